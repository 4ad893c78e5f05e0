// Sherry 3:4 ternary GEMM for a few tokens (M <= 8): the decode path.
//
// What it computes (Sherry page, pnsm.cn/news/1195499, sec. 2.2 steps 1-4,
// sec. 3.1): acc[m][n] = sum_k q[m][k] * T[n][k] exactly in int32, and
// y[m][n] = (float)((float)acc * alpha[n]) * s[m].  With FUSED the kernel
// also quantises the fp32 activations (sec. 2.2 step 1, the rule of
// quant.cuh), so one launch covers a whole layer call.
//
// Mapping to the B200.  At a few tokens a layer call moves a few MB and its
// time is latency: the kernel boundary, one activation fetch, the decode of
// every 5-bit code, one store of y.  The design keeps that chain short.
//   * One CTA per SM (more only when its codes would not fit in shared
//     memory), each owning a contiguous, balanced range of whole output rows
//     over the full K: no split-K, no cross-CTA reduction, no atomics, no
//     workspace, no clusters.
//   * Before griddepcontrol.wait the CTA streams its rows' codes (the rotated
//     word planes of the native layout) into shared memory with 4-byte
//     cp.async copies: weights never depend on the previous kernel, so their
//     fetch overlaps its decode.  The CTA lets the next kernel start only once
//     its own activations are in shared memory, so that the next kernel's
//     weight stream does not queue in front of those latency-critical reads.  The CTA is small enough in shared memory,
//     threads and registers for the next layer's CTA to be resident at the
//     same time and do the same.
//   * After the wait every CTA reads the activations of its tokens (all of
//     K), takes the absmax, quantises into shared memory; then thread
//     (row i, K-part p) walks the chunks of its part: one 32-entry table
//     load turns a code into int8x4 {-1,0,+1}, one dp4a per token adds it.
//   * The K-parts of a row are summed in shared memory and the epilogue
//     writes y (and acc) with coalesced stores.
#pragma once

#include <cstdint>

#include "ptx.cuh"
#include "quant.cuh"
#include "sherry_internal.h"

namespace sherry {
namespace decode {

constexpr int kMaxM = 8;
constexpr int kMaxThreads = 512;
constexpr int kSmemBudget = 100 * 1024;     // two CTAs (this layer, the next) per SM
constexpr int kXV = 8;                      // fused: float4 activations per thread held in registers

struct Params {
    const uint8_t* wnative;
    const int8_t* xq;            // [M][K] int8 activations (not FUSED)
    const float* x_scale;        // [M] (not FUSED)
    const float* x;              // [M][K] fp32 activations (FUSED)
    int8_t* xq_out;              // FUSED, optional: [M][K] int8 activations (written by CTA 0)
    float* xs_out;               // FUSED, optional: [M] scales (written by CTA 0)
    const float* alpha;          // [N]
    float* y;                    // [M][N] or null
    int32_t* acc;                // [M][N] or null
    int64_t M, N, K, Kc;
    int G;                       // CTAs; CTA c owns rows [row_begin(c), row_begin(c+1))
    int R;                       // largest row count of a CTA, a multiple of 4
    int P;                       // K-parts per row
    int CPT;                     // chunks per K-part
};

// Shared memory: table | scales | warp maxima (two token slots) | partial sums [P][M][R] |
// alpha [R] | codes [Kc][5][R] words | activations [M][Kc*128] int8.
constexpr int kOffTable = 0;                              // 32 x u32, 128-byte aligned inside 256 bytes
constexpr int kOffScale = 256;                            // [kMaxM] f32 s
constexpr int kOffWarpMax = kOffScale + kMaxM * 4;        // [2][16 warps] f32
constexpr int kOffRed = kOffWarpMax + 2 * 16 * 4;
static_assert(kMaxThreads / 32 <= 16, "warp-maximum slots");
__host__ __device__ inline int off_alpha(int M, int P, int R) { return (kOffRed + P * M * R * 4 + 15) & ~15; }
__host__ __device__ inline int off_codes(int M, int P, int R) { return (off_alpha(M, P, R) + R * 4 + 15) & ~15; }
__host__ __device__ inline int off_q(int M, int P, int R, int64_t Kc)
{
    return (off_codes(M, P, R) + (int)Kc * SHERRY_CHUNK_WORDS * R * 4 + 15) & ~15;
}
__host__ __device__ inline int smem_bytes(int M, int P, int R, int64_t Kc)
{
    return off_q(M, P, R, Kc) + M * (int)Kc * SHERRY_KCHUNK;
}

__device__ __forceinline__ uint32_t expand_code(uint32_t c)
{
    const uint32_t z = c & 3u;
    uint32_t word = 0, slot = 2;
#pragma unroll
    for (uint32_t i = 0; i < 4; ++i) {
        if (i == z) continue;
        word |= (((c >> slot) & 1u) ? 0xFFu : 0x01u) << (8 * i);
        ++slot;
    }
    return word;
}

// First row of row group g of G: balanced, rounded up to a multiple of 4.
__host__ __device__ inline int64_t row_begin(int64_t N, int64_t g, int64_t G)
{
    const int64_t b = (N * g / G + 3) & ~int64_t(3);
    return b < N ? b : N;
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }


// N consecutive 32-bit words from a shared address (aligned to 4 N bytes).
template <int N>
__device__ __forceinline__ void lds_vec(uint32_t addr, uint32_t (&v)[N]);
template <>
__device__ __forceinline__ void lds_vec<1>(uint32_t addr, uint32_t (&v)[1])
{
    asm("ld.shared.u32 %0, [%1];" : "=r"(v[0]) : "r"(addr));
}
template <>
__device__ __forceinline__ void lds_vec<2>(uint32_t addr, uint32_t (&v)[2])
{
    asm("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v[0]), "=r"(v[1]) : "r"(addr));
}
template <>
__device__ __forceinline__ void lds_vec<4>(uint32_t addr, uint32_t (&v)[4])
{
    asm("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]) : "r"(addr));
}

template <int MT, bool FUSED>
__global__ void __launch_bounds__(kMaxThreads, 2)
    sherry_decode_kernel(const Params p)
{
    extern __shared__ __align__(16) uint8_t smem[];
    const int M = (int)p.M;
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int64_t r0 = row_begin(p.N, blockIdx.x, p.G), r1 = row_begin(p.N, blockIdx.x + 1, p.G);
    const int Rc = (int)(r1 - r0);
    const int R = p.R, P = p.P;
    const uint32_t s_base = ptx::smem_u32(smem);
    const uint32_t codes_s = s_base + off_codes(M, P, R);
    const int qoff = off_q(M, P, R, p.Kc);
    int8_t* qbuf = reinterpret_cast<int8_t*>(smem + qoff);
    const int QK = (int)p.Kc * SHERRY_KCHUNK;              // bytes per token row of qbuf

    // ---- before the wait: this CTA's codes, alpha, the decode table -------------
    // Row groups start at multiples of 4 rows, so 4 consecutive rows of one word
    // plane are 16 aligned bytes: thread t copies 4-row piece t % R4 of every
    // (nthr / R4)-th chunk with 16-byte cp.async (4-byte copies for a ragged end);
    // consecutive lanes read consecutive positions of the plane.
    {
        const int R4 = (Rc + 3) >> 2;
        const int cstride = R4 > 0 ? nthr / R4 : 0;
        const int pi = R4 > 0 ? tid % R4 : 0, cs = R4 > 0 ? tid / R4 : 0;
        if (cs < cstride) {
            const int64_t r = r0 + 4 * pi;
            const int rr = (int)(r & 127);
            const int nr = min(4, Rc - 4 * pi);
            const uint32_t* src = reinterpret_cast<const uint32_t*>(p.wnative) +
                                  (r >> 7) * p.Kc * (SHERRY_CHUNK_WORDS * SHERRY_TILE_ROWS);
            int pos[SHERRY_CHUNK_WORDS];
#pragma unroll
            for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j) pos[j] = sherry_word_pos(j, rr);
            uint32_t dst = codes_s + 4u * (uint32_t)(cs * SHERRY_CHUNK_WORDS * R + 4 * pi);
            const uint32_t dstep = 4u * (uint32_t)(cstride * SHERRY_CHUNK_WORDS * R);
            for (int c = cs; c < (int)p.Kc; c += cstride) {
                const uint32_t* sc = src + (int64_t)c * (SHERRY_CHUNK_WORDS * SHERRY_TILE_ROWS);
                if (nr == 4) {
#pragma unroll
                    for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j) cp_async16(dst + 4u * (uint32_t)(j * R), sc + pos[j]);
                } else {
                    for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j)
                        for (int e = 0; e < nr; ++e) cp_async4(dst + 4u * (uint32_t)(j * R + e), sc + pos[j] + e);
                }
                dst += dstep;
            }
        }
        const uint32_t alpha_s = s_base + off_alpha(M, P, R);
        for (int ii = tid; ii < Rc; ii += nthr) cp_async4(alpha_s + 4u * (uint32_t)ii, p.alpha + r0 + ii);
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    // the decode table at a 128-byte aligned shared address, so that a lookup
    // address is one LOP3: (code * 4) | table
    const uint32_t table_s = (s_base + kOffTable + 127u) & ~127u;
    if (tid < 32) ptx::sts_u32(table_s + 4u * (uint32_t)tid, expand_code((uint32_t)tid));
    ptx::pdl_wait();

    // ---- activations -------------------------------------------------------------
    float* scale_s = reinterpret_cast<float*>(smem + kOffScale);
    const int K4 = (int)(p.K >> 2);
    if constexpr (FUSED) {
        // per token: the thread's float4s stay in registers (all loads in
        // flight at once), block absmax, then quantise from the registers
        float* warp_max = reinterpret_cast<float*>(smem + kOffWarpMax);
        const int nwarps = (nthr + 31) >> 5;
        const bool in_regs = K4 <= kXV * nthr;
        for (int m = 0; m < M; ++m) {
            const float4* xr = reinterpret_cast<const float4*>(p.x + (int64_t)m * p.K);
            uint32_t* qr = reinterpret_cast<uint32_t*>(qbuf + m * QK);
            float4 v[kXV];
            float mx = 0.0f;
            if (in_regs) {
                // predicated loads, all in flight at once; slots past the row
                // hold zeros, which leave the maximum unchanged
#pragma unroll
                for (int u = 0; u < kXV; ++u) {
                    const int idx = tid + u * nthr;
                    v[u] = idx < K4 ? xr[idx] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                }
#pragma unroll
                for (int u = 0; u < kXV; ++u) mx = fmaxf(mx, quant::absmax4(v[u]));
            } else {
#pragma unroll 4
                for (int i = tid; i < K4; i += nthr) mx = fmaxf(mx, quant::absmax4(xr[i]));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
            if (lane == 0) warp_max[(m & 1) * 16 + warp] = mx;
            __syncthreads();
            // every warp combines the (at most 16) warp maxima: one load per
            // lane and a shuffle tree, not a chain of dependent loads
            float a = lane < nwarps ? warp_max[(m & 1) * 16 + lane] : 0.0f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
            const quant::Scale sc = quant::make_scale(a);
            if (tid == 0) {
                scale_s[m] = sc.s;
                if (p.xs_out && blockIdx.x == 0) p.xs_out[m] = sc.s;
            }
            uint32_t* qo = (p.xq_out && blockIdx.x == 0) ? reinterpret_cast<uint32_t*>(p.xq_out + (int64_t)m * p.K)
                                                          : nullptr;
            if (in_regs) {
#pragma unroll
                for (int u = 0; u < kXV; ++u) {
                    const int idx = tid + u * nthr;
                    if (idx < K4) {
                        const uint32_t w = quant::quantise4(v[u], sc);
                        qr[idx] = w;
                        if (qo) qo[idx] = w;
                    }
                }
            } else {
                for (int i = tid; i < K4; i += nthr) {
                    const uint32_t w = quant::quantise4(xr[i], sc);
                    qr[i] = w;
                    if (qo) qo[i] = w;
                }
            }
        }
    } else {
        const int K16 = (int)(p.K >> 4);
        for (int m = 0; m < M; ++m)
            for (int i = tid; i < K16; i += nthr)
                cp_async16(s_base + (uint32_t)(qoff + m * QK + 16 * i), p.xq + (int64_t)m * p.K + 16 * i);
        asm volatile("cp.async.commit_group;" ::: "memory");
        if (tid < M) scale_s[tid] = p.x_scale[tid];
    }
    // zero the activation tail of the last chunk: its padding codes decode to nonzero weights
    {
        const int tail = QK - (int)p.K;                    // multiple of 32
        for (int i = tid; i < M * tail; i += nthr) {
            const int m = i / tail;
            qbuf[m * QK + (int)p.K + (i - m * tail)] = 0;
        }
    }
    cp_async_wait_all();
    __syncthreads();
    // the next kernel may start now: its weight prefetch overlaps this decode
    // instead of queueing in front of this CTA's activation reads
    ptx::pdl_launch_dependents();

    // ---- decode + dp4a: one row per thread ----------------------------------------
    // All 32 table loads of a chunk are issued before its dp4a run, which keeps
    // enough loads in flight with one CTA per SM; the next chunk's code words
    // are fetched during the current one.
    const int i = tid % R, part = tid / R;
    int32_t acc[MT][4];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0;
    if (part < P && i < Rc) {
        const uint32_t cbase = codes_s + 4u * (uint32_t)i;
        const uint32_t q_s = s_base + (uint32_t)qoff;
        const int cb = part * p.CPT;
        const int ce = min((int)p.Kc, cb + p.CPT);
        uint32_t wn[SHERRY_CHUNK_WORDS];
#pragma unroll
        for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j)
            wn[j] = ptx::lds_u32_nv(cbase + 4u * (uint32_t)((cb * SHERRY_CHUNK_WORDS + j) * R));
#pragma unroll 1
        for (int c = cb; c < ce; ++c) {
            uint32_t w[SHERRY_CHUNK_WORDS + 1];
#pragma unroll
            for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j) w[j] = wn[j];
            w[SHERRY_CHUNK_WORDS] = 0;
            if (c + 1 < ce) {
#pragma unroll
                for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j)
                    wn[j] = ptx::lds_u32_nv(cbase + 4u * (uint32_t)(((c + 1) * SHERRY_CHUNK_WORDS + j) * R));
            }
            // table entries of the chunk's 32 codes
            uint32_t e[32];
#pragma unroll
            for (int g = 0; g < 32; ++g) {
                // byte offset of group g's code in the table: (bits [5g, 5g+5)) * 4
                const int bit = 5 * g, wi = bit >> 5, off = bit & 31;
                uint32_t v;
                if (off == 0) v = w[wi] << 2;
                else if (off == 1) v = w[wi] << 1;
                else if (off <= 27) v = w[wi] >> (off - 2);
                else v = __funnelshift_r(w[wi], w[wi + 1], off - 2);
                e[g] = ptx::lds_u32_nv((v & 0x7Cu) | table_s);
            }
            const uint32_t qc = q_s + (uint32_t)(c * SHERRY_KCHUNK);
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= M) break;
#pragma unroll
                for (int g4 = 0; g4 < 8; ++g4) {
                    uint32_t qv[4];
                    lds_vec<4>(qc + (uint32_t)(m * QK + 16 * g4), qv);
                    acc[m][0] = __dp4a((int)e[4 * g4 + 0], (int)qv[0], acc[m][0]);
                    acc[m][1] = __dp4a((int)e[4 * g4 + 1], (int)qv[1], acc[m][1]);
                    acc[m][2] = __dp4a((int)e[4 * g4 + 2], (int)qv[2], acc[m][2]);
                    acc[m][3] = __dp4a((int)e[4 * g4 + 3], (int)qv[3], acc[m][3]);
                }
            }
        }
    }

    // ---- sum the K-parts of each row, epilogue ----------------------------------------
    int32_t* red = reinterpret_cast<int32_t*>(smem + kOffRed);      // [P][M][R]
    const float* alpha_sm = reinterpret_cast<const float*>(smem + off_alpha(M, P, R));
    if (part < P) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
            if (m < M) red[(part * M + m) * R + i] = (acc[m][0] + acc[m][1]) + (acc[m][2] + acc[m][3]);
    }
    __syncthreads();
    for (int idx = tid; idx < M * Rc; idx += nthr) {
        const int m = idx / Rc, ii = idx - m * Rc;
        int32_t a32 = 0;
        for (int pp = 0; pp < P; ++pp) a32 += red[(pp * M + m) * R + ii];
        const int64_t n = r0 + ii;
        if (p.acc) p.acc[m * p.N + n] = a32;
        if (p.y) p.y[m * p.N + n] = __fmul_rn(__fmul_rn((float)a32, alpha_sm[ii]), scale_s[m]);
    }
}

}  // namespace decode
}  // namespace sherry
