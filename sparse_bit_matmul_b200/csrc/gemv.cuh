// Sherry 3:4 ternary decode GEMV (few tokens) on the sm_100a CUDA cores.
//
// What it computes (Sherry page, pnsm.cn/news/1195499, sec. 2.2 steps 1-4):
// the page's table-lookup inference.  For every 4-element activation segment
// x_g = (x[4g], .., x[4g+3]) of a token, a table holds the dot product of x_g
// with each of the 32 ternary groups (the 16 patterns of the page times the
// sign bit, folded together so no sign has to be applied afterwards):
//     lut[m][g][c] = sum_i T_i(c) * x_i8[m][4g + i]        (int16, |.| <= 381)
// Then acc[m][n] = sum_g lut[m][g][code(n, g)], exact in int32, and
// y[m][n] = (float)((float)acc * alpha[n]) * x_scale[m].
//
// Mapping to the B200 (the page's AVX2/NEON/Jetson kernels are prior art):
//   * a CTA owns one K-slice (SL chunks of 128 weights) of one 128-row tile;
//     the codes of a (tile, slice) are one contiguous block of the native
//     layout, fetched with a single bulk copy into shared memory;
//   * the tables of the slice (SL * 32 groups * 32 entries * M tokens) are
//     built in shared memory by the CTA; then two threads share a weight row
//     (alternate chunks), and per group need one shift, one LOP3 (the 5-bit
//     code times 2 OR-ed into the table base), one ld.shared.s16 and one add
//     per token: the 32 lanes of a warp read one group's 64-byte table, so
//     there are no bank conflicts whatever the codes;
//   * the NS K-slices of a tile run as one thread-block cluster: CTA r owns
//     rows [r*128/NS, (r+1)*128/NS); every CTA adds its int32 partial sums
//     of those rows into CTA r's shared memory with red.shared::cluster, and
//     after one cluster barrier each CTA writes y for its own rows -- exact,
//     no global atomics, no workspace (the receive buffers are zeroed and
//     announced with an early non-blocking cluster arrive);
//   * launched with programmatic dependent launch: the weight copy is issued
//     before griddepcontrol.wait (weights never depend on the previous
//     kernel), activations and the workspace are touched only after it.
#pragma once

#include <cstdint>

#include "ptx.cuh"
#include "sherry_internal.h"

namespace sherry {
namespace gemv {

constexpr int kThreads = 256;          // two threads per row of a 128-row tile
constexpr int kMaxSL = 16;             // chunks per K-slice (2048 weights)
constexpr int kMaxNS = 8;              // K-slices per tile = cluster size
constexpr int kLutTokenStride = kMaxSL * 32 * 64;   // bytes of one token's tables
constexpr uint64_t kWaitLimitNs = 2000000000ull;

struct Params {
    const uint8_t* wnative;
    const int8_t* x;            // [M][K]
    const float* x_scale;       // [M]
    const float* alpha;         // [N]
    float* y;                   // [M][N] or null
    int32_t* acc;               // [M][N] or null
    unsigned* status;
    int64_t M, N, K;
    int64_t TN, Kc;
    int SL, NS;                 // chunks per slice, slices per tile (cluster size)
};

// Shared memory of one CTA for MT tokens and SL chunks per slice: the tables
// (token stride fixed so that the token offset is an immediate), the codes,
// the partial sums [2][MT][128] int32 (the second half doubles as the receive
// buffer of the cluster reduction), one mbarrier.
__host__ __device__ inline int lut_bytes(int mt, int sl) { return (mt - 1) * kLutTokenStride + sl * 2048; }
__host__ __device__ inline int code_offset(int mt, int sl) { return (lut_bytes(mt, sl) + 127) & ~127; }
__host__ __device__ inline int red_offset(int mt, int sl)
{
    return code_offset(mt, sl) + sl * SHERRY_CHUNK_BYTES_PER_TILE;
}
__host__ __device__ inline int bar_offset(int mt, int sl) { return red_offset(mt, sl) + 2 * mt * 128 * 4; }
__host__ __device__ inline int smem_bytes(int mt, int sl) { return bar_offset(mt, sl) + 64; }

// 32 table entries of one activation segment, packed as 16 pairs of int16
// (entry c at half-word c).
__device__ __forceinline__ void segment_table(uint32_t xw, uint32_t (&out)[16])
{
    const int a[4] = {(int)(int8_t)(xw & 0xFF), (int)(int8_t)((xw >> 8) & 0xFF),
                      (int)(int8_t)((xw >> 16) & 0xFF), (int)(int8_t)(xw >> 24)};
    int e[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) {
        const int z = c & 3;
        int v = 0, slot = 2;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (i == z) continue;
            v += ((c >> slot) & 1) ? -a[i] : a[i];
            ++slot;
        }
        e[c] = v;
    }
#pragma unroll
    for (int p = 0; p < 16; ++p)
        out[p] = ((uint32_t)e[2 * p] & 0xFFFFu) | ((uint32_t)e[2 * p + 1] << 16);
}

template <int MT>
__global__ void __launch_bounds__(kThreads)
    sherry_gemv_kernel(const Params p)
{
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t* lut = smem;                                           // [MT][SL*32][32] int16, token stride 32 KB
    const uint32_t* codes = reinterpret_cast<const uint32_t*>(smem + code_offset(MT, p.SL));   // [SL][5][128]
    int32_t* red = reinterpret_cast<int32_t*>(smem + red_offset(MT, p.SL));                    // [2][MT][128]
    const uint32_t bar_a = ptx::smem_u32(smem + bar_offset(MT, p.SL));

    const int64_t tile = blockIdx.x;
    const int slice = blockIdx.y;               // = rank in the cluster when NS > 1
    const int c0 = slice * p.SL;
    int nch = (int)(p.Kc - c0);
    nch = nch < 0 ? 0 : (nch > p.SL ? p.SL : nch);

    // weights first: they do not depend on any earlier kernel
    if (threadIdx.x == 0) {
        ptx::mbar_init(bar_a, 1);
        ptx::fence_mbar_init();
        const uint32_t bytes = (uint32_t)nch * SHERRY_CHUNK_BYTES_PER_TILE;
        ptx::mbar_arrive_expect_tx(bar_a, bytes);
        if (bytes)
            ptx::bulk_g2s(ptx::smem_u32(codes), p.wnative + (tile * p.Kc + c0) * SHERRY_CHUNK_BYTES_PER_TILE, bytes,
                          bar_a);
    }
    // receive buffer of the cluster reduction, zeroed and announced early
    int32_t* recv = red + MT * 128;
    for (int i = threadIdx.x; i < MT * 128; i += kThreads) recv[i] = 0;
    if (p.NS > 1) {
        __syncthreads();
        ptx::cluster_arrive_release();
    }
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();

    // tables of this K-slice: one (token, group) per thread and step
    const int G = nch * 32;
    const int64_t K4 = p.K / 4;
    for (int idx = threadIdx.x; idx < MT * G; idx += kThreads) {
        const int m = idx / G, g = idx - m * G;
        const int64_t gg = (int64_t)c0 * 32 + g;
        uint32_t xw = 0;
        if (m < p.M && gg < K4) xw = *reinterpret_cast<const uint32_t*>(p.x + m * p.K + 4 * gg);
        uint32_t t[16];
        segment_table(xw, t);
        uint4* dst = reinterpret_cast<uint4*>(lut + m * kLutTokenStride + g * 64);
#pragma unroll
        for (int q = 0; q < 4; ++q) dst[q] = make_uint4(t[4 * q], t[4 * q + 1], t[4 * q + 2], t[4 * q + 3]);
    }
    __syncthreads();

    const int row = threadIdx.x & 127;
    const int sub = threadIdx.x >> 7;           // this thread takes chunks sub, sub + 2, ...
    const int lane = threadIdx.x & 31;
    bool ok = ptx::mbar_wait_bounded(bar_a, 0, kWaitLimitNs);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok && lane == 0) atomicCAS(p.status, 0u, (unsigned)SHERRY_DEV_TIMEOUT_DECODER);

    int32_t acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0;
    const uint32_t lut_base = ptx::smem_u32(lut);
#pragma unroll 1
    for (int j = sub; ok && j < nch; j += 2) {
        uint32_t w[SHERRY_CHUNK_WORDS];
#pragma unroll
        for (int k = 0; k < SHERRY_CHUNK_WORDS; ++k)
            w[k] = codes[j * (SHERRY_CHUNK_WORDS * SHERRY_TILE_ROWS) + sherry_word_pos(k, row)];
        const uint32_t base = lut_base + (uint32_t)j * 2048u;   // 64-byte aligned
#pragma unroll
        for (int g = 0; g < 32; ++g) {
            // twice the 5-bit code of group g, i.e. its byte offset in the table
            const int bit = 5 * g, wi = bit >> 5, off = bit & 31;
            uint32_t v;
            if (off == 0) v = w[wi] << 1;
            else if (off <= 27) v = w[wi] >> (off - 1);
            else v = __funnelshift_r(w[wi], w[wi + 1], off - 1);
            const uint32_t a = (v & 0x3Eu) | base;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                int16_t e;
                asm volatile("ld.shared.s16 %0, [%1];" : "=h"(e) : "r"(a + (uint32_t)(m * kLutTokenStride + g * 64)));
                acc[m] += (int32_t)e;
            }
        }
    }
    // the two threads of a row combine in red[0..MT*128)
    if (sub == 1) {
#pragma unroll
        for (int m = 0; m < MT; ++m) red[m * 128 + row] = acc[m];
    }
    __syncthreads();
    const int rows = 128 / p.NS;
    if (sub == 0) {
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[m] += red[m * 128 + row];
        if (p.NS == 1) {
#pragma unroll
            for (int m = 0; m < MT; ++m) recv[m * 128 + row] = acc[m];
        } else {
            ptx::cluster_wait_acquire();             // every peer has zeroed its receive buffer
            const uint32_t owner = (uint32_t)(row / rows);
#pragma unroll
            for (int m = 0; m < MT; ++m) ptx::red_cluster_add_s32(ptx::smem_u32(recv + m * 128 + row), owner, acc[m]);
        }
    } else if (p.NS > 1) {
        ptx::cluster_wait_acquire();
    }
    if (p.NS > 1) {
        ptx::cluster_arrive_release();               // partial sums sent
        ptx::cluster_wait_acquire();                 // ... and received from every peer
    } else {
        __syncthreads();
    }
    // y for the rows this CTA owns
    const int r0 = (p.NS == 1) ? 0 : slice * rows;
    for (int idx = threadIdx.x; idx < MT * rows; idx += kThreads) {
        const int m = idx / rows, r = r0 + (idx - m * rows);
        const int64_t n = tile * SHERRY_TILE_ROWS + r;
        if (m >= p.M || n >= p.N) continue;
        const int32_t a32 = recv[m * 128 + r];
        if (p.acc) p.acc[m * p.N + n] = a32;
        if (p.y) p.y[m * p.N + n] = __fmul_rn(__fmul_rn((float)a32, p.alpha[n]), p.x_scale[m]);
    }
}

}  // namespace gemv
}  // namespace sherry
