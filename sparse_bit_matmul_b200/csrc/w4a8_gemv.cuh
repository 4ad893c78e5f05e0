// W4A8 FastGEMM for a few tokens (M <= 4) on the CUDA cores.
//
// What it computes (OdysseyLLM review page,
// xllm-io.github.io/paper-review/blog/odysseyllm, sec. 3.1-3.2, 5.2):
//   acc[m][n] = (sum_k x_i8[m][k] * 16 w[n][k]) / 16      (exact int32)
//   y[m][n]   = (float)((float)acc[m][n] * S[n]) * x_scale[m]
// where 16 w is the SINT4 weight moved into the high half of a byte (the
// page's SINT4toS8 shift), here by one shift and two masks per 8 weights of
// the native layout, and the products are summed with dp4a.
//
// With one to four tokens the weights are read once and each weight byte
// meets at most 8 multiply-adds, so this kernel skips the tcgen05 pipeline
// and its role hand-offs.  It is a comparison kernel: at K=4096, N=14336 it
// measured 11.5 us (M=1) and 20.0 us (M=4) per call, slower than the
// tensor-core kernel, which stays the default for every M.  A CTA owns 32 consecutive rows (lane = row: a warp's 16-byte
// loads of one piece cover 512 contiguous bytes of the native layout) and
// its PARTS warps split K into equal runs of 32-weight pieces; the partial
// sums meet in shared memory and the first MT warps write the outputs.
// Programmatic dependent launch: the first weight loads are issued before
// the wait for the previous kernel on the stream (they do not depend on it);
// the activations, scales and outputs are touched only after it.
#pragma once

#include <cstdint>

#include "sherry_internal.h"

namespace sherry {
namespace w4gemv {

constexpr int kRows = 32;           // rows per CTA, one per lane
constexpr int kBatch = 4;           // 16-byte pieces in flight per thread

__device__ __forceinline__ int dot8(uint32_t v, int x_lo, int x_hi, int acc)
{
    // byte b of v: w[k0+b] in bits 0-3, w[k0+4+b] in bits 4-7
    acc = __dp4a((int)((v << 4) & 0xF0F0F0F0u), x_lo, acc);
    return __dp4a((int)(v & 0xF0F0F0F0u), x_hi, acc);
}

template <int MT, int PARTS>
__global__ void __launch_bounds__(kRows * PARTS)
    w4a8_gemv_kernel(const int8_t* __restrict__ x, const float* __restrict__ x_scale,
                     const uint8_t* __restrict__ wn, const float* __restrict__ scale, float* __restrict__ y,
                     int32_t* __restrict__ acc_out, int64_t M, int64_t N, int64_t K)
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int lane = threadIdx.x & 31, part = threadIdx.x >> 5;
    const int64_t n = (int64_t)blockIdx.x * kRows + lane;        // < ceil(N/128)*128: inside the layout
    const int64_t Kc = sherry_k_chunks(K);
    const int64_t P = K / 32;                                     // pieces holding weights (K % 32 == 0)
    const int64_t per = (P + PARTS - 1) / PARTS;
    const int64_t p0 = part * per;
    const int64_t p1 = p0 + per < P ? p0 + per : P;

    int acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0;

    uint4 w[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b)
        if (p0 + b < p1) w[b] = __ldg(reinterpret_cast<const uint4*>(wn + sherry_w4_piece_offset(n, Kc, p0 + b)));
    asm volatile("griddepcontrol.wait;" ::: "memory");

    for (int64_t p = p0; p < p1; p += kBatch) {
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            if (p + b >= p1) break;
            const uint4 v = w[b];
            const int64_t k0 = (p + b) * 32;
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                if (m >= M) break;
                const int4* xr = reinterpret_cast<const int4*>(x + m * K + k0);
                const int4 xa = __ldg(xr), xb = __ldg(xr + 1);
                int a = acc[m];
                a = dot8(v.x, xa.x, xa.y, a);
                a = dot8(v.y, xa.z, xa.w, a);
                a = dot8(v.z, xb.x, xb.y, a);
                a = dot8(v.w, xb.z, xb.w, a);
                acc[m] = a;
            }
            // refill this slot with the piece kBatch ahead
            if (p + b + kBatch < p1)
                w[b] = __ldg(reinterpret_cast<const uint4*>(wn + sherry_w4_piece_offset(n, Kc, p + b + kBatch)));
        }
    }

    __shared__ int red[PARTS][MT][kRows];
#pragma unroll
    for (int m = 0; m < MT; ++m) red[part][m][lane] = acc[m];
    __syncthreads();
    if (part < MT && part < M && n < N) {
        const int m = part;
        int s16 = 0;
#pragma unroll
        for (int q = 0; q < PARTS; ++q) s16 += red[q][m][lane];
        const int32_t a = s16 >> 4;                               // exact: every term is a multiple of 16
        if (acc_out) acc_out[m * N + n] = a;
        if (y) y[m * N + n] = __fmul_rn(__fmul_rn((float)a, __ldg(scale + n)), __ldg(x_scale + m));
    }
}

}  // namespace w4gemv
}  // namespace sherry
