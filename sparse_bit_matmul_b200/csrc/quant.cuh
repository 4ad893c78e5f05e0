// Per-token int8 activation quantiser arithmetic shared by the quantiser
// kernel and the fused decode kernel.
//
// Rule (the Sherry page, pnsm.cn/news/1195499, sec. 2.2 step 1 leaves it
// open; this is symmetric absmax/127): s = a / 127 with a = max |x| (IEEE
// fp32 division), q = clamp(rint(fl(x / s)), -127, 127), round half to even;
// a == 0 gives s = 0 and q = 0.
//
// q is computed without a division for almost every element: with
// r = fl(1 / s) and t = fl(x * r), |t - x/s| <= |x/s| * (2^-23 + 2^-48) and
// |fl(x/s) - x/s| <= 2^-24 |x/s|, so |t - fl(x/s)| < 2.3e-5 for
// |x/s| <= 127.0001.  Unless t lies within kHalfEps = 4e-5 of a half
// integer, t and fl(x/s) are strictly on the same side of every rounding
// boundary and rint(t) == rint(fl(x/s)).  Near a boundary (and whenever
// 1/s is not a finite normal number) the element takes the exact IEEE
// division.  |rint| never exceeds 127 on the fast path because |x| <= a.
#pragma once

#include <cstdint>

namespace sherry {
namespace quant {

constexpr float kHalfEps = 4.0e-5f;

struct Scale {
    float s;        // a / 127 (IEEE), 0 when a == 0
    float r;        // fl(1 / s)
    bool zero;      // a == 0: every q is 0
    bool fast;      // the reciprocal path is valid for this token
};

__device__ __forceinline__ Scale make_scale(float a)
{
    Scale sc;
    sc.s = __fdiv_rn(a, 127.0f);
    sc.zero = (a == 0.0f);
    sc.r = __frcp_rn(sc.s);
    sc.fast = !sc.zero && sc.s >= 1.0e-30f && isfinite(sc.r) && sc.r < 1.0e30f;
    if (sc.zero) sc.s = 0.0f;
    return sc;
}

__device__ __forceinline__ int quantise_exact(float x, float s)
{
    int r = __float2int_rn(__fdiv_rn(x, s));
    return r > 127 ? 127 : (r < -127 ? -127 : r);
}

__device__ __forceinline__ int quantise(float x, const Scale& sc)
{
    if (sc.zero) return 0;
    if (sc.fast) {
        const float t = __fmul_rn(x, sc.r);
        const float rt = rintf(t);
        if (fabsf(t - rt) < 0.5f - kHalfEps) return (int)rt;
    }
    return quantise_exact(x, sc.s);
}

// Four consecutive activations -> four int8 codes packed little endian.
__device__ __forceinline__ uint32_t quantise4(const float4& v, const Scale& sc)
{
    const uint32_t a = (uint32_t)quantise(v.x, sc) & 0xFFu;
    const uint32_t b = (uint32_t)quantise(v.y, sc) & 0xFFu;
    const uint32_t c = (uint32_t)quantise(v.z, sc) & 0xFFu;
    const uint32_t d = (uint32_t)quantise(v.w, sc) & 0xFFu;
    return a | (b << 8) | (c << 16) | (d << 24);
}

__device__ __forceinline__ float absmax4(const float4& v)
{
    return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

}  // namespace quant
}  // namespace sherry
