// Per-token int8 activation quantiser arithmetic shared by the quantiser
// kernel and the fused decode kernel.
//
// Rule (the Sherry page, pnsm.cn/news/1195499, sec. 2.2 step 1 leaves it
// open; this is symmetric absmax/127): s = a / 127 with a = max |x| (IEEE
// fp32 division), q = clamp(rint(fl(x / s)), -127, 127), round half to even;
// a == 0 gives s = 0 and q = 0.
//
// q is computed without a division for almost every element: r is the
// hardware reciprocal approximation of s (rcp.approx, at most 1 ulp off:
// relative error <= 2^-23) and t = fl(x * r), so |t - x/s| <= |x/s| *
// (2^-23 + 2^-24 + 2^-47), and |fl(x/s) - x/s| <= 2^-24 |x/s|: together
// |t - fl(x/s)| < 3.0e-5 for |x/s| <= 127.0001.  Unless t lies within
// kHalfEps = 4e-5 of a half integer, t and fl(x/s) are strictly on the same
// side of every rounding boundary and rint(t) == rint(fl(x/s)).  Near a
// boundary (and whenever s is tiny or r is not finite) the element takes the
// exact IEEE division, kept out of line.  |rint| never exceeds 127 on the
// fast path because |x| <= a.
//
// On the fast path rint(t) is taken without conversion instructions (they
// issue at a quarter of the ALU rate): for |t| < 2^22, fl(t + 1.5 * 2^23) is
// 1.5 * 2^23 + rint(t), rounded half to even by the addition itself, so the
// low byte of that float's encoding is the two's-complement byte of rint(t),
// and subtracting 1.5 * 2^23 again gives rint(t) as a float, exactly.
#pragma once

#include <cstdint>

namespace sherry {
namespace quant {

constexpr float kHalfEps = 4.0e-5f;
constexpr float kRoundMagic = 12582912.0f;      // 1.5 * 2^23

struct Scale {
    float s;        // a / 127 (IEEE), 0 when a == 0
    float r;        // fl(1 / s)
    bool zero;      // a == 0: every q is 0
    bool fast;      // the reciprocal path is valid for this token
};

__device__ __forceinline__ float rcp_approx(float s)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(s));
    return r;
}

__device__ __forceinline__ Scale make_scale(float a)
{
    Scale sc;
    sc.s = __fdiv_rn(a, 127.0f);
    sc.zero = (a == 0.0f);
    sc.r = rcp_approx(sc.s);
    sc.fast = !sc.zero && sc.s >= 1.0e-30f && isfinite(sc.r) && sc.r < 1.0e30f;
    if (sc.zero) sc.s = 0.0f;
    return sc;
}

__device__ __forceinline__ int quantise_exact(float x, float s)
{
    int r = __float2int_rn(__fdiv_rn(x, s));
    return r > 127 ? 127 : (r < -127 ? -127 : r);
}

// The exact path for a whole group of four, out of line: rare, and it keeps
// the division's code and registers away from the common path.
__device__ __noinline__ uint32_t quantise4_exact(float4 v, float s)
{
    const uint32_t a = (uint32_t)quantise_exact(v.x, s) & 0xFFu;
    const uint32_t b = (uint32_t)quantise_exact(v.y, s) & 0xFFu;
    const uint32_t c = (uint32_t)quantise_exact(v.z, s) & 0xFFu;
    const uint32_t d = (uint32_t)quantise_exact(v.w, s) & 0xFFu;
    return a | (b << 8) | (c << 16) | (d << 24);
}

// Four consecutive activations -> four int8 codes packed little endian.
__device__ __forceinline__ uint32_t quantise4(const float4& v, const Scale& sc)
{
    if (sc.zero) return 0u;
    const float in[4] = {v.x, v.y, v.z, v.w};
    // byte e of the result <- low byte of element e's rounded encoding
    constexpr uint32_t kSel[4] = {0x3214u, 0x3240u, 0x3410u, 0x4210u};
    uint32_t packed = 0;
    bool near = !sc.fast;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float t = __fmul_rn(in[e], sc.r);
        const float tm = __fadd_rn(t, kRoundMagic);
        near |= !(fabsf(__fsub_rn(t, __fsub_rn(tm, kRoundMagic))) < 0.5f - kHalfEps);
        packed = __byte_perm(packed, __float_as_uint(tm), kSel[e]);
    }
    return near ? quantise4_exact(v, sc.s) : packed;
}

__device__ __forceinline__ float absmax4(const float4& v)
{
    return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

}  // namespace quant
}  // namespace sherry
