// Host half of libsherry_b200: offline ternarisation and packing (Sherry page,
// pnsm.cn/news/1195499, sec. 3.1 objective and sec. 2.1 5-bit encoding), the
// unpacker, and the size and status helpers of the C ABI.
//
// Group rule (sec. 3.1: keep the 3 largest |w| with their signs): the
// element with the smallest magnitude is zeroed.  Magnitudes are compared as
// the IEEE bit pattern with the sign cleared, which orders finite floats
// exactly like |w| and makes -0.0 and +0.0 equal; the first (lowest index)
// of equal minima is zeroed.  A kept weight is negative only when w < 0.0f,
// so -0.0 counts as positive.
#include <cmath>
#include <cstdint>
#include <cstring>

#include "sherry.h"
#include "sherry_internal.h"

namespace {

inline uint32_t float_bits(float f)
{
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return u;
}

// 5-bit code of one group plus its kept-magnitude sum (fp64, in position order).
inline uint32_t encode_group(const float* w, double* kept_sum)
{
    uint32_t mag[4], neg[4];
    for (int i = 0; i < 4; ++i) {
        uint32_t b = float_bits(w[i]);
        mag[i] = b & 0x7fffffffu;
        neg[i] = (b >> 31) & (mag[i] != 0u);
    }
    // zero position: first index attaining the minimum magnitude
    uint32_t z = 0, best = mag[0];
    for (uint32_t i = 1; i < 4; ++i) {
        bool smaller = mag[i] < best;
        z = smaller ? i : z;
        best = smaller ? mag[i] : best;
    }
    uint32_t code = z, slot = 2;
    double s = *kept_sum;
    for (uint32_t i = 0; i < 4; ++i) {
        if (i == z) continue;
        code |= neg[i] << slot;
        ++slot;
        s += (double)std::fabs(w[i]);
    }
    *kept_sum = s;
    return code;
}

}  // namespace

extern "C" {

const char* sherry_status_string(int status)
{
    switch (status) {
    case SHERRY_OK: return "ok";
    case SHERRY_ERR_INVALID_ARG: return "invalid argument";
    case SHERRY_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case SHERRY_ERR_NONFINITE: return "non-finite weight";
    case SHERRY_ERR_CUDA: return "CUDA error";
    case SHERRY_ERR_DEVICE: return "unsupported device";
    case SHERRY_ERR_WORKSPACE: return "workspace too small: call sherry_reserve first";
    default: return "unknown status";
    }
}

int sherry_version(void) { return 10000; }

size_t sherry_packed_bytes(int64_t N, int64_t K)
{
    if (!sherry_shape_ok(1, N, K)) return 0;
    return (size_t)N * (size_t)(K / 32) * 5u;
}

size_t sherry_native_bytes(int64_t N, int64_t K)
{
    if (!sherry_shape_ok(1, N, K)) return 0;
    return (size_t)sherry_row_tiles(N) * (size_t)sherry_k_chunks(K) * SHERRY_CHUNK_BYTES_PER_TILE;
}

int sherry_pack(const float* W, int64_t N, int64_t K, uint8_t* codes, float* alpha)
{
    if (!W || !codes || !alpha) return SHERRY_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0) return SHERRY_ERR_INVALID_ARG;
    if (!sherry_shape_ok(1, N, K)) return SHERRY_ERR_UNSUPPORTED_SHAPE;

    int nonfinite = 0;
#pragma omp parallel for schedule(static) reduction(| : nonfinite)
    for (int64_t n = 0; n < N; ++n) {
        const float* w = W + n * K;
        for (int64_t k = 0; k < K; ++k)
            nonfinite |= ((float_bits(w[k]) & 0x7f800000u) == 0x7f800000u);
    }
    if (nonfinite) return SHERRY_ERR_NONFINITE;

    const int64_t row_bytes = K / 32 * 5;
    const double denom = 0.75 * (double)K;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const float* w = W + n * K;
        uint8_t* out = codes + n * row_bytes;
        double kept = 0.0;
        // 8 groups (32 weights) fill exactly 40 bits = 5 bytes
        for (int64_t blk = 0; blk < K / 32; ++blk) {
            uint64_t bits = 0;
            for (int g = 0; g < 8; ++g)
                bits |= (uint64_t)encode_group(w + blk * 32 + g * 4, &kept) << (5 * g);
            for (int b = 0; b < 5; ++b) out[blk * 5 + b] = (uint8_t)(bits >> (8 * b));
        }
        alpha[n] = (float)(kept / denom);
    }
    return SHERRY_OK;
}

int sherry_unpack(const uint8_t* codes, int64_t N, int64_t K, int8_t* T)
{
    if (!codes || !T) return SHERRY_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0) return SHERRY_ERR_INVALID_ARG;
    if (!sherry_shape_ok(1, N, K)) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    const int64_t row_bytes = K / 32 * 5;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t* in = codes + n * row_bytes;
        int8_t* t = T + n * K;
        for (int64_t blk = 0; blk < K / 32; ++blk) {
            uint64_t bits = 0;
            for (int b = 0; b < 5; ++b) bits |= (uint64_t)in[blk * 5 + b] << (8 * b);
            for (int g = 0; g < 8; ++g) {
                uint32_t c = (uint32_t)(bits >> (5 * g)) & 31u;
                uint32_t z = c & 3u, slot = 2;
                int8_t* o = t + blk * 32 + g * 4;
                for (uint32_t i = 0; i < 4; ++i) {
                    if (i == z) {
                        o[i] = 0;
                    } else {
                        o[i] = ((c >> slot) & 1u) ? (int8_t)-1 : (int8_t)1;
                        ++slot;
                    }
                }
            }
        }
    }
    return SHERRY_OK;
}

// ---------------------------------------------------------------------------
// W4A8 FastGEMM weights (OdysseyLLM review page,
// xllm-io.github.io/paper-review/blog/odysseyllm, sec. 3.3 and 5.2): one
// symmetric scale per output channel, S = a / 7 with a the largest |w| of
// the row (the clipping factors taken as 1), w_q = clamp(rint(w / S), -8, 7)
// in fp32 (IEEE division, ties to even); a == 0 gives S = 0 and w_q = 0.
// Stored as 4-bit two's complement, two per byte, even k in the low nibble.
// ---------------------------------------------------------------------------

static bool w4a8_shape_ok(int64_t M, int64_t N, int64_t K)
{
    return sherry_shape_ok(M, N, K) && K <= SHERRY_W4_MAX_K;
}

size_t sherry_w4a8_packed_bytes(int64_t N, int64_t K)
{
    if (!w4a8_shape_ok(1, N, K)) return 0;
    return (size_t)N * (size_t)(K / 2);
}

size_t sherry_w4a8_native_bytes(int64_t N, int64_t K)
{
    if (!w4a8_shape_ok(1, N, K)) return 0;
    return (size_t)sherry_row_tiles(N) * (size_t)sherry_k_chunks(K) * SHERRY_W4_CHUNK_BYTES;
}

int sherry_w4a8_pack(const float* W, int64_t N, int64_t K, uint8_t* w4, float* scale)
{
    if (!W || !w4 || !scale) return SHERRY_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0) return SHERRY_ERR_INVALID_ARG;
    if (!w4a8_shape_ok(1, N, K)) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    int nonfinite = 0;
#pragma omp parallel for schedule(static) reduction(| : nonfinite)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) nonfinite |= ((float_bits(W[n * K + k]) & 0x7f800000u) == 0x7f800000u);
    if (nonfinite) return SHERRY_ERR_NONFINITE;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const float* w = W + n * K;
        uint8_t* out = w4 + n * (K / 2);
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k) a = std::fmax(a, std::fabs(w[k]));
        const float S = a / 7.0f;
        scale[n] = S;
        for (int64_t k = 0; k < K; k += 2) {
            uint32_t nib[2] = {0u, 0u};
            if (a != 0.0f) {
                for (int e = 0; e < 2; ++e) {
                    const float r = std::fmin(std::fmax(std::rint(w[k + e] / S), -8.0f), 7.0f);
                    nib[e] = (uint32_t)(int32_t)r & 0xFu;
                }
            }
            out[k / 2] = (uint8_t)(nib[0] | (nib[1] << 4));
        }
    }
    return SHERRY_OK;
}

int sherry_w4a8_unpack(const uint8_t* w4, int64_t N, int64_t K, int8_t* Wq)
{
    if (!w4 || !Wq) return SHERRY_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0) return SHERRY_ERR_INVALID_ARG;
    if (!w4a8_shape_ok(1, N, K)) return SHERRY_ERR_UNSUPPORTED_SHAPE;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 2; ++j) {
            const uint8_t b = w4[n * (K / 2) + j];
            // sign-extend each nibble: (v ^ 8) - 8
            Wq[n * K + 2 * j] = (int8_t)((int)((b & 0xFu) ^ 8u) - 8);
            Wq[n * K + 2 * j + 1] = (int8_t)((int)((b >> 4) ^ 8u) - 8);
        }
    return SHERRY_OK;
}

}  // extern "C"
