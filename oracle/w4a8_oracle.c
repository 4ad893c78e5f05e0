/*
 * ORACLE -- test infrastructure only.
 *
 * A plain, slow, obviously correct CPU statement of the W4A8 FastGEMM path:
 * per-channel symmetric int4 weights, int8 activations, the int4 -> int8
 * conversion by a 4-bit left shift, an int8 contraction with int32 sums and
 * a division by 16 before dequantisation.  Only the tests, the smoke check
 * and the CPU baseline leg of the benchmark may load this file's library.  It
 * shares no code, header, table or constant with the CUDA library under
 * sparse_bit_matmul_b200/.
 *
 * Source: "OdysseyLLM: A Speed Odyssey for Deployable Quantization of LLMs"
 * (review page, xllm-io.github.io/paper-review/blog/odysseyllm):
 *   sec. 3.1 (Figure 2)  the W4A8 row: SINT4 weights, INT8 activations,
 *                        per-channel; SINT4 -> SINT8 (x16) -> INT8 GEMM ->
 *                        dequantise after dividing by 16
 *   sec. 3.2 (Figure 4)  SINT4toS8: the 4-bit two's complement value moved to
 *                        the high half of a byte (shift left by 4) is the
 *                        int8 value 16*w; no subtraction, no int32 unpacking
 *   sec. 3.3             weight scale S = max(|gamma max W|, |beta min W|) /
 *                        (2^(N-1) - 1), W_q = clamp(W / S, -2^(N-1),
 *                        2^(N-1) - 1), N = 4 bits
 *   sec. 5.2             two's complement table of SINT4, the worked
 *                        conversion -7 = 1001 -> 1001 0000 = -112, and the
 *                        identity sum(A*W*16)/16 = sum(A*W)
 *
 * Readings taken where the page is silent, each with its reason:
 *   - gamma = beta = 1: the learnable clipping factors need calibration data,
 *     which this path does not have; "per-channel" = one S per output row n
 *     of W [N][K];
 *   - S = a / 7.0f in fp32 (a = max(|max_k W|, |min_k W|)), W_q =
 *     clamp(rint(W / S), -8, 7) with fp32 IEEE division and round half to
 *     even; a == 0 gives S = 0 and W_q = 0: the page gives no rounding
 *     rule, and these are the activation quantiser's rules;
 *   - activations: per-token absmax int8 (s = a / 127), the same quantiser as
 *     the Sherry path (oracle_quant_act);
 *   - storage: row n starts at byte n * K/2; byte j holds weight 2j in its
 *     low nibble and weight 2j+1 in its high nibble (two's complement): the
 *     page shows single values only, and low-first matches the Sherry stream;
 *   - y[m][n] = (float)((float)acc[m][n] * S[n]) * s[m], two separately
 *     rounded fp32 products in this order, acc = the int32 sum after the
 *     division by 16: the same order as the Sherry epilogue, so y is
 *     reproducible bit for bit.
 *
 * Compile with -ffp-contract=off so that no multiply-add is fused.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define W4_OK 0
#define W4_BAD_ARG 1
#define W4_BAD_SHAPE 2
#define W4_NONFINITE 3
#define W4_OVERFLOW 4
#define W4_NOT_MULTIPLE 5

/* ---- weight quantisation (sec. 3.3, gamma = beta = 1) -------------------- */
int w4a8_oracle_quantise(const float* W, int64_t N, int64_t K, int8_t* Wq, float* S)
{
    if (!W || !Wq || !S || N <= 0 || K <= 0) return W4_BAD_ARG;
    for (int64_t i = 0; i < N * K; ++i)
        if (!isfinite(W[i])) return W4_NONFINITE;
    const float qmax = 7.0f;                 /* 2^(4-1) - 1 */
    for (int64_t n = 0; n < N; ++n) {
        const float* w = W + n * K;
        float hi = w[0], lo = w[0];
        for (int64_t k = 1; k < K; ++k) {
            if (w[k] > hi) hi = w[k];
            if (w[k] < lo) lo = w[k];
        }
        float a = fabsf(hi);
        if (fabsf(lo) > a) a = fabsf(lo);
        if (a == 0.0f) {
            S[n] = 0.0f;
            memset(Wq + n * K, 0, (size_t)K);
            continue;
        }
        const float sc = a / qmax;
        S[n] = sc;
        for (int64_t k = 0; k < K; ++k) {
            float r = rintf(w[k] / sc);
            if (r > 7.0f) r = 7.0f;
            if (r < -8.0f) r = -8.0f;
            Wq[n * K + k] = (int8_t)r;
        }
    }
    return W4_OK;
}

/* ---- storage of SINT4 values (sec. 5.2 two's complement) ----------------- */
int64_t w4a8_oracle_row_bytes(int64_t K) { return K / 2; }

int w4a8_oracle_pack(const int8_t* Wq, int64_t N, int64_t K, uint8_t* packed)
{
    if (!Wq || !packed || N <= 0 || K <= 0) return W4_BAD_ARG;
    if (K % 2 != 0) return W4_BAD_SHAPE;
    for (int64_t i = 0; i < N * K; ++i)
        if (Wq[i] < -8 || Wq[i] > 7) return W4_BAD_ARG;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t j = 0; j < K / 2; ++j) {
            /* the low 4 bits of a two's complement int8 are the SINT4 bits */
            unsigned lo = (unsigned)(uint8_t)Wq[n * K + 2 * j] & 0xFu;
            unsigned hi = (unsigned)(uint8_t)Wq[n * K + 2 * j + 1] & 0xFu;
            packed[n * (K / 2) + j] = (uint8_t)(lo | (hi << 4));
        }
    return W4_OK;
}

/* SINT4 bits -> value: bit 3 has weight -8 (two's complement). */
static int sint4_value(unsigned nib)
{
    return (int)(nib & 7u) - (int)(nib & 8u);
}

int w4a8_oracle_unpack(const uint8_t* packed, int64_t N, int64_t K, int8_t* Wq)
{
    if (!packed || !Wq || N <= 0 || K <= 0) return W4_BAD_ARG;
    if (K % 2 != 0) return W4_BAD_SHAPE;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t b = packed[n * (K / 2) + k / 2];
            unsigned nib = (k % 2 == 0) ? (b & 0xFu) : (unsigned)(b >> 4);
            Wq[n * K + k] = (int8_t)sint4_value(nib);
        }
    return W4_OK;
}

/* ---- SINT4toS8 (sec. 3.2, 5.2): the 4 bits become the high half of a byte */
int w4a8_oracle_sint4_to_s8(int nibble)
{
    uint8_t byte = (uint8_t)(((unsigned)nibble & 0xFu) << 4);
    return (int)(int8_t)byte;
}

/* ---- contraction (sec. 3.1 W4A8 row, sec. 5.2) --------------------------
 * acc16[m][n] = sum_k q[m][k] * SINT4toS8(w[n][k]) is what an int8 GEMM with
 * an int32 accumulator computes (checked to fit int32); it is a multiple of
 * 16 (checked), and acc = acc16 / 16. */
int w4a8_oracle_gemm(const int8_t* q, const uint8_t* packed, int64_t M, int64_t N, int64_t K,
                     int32_t* acc)
{
    if (!q || !packed || !acc || M <= 0 || N <= 0 || K <= 0) return W4_BAD_ARG;
    if (K % 2 != 0) return W4_BAD_SHAPE;
    int bad = W4_OK;
    for (int64_t n = 0; n < N && bad == W4_OK; ++n) {
        const uint8_t* row = packed + n * (K / 2);
        for (int64_t m = 0; m < M; ++m) {
            int64_t sum16 = 0;
            for (int64_t k = 0; k < K; ++k) {
                unsigned nib = (k % 2 == 0) ? (row[k / 2] & 0xFu) : (unsigned)(row[k / 2] >> 4);
                sum16 += (int64_t)q[m * K + k] * (int64_t)w4a8_oracle_sint4_to_s8((int)nib);
            }
            if (sum16 > INT32_MAX || sum16 < INT32_MIN) {
                bad = W4_OVERFLOW;
                break;
            }
            if (sum16 % 16 != 0) {
                bad = W4_NOT_MULTIPLE;
                break;
            }
            acc[m * N + n] = (int32_t)(sum16 / 16);
        }
    }
    return bad;
}

/* ---- dequantisation ------------------------------------------------------ */
void w4a8_oracle_epilogue(const int32_t* acc, const float* S, const float* s, int64_t M, int64_t N,
                          float* y)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float t = (float)acc[m * N + n] * S[n];
            y[m * N + n] = t * s[m];
        }
}
