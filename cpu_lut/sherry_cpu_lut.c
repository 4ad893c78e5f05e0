/*
 * CPU COMPARISON KERNEL -- the stronger timed CPU baseline of bench.py.
 *
 * The Sherry page's own CPU inference scheme ("Sherry framework: ternary
 * quantisation and 3:4 sparsity for LLM inference", pnsm.cn/news/1195499,
 * sec. 2.2 steps 1-4 and sec. 5.1), on x86 with AVX2:
 *   1. every 4-element segment of the int8 activations gets a 16-entry
 *      table: entry p is the segment's dot product with the ternary group
 *      of pattern p whose first kept weight is +1;
 *   2. the tables are read with vpshufb (_mm256_shuffle_epi8), 32 weight
 *      rows per instruction, indexed by the rows' 4-bit patterns;
 *   3. the group's sign bit negates the looked-up value;
 *   4. the values are summed in integers, then scaled once in fp32.
 *
 * It is neither the oracle nor part of the GPU library: nothing under
 * sparse_bit_matmul_b200/ links, imports or calls it, and it shares no code
 * with either.  Only tests/ and bench.py load it.
 *
 * Readings:
 *   - code -> (pattern, sign): pattern4 = z | (s1^s0)<<2 | (s2^s0)<<3,
 *     sign = s0, for code = z | s0<<2 | s1<<3 | s2<<4 (the bijection of the
 *     page's 4-bit pattern plus one sign bit);
 *   - table entries are 16-bit: with int8 activations a group sum reaches
 *     +-381, more than a byte holds, so each table is kept as a low-byte and
 *     a high-byte table (two vpshufb per lookup) and the sign is applied to
 *     16-bit lanes (_mm256_sign_epi16) where the page's listing applies the
 *     byte form;
 *   - y[m][n] = (float)((float)acc[m][n] * alpha[n]) * s[m].
 * Compile with -ffp-contract=off.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif
#if defined(__x86_64__) || defined(__i386__)
#include <immintrin.h>
#define LUT_HAVE_X86 1
#else
#define LUT_HAVE_X86 0
#endif

#define LUT_OK 0
#define LUT_BAD_ARG 1
#define LUT_BAD_SHAPE 2
#define LUT_ROWS 32        /* rows per lookup: the 32 bytes of a 256-bit vpshufb */
#define LUT_RUN 64         /* groups summed in int16 before widening: 64 * 381 < 32767 */

static int64_t row_blocks(int64_t N) { return (N + LUT_ROWS - 1) / LUT_ROWS; }

/* Bytes of the prepared weights: [row block][group][32 index bytes]. */
int64_t lut_prepared_bytes(int64_t N, int64_t K) { return row_blocks(N) * LUT_ROWS * (K / 4); }

/* 5-bit code g of a canonical row (stream bits [5g, 5g+5), LSB first). */
static unsigned code_at(const uint8_t* row, int64_t g)
{
    const int64_t bit = 5 * g;
    unsigned v = row[bit >> 3];
    if ((bit & 7) > 3) v |= (unsigned)row[(bit >> 3) + 1] << 8;
    return (v >> (bit & 7)) & 31u;
}

/* Canonical codes [N][5K/32] -> index bytes pattern4 | sign << 4, 32 rows
 * of one group side by side.  Rows past N get byte 0 (their sums are never
 * stored). */
int lut_prepare(const uint8_t* codes, int64_t N, int64_t K, uint8_t* prepared)
{
    if (!codes || !prepared || N <= 0 || K <= 0) return LUT_BAD_ARG;
    if (K % 32 != 0) return LUT_BAD_SHAPE;
    const int64_t G = K / 4, rb_count = row_blocks(N), row_bytes = K / 32 * 5;
#pragma omp parallel for schedule(static)
    for (int64_t rb = 0; rb < rb_count; ++rb)
        for (int r = 0; r < LUT_ROWS; ++r) {
            const int64_t n = rb * LUT_ROWS + r;
            for (int64_t g = 0; g < G; ++g) {
                uint8_t b = 0;
                if (n < N) {
                    const unsigned c = code_at(codes + n * row_bytes, g);
                    const unsigned z = c & 3u, s0 = (c >> 2) & 1u, s1 = (c >> 3) & 1u, s2 = (c >> 4) & 1u;
                    b = (uint8_t)(z | ((s1 ^ s0) << 2) | ((s2 ^ s0) << 3) | (s0 << 4));
                }
                prepared[(rb * G + g) * LUT_ROWS + r] = b;
            }
        }
    return LUT_OK;
}

/* Step 1: the 16 entries of every segment, split into low and high bytes. */
static void build_tables(const int8_t* q, int64_t G, uint8_t* tlo, uint8_t* thi)
{
#pragma omp parallel for schedule(static)
    for (int64_t g = 0; g < G; ++g) {
        const int8_t* seg = q + 4 * g;
        for (int p = 0; p < 16; ++p) {
            const int z = p & 3;
            int t = 0, j = 0;
            for (int i = 0; i < 4; ++i) {
                if (i == z) continue;
                /* kept weight j: +1 for the first, then bits 2 and 3 of p */
                const int neg = (j == 0) ? 0 : (p >> (1 + j)) & 1;
                t += neg ? -seg[i] : seg[i];
                ++j;
            }
            tlo[g * 16 + p] = (uint8_t)(t & 0xFF);
            thi[g * 16 + p] = (uint8_t)((t >> 8) & 0xFF);
        }
    }
}

static void block_scalar(const uint8_t* idx, const uint8_t* tlo, const uint8_t* thi, int64_t G, int32_t acc[LUT_ROWS])
{
    for (int r = 0; r < LUT_ROWS; ++r) acc[r] = 0;
    for (int64_t g = 0; g < G; ++g)
        for (int r = 0; r < LUT_ROWS; ++r) {
            const unsigned b = idx[g * LUT_ROWS + r], p = b & 15u;
            const int16_t v = (int16_t)(uint16_t)(tlo[g * 16 + p] | (thi[g * 16 + p] << 8));
            acc[r] += (b & 16u) ? -v : v;
        }
}

#if LUT_HAVE_X86
/* Steps 2-4 for one block of 32 rows: two vpshufb per group (low and high
 * bytes of the entries), the sign on 16-bit lanes, int16 sums widened every
 * LUT_RUN groups. */
__attribute__((target("avx2"))) static void block_avx2(const uint8_t* idx, const uint8_t* tlo,
                                                       const uint8_t* thi, int64_t G, int32_t acc[LUT_ROWS])
{
    const __m256i nib = _mm256_set1_epi8(0x0F), sbit = _mm256_set1_epi8(0x10), one = _mm256_set1_epi16(1);
    for (int r = 0; r < LUT_ROWS; ++r) acc[r] = 0;
    for (int64_t g0 = 0; g0 < G; g0 += LUT_RUN) {
        const int64_t g1 = g0 + LUT_RUN < G ? g0 + LUT_RUN : G;
        __m256i a_lo = _mm256_setzero_si256(), a_hi = _mm256_setzero_si256();
        for (int64_t g = g0; g < g1; ++g) {
            const __m256i ix = _mm256_loadu_si256((const __m256i*)(idx + g * LUT_ROWS));
            const __m256i tl = _mm256_broadcastsi128_si256(_mm_loadu_si128((const __m128i*)(tlo + g * 16)));
            const __m256i th = _mm256_broadcastsi128_si256(_mm_loadu_si128((const __m128i*)(thi + g * 16)));
            const __m256i pi = _mm256_and_si256(ix, nib);
            const __m256i L = _mm256_shuffle_epi8(tl, pi), H = _mm256_shuffle_epi8(th, pi);
            const __m256i sm = _mm256_cmpeq_epi8(_mm256_and_si256(ix, sbit), sbit);   /* 0xFF: negative group */
            const __m256i s_lo = _mm256_or_si256(_mm256_unpacklo_epi8(sm, sm), one);  /* -1 or +1 */
            const __m256i s_hi = _mm256_or_si256(_mm256_unpackhi_epi8(sm, sm), one);
            a_lo = _mm256_add_epi16(a_lo, _mm256_sign_epi16(_mm256_unpacklo_epi8(L, H), s_lo));
            a_hi = _mm256_add_epi16(a_hi, _mm256_sign_epi16(_mm256_unpackhi_epi8(L, H), s_hi));
        }
        int16_t lo[16], hi[16];
        _mm256_storeu_si256((__m256i*)lo, a_lo);
        _mm256_storeu_si256((__m256i*)hi, a_hi);
        /* unpack works inside 128-bit lanes: a_lo holds rows 0-7 and 16-23,
         * a_hi rows 8-15 and 24-31 */
        for (int e = 0; e < 8; ++e) {
            acc[e] += lo[e];
            acc[e + 16] += lo[e + 8];
            acc[e + 8] += hi[e];
            acc[e + 24] += hi[e + 8];
        }
    }
}
#endif

int lut_has_avx2(void)
{
#if LUT_HAVE_X86
    __builtin_cpu_init();
    return __builtin_cpu_supports("avx2") ? 1 : 0;
#else
    return 0;
#endif
}

/* y fp32 [M][N] (and acc int32 [M][N] when not NULL) from int8 activations
 * q [M][K] with scales s [M], prepared weights and alpha [N].  force_scalar
 * selects the plain-C lookup loop. */
int lut_gemm(const int8_t* q, const float* s, const uint8_t* prepared, const float* alpha, int64_t M, int64_t N,
             int64_t K, float* y, int32_t* acc_out, int force_scalar)
{
    if (!q || !s || !prepared || !alpha || !y || M <= 0 || N <= 0 || K <= 0) return LUT_BAD_ARG;
    if (K % 32 != 0) return LUT_BAD_SHAPE;
    const int64_t G = K / 4, rb_count = row_blocks(N);
    uint8_t* tlo = (uint8_t*)malloc((size_t)(G * 16));
    uint8_t* thi = (uint8_t*)malloc((size_t)(G * 16));
    if (!tlo || !thi) {
        free(tlo);
        free(thi);
        return LUT_BAD_ARG;
    }
    const int use_avx2 = !force_scalar && lut_has_avx2();
    for (int64_t m = 0; m < M; ++m) {
        build_tables(q + m * K, G, tlo, thi);
#pragma omp parallel for schedule(static)
        for (int64_t rb = 0; rb < rb_count; ++rb) {
            int32_t acc[LUT_ROWS];
            const uint8_t* idx = prepared + rb * G * LUT_ROWS;
#if LUT_HAVE_X86
            if (use_avx2) block_avx2(idx, tlo, thi, G, acc);
            else block_scalar(idx, tlo, thi, G, acc);
#else
            (void)use_avx2;
            block_scalar(idx, tlo, thi, G, acc);
#endif
            for (int r = 0; r < LUT_ROWS; ++r) {
                const int64_t n = rb * LUT_ROWS + r;
                if (n >= N) break;
                if (acc_out) acc_out[m * N + n] = acc[r];
                const float t = (float)acc[r] * alpha[n];
                y[m * N + n] = t * s[m];
            }
        }
    }
    free(tlo);
    free(thi);
    return LUT_OK;
}

int lut_num_threads(void)
{
    int n = 1;
#ifdef _OPENMP
#pragma omp parallel
    {
#pragma omp single
        n = omp_get_num_threads();
    }
#endif
    return n;
}
