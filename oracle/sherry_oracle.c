/*
 * ORACLE -- test infrastructure only.
 *
 * A plain, slow, obviously correct CPU statement of what the Sherry 3:4
 * ternary matmul computes.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this file's library.  It shares no
 * code, header, table or constant with the CUDA library under
 * sparse_bit_matmul_b200/.
 *
 * Source: "Sherry framework: ternary quantisation and 3:4 sparsity for LLM
 * inference" (pnsm.cn/news/1195499):
 *   sec. 1.1        3:4 pattern: every 4 weights hold exactly 3 nonzeros
 *   sec. 2.1        offline compression to 1.25 bit/weight (one 5-bit code per
 *                   group of 4: a pattern part plus a sign bit)
 *   sec. 2.2        online inference: 4-element activation segments, a
 *                   16-entry table per segment, sign application, integer
 *                   accumulation, one float scale at the end
 *   sec. 3.1        objective  min ||W - alpha T||^2,  T in {-1,0,+1}^4,
 *                   ||T||_0 = 3; solution: keep the 3 largest |w| with their
 *                   signs
 *
 * Readings taken where the page is silent or garbled, each with its reason:
 *   - groups run along K, the reduction axis: the page's 4-element activation
 *     segments only line up with weight groups along K;
 *   - alpha is one scale per output row n: sum of kept |w| (fp64, ascending k)
 *     divided by 0.75*K, rounded once to fp32.  One fp32 alpha per group of
 *     4 would cost 8 bit/weight against the page's 1.25, and with exactly 3
 *     nonzeros per group ||T||^2 = 0.75 K is fixed, so this alpha and the
 *     per-group choice of T minimise ||W - alpha T||^2 together;
 *   - ties in |w|: the lowest index is the one zeroed (every choice gives the
 *     same error; one is needed for bit-exact codes);
 *   - sign of a kept weight: negative iff w < 0.0f (so -0.0 and +0.0 are +),
 *     the plain IEEE comparison;
 *   - code = z | s0<<2 | s1<<3 | s2<<4, z = zeroed position, s_j = sign bit
 *     of the j-th kept position in ascending order (1 = negative): the page
 *     fixes only the size, 5 bits;
 *   - the page's (4-bit pattern, 1 dominant-sign bit) form is the bijection
 *     pattern4 = z | (s1^s0)<<2 | (s2^s0)<<3, sign = s0: a literal "which 3
 *     of 4 are nonzero" mask gives only 8 states with the sign bit and cannot
 *     hold the page's own mixed-sign example block [-1, 0, +1, -1];
 *   - row n's code stream starts at byte n*(5K/32); code j occupies stream
 *     bits [5j, 5j+5), least significant bit first; K % 32 == 0 (rows of
 *     whole bytes; every workload's K qualifies);
 *   - activations: per token absmax a; s = a/127 (fp32 division); q =
 *     clamp(rint(x/s), -127, 127) with round-half-to-even; a == 0 gives
 *     s = 0 and q = 0: the page gives no rule, and this is the plainest
 *     symmetric one (it never produces -128);
 *   - y[m][n] = (float)((float)acc[m][n] * alpha[n]) * s[m], two separately
 *     rounded fp32 products in this order: the page says one float scale at
 *     the end; a fixed order keeps y reproducible bit for bit, and
 *     float(acc) is exact because |acc| <= 127 * 0.75 K < 2^24.
 *
 * Compile with -ffp-contract=off so that no multiply-add is fused.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- status codes ------------------------------------------------------ */
#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_BAD_SHAPE 2
#define ORACLE_NONFINITE 3
#define ORACLE_OVERFLOW 4

/* ---- ternarisation of one group (sec. 3.1) ------------------------------ */
/* Index of the group element with the smallest |w|; lowest index on ties. */
static int smallest_magnitude_index(const float w[4])
{
    int z = 0;
    for (int i = 1; i < 4; ++i)
        if (fabsf(w[i]) < fabsf(w[z])) z = i;
    return z;
}

/* T for one group: zero at z, sign of w elsewhere (+1 for w >= 0). */
static void ternarise_group(const float w[4], int8_t t[4])
{
    int z = smallest_magnitude_index(w);
    for (int i = 0; i < 4; ++i)
        t[i] = (i == z) ? 0 : (w[i] < 0.0f ? -1 : 1);
}

/*
 * Quantise W[N][K] (row-major) to T[N][K] in {-1,0,+1} and alpha[N].
 * alpha64 (optional) receives the fp64 scale before rounding to fp32.
 */
int oracle_quantise(const float* W, int64_t N, int64_t K, int8_t* T, float* alpha,
                    double* alpha64)
{
    if (!W || !T || !alpha || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    if (K % 4 != 0) return ORACLE_BAD_SHAPE;
    for (int64_t i = 0; i < N * K; ++i)
        if (!isfinite(W[i])) return ORACLE_NONFINITE;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        const float* w = W + n * K;
        int8_t* t = T + n * K;
        double kept = 0.0;
        for (int64_t g = 0; g < K / 4; ++g) {
            ternarise_group(w + 4 * g, t + 4 * g);
        }
        for (int64_t k = 0; k < K; ++k)
            if (t[k] != 0) kept += fabs((double)w[k]);
        double a = kept / (0.75 * (double)K);
        if (alpha64) alpha64[n] = a;
        alpha[n] = (float)a;
    }
    return ORACLE_OK;
}

/* ---- 5-bit code of a group (sec. 2.1) ----------------------------------- */
/* Returns -1 if t is not a valid 3:4 ternary group. */
int oracle_encode_group(const int8_t t[4])
{
    int z = -1, nz = 0;
    for (int i = 0; i < 4; ++i) {
        if (t[i] == 0) {
            if (z >= 0) return -1;
            z = i;
        } else if (t[i] == 1 || t[i] == -1) {
            ++nz;
        } else {
            return -1;
        }
    }
    if (z < 0 || nz != 3) return -1;
    int code = z, j = 0;
    for (int i = 0; i < 4; ++i) {
        if (i == z) continue;
        if (t[i] < 0) code |= 1 << (2 + j);
        ++j;
    }
    return code;
}

void oracle_decode_group(int code, int8_t t[4])
{
    int z = code & 3, j = 0;
    for (int i = 0; i < 4; ++i) {
        if (i == z) {
            t[i] = 0;
        } else {
            t[i] = ((code >> (2 + j)) & 1) ? -1 : 1;
            ++j;
        }
    }
}

/* The page's (pattern, sign) form and back. */
void oracle_code_to_pattern_sign(int code, int* pattern4, int* sign)
{
    int z = code & 3, s0 = (code >> 2) & 1, s1 = (code >> 3) & 1, s2 = (code >> 4) & 1;
    *pattern4 = z | ((s1 ^ s0) << 2) | ((s2 ^ s0) << 3);
    *sign = s0;
}

int oracle_pattern_sign_to_code(int pattern4, int sign)
{
    int z = pattern4 & 3, d1 = (pattern4 >> 2) & 1, d2 = (pattern4 >> 3) & 1;
    int s0 = sign & 1;
    return z | (s0 << 2) | ((d1 ^ s0) << 3) | ((d2 ^ s0) << 4);
}

/* ---- bit stream packing ------------------------------------------------- */
static void put_bit(uint8_t* stream, int64_t bit, int v)
{
    if (v) stream[bit >> 3] |= (uint8_t)(1u << (bit & 7));
}

static int get_bit(const uint8_t* stream, int64_t bit)
{
    return (stream[bit >> 3] >> (bit & 7)) & 1;
}

int64_t oracle_row_bytes(int64_t K) { return K * 5 / 32; }

/* T[N][K] -> codes[N][5K/32]. */
int oracle_pack(const int8_t* T, int64_t N, int64_t K, uint8_t* codes)
{
    if (!T || !codes || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    if (K % 32 != 0) return ORACLE_BAD_SHAPE;
    int64_t rb = oracle_row_bytes(K);
    memset(codes, 0, (size_t)(N * rb));
    for (int64_t n = 0; n < N; ++n) {
        uint8_t* row = codes + n * rb;
        for (int64_t g = 0; g < K / 4; ++g) {
            int c = oracle_encode_group(T + n * K + 4 * g);
            if (c < 0) return ORACLE_BAD_ARG;
            for (int b = 0; b < 5; ++b) put_bit(row, 5 * g + b, (c >> b) & 1);
        }
    }
    return ORACLE_OK;
}

/* codes[N][5K/32] -> T[N][K]. */
int oracle_unpack(const uint8_t* codes, int64_t N, int64_t K, int8_t* T)
{
    if (!T || !codes || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    if (K % 32 != 0) return ORACLE_BAD_SHAPE;
    int64_t rb = oracle_row_bytes(K);
    for (int64_t n = 0; n < N; ++n) {
        const uint8_t* row = codes + n * rb;
        for (int64_t g = 0; g < K / 4; ++g) {
            int c = 0;
            for (int b = 0; b < 5; ++b) c |= get_bit(row, 5 * g + b) << b;
            oracle_decode_group(c, T + n * K + 4 * g);
        }
    }
    return ORACLE_OK;
}

/* ---- activation quantisation -------------------------------------------- */
int oracle_quant_act(const float* x, int64_t M, int64_t K, int8_t* q, float* s)
{
    if (!x || !q || !s || M <= 0 || K <= 0) return ORACLE_BAD_ARG;
    for (int64_t m = 0; m < M; ++m) {
        const float* xr = x + m * K;
        float a = 0.0f;
        for (int64_t k = 0; k < K; ++k)
            if (fabsf(xr[k]) > a) a = fabsf(xr[k]);
        if (a == 0.0f) {
            s[m] = 0.0f;
            memset(q + m * K, 0, (size_t)K);
            continue;
        }
        float sc = a / 127.0f;
        s[m] = sc;
        for (int64_t k = 0; k < K; ++k) {
            float r = rintf(xr[k] / sc);
            if (r > 127.0f) r = 127.0f;
            if (r < -127.0f) r = -127.0f;
            q[m * K + k] = (int8_t)r;
        }
    }
    return ORACLE_OK;
}

/* ---- integer contraction (addition-only in effect: T in {-1,0,1}) -------- */
/* acc[m][n] = sum_k q[m][k] * T[n][k]; exact in int64, must fit int32. */
int oracle_gemm(const int8_t* q, const int8_t* T, int64_t M, int64_t N, int64_t K,
                int32_t* acc)
{
    if (!q || !T || !acc || M <= 0 || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t m = 0; m < M; ++m) {
            int64_t sum = 0;
            for (int64_t k = 0; k < K; ++k)
                sum += (int64_t)q[m * K + k] * (int64_t)T[n * K + k];
            if (sum > INT32_MAX || sum < INT32_MIN) bad = 1;
            acc[m * N + n] = (int32_t)sum;
        }
    }
    return bad ? ORACLE_OVERFLOW : ORACLE_OK;
}

/*
 * The page's table form of the same contraction (sec. 2.2): for every
 * 4-element activation segment build 16 entries, entry p = segment . P[p]
 * where P[p] is the ternary group of pattern p with a +1 sign bit; look up
 * with the pattern of the weight group, negate when the sign bit is set,
 * accumulate in integers.  codes are the packed rows; acc[m][n].
 */
int oracle_gemm_lut(const int8_t* q, const uint8_t* codes, int64_t M, int64_t N, int64_t K,
                    int32_t* acc)
{
    if (!q || !codes || !acc || M <= 0 || N <= 0 || K <= 0) return ORACLE_BAD_ARG;
    if (K % 32 != 0) return ORACLE_BAD_SHAPE;
    int8_t P[16][4];
    for (int p = 0; p < 16; ++p) oracle_decode_group(oracle_pattern_sign_to_code(p, 0), P[p]);
    int64_t G = K / 4, rb = oracle_row_bytes(K);
    int32_t* lut = (int32_t*)malloc((size_t)(G * 16) * sizeof(int32_t));
    if (!lut) return ORACLE_BAD_ARG;
    for (int64_t m = 0; m < M; ++m) {
        for (int64_t g = 0; g < G; ++g)
            for (int p = 0; p < 16; ++p) {
                int32_t e = 0;
                for (int i = 0; i < 4; ++i) e += (int32_t)q[m * K + 4 * g + i] * P[p][i];
                lut[g * 16 + p] = e;
            }
#pragma omp parallel for schedule(static)
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t* row = codes + n * rb;
            int64_t sum = 0;
            for (int64_t g = 0; g < G; ++g) {
                int c = 0;
                for (int b = 0; b < 5; ++b) c |= get_bit(row, 5 * g + b) << b;
                int pat, sg;
                oracle_code_to_pattern_sign(c, &pat, &sg);
                int32_t v = lut[g * 16 + pat];
                sum += sg ? -v : v;
            }
            acc[m * N + n] = (int32_t)sum;
        }
    }
    free(lut);
    return ORACLE_OK;
}

/* ---- epilogue ------------------------------------------------------------ */
void oracle_epilogue(const int32_t* acc, const float* alpha, const float* s, int64_t M,
                     int64_t N, float* y)
{
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            float t = (float)acc[m * N + n] * alpha[n];
            y[m * N + n] = t * s[m];
        }
}

/* ---- the whole path from packed codes, for the timed CPU baseline -------- */
/* unpack -> contract -> epilogue; acc may be NULL (a temporary is used). */
int oracle_forward(const int8_t* q, const float* s, const uint8_t* codes, const float* alpha,
                   int64_t M, int64_t N, int64_t K, float* y, int32_t* acc)
{
    if (!q || !s || !codes || !alpha || !y || M <= 0 || N <= 0 || K <= 0)
        return ORACLE_BAD_ARG;
    int8_t* T = (int8_t*)malloc((size_t)(N * K));
    int32_t* a = acc ? acc : (int32_t*)malloc((size_t)(M * N) * sizeof(int32_t));
    if (!T || !a) {
        free(T);
        if (!acc) free(a);
        return ORACLE_BAD_ARG;
    }
    int rc = oracle_unpack(codes, N, K, T);
    if (rc == ORACLE_OK) rc = oracle_gemm(q, T, M, N, K, a);
    if (rc == ORACLE_OK) oracle_epilogue(a, alpha, s, M, N, y);
    free(T);
    if (!acc) free(a);
    return rc;
}

int oracle_num_threads(void)
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
