// Host-side check of the decode kernel's work split and shared-memory
// indexing (decode::plan and the index expressions of sherry_decode_kernel,
// compiled from the kernel's own header for the host).  For many (M, N, K)
// and SM counts it checks that:
//   * the CTAs' row ranges tile [0, N) with 1 <= rows <= R, R % 4 == 0,
//     R % RT == 0, Q = R / RT, Q * P <= threads <= 512, and the K-parts tile
//     the chunks with no empty part;
//   * the shared-memory regions are in order, 16-byte aligned and end at
//     smem_bytes <= the budget; the activation chunk stride S is a multiple of
//     16 of at least 128;
//   * every shared-memory index the kernel forms (code prefetch, code loads
//     of each row group, activation loads and stores, the tail, partial sums,
//     row totals) and every native-layout word the prefetch reads stays
//     inside its region or buffer;
//   * every (row, K chunk) pair of a CTA is walked by exactly one thread, and
//     every piece of every ring step is copied exactly once into its slot.
// Prints "ok" and exits 0, or prints the first violation and exits 1.
#include <cstdio>
#include <cstdint>
#include <vector>

#include "decode.cuh"

using namespace sherry;

static int fail(const char* what, int64_t M, int64_t N, int64_t K, int sms)
{
    std::printf("%s: M=%lld N=%lld K=%lld sms=%d\n", what, (long long)M, (long long)N, (long long)K, sms);
    return 1;
}

static int check(int64_t M, int64_t N, int64_t K, int sms)
{
    const int64_t Kc = sherry_k_chunks(K);
    decode::Plan pl;
    if (!decode::plan(N, Kc, M, sms, &pl)) {
        // the launcher reports an unsupported shape; every M <= 8 with K up
        // to 16384 must have a plan
        if (M <= 8 && K <= 16384) return fail("no plan", M, N, K, sms);
        return 0;
    }
    const int R = pl.R, RT = pl.RT, Q = pl.Q, P = pl.P, CPT = pl.CPT, S = pl.S, G = pl.G, NS = pl.NS;
    if (!(NS == CPT || (NS >= 2 && NS <= decode::kMaxRing && NS < CPT))) return fail("ring slots", M, N, K, sms);
    const int nthr = pl.threads;
    if (R % 4 || R % RT || Q * RT != R || Q * P > nthr || nthr > decode::kMaxThreads || nthr % 32)
        return fail("row groups / threads", M, N, K, sms);
    if ((int64_t)P * CPT < Kc || (int64_t)(P - 1) * CPT >= Kc) return fail("K parts", M, N, K, sms);
    if (S < 128 || S % 16) return fail("activation stride", M, N, K, sms);
    const int Mi = (int)M;
    const int o_red = decode::kOffRed, o_alpha = decode::off_alpha(Mi, P, R);
    const int o_codes = decode::off_codes(Mi, P, R), o_q = decode::off_q(Mi, P, R, NS);
    const int smem = decode::smem_bytes(Mi, P, R, NS, Kc, S);
    if (smem != pl.smem || smem > decode::kSmemBudgetMax) return fail("smem size", M, N, K, sms);
    if (smem > decode::kSmemBudget && decode::plan_within(N, Kc, M, sms, decode::kSmemBudget, &pl))
        return fail("a two-CTA plan exists but was not taken", M, N, K, sms);
    if (o_red + P * Mi * R * 4 > o_alpha || o_alpha + R * 4 > o_codes ||
        o_codes + NS * P * 5 * R * 4 > o_q || (o_alpha | o_codes | o_q) % 16)
        return fail("smem regions", M, N, K, sms);
    const int64_t native_words = sherry_row_tiles(N) * Kc * SHERRY_CHUNK_WORDS * SHERRY_TILE_ROWS;
    const int QK = (int)Kc * S;
    int64_t covered = 0;
    for (int b = 0; b < G; ++b) {
        const int64_t r0 = decode::row_begin(N, b, G), r1 = decode::row_begin(N, b + 1, G);
        if (r0 != covered) return fail("row ranges not contiguous", M, N, K, sms);
        const int Rc = (int)(r1 - r0);
        if (Rc < 1 || Rc > R) return fail("rows per CTA", M, N, K, sms);
        covered = r1;
        if (NS == CPT || RT != 4) {
            // ring steps: thread t copies piece t % R4 of part t / R4 (t < P * R4)
            // at every step k into slot k % NS; every (step, part, piece) exactly
            // once, in bounds
            const int R4 = (Rc + 3) >> 2;
            if ((int64_t)P * R4 > nthr) return fail("more pieces than threads", M, N, K, sms);
            std::vector<uint8_t> got((size_t)CPT * P * R4, 0);
            for (int tid = 0; tid < P * R4; ++tid) {
                const int fpart = tid / R4, fpi = tid % R4;
                for (int k = 0; k < CPT; ++k) {
                    const int c = fpart * CPT + k;
                    if (c >= (int)Kc) continue;
                    got[((size_t)k * P + fpart) * R4 + fpi]++;
                    const int64_t r = r0 + 4 * fpi;
                    const int nr = Rc - 4 * fpi < 4 ? Rc - 4 * fpi : 4;
                    if (((r & 127) + nr - 1) > 127) return fail("piece crosses a tile", M, N, K, sms);
                    for (int j = 0; j < 5; ++j) {
                        const int64_t src = ((r >> 7) * Kc + c) * 640 + sherry_word_pos(j, (int)(r & 127));
                        if (src < 0 || src + nr > native_words) return fail("prefetch source", M, N, K, sms);
                        const int64_t dst = (int64_t)(k % NS) * P * 5 * R + (int64_t)(fpart * 5 + j) * R + 4 * fpi;
                        if (dst < 0 || dst + nr > (int64_t)NS * P * 5 * R) return fail("prefetch destination", M, N, K, sms);
                    }
                }
            }
            for (int k = 0; k < CPT; ++k)
                for (int pp = 0; pp < P; ++pp)
                    for (int pi = 0; pi < R4; ++pi)
                        if (got[((size_t)k * P + pp) * R4 + pi] != (pp * CPT + k < (int)Kc ? 1 : 0))
                            return fail("step pieces not copied exactly once", M, N, K, sms);
        } else {
            // streaming ring of 4 rows per thread: thread (qi, part) copies its
            // own rows of every step (row0 = qi * RT, ragged last group in 4-byte words); every
            // (step, part, row) exactly once, in bounds, RT-word aligned
            std::vector<uint8_t> got((size_t)CPT * P * Rc, 0);
            for (int tid = 0; tid < nthr; ++tid) {
                const int qi = tid % Q, part = tid / Q;
                if (part >= P || qi * RT >= Rc) continue;
                const int row0 = qi * RT, nr = Rc - row0 < RT ? Rc - row0 : RT;
                const int64_t r = r0 + row0;
                if (((r & 127) + nr - 1) > 127) return fail("own rows cross a tile", M, N, K, sms);
                for (int k = 0; k < CPT; ++k) {
                    const int c = part * CPT + k;
                    if (c >= (int)Kc) continue;
                    for (int e = 0; e < nr; ++e) got[((size_t)k * P + part) * Rc + row0 + e]++;
                    for (int j = 0; j < 5; ++j) {
                        const int64_t src = ((r >> 7) * Kc + c) * 640 + sherry_word_pos(j, (int)(r & 127));
                        if (src < 0 || src + nr > native_words) return fail("own copy source", M, N, K, sms);
                        const int64_t dst = (int64_t)(k % NS) * P * 5 * R + (int64_t)(part * 5 + j) * R + row0;
                        if (dst < 0 || dst + nr > (int64_t)NS * P * 5 * R) return fail("own copy destination", M, N, K, sms);
                        if (nr == RT && (src % RT || dst % RT)) return fail("own copy alignment", M, N, K, sms);
                        for (int e = 1; e < nr; ++e)
                            if (((r >> 7) * Kc + c) * 640 + sherry_word_pos(j, (int)((r + e) & 127)) != src + e)
                                return fail("own rows not consecutive", M, N, K, sms);
                    }
                }
            }
            for (int k = 0; k < CPT; ++k)
                for (int pp = 0; pp < P; ++pp)
                    for (int rr = 0; rr < Rc; ++rr)
                        if (got[((size_t)k * P + pp) * Rc + rr] != (pp * CPT + k < (int)Kc ? 1 : 0))
                            return fail("step rows not copied exactly once", M, N, K, sms);
        }
        // main loop and partial sums
        std::vector<uint8_t> walk((size_t)Rc * Kc, 0);
        for (int tid = 0; tid < nthr; ++tid) {
            const int qi = tid % Q, part = tid / Q;
            if (part >= P) continue;
            for (int r = 0; r < RT; ++r) {
                const int64_t red = (int64_t)(part * Mi + (Mi - 1)) * R + qi * RT + r;
                if (red >= (int64_t)P * Mi * R) return fail("partial sums index", M, N, K, sms);
            }
            if (qi * RT >= Rc) continue;
            if (part * CPT >= (int)Kc) return fail("empty K part", M, N, K, sms);
            for (int k = 0; k < CPT; ++k) {
                const int c = part * CPT + k;
                if (c >= (int)Kc) continue;
                for (int j = 0; j < 5; ++j) {
                    const int64_t w = (int64_t)(k % NS) * P * 5 * R + (int64_t)(part * 5 + j) * R + qi * RT;
                    if (w + RT > (int64_t)NS * P * 5 * R) return fail("code load", M, N, K, sms);
                }
                const int64_t a = (int64_t)(Mi - 1) * QK + (int64_t)c * S + 16 * 7 + 16;
                if (a > (int64_t)Mi * QK) return fail("activation load", M, N, K, sms);
                for (int r = 0; r < RT; ++r)
                    if (qi * RT + r < Rc) walk[(size_t)(qi * RT + r) * Kc + c]++;
            }
        }
        for (uint8_t v : walk)
            if (v != 1) return fail("(row, chunk) not walked exactly once", M, N, K, sms);
    }
    if (covered != N) return fail("rows not covered", M, N, K, sms);
    // activation stores: fused words and int8 16-byte copies, and the tail
    const int64_t K4 = K / 4, K16 = K / 16;
    if ((int64_t)(Mi - 1) * QK + ((K4 - 1) >> 5) * S + 4 * ((K4 - 1) & 31) + 4 > (int64_t)Mi * QK)
        return fail("fused activation store", M, N, K, sms);
    if ((int64_t)(Mi - 1) * QK + ((K16 - 1) >> 3) * S + 16 * ((K16 - 1) & 7) + 16 > (int64_t)Mi * QK)
        return fail("activation copy", M, N, K, sms);
    const int used = (int)(K - (Kc - 1) * 128);
    if (used <= 0 || used > 128 || (128 - used) % 32) return fail("tail", M, N, K, sms);
    return 0;
}

int main()
{
    const int64_t Ns[] = {1, 3, 4, 5, 37, 77, 128, 129, 200, 257, 300, 333, 388, 512, 640, 777, 1000, 1024,
                          2000, 4096, 4100, 5120, 6400, 8192, 14336, 19072, 28672, 65536};
    const int64_t Ks[] = {32, 96, 128, 160, 224, 256, 512, 640, 1024, 1184, 2048, 4096, 8192, 9216, 14336, 16384};
    const int64_t Ms[] = {1, 2, 3, 4, 5, 7, 8};
    const int sm_list[] = {148, 132, 1, 7};
    int64_t n = 0;
    for (int sms : sm_list)
        for (int64_t M : Ms)
            for (int64_t N : Ns)
                for (int64_t K : Ks) {
                    if (check(M, N, K, sms)) return 1;
                    ++n;
                }
    std::printf("ok %lld shapes\n", (long long)n);
    return 0;
}
