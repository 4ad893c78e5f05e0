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
//     over the full K: no split-K, no cross-CTA reduction, no atomics in
//     global memory, no workspace, no clusters.
//   * Before griddepcontrol.wait the CTA streams its rows' codes (the rotated
//     word planes of the native layout) into shared memory with 16-byte
//     cp.async copies.  Weights never depend
//     on the previous kernel, so their fetch overlaps its decode.  The CTA
//     lets the next kernel start only once its own activations are in
//     shared memory, so that the next kernel's weight stream does not queue
//     in front of those latency-critical reads.  The CTA is small enough in
//     shared memory, threads and registers for the next layer's CTA to be
//     resident at the same time and do the same.
//   * After the wait every CTA reads the activations of its tokens (all of
//     K), takes the absmax, quantises into shared memory.
//   * Thread (row group i, K-part p) owns RT consecutive rows and walks the
//     chunks of its part.  Per group: one 32-entry table load turns the
//     5-bit code into int8x4 {-1,0,+1}, one dp4a per token adds it.  The
//     shared-memory pipe is the limit of that loop (measured on B200: one
//     conflict-free 32-bit lookup per clock per SM, a broadcast 128-bit
//     activation load about 2.6 clocks): one 16-byte activation load serves
//     all RT rows of a thread, so the table lookups are most of the pipe's
//     work.  Consecutive lanes own consecutive row groups, so their code
//     loads are consecutive 4*RT-byte pieces and their activation loads are
//     broadcasts.  Activation chunks sit S >= 128 bytes apart, S chosen on
//     the host so that the few K-parts that share a warp read different
//     banks.
//   * The K-parts of a row are summed in shared memory and the epilogue writes
//     y (and acc) with coalesced stores.
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
constexpr int kSmemBudgetMax = 200 * 1024;  // one CTA per SM: shapes whose activations alone need more
constexpr int kXV = 7;                      // fused: float4 activations per thread held in registers (K <= 14336 at 512 threads)

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
    int Q;                       // row groups of RT rows: R / RT
    int P;                       // K-parts per row
    int CPT;                     // chunks per K-part: the loop steps; step k covers chunk p * CPT + k of part p
    int NS;                      // ring slots of code steps held in shared memory (NS >= CPT: all of them)
    int S;                       // bytes between consecutive K chunks of the int8 activation buffer
};

// Shared memory: table | scales | warp maxima (two token slots) | partial sums [P][M][R] |
// alpha [R] | code ring [NS][P][5][R] words | activations [M][Kc][S] int8.
constexpr int kOffTable = 0;                              // 32 x u32, 128-byte aligned inside 256 bytes
constexpr int kOffScale = 256;                            // [kMaxM] f32 s
constexpr int kOffWarpMax = kOffScale + kMaxM * 4;        // [2][16 warps] f32
constexpr int kOffRed = kOffWarpMax + 2 * 16 * 4;
static_assert(kMaxThreads / 32 <= 16, "warp-maximum slots");
static_assert(kOffRed % 16 == 0, "alignment");
__host__ __device__ inline int off_alpha(int M, int P, int R) { return (kOffRed + P * M * R * 4 + 15) & ~15; }
__host__ __device__ inline int off_codes(int M, int P, int R) { return (off_alpha(M, P, R) + R * 4 + 15) & ~15; }
__host__ __device__ inline int off_q(int M, int P, int R, int NS)
{
    return (off_codes(M, P, R) + NS * P * SHERRY_CHUNK_WORDS * R * 4 + 15) & ~15;
}
__host__ __device__ inline int smem_bytes(int M, int P, int R, int NS, int64_t Kc, int S)
{
    return off_q(M, P, R, NS) + M * (int)Kc * S;
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
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
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

// The same loads, kept in program order with this thread's copies into the
// ring (volatile: a refill of the slot is never issued ahead of them).
template <int N>
__device__ __forceinline__ void lds_vec_ordered(uint32_t addr, uint32_t (&v)[N]);
template <>
__device__ __forceinline__ void lds_vec_ordered<1>(uint32_t addr, uint32_t (&v)[1])
{
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v[0]) : "r"(addr));
}
template <>
__device__ __forceinline__ void lds_vec_ordered<2>(uint32_t addr, uint32_t (&v)[2])
{
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v[0]), "=r"(v[1]) : "r"(addr));
}
template <>
__device__ __forceinline__ void lds_vec_ordered<4>(uint32_t addr, uint32_t (&v)[4])
{
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]) : "r"(addr));
}

// Byte offset, in the table, of group g's code within a row's five chunk
// words w[0..4] (w[5] = 0): (bits [5g, 5g+5)) * 4.  g is a compile-time
// constant after unrolling, so this is one shift or funnel shift.
template <int G>
__device__ __forceinline__ uint32_t code_x4(const uint32_t (&w)[SHERRY_CHUNK_WORDS + 1])
{
    constexpr int bit = 5 * G, wi = bit >> 5, off = bit & 31;
    uint32_t v;
    if constexpr (off == 0) v = w[wi] << 2;
    else if constexpr (off == 1) v = w[wi] << 1;
    else if constexpr (off <= 27) v = w[wi] >> (off - 2);
    else v = __funnelshift_r(w[wi], w[wi + 1], off - 2);
    return v & 0x7Cu;
}

// The decode table: in a static shared array (ST: a lookup is one load at
// code * 4 plus the array's constant offset) or at a 128-byte aligned
// address of the dynamic window (a lookup address is (code * 4) | table).
// Which one measures faster depends on the instantiation (the one-row
// fused loop keeps the dynamic form).
struct TableRef {
    uint32_t addr;              // dynamic form: shared address
    const uint32_t* ptr;        // static form
};
template <bool ST>
__device__ __forceinline__ uint32_t table_at(const TableRef& t, uint32_t code_x4)
{
    if constexpr (ST) return *reinterpret_cast<const uint32_t*>(reinterpret_cast<const char*>(t.ptr) + code_x4);
    else return ptx::lds_u32_nv(code_x4 | t.addr);
}

// The 4 groups of piece G4 (groups 4 G4 .. 4 G4 + 3) of RT rows: table entries.
template <int G4, int RT, bool ST>
__device__ __forceinline__ void lookup_piece(const uint32_t (&w)[RT][SHERRY_CHUNK_WORDS + 1], const TableRef& tab,
                                             uint32_t (&e)[RT][4])
{
#pragma unroll
    for (int r = 0; r < RT; ++r) {
        e[r][0] = table_at<ST>(tab, code_x4<4 * G4 + 0>(w[r]));
        e[r][1] = table_at<ST>(tab, code_x4<4 * G4 + 1>(w[r]));
        e[r][2] = table_at<ST>(tab, code_x4<4 * G4 + 2>(w[r]));
        e[r][3] = table_at<ST>(tab, code_x4<4 * G4 + 3>(w[r]));
    }
}

template <int G4, int MT, int RT, bool ST>
__device__ __forceinline__ void piece(const uint32_t (&w)[RT][SHERRY_CHUNK_WORDS + 1], const TableRef& tab,
                                      uint32_t qc, int QK, int M, int32_t (&acc)[RT][MT])
{
    uint32_t e[RT][4];
    lookup_piece<G4, RT, ST>(w, tab, e);
#pragma unroll
    for (int m = 0; m < MT; ++m) {
        if (m >= M) break;
        uint32_t qv[4];
        lds_vec<4>(qc + (uint32_t)(m * QK + 16 * G4), qv);
#pragma unroll
        for (int r = 0; r < RT; ++r) {
            int32_t a = acc[r][m];
            a = __dp4a((int)e[r][0], (int)qv[0], a);
            a = __dp4a((int)e[r][1], (int)qv[1], a);
            a = __dp4a((int)e[r][2], (int)qv[2], a);
            a = __dp4a((int)e[r][3], (int)qv[3], a);
            acc[r][m] = a;
        }
    }
}

inline int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
inline int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }
inline int min_i(int a, int b) { return a < b ? a : b; }

// Work split of the decode kernel: G CTAs of at most R rows, row groups of
// RT rows (Q = R / RT of them), P K-parts of CPT chunks per row, Q * P <=
// kMaxThreads.  RT is the largest that the token count's registers allow and
// that still gives the CTA at least kMinBusyThreads working threads.  The
// codes live in a ring of NS loop steps (step k holds chunk p * CPT + k of
// every part p for all R rows): when every step fits (NS = CPT), all of a
// CTA's codes are fetched before the dependency wait, overlapping the
// previous kernel; otherwise the CTA streams them, fetching step k + NS while
// it decodes step k, and the grid takes two CTAs per SM so that the decode
// runs with twice the warps.
struct Plan {
    int G, R, RT, Q, P, CPT, NS, threads, smem, S;
};

constexpr int kMinBusyThreads = 320;
constexpr int kMaxRing = 4;                 // ring slots when the codes stream

// Rows per thread that the registers allow for MT tokens: RT x MT
// accumulators plus RT x 5 code words and RT x 4 table entries live at once.
inline int rt_max(int64_t M) { return M <= 2 ? 4 : 2; }
// Rows per thread tried first: one token takes one row per thread (its loop
// keeps a whole chunk's table loads in flight; measured faster live than
// several rows per thread) unless its codes stream.
inline int rt_first(int64_t M) { return M == 1 ? 1 : rt_max(M); }

// Bytes between K chunks of the int8 activation buffer: 128 + 16 sigma.  The
// K-parts that share a warp read their chunks at the same loop step; their
// 16-byte pieces sit sigma * 4 * dc banks apart (dc: chunk distance), so
// sigma is chosen to keep the pieces of a warp in different banks.
inline int act_stride(int Q, int P, int CPT, int threads)
{
    int best = 0, best_bad = 1 << 30;
    for (int sigma = 0; sigma < 8; ++sigma) {
        const int S = 128 + 16 * sigma;
        int bad = 0;
        for (int w0 = 0; w0 < threads; w0 += 32) {
            const int pa = w0 / Q, pb = min_i(P - 1, (w0 + 31) / Q);
            for (int p1 = pa; p1 <= pb; ++p1)
                for (int p2 = p1 + 1; p2 <= pb; ++p2) {
                    const int banks = (int)(((int64_t)(p2 - p1) * CPT * S / 4) % 32);
                    if (banks < 4 || banks > 28) ++bad;
                }
        }
        if (bad < best_bad) {
            best_bad = bad;
            best = S;
        }
        if (bad == 0) break;
    }
    return best;
}

// Row groups and K-parts for CTAs of R rows.
inline bool split_rows(int64_t R, int64_t Kc, int rtmax, int64_t* RT, int64_t* Q, int64_t* P, int64_t* CPT)
{
    for (*RT = rtmax;; *RT /= 2) {
        *Q = R / *RT;
        if (*Q > kMaxThreads) return false;
        *P = max64(1, min64(Kc, kMaxThreads / *Q));
        *CPT = (Kc + *P - 1) / *P;
        *P = (Kc + *CPT - 1) / *CPT;
        if (*Q * *P >= kMinBusyThreads || *RT == 1 || R / (*RT / 2) > kMaxThreads) return true;
    }
}

// The plan for G CTAs within `budget` bytes of shared memory each; false
// when it does not fit (ring of at least two steps, or every step).
inline bool plan_for(int64_t N, int64_t Kc, int64_t M, int64_t G, int budget, int rtmax, Plan* out)
{
    const int64_t R = ((N + G - 1) / G + 3 + 3) & ~int64_t(3);     // rows of a CTA at most, a multiple of 4
    if (R > (int64_t)rtmax * kMaxThreads || G > 0x7fffffff) return false;
    int64_t RT, Q, P, CPT;
    if (!split_rows(R, Kc, rtmax, &RT, &Q, &P, &CPT)) return false;
    for (int shrink = 0; shrink < 4; ++shrink) {
        int S = act_stride((int)Q, (int)P, (int)CPT, (int)(Q * P));
        for (int pass = 0; pass < 2; ++pass) {
            // every step held when it fits, else the deepest ring of up to kMaxRing slots
            int NS = (int)min64(CPT, kMaxRing);
            const int64_t all = smem_bytes((int)M, (int)P, (int)R, (int)CPT, Kc, S);
            if (all <= budget) NS = (int)CPT;
            else
                while (NS >= 2 && smem_bytes((int)M, (int)P, (int)R, NS, Kc, S) > budget) --NS;
            if ((NS >= 2 || NS == CPT) && smem_bytes((int)M, (int)P, (int)R, NS, Kc, S) <= budget) {
                out->G = (int)G;
                out->R = (int)R;
                out->RT = (int)RT;
                out->Q = (int)Q;
                out->P = (int)P;
                out->CPT = (int)CPT;
                out->NS = NS;
                out->threads = (int)max64(32, (Q * P + 31) / 32 * 32);
                out->smem = smem_bytes((int)M, (int)P, (int)R, NS, Kc, S);
                out->S = S;
                return true;
            }
            if (S == SHERRY_KCHUNK) break;
            S = SHERRY_KCHUNK;                                     // plain 128-byte activation chunks
        }
        if (P == 1) break;
        CPT *= 2;                                                  // fewer K-parts: fewer partial sums
        P = (Kc + CPT - 1) / CPT;
    }
    return false;
}

inline bool plan_rt(int64_t N, int64_t Kc, int64_t M, int sms, int budget, int rtmax, Plan* out)
{
    // at least 4 rows per CTA: row boundaries rounded to 4 rows then leave no CTA empty
    const int64_t gmax = max64(1, N / 4);
    const int64_t cap = (int64_t)rtmax * kMaxThreads - 8;           // rows per CTA: at most ceil(N / G) + 6
    int64_t G = min64(gmax, max64(sms, (N + cap - 1) / cap));
    for (int iter = 0; iter < 64; ++iter) {
        if (plan_for(N, Kc, M, G, budget, rtmax, out)) {
            // codes that stream: two CTAs per SM (half the rows each) decode with twice the warps
            Plan two;
            if (out->NS < out->CPT && G == sms && 2 * G <= gmax && plan_for(N, Kc, M, 2 * G, budget, rtmax, &two))
                *out = two;
            return true;
        }
        if (G >= gmax) return false;
        G = min64(gmax, 2 * G);                                       // about half the rows per CTA
    }
    return false;
}

// One row per thread for one token when its codes stay resident; several rows
// per thread otherwise (and whenever the first choice finds no plan).
inline bool plan_within(int64_t N, int64_t Kc, int64_t M, int sms, int budget, Plan* out)
{
    if (rt_first(M) != rt_max(M) && plan_rt(N, Kc, M, sms, budget, rt_first(M), out) && out->NS == out->CPT)
        return true;
    return plan_rt(N, Kc, M, sms, budget, rt_max(M), out);
}

// The plan of a launch: within kSmemBudget (two CTAs per SM, so the next
// layer's CTA can start its weight fetch beside this one) when possible, else
// within kSmemBudgetMax (one CTA per SM).
inline bool plan(int64_t N, int64_t Kc, int64_t M, int sms, Plan* out)
{
    return plan_within(N, Kc, M, sms, kSmemBudget, out) || plan_within(N, Kc, M, sms, kSmemBudgetMax, out);
}

// This thread's copies of one ring step: the 16-byte pieces (4 rows of one
// word plane) of the 4-row piece pi of part p's chunk at that step.  Row groups
// start at multiples of 4 rows, so 4 consecutive rows of one plane are 16
// aligned bytes in the native layout (4-byte copies for a ragged last piece).
__device__ __forceinline__ void fetch_piece(const Params& p, int64_t r0, int Rc, int pi, int part, int step,
                                            uint32_t slot_s)
{
    const int c = part * p.CPT + step;
    if (pi < 0 || c >= (int)p.Kc) return;
    const int64_t r = r0 + 4 * pi;
    const int nr = min(4, Rc - 4 * pi);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(p.wnative) +
                          ((r >> 7) * p.Kc + c) * (SHERRY_CHUNK_WORDS * SHERRY_TILE_ROWS);
    const int rr = (int)(r & 127);
    const uint32_t dst = slot_s + 4u * (uint32_t)(part * SHERRY_CHUNK_WORDS * p.R + 4 * pi);
    if (nr == 4) {
#pragma unroll
        for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j)
            cp_async16(dst + 4u * (uint32_t)(j * p.R), src + sherry_word_pos(j, rr));
    } else {
        for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j)
            for (int e = 0; e < nr; ++e) cp_async4(dst + 4u * (uint32_t)(j * p.R + e), src + sherry_word_pos(j, rr) + e);
    }
}

// Streaming rings: the code words a thread decodes at one step (rows row0 ..
// row0 + RT - 1 of the CTA, part `part`'s chunk at that step, five planes),
// copied by that thread itself, so that waiting for its own copy groups is
// all the synchronisation the ring needs.  row0 is a multiple of RT and the
// CTA's first row a multiple of 4, so the RT words of a plane are 4 RT
// aligned bytes in the native layout (4-byte copies for a ragged last group).
template <int RT>
__device__ __forceinline__ void fetch_own(const Params& p, int64_t r0, int Rc, int row0, int part, int step,
                                          uint32_t slot_s)
{
    const int c = part * p.CPT + step;
    if (row0 >= Rc || c >= (int)p.Kc) return;
    const int64_t r = r0 + row0;
    const int nr = min(RT, Rc - row0);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(p.wnative) +
                          ((r >> 7) * p.Kc + c) * (SHERRY_CHUNK_WORDS * SHERRY_TILE_ROWS);
    const int rr = (int)(r & 127);
    const uint32_t dst = slot_s + 4u * (uint32_t)(part * SHERRY_CHUNK_WORDS * p.R + row0);
    if (nr == RT) {
#pragma unroll
        for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j) {
            if constexpr (RT == 4) cp_async16(dst + 4u * (uint32_t)(j * p.R), src + sherry_word_pos(j, rr));
            else if constexpr (RT == 2) cp_async8(dst + 4u * (uint32_t)(j * p.R), src + sherry_word_pos(j, rr));
            else cp_async4(dst + 4u * (uint32_t)(j * p.R), src + sherry_word_pos(j, rr));
        }
    } else {
        for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j)
            for (int e = 0; e < nr; ++e) cp_async4(dst + 4u * (uint32_t)(j * p.R + e), src + sherry_word_pos(j, rr) + e);
    }
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Waits until at most n of this thread's committed copy groups are pending (n <= 3).
__device__ __forceinline__ void cp_async_wait_pending(int n)
{
    if (n <= 0) asm volatile("cp.async.wait_group 0;" ::: "memory");
    else if (n == 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
    else if (n == 2) asm volatile("cp.async.wait_group 2;" ::: "memory");
    else asm volatile("cp.async.wait_group 3;" ::: "memory");
}

// The fused activation phase: per token, absmax over the row, s = a / 127 and
// int8 codes into the shared activation buffer (qbuf: token m's K chunk c at
// byte m * QK + c * S), scales into scale_s.  XV float4 slots per thread hold
// the row in registers (all loads in flight at once); XV = 0 streams it from
// global memory twice.  Whether the row is in registers is a compile-time
// property of each instantiation.
template <int XV>
__device__ __forceinline__ void fused_activations(const Params& p, int8_t* qbuf, int QK, int S, float* scale_s,
                                                  float* warp_max, int M, int K4)
{
    const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = (nthr + 31) >> 5;
    constexpr bool in_regs = XV > 0;
    constexpr int NV = XV > 0 ? XV : 1;
    for (int m = 0; m < M; ++m) {
        const float4* xr = reinterpret_cast<const float4*>(p.x + (int64_t)m * p.K);
        int8_t* qr = qbuf + m * QK;
        float4 v[NV];
        float mx = 0.0f;
        // slots this thread holds (words tid, tid + nthr, ...); the same for
        // every lane of a warp except in a row's last, partial warp, so the
        // slots past the row are branched over rather than issued
        const int nsl = tid < K4 ? (K4 - 1 - tid) / nthr + 1 : 0;
        if constexpr (in_regs) {
            // all loads in flight at once
#pragma unroll
            for (int u = 0; u < XV; ++u)
                if (u < nsl) v[u] = xr[tid + u * nthr];
#pragma unroll
            for (int u = 0; u < XV; ++u)
                if (u < nsl) mx = fmaxf(mx, quant::absmax4(v[u]));
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
        // word idx (activations 4 idx .. 4 idx + 3) sits in chunk idx / 32
        if constexpr (in_regs) {
#pragma unroll
            for (int u = 0; u < XV; ++u) {
                const int idx = tid + u * nthr;
                if (u < nsl) {
                    const uint32_t w = quant::quantise4(v[u], sc);
                    *reinterpret_cast<uint32_t*>(qr + (idx >> 5) * S + 4 * (idx & 31)) = w;
                    if (qo) qo[idx] = w;
                }
            }
        } else {
            for (int i = tid; i < K4; i += nthr) {
                const uint32_t w = quant::quantise4(xr[i], sc);
                *reinterpret_cast<uint32_t*>(qr + (i >> 5) * S + 4 * (i & 31)) = w;
                if (qo) qo[i] = w;
            }
        }
    }
}

template <int MT, bool FUSED, int RT>
__global__ void __launch_bounds__(kMaxThreads, 2)
    sherry_decode_kernel(const Params p)
{
    static_assert(RT == 1 || RT == 2 || RT == 4, "rows per thread");
    static_assert(kMaxRing <= 4, "cp_async_wait_pending covers up to 3 pending groups");
    extern __shared__ __align__(16) uint8_t smem[];
    const int M = (int)p.M;
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int64_t r0 = row_begin(p.N, blockIdx.x, p.G), r1 = row_begin(p.N, blockIdx.x + 1, p.G);
    const int Rc = (int)(r1 - r0);
    const int R = p.R, P = p.P, S = p.S, NS = p.NS, CPT = p.CPT;
    const uint32_t s_base = ptx::smem_u32(smem);
    const uint32_t codes_s = s_base + off_codes(M, P, R);
    const uint32_t slot_bytes = 4u * (uint32_t)(P * SHERRY_CHUNK_WORDS * R);
    const int qoff = off_q(M, P, R, NS);
    int8_t* qbuf = reinterpret_cast<int8_t*>(smem + qoff);
    const int QK = (int)p.Kc * S;                          // bytes per token row of qbuf

    // ---- before the wait: the first ring steps of this CTA's codes, alpha, the table ----
    // Thread (qi, part) decodes rows qi * RT .. qi * RT + RT - 1 of K part `part`.
    // Resident rings (every step fits): thread t copies piece pi = t % R4 of
    // part t / R4 at every step (P * R4 <= threads: at most one piece per
    // thread and step), consecutive lanes reading consecutive positions of a
    // plane, and one barrier publishes them.  Streaming rings of 4 rows per
    // thread: every thread copies what it decodes (fetch_own, one 16-byte copy
    // per plane), so steps need no barrier; with 1 or 2 rows per thread the
    // pieces are copied as for resident rings and two barriers a step publish
    // and release them (smaller own copies measured slower there).
    const bool streaming = NS < CPT;
    const bool own = streaming && RT == 4;
    const int qi = tid % p.Q, part = tid / p.Q;
    const bool busy = part < P && qi * RT < Rc;
    const int R4 = (Rc + 3) >> 2;
    const int fpi = (R4 > 0 && tid < P * R4) ? tid % R4 : -1;
    const int fpart = R4 > 0 ? tid / R4 : 0;
    const int first = CPT < NS ? CPT : NS;                 // steps fetched before the wait
    {
        const uint32_t alpha_s = s_base + off_alpha(M, P, R);
        for (int ii = tid; ii < Rc; ii += nthr) cp_async4(alpha_s + 4u * (uint32_t)ii, p.alpha + r0 + ii);
    }
    for (int k = 0; k < first; ++k) {
        if (!own) fetch_piece(p, r0, Rc, fpi, fpart, k, codes_s + (uint32_t)k * slot_bytes);
        else if (busy) fetch_own<RT>(p, r0, Rc, qi * RT, part, k, codes_s + (uint32_t)k * slot_bytes);
        cp_async_commit();
    }
    // the decode table (see TableRef): static for every instantiation but the
    // fused one-row one, which measured faster with the dynamic form
    constexpr bool kStaticTable = !(FUSED && RT == 1);
    __shared__ __align__(128) uint32_t s_table[32];
    TableRef tab;
    tab.addr = (s_base + kOffTable + 127u) & ~127u;
    tab.ptr = s_table;
    if (tid < 32) {
        if constexpr (kStaticTable) s_table[tid] = expand_code((uint32_t)tid);
        else ptx::sts_u32(tab.addr + 4u * (uint32_t)tid, expand_code((uint32_t)tid));
    }
    ptx::pdl_wait();

    // ---- activations -------------------------------------------------------------
    // qbuf holds token m's K chunk c at byte m * QK + c * S.
    float* scale_s = reinterpret_cast<float*>(smem + kOffScale);
    const int K4 = (int)(p.K >> 2);
    if constexpr (FUSED) {
        // rows of up to kXV float4s per thread are held in registers; longer
        // rows stream from global memory (XV = 0)
        float* warp_max = reinterpret_cast<float*>(smem + kOffWarpMax);
        if (K4 <= kXV * nthr) fused_activations<kXV>(p, qbuf, QK, S, scale_s, warp_max, M, K4);
        else fused_activations<0>(p, qbuf, QK, S, scale_s, warp_max, M, K4);
    } else {
        // plain 16-byte loads, so that the copy groups in flight are the code steps only
        const int K16 = (int)(p.K >> 4);
        for (int m = 0; m < M; ++m)
            for (int i = tid; i < K16; i += nthr) {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.xq + (int64_t)m * p.K) + i);
                *reinterpret_cast<uint4*>(qbuf + m * QK + (i >> 3) * S + 16 * (i & 7)) = v;
            }
        if (tid < M) scale_s[tid] = p.x_scale[tid];
    }
    // zero the activation tail of the last chunk: its padding codes decode to nonzero weights
    {
        const int used = (int)(p.K - (p.Kc - 1) * SHERRY_KCHUNK);      // bytes of the last chunk in K
        const int tail = SHERRY_KCHUNK - used;                          // multiple of 32
        for (int i = tid; i < M * tail; i += nthr) {
            const int m = i / tail;
            qbuf[m * QK + (int)(p.Kc - 1) * S + used + (i - m * tail)] = 0;
        }
    }
    // every step in the ring (the codes did not stream): all copies landed
    if (!streaming) cp_async_wait_all();
    __syncthreads();
    // the next kernel may start now: its weight prefetch overlaps this decode
    // instead of queueing in front of this CTA's activation reads
    ptx::pdl_launch_dependents();

    // ---- decode + dp4a: RT rows per thread, one ring step at a time -----------------
    // Step k holds chunk part * CPT + k of every part.  When the codes stream,
    // each thread waits for its own copies of step k; with own copies it
    // decodes the step and refills the slot with its rows of step k + NS,
    // otherwise a barrier makes every thread's copies visible first and a
    // second one (the slot is no longer read) precedes the refill.
    int32_t acc[RT][MT];
#pragma unroll
    for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0;
    const uint32_t q_s = s_base + (uint32_t)qoff;
    if (RT == 1 && !streaming) {
        // One row per thread over the whole ring (every step resident): all 32
        // table loads of a chunk are issued before its dp4a run, and the next
        // chunk's code words are loaded during the current one.  With the few
        // warps a CTA has beside the next layer's prefetching CTA, this keeps
        // more loads in flight than walking the chunk piece by piece.
        const int nch = busy ? min(CPT, (int)p.Kc - part * CPT) : 0;
        if (nch > 0) {
            const uint32_t base = codes_s + 4u * (uint32_t)(part * SHERRY_CHUNK_WORDS * R + qi);
            int32_t a4[MT][4];
#pragma unroll
            for (int m = 0; m < MT; ++m) a4[m][0] = a4[m][1] = a4[m][2] = a4[m][3] = 0;
            uint32_t wn[SHERRY_CHUNK_WORDS];
#pragma unroll
            for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j) wn[j] = ptx::lds_u32_nv(base + 4u * (uint32_t)(j * R));
#pragma unroll 1
            for (int k = 0; k < nch; ++k) {
                uint32_t w[SHERRY_CHUNK_WORDS + 1];
#pragma unroll
                for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j) w[j] = wn[j];
                w[SHERRY_CHUNK_WORDS] = 0;
                if (k + 1 < nch) {
#pragma unroll
                    for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j)
                        wn[j] = ptx::lds_u32_nv(base + (uint32_t)(k + 1) * slot_bytes + 4u * (uint32_t)(j * R));
                }
                uint32_t e[32];
#pragma unroll
                for (int g = 0; g < 32; ++g) {
                    const int bit = 5 * g, wi = bit >> 5, off = bit & 31;
                    uint32_t v;
                    if (off == 0) v = w[wi] << 2;
                    else if (off == 1) v = w[wi] << 1;
                    else if (off <= 27) v = w[wi] >> (off - 2);
                    else v = __funnelshift_r(w[wi], w[wi + 1], off - 2);
                    e[g] = table_at<kStaticTable>(tab, v & 0x7Cu);
                }
                const uint32_t qc = q_s + (uint32_t)((part * CPT + k) * S);
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (m >= M) break;
#pragma unroll
                    for (int g4 = 0; g4 < 8; ++g4) {
                        uint32_t qv[4];
                        lds_vec<4>(qc + (uint32_t)(m * QK + 16 * g4), qv);
                        a4[m][0] = __dp4a((int)e[4 * g4 + 0], (int)qv[0], a4[m][0]);
                        a4[m][1] = __dp4a((int)e[4 * g4 + 1], (int)qv[1], a4[m][1]);
                        a4[m][2] = __dp4a((int)e[4 * g4 + 2], (int)qv[2], a4[m][2]);
                        a4[m][3] = __dp4a((int)e[4 * g4 + 3], (int)qv[3], a4[m][3]);
                    }
                }
            }
#pragma unroll
            for (int m = 0; m < MT; ++m) acc[0][m] = (a4[m][0] + a4[m][1]) + (a4[m][2] + a4[m][3]);
        }
    } else {
    int committed = first;
#pragma unroll 1
    for (int k = 0; k < CPT; ++k) {
        if (streaming) {
            cp_async_wait_pending(committed - (k + 1));
            if (!own) __syncthreads();
        }
        const int c = part * CPT + k;
        if (busy && c < (int)p.Kc) {
            // the five code words of each of the RT rows: one RT-word load per plane
            const uint32_t cbase = codes_s + (uint32_t)(k % NS) * slot_bytes +
                                   4u * (uint32_t)(part * SHERRY_CHUNK_WORDS * R + qi * RT);
            uint32_t w[RT][SHERRY_CHUNK_WORDS + 1];
#pragma unroll
            for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j) {
                uint32_t t[RT];
                lds_vec_ordered<RT>(cbase + 4u * (uint32_t)(j * R), t);
#pragma unroll
                for (int r = 0; r < RT; ++r) w[r][j] = t[r];
            }
#pragma unroll
            for (int r = 0; r < RT; ++r) w[r][SHERRY_CHUNK_WORDS] = 0;
            const uint32_t qc = q_s + (uint32_t)(c * S);
            piece<0, MT, RT, kStaticTable>(w, tab, qc, QK, M, acc);
            piece<1, MT, RT, kStaticTable>(w, tab, qc, QK, M, acc);
            piece<2, MT, RT, kStaticTable>(w, tab, qc, QK, M, acc);
            piece<3, MT, RT, kStaticTable>(w, tab, qc, QK, M, acc);
            piece<4, MT, RT, kStaticTable>(w, tab, qc, QK, M, acc);
            piece<5, MT, RT, kStaticTable>(w, tab, qc, QK, M, acc);
            piece<6, MT, RT, kStaticTable>(w, tab, qc, QK, M, acc);
            piece<7, MT, RT, kStaticTable>(w, tab, qc, QK, M, acc);
        }
        if (streaming && k + NS < CPT) {
            if (own) {
                if (busy) fetch_own<RT>(p, r0, Rc, qi * RT, part, k + NS, codes_s + (uint32_t)(k % NS) * slot_bytes);
            } else {
                __syncthreads();
                fetch_piece(p, r0, Rc, fpi, fpart, k + NS, codes_s + (uint32_t)(k % NS) * slot_bytes);
            }
            cp_async_commit();
            ++committed;
        }
    }

    }

    // ---- sum the K-parts of each row, epilogue ----------------------------------------
    int32_t* red = reinterpret_cast<int32_t*>(smem + kOffRed);      // [P][M][R]
    const float* alpha_sm = reinterpret_cast<const float*>(smem + off_alpha(M, P, R));
    if (part < P) {
#pragma unroll
        for (int m = 0; m < MT; ++m)
            if (m < M)
#pragma unroll
                for (int r = 0; r < RT; ++r) red[(part * M + m) * R + qi * RT + r] = acc[r][m];
    }
    __syncthreads();
    const int O = M * Rc;
    // output o = (token m, row i): one thread sums its P partials
    for (int idx = tid; idx < O; idx += nthr) {
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
