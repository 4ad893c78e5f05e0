// Sherry 3:4 ternary GEMM on the sm_100a tensor cores.
//
// What it computes (Sherry page, pnsm.cn/news/1195499, sec. 2.2 steps 2-4):
//   acc[m][n] = sum_k x_i8[m][k] * T[n][k]           (exact int32)
//   y[m][n]   = (float)((float)acc[m][n] * alpha[n]) * x_scale[m]
// with T decoded from the 5-bit group codes of sec. 2.1.
//
// How (the page's CPU/Jetson table-lookup kernels are prior art only): the
// problem is run "swap-AB" on tcgen05.mma.kind::i8 with M = 128 weight rows,
// N = BN tokens and K = 32 per instruction.
//   * A (weights) lives in tensor memory.  Decoder warps read the packed
//     codes of their row from shared memory, turn every 5-bit code into the
//     four int8 weights {-1,0,+1} of its group with one lookup in a 32-entry
//     table, and store them with tcgen05.st: one 32-bit TMEM cell is one
//     group, so a 128-wide K chunk of a row is 32 consecutive columns of that
//     row's lane.
//   * B (activations) is loaded by TMA into shared memory, K-major with the
//     128-byte swizzle, and described to the MMA by a shared-memory matrix
//     descriptor; rows past M and columns past K are zero-filled by TMA.
//   * D (int32 accumulators) lives in tensor memory; epilogue warps read it
//     with tcgen05.ld and apply the two fp32 products.
// Work is split so that every SM gets the same number of K chunks whatever
// the shape (one CTA per SM): each CTA first takes an even share of the
// units (token tile, row tile, K chunk) of the T mod G tiles left over, then
// T div G whole tiles of its own (SegWalk).  A tile whose K range spans
// several CTAs is summed exactly with int32 red.add into a workspace slot;
// the last contributor (an atomic counter) runs the epilogue and clears the
// slot and counter, so the workspace is all zero between calls.  The split
// tiles come first, so their reductions overlap the whole tiles after them.
//
// A pipeline stage carries SC consecutive K chunks of one tile (one bulk copy
// of SC * 2560 bytes of codes, SC 2D TMA boxes of activations, SC * 4 MMAs),
// so that the fixed cost of a stage's barriers is paid once per SC chunks.
//
// Warp roles (576 threads; 448 for 192-token tiles with two-chunk stages,
// which have two decoder groups):
//   warp 0       producer: per stage one bulk copy of the codes (completing
//                the stage's code barrier, which the decoders wait for) and
//                one 2D TMA of the activation tile per chunk (completing its
//                full barrier, which the MMA warp waits for); the codes of
//                the first ring round go out before the dependency wait, so
//                the decoders work while the previous kernel finishes
//   warp 1       TMEM allocation and MMA issue (an elected lane)
//   warps 2-13   three decoder groups of four warps (each group covers the
//                four TMEM lane quadrants), taking stages in turn
//   warps 14-17  epilogue (one warp per lane quadrant)
// Loop indices (stage, phase, tile coordinates) advance incrementally: no
// integer division on the per-chunk path.
// Every wait is bounded in wall time; when a bound runs out the kernel
// records a status code, stops issuing work, waits (bounded) for what it has
// in flight, frees its tensor memory and returns.
//
// The same kernel runs the W4A8 FastGEMM of the OdysseyLLM review page
// (xllm-io.github.io/paper-review/blog/odysseyllm, sec. 3.1-3.2, 5.2) when
// WF = kWeightInt4: the weights are per-channel SINT4 (8 KB per 128 x 128
// chunk instead of 2560 bytes of codes), the decoders turn each 4-bit two's
// complement value into the int8 16 w by moving it into the high half of a
// byte (shift and mask, no table), the MMAs sum q * 16 w exactly in int32,
// and the epilogue divides those sums by 16 (an exact arithmetic shift)
// before the two fp32 products with the channel scale and the token scale.
#pragma once

#include <cstdint>
#include <cuda.h>

#include "ptx.cuh"
#include "sherry_internal.h"

namespace sherry {
namespace tc {

constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kDecWarp0 = 2;
constexpr int kTmemCols = 512;
constexpr uint64_t kWaitLimitNs = 2000000000ull;              // 2 s per wait

// weight formats
constexpr int kWeightSherry = 0;     // 5-bit 3:4 ternary group codes
constexpr int kWeightInt4 = 1;       // SINT4, two per byte

template <int BN, int SC, int WF = kWeightSherry>
struct Cfg {
    static_assert(BN == 16 || BN == 32 || BN == 64 || BN == 128 || BN == 192, "BN");
    // 192-token tiles: two 192-column accumulators leave 128 TMEM columns:
    // four one-chunk A slots (SC = 1, three decoder groups, the form used)
    // or two two-chunk slots (SC = 2, then only two groups: the rings must be
    // at least as deep as the number of groups)
    static constexpr int kDecGroups = (BN == 192 && SC == 2) ? 2 : 3;
    static constexpr int kEpiWarp0 = kDecWarp0 + 4 * kDecGroups;
    static constexpr int kThreads = 32 * (kEpiWarp0 + 4);
    static_assert(SC >= 1 && SC <= 4, "SC");
    static_assert(WF == kWeightSherry || WF == kWeightInt4, "WF");
    // weight bytes of one (row tile, K chunk) block
    static constexpr int kChunkWBytes = WF == kWeightSherry ? SHERRY_CHUNK_BYTES_PER_TILE : SHERRY_W4_CHUNK_BYTES;
    // int32 sums of q * 16 w are divided by 16 before the epilogue uses them
    static constexpr int kAccShift = WF == kWeightInt4 ? 4 : 0;
    static constexpr int kBChunkBytes = BN * 128;
    static constexpr int kBStageBytes = SC * kBChunkBytes;
    static constexpr int kCodeStageBytes = SC * kChunkWBytes;
    static constexpr int kStageBytes = kBStageBytes + kCodeStageBytes;
    static constexpr int kStagesRaw = (192 * 1024) / kStageBytes;
    static constexpr int kStagesCap = kStagesRaw > 12 ? 12 : kStagesRaw;
    // A whole number of rounds of decoder groups: stage s is then always
    // decoded by group s mod kDecGroups (see the ring rules below).
    static constexpr int kStages = kStagesCap - kStagesCap % kDecGroups;
    static constexpr int kACols = 32 * SC;                          // TMEM columns of one A stage
    static constexpr int kDBufs = (2 * BN + 2 * kACols <= kTmemCols) ? 2 : 1;
    static constexpr int kAStagesRaw = (kTmemCols - kDBufs * BN) / kACols;
    static constexpr int kAStages = kAStagesRaw > 8 ? 8 : kAStagesRaw;
    // A decoder group takes every kDecGroups-th stage.  A parity wait is exact
    // only while the waiter is not a whole phase ahead of the barrier: a wait
    // for phase k on a barrier still in phase k-1 sees the parity of phase
    // k-2, complete, and returns at once.
    //  - code(s) (the stage's codes; the decoders wait for it): the copies of
    //    different stages may land in any order, so the group waiting for the
    //    fill of iteration i must itself have seen the fill of iteration
    //    i - kStages: kStages a multiple of kDecGroups makes it the same
    //    group.  It cannot be two phases behind either: the next refill of
    //    stage s needs this group's arrival on empty(s).
    //  - full(s) (the stage's activation boxes): waited for by the MMA warp
    //    alone, in stage order; its refill needs the MMA's commit on empty(s).
    //  - aempty(a): completed by tcgen05.commit of the one MMA thread, in
    //    issue order; a group that saw its previous slot freed has seen every
    //    earlier MMA complete, which covers slot a's previous use once the
    //    ring is at least kDecGroups deep.
    static_assert(kStages >= kDecGroups && kStages % kDecGroups == 0, "stage ring not whole rounds of decoder groups");
    static_assert(kAStages >= kDecGroups, "A ring shallower than decoder groups");
    static constexpr int kACol0 = kDBufs * BN;
    // shared memory: [B stages][code stages][barriers + misc]
    static constexpr int kOffCodes = kStages * kBStageBytes;
    static constexpr int kOffBars = kOffCodes + kStages * kCodeStageBytes;
    static constexpr int kNumBars = 3 * kStages + 2 * kAStages + 2 * kDBufs + 1;
    static constexpr int kOffMisc = kOffBars + 8 * kNumBars;
    static constexpr int kMiscBytes = 64 + 2 * BN * 4;   // tmem holder, flags, token scales [2][BN]
    // output staging for TMA stores: per epilogue warp two slices of
    // [kSlice tokens][32 rows] fp32
    static constexpr int kSlice = BN < 32 ? BN : 32;
    static constexpr int kOffStaging = (kOffMisc + kMiscBytes + 127) & ~127;
    static constexpr int kStagingBytes = 4 * 2 * kSlice * 32 * 4;
    static constexpr int kSmemBytes = kOffStaging + kStagingBytes + 1024;   // + alignment slack
    // dynamic plus static (the table of the code path, 1 KB as compiled)
    // within the 227 KB per-block limit
    static_assert(kSmemBytes + (WF == kWeightSherry ? 1024 : 0) <= 232448, "shared memory");
    // instruction descriptor: s32 accumulate, signed int8 A and B, both
    // K-major, N = BN, M = 128
    static constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                                       (uint32_t(128 >> 4) << 24);
};

struct Params {
    const uint8_t* wnative;     // kernel-native codes
    const float* alpha;         // [N]
    const float* x_scale;       // [M]
    float* y;                   // [M][N] or null
    int32_t* acc;               // [M][N] or null
    int32_t* ws;                // split-K slots [grid][BN][128]
    uint32_t* counters;         // [grid]
    unsigned* status;           // device status word
    int64_t M, N, K;
    int64_t TM, TN, Kc;         // token tiles, row tiles, K chunks
    int64_t U;                  // total units TM*TN*Kc
    int y_tma;                  // y rows 16-byte multiples: complete tiles leave through TMA stores
};

// The work of one CTA as a sequence of tile segments (a segment = chunks
// [cb, ce) of one tile; units are numbered tile-major, unit = tile * Kc +
// chunk).  With T tiles and G CTAs, the last R = T mod G tiles are split
// stream-K: their RU = R * Kc units are cut into G contiguous shares (each
// under one tile; when RU < G, one unit to each of the first RU CTAs, so
// that no share is empty), walked first.  Then every CTA walks F = T div G whole tiles of
// its own.  So every CTA gets the same number of units within one, the
// tiles summed across CTAs come first (their reductions overlap the later
// tiles), and every CTA ends on whole tiles.  All roles walk this sequence.
struct SegWalk {
    int64_t Kc, tile, cb, ce, end_u, r1_tile, r1_end_tile;
    int range;                                  // 0 split share, 1 own tiles, 2 done
    SHERRY_HD SegWalk(const Params& p, int64_t b, int64_t G)
    {
        Kc = p.Kc;
        const int64_t T = p.TM * p.TN;
        const int64_t F = T / G, R = T - F * G;
        const int64_t L0 = (T - R) * Kc, RU = R * Kc;
        r1_tile = b * F;
        r1_end_tile = (b + 1) * F;
        int64_t a0, a1;
        if (RU >= G) {
            a0 = L0 + RU * b / G;
            a1 = L0 + RU * (b + 1) / G;
        } else {
            a0 = L0 + b;
            a1 = a0 + (b < RU ? 1 : 0);
        }
        if (a0 < a1) {
            range = 0;
            end_u = a1;
            tile = a0 / Kc;
            cb = a0 - tile * Kc;
            const int64_t te = (tile + 1) * Kc;
            ce = (te < a1 ? te : a1) - tile * Kc;
        } else {
            start_own();
        }
    }
    SHERRY_HD void start_own()
    {
        if (r1_tile < r1_end_tile) {
            range = 1;
            tile = r1_tile;
            cb = 0;
            ce = Kc;
        } else {
            range = 2;
        }
    }
    SHERRY_HD bool done() const { return range == 2; }
    SHERRY_HD bool complete() const { return cb == 0 && ce == Kc; }
    SHERRY_HD void next()
    {
        if (range == 0) {
            const int64_t u = tile * Kc + ce;
            if (u < end_u) {
                ++tile;
                cb = 0;
                ce = (end_u - u) < Kc ? (end_u - u) : Kc;
            } else {
                start_own();
            }
        } else if (++tile >= r1_end_tile) {
            range = 2;
        }
    }
};

// First and last CTA of a split tile t (one of the last R tiles): the owners
// of its first and last unit among the G shares of the split units.
SHERRY_HD inline void split_owners(const Params& p, int64_t t, int64_t G, int64_t* bf, int64_t* bl)
{
    const int64_t T = p.TM * p.TN;
    const int64_t R = T - (T / G) * G;
    const int64_t RU = R * p.Kc;
    const int64_t u = (t - (T - R)) * p.Kc;
    if (RU >= G) {
        *bf = ((u + 1) * G - 1) / RU;
        *bl = ((u + p.Kc) * G - 1) / RU;
    } else {
        *bf = u;
        *bl = u + p.Kc - 1;
    }
}

__device__ __forceinline__ uint64_t b_desc_sw128(uint32_t smem_addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((smem_addr >> 4) & 0x3FFFu);          // start address
    d |= (uint64_t)1u << 16;                               // leading byte offset (unused, 16 B)
    d |= (uint64_t)(1024u >> 4) << 32;                     // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1u << 46;                               // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                               // 128-byte swizzle
    return d;
}

__device__ __forceinline__ void report(unsigned* status, volatile int* abort_flag, unsigned code)
{
    atomicCAS(status, 0u, code);
    *abort_flag = 1;
}

template <int BN, int SC, int WF = kWeightSherry>
__global__ void __launch_bounds__(Cfg<BN, SC, WF>::kThreads, 1)
    sherry_gemm_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap ymap,
                          const Params p)
{
    using C = Cfg<BN, SC, WF>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    __shared__ __align__(128) uint32_t table[32];
    // 1024-byte aligned start, computed by pointer arithmetic so that the
    // compiler keeps the shared address space (plain ld.shared/st.shared)
    uint8_t* smem = smem_raw + ((1024u - (ptx::smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t bar0 = sbase + C::kOffBars;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
    auto afull_bar = [&](int a) { return bar0 + 8u * (2 * C::kStages + a); };
    auto aempty_bar = [&](int a) { return bar0 + 8u * (2 * C::kStages + C::kAStages + a); };
    auto dfull_bar = [&](int d) { return bar0 + 8u * (2 * C::kStages + 2 * C::kAStages + d); };
    auto dempty_bar = [&](int d) { return bar0 + 8u * (2 * C::kStages + 2 * C::kAStages + C::kDBufs + d); };
    const uint32_t drain_bar = bar0 + 8u * (2 * C::kStages + 2 * C::kAStages + 2 * C::kDBufs);
    // a stage's codes land on code(s) (the decoders wait for it), its
    // activation boxes on full(s) (the MMA warp waits for it): the codes of
    // the first ring round are copied, and decoded, before the dependency wait
    auto code_bar = [&](int s) { return bar0 + 8u * (2 * C::kStages + 2 * C::kAStages + 2 * C::kDBufs + 1 + s); };
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
    volatile int* last_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 8);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const int64_t G = gridDim.x;

    if (WF == kWeightSherry && threadIdx.x < 32) {
        // code -> four int8 weights of the group, byte i = position i
        const uint32_t c = threadIdx.x, z = c & 3u;
        uint32_t word = 0, slot = 2;
        for (uint32_t i = 0; i < 4; ++i) {
            uint32_t b = 0;
            if (i != z) {
                b = ((c >> slot) & 1u) ? 0xFFu : 0x01u;
                ++slot;
            }
            word |= b << (8 * i);
        }
        table[c] = word;
    }
    if (threadIdx.x == 32) {
        for (int s = 0; s < C::kStages; ++s) {
            ptx::mbar_init(full_bar(s), 1);
            ptx::mbar_init(code_bar(s), 1);
            ptx::mbar_init(empty_bar(s), 4 + 1);
        }
        for (int a = 0; a < C::kAStages; ++a) {
            ptx::mbar_init(afull_bar(a), 4);
            ptx::mbar_init(aempty_bar(a), 1);
        }
        for (int d = 0; d < C::kDBufs; ++d) {
            ptx::mbar_init(dfull_bar(d), 1);
            ptx::mbar_init(dempty_bar(d), 4);
        }
        ptx::mbar_init(drain_bar, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    __syncwarp();
    if (warp == kMmaWarp) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_holder), kTmemCols);
        ptx::tmem_relinquish();
    }
    if (threadIdx.x == 0) ptx::prefetch_tensormap(&xmap);
    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // Programmatic dependent launch: everything above (barriers, tensor
    // memory, table) overlaps the end of the previous kernel on the stream.
    // The roles that touch global memory the previous kernel may write or
    // read (the producer: activations; the epilogue: scales, y, acc and the
    // split-K workspace) wait for it to complete; the decoders and the MMA
    // warp only use this CTA's shared and tensor memory.
    ptx::pdl_launch_dependents();

    if (warp == kProducerWarp) {
        // Converged warp, elected-lane issue and a non-blocking test of the
        // next slot, for the same reason as the MMA loop below: a copy issued
        // late delays every role after it.
        //
        // The codes do not depend on the previous kernel: the first ring
        // round's code copies are issued before the dependency wait, so that
        // they (and their decoding) overlap the end of the previous kernel;
        // their activation boxes follow after the wait.
        int64_t npre = 0;
        {
            SegWalk w(p, blockIdx.x, G);
            while (!w.done() && npre < C::kStages) {
                const int64_t tn = w.tile % p.TN;
                int c = (int)w.cb;
                int left = (int)(w.ce - w.cb);
                while (left > 0 && npre < C::kStages) {
                    const int nch = left < SC ? left : SC;
                    const uint32_t st = (uint32_t)npre;          // first round: slot npre, no wait
                    ptx::mbar_arrive_expect_tx_elect(code_bar((int)st), (uint32_t)(nch * C::kChunkWBytes));
                    ptx::bulk_g2s_elect(sbase + C::kOffCodes + st * C::kCodeStageBytes,
                                        p.wnative + (tn * p.Kc + c) * (int64_t)C::kChunkWBytes,
                                        (uint32_t)(nch * C::kChunkWBytes), code_bar((int)st));
                    c += nch;
                    left -= nch;
                    ++npre;
                }
                w.next();
            }
        }
        ptx::pdl_wait();
        int s = 0;
        uint32_t ph = 0;
        bool ready = false;                      // empty(s) already seen complete
        bool ok = true;
        int64_t issued = 0;
        SegWalk w(p, blockIdx.x, G);
        while (!w.done()) {
            const int64_t tm = w.tile / p.TN, tn = w.tile - tm * p.TN;
            int c = (int)w.cb;                     // K chunk within the tile
            const uint8_t* src = p.wnative + (tn * p.Kc + c) * (int64_t)C::kChunkWBytes;
            const int32_t ty = (int32_t)(tm * BN);
            int left = (int)(w.ce - w.cb);
            while (left > 0) {
                const int nch = left < SC ? left : SC;
                const bool pre = issued < npre;      // codes already in flight, empty(s) fresh
                if (!ready && !pre) {
                    ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(empty_bar(s), ph ^ 1u, kWaitLimitNs));
                    if (!ok) break;
                }
                const int s1 = (s + 1 == C::kStages) ? 0 : s + 1;
                const uint32_t ph1 = (s + 1 == C::kStages) ? ph ^ 1u : ph;
                const uint32_t t_e = ptx::mbar_test(empty_bar(s1), ph1 ^ 1u);
                if (!pre) {
                    ptx::mbar_arrive_expect_tx_elect(code_bar(s), (uint32_t)(nch * C::kChunkWBytes));
                    ptx::bulk_g2s_elect(sbase + C::kOffCodes + (uint32_t)s * C::kCodeStageBytes, src,
                                        (uint32_t)(nch * C::kChunkWBytes), code_bar(s));
                }
                ptx::mbar_arrive_expect_tx_elect(full_bar(s), (uint32_t)(nch * C::kBChunkBytes));
                if (nch == SC) {
#pragma unroll
                    for (int j = 0; j < SC; ++j)
                        ptx::tma_load_2d_elect(sbase + (uint32_t)(s * C::kBStageBytes + j * C::kBChunkBytes), &xmap,
                                               (c + j) * SHERRY_KCHUNK, ty, full_bar(s));
                } else {
                    for (int j = 0; j < nch; ++j)
                        ptx::tma_load_2d_elect(sbase + (uint32_t)(s * C::kBStageBytes + j * C::kBChunkBytes), &xmap,
                                               (c + j) * SHERRY_KCHUNK, ty, full_bar(s));
                }
                src += nch * C::kChunkWBytes;
                c += nch;
                left -= nch;
                ++issued;
                s = s1;
                ph = ph1;
                ready = __all_sync(0xffffffffu, t_e != 0u);
            }
            if (!ok) break;
            w.next();
        }
        if (!ok && lane == 0) report(p.status, abort_flag, SHERRY_DEV_TIMEOUT_PRODUCER);
        // every copy issued has landed before the CTA may exit (in the
        // normal flow the consumers already waited for all of them)
        const int64_t from = issued > C::kStages ? issued - C::kStages : 0;
        int ds = (int)(from % C::kStages);
        uint32_t dph = (uint32_t)((from / C::kStages) & 1);
        for (int64_t i = from; i < issued; ++i) {
            const bool landed = ptx::mbar_wait_bounded(full_bar(ds), dph, kWaitLimitNs) &&
                                ptx::mbar_wait_bounded(code_bar(ds), dph, kWaitLimitNs);
            if (!__all_sync(0xffffffffu, landed)) {
                if (lane == 0) atomicCAS(p.status, 0u, (unsigned)SHERRY_DEV_TIMEOUT_DRAIN);
                break;
            }
            if (++ds == C::kStages) { ds = 0; dph ^= 1u; }
        }
    } else if (warp == kMmaWarp) {
        // The MMA issue blocks while the tensor pipe is busy and the pipe holds
        // almost no queued work, so every instruction between two MMAs is a
        // bubble.  Hence: the whole warp runs the loop converged, with every
        // loop value warp-uniform (votes make the wait results uniform), and
        // one elected lane issues inside the MMA's own instruction sequence;
        // and the next stage's barriers are tested (non-blocking) before the
        // current stage's MMAs, so a stage whose inputs are ready starts with
        // no wait.
        int s = 0, a = 0, d = 0;
        uint32_t sph = 0, aph = 0, dph = 0;
        bool issued_any = false, ok = true;
        bool ready = false;                      // this stage's full and afull already seen complete
        SegWalk w(p, blockIdx.x, G);
        while (!w.done()) {
            int left = (int)(w.ce - w.cb);         // chunks of this tile segment
            ok = __all_sync(0xffffffffu, ptx::mbar_wait_bounded(dempty_bar(d), dph ^ 1u, kWaitLimitNs));
            if (!ok) break;
            const uint32_t d_tmem = tmem + (uint32_t)(d * BN);
            uint32_t acc0 = 0u;
            while (left > 0) {
                if (!ready) {
                    ok = ptx::mbar_wait_bounded(full_bar(s), sph, kWaitLimitNs) &&
                         ptx::mbar_wait_bounded(afull_bar(a), aph, kWaitLimitNs);
                    ok = __all_sync(0xffffffffu, ok);
                    if (!ok) break;
                }
                ptx::tc_fence_after();
                const int s1 = (s + 1 == C::kStages) ? 0 : s + 1;
                const int a1 = (a + 1 == C::kAStages) ? 0 : a + 1;
                const uint32_t sph1 = (s + 1 == C::kStages) ? sph ^ 1u : sph;
                const uint32_t aph1 = (a + 1 == C::kAStages) ? aph ^ 1u : aph;
                // both tests issue before the MMAs; their results are read
                // only after the stage's last MMA
                const uint32_t t_full = ptx::mbar_test(full_bar(s1), sph1);
                const uint32_t t_a = ptx::mbar_test(afull_bar(a1), aph1);
                const uint32_t a_tmem = tmem + (uint32_t)(C::kACol0 + a * C::kACols);
                // descriptor of the stage's first K step; later steps only
                // add to the start-address field (16-byte units)
                const uint64_t desc0 = b_desc_sw128(sbase + (uint32_t)s * C::kBStageBytes);
                if (left >= SC) {
#pragma unroll
                    for (int j = 0; j < SC; ++j)
                        ptx::mma_i8_ts_chunk_elect(d_tmem, a_tmem + (uint32_t)(32 * j),
                                                   desc0 + (uint64_t)((j * C::kBChunkBytes) >> 4), C::kIdesc,
                                                   j == 0 ? acc0 : 1u);
                    left -= SC;
                } else {
                    for (int j = 0; j < left; ++j)
                        ptx::mma_i8_ts_chunk_elect(d_tmem, a_tmem + (uint32_t)(32 * j),
                                                   desc0 + (uint64_t)((j * C::kBChunkBytes) >> 4), C::kIdesc,
                                                   j == 0 ? acc0 : 1u);
                    left = 0;
                }
                ptx::tc_commit_elect(empty_bar(s));
                ptx::tc_commit_elect(aempty_bar(a));
                issued_any = true;
                acc0 = 1u;
                s = s1; a = a1; sph = sph1; aph = aph1;
                ready = __all_sync(0xffffffffu, (t_full & t_a) != 0u);
            }
            if (!ok) break;
            ptx::tc_commit_elect(dfull_bar(d));
            if (++d == C::kDBufs) { d = 0; dph ^= 1u; }
            w.next();
        }
        if (!ok && lane == 0) report(p.status, abort_flag, SHERRY_DEV_TIMEOUT_MMA);
        if (issued_any) {
            // all MMAs of this warp complete before tensor memory is freed
            ptx::tc_commit_elect(drain_bar);
            const bool done = ptx::mbar_wait_bounded(drain_bar, 0, kWaitLimitNs);
            if (!__all_sync(0xffffffffu, done) && lane == 0)
                atomicCAS(p.status, 0u, (unsigned)SHERRY_DEV_TIMEOUT_DRAIN);
        }
    } else if (warp >= kDecWarp0 && warp < kDecWarp0 + 4 * C::kDecGroups) {
        const int grp = (warp - kDecWarp0) / 4;
        const int quad = warp & 3;                 // TMEM lane quadrant of this warp
        const int row = quad * 32 + lane;          // row within the 128-row tile
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        // 128-byte aligned: a code's entry address is (code * 4) | table_s
        const uint32_t table_s = ptx::smem_u32(table);
        // byte offsets of this row's five code words within a chunk
        uint32_t wpos[SHERRY_CHUNK_WORDS];
#pragma unroll
        for (int k = 0; k < SHERRY_CHUNK_WORDS; ++k) wpos[k] = 4u * (uint32_t)sherry_word_pos(k, row);
        int s = 0, a = 0;
        uint32_t sph = 0, aph = 0;
        int turn = 0;                               // iteration index modulo C::kDecGroups
        bool quit = false;
        SegWalk w(p, blockIdx.x, G);
        for (; !w.done() && !quit; w.next()) {
          for (int left = (int)(w.ce - w.cb); left > 0; left -= SC, turn = (turn + 1 == C::kDecGroups) ? 0 : turn + 1) {
            const int nch = left < SC ? left : SC;
            const bool mine = turn == grp;
            if (mine) {
                // no per-stage abort poll: after another role gave up, this
                // wait runs out by itself and the group leaves
                bool ok = ptx::mbar_wait_bounded(code_bar(s), sph, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, ok)) {
                    if (lane == 0) report(p.status, abort_flag, SHERRY_DEV_TIMEOUT_DECODER);
                    quit = true;
                    break;
                }
                const uint32_t codes_s = sbase + (uint32_t)(C::kOffCodes + s * C::kCodeStageBytes);
                if constexpr (WF == kWeightInt4) {
                    // SINT4 -> int8 16 w (shift into the high half of each
                    // byte); the stage's weights are read while its A slot is
                    // filled, then both are released
                    ok = ptx::mbar_wait_bounded(aempty_bar(a), aph ^ 1u, kWaitLimitNs);
                    if (!__all_sync(0xffffffffu, ok)) {
                        if (lane == 0) report(p.status, abort_flag, SHERRY_DEV_TIMEOUT_DECODER);
                        quit = true;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t wrow = codes_s + (uint32_t)(16 * row);
#pragma unroll
                    for (int j = 0; j < SC; ++j) {
                        if (j >= nch) break;
                        uint32_t a_vals[32];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            uint32_t v[4];
                            ptx::lds_v4_u32(wrow + (uint32_t)(j * C::kChunkWBytes + q * SHERRY_TILE_ROWS * 16), v);
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                a_vals[8 * q + 2 * i] = (v[i] << 4) & 0xF0F0F0F0u;
                                a_vals[8 * q + 2 * i + 1] = v[i] & 0xF0F0F0F0u;
                            }
                        }
                        ptx::tmem_st_32x32b_x32(lane_base + (uint32_t)(C::kACol0 + a * C::kACols + 32 * j), a_vals);
                    }
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(empty_bar(s));
                    ptx::tmem_wait_st();
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(afull_bar(a));
                } else {
                uint32_t w[SC][SHERRY_CHUNK_WORDS];
#pragma unroll
                for (int j = 0; j < SC; ++j)
#pragma unroll
                    for (int k = 0; k < SHERRY_CHUNK_WORDS; ++k)
                        w[j][k] = (j < nch) ? ptx::lds_u32(codes_s + (uint32_t)(j * C::kChunkWBytes) + wpos[k]) : 0u;
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(empty_bar(s));
                ok = ptx::mbar_wait_bounded(aempty_bar(a), aph ^ 1u, kWaitLimitNs);
                if (!__all_sync(0xffffffffu, ok)) {
                    if (lane == 0) report(p.status, abort_flag, SHERRY_DEV_TIMEOUT_DECODER);
                    quit = true;
                    break;
                }
                ptx::tc_fence_after();
#pragma unroll
                for (int j = 0; j < SC; ++j) {
                    if (j >= nch) break;
                    uint32_t a_vals[32];
#pragma unroll
                    for (int g = 0; g < 32; ++g) {
                        // byte offset of the group's table entry: code * 4
                        const int bit = 5 * g, wi = bit >> 5, off = bit & 31;
                        uint32_t v;
                        if (off == 0) v = w[j][wi] << 2;
                        else if (off == 1) v = w[j][wi] << 1;
                        else if (off <= 27) v = w[j][wi] >> (off - 2);
                        else v = __funnelshift_r(w[j][wi], w[j][wi + 1], off - 2);
                        a_vals[g] = ptx::lds_u32_nv((v & 0x7Cu) | table_s);
                    }
                    ptx::tmem_st_32x32b_x32(lane_base + (uint32_t)(C::kACol0 + a * C::kACols + 32 * j), a_vals);
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(afull_bar(a));
                }
            }
            if (++s == C::kStages) { s = 0; sph ^= 1u; }
            if (++a == C::kAStages) { a = 0; aph ^= 1u; }
          }
        }
    } else if (warp >= C::kEpiWarp0) {
        ptx::pdl_wait();
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const int etid = threadIdx.x - C::kEpiWarp0 * 32;     // 0..127
        int64_t seg = 0;
        int d = 0;
        uint32_t dph = 0;
        uint32_t stage_slice = 0;                  // output slices staged so far
        SegWalk w(p, blockIdx.x, G);
        for (; !w.done(); w.next()) {
            const int64_t tile = w.tile;
            const int64_t tm = tile / p.TN, tn = tile - tm * p.TN;
            const int64_t n = tn * SHERRY_TILE_ROWS + r;
            const bool complete = w.complete();
            // the tile's token scales and this row's alpha do not depend on
            // the MMAs: fetch them into shared memory (double-buffered by
            // segment) before waiting for the accumulators
            float* sc_s = reinterpret_cast<float*>(smem + C::kOffMisc + 64) + (seg & 1) * BN;
            for (int i = etid; i < BN; i += 128) {
                const int64_t m = tm * BN + i;
                sc_s[i] = (m < p.M) ? __ldg(p.x_scale + m) : 0.0f;
            }
            const float al = (n < p.N) ? __ldg(p.alpha + n) : 0.0f;
            // every epilogue thread waits; the AND over the 128 of them makes
            // the leave-or-stay decision uniform
            bool ok = !*abort_flag && ptx::mbar_wait_bounded(dfull_bar(d), dph, kWaitLimitNs);
            ok = ptx::named_bar_and(1, 128, ok);
            if (!ok) {
                if (etid == 0) report(p.status, abort_flag, SHERRY_DEV_TIMEOUT_EPILOGUE);
                break;
            }
            ptx::tc_fence_after();
            int64_t slot = 0, nparts = 1;
            if (!complete) {
                int64_t bf = 0, bl = 0;
                split_owners(p, tile, G, &bf, &bl);
                slot = bf;
                nparts = bl - bf + 1;
            }
            int32_t* wsl = p.ws + slot * (int64_t)BN * SHERRY_TILE_ROWS;
            const bool via_tma = complete && p.y_tma && p.y && !p.acc;
            if (via_tma) {
                // Each warp stores its own 32 rows x kSlice tokens through TMA
                // from its own double-buffered staging, with its own bulk
                // groups: no barrier across the epilogue warps per slice.
                constexpr int SL = C::kSlice;
                float* stg_w = reinterpret_cast<float*>(smem + C::kOffStaging) + quad * (2 * SL * 32);
#pragma unroll 1
                for (int j0 = 0; j0 < BN; j0 += SL) {
                    if (tm * BN + j0 >= p.M) break;     // tokens past M: nothing to store
                    uint32_t v[SL];
                    if constexpr (SL == 32) ptx::tmem_ld_32x32b_x32(lane_base + (uint32_t)(d * BN + j0), v);
                    else ptx::tmem_ld_32x32b_x16(lane_base + (uint32_t)(d * BN + j0), v);
                    // this slice's buffer is free once the store issued two
                    // slices ago has read it
                    if (lane == 0) ptx::bulk_wait_group_read<1>();
                    __syncwarp();
                    ptx::tmem_wait_ld();
                    float* stg = stg_w + (stage_slice & 1) * (SL * 32);
#pragma unroll
                    for (int jj = 0; jj < SL; ++jj)
                        stg[jj * 32 + lane] =
                            __fmul_rn(__fmul_rn((float)((int32_t)v[jj] >> C::kAccShift), al), sc_s[j0 + jj]);
                    ptx::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        ptx::tma_store_2d(&ymap, (int32_t)(tn * SHERRY_TILE_ROWS + quad * 32), (int32_t)(tm * BN + j0),
                                          ptx::smem_u32(stg));
                        ptx::bulk_commit_group();
                    }
                    ++stage_slice;
                }
            }
#pragma unroll 1
            for (int j0 = 0; j0 < (via_tma ? 0 : BN); j0 += 16) {
                uint32_t v[16];
                ptx::tmem_ld_32x32b_x16(lane_base + (uint32_t)(d * BN + j0), v);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    const int64_t m = tm * BN + j0 + jj;
                    if (m >= p.M) continue;
                    const int32_t a32 = (int32_t)v[jj];      // a partial sum goes to the slot as is
                    if (complete) {
                        const int32_t af = a32 >> C::kAccShift;
                        if (n < p.N) {
                            if (p.acc) p.acc[m * p.N + n] = af;
                            if (p.y) p.y[m * p.N + n] = __fmul_rn(__fmul_rn((float)af, al), sc_s[j0 + jj]);
                        }
                    } else {
                        ptx::red_add_s32(wsl + (j0 + jj) * SHERRY_TILE_ROWS + r, a32);
                    }
                }
            }
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(dempty_bar(d));
            ++seg;
            if (++d == C::kDBufs) { d = 0; dph ^= 1u; }
            const int64_t cur_tm = tm;
            if (!complete) {
                __threadfence();
                ptx::named_bar_sync(1, 128);
                if (etid == 0) {
                    const uint32_t old = atomicAdd(p.counters + slot, 1u);
                    *last_flag = (old == (uint32_t)(nparts - 1)) ? 1 : 0;
                }
                __syncwarp();
                ptx::named_bar_sync(1, 128);
                if (*last_flag) {
                    __threadfence();
                    // 16 independent L2 loads in flight per batch: one round
                    // trip per 16 tokens, not one per token
                    const int64_t mleft = p.M - cur_tm * BN;
                    const int jn = mleft < BN ? (int)mleft : BN;
                    for (int j0 = 0; j0 < jn; j0 += 16) {
                        int32_t v[16];
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj)
                            v[jj] = (j0 + jj < jn) ? __ldcg(wsl + (j0 + jj) * SHERRY_TILE_ROWS + r) : 0;
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) {
                            const int j = j0 + jj;
                            if (j >= jn) break;
                            const int64_t m = cur_tm * BN + j;
                            wsl[j * SHERRY_TILE_ROWS + r] = 0;
                            const int32_t af = v[jj] >> C::kAccShift;
                            if (n < p.N) {
                                if (p.acc) p.acc[m * p.N + n] = af;
                                if (p.y) p.y[m * p.N + n] = __fmul_rn(__fmul_rn((float)af, al), sc_s[j]);
                            }
                        }
                    }
                    if (etid == 0) atomicExch(p.counters + slot, 0u);
                }
                __syncwarp();
                ptx::named_bar_sync(1, 128);
            }
        }
        // shared memory stays valid until every TMA store has read it
        if (lane == 0) ptx::bulk_wait_group<0>();
    }

    __syncwarp();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == kMmaWarp) ptx::tmem_dealloc(tmem, kTmemCols);
}

}  // namespace tc
}  // namespace sherry
