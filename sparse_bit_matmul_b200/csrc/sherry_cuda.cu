// Device half of libsherry_b200: activation quantiser, repack, the SIMT
// comparison kernel, the tcgen05 GEMM launcher and the device entry points of
// the C ABI (include/sherry.h).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdlib>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "sherry.h"
#include "sherry_internal.h"
#include "gemv.cuh"
#include "decode.cuh"
#include "quant.cuh"
#include "tc_gemm.cuh"
#include "w4a8_gemv.cuh"

namespace sherry {

__device__ unsigned g_device_status = 0;

// ---------------------------------------------------------------------------
// Activation quantiser: one CTA per token.  a = max |x| (exact), s = a / 127
// (IEEE fp32 division), q = clamp(rint(x / s), -127, 127) with rint rounding
// half to even; a == 0 gives s = 0 and q = 0 (the arithmetic of quant.cuh).
// Each thread keeps its float4s in registers between the absmax and the
// quantisation (one read of x, all loads in flight at once) when the row
// fits (K <= 4 * kQuantXV * kQuantThreads); longer rows are read twice.
// ---------------------------------------------------------------------------
constexpr int kQuantThreads = 512;
constexpr int kQuantXV = 8;

__global__ void __launch_bounds__(kQuantThreads)
    quant_act_kernel(const float* __restrict__ x, int64_t K, int8_t* __restrict__ q, float* __restrict__ scale)
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t m = blockIdx.x;
    const float4* xr = reinterpret_cast<const float4*>(x + m * K);
    uint32_t* qw = reinterpret_cast<uint32_t*>(q + m * K);
    const int K4 = (int)(K / 4);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const bool in_regs = K4 <= kQuantXV * kQuantThreads;

    float4 v[kQuantXV];
    float a = 0.0f;
    if (in_regs) {
#pragma unroll
        for (int u = 0; u < kQuantXV; ++u) {
            const int idx = tid + u * kQuantThreads;
            v[u] = idx < K4 ? xr[idx] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
#pragma unroll
        for (int u = 0; u < kQuantXV; ++u) a = fmaxf(a, quant::absmax4(v[u]));
    } else {
#pragma unroll 4
        for (int i = tid; i < K4; i += kQuantThreads) a = fmaxf(a, quant::absmax4(xr[i]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    __shared__ float warp_max[kQuantThreads / 32];
    if (lane == 0) warp_max[warp] = a;
    __syncthreads();
    // every warp combines the warp maxima: one load per lane and a shuffle tree
    a = lane < kQuantThreads / 32 ? warp_max[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));

    const quant::Scale sc = quant::make_scale(a);
    if (tid == 0) scale[m] = sc.s;
    if (in_regs) {
#pragma unroll
        for (int u = 0; u < kQuantXV; ++u) {
            const int idx = tid + u * kQuantThreads;
            if (idx < K4) qw[idx] = quant::quantise4(v[u], sc);
        }
    } else {
#pragma unroll 4
        for (int i = tid; i < K4; i += kQuantThreads) qw[i] = quant::quantise4(xr[i], sc);
    }
}

// ---------------------------------------------------------------------------
// Self-test of failure detection: one warp initialises an mbarrier that
// nothing ever arrives on and waits for its first phase with the bounded
// wait every kernel of the library uses.  When the bound runs out it records
// SHERRY_DEV_TIMEOUT_SELFTEST in the device status word and returns.  No
// bulk copy and no tensor memory is involved, so nothing is in flight when
// the wait gives up.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32) wait_selftest_kernel(uint64_t limit_ns, unsigned* status)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = ptx::smem_u32(&bar);
    if (threadIdx.x == 0) {
        ptx::mbar_init(b, 1);
        ptx::fence_mbar_init();
    }
    __syncwarp();
    const bool done = ptx::mbar_wait_bounded(b, 0, limit_ns);
    if (!__all_sync(0xffffffffu, done) && threadIdx.x == 0)
        atomicCAS(status, 0u, (unsigned)SHERRY_DEV_TIMEOUT_SELFTEST);
}

// ---------------------------------------------------------------------------
// Repack: canonical stream -> kernel-native layout (one thread per word).
// ---------------------------------------------------------------------------
__global__ void repack_kernel(const uint8_t* __restrict__ codes, int64_t N, int64_t K, uint32_t* __restrict__ out,
                              int64_t total_words)
{
    const int64_t row_bytes = K / 32 * 5;
    const int64_t Kc = sherry_k_chunks(K);
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total_words;
         idx += (int64_t)gridDim.x * blockDim.x) {
        const int64_t j = (idx / SHERRY_TILE_ROWS) % SHERRY_CHUNK_WORDS;
        const int64_t r = (idx - 8 * j) & (SHERRY_TILE_ROWS - 1);    // position idx % 128 holds row r
        const int64_t c = (idx / (SHERRY_TILE_ROWS * SHERRY_CHUNK_WORDS)) % Kc;
        const int64_t t = idx / (SHERRY_TILE_ROWS * SHERRY_CHUNK_WORDS * Kc);
        const int64_t n = t * SHERRY_TILE_ROWS + r;
        const int64_t b0 = c * (SHERRY_CHUNK_WORDS * 4) + 4 * j;
        uint32_t w = 0;
        if (n < N) {
#pragma unroll
            for (int b = 0; b < 4; ++b)
                if (b0 + b < row_bytes) w |= (uint32_t)codes[n * row_bytes + b0 + b] << (8 * b);
        }
        out[idx] = w;
    }
}

// ---------------------------------------------------------------------------
// W4A8 repack: canonical SINT4 rows [N][K/2] (even k in the low nibble) ->
// the native blocks of sherry_internal.h (one thread per native word).
// Rows past N and chunks past K are zero.
// ---------------------------------------------------------------------------
__global__ void repack_w4_kernel(const uint8_t* __restrict__ w4, int64_t N, int64_t K, uint32_t* __restrict__ out,
                                 int64_t total_words)
{
    const int64_t Kc = sherry_k_chunks(K);
    for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < total_words;
         idx += (int64_t)gridDim.x * blockDim.x)
        out[idx] = sherry_w4_native_word(w4, N, K, Kc, idx);
}

// ---------------------------------------------------------------------------
// SIMT comparison kernel: thread = weight row, MT tokens per CTA, decode
// through a 32-entry shared table, dp4a against the activations.
// ---------------------------------------------------------------------------
constexpr int kSimtMT = 8;

__global__ void __launch_bounds__(SHERRY_TILE_ROWS)
    simt_gemm_kernel(const int8_t* __restrict__ xq, const float* __restrict__ xs,
                     const uint32_t* __restrict__ wn, const float* __restrict__ alpha, float* __restrict__ y,
                     int32_t* __restrict__ acc_out, int64_t M, int64_t N, int64_t K)
{
    __shared__ uint32_t table[32];
    if (threadIdx.x < 32) {
        const uint32_t c = threadIdx.x, z = c & 3u;
        uint32_t word = 0, slot = 2;
        for (uint32_t i = 0; i < 4; ++i) {
            if (i == z) continue;
            word |= (((c >> slot) & 1u) ? 0xFFu : 0x01u) << (8 * i);
            ++slot;
        }
        table[c] = word;
    }
    __syncthreads();
    const int64_t t = blockIdx.x;
    const int r = threadIdx.x;
    const int64_t n = t * SHERRY_TILE_ROWS + r;
    const int64_t m0 = (int64_t)blockIdx.y * kSimtMT;
    const int64_t Kc = sherry_k_chunks(K);
    int32_t acc[kSimtMT];
#pragma unroll
    for (int i = 0; i < kSimtMT; ++i) acc[i] = 0;
    for (int64_t c = 0; c < Kc; ++c) {
        const uint32_t* blk = wn + (t * Kc + c) * (SHERRY_TILE_ROWS * SHERRY_CHUNK_WORDS);
        uint32_t w[SHERRY_CHUNK_WORDS + 1];
#pragma unroll
        for (int j = 0; j < SHERRY_CHUNK_WORDS; ++j) w[j] = blk[sherry_word_pos(j, r)];
        w[SHERRY_CHUNK_WORDS] = 0;
        for (int g = 0; g < 32; ++g) {
            const int64_t k = c * SHERRY_KCHUNK + 4 * g;
            if (k >= K) break;
            const int bit = 5 * g;
            const uint32_t v = __funnelshift_r(w[bit >> 5], w[(bit >> 5) + 1], bit & 31);
            const int W4 = (int)table[v & 31u];
#pragma unroll
            for (int i = 0; i < kSimtMT; ++i) {
                const int64_t m = m0 + i;
                if (m < M) acc[i] = __dp4a(W4, *reinterpret_cast<const int*>(xq + m * K + k), acc[i]);
            }
        }
    }
    if (n >= N) return;
    const float al = alpha[n];
#pragma unroll
    for (int i = 0; i < kSimtMT; ++i) {
        const int64_t m = m0 + i;
        if (m >= M) break;
        if (acc_out) acc_out[m * N + n] = acc[i];
        if (y) y[m * N + n] = __fmul_rn(__fmul_rn((float)acc[i], al), xs[m]);
    }
}

// ---------------------------------------------------------------------------
// host helpers
// ---------------------------------------------------------------------------
namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? SHERRY_OK : SHERRY_ERR_CUDA; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

struct DeviceInfo {
    bool checked = false;
    bool ok = false;
    int sms = 0;
    int max_smem_optin = 0;
};

std::mutex g_mutex;
std::vector<DeviceInfo> g_dev;

struct Workspace {
    void* ptr = nullptr;
    size_t bytes = 0;
};
std::vector<Workspace> g_ws;

int device_info(DeviceInfo* out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SHERRY_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((int)g_dev.size() <= dev) g_dev.resize(dev + 1);
    DeviceInfo& d = g_dev[dev];
    if (!d.checked) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return SHERRY_ERR_CUDA;
        d.ok = (prop.major == 10 && prop.minor == 0);
        d.sms = prop.multiProcessorCount;
        d.max_smem_optin = (int)prop.sharedMemPerBlockOptin;
        d.checked = true;
    }
    *out = d;
    return d.ok ? SHERRY_OK : SHERRY_ERR_DEVICE;
}

// Zero-initialised per-device workspace of at least `bytes`, ordered on `stream`.
// CTAs of a tensor-core launch with T output tiles of BN tokens and Kc K
// chunks each (U = T * Kc units).
// T >= SMs: one CTA per SM (whole tiles plus an even share of the leftover
// tiles, split across CTAs; their sums overlap the whole tiles).
// T < SMs: the sums of split tiles come at the end of the kernel, where they
// were measured at ~18 us for 128-token tiles (2 + 16 * BN / 128 us is the
// estimate used here), against ~0.27 us per K chunk walked.  So every tile is
// split into S = SMs div T equal K shares (T * S CTAs) only when that saves
// more chunk time than the sums cost; otherwise S = 1: one CTA per tile, no
// tile split, no cross-CTA sum.
int64_t tc_grid(int64_t T, int64_t U, int64_t sms, int64_t Kc, int bn)
{
    int64_t g = sms;
    if (T < sms) {
        const int64_t S = sms / T;
        const double saved_us = 0.27 * (double)Kc * (1.0 - 1.0 / (double)S);
        const double sums_us = 2.0 + 16.0 * (double)bn / 128.0;
        g = (S > 1 && saved_us > sums_us) ? T * S : T;
    }
    return std::min<int64_t>(g, U);
}

// The per-device split-K workspace set aside by sherry_reserve: never
// allocated here (the asynchronous entry points allocate nothing and never
// synchronise); SHERRY_ERR_WORKSPACE when it is smaller than a call needs.
int get_workspace(size_t bytes, void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SHERRY_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((int)g_ws.size() <= dev || g_ws[dev].bytes < bytes) return SHERRY_ERR_WORKSPACE;
    *out = g_ws[dev].ptr;
    return SHERRY_OK;
}

// Token tile of the tensor-core kernel for M tokens (the dispatch of
// sherry_gemm_tc and sherry_w4a8_gemm_tc).
int tc_token_tile(int64_t M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : M < 1536 ? 128 : 192; }

// Split-K workspace for every launch of up to M tokens on `sms` SMs: the
// partial-sum slots of at most one CTA per SM, BN tokens x 128 rows each, and
// one arrival counter per CTA.
size_t tc_workspace_bytes(int64_t M, int sms)
{
    return (size_t)sms * tc_token_tile(M) * SHERRY_TILE_ROWS * sizeof(int32_t) + (size_t)sms * sizeof(uint32_t);
}

// fp32 y [M][N]: boxes of 32 rows n x box_m tokens m (no swizzle), one per
// epilogue warp; needs rows of whole 16-byte units (N % 4 == 0) and a
// 16-byte aligned base.
int make_y_map(CUtensorMap* map, const float* y, int64_t M, int64_t N, int box_m)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return SHERRY_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)N * 4};
    cuuint32_t box[2] = {32, (cuuint32_t)box_m};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(y), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? SHERRY_OK : SHERRY_ERR_CUDA;
}

int make_x_map(CUtensorMap* map, const int8_t* x, int64_t M, int64_t K, int bn)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return SHERRY_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {SHERRY_KCHUNK, (cuuint32_t)bn};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t*>(x), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? SHERRY_OK : SHERRY_ERR_CUDA;
}

unsigned* device_status_ptr()
{
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    return static_cast<unsigned*>(p);
}

// Launch with programmatic dependent launch: the kernel may start while the
// previous kernel on the stream finishes; it orders itself with
// griddepcontrol.wait before touching anything that kernel may write.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <int BN, int SC, int WF = tc::kWeightSherry>
int launch_tc(const int8_t* x, const float* xs, const void* wn, const float* alpha, float* y, int32_t* acc,
              int64_t M, int64_t N, int64_t K, cudaStream_t stream)
{
    using C = tc::Cfg<BN, SC, WF>;
    DeviceInfo di;
    int st = device_info(&di);
    if (st != SHERRY_OK) return st;
    tc::Params p;
    p.wnative = static_cast<const uint8_t*>(wn);
    p.alpha = alpha;
    p.x_scale = xs;
    p.y = y;
    p.acc = acc;
    p.M = M;
    p.N = N;
    p.K = K;
    p.TM = (M + BN - 1) / BN;
    p.TN = sherry_row_tiles(N);
    p.Kc = sherry_k_chunks(K);
    p.U = p.TM * p.TN * p.Kc;
    const int64_t grid = tc_grid(p.TM * p.TN, p.U, di.sms, p.Kc, BN);
    // the workspace is touched only by tiles whose K range is split across
    // CTAs: the last T mod G tiles (none when every CTA takes whole tiles)
    p.ws = nullptr;
    p.counters = nullptr;
    if ((p.TM * p.TN) % grid != 0) {
        void* ws = nullptr;
        const size_t ws_acc = (size_t)grid * BN * SHERRY_TILE_ROWS * sizeof(int32_t);
        st = get_workspace(ws_acc + (size_t)grid * sizeof(uint32_t), &ws);
        if (st != SHERRY_OK) return st;
        p.ws = static_cast<int32_t*>(ws);
        p.counters = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + ws_acc);
    }
    p.status = device_status_ptr();
    if (!p.status) return SHERRY_ERR_CUDA;

    CUtensorMap map, ymap;
    st = make_x_map(&map, x, M, K, BN);
    if (st != SHERRY_OK) return st;
    std::memset(&ymap, 0, sizeof(ymap));
    p.y_tma = (y && N % 4 == 0 && aligned16(y)) ? 1 : 0;
    if (p.y_tma && make_y_map(&ymap, y, M, N, C::kSlice) != SHERRY_OK) p.y_tma = 0;

    // at least half of the SM's shared memory so that exactly one CTA (and
    // one 512-column tensor-memory allocation) lives on each SM
    const int smem = std::max(C::kSmemBytes, 120 * 1024);
    if (smem > di.max_smem_optin) return SHERRY_ERR_DEVICE;
    cudaError_t e = cudaFuncSetAttribute(tc::sherry_gemm_tc_kernel<BN, SC, WF>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return SHERRY_ERR_CUDA;
    e = launch_pdl(tc::sherry_gemm_tc_kernel<BN, SC, WF>, dim3((unsigned)grid), dim3(C::kThreads), (size_t)smem,
                   stream, map, ymap, p);
    if (e != cudaSuccess) return cuda_status(e);
    return cuda_status(cudaGetLastError());
}


// W4A8 GEMV for M <= MT tokens: 32 rows per CTA; 16 K parts (512 threads)
// when there are at least two CTAs per SM, else 32 (1024 threads) so that
// each SM keeps enough 16-byte loads in flight.
template <int MT>
int launch_w4_gemv(const int8_t* x, const float* xs, const void* wn, const float* scale, float* y, int32_t* acc,
                   int64_t M, int64_t N, int64_t K, cudaStream_t stream)
{
    DeviceInfo di;
    const int st = device_info(&di);
    if (st != SHERRY_OK) return st;
    const int64_t ctas = (N + w4gemv::kRows - 1) / w4gemv::kRows;
    const uint8_t* w = static_cast<const uint8_t*>(wn);
    cudaError_t e;
    if (ctas >= 2 * (int64_t)di.sms)
        e = launch_pdl(w4gemv::w4a8_gemv_kernel<MT, 16>, dim3((unsigned)ctas), dim3(w4gemv::kRows * 16), 0, stream,
                       x, xs, w, scale, y, acc, M, N, K);
    else
        e = launch_pdl(w4gemv::w4a8_gemv_kernel<MT, 32>, dim3((unsigned)ctas), dim3(w4gemv::kRows * 32), 0, stream,
                       x, xs, w, scale, y, acc, M, N, K);
    if (e != cudaSuccess) return cuda_status(e);
    return cuda_status(cudaGetLastError());
}

template <int MT>
int launch_gemv(const int8_t* x, const float* xs, const void* wn, const float* alpha, float* y, int32_t* acc,
                int64_t M, int64_t N, int64_t K, cudaStream_t stream)
{
    DeviceInfo di;
    int st = device_info(&di);
    if (st != SHERRY_OK) return st;
    gemv::Params p;
    p.wnative = static_cast<const uint8_t*>(wn);
    p.x = x;
    p.x_scale = xs;
    p.alpha = alpha;
    p.y = y;
    p.acc = acc;
    p.M = M;
    p.N = N;
    p.K = K;
    p.TN = sherry_row_tiles(N);
    p.Kc = sherry_k_chunks(K);
    if (p.Kc > (int64_t)gemv::kMaxSL * gemv::kMaxNS || p.TN > 0x7fffffff) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    // K-slices per tile (the cluster size): enough for at most kMaxSL chunks
    // per slice, more while the grid has fewer than two CTAs per SM
    int NS = 1;
    while (NS < gemv::kMaxNS && NS < p.Kc &&
           ((p.Kc + NS - 1) / NS > gemv::kMaxSL || p.TN * NS < 2 * (int64_t)di.sms))
        NS *= 2;
    p.NS = NS;
    p.SL = (int)((p.Kc + NS - 1) / NS);
    p.status = device_status_ptr();
    if (!p.status) return SHERRY_ERR_CUDA;
    const int smem = gemv::smem_bytes(MT, p.SL);
    if (smem > di.max_smem_optin) return SHERRY_ERR_DEVICE;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(gemv::sherry_gemv_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
        return SHERRY_ERR_CUDA;
    if (cudaFuncSetAttribute(gemv::sherry_gemv_kernel<MT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return SHERRY_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)p.TN, (unsigned)NS);
    cfg.blockDim = dim3(gemv::kThreads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = (unsigned)NS;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cuda_status(cudaLaunchKernelEx(&cfg, gemv::sherry_gemv_kernel<MT>, p));
}

template <int MT, bool FUSED, int RT>
int launch_decode_rt(const decode::Params& p, const decode::Plan& pl, cudaStream_t stream)
{
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    // One shared-memory carveout for every shape: left to the driver, the
    // L1/shared split follows each launch's request, and consecutive layers
    // of different shapes (27, 70 and 88 KB) then cannot share an SM, so the
    // next layer's CTAs lose their early start (measured: 11.2 us per call
    // alternating two shapes that take 7.6 and 9.0 us on their own).
    std::call_once(attr_once, [&] {
        attr_err = cudaFuncSetAttribute(decode::sherry_decode_kernel<MT, FUSED, RT>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, decode::kSmemBudgetMax);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(decode::sherry_decode_kernel<MT, FUSED, RT>,
                                            cudaFuncAttributePreferredSharedMemoryCarveout,
                                            cudaSharedmemCarveoutMaxShared);
    });
    if (attr_err != cudaSuccess) return SHERRY_ERR_CUDA;
    return cuda_status(launch_pdl(decode::sherry_decode_kernel<MT, FUSED, RT>, dim3((unsigned)pl.G),
                                  dim3((unsigned)pl.threads), (size_t)pl.smem, stream, p));
}

template <int MT, bool FUSED>
int launch_decode(const decode::Params& p0, cudaStream_t stream)
{
    DeviceInfo di;
    int st = device_info(&di);
    if (st != SHERRY_OK) return st;
    decode::Params p = p0;
    p.Kc = sherry_k_chunks(p.K);
    if (p.M > MT) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    decode::Plan pl;
    if (!decode::plan(p.N, p.Kc, p.M, di.sms, &pl)) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    p.G = pl.G;
    p.R = pl.R;
    p.Q = pl.Q;
    p.P = pl.P;
    p.CPT = pl.CPT;
    p.NS = pl.NS;
    p.S = pl.S;
    if (pl.smem > di.max_smem_optin) return SHERRY_ERR_DEVICE;
    if (pl.RT == 4) {
        if constexpr (MT <= 2) return launch_decode_rt<MT, FUSED, 4>(p, pl, stream);
        else return SHERRY_ERR_UNSUPPORTED_SHAPE;
    }
    if (pl.RT == 2) return launch_decode_rt<MT, FUSED, 2>(p, pl, stream);
    return launch_decode_rt<MT, FUSED, 1>(p, pl, stream);
}

// Per-device buffer for the int8 activations and scales of sherry_linear
// when the caller passes none and the fused kernel does not apply; set aside
// by sherry_reserve, never allocated here.
std::vector<Workspace> g_act;

size_t act_buffer_bytes(int64_t M, int64_t K) { return (((size_t)M * (size_t)K + 255) & ~size_t(255)) + 4 * (size_t)M; }

int get_act_buffer(size_t bytes, void** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SHERRY_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((int)g_act.size() <= dev || g_act[dev].bytes < bytes) return SHERRY_ERR_WORKSPACE;
    *out = g_act[dev].ptr;
    return SHERRY_OK;
}

// Grow one per-device buffer to at least `bytes` (host-synchronous; the
// device is idle before an older, smaller buffer is freed), zero-filled.
int grow_buffer(Workspace& w, size_t bytes)
{
    if (w.bytes >= bytes) return SHERRY_OK;
    if (w.ptr) {
        if (cudaDeviceSynchronize() != cudaSuccess) return SHERRY_ERR_CUDA;
        cudaFree(w.ptr);
        w.ptr = nullptr;
        w.bytes = 0;
    }
    void* ptr = nullptr;
    if (cudaMalloc(&ptr, bytes) != cudaSuccess) return SHERRY_ERR_CUDA;
    if (cudaMemset(ptr, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
        cudaFree(ptr);
        return SHERRY_ERR_CUDA;
    }
    w.ptr = ptr;
    w.bytes = bytes;
    return SHERRY_OK;
}

int check_gemm_args(const int8_t* x, const float* xs, const void* wn, const float* alpha, const float* y,
                    const int32_t* acc, int64_t M, int64_t N, int64_t K)
{
    if (!x || !xs || !wn || !alpha || (!y && !acc)) return SHERRY_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0) return SHERRY_ERR_INVALID_ARG;
    if (!sherry_shape_ok(M, N, K)) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(wn)) return SHERRY_ERR_INVALID_ARG;
    return SHERRY_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// Fixed scratch for sherry_gemm_noalloc: the split-K partial sums and arrival
// counters of at most kNoAllocMaxCtas CTAs for token tiles of up to
// kNoAllocMaxBN tokens (M <= 32).  It lives in the library's own device
// image, so it is reserved on every GPU that loads the library until exit.
// ---------------------------------------------------------------------------
constexpr int kNoAllocMaxCtas = 160;
constexpr int kNoAllocMaxBN = 32;
constexpr size_t kNoAllocAccWords = (size_t)kNoAllocMaxCtas * kNoAllocMaxBN * SHERRY_TILE_ROWS;
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocAccWords + kNoAllocMaxCtas];

namespace {

std::mutex g_noalloc_mutex;
std::vector<int32_t*> g_noalloc_ptr;   // device address of g_noalloc_scratch, per device

// Host code may not use g_noalloc_scratch's name as a device address: it is a
// host-side stand-in.  The address is looked up once per device, with that
// device current.
int noalloc_scratch(int32_t** out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SHERRY_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_noalloc_mutex);
    if ((int)g_noalloc_ptr.size() <= dev) g_noalloc_ptr.resize(dev + 1, nullptr);
    if (!g_noalloc_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return SHERRY_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<int32_t*>(ptr);
    }
    *out = g_noalloc_ptr[dev];
    return SHERRY_OK;
}

template <int BN, int SC>
int launch_tc_noalloc(const int8_t* x, const float* xs, const void* wn, const float* alpha, float* y,
                      int32_t* acc, int64_t M, int64_t N, int64_t K, cudaStream_t stream)
{
    using C = tc::Cfg<BN, SC>;
    static_assert(BN <= kNoAllocMaxBN, "token tile larger than the fixed scratch");
    DeviceInfo di;
    int st = device_info(&di);
    if (st != SHERRY_OK) return st;
    int32_t* scratch = nullptr;
    st = noalloc_scratch(&scratch);
    if (st != SHERRY_OK) return st;
    tc::Params p;
    p.wnative = static_cast<const uint8_t*>(wn);
    p.alpha = alpha;
    p.x_scale = xs;
    p.y = y;
    p.acc = acc;
    p.M = M;
    p.N = N;
    p.K = K;
    p.TM = (M + BN - 1) / BN;
    p.TN = sherry_row_tiles(N);
    p.Kc = sherry_k_chunks(K);
    p.U = p.TM * p.TN * p.Kc;
    const int64_t grid = std::min<int64_t>(tc_grid(p.TM * p.TN, p.U, di.sms, p.Kc, BN), kNoAllocMaxCtas);
    p.ws = scratch;
    p.counters = reinterpret_cast<uint32_t*>(scratch + kNoAllocAccWords);
    p.status = device_status_ptr();
    if (!p.status) return SHERRY_ERR_CUDA;
    // slots and counters this launch uses start at zero, whatever an earlier
    // (possibly aborted) call left behind
    if (cudaMemsetAsync(p.ws, 0, (size_t)grid * BN * SHERRY_TILE_ROWS * sizeof(int32_t), stream) != cudaSuccess ||
        cudaMemsetAsync(p.counters, 0, (size_t)grid * sizeof(uint32_t), stream) != cudaSuccess)
        return SHERRY_ERR_CUDA;
    CUtensorMap map, ymap;
    st = make_x_map(&map, x, M, K, BN);
    if (st != SHERRY_OK) return st;
    std::memset(&ymap, 0, sizeof(ymap));
    p.y_tma = (y && N % 4 == 0 && aligned16(y)) ? 1 : 0;
    if (p.y_tma && make_y_map(&ymap, y, M, N, C::kSlice) != SHERRY_OK) p.y_tma = 0;
    const int smem = std::max(C::kSmemBytes, 120 * 1024);
    if (smem > di.max_smem_optin) return SHERRY_ERR_DEVICE;
    if (cudaFuncSetAttribute(tc::sherry_gemm_tc_kernel<BN, SC>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
        return SHERRY_ERR_CUDA;
    const cudaError_t e = launch_pdl(tc::sherry_gemm_tc_kernel<BN, SC>, dim3((unsigned)grid), dim3(C::kThreads),
                                     (size_t)smem, stream, map, ymap, p);
    if (e != cudaSuccess) return cuda_status(e);
    return cuda_status(cudaGetLastError());
}

}  // namespace

}  // namespace sherry

using namespace sherry;

extern "C" {

int sherry_repack(const uint8_t* codes_dev, int64_t N, int64_t K, void* native_dev, void* stream)
{
    if (!codes_dev || !native_dev) return SHERRY_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0) return SHERRY_ERR_INVALID_ARG;
    if (!sherry_shape_ok(1, N, K)) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(native_dev)) return SHERRY_ERR_INVALID_ARG;
    const int64_t words = (int64_t)(sherry_native_bytes(N, K) / 4);
    const int threads = 256;
    const int64_t blocks = std::min<int64_t>((words + threads - 1) / threads, 148 * 32);
    repack_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
        codes_dev, N, K, static_cast<uint32_t*>(native_dev), words);
    return cuda_status(cudaGetLastError());
}

int sherry_w4a8_repack(const uint8_t* w4_dev, int64_t N, int64_t K, void* native_dev, void* stream)
{
    if (!w4_dev || !native_dev) return SHERRY_ERR_INVALID_ARG;
    if (N <= 0 || K <= 0) return SHERRY_ERR_INVALID_ARG;
    const size_t bytes = sherry_w4a8_native_bytes(N, K);
    if (bytes == 0) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(native_dev)) return SHERRY_ERR_INVALID_ARG;
    const int64_t words = (int64_t)(bytes / 4);
    const int threads = 256;
    const int64_t blocks = std::min<int64_t>((words + threads - 1) / threads, 148 * 32);
    repack_w4_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
        w4_dev, N, K, static_cast<uint32_t*>(native_dev), words);
    return cuda_status(cudaGetLastError());
}

int sherry_w4a8_gemm_gemv(const int8_t* x_i8, const float* x_scale, const void* W4native, const float* scale,
                          float* y, int32_t* acc, int64_t M, int64_t N, int64_t K, void* stream)
{
    int st = check_gemm_args(x_i8, x_scale, W4native, scale, y, acc, M, N, K);
    if (st != SHERRY_OK) return st;
    if (K > SHERRY_W4_MAX_K || M > SHERRY_W4A8_GEMV_MAX_M) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M == 1) return launch_w4_gemv<1>(x_i8, x_scale, W4native, scale, y, acc, M, N, K, s);
    if (M == 2) return launch_w4_gemv<2>(x_i8, x_scale, W4native, scale, y, acc, M, N, K, s);
    return launch_w4_gemv<4>(x_i8, x_scale, W4native, scale, y, acc, M, N, K, s);
}

int sherry_w4a8_gemm_tc(const int8_t* x_i8, const float* x_scale, const void* W4native, const float* scale,
                        float* y, int32_t* acc, int64_t M, int64_t N, int64_t K, void* stream)
{
    int st = check_gemm_args(x_i8, x_scale, W4native, scale, y, acc, M, N, K);
    if (st != SHERRY_OK) return st;
    if (K > SHERRY_W4_MAX_K) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    constexpr int W4 = tc::kWeightInt4;
    // int4 stages carry 3.2x the weight bytes of code stages: two-chunk
    // stages from 32 tokens on keep at least three stages in the ring
    if (M <= 16) return launch_tc<16, 4, W4>(x_i8, x_scale, W4native, scale, y, acc, M, N, K, s);
    if (M <= 32) return launch_tc<32, 2, W4>(x_i8, x_scale, W4native, scale, y, acc, M, N, K, s);
    if (M <= 64) return launch_tc<64, 2, W4>(x_i8, x_scale, W4native, scale, y, acc, M, N, K, s);
    if (M < 1536) return launch_tc<128, 2, W4>(x_i8, x_scale, W4native, scale, y, acc, M, N, K, s);
    return launch_tc<192, 1, W4>(x_i8, x_scale, W4native, scale, y, acc, M, N, K, s);
}

// Every M runs on the tensor cores: at M = 1 and 4 (K=4096, N=14336) the
// CUDA-core GEMV measured 11.5 and 20.0 us per call against about 9.3-10.2
// us for the tensor-core kernel.
int sherry_w4a8_gemm_acc(const int8_t* x_i8, const float* x_scale, const void* W4native, const float* scale,
                         float* y, int32_t* acc, int64_t M, int64_t N, int64_t K, void* stream)
{
    return sherry_w4a8_gemm_tc(x_i8, x_scale, W4native, scale, y, acc, M, N, K, stream);
}

int sherry_w4a8_gemm(const int8_t* x_i8, const float* x_scale, const void* W4native, const float* scale, float* y,
                     int64_t M, int64_t N, int64_t K, void* stream)
{
    if (!y) return SHERRY_ERR_INVALID_ARG;
    return sherry_w4a8_gemm_acc(x_i8, x_scale, W4native, scale, y, nullptr, M, N, K, stream);
}

int sherry_quant_act(const float* x, int64_t M, int64_t K, int8_t* x_i8, float* x_scale, void* stream)
{
    if (!x || !x_i8 || !x_scale) return SHERRY_ERR_INVALID_ARG;
    if (M <= 0 || K <= 0) return SHERRY_ERR_INVALID_ARG;
    if (!sherry_shape_ok(M, 1, K)) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(x_i8)) return SHERRY_ERR_INVALID_ARG;
    return cuda_status(launch_pdl(quant_act_kernel, dim3((unsigned)M), dim3(kQuantThreads), 0,
                                  static_cast<cudaStream_t>(stream), x, K, x_i8, x_scale));
}

int sherry_gemm_acc(const int8_t* x_i8, const float* x_scale, const void* Wnative, const float* alpha, float* y,
                    int32_t* acc, int64_t M, int64_t N, int64_t K, void* stream)
{
    int st = check_gemm_args(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K);
    if (st != SHERRY_OK) return st;
    if (M <= SHERRY_GEMM_DECODE_AUTO_MAX_M) {
        DeviceInfo di;
        st = device_info(&di);
        if (st != SHERRY_OK) return st;
        decode::Plan pl;
        if (decode::plan(N, sherry_k_chunks(K), M, di.sms, &pl))
            return sherry_gemm_decode(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, stream);
    }
    return sherry_gemm_tc(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, stream);
}

int sherry_gemm_decode(const int8_t* x_i8, const float* x_scale, const void* Wnative, const float* alpha,
                       float* y, int32_t* acc, int64_t M, int64_t N, int64_t K, void* stream)
{
    int st = check_gemm_args(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K);
    if (st != SHERRY_OK) return st;
    if (M > SHERRY_DECODE_MAX_M) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    decode::Params p = {};
    p.wnative = static_cast<const uint8_t*>(Wnative);
    p.xq = x_i8;
    p.x_scale = x_scale;
    p.alpha = alpha;
    p.y = y;
    p.acc = acc;
    p.M = M;
    p.N = N;
    p.K = K;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M == 1) return launch_decode<1, false>(p, s);
    if (M == 2) return launch_decode<2, false>(p, s);
    if (M <= 4) return launch_decode<4, false>(p, s);
    return launch_decode<8, false>(p, s);
}

int sherry_linear_ex(const float* x, const void* Wnative, const float* alpha, float* y, int32_t* acc,
                     int8_t* x_i8, float* x_scale, int64_t M, int64_t N, int64_t K, void* stream)
{
    if (!x || !Wnative || !alpha || (!y && !acc)) return SHERRY_ERR_INVALID_ARG;
    if ((x_i8 == nullptr) != (x_scale == nullptr)) return SHERRY_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || K <= 0) return SHERRY_ERR_INVALID_ARG;
    if (!sherry_shape_ok(M, N, K)) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(Wnative) || (x_i8 && !aligned16(x_i8))) return SHERRY_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M <= SHERRY_LINEAR_FUSED_MAX_M) {
        DeviceInfo di;
        int st = device_info(&di);
        if (st != SHERRY_OK) return st;
        decode::Plan pl;
        if (decode::plan(N, sherry_k_chunks(K), M, di.sms, &pl)) {
            decode::Params p = {};
            p.wnative = static_cast<const uint8_t*>(Wnative);
            p.x = x;
            p.xq_out = x_i8;
            p.xs_out = x_scale;
            p.alpha = alpha;
            p.y = y;
            p.acc = acc;
            p.M = M;
            p.N = N;
            p.K = K;
            static_assert(SHERRY_LINEAR_FUSED_MAX_M <= 4, "fused launches instantiated for up to 4 tokens");
            if (M == 1) return launch_decode<1, true>(p, s);
            if (M == 2) return launch_decode<2, true>(p, s);
            return launch_decode<4, true>(p, s);
        }
    }
    if (!x_i8) {
        void* buf = nullptr;
        const size_t qbytes = ((size_t)M * (size_t)K + 255) & ~size_t(255);
        int st = get_act_buffer(act_buffer_bytes(M, K), &buf);
        if (st != SHERRY_OK) return st;
        x_i8 = static_cast<int8_t*>(buf);
        x_scale = reinterpret_cast<float*>(static_cast<uint8_t*>(buf) + qbytes);
    }
    int st = sherry_quant_act(x, M, K, x_i8, x_scale, stream);
    if (st != SHERRY_OK) return st;
    return sherry_gemm_acc(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, stream);
}

int sherry_linear(const float* x, const void* Wnative, const float* alpha, float* y, int64_t M, int64_t N,
                  int64_t K, void* stream)
{
    if (!y) return SHERRY_ERR_INVALID_ARG;
    return sherry_linear_ex(x, Wnative, alpha, y, nullptr, nullptr, nullptr, M, N, K, stream);
}

int sherry_gemm_tc(const int8_t* x_i8, const float* x_scale, const void* Wnative, const float* alpha, float* y,
                   int32_t* acc, int64_t M, int64_t N, int64_t K, void* stream)
{
    int st = check_gemm_args(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K);
    if (st != SHERRY_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M <= 16) return launch_tc<16, 4>(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, s);
    if (M <= 32) return launch_tc<32, 4>(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, s);
    if (M <= 64) return launch_tc<64, 4>(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, s);
    // 192-token tiles decode each weight tile for 1.5x the tokens; measured
    // faster from M ~ 1536 on (M=2048: 115.5 -> 111.5 us, M=8192: 407 -> 380
    // us at K=4096, N=14336), slower where their padding is large (M=1024).
    // One-chunk stages: four A slots and three decoder groups beat two-chunk
    // stages with two (M=8192: 398 -> 380 us, K=14336 -> N=4096: 99 -> 96.5).
    if (M < 1536) return launch_tc<128, 2>(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, s);
    return launch_tc<192, 1>(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, s);
}

int sherry_gemm_gemv(const int8_t* x_i8, const float* x_scale, const void* Wnative, const float* alpha, float* y,
                     int32_t* acc, int64_t M, int64_t N, int64_t K, void* stream)
{
    int st = check_gemm_args(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K);
    if (st != SHERRY_OK) return st;
    if (M > SHERRY_GEMV_MAX_M || sherry_k_chunks(K) > (int64_t)gemv::kMaxSL * gemv::kMaxNS)
        return SHERRY_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (M == 1) return launch_gemv<1>(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, s);
    if (M == 2) return launch_gemv<2>(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, s);
    return launch_gemv<4>(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, s);
}

int sherry_gemm(const int8_t* x_i8, const float* x_scale, const void* Wnative, const float* alpha, float* y,
                int64_t M, int64_t N, int64_t K, void* stream)
{
    if (!y) return SHERRY_ERR_INVALID_ARG;
    return sherry_gemm_acc(x_i8, x_scale, Wnative, alpha, y, nullptr, M, N, K, stream);
}

int sherry_gemm_simt(const int8_t* x_i8, const float* x_scale, const void* Wnative, const float* alpha, float* y,
                     int32_t* acc, int64_t M, int64_t N, int64_t K, void* stream)
{
    int st = check_gemm_args(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K);
    if (st != SHERRY_OK) return st;
    DeviceInfo di;
    st = device_info(&di);
    if (st != SHERRY_OK) return st;
    dim3 grid((unsigned)sherry_row_tiles(N), (unsigned)((M + kSimtMT - 1) / kSimtMT));
    if ((M + kSimtMT - 1) / kSimtMT > 65535) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    simt_gemm_kernel<<<grid, SHERRY_TILE_ROWS, 0, static_cast<cudaStream_t>(stream)>>>(
        x_i8, x_scale, static_cast<const uint32_t*>(Wnative), alpha, y, acc, M, N, K);
    return cuda_status(cudaGetLastError());
}

int sherry_gemm_noalloc(const int8_t* x_i8, const float* x_scale, const void* Wnative, const float* alpha,
                        float* y, int32_t* acc, int64_t M, int64_t N, int64_t K, void* stream)
{
    int st = check_gemm_args(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K);
    if (st != SHERRY_OK) return st;
    if (M > kNoAllocMaxBN) return SHERRY_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // the decode kernel needs no workspace at all: the same choice as sherry_gemm
    if (M <= SHERRY_GEMM_DECODE_AUTO_MAX_M) {
        DeviceInfo di;
        st = device_info(&di);
        if (st != SHERRY_OK) return st;
        decode::Plan pl;
        if (decode::plan(N, sherry_k_chunks(K), M, di.sms, &pl))
            return sherry_gemm_decode(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, stream);
    }
    if (M <= 16) return launch_tc_noalloc<16, 4>(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, s);
    return launch_tc_noalloc<32, 4>(x_i8, x_scale, Wnative, alpha, y, acc, M, N, K, s);
}

int sherry_selftest_wait(uint64_t limit_ns, void* stream)
{
    if (limit_ns == 0 || limit_ns > 1000000000ull) return SHERRY_ERR_INVALID_ARG;
    DeviceInfo di;
    int st = device_info(&di);
    if (st != SHERRY_OK) return st;
    unsigned* status = device_status_ptr();
    if (!status) return SHERRY_ERR_CUDA;
    wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, status);
    return cuda_status(cudaGetLastError());
}

size_t sherry_workspace_bytes(int64_t max_M, int64_t max_K)
{
    if (max_M < 1 || max_K < 1) return 0;
    DeviceInfo di;
    if (device_info(&di) != SHERRY_OK) return 0;
    return tc_workspace_bytes(max_M, di.sms) + act_buffer_bytes(max_M, max_K);
}

int sherry_reserve(int64_t max_M, int64_t max_K)
{
    if (max_M < 1 || max_K < 1 || max_M > SHERRY_MAX_DIM || max_K > SHERRY_MAX_K) return SHERRY_ERR_INVALID_ARG;
    DeviceInfo di;
    int st = device_info(&di);
    if (st != SHERRY_OK) return st;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SHERRY_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mutex);
    if ((int)g_ws.size() <= dev) g_ws.resize(dev + 1);
    if ((int)g_act.size() <= dev) g_act.resize(dev + 1);
    st = grow_buffer(g_ws[dev], tc_workspace_bytes(max_M, di.sms));
    if (st != SHERRY_OK) return st;
    return grow_buffer(g_act[dev], act_buffer_bytes(max_M, max_K));
}

int sherry_last_device_status(int reset)
{
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return -1;
    if (reset) {
        // A launch whose bounded wait ran out may have left split-K partial
        // sums and arrival counters behind: the workspace of this device is
        // zeroed again before the next call can use it.
        if (v != 0) {
            int dev = 0;
            if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) return -1;
            std::lock_guard<std::mutex> lk(g_mutex);
            if ((int)g_ws.size() > dev && g_ws[dev].ptr &&
                (cudaMemset(g_ws[dev].ptr, 0, g_ws[dev].bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess))
                return -1;
        }
        unsigned z = 0;
        if (cudaMemcpyToSymbol(g_device_status, &z, sizeof(z)) != cudaSuccess) return -1;
    }
    return (int)v;
}

}  // extern "C"
