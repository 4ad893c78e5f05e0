/*
 * sherry.h -- C ABI of libsherry_b200.so: the Sherry 3:4 ternary-weight matmul
 * on NVIDIA B200 (sm_100a).
 *
 * The method (Sherry page, pnsm.cn/news/1195499, "Sherry framework: ternary
 * quantisation and 3:4 sparsity for LLM inference"):
 *   - sec. 3.1: every group of 4 consecutive weights along K is replaced by
 *     T in {-1,0,+1}^4 with exactly 3 nonzeros -- the 3 largest |w| keep
 *     their signs -- times a least-squares scale alpha (one per output row n);
 *   - sec. 2.1: each group is stored as one 5-bit code (1.25 bit/weight);
 *   - sec. 2.2: activations are integers, the contraction is additions and
 *     subtractions accumulated exactly, followed by float scaling.
 *
 * Data conventions (all row-major):
 *   W      fp32 [N][K]      output feature n is row n (Linear.weight layout)
 *   x      fp32 [M][K]      M tokens
 *   x_i8   int8 [M][K]      quantised activations, x_scale fp32 [M]
 *   y      fp32 [M][N]      y[m][n] = (float)((float)acc[m][n] * alpha[n]) * x_scale[m]
 *   acc    int32 [M][N]     acc[m][n] = sum_k x_i8[m][k] * T[n][k]  (exact)
 *
 * Canonical code of a group (z = position of the zero, s_j = 1 when the j-th
 * kept weight in ascending position is negative):
 *     code = z | s0 << 2 | s1 << 3 | s2 << 4
 * Canonical stream: row n starts at byte n * (5K/32); code g occupies stream
 * bits [5g, 5g+5), least significant bit first (bit b is bit b%8 of byte b/8).
 *
 * Shape rules: M, N, K >= 1 and K % 32 == 0 (rows of whole bytes).
 *
 * Ownership: the caller owns every buffer passed in.  Host functions take host
 * pointers; device functions take device pointers and a cudaStream_t passed
 * as void* (NULL = legacy default stream).  Device functions are asynchronous
 * on that stream: none of them allocates, frees or synchronises.  The device
 * memory the library owns is, per device:
 *   - the workspace set aside by sherry_reserve (host, synchronous): the
 *     split-K partial sums and arrival counters of the tensor-core kernel,
 *     all zero between calls, and the int8 activations and scales that
 *     sherry_linear uses when the caller passes none.  A call that needs more
 *     than was reserved returns SHERRY_ERR_WORKSPACE and launches nothing;
 *   - the fixed scratch array of sherry_gemm_noalloc and the device status
 *     word, both in the library's own device image.
 * Calls that use the reserved workspace share it: calls that may run at the
 * same time on different streams of one device must not be issued
 * (serialise them on one stream or with events).
 *
 * Errors: every function returns a sherry_status.  Argument errors are
 * reported before anything is launched.  SHERRY_ERR_CUDA means a CUDA call
 * (launch, copy, allocation) failed; the CUDA error is then also left for
 * cudaGetLastError.  Kernels never trap: a wait that exceeds its bound sets a
 * device status word (read with sherry_last_device_status) and the kernel
 * returns.
 */
#ifndef SHERRY_H
#define SHERRY_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SHERRY_OK = 0,
    SHERRY_ERR_INVALID_ARG = 1,       /* null pointer, non-positive size, misaligned pointer */
    SHERRY_ERR_UNSUPPORTED_SHAPE = 2, /* K % 32 != 0, or a size beyond the int32 index range */
    SHERRY_ERR_NONFINITE = 3,         /* NaN or Inf in W (sherry_pack) */
    SHERRY_ERR_CUDA = 4,              /* a CUDA runtime call failed */
    SHERRY_ERR_DEVICE = 5,            /* the device is not sm_100 or lacks a needed feature */
    SHERRY_ERR_WORKSPACE = 6          /* the call needs more workspace than sherry_reserve set aside */
} sherry_status;

/* Short English text for a status value; never NULL. */
const char* sherry_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
int sherry_version(void);

/* Bytes of the canonical code stream for an N x K weight: N * K * 5 / 32
 * (sec. 2.1, 1.25 bit/weight).  Returns 0 for invalid shapes. */
size_t sherry_packed_bytes(int64_t N, int64_t K);

/* Bytes of the kernel-native layout written by sherry_repack and read by
 * sherry_gemm: rows padded to a multiple of 128 and K to a multiple of 128,
 * 20 bytes per (row, 128-wide K chunk).  Returns 0 for invalid shapes. */
size_t sherry_native_bytes(int64_t N, int64_t K);

/*
 * sherry_pack -- host, synchronous.  Offline ternarisation and packing
 * (sec. 3.1 objective, sec. 2.1 encoding).
 *   W      [in]  fp32 [N][K], host memory, finite values only
 *   codes  [out] uint8 [N][5K/32], host memory (canonical stream)
 *   alpha  [out] fp32 [N], host memory: sum of kept |w| (fp64, ascending k)
 *                / (0.75 K), rounded once to fp32
 * Per group the smallest |w| is zeroed (lowest index on ties); kept weights
 * keep their sign (w < 0 is negative, so -0.0 counts as +).
 * Returns SHERRY_ERR_NONFINITE (outputs unspecified) if W holds NaN or Inf.
 * Uses the host's cores (OpenMP over rows); results do not depend on the
 * number of threads.
 */
int sherry_pack(const float* W, int64_t N, int64_t K, uint8_t* codes, float* alpha);

/*
 * sherry_unpack -- host, synchronous.  Canonical codes -> T int8 [N][K] in
 * {-1,0,+1} (exactly 3 nonzeros per group).  Every 5-bit value is a valid
 * code, so any byte stream decodes.
 */
int sherry_unpack(const uint8_t* codes, int64_t N, int64_t K, int8_t* T);

/*
 * sherry_repack -- device, asynchronous on `stream`.  Rearranges a canonical
 * code stream already copied to the device into the kernel-native layout
 * (same codes, tile-interleaved so that 128 consecutive rows of one 128-wide
 * K chunk are one contiguous 2560-byte block).  Inside a block, word j
 * (canonical bytes [20c+4j, 20c+4j+4) of the row, little endian) of row r
 * sits at 32-bit index 128 j + ((r + 8 j) mod 128): five word planes, plane
 * j rotated by 8 j rows so that the kernels' shared-memory reads of it are
 * free of bank conflicts.
 *   codes_dev  [in]  uint8 [N][5K/32], device memory
 *   native_dev [out] sherry_native_bytes(N, K) bytes, device memory, 16-byte aligned
 * Padding bytes are written as zero.
 */
int sherry_repack(const uint8_t* codes_dev, int64_t N, int64_t K, void* native_dev,
                  void* stream);

/*
 * sherry_quant_act -- device, asynchronous.  Per-token int8 activation
 * quantisation (sec. 2.2 step 1 leaves the rule open; this is symmetric
 * absmax/127 with round-half-to-even and IEEE fp32 division):
 *   a = max_k |x[m][k]|;  x_scale[m] = a / 127;
 *   x_i8[m][k] = clamp(rint(x[m][k] / x_scale[m]), -127, 127);
 *   a == 0 gives x_scale[m] = 0 and a zero row.
 *   x       [in]  fp32 [M][K], device memory, 16-byte aligned
 *   x_i8    [out] int8 [M][K], device memory, 16-byte aligned
 *   x_scale [out] fp32 [M], device memory
 * NaN or Inf in x gives unspecified values (no error is reported).
 */
int sherry_quant_act(const float* x, int64_t M, int64_t K, int8_t* x_i8, float* x_scale,
                     void* stream);

/* Largest M of the table-lookup GEMV kernel, sherry_gemm_gemv. */
#define SHERRY_GEMV_MAX_M 4
/* Largest M of the decode kernel, sherry_gemm_decode. */
#define SHERRY_DECODE_MAX_M 8
/* Largest M for which sherry_gemm chooses the decode kernel: measured on
 * B200 over the (4096,4096), (4096,14336), (14336,4096) projections, the
 * tensor-core kernel is faster from M = 3 on. */
#define SHERRY_GEMM_DECODE_AUTO_MAX_M 2
/* Largest M for which sherry_linear is a single fused launch (quantiser and
 * decode kernel); from M = 2 on the two-launch path measured faster. */
#define SHERRY_LINEAR_FUSED_MAX_M 1

/*
 * sherry_gemm -- device, asynchronous.  y = epilogue(x_i8 . T^T) (sec. 2.2
 * steps 2-4): exact int32 accumulation, then
 * y[m][n] = (float)((float)acc * alpha[n]) * x_scale[m].
 * M <= SHERRY_GEMM_DECODE_AUTO_MAX_M runs sherry_gemm_decode (when a CTA's
 * share of the codes fits in shared memory, i.e. K up to about 600000
 * weights), any other shape sherry_gemm_tc (tensor cores); all kernels give
 * identical results.
 *   x_i8     [in]  int8 [M][K], device memory, 16-byte aligned
 *   x_scale  [in]  fp32 [M], device memory
 *   Wnative  [in]  kernel-native codes from sherry_repack, device memory, 16-byte aligned
 *   alpha    [in]  fp32 [N], device memory
 *   y        [out] fp32 [M][N], device memory
 * Uses the workspace set aside by sherry_reserve when its tensor-core launch
 * splits a tile over several CTAs (SHERRY_ERR_WORKSPACE when too small).
 */
int sherry_gemm(const int8_t* x_i8, const float* x_scale, const void* Wnative,
                const float* alpha, float* y, int64_t M, int64_t N, int64_t K, void* stream);

/*
 * sherry_gemm_acc -- as sherry_gemm, and also writes the exact int32
 * accumulators acc[M][N] (device memory) when acc != NULL.  y may be NULL
 * when only acc is wanted.
 */
int sherry_gemm_acc(const int8_t* x_i8, const float* x_scale, const void* Wnative,
                    const float* alpha, float* y, int32_t* acc, int64_t M, int64_t N,
                    int64_t K, void* stream);

/*
 * sherry_gemm_tc -- device, asynchronous.  The contraction on the tensor
 * cores for any M: the ternary weights are decoded from the 5-bit codes
 * into tensor memory (one 32-bit cell per group of 4) and multiplied with
 * tcgen05.mma kind::i8 against the int8 activations (TMA-loaded, 128-byte
 * swizzle); K is split over all SMs with exact int32 partial sums in the
 * per-device workspace.  Launched with programmatic dependent launch: the
 * codes of each CTA's first pipeline round are copied before the previous
 * kernel on the stream ends; activations, scales and outputs are touched
 * only after it completed.  So, as for sherry_gemm_decode, Wnative must not
 * be written by the kernel launched just before on the same stream unless
 * that kernel ends without triggering its dependents early (every ordinary
 * kernel, and sherry_repack, does so).  Arguments as sherry_gemm_acc.
 */
int sherry_gemm_tc(const int8_t* x_i8, const float* x_scale, const void* Wnative,
                   const float* alpha, float* y, int32_t* acc, int64_t M, int64_t N,
                   int64_t K, void* stream);

/*
 * sherry_gemm_decode -- device, asynchronous.  The decode kernel for
 * M <= SHERRY_DECODE_MAX_M tokens, on the CUDA cores.  One CTA per SM owns a
 * balanced range of whole output rows over the full K: its codes are
 * streamed into shared memory, each 5-bit code becomes four int8 weights in
 * {-1,0,+1} through a 32-entry table, and dp4a adds them against the int8
 * activations; partial sums of a row never leave the CTA (no workspace, no
 * atomics).  Launched with programmatic dependent launch: the weight copy
 * starts before the previous kernel on the stream ends; activations are
 * read only after it completed, so Wnative and alpha must not be written by
 * the kernel launched just before on the same stream unless that kernel
 * ends without triggering its dependents early (every ordinary kernel, and
 * sherry_repack, does so).  Returns SHERRY_ERR_UNSUPPORTED_SHAPE for M > 8
 * or when one row's codes do not fit in shared memory.  Arguments as
 * sherry_gemm_acc.
 */
int sherry_gemm_decode(const int8_t* x_i8, const float* x_scale, const void* Wnative,
                       const float* alpha, float* y, int32_t* acc, int64_t M, int64_t N,
                       int64_t K, void* stream);

/*
 * sherry_linear -- device, asynchronous.  The whole online step of the page
 * (sec. 2.2 steps 1-4) from fp32 activations: the sherry_quant_act rule
 * followed by the sherry_gemm contraction and epilogue, with bit-identical
 * results.  For M <= SHERRY_LINEAR_FUSED_MAX_M (one token) it is one launch
 * of the decode kernel that also quantises (every CTA reads the whole
 * activation row, takes its absmax and quantises it into its shared memory).
 * Other shapes run sherry_quant_act into x_i8 / x_scale (sherry_linear_ex),
 * or into the activation buffer that sherry_reserve set aside, and then
 * sherry_gemm.
 *   x        [in]  fp32 [M][K], device memory, 16-byte aligned
 *   Wnative  [in]  kernel-native codes, device memory, 16-byte aligned
 *   alpha    [in]  fp32 [N], device memory
 *   y        [out] fp32 [M][N], device memory
 * Concurrency as sherry_gemm.  (The page describes these steps as one
 * inference pass; the single entry point is this library's.)
 */
int sherry_linear(const float* x, const void* Wnative, const float* alpha, float* y,
                  int64_t M, int64_t N, int64_t K, void* stream);

/*
 * sherry_linear_ex -- as sherry_linear, with optional outputs: acc int32
 * [M][N], and x_i8 int8 [M][K] (16-byte aligned) with x_scale fp32 [M], the
 * quantised activations (both or neither; when given they are also used
 * instead of the library's buffer).  y may be NULL when acc is given.
 */
int sherry_linear_ex(const float* x, const void* Wnative, const float* alpha, float* y,
                     int32_t* acc, int8_t* x_i8, float* x_scale, int64_t M, int64_t N,
                     int64_t K, void* stream);

/*
 * sherry_gemm_gemv -- device, asynchronous.  Decode GEMV for M <= 
 * SHERRY_GEMV_MAX_M tokens on the CUDA cores, following the page's
 * inference scheme (sec. 2.2): per 4-element activation segment a table of
 * its dot products with all 32 ternary groups is built in shared memory;
 * each weight group then costs one table lookup and one add.  Launched with
 * programmatic dependent launch (it may start before the previous kernel on
 * the stream ends; it reads activations only after that kernel completed).
 * The K-slices of a 128-row tile run as one thread-block cluster and are
 * summed exactly through distributed shared memory (no workspace).  M > 4
 * or K > 16384 returns SHERRY_ERR_UNSUPPORTED_SHAPE.  sherry_gemm does not
 * dispatch to it; it is the page's own scheme, kept for comparison with
 * sherry_gemm_decode.  Arguments as sherry_gemm_acc.
 */
int sherry_gemm_gemv(const int8_t* x_i8, const float* x_scale, const void* Wnative,
                     const float* alpha, float* y, int32_t* acc, int64_t M, int64_t N,
                     int64_t K, void* stream);

/*
 * sherry_gemm_simt -- device, asynchronous.  The same contraction and
 * epilogue on the CUDA cores (shared-memory code table + dp4a), kept as an
 * independent second kernel for A/B comparison.  Same arguments as
 * sherry_gemm_acc; needs no workspace.
 */
int sherry_gemm_simt(const int8_t* x_i8, const float* x_scale, const void* Wnative,
                     const float* alpha, float* y, int32_t* acc, int64_t M, int64_t N,
                     int64_t K, void* stream);

/*
 * sherry_gemm_noalloc -- device, asynchronous.  The same contraction and
 * epilogue as sherry_gemm_acc, for callers that must not allocate device
 * memory once they are running: programs whose device memory is handed out
 * by their own pool sized at start-up, or whose request loop may not make
 * the synchronising cudaMalloc/cudaFree calls.  (This entry point is an
 * addition of this library; the Sherry page has no counterpart.)
 * Instead of the per-device workspace of sherry_gemm, it uses a fixed
 * scratch array compiled into the library: 2.6 MB, reserved on every GPU
 * that loads the library until the process exits.  It therefore serves
 * decode shapes only: M <= 32 tokens, otherwise SHERRY_ERR_UNSUPPORTED_SHAPE
 * is returned before anything is launched.  For M <=
 * SHERRY_GEMM_DECODE_AUTO_MAX_M it runs the decode kernel, which needs no
 * scratch at all, as sherry_gemm would.  It calls no cudaMalloc or
 * cudaFree.  Each call first clears (cudaMemsetAsync on `stream`) the part
 * of the scratch it uses.
 * The first call on a device looks up the scratch's device address with that
 * device current; make that first call before any stream capture.
 * All calls share the one scratch array: calls that may overlap on the GPU
 * (different streams without ordering between them) race and give wrong
 * results.  Arguments as sherry_gemm_acc.
 */
int sherry_gemm_noalloc(const int8_t* x_i8, const float* x_scale, const void* Wnative,
                        const float* alpha, float* y, int32_t* acc, int64_t M, int64_t N,
                        int64_t K, void* stream);

/* ===========================================================================
 * W4A8 FastGEMM -- the second workload of this library: per-channel SINT4
 * weights times int8 activations on the same tcgen05 kernel.
 * (OdysseyLLM review page, xllm-io.github.io/paper-review/blog/odysseyllm,
 * "OdysseyLLM: A Speed Odyssey for Deployable Quantization of LLMs".)
 *   - sec. 3.3: symmetric per-channel weight scale
 *     S[n] = max(|max_k W[n][k]|, |min_k W[n][k]|) / 7, and
 *     W_q = clamp(rint(W / S), -8, 7) (fp32 IEEE division, ties to even).
 *     The page's learnable clipping factors are taken as 1.  S = 0 and
 *     W_q = 0 for an all-zero row.
 *   - sec. 3.2 / 5.2: SINT4toS8.  The 4-bit two's complement value becomes
 *     the int8 value 16 w by moving it into the high half of a byte.  An
 *     int8 GEMM sums q * 16 w exactly in int32.
 *   - sec. 3.1 (Figure 2, the W4A8 row): those sums are divided by 16
 *     (exact) before dequantisation:
 *         acc[m][n] = (sum_k x_i8[m][k] * 16 W_q[n][k]) / 16
 *         y[m][n]   = (float)((float)acc[m][n] * S[n]) * x_scale[m]
 * Activations come from sherry_quant_act (per-token absmax / 127).
 * Canonical SINT4 rows: row n starts at byte n * K/2; byte j holds W_q[n][2j]
 * in bits 0-3 and W_q[n][2j+1] in bits 4-7 (two's complement nibbles).
 * Shape rules: those of the Sherry path, and K <= 132104 (so K <= 132096
 * with K % 32 == 0) so that
 * |sum q * 16 w| <= 127 * 128 * K stays below 2^31.
 * =========================================================================== */

/* Bytes of canonical SINT4 rows: N * K/2; 0 when (N, K) is not supported. */
size_t sherry_w4a8_packed_bytes(int64_t N, int64_t K);
/* Bytes of the kernel-native SINT4 layout written by sherry_w4a8_repack:
 * ceil(N/128) * ceil(K/128) * 8192; 0 when (N, K) is not supported. */
size_t sherry_w4a8_native_bytes(int64_t N, int64_t K);

/*
 * sherry_w4a8_pack -- host, synchronous.  Quantises W (sec. 3.3 above) and
 * packs it into canonical SINT4 rows.
 *   W      [in]  fp32 [N][K], host memory
 *   w4     [out] sherry_w4a8_packed_bytes(N, K) bytes, host memory
 *   scale  [out] fp32 [N] per-channel scales S, host memory
 * Returns SHERRY_ERR_NONFINITE (nothing written) when W holds a NaN or Inf,
 * SHERRY_ERR_UNSUPPORTED_SHAPE for K % 32 != 0 or K > 132104.
 */
int sherry_w4a8_pack(const float* W, int64_t N, int64_t K, uint8_t* w4, float* scale);

/* sherry_w4a8_unpack -- host, synchronous.  Canonical SINT4 rows -> int8
 * W_q [N][K] with values in [-8, 7] (tests and inspection). */
int sherry_w4a8_unpack(const uint8_t* w4, int64_t N, int64_t K, int8_t* Wq);

/*
 * sherry_w4a8_repack -- device, asynchronous on `stream`.  Rearranges
 * canonical SINT4 rows into the layout sherry_w4a8_gemm reads.  Run it once
 * per weight matrix; the output does not depend on the GPU.
 *   w4_dev     [in]  canonical rows, device memory
 *   native_dev [out] sherry_w4a8_native_bytes(N, K) bytes, device memory,
 *                    16-byte aligned
 */
int sherry_w4a8_repack(const uint8_t* w4_dev, int64_t N, int64_t K, void* native_dev,
                       void* stream);

/* Largest M the CUDA-core GEMV (sherry_w4a8_gemm_gemv) serves. */
#define SHERRY_W4A8_GEMV_MAX_M 4

/*
 * sherry_w4a8_gemm_acc -- device, asynchronous.  The W4A8 contraction and
 * dequantisation above, for every M on the tensor-core kernel
 * (sherry_w4a8_gemm_tc; it measured faster than the GEMV at M = 1 and 4).
 *   x_i8, x_scale  [in]  from sherry_quant_act, device memory (x_i8 16-byte aligned)
 *   W4native       [in]  from sherry_w4a8_repack, device memory, 16-byte aligned
 *   scale          [in]  fp32 [N] per-channel S from sherry_w4a8_pack, device memory
 *   y              [out] fp32 [M][N] or NULL
 *   acc            [out] int32 [M][N] (the sums after the division by 16) or NULL
 * At least one of y and acc must be non-NULL.  The tensor-core kernel uses
 * the split-K workspace described at the top of this file.
 */
int sherry_w4a8_gemm_acc(const int8_t* x_i8, const float* x_scale, const void* W4native,
                         const float* scale, float* y, int32_t* acc, int64_t M, int64_t N,
                         int64_t K, void* stream);

/*
 * sherry_w4a8_gemm_tc -- device, asynchronous.  The same, on the tcgen05
 * tensor-core kernel for every M.  The SINT4toS8 conversion runs in the
 * kernel's decoder warps, between the shared-memory copy of the weights and
 * the tensor memory the MMAs read.  Arguments as sherry_w4a8_gemm_acc.
 */
int sherry_w4a8_gemm_tc(const int8_t* x_i8, const float* x_scale, const void* W4native,
                        const float* scale, float* y, int32_t* acc, int64_t M, int64_t N,
                        int64_t K, void* stream);

/*
 * sherry_w4a8_gemm_gemv -- device, asynchronous.  The same, for M <=
 * SHERRY_W4A8_GEMV_MAX_M, on the CUDA cores (a comparison kernel: the
 * default path is the tensor-core kernel).  A CTA owns 32 rows and splits
 * K among its warps; the shift into int8 and dp4a run in registers.  Larger
 * M returns SHERRY_ERR_UNSUPPORTED_SHAPE.  Needs no workspace.  Arguments as
 * sherry_w4a8_gemm_acc.
 */
int sherry_w4a8_gemm_gemv(const int8_t* x_i8, const float* x_scale, const void* W4native,
                          const float* scale, float* y, int32_t* acc, int64_t M, int64_t N,
                          int64_t K, void* stream);

/* sherry_w4a8_gemm -- sherry_w4a8_gemm_acc without the int32 output (y required). */
int sherry_w4a8_gemm(const int8_t* x_i8, const float* x_scale, const void* W4native,
                     const float* scale, float* y, int64_t M, int64_t N, int64_t K,
                     void* stream);

/*
 * sherry_selftest_wait -- device, asynchronous.  A check of failure
 * detection (no counterpart on the page): one warp waits, with the bounded
 * wait every kernel of the library uses, for an mbarrier phase that nothing
 * completes.  After limit_ns nanoseconds of wall time (1 to 10^9) the wait
 * gives up, the kernel records 0x107 in the device status word (read with
 * sherry_last_device_status) and returns; the context stays usable.  No
 * copy is in flight and no tensor memory is held when it gives up.
 */
int sherry_selftest_wait(uint64_t limit_ns, void* stream);

/*
 * sherry_workspace_bytes -- host.  Device bytes that sherry_reserve(max_M,
 * max_K) sets aside on the current device: the tensor-core kernel's split-K
 * slots (one per SM, the token tile of max_M tokens x 128 rows of int32)
 * and counters, plus max_M x max_K int8 activations and max_M scales for
 * sherry_linear.  0 for non-positive sizes or an unsupported device.
 */
size_t sherry_workspace_bytes(int64_t max_M, int64_t max_K);

/*
 * sherry_reserve -- host, synchronous.  Sets aside, on the current device,
 * the workspace of every later call with M <= max_M and K <= max_K (any N):
 * sherry_gemm, sherry_gemm_acc, sherry_gemm_tc, sherry_linear(_ex) and the
 * W4A8 tensor-core entry points.  Grows what an earlier call reserved (never
 * shrinks it); when it grows it first waits for the device to be idle, then
 * frees the old buffer, allocates and zero-fills the new one.  Call it before
 * capturing a stream into a CUDA graph and before timing.  The asynchronous
 * entry points never allocate: without enough workspace they return
 * SHERRY_ERR_WORKSPACE.  Calls whose tensor-core launch splits no tile over
 * several CTAs, the decode kernel (M <= SHERRY_DECODE_MAX_M), the fused
 * sherry_linear launch and sherry_gemm_noalloc need no workspace.
 */
int sherry_reserve(int64_t max_M, int64_t max_K);

/*
 * sherry_last_device_status -- host, synchronous (copies one word from the
 * current device).  0 when no kernel of this library has reported a bounded
 * wait running out since the last reset; otherwise a nonzero code naming the
 * wait.  reset != 0 clears it; when the word was nonzero the reset also waits
 * for the device to be idle and zero-fills the reserved workspace again,
 * since a launch that gave up may have left partial sums and arrival
 * counters in it.  After a nonzero status, reset it before the next call.
 */
int sherry_last_device_status(int reset);

#ifdef __cplusplus
}
#endif

#endif /* SHERRY_H */
