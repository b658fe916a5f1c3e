/*
 * wq.h -- C ABI of libwq.so: weight-only integer-quantised GEMM for NVIDIA
 * B200 (sm_100a).
 *
 * Weights W (fp16, [N, K] row-major, the nn.Linear layout) are stored as b-bit
 * integer codes (b = 2, 3, 4 or 8) on the uniform asymmetric min-max grid, one
 * grid per row or per group of `group` consecutive input columns:
 *
 *   lo = min(0, min w), hi = max(0, max w)           over the row / group
 *   scale = fp16_rne((hi - lo) / (2^b - 1))          (1.0 if that rounds to 0)
 *   zero  = rint(-lo / scale)                        (0 when scale was 0)
 *   q     = clamp(rint(w / scale) + zero, 0, 2^b - 1)   rint: half to even
 *   w'    = scale * (q - zero)
 *
 * Sources: "OPTQ: Accurate Quantization for Generative Pre-trained
 * Transformers" (reproducibility summary, row "Experiment Setup": uniform
 * per-row asymmetric quantisation on the min-max grid); "Platform For AI:
 * BladeLLM model quantization" (section "block_wise_quant": one parameter set
 * per block of input channels; section "Quantization algorithms > MinMax":
 * round to nearest, no calibration data).  The range always containing 0, the
 * half-to-even rounding, the fp16 rounding of the scale and the degenerate
 * scale rule are this library's readings of what those pages leave open.
 *
 * Packed code layout ("[Feature Request] 4bit and 2bit and 1bit quantization
 * support", onnxruntime issue 14997: several low-bit codes per machine word):
 * codes are uint32 [N, K*b/32] row-major, least-significant bits first along K.
 *   b = 2, 4, 8: code k of a row is in word k/(32/b) at bit b*(k mod 32/b)
 *                (16, 8, 4 codes per word);
 *   b = 3:       the 32 codes of unit u = k/32 fill the 96-bit little-endian
 *                value of words 3u, 3u+1, 3u+2; code j = k mod 32 sits at bit 3j
 *                (codes 10 and 21 of each unit straddle two words).
 * Scales and zeros are fp16 [N, G] row-major, G = K/group (G = 1 per row);
 * every zero is a non-negative integer, exact in fp16.
 *
 * Common rules for the compute calls:
 *   - every pointer is a DEVICE pointer on the current CUDA device, 16-byte
 *     aligned; the caller allocates and owns every buffer, the library never
 *     allocates, frees or keeps a pointer after the call returns;
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream); the work
 *     is enqueued on it and the call returns without synchronising;
 *   - `group` is 0 or K (one grid per row), or a multiple of 32 dividing K;
 *   - K must be a multiple of 32; M, N, K >= 1;
 *   - arguments are checked before anything is launched; on any non-OK status
 *     nothing is launched and no output byte is written;
 *   - WQ_ERR_CUDA reports a launch error (the CUDA error is left for
 *     cudaGetLastError to read);
 *   - W must be finite (not checked).
 */
#ifndef WQ_H
#define WQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  WQ_OK = 0,
  WQ_ERR_NULL = 1,                /* a required pointer is NULL */
  WQ_ERR_BITS = 2,                /* bits not in {2, 3, 4, 8} */
  WQ_ERR_GROUP = 3,               /* group not 0, K, or a multiple of 32 dividing K */
  WQ_ERR_SHAPE = 4,               /* M, N or K < 1, K not a multiple of 32, or too large */
  WQ_ERR_ALIGN = 5,               /* a pointer is not 16-byte aligned */
  WQ_ERR_UNSUPPORTED_DEVICE = 6,  /* current device is not compute capability 10.0 */
  WQ_ERR_CUDA = 7,                /* a CUDA runtime call or launch failed */
  WQ_ERR_DEVICE_TIMEOUT = 8,      /* a bounded device-side wait expired (see below) */
  WQ_ERR_WORKSPACE = 9            /* workspace NULL or smaller than the call needs */
} wq_status;

/*
 * wq_quantize_rtn -- round-to-nearest quantisation and packing of W.
 * (Grid: OPTQ page, "Experiment Setup"; groups: BladeLLM page,
 * "block_wise_quant"; rounding: BladeLLM page, "Quantization algorithms >
 * MinMax".)
 *
 *   W_f16      in   fp16 [N, K] row-major
 *   N, K            rows (outputs) and columns (inputs)
 *   bits            2, 3, 4 or 8
 *   group           0 or K (per row), or a multiple of 32 dividing K
 *   codes      out  uint32 [N, wq_codes_words(N, K, bits) / N], layout above
 *   scales_f16 out  fp16 [N, G]
 *   zeros_f16  out  fp16 [N, G]
 *   stream          cudaStream_t
 *
 * Results are bit-exact: codes, scales and zeros are the unique values the
 * grid definition above gives (fp64 scale rounding, IEEE fp32 division and
 * half-to-even rint for zero and codes).
 */
wq_status wq_quantize_rtn(const void* W_f16, int64_t N, int64_t K, int bits, int64_t group,
                          uint32_t* codes, void* scales_f16, void* zeros_f16, void* stream);

/*
 * wq_quantize_rtn_sym -- round-to-nearest quantisation on the symmetric grid
 * ("Platform For AI: BladeLLM model quantization", "Quantization modes >
 * weight_only_quant": signed symmetric quantisation is the default; groups as
 * in "block_wise_quant").  Per row or group:
 *
 *   a = max |w|,  scale = fp16_rne(a / (2^(b-1) - 1))  (1.0 if that rounds to 0)
 *   zero = 2^(b-1) (fixed, not stored)
 *   q = clamp(rint(w / scale) + 2^(b-1), 0, 2^b - 1),   w' = scale * (q - 2^(b-1))
 *
 * so +-a map to the signed codes +-(2^(b-1) - 1).  Arguments as for
 * wq_quantize_rtn, without zeros_f16.  Pass zeros_f16 = NULL to wq_gemm and
 * wq_gemm_grouped for codes written by this call.  Bit-exact like
 * wq_quantize_rtn (the scale divisor 2^(b-1) - 1 is this library's reading).
 */
wq_status wq_quantize_rtn_sym(const void* W_f16, int64_t N, int64_t K, int bits, int64_t group,
                              uint32_t* codes, void* scales_f16, void* stream);

/*
 * wq_gemm -- y = x . W'^T with W' dequantised on the fly from the codes.
 * (Dequantise-in-the-matmul: onnxruntime issue 14997, weights kept in 4 bit and
 * converted to float when used; BladeLLM page, "Background information >
 * Solutions" and "Quantization modes > weight_only_quant": low-bit weights cut
 * the bytes moved from GPU memory, the bound in memory-limited decoding.)
 *
 *   x_bf16     in   bf16 [M, K] row-major
 *   M, N, K         batch rows, output features, input features
 *   codes      in   packed codes as written by wq_quantize_rtn
 *   scales_f16 in   fp16 [N, G]
 *   zeros_f16  in   fp16 [N, G], or NULL for the symmetric grid of
 *                   wq_quantize_rtn_sym (every zero 2^(bits-1))
 *   bits, group     as given to wq_quantize_rtn
 *   y_bf16     out  bf16 [M, N] row-major; must not overlap the inputs
 *   stream          cudaStream_t
 *
 * Products and sums are fp32; y is rounded once to bf16 (RNE).  Which kernel
 * runs depends on the batch M (every path streams the packed codes once and
 * unpacks them on chip; K below means "K, and K * bits, allow TMA staging"):
 *   M = 1        CUDA-core GEMV: codes staged by TMA, unpacked in registers,
 *                exact x * q products (K * bits a multiple of 128);
 *   M = 2..8     warp-level tensor-core GEMV (mma.sync, bf16 in, fp32 out):
 *                codes unpacked in registers into the A operand, the tokens
 *                are the MMA's columns (K and group multiples of 128);
 *   M = 2..16    otherwise: tcgen05 GEMV with the unpacked codes in tensor
 *                memory (K a multiple of 128; 3-bit codes need groups that
 *                are multiples of 128), else a CUDA-core GEMV;
 *   M > 16       tcgen05 GEMM (operands staged by TMA, W' dequantised to
 *                bf16 in shared memory, accumulators in tensor memory) when K
 *                is a multiple of 128, else the GEMV 16 batch rows at a time.
 * The decode paths use tensor cores from M = 2 on because a CUDA-core dot
 * product costs one FMA per code and token, so its cost grows with M while
 * the bytes read do not.  Accuracy: every product is exact or rounded once
 * (w' to bf16 on the tensor-core GEMM with grouped grids), sums are fp32, and
 * y carries one bf16 rounding (up to 2^-8 |y|); on realistic inputs each y
 * element lies within 2e-3 * sum_k |x w'| + 2^-8 |y| + 1e-3 of the exact
 * value (arithmetic error, the output rounding, an absolute floor), which is
 * the acceptance bound the tests use.  Range of x: |x| must stay below 2^63.
 * The decode paths form each product at a fixed power-of-two scale (2^-85 on
 * CUDA cores, 2^-69 on the tensor cores); entries with |x| below about 2^-57
 * give products under the fp32 normal range, which the tensor cores may flush
 * to zero: such entries may contribute nothing, an absolute error below
 * 2^-57 * sum_k |w'_k|, far under the 1e-3 floor.
 */
wq_status wq_gemm(const void* x_bf16, int64_t M, int64_t N, int64_t K, const uint32_t* codes,
                  const void* scales_f16, const void* zeros_f16, int bits, int64_t group,
                  void* y_bf16, void* stream);

/*
 * One linear y = x . W'^T of a grouped call: every field as for wq_gemm
 * (x bf16 [M, K], codes/scales/zeros of W [N, K] as wq_quantize_rtn wrote
 * them, zeros NULL for a symmetric grid, y bf16 [M, N]).  The linears of a
 * call share M and bits; each has its own x, shape, group and grid.
 */
typedef struct {
  const void* x_bf16;
  const uint32_t* codes;
  const void* scales_f16;
  const void* zeros_f16;
  void* y_bf16;
  int64_t N, K, group;
} wq_linear;

/*
 * wq_gemm_grouped -- y_l = x_l . W'_l^T for `count` independent linears in as
 * few launches as possible (the decode step of a transformer layer stack: the
 * same dequantise-in-the-matmul as wq_gemm, with the bandwidth argument of
 * the BladeLLM page, "Background information > Solutions").
 *
 *   linears    in   host array of `count` descriptors (read during the call only)
 *   count           >= 1
 *   M               batch rows, common to all linears
 *   bits            2, 3, 4 or 8, common to all linears
 *   workspace       device buffer of at least wq_gemm_grouped_workspace_size()
 *                   bytes, 16-byte aligned, ZERO-FILLED by the caller before
 *                   its first use; every completed call leaves its counters
 *                   at zero again (a call that ends in WQ_ERR_DEVICE_TIMEOUT
 *                   may not: zero the workspace again after one).  Calls that
 *                   share a workspace must be ordered (same stream).  May be
 *                   NULL when the size is 0.
 *   workspace_bytes its size
 *   stream          cudaStream_t
 *
 * For M <= 16, linears whose K and group are multiples of 128 (or per-row
 * grids with K a multiple of 128) run in one persistent kernel per 128
 * linears: every linear is cut into 32-row tiles and 1024-code stages, the
 * stage sequence of all linears is split evenly over the CTAs (a tile cut
 * between two CTAs is finished through the workspace in a fixed order, so
 * results do not depend on timing), and the codes stream through a TMA ring
 * that never drains between tiles or linears.  A short preparation kernel
 * first writes each x, pre-scaled for the tensor cores, into the workspace.
 * The multiply-adds run on warp-level MMAs (mma.sync, bf16 in, fp32 out),
 * with the same exact products and the same accuracy bound as wq_gemm.
 * For 17 <= M <= 255, linears whose K is a multiple of 128 run the swap-AB
 * tensor-core GEMM of wq_gemm in one launch per 64 linears, one CTA per
 * 128-row tile over all of K (no workspace is needed).  Other linears run as
 * wq_gemm would run them.  Every argument of every linear is checked before
 * anything is launched, as for wq_gemm; outputs must not overlap any input or
 * each other.
 */
wq_status wq_gemm_grouped(const wq_linear* linears, int count, int64_t M, int bits, void* workspace,
                          size_t workspace_bytes, void* stream);

/* Workspace bytes wq_gemm_grouped needs for these linears, M and bits (0 if
 * none is needed or an argument is invalid).  Needs no device. */
size_t wq_gemm_grouped_workspace_size(const wq_linear* linears, int count, int64_t M, int bits);

/*
 * wq_gemm_grouped_noalloc -- wq_gemm_grouped for callers that cannot allocate
 * device memory at the point of the call (a serving runtime that hands all
 * GPU memory to its own pool at start-up, code running during CUDA graph
 * capture, a real-time decode loop in which an allocation could synchronise
 * the device or fail).  The pages have no counterpart: this is an interface
 * convenience of this library, not a step of the method.
 *
 * Same arguments, checks, kernels and results as wq_gemm_grouped, without the
 * workspace: the library keeps one built-in workspace of 8 MiB per GPU (a
 * device array that every GPU loading the library holds until the process
 * exits).  A call whose linears need more than 8 MiB of workspace (see
 * wq_gemm_grouped_workspace_size) returns WQ_ERR_WORKSPACE before anything
 * is launched.  The call allocates and frees nothing; each call clears the
 * workspace's tile counters on `stream` before its kernels run.
 *   - The first call on a device looks up the array's device address (and
 *     sets the kernels' attributes); make that first call before any stream
 *     capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents: calls whose kernels overlap on the GPU (different streams
 *     without ordering, or several host threads) race and give wrong results.
 *     Order them on one stream.
 */
wq_status wq_gemm_grouped_noalloc(const wq_linear* linears, int count, int64_t M, int bits, void* stream);

/* Number of uint32 words of packed codes for an [N, K] matrix: N*K*bits/32
 * (0 if bits or K are invalid). */
size_t wq_codes_words(int64_t N, int64_t K, int bits);

/* Number of fp16 scales (and of zeros): N * G, G = K/group or 1 per row
 * (0 if group or K are invalid). */
size_t wq_params_count(int64_t N, int64_t K, int64_t group);

/* Static, NUL-terminated description of a status code. */
const char* wq_status_string(wq_status status);

/*
 * wq_last_device_error -- WQ_ERR_DEVICE_TIMEOUT if, since the previous call, a
 * kernel on the current device gave up a bounded wait (a pipeline barrier that
 * never completed); WQ_OK otherwise.  Synchronises the device and clears the
 * flag.  A kernel that gives up leaves its outputs undefined but the CUDA
 * context usable.
 */
wq_status wq_last_device_error(void);

#ifdef __cplusplus
}
#endif

#endif /* WQ_H */
