// wq_internal.cuh -- declarations shared by the translation units of libwq.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace wq {

// Largest M served by the CUDA-core GEMV; larger batches use the tensor cores.
constexpr int kGemvMaxM = 16;

// Effective group length: K for a per-row grid (group 0 or K).
inline int64_t effective_group(int64_t K, int64_t group) { return (group == 0) ? K : group; }

// Division of non-negative 32-bit n (< 2^31) by a fixed divisor d >= 1 with a
// multiply-high and a shift (division by invariant integers using
// multiplication, Granlund & Montgomery 1994): l = ceil(log2 d),
// m = floor(2^32 (2^l - d) / d) + 1, n / d = (mulhi(n, m) + n) >> l.
struct FastDiv {
  uint32_t m = 1, l = 0, d = 1;
  FastDiv() = default;
  explicit FastDiv(uint32_t d_) : d(d_) {
    l = 0;
    while ((uint64_t(1) << l) < d) ++l;
    m = uint32_t(((uint64_t(1) << 32) * ((uint64_t(1) << l) - d)) / d + 1);
  }
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    return uint32_t((uint64_t(__umulhi(n, m)) + n) >> l);
  }
};

// ---- unpacking a 32-code unit with one AND per code ---------------------
// A code q at bit p of a 32-bit word, with every other bit cleared, is the
// subnormal float q * 2^(p-149) (no exponent bits, no implicit one).  Codes
// above bit 23 - b are first brought down by one shift shared by the word
// (a funnel shift for the 3-bit codes that straddle two words).
// Position p (after its shift) of code i of a unit, and whether it needs the
// shifted view.  Host-and-device so the lane's x scale can use it at run time.
template <int BITS>
__host__ __device__ constexpr int code_p(int i) {
  const int P = (BITS * i) % 32;
  if (P + BITS <= 23) return P;
  return P - (BITS == 2 ? 10 : BITS == 8 ? 16 : 12);
}
template <int BITS>
__host__ __device__ constexpr bool code_shifted(int i) {
  return (BITS * i) % 32 + BITS > 23;
}

template <int BITS, int I>
__device__ __forceinline__ float code_subnormal(const uint32_t (&w)[BITS]) {
  constexpr int a = (BITS * I) / 32;
  constexpr int p = code_p<BITS>(I);
  constexpr uint32_t mask = ((1u << BITS) - 1u) << p;
  uint32_t v;
  if constexpr (!code_shifted<BITS>(I)) {
    v = w[a];
  } else if constexpr (BITS == 3) {
    v = (a < 2) ? __funnelshift_r(w[a], w[a + 1 < 3 ? a + 1 : 2], 12) : (w[a] >> 12);
  } else {
    v = w[a] >> (BITS == 2 ? 10 : BITS == 8 ? 16 : 12);
  }
  return __uint_as_float(v & mask);
}


// ---- launchers (arguments already validated by the C ABI layer) ----------
cudaError_t launch_quantize(const __half* W, int64_t N, int64_t K, int bits, int64_t g,
                            uint32_t* codes, __half* scales, __half* zeros, cudaStream_t st);

cudaError_t launch_gemv(const __nv_bfloat16* x, int M, int64_t N, int64_t K,
                        const uint32_t* codes, const __half* scales, const __half* zeros,
                        int bits, int64_t g, __nv_bfloat16* y, cudaStream_t st);

// M = 1 decode GEMV with TMA-staged codes and x; needs 16-byte aligned code
// rows and a 16-byte aligned x.
bool gemv_m1_tma_supported(const void* x, const void* codes, int64_t K, int bits);
cudaError_t launch_gemv_m1_tma(const __nv_bfloat16* x, int64_t N, int64_t K,
                               const uint32_t* codes, const __half* scales, const __half* zeros,
                               int bits, int64_t g, __nv_bfloat16* y, cudaStream_t st);
bool gemv_m1_tma_read_and_clear_timeout(cudaError_t* err);

// Decode GEMV for 2..8 tokens on warp-level MMAs (gemv_mma.cu): K and the group
// length multiples of 128, x rows and code rows 16-byte aligned.
bool gemv_mma_supported(int M, const void* x, const void* codes, int64_t K, int64_t g);
cudaError_t launch_gemv_mma(const __nv_bfloat16* x, int M, int64_t N, int64_t K, const uint32_t* codes,
                            const __half* scales, const __half* zeros, int bits, int64_t g,
                            __nv_bfloat16* y, cudaStream_t st);
bool gemv_mma_read_and_clear_timeout(cudaError_t* err);

// True when the tensor-core path can stage this K with TMA (K a multiple of 128).
bool gemm_tc_supported(int64_t K, int bits);

// Batches of 17..255 rows on the tensor cores with the weight rows on the
// MMA's M side (gemm_sw.cu); K a multiple of 128.
bool gemm_sw_supported(int64_t M, int64_t K);
cudaError_t launch_gemm_sw(const __nv_bfloat16* x, int64_t M, int64_t N, int64_t K, const uint32_t* codes,
                           const __half* scales, const __half* zeros, int bits, int64_t g, __nv_bfloat16* y,
                           cudaStream_t st);
bool gemm_sw_read_and_clear_timeout(cudaError_t* err);

cudaError_t launch_gemm_tc(const __nv_bfloat16* x, int64_t M, int64_t N, int64_t K,
                           const uint32_t* codes, const __half* scales, const __half* zeros,
                           int bits, int64_t g, __nv_bfloat16* y, cudaStream_t st);

// Tensor-core decode GEMV (gemv_tc.cu): 2 <= M <= 16, K % 128 == 0, and for
// 3-bit codes groups that are whole multiples of 128.
bool gemv_tc_supported(int M, int64_t K, int bits, int64_t g);
cudaError_t launch_gemv_tc(const __nv_bfloat16* x, int M, int64_t N, int64_t K,
                           const uint32_t* codes, const __half* scales, const __half* zeros,
                           int bits, int64_t g, __nv_bfloat16* y, cudaStream_t st);
bool gemv_tc_read_and_clear_timeout(cudaError_t* err);

// Reads and clears the device-side "bounded wait expired" flags of the current
// device (synchronises the device).  Returns true if one was set.
bool gemm_tc_read_and_clear_timeout(cudaError_t* err);

// TMA tensor maps (a CUtensorMap is 128 bytes, 64-byte aligned).
enum class TmaType { kU32, kBF16 };
bool make_tensor_map_2d(void* map, TmaType type, const void* base, uint64_t inner, uint64_t outer,
                        uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, int swizzle_bytes);

}  // namespace wq
