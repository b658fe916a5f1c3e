// gemv_tma.cu -- decode GEMV for one token (M = 1): y = x . W'^T on CUDA cores,
// codes streamed by TMA.
//
// Dequantise inside the matmul ("[Feature Request] 4bit and 2bit and 1bit
// quantization support": packed weights are turned into floats on the GPU;
// "Platform For AI: BladeLLM model quantization", "Quantization modes >
// weight_only_quant": decoding is bound by the bytes read from GPU memory).
//
// Work split.  A CTA owns 32 output rows; its W warps split K (split-K across
// warps), each warp taking a contiguous range of "box columns" (4 units of 32
// codes = 128 inputs).  Per box column one lane issues a 2-D TMA copy of the
// packed codes of all 32 rows (32 x 16b bytes, rows past N and columns past K
// zero-filled) into the warp's ring of D stages; the copy completes on the
// stage's mbarrier.  Lane l works on rows lr, lr+8, lr+16, lr+24 (lr = l % 8)
// and on unit kq = l / 8 of the column, so every code is touched once.
// Partial sums are reduced over the 4 kq lanes with shuffles and over the W
// warps through shared memory; y is rounded once to bf16.
//
// Unpacking with one AND per code.  A code q at bit p of a 32-bit word, with
// every other bit cleared, is the subnormal float q * 2^(p-149): no exponent
// bits, no implicit leading one, nothing to subtract.  Codes above bit 23 - b
// are first brought down by one shared shift (a funnel shift for the 3-bit
// straddles).  The x value multiplied with code position i is stored scaled by
// 2^(S - p_i), so every product x * q lands exactly at the common scale
// 2^(S-149) (S = 64): products are exact (an 8-bit significand times a code of
// at most 8 bits), sums are fp32, and the unit's dot product is brought back
// with one exact multiplication by 2^(149-S).  The zero is applied per unit as
// s * (dot - z * sum x); sum x of each unit comes from a shuffle reduction of
// the staged x values.  Results far below the fp32 normal range (|x q| < 2^-41)
// keep an absolute accuracy of 2^-64; |x| must stay below 2^63.
#include <cuda.h>   // CUtensorMap

#include "wq_internal.cuh"

namespace wq {
namespace {

constexpr int kScaleS = 64;
constexpr uint64_t kWaitNs = 1000000000ull;

__device__ unsigned int g_gemv_tma_timeout;

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

// d[I % 4] += x'[I] * f_I for I = I0..31 (four independent chains).
template <int BITS, int I>
struct Dot {
  __device__ __forceinline__ static void run(const uint32_t (&w)[BITS], const float (&xp)[32],
                                             float (&d)[4]) {
    d[I & 3] = fmaf(xp[I], code_subnormal<BITS, I>(w), d[I & 3]);
    if constexpr (I + 1 < 32) Dot<BITS, I + 1>::run(w, xp, d);
  }
};

__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __noinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = now_ns();
  while (!mbar_try(bar, parity)) {
    if (now_ns() - t0 > kWaitNs) {
      atomicExch(&g_gemv_tma_timeout, 1u);
      return false;
    }
  }
  return true;
}

template <int BITS>
__device__ __forceinline__ void lds_words(uint32_t a, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 2) {
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(a));
  } else if constexpr (BITS == 4) {
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(a));
  } else if constexpr (BITS == 8) {
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(a));
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7]) : "r"(a + 16));
  } else {
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[0]) : "r"(a));
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[1]) : "r"(a + 4));
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[2]) : "r"(a + 8));
  }
}

template <int BITS, int D>
struct M1Cfg {
  static constexpr int COL_BYTES = 32 * 16 * BITS;        // one box: 32 rows x 4 units
  static constexpr int XS_BYTES = 2 * 128 * 4;             // staged x', double-buffered
  // per-warp region, kept a multiple of 128 bytes (TMA destination alignment)
  static constexpr int WARP_BYTES = (D * COL_BYTES + XS_BYTES + D * 8 + 127) / 128 * 128;
};
template <int BITS>
constexpr int ring_depth() { return BITS == 8 ? 3 : 4; }

template <int BITS, int W, int D>
__global__ void __launch_bounds__(32 * W)
gemv_m1_tma_kernel(const __grid_constant__ CUtensorMap tm_codes, const __nv_bfloat16* __restrict__ x,
                   int64_t N, int64_t K, const __half* __restrict__ scales,
                   const __half* __restrict__ zeros, FastDiv units_per_group,
                   __nv_bfloat16* __restrict__ y) {
  using Cfg = M1Cfg<BITS, D>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float red[W][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int lr = lane & 7, kq = lane >> 3;
  uint8_t* wbase = smem + warp * Cfg::WARP_BYTES;
  const uint32_t ring = saddr(wbase);
  float* xs = reinterpret_cast<float*>(wbase + D * Cfg::COL_BYTES);
  const uint32_t bar0 = saddr(wbase + D * Cfg::COL_BYTES + Cfg::XS_BYTES);

  const int64_t row0 = int64_t(blockIdx.x) * 32;
  const int64_t KU = K / 32;
  const int KC = int((KU + 3) / 4);
  const int c0 = int(int64_t(KC) * warp / W), c1 = int(int64_t(KC) * (warp + 1) / W);
  const int64_t G = K / (int64_t(units_per_group.d) * 32);

  // x scale of code position `lane` (the position this lane stages).
  const float xscale = __uint_as_float(uint32_t(127 + kScaleS - code_p<BITS>(lane)) << 23);

  if (lane == 0) {
    for (int s = 0; s < D; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8 * s));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();
  auto issue = [&](int c) {   // lane 0
    if (c < c1) {
      const int s = (c - c0) % D;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar0 + 8 * s),
                   "r"(uint32_t(Cfg::COL_BYTES))
                   : "memory");
      asm volatile(
          "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
          " [%0], [%1, {%3, %4}], [%2];" ::"r"(ring + s * Cfg::COL_BYTES),
          "l"(&tm_codes), "r"(bar0 + 8 * s), "r"(c * 4 * BITS), "r"(int(row0))
          : "memory");
    }
  };
  // x of column c, position `lane` of its 4 units.
  auto load_x = [&](int c, float (&xv)[4]) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t k = (int64_t(c) * 4 + u) * 32 + lane;
      xv[u] = (c < c1 && k < K) ? __bfloat162float(x[k]) : 0.0f;
    }
  };
  // stage x' of a column and return sum x of this lane's unit kq.
  auto stage_x = [&](int c, const float (&xv)[4]) {
    float* dst = xs + ((c - c0) & 1) * 128;
#pragma unroll
    for (int u = 0; u < 4; ++u) dst[u * 32 + lane] = xv[u] * xscale;
    const bool h16 = lane & 16, h8 = lane & 8;
    float a = (h16 ? xv[2] : xv[0]) + __shfl_xor_sync(0xffffffffu, h16 ? xv[0] : xv[2], 16);
    float b = (h16 ? xv[3] : xv[1]) + __shfl_xor_sync(0xffffffffu, h16 ? xv[1] : xv[3], 16);
    float e = (h8 ? b : a) + __shfl_xor_sync(0xffffffffu, h8 ? a : b, 8);
    e += __shfl_xor_sync(0xffffffffu, e, 4);
    e += __shfl_xor_sync(0xffffffffu, e, 2);
    e += __shfl_xor_sync(0xffffffffu, e, 1);
    return e;
  };
  auto load_sz = [&](int c, float (&sc)[4], float (&zz)[4]) {
    const int64_t ug = int64_t(c) * 4 + kq;
    const uint32_t grp = units_per_group.div(uint32_t(ug < KU ? ug : 0));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t n = row0 + lr + 8 * i;
      const bool ok = c < c1 && ug < KU && n < N;
      sc[i] = ok ? __half2float(scales[n * G + grp]) : 0.0f;
      zz[i] = ok ? __half2float(zeros[n * G + grp]) : 0.0f;
    }
  };

  if (lane == 0)
    for (int c = c0; c < c0 + D; ++c) issue(c);
  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  float xv[4], sc[4], zz[4];
  load_x(c0, xv);
  float sx = stage_x(c0, xv);
  load_sz(c0, sc, zz);
  bool ok = true;
  int c = c0;
  for (; c < c1; ++c) {
    float xn[4], scn[4], zzn[4];
    load_x(c + 1, xn);
    load_sz(c + 1, scn, zzn);
    const int s = (c - c0) % D;
    ok = mbar_wait_bounded(bar0 + 8 * s, uint32_t(((c - c0) / D) & 1));
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) break;
    __syncwarp();                      // x' of column c is visible
    float xp[32];
    const float4* xq = reinterpret_cast<const float4*>(xs + ((c - c0) & 1) * 128 + kq * 32);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 v = xq[j];
      xp[4 * j] = v.x; xp[4 * j + 1] = v.y; xp[4 * j + 2] = v.z; xp[4 * j + 3] = v.w;
    }
    const uint32_t col = ring + uint32_t(s * Cfg::COL_BYTES);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t w[BITS];
      lds_words<BITS>(col + uint32_t((lr + 8 * i) * 16 * BITS + kq * 4 * BITS), w);
      float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      Dot<BITS, 0>::run(w, xp, d);
      const float dot = (d[0] + d[1]) + (d[2] + d[3]);
      acc[i] = fmaf(sc[i], fmaf(dot, 0x1p85f, -zz[i] * sx), acc[i]);
    }
    __syncwarp();                      // stage s and x' buffer (c - c0) & 1 are free again
    if (lane == 0) issue(c + D);
    sx = stage_x(c + 1, xn);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      sc[i] = scn[i];
      zz[i] = zzn[i];
    }
  }
  if (!ok) {                           // copies still in flight land before the CTA exits
    if (lane == 0)
      for (int k = c; k < c1 && k < c + D; ++k) {
        const uint64_t t0 = now_ns();
        while (!mbar_try(bar0 + 8 * ((k - c0) % D), uint32_t(((k - c0) / D) & 1)) &&
               now_ns() - t0 < kWaitNs / 5) {
        }
      }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float v = acc[i];
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    if (kq == 0) red[warp][lr + 8 * i] = v;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < W; ++w) v += red[w][threadIdx.x];
    const int64_t n = row0 + threadIdx.x;
    if (n < N && ok) y[n] = __float2bfloat16_rn(v);
  }
}

template <int BITS, int W>
cudaError_t launch_w(const CUtensorMap& tm, const __nv_bfloat16* x, int64_t N, int64_t K,
                     const __half* scales, const __half* zeros, const FastDiv& upg,
                     __nv_bfloat16* y, cudaStream_t st) {
  constexpr int D = ring_depth<BITS>();
  constexpr int smem = W * M1Cfg<BITS, D>::WARP_BYTES;
  static_assert(smem + W * 32 * 4 <= 232448, "shared memory");
  static bool attr_set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(gemv_m1_tma_kernel<BITS, W, D>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  const dim3 grid(unsigned((N + 31) / 32));
  gemv_m1_tma_kernel<BITS, W, D><<<grid, 32 * W, smem, st>>>(tm, x, N, K, scales, zeros, upg, y);
  return cudaGetLastError();
}

template <int BITS>
cudaError_t launch_bits(const __nv_bfloat16* x, int64_t N, int64_t K, const uint32_t* codes,
                        const __half* scales, const __half* zeros, int64_t g, __nv_bfloat16* y,
                        cudaStream_t st) {
  alignas(64) CUtensorMap tm;
  if (!make_tensor_map_2d(&tm, TmaType::kU32, codes, uint64_t(K * BITS / 32), uint64_t(N),
                          uint64_t(K * BITS / 8), 4 * BITS, 32, false))
    return cudaErrorInvalidValue;
  const FastDiv upg(uint32_t(g / 32));
  // Warps per CTA: enough warps in total to cover every SM several times, but
  // no more warps than box columns in a row.
  const int64_t ctas = (N + 31) / 32;
  const int64_t cols = (K / 32 + 3) / 4;
  const int64_t want = (148 * 24 + ctas - 1) / ctas;
  if (BITS != 8 && want >= 16 && cols >= 16)
    return launch_w<BITS, (BITS == 8 ? 8 : 16)>(tm, x, N, K, scales, zeros, upg, y, st);
  if (want >= 8 && cols >= 8) return launch_w<BITS, 8>(tm, x, N, K, scales, zeros, upg, y, st);
  return launch_w<BITS, 4>(tm, x, N, K, scales, zeros, upg, y, st);
}

}  // namespace

bool gemv_m1_tma_supported(int64_t K, int bits) { return (K * bits) % 128 == 0; }

cudaError_t launch_gemv_m1_tma(const __nv_bfloat16* x, int64_t N, int64_t K,
                               const uint32_t* codes, const __half* scales, const __half* zeros,
                               int bits, int64_t g, __nv_bfloat16* y, cudaStream_t st) {
  switch (bits) {
    case 2: return launch_bits<2>(x, N, K, codes, scales, zeros, g, y, st);
    case 3: return launch_bits<3>(x, N, K, codes, scales, zeros, g, y, st);
    case 4: return launch_bits<4>(x, N, K, codes, scales, zeros, g, y, st);
    default: return launch_bits<8>(x, N, K, codes, scales, zeros, g, y, st);
  }
}

bool gemv_m1_tma_read_and_clear_timeout(cudaError_t* err) {
  unsigned int v = 0;
  const unsigned int zero = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&v, g_gemv_tma_timeout, sizeof(v));
  if (e == cudaSuccess && v) e = cudaMemcpyToSymbol(g_gemv_tma_timeout, &zero, sizeof(zero));
  *err = e;
  return v != 0;
}

}  // namespace wq
