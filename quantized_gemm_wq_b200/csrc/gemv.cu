// gemv.cu -- decode-time y = x . W'^T for small batches (M <= 16) on CUDA cores.
//
// Dequantise inside the matmul: "[Feature Request] 4bit and 2bit and 1bit
// quantization support" (weights stay packed in memory and are turned into
// floats by the GPU when used); "Platform For AI: BladeLLM model quantization",
// "Background information > Solutions" and "Quantization modes >
// weight_only_quant" (low-bit weights cut the bytes read from GPU memory, the
// bound when memory bandwidth limits decoding).  At M <= 16 the work is a scan
// of the packed codes: every code byte is read from HBM exactly once.
//
// Work split.  A CTA owns 32 consecutive output rows (one per lane) and splits
// their K dimension across its 8 warps (split-K across warps): warp w takes
// tiles of U consecutive 32-code blocks, interleaved over warps.  Per block a
// lane loads the b packed words of its row with one vector load (b = 2, 4, 8;
// three 32-bit loads for b = 3), unpacks the 32 codes in registers and
// accumulates  s * sum_k x[m,k] (q_k - z)  in fp32 for every batch row m.
// The 32 x values of a block are staged once per warp in shared memory and read
// as broadcasts.  Partial sums of the 8 warps are added through shared memory
// at the end and y is rounded once to bf16.
//
// Exactness of the dequantisation: q - z is formed exactly as
// float(0x4B000000 | q) - (2^23 + z): both terms are exact in fp32 (integers
// below 2^24), so w' = s (q - z) is exact before the product with x.
#include "wq_internal.cuh"

namespace wq {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;

template <int MT>
struct GemvCfg {
  static constexpr int U = MT <= 4 ? 4 : 2;   // blocks per warp tile (loads in flight)
};

template <int BITS>
__device__ __forceinline__ void load_codes(const uint32_t* __restrict__ p, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 2) {
    uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = v.x; w[1] = v.y;
  } else if constexpr (BITS == 4) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (BITS == 8) {
    uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else {
    w[0] = __ldg(p); w[1] = __ldg(p + 1); w[2] = __ldg(p + 2);
  }
}

// Code i (0..31) of a 32-code block, per the packed layout.
template <int BITS>
__device__ __forceinline__ uint32_t code_at(const uint32_t (&w)[BITS], int i) {
  if constexpr (BITS == 3) {
    const int bit = 3 * i, a = bit >> 5, sh = bit & 31;
    const uint32_t nxt = (a + 1 < 3) ? w[(a + 1) % 3] : 0u;
    return __funnelshift_r(w[a], nxt, sh) & 7u;
  } else {
    constexpr int per = 32 / BITS;
    return (w[i / per] >> (BITS * (i % per))) & ((1u << BITS) - 1u);
  }
}

template <int BITS, int MT>
__global__ void __launch_bounds__(kThreads)
gemv_kernel(const __nv_bfloat16* __restrict__ x, int M, int64_t N, int64_t K,
            const uint32_t* __restrict__ codes, const __half* __restrict__ scales,
            const __half* __restrict__ zeros, int64_t g, FastDiv blocks_per_group,
            __nv_bfloat16* __restrict__ y) {
  constexpr int U = GemvCfg<MT>::U;
  constexpr int kStage = kWarps * U * MT * 32;
  constexpr int kRed = kWarps * MT * 32;
  __shared__ __align__(16) float smem[kStage > kRed ? kStage : kRed];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n = int64_t(blockIdx.x) * 32 + lane;
  const bool row_ok = n < N;
  const int64_t KB = K / 32;
  const int64_t KW = K * BITS / 32;
  const int64_t G = K / g;
  const uint32_t* crow = codes + (row_ok ? n : 0) * KW;
  const __half* srow = scales + (row_ok ? n : 0) * G;
  const __half* zrow = zeros + (row_ok ? n : 0) * G;
  float* xs = smem + warp * (U * MT * 32);

  float acc[MT];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.0f;

  for (int64_t t0 = int64_t(warp) * U; t0 < KB; t0 += int64_t(kWarps) * U) {
    uint32_t cw[U][BITS];
    float sc[U], zb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t kb = t0 + u;
      if (row_ok && kb < KB) {
        load_codes<BITS>(crow + kb * BITS, cw[u]);
        const uint32_t grp = blocks_per_group.div(uint32_t(kb));
        sc[u] = __half2float(srow[grp]);
        zb[u] = 8388608.0f + __half2float(zrow[grp]);
      } else {
#pragma unroll
        for (int i = 0; i < BITS; ++i) cw[u][i] = 0u;
        sc[u] = 0.0f;
        zb[u] = 8388608.0f;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t kb = t0 + u;
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        float v = 0.0f;
        if (m < M && kb < KB) v = __bfloat162float(x[int64_t(m) * K + kb * 32 + lane]);
        xs[(u * MT + m) * 32 + lane] = v;
      }
    }
    __syncwarp();
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float qz[32];
#pragma unroll
      for (int i = 0; i < 32; ++i)
        qz[i] = __int_as_float(0x4B000000 | int(code_at<BITS>(cw[u], i))) - zb[u];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < M) {
          const float4* xv = reinterpret_cast<const float4*>(xs + (u * MT + m) * 32);
          float d0 = 0.0f, d1 = 0.0f;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 xx = xv[i];
            d0 = fmaf(xx.x, qz[4 * i + 0], d0);
            d1 = fmaf(xx.y, qz[4 * i + 1], d1);
            d0 = fmaf(xx.z, qz[4 * i + 2], d0);
            d1 = fmaf(xx.w, qz[4 * i + 3], d1);
          }
          acc[m] = fmaf(sc[u], d0 + d1, acc[m]);
        }
      }
    }
    __syncwarp();
  }

  __syncthreads();   // staging area is reused for the cross-warp reduction
#pragma unroll
  for (int m = 0; m < MT; ++m) smem[(warp * MT + m) * 32 + lane] = acc[m];
  __syncthreads();
  for (int idx = threadIdx.x; idx < MT * 32; idx += kThreads) {
    const int m = idx >> 5, l = idx & 31;
    const int64_t nn = int64_t(blockIdx.x) * 32 + l;
    if (m < M && nn < N) {
      float s = 0.0f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) s += smem[(w * MT + m) * 32 + l];
      y[int64_t(m) * N + nn] = __float2bfloat16_rn(s);
    }
  }
}

template <int BITS>
cudaError_t launch_bits(const __nv_bfloat16* x, int M, int64_t N, int64_t K,
                        const uint32_t* codes, const __half* scales, const __half* zeros,
                        int64_t g, __nv_bfloat16* y, cudaStream_t st) {
  const dim3 grid(unsigned((N + 31) / 32));
  const FastDiv bpg(uint32_t(g / 32));
  if (M <= 1) gemv_kernel<BITS, 1><<<grid, kThreads, 0, st>>>(x, M, N, K, codes, scales, zeros, g, bpg, y);
  else if (M <= 2) gemv_kernel<BITS, 2><<<grid, kThreads, 0, st>>>(x, M, N, K, codes, scales, zeros, g, bpg, y);
  else if (M <= 4) gemv_kernel<BITS, 4><<<grid, kThreads, 0, st>>>(x, M, N, K, codes, scales, zeros, g, bpg, y);
  else if (M <= 8) gemv_kernel<BITS, 8><<<grid, kThreads, 0, st>>>(x, M, N, K, codes, scales, zeros, g, bpg, y);
  else gemv_kernel<BITS, 16><<<grid, kThreads, 0, st>>>(x, M, N, K, codes, scales, zeros, g, bpg, y);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemv(const __nv_bfloat16* x, int M, int64_t N, int64_t K,
                        const uint32_t* codes, const __half* scales, const __half* zeros,
                        int bits, int64_t g, __nv_bfloat16* y, cudaStream_t st) {
  switch (bits) {
    case 2: return launch_bits<2>(x, M, N, K, codes, scales, zeros, g, y, st);
    case 3: return launch_bits<3>(x, M, N, K, codes, scales, zeros, g, y, st);
    case 4: return launch_bits<4>(x, M, N, K, codes, scales, zeros, g, y, st);
    default: return launch_bits<8>(x, M, N, K, codes, scales, zeros, g, y, st);
  }
}

}  // namespace wq
