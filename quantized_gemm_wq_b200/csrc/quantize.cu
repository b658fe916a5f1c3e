// quantize.cu -- round-to-nearest quantisation of fp16 weights onto the
// uniform asymmetric min-max grid, and packing of the codes.
//
// Grid: "OPTQ: Accurate Quantization for Generative Pre-trained Transformers"
// (reproducibility summary, row "Experiment Setup"): per-row asymmetric
// quantisation on the min-max grid.  Groups: "Platform For AI: BladeLLM model
// quantization", section "block_wise_quant" (one scale set per block of input
// channels).  Rounding: same page, "Quantization algorithms > MinMax"
// (round-to-nearest).  Packing: "[Feature Request] 4bit and 2bit and 1bit
// quantization support" (several codes per word; the exact layout is the
// library's own, see include/wq.h).
//
// A "segment" is one (row, group) pair: g consecutive weights of one row that
// share a scale and a zero.  A segment is split into 32-weight blocks; each
// thread owns whole blocks, so the b words that one block packs into are
// produced and stored by a single thread (b = 3 included).
//
// Arithmetic (bit-exact with the exact definition):
//   * lo/hi: exact fp32 min/max of fp16 values, seeded with 0 (range holds 0);
//   * scale: (hi - lo) in fp64 is exact, one fp64 division, then one RNE to
//     fp16.  The fp64 quotient can never cross or land on an fp16 rounding
//     midpoint unless the exact quotient does, so this equals exact rounding;
//   * zero and codes: rint of an IEEE fp32 division (div.rn, never a multiply
//     by a reciprocal).  With 11-bit operands a non-tie quotient lies farther
//     from a half-integer than fp32 rounding can move it, so this also equals
//     exact rounding (checked on the host over every finite fp16 weight).
#include "wq_internal.cuh"

namespace wq {
namespace {

constexpr int kThreads = 256;

struct Block32 {
  float v[32];
};

__device__ __forceinline__ void load_block(const __half* __restrict__ p, Block32& b) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 u = __ldg(q + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      __half2 h = *reinterpret_cast<const __half2*>(&w[j]);
      float2 f = __half22float2(h);
      b.v[8 * i + 2 * j] = f.x;
      b.v[8 * i + 2 * j + 1] = f.y;
    }
  }
}

// Pack 32 codes of `BITS` bits into BITS words (layout of include/wq.h).
template <int BITS>
__device__ __forceinline__ void pack32(const uint32_t (&c)[32], uint32_t (&w)[BITS]) {
#pragma unroll
  for (int i = 0; i < BITS; ++i) w[i] = 0u;
  if constexpr (BITS == 3) {
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int bit = 3 * j, wi = bit >> 5, off = bit & 31;
      w[wi] |= c[j] << off;
      if (off > 29) w[wi + 1] |= c[j] >> (32 - off);
    }
  } else {
    constexpr int per = 32 / BITS;
#pragma unroll
    for (int j = 0; j < 32; ++j) w[j / per] |= c[j] << (BITS * (j % per));
  }
}

template <int BITS>
__device__ __forceinline__ void store_words(uint32_t* __restrict__ dst, const uint32_t (&w)[BITS]) {
  if constexpr (BITS == 2) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else if constexpr (BITS == 4) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else if constexpr (BITS == 8) {
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else {
    dst[0] = w[0];
    dst[1] = w[1];
    dst[2] = w[2];
  }
}

struct Grid {
  float s;     // stored scale as fp32 (exact)
  float z;     // stored zero (integer, exact)
  __half sh;
};

// Asymmetric grid (sym false): scale from the range [lo, hi], zero rint(-lo /
// scale).  Symmetric grid (sym true; "Platform For AI: BladeLLM model
// quantization", "Quantization modes > weight_only_quant": signed symmetric by
// default): a = max(-lo, hi) = max |w|, scale = fp16(a / (2^(b-1) - 1)), zero
// fixed at 2^(b-1) and not stored.  One fp64 division then one RNE to fp16
// equals exact rounding for the divisors 1, 3, 7, 127 as for 3, 7, 15, 255.
template <int BITS>
__device__ __forceinline__ Grid make_grid(float lo, float hi, bool sym) {
  constexpr double qmax = double((1 << BITS) - 1);
  constexpr double top = double((1 << (BITS - 1)) - 1);
  const double d = sym ? double(fmaxf(0.0f - lo, hi)) / top
                       : (double(hi) - double(lo)) / qmax;   // exact difference, one rounding
  Grid gr;
  gr.sh = __double2half(d);                           // one RNE to fp16
  gr.s = __half2float(gr.sh);
  if (gr.s == 0.0f) {                                  // degenerate range
    gr.s = 1.0f;
    gr.sh = __float2half_rn(1.0f);
    gr.z = sym ? float(1 << (BITS - 1)) : 0.0f;
  } else if (sym) {
    gr.z = float(1 << (BITS - 1));
  } else {
    gr.z = rintf(__fdiv_rn(0.0f - lo, gr.s));          // 0 - lo is never -0
  }
  return gr;
}

template <int BITS>
__device__ __forceinline__ void encode_block(const Block32& b, const Grid& gr,
                                             uint32_t* __restrict__ dst) {
  constexpr float qmax = float((1 << BITS) - 1);
  uint32_t c[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float q = rintf(__fdiv_rn(b.v[i], gr.s)) + gr.z;
    q = fminf(fmaxf(q, 0.0f), qmax);
    c[i] = uint32_t(q);
  }
  uint32_t w[BITS];
  pack32<BITS>(c, w);
  store_words<BITS>(dst, w);
}

// Segments of at most 32 blocks: TPS threads (a power of two <= 32) per
// segment, several segments per CTA, min/max reduced with shuffles.
template <int BITS, int TPS>
__global__ void __launch_bounds__(kThreads)
quantize_small_kernel(const __half* __restrict__ W, int64_t nseg, int64_t K, int64_t g,
                      uint32_t* __restrict__ codes, __half* __restrict__ scales,
                      __half* __restrict__ zeros) {
  const int64_t seg = int64_t(blockIdx.x) * (kThreads / TPS) + threadIdx.x / TPS;
  const int sub = threadIdx.x % TPS;
  const bool active = seg < nseg;
  const int64_t G = K / g;
  const int64_t n = active ? seg / G : 0, j = active ? seg % G : 0;
  const int nblk = int(g / 32);
  const __half* wseg = W + n * K + j * g;
  uint32_t* cseg = codes + n * (K * BITS / 32) + j * (g / 32) * BITS;

  float lo = 0.0f, hi = 0.0f;
  if (active) {
    for (int blk = sub; blk < nblk; blk += TPS) {
      Block32 b;
      load_block(wseg + 32 * blk, b);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        lo = fminf(lo, b.v[i]);
        hi = fmaxf(hi, b.v[i]);
      }
    }
  }
#pragma unroll
  for (int off = TPS / 2; off > 0; off >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off, TPS));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off, TPS));
  }
  if (!active) return;
  const Grid gr = make_grid<BITS>(lo, hi, zeros == nullptr);
  if (sub == 0) {
    scales[seg] = gr.sh;
    if (zeros) zeros[seg] = __float2half_rn(gr.z);
  }
  for (int blk = sub; blk < nblk; blk += TPS) {
    Block32 b;
    load_block(wseg + 32 * blk, b);
    encode_block<BITS>(b, gr, cseg + blk * BITS);
  }
}

// Long segments (more than 32 blocks, e.g. one grid per row of a wide layer):
// one CTA per segment, min/max reduced through shared memory.
template <int BITS>
__global__ void __launch_bounds__(kThreads)
quantize_large_kernel(const __half* __restrict__ W, int64_t K, int64_t g,
                      uint32_t* __restrict__ codes, __half* __restrict__ scales,
                      __half* __restrict__ zeros) {
  __shared__ float s_lo[kThreads / 32], s_hi[kThreads / 32];
  const int64_t seg = blockIdx.x;
  const int64_t G = K / g;
  const int64_t n = seg / G, j = seg % G;
  const int nblk = int(g / 32);
  const __half* wseg = W + n * K + j * g;
  uint32_t* cseg = codes + n * (K * BITS / 32) + j * (g / 32) * BITS;

  float lo = 0.0f, hi = 0.0f;
  for (int blk = threadIdx.x; blk < nblk; blk += kThreads) {
    Block32 b;
    load_block(wseg + 32 * blk, b);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      lo = fminf(lo, b.v[i]);
      hi = fmaxf(hi, b.v[i]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
  if ((threadIdx.x & 31) == 0) {
    s_lo[threadIdx.x / 32] = lo;
    s_hi[threadIdx.x / 32] = hi;
  }
  __syncthreads();
  lo = s_lo[0];
  hi = s_hi[0];
#pragma unroll
  for (int w = 1; w < kThreads / 32; ++w) {
    lo = fminf(lo, s_lo[w]);
    hi = fmaxf(hi, s_hi[w]);
  }
  const Grid gr = make_grid<BITS>(lo, hi, zeros == nullptr);
  if (threadIdx.x == 0) {
    scales[seg] = gr.sh;
    if (zeros) zeros[seg] = __float2half_rn(gr.z);
  }
  for (int blk = threadIdx.x; blk < nblk; blk += kThreads) {
    Block32 b;
    load_block(wseg + 32 * blk, b);
    encode_block<BITS>(b, gr, cseg + blk * BITS);
  }
}

template <int BITS>
cudaError_t launch_bits(const __half* W, int64_t N, int64_t K, int64_t g, uint32_t* codes,
                        __half* scales, __half* zeros, cudaStream_t st) {
  const int64_t nseg = N * (K / g);
  const int nblk = int(g / 32);
  if (nblk > 32) {
    quantize_large_kernel<BITS><<<dim3(unsigned(nseg)), kThreads, 0, st>>>(W, K, g, codes, scales, zeros);
    return cudaGetLastError();
  }
  int tps = 1;
  while (tps * 2 <= nblk) tps *= 2;
  const int64_t per_cta = kThreads / tps;
  const unsigned grid = unsigned((nseg + per_cta - 1) / per_cta);
  switch (tps) {
    case 1: quantize_small_kernel<BITS, 1><<<grid, kThreads, 0, st>>>(W, nseg, K, g, codes, scales, zeros); break;
    case 2: quantize_small_kernel<BITS, 2><<<grid, kThreads, 0, st>>>(W, nseg, K, g, codes, scales, zeros); break;
    case 4: quantize_small_kernel<BITS, 4><<<grid, kThreads, 0, st>>>(W, nseg, K, g, codes, scales, zeros); break;
    case 8: quantize_small_kernel<BITS, 8><<<grid, kThreads, 0, st>>>(W, nseg, K, g, codes, scales, zeros); break;
    case 16: quantize_small_kernel<BITS, 16><<<grid, kThreads, 0, st>>>(W, nseg, K, g, codes, scales, zeros); break;
    default: quantize_small_kernel<BITS, 32><<<grid, kThreads, 0, st>>>(W, nseg, K, g, codes, scales, zeros); break;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize(const __half* W, int64_t N, int64_t K, int bits, int64_t g,
                            uint32_t* codes, __half* scales, __half* zeros, cudaStream_t st) {
  switch (bits) {
    case 2: return launch_bits<2>(W, N, K, g, codes, scales, zeros, st);
    case 3: return launch_bits<3>(W, N, K, g, codes, scales, zeros, st);
    case 4: return launch_bits<4>(W, N, K, g, codes, scales, zeros, st);
    default: return launch_bits<8>(W, N, K, g, codes, scales, zeros, st);
  }
}

}  // namespace wq
