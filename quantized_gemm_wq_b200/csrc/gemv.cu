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
// Work split.  Each warp owns R consecutive output rows over the whole K.  A
// lane owns one 32-code unit (b packed words) of every row per step, so one
// warp-wide load reads 32 consecutive units of a row: 256/384/512/1024 bytes
// contiguous for b = 2/3/4/8 (fully coalesced).  Steps are unrolled so that
// R x S loads per lane are in flight before the first is used.  Each lane
// keeps fp32 partial sums for its rows; a shuffle reduction across the 32
// lanes (split-K over lanes) finishes every row.
//
// Unpacking.  A code q sitting at bit p of a 32-bit word becomes a float with
// one AND-OR (lop3): bits (word & (mask << p)) | ((150 - p) << 23) are the
// float 2^(23-p) + q exactly (exponent 23 - p, q in the mantissa).  Every code
// is brought to a position p in [8, 23 - b] by one of three shared word views
// (word << 8 or 12, word, word >> 10..16 / a funnel shift for the b = 3
// straddles), so a code costs one lop3.
//   One FADD with the compile-time constant 2^(23-p) then gives q exactly, and
//   q - z is formed exactly (M = 1: the zero is applied once per unit as
//   s * (sum x q - z sum x), with sum x shared by the R rows; M > 1: q - z per
//   code, reused for every batch row).  The constant is never folded into the
//   accumulator: its rounding error would scale with sum |x| rather than with
//   sum |x w'|, and rows whose codes sit mostly at the zero (outlier-heavy
//   per-row grids) would lose the accuracy contract.
// All products x * q and x * (q - z) are exact in fp32 (8-bit x significand
// times a code of at most 9 bits); y is rounded once to bf16.
#include "wq_internal.cuh"

namespace wq {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;


// ---------------------------------------------------------------- unpack plan
// For code i (0..31) of a unit: the word it starts in, the view of that word
// (0: shifted left, 1: as is, 2: shifted right / funnel), and its bit position
// p in that view.
struct Slot {
  int word, view, p;
};

template <int BITS>
__host__ __device__ constexpr int left_shift() { return BITS == 4 ? 12 : 8; }
template <int BITS>
__host__ __device__ constexpr int right_shift() {
  return BITS == 2 ? 10 : BITS == 3 ? 12 : BITS == 4 ? 12 : 16;
}

template <int BITS>
__host__ __device__ constexpr Slot slot(int i) {
  const int bit = BITS * i;
  const int word = bit / 32, P = bit % 32;
  constexpr int L = left_shift<BITS>(), Rs = right_shift<BITS>();
  if (BITS == 8) {           // one code per byte: a view per byte position
    if (P == 0) return {word, 0, 8};
    if (P == 8) return {word, 1, 8};
    if (P == 16) return {word, 3, 8};   // >> 8
    return {word, 2, 8};                // >> 16
  }
  if (P + L + BITS <= 23 && P + L >= 8) return {word, 0, P + L};
  if (P + BITS <= 23 && P >= 8) return {word, 1, P};
  return {word, 2, P - Rs};
}

template <int BITS>
struct Views {
  uint32_t v[BITS][4];
};

template <int BITS>
__device__ __forceinline__ void make_views(const uint32_t (&w)[BITS], Views<BITS>& vw) {
  constexpr int L = left_shift<BITS>(), Rs = right_shift<BITS>();
#pragma unroll
  for (int a = 0; a < BITS; ++a) {
    vw.v[a][0] = w[a] << L;
    vw.v[a][1] = w[a];
    if constexpr (BITS == 3) {
      vw.v[a][2] = (a < 2) ? __funnelshift_r(w[a], w[a + 1 < 3 ? a + 1 : 2], Rs) : (w[a] >> Rs);
    } else {
      vw.v[a][2] = w[a] >> Rs;
    }
    vw.v[a][3] = w[a] >> 8;
  }
}

// (a & mask) | c in one lop3, mask an immediate and c a register.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(MASK), "r"(c));
  return d;
}

// The float 2^(23-p) + q for code i.
template <int BITS, int I>
__device__ __forceinline__ float code_float(const Views<BITS>& vw) {
  constexpr Slot s = slot<BITS>(I);
  constexpr uint32_t mask = ((1u << BITS) - 1u) << s.p;
  constexpr uint32_t expo = uint32_t(150 - s.p) << 23;
  return __uint_as_float(and_or<mask>(vw.v[s.word][s.view], expo));
}
template <int BITS, int I>
__host__ __device__ constexpr float code_bias() {
  return float(1u << (23 - slot<BITS>(I).p));
}

// ---------------------------------------------------------------- loads
template <int BITS>
__device__ __forceinline__ void load_unit(const uint32_t* __restrict__ p, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 2) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p));
    w[0] = v.x; w[1] = v.y;
  } else if constexpr (BITS == 4) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (BITS == 8) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(p));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(p) + 1);
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else {
    w[0] = __ldg(p); w[1] = __ldg(p + 1); w[2] = __ldg(p + 2);
  }
}

// 32 bf16 of x (one unit's k-range) as fp32.
__device__ __forceinline__ void load_x32(const __nv_bfloat16* __restrict__ p, float (&x)[32]) {
  const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 u = __ldg(q + j);
    const uint32_t r[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      x[8 * j + 2 * t] = __uint_as_float(r[t] << 16);
      x[8 * j + 2 * t + 1] = __uint_as_float(r[t] & 0xFFFF0000u);
    }
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int BITS, int I>
struct Unroll {
  // sum_i x_i * f_i over codes I..31 (f: 2^(23-p) + q), and sum_i x_i 2^(23-p_i)
  __device__ __forceinline__ static void dot(const float (&x)[32], const Views<BITS>& vw, float& d0,
                                             float& d1) {
    d0 = fmaf(x[I], code_float<BITS, I>(vw) - code_bias<BITS, I>(), d0);
    if constexpr (I + 1 < 32) {
      d1 = fmaf(x[I + 1], code_float<BITS, I + 1>(vw) - code_bias<BITS, I + 1>(), d1);
      Unroll<BITS, I + 2>::dot(x, vw, d0, d1);
    }
  }
  __device__ __forceinline__ static void xsum(const float (&x)[32], float& s) {
    s += x[I];
    if constexpr (I + 1 < 32) Unroll<BITS, I + 1>::xsum(x, s);
  }
  // exact q - z for codes I..I+7 (c: per-row zero; q = f - 2^(23-p) exactly)
  __device__ __forceinline__ static void qz8(const Views<BITS>& vw, float z, float (&out)[8]) {
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      out[t] = 0.0f;
    }
    Fill<0>::run(vw, z, out);
  }
  template <int T>
  struct Fill {
    __device__ __forceinline__ static void run(const Views<BITS>& vw, float z, float (&out)[8]) {
      out[T] = (code_float<BITS, I + T>(vw) - code_bias<BITS, I + T>()) - z;
      if constexpr (T + 1 < 8) Fill<T + 1>::run(vw, z, out);
    }
  };
};
template <int BITS>
struct Unroll<BITS, 32> {
  __device__ __forceinline__ static void dot(const float (&)[32], const Views<BITS>&, float&, float&) {}
  __device__ __forceinline__ static void xsum(const float (&)[32], float&) {}
};

// ---------------------------------------------------------------- M = 1
template <int BITS, int R>
struct Step {
  uint32_t w[R][BITS];
  float s[R], z[R];
};

template <int BITS, int R>
__device__ __forceinline__ void load_step(Step<BITS, R>& st, const uint32_t* __restrict__ codes,
                                          const __half* __restrict__ scales,
                                          const __half* __restrict__ zeros, int64_t row0,
                                          int64_t N, int64_t KW, int64_t G, int64_t u, int64_t KU,
                                          const FastDiv& upg) {
  const uint32_t grp = upg.div(uint32_t(u < KU ? u : 0));
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const int64_t n = row0 + r;
    if (u < KU && n < N) {
      load_unit<BITS>(codes + n * KW + u * BITS, st.w[r]);
      st.s[r] = __half2float(scales[n * G + grp]);
      st.z[r] = zeros ? __half2float(zeros[n * G + grp]) : float(1 << (BITS - 1));
    } else {
#pragma unroll
      for (int i = 0; i < BITS; ++i) st.w[r][i] = 0u;
      st.s[r] = 0.0f;
      st.z[r] = 0.0f;
    }
  }
}

template <int BITS, int R>
__device__ __forceinline__ void compute_step(const Step<BITS, R>& st, const __nv_bfloat16* __restrict__ xu,
                                             float (&acc)[R]) {
  float xf[32];
  load_x32(xu, xf);
  float sx = 0.0f;
  Unroll<BITS, 0>::xsum(xf, sx);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    Views<BITS> vw;
    make_views<BITS>(st.w[r], vw);
    float d0 = 0.0f, d1 = 0.0f;
    Unroll<BITS, 0>::dot(xf, vw, d0, d1);
    acc[r] = fmaf(st.s[r], fmaf(-st.z[r], sx, d0 + d1), acc[r]);
  }
}

template <int BITS, int R>
__global__ void __launch_bounds__(kThreads, 4)
gemv1_kernel(const __nv_bfloat16* __restrict__ x, int64_t N, int64_t K,
             const uint32_t* __restrict__ codes, const __half* __restrict__ scales,
             const __half* __restrict__ zeros, FastDiv units_per_group,
             __nv_bfloat16* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int64_t row0 = (int64_t(blockIdx.x) * kWarps + (threadIdx.x >> 5)) * R;
  if (row0 >= N) return;
  const int64_t KU = K / 32;                 // units per row
  const int64_t KW = K * BITS / 32;          // words per row
  const int64_t G = K / (int64_t(units_per_group.d) * 32);
  float acc[R];
#pragma unroll
  for (int r = 0; r < R; ++r) acc[r] = 0.0f;

  // Two register buffers: the next step's codes are in flight while the
  // current step is unpacked.
  Step<BITS, R> a, b;
  int64_t u = lane;
  load_step<BITS, R>(a, codes, scales, zeros, row0, N, KW, G, u, KU, units_per_group);
  while (u < KU) {
    load_step<BITS, R>(b, codes, scales, zeros, row0, N, KW, G, u + 32, KU, units_per_group);
    compute_step<BITS, R>(a, x + u * 32, acc);
    u += 32;
    if (u >= KU) break;
    load_step<BITS, R>(a, codes, scales, zeros, row0, N, KW, G, u + 32, KU, units_per_group);
    compute_step<BITS, R>(b, x + u * 32, acc);
    u += 32;
  }
#pragma unroll
  for (int r = 0; r < R; ++r) {
    const float v = warp_sum(acc[r]);
    if (lane == r && row0 + r < N) y[row0 + r] = __float2bfloat16_rn(v);
  }
}

// ---------------------------------------------------------------- 2 <= M <= 16
template <int BITS, int MT, int R>
__global__ void __launch_bounds__(kThreads)
gemvm_kernel(const __nv_bfloat16* __restrict__ x, int M, int64_t N, int64_t K,
             const uint32_t* __restrict__ codes, const __half* __restrict__ scales,
             const __half* __restrict__ zeros, FastDiv units_per_group,
             __nv_bfloat16* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int64_t row0 = (int64_t(blockIdx.x) * kWarps + (threadIdx.x >> 5)) * R;
  if (row0 >= N) return;
  const int64_t KU = K / 32;
  const int64_t KW = K * BITS / 32;
  const int64_t G = K / (int64_t(units_per_group.d) * 32);
  float acc[R][MT];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;

  for (int64_t u = lane; u < KU; u += 32) {
    const uint32_t grp = units_per_group.div(uint32_t(u));
    Views<BITS> vw[R];
    float sc[R], zz[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int64_t n = row0 + r;
      uint32_t w[BITS];
      if (n < N) {
        load_unit<BITS>(codes + n * KW + u * BITS, w);
        sc[r] = __half2float(scales[n * G + grp]);
        zz[r] = zeros ? __half2float(zeros[n * G + grp]) : float(1 << (BITS - 1));
      } else {
#pragma unroll
        for (int i = 0; i < BITS; ++i) w[i] = 0u;
        sc[r] = 0.0f;
        zz[r] = 0.0f;
      }
      make_views<BITS>(w, vw[r]);
    }
    float d[R][MT];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) d[r][m] = 0.0f;
    // 4 chunks of 8 codes: q - z per row once, then every batch row
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float qz[R][8];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        if (c == 0) Unroll<BITS, 0>::qz8(vw[r], zz[r], qz[r]);
        else if (c == 1) Unroll<BITS, 8>::qz8(vw[r], zz[r], qz[r]);
        else if (c == 2) Unroll<BITS, 16>::qz8(vw[r], zz[r], qz[r]);
        else Unroll<BITS, 24>::qz8(vw[r], zz[r], qz[r]);
      }
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        if (m < M) {
          const uint4 xv = __ldg(reinterpret_cast<const uint4*>(x + int64_t(m) * K + u * 32 + 8 * c));
          const uint32_t xr[4] = {xv.x, xv.y, xv.z, xv.w};
          float xf[8];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            xf[2 * t] = __uint_as_float(xr[t] << 16);
            xf[2 * t + 1] = __uint_as_float(xr[t] & 0xFFFF0000u);
          }
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int t = 0; t < 8; ++t) d[r][m] = fmaf(xf[t], qz[r][t], d[r][m]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[r][m] = fmaf(sc[r], d[r][m], acc[r][m]);
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      const float v = warp_sum(acc[r][m]);
      if (lane == 0 && m < M && row0 + r < N) y[int64_t(m) * N + row0 + r] = __float2bfloat16_rn(v);
    }
}

template <int BITS>
cudaError_t launch_bits(const __nv_bfloat16* x, int M, int64_t N, int64_t K,
                        const uint32_t* codes, const __half* scales, const __half* zeros,
                        int64_t g, __nv_bfloat16* y, cudaStream_t st) {
  const FastDiv upg(uint32_t(g / 32));
  auto grid_for = [&](int R) { return dim3(unsigned((N + int64_t(kWarps) * R - 1) / (int64_t(kWarps) * R))); };
  if (M <= 1) {
    if (gemv_m1_tma_supported(x, codes, K, BITS))   // TMA-staged codes and x
      return launch_gemv_m1_tma(x, N, K, codes, scales, zeros, BITS, g, y, st);
    constexpr int R = BITS == 8 ? 2 : 4;
    gemv1_kernel<BITS, R><<<grid_for(R), kThreads, 0, st>>>(x, N, K, codes, scales, zeros, upg, y);
  } else if (M <= 2) {
    gemvm_kernel<BITS, 2, 4><<<grid_for(4), kThreads, 0, st>>>(x, M, N, K, codes, scales, zeros, upg, y);
  } else if (M <= 4) {
    gemvm_kernel<BITS, 4, 4><<<grid_for(4), kThreads, 0, st>>>(x, M, N, K, codes, scales, zeros, upg, y);
  } else if (M <= 8) {
    gemvm_kernel<BITS, 8, 2><<<grid_for(2), kThreads, 0, st>>>(x, M, N, K, codes, scales, zeros, upg, y);
  } else {
    gemvm_kernel<BITS, 16, 2><<<grid_for(2), kThreads, 0, st>>>(x, M, N, K, codes, scales, zeros, upg, y);
  }
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
