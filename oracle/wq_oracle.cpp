// wq_oracle.cpp -- the CPU oracle for weight-only integer-quantised GEMM.
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously correct
// statement of what the library computes; only the tests, the smoke check and
// the benchmark's CPU-baseline leg may load it.  It shares no code, header,
// table or constant with the CUDA library, and the CUDA library never calls it.
//
// What it computes, and where that is defined:
//
//   * The grid.  "OPTQ: Accurate Quantization for Generative Pre-trained
//     Transformers" (reproducibility summary, row "Experiment Setup"): standard
//     uniform asymmetric quantisation on the min-max grid, one grid per row.
//     "Platform For AI: BladeLLM model quantization", section "block_wise_quant":
//     the same parameters per block of input channels instead of per output
//     channel (one (scale, zero) per g consecutive inputs of a row).
//     Written out: scale = (max - min) / (2^b - 1), zero = round(-min / scale),
//     q = clamp(round(w / scale) + zero, 0, 2^b - 1), w' = scale * (q - zero).
//   * Round to nearest.  Same BladeLLM page, "Quantization algorithms > MinMax":
//     codes are the nearest grid point, no calibration data.
//   * Packing.  "[Feature Request] 4bit and 2bit and 1bit quantization support"
//     (onnxruntime issue 14997): several low-bit codes share one machine word
//     (two 4-bit codes per byte; sixteen 2-bit codes per 32-bit word).
//   * Dequantise inside the matmul.  Same issue page (weights stored in 4 bit,
//     converted to float at run time) and the BladeLLM page, section
//     "Background information > Solutions": y = x . W'^T with W' rebuilt from
//     the codes.
//
// Readings where the pages (and the formulas above) leave a point open:
//   R1 the range always contains 0: lo = min(0, min w), hi = max(0, max w);
//   R2 round() is round-half-to-even;
//   R3 scale is stored as fp16 = RNE(exact (hi-lo)/(2^b-1)); zero and codes
//      are computed from that stored fp16 scale;
//   R4 a zero stored scale (all-zero group, or a range that underflows fp16)
//      becomes scale 1, zero 0;
//   R5 zero is not clamped; it is a non-negative integer stored exactly in fp16,
//      with a clear sign bit;
//   R6 group 0 or group K means one (scale, zero) per row;
//   S1 the symmetric grid ("Platform For AI: BladeLLM model quantization",
//      "Quantization modes > weight_only_quant": signed symmetric quantisation
//      by default): a = max |w| over the group, scale = fp16 RNE of
//      a / (2^(b-1) - 1) (1 if that is 0), the zero fixed at 2^(b-1) and not
//      stored; the codes are the same RTN codes on that grid, so the signed
//      value q - 2^(b-1) of +-a is +-(2^(b-1) - 1), and the extra code 0 is
//      only reached by rounding or a scale rounded down;
//   R7 packing is LSB-first along K: for b in {2,4,8} code k sits in word
//      k / (32/b) at bit b*(k mod 32/b); for b = 3 the 32 codes of unit
//      u = k/32 fill the 96-bit little-endian value of words 3u..3u+2, code
//      j = k mod 32 at bit 3j (codes 10 and 21 straddle two words).
//
//   * Error-compensating quantisation (OPTQ).  "OPTQ: Accurate Quantization
//     for Generative Pre-trained Transformers" (reproducibility summary, rows
//     "Experiment Setup" and "Pseudocode") and "Platform For AI: BladeLLM model
//     quantization", "Quantization algorithms > GPTQ": the columns of a row are
//     quantised one after another; after each, the error it leaves is made up
//     by adjusting the columns not yet quantised through the inverse of the
//     layer Hessian of the calibration activations.  Readings:
//   O1 the Hessian is H = (2 / S) X^T X over S calibration rows x (any positive
//      factor gives the same codes: it cancels, damping included);
//   O2 damping: H + d I with d = percdamp * mean(diag H) (percdamp 0.01 by
//      default); if every diagonal entry is 0, H is replaced by I;
//   O3 a group's grid (R1-R5) is computed from the compensated weights of the
//      whole group when its first column comes up, and then stays fixed;
//   O4 columns are taken in their natural order; the grid rules apply to the
//      fp64 compensated weights as they are (no rounding to fp16 first);
//   O5 each step's compensation is the least-squares re-fit: after columns
//      0..k are fixed to their grid values w', the free columns F = k+1..K-1
//      become w0_F - H_FF^-1 H_F,Q (w'_Q - w0_Q) (Q = 0..k, w0 the fp16
//      weights, H damped).  Carried out step by step this is
//        e = (w_k - w'_k) / A_kk;  w_j -= e A_kj  (j > k)
//      with A the inverse of H restricted to the columns free before step k;
//      A is then reduced by eliminating column k.
//
// Everything is computed in fp64.  fp16 and bf16 are decoded and rounded here
// from the IEEE 754 binary16 / bfloat16 definitions (no library conversion).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

// ---------------------------------------------------------------- formats
// A small binary floating-point format with `ebits` exponent bits and `mbits`
// stored fraction bits (binary16: 5/10, bfloat16: 8/7).
struct Fmt {
  int ebits, mbits;
  int bias() const { return (1 << (ebits - 1)) - 1; }
  int emin() const { return 1 - bias(); }   // exponent of the smallest normal
  int emax() const { return bias(); }       // exponent of the largest finite
};
constexpr Fmt kF16{5, 10};
constexpr Fmt kBF16{8, 7};

double decode(uint32_t bits, Fmt f) {
  const uint32_t sign = bits >> (f.ebits + f.mbits);
  const uint32_t e = (bits >> f.mbits) & ((1u << f.ebits) - 1);
  const uint32_t m = bits & ((1u << f.mbits) - 1);
  double v;
  if (e == 0) {
    v = std::ldexp(double(m), f.emin() - f.mbits);              // subnormal or zero
  } else if (e == (1u << f.ebits) - 1) {
    v = m ? std::nan("") : INFINITY;
  } else {
    v = std::ldexp(double(m | (1u << f.mbits)), int(e) - f.bias() - f.mbits);
  }
  return sign ? -v : v;
}

// Round a double to the nearest value of format f, ties to even; returns bits.
uint32_t encode_rne(double d, Fmt f) {
  const int nb = f.ebits + f.mbits;
  const uint32_t sign = std::signbit(d) ? (1u << nb) : 0u;
  const uint32_t inf = ((1u << f.ebits) - 1) << f.mbits;
  if (std::isnan(d)) return inf | (1u << (f.mbits - 1));
  const double a = std::fabs(d);
  // Largest finite is (2 - 2^-mbits) * 2^emax; halfway to the next binade's
  // first value rounds to it (its fraction is odd), so that halfway overflows.
  const double overflow = std::ldexp(2.0 - std::ldexp(1.0, -f.mbits - 1), f.emax());
  if (a >= overflow) return sign | inf;
  if (a == 0.0) return sign;
  int e2;
  std::frexp(a, &e2);            // a in [2^(e2-1), 2^e2)
  int E = std::max(e2 - 1, f.emin());
  const double quantum = std::ldexp(1.0, E - f.mbits);
  const double r = std::nearbyint(a / quantum);   // exact scaling; RNE
  const double v = r * quantum;                   // representable in f
  if (v == 0.0) return sign;
  std::frexp(v, &e2);
  E = e2 - 1;
  if (E < f.emin()) {            // subnormal
    return sign | uint32_t(v / std::ldexp(1.0, f.emin() - f.mbits));
  }
  const uint32_t frac = uint32_t(v / std::ldexp(1.0, E - f.mbits)) - (1u << f.mbits);
  return sign | (uint32_t(E + f.bias()) << f.mbits) | frac;
}

double f16(uint16_t h) { return decode(h, kF16); }
uint16_t to_f16(double d) { return uint16_t(encode_rne(d, kF16)); }
double bf16(uint16_t h) { return decode(h, kBF16); }

// ---------------------------------------------------------------- checks
bool valid_bits(int b) { return b == 2 || b == 3 || b == 4 || b == 8; }

// Per-row when group is 0 or K (R6); otherwise a multiple of 32 dividing K.
int64_t effective_group(int64_t K, int64_t group) {
  if (group == 0 || group == K) return K;
  if (group < 0 || group % 32 != 0 || K % group != 0) return -1;
  return group;
}

int64_t words_per_row(int64_t K, int bits) { return K * bits / 32; }

template <class F>
void parallel_rows(int64_t n, int nthreads, F&& body) {
  if (nthreads <= 0) nthreads = int(std::max(1u, std::thread::hardware_concurrency()));
  nthreads = int(std::min<int64_t>(nthreads, std::max<int64_t>(n, 1)));
  if (nthreads <= 1) {
    for (int64_t i = 0; i < n; ++i) body(i);
    return;
  }
  std::vector<std::thread> pool;
  for (int t = 0; t < nthreads; ++t) {
    pool.emplace_back([&, t] {
      for (int64_t i = t; i < n; i += nthreads) body(i);
    });
  }
  for (auto& th : pool) th.join();
}

// ---------------------------------------------------------------- packing (R7)
void pack_row(const uint8_t* q, int64_t K, int bits, uint32_t* w) {
  const int64_t nw = words_per_row(K, bits);
  std::memset(w, 0, size_t(nw) * 4);
  if (bits == 3) {
    for (int64_t k = 0; k < K; ++k) {
      const int64_t u = k / 32, j = k % 32;
      const int bit = int(3 * j);
      const int64_t wi = 3 * u + bit / 32;
      const int off = bit % 32;
      w[wi] |= uint32_t(q[k]) << off;
      if (off > 29) w[wi + 1] |= uint32_t(q[k]) >> (32 - off);
    }
  } else {
    const int per = 32 / bits;
    for (int64_t k = 0; k < K; ++k)
      w[k / per] |= uint32_t(q[k]) << (bits * (k % per));
  }
}

void unpack_row(const uint32_t* w, int64_t K, int bits, uint8_t* q) {
  const uint32_t mask = (1u << bits) - 1;
  if (bits == 3) {
    for (int64_t k = 0; k < K; ++k) {
      const int64_t u = k / 32, j = k % 32;
      const int bit = int(3 * j);
      const int64_t wi = 3 * u + bit / 32;
      const int off = bit % 32;
      uint32_t v = w[wi] >> off;
      if (off > 29) v |= w[wi + 1] << (32 - off);
      q[k] = uint8_t(v & mask);
    }
  } else {
    const int per = 32 / bits;
    for (int64_t k = 0; k < K; ++k) q[k] = uint8_t((w[k / per] >> (bits * (k % per))) & mask);
  }
}

}  // namespace

extern "C" {

// ------------------------------------------------ format conversions (tests)
void orc_f16_to_f64(const uint16_t* h, double* d, int64_t n) {
  for (int64_t i = 0; i < n; ++i) d[i] = f16(h[i]);
}
void orc_f64_to_f16(const double* d, uint16_t* h, int64_t n) {
  for (int64_t i = 0; i < n; ++i) h[i] = to_f16(d[i]);
}
void orc_bf16_to_f64(const uint16_t* h, double* d, int64_t n) {
  for (int64_t i = 0; i < n; ++i) d[i] = bf16(h[i]);
}
void orc_f64_to_bf16(const double* d, uint16_t* h, int64_t n) {
  for (int64_t i = 0; i < n; ++i) h[i] = uint16_t(encode_rne(d[i], kBF16));
}

// ------------------------------------------------ quantise (round to nearest)
// W: fp16 bit patterns [N, K] row-major.  Outputs: unpacked codes q [N, K]
// (uint8), scales and zeros as fp16 bit patterns [N, G] with G = K / group
// (G = 1 per-row).  Returns 0, or -1 on an invalid argument (nothing written).
int orc_quantize_rtn(const uint16_t* W, int64_t N, int64_t K, int bits, int64_t group,
                     uint8_t* q, uint16_t* scales, uint16_t* zeros, int nthreads) {
  if (!W || !q || !scales || !zeros || N < 1 || K < 1 || K % 32 != 0 || !valid_bits(bits))
    return -1;
  const int64_t g = effective_group(K, group);
  if (g < 0) return -1;
  const int64_t G = K / g;
  const double qmax = double((1 << bits) - 1);
  parallel_rows(N, nthreads, [&](int64_t n) {
    const uint16_t* wr = W + n * K;
    for (int64_t j = 0; j < G; ++j) {
      // R1: the range always includes 0.
      double lo = 0.0, hi = 0.0;
      for (int64_t k = j * g; k < (j + 1) * g; ++k) {
        const double w = f16(wr[k]);
        lo = std::min(lo, w);
        hi = std::max(hi, w);
      }
      // R3: fp16 scale, one rounding of the (exact in fp64) quotient.
      double s = f16(to_f16((hi - lo) / qmax));
      double z;
      if (s == 0.0) {           // R4
        s = 1.0;
        z = 0.0;
      } else {
        z = std::nearbyint((0.0 - lo) / s);   // R2, R5 (0.0 - lo is never -0)
      }
      scales[n * G + j] = to_f16(s);
      zeros[n * G + j] = to_f16(z);
      for (int64_t k = j * g; k < (j + 1) * g; ++k) {
        double c = std::nearbyint(f16(wr[k]) / s) + z;
        c = std::min(std::max(c, 0.0), qmax);
        q[n * K + k] = uint8_t(c);
      }
    }
  });
  return 0;
}

// ------------------------------------------------ quantise, symmetric grid (S1)
// Same layout as orc_quantize_rtn; no zeros output (every zero is 2^(b-1)).
int orc_quantize_rtn_sym(const uint16_t* W, int64_t N, int64_t K, int bits, int64_t group,
                         uint8_t* q, uint16_t* scales, int nthreads) {
  if (!W || !q || !scales || N < 1 || K < 1 || K % 32 != 0 || !valid_bits(bits)) return -1;
  const int64_t g = effective_group(K, group);
  if (g < 0) return -1;
  const int64_t G = K / g;
  const double qmax = double((1 << bits) - 1);
  const double z = double(1 << (bits - 1));
  const double top = z - 1.0;                 // signed code of +a
  parallel_rows(N, nthreads, [&](int64_t n) {
    const uint16_t* wr = W + n * K;
    for (int64_t j = 0; j < G; ++j) {
      double a = 0.0;
      for (int64_t k = j * g; k < (j + 1) * g; ++k) a = std::max(a, std::fabs(f16(wr[k])));
      double s = f16(to_f16(a / top));
      if (s == 0.0) s = 1.0;                  // all-zero group or underflow (as R4)
      scales[n * G + j] = to_f16(s);
      for (int64_t k = j * g; k < (j + 1) * g; ++k) {
        double c = std::nearbyint(f16(wr[k]) / s) + z;
        c = std::min(std::max(c, 0.0), qmax);
        q[n * K + k] = uint8_t(c);
      }
    }
  });
  return 0;
}

// ------------------------------------------------ quantise with error compensation (OPTQ)
// W: fp16 bit patterns [N, K]; H: fp64 [K, K], symmetric positive
// semi-definite (only its lower triangle is read).  Outputs as for
// orc_quantize_rtn; u (optional, fp64 [N, K]) receives each weight as it was
// when its column came up (after the compensation of the earlier columns).
// Returns 0, -1 on an invalid argument, -2 if the damped H is not positive
// definite (nothing written).
int orc_quantize_optq(const uint16_t* W, const double* H, int64_t N, int64_t K, int bits,
                      int64_t group, double percdamp, uint8_t* q, uint16_t* scales,
                      uint16_t* zeros, double* u, int nthreads) {
  if (!W || !H || !q || !scales || !zeros || N < 1 || K < 1 || !valid_bits(bits) ||
      !(percdamp >= 0.0))
    return -1;
  const int64_t g = effective_group(K, group);
  if (g < 0) return -1;
  const int64_t G = K / g;
  const double qmax = double((1 << bits) - 1);
  const size_t KK = size_t(K) * size_t(K);

  // O2: damped Hessian (lower triangle, full storage).
  std::vector<double> Hd(KK, 0.0);
  double mean_diag = 0.0;
  for (int64_t i = 0; i < K; ++i) mean_diag += H[i * K + i];
  mean_diag /= double(K);
  for (int64_t i = 0; i < K; ++i)
    for (int64_t j = 0; j <= i; ++j)
      Hd[i * K + j] = mean_diag == 0.0 ? (i == j ? 1.0 : 0.0) : H[i * K + j];
  if (mean_diag != 0.0)
    for (int64_t i = 0; i < K; ++i) Hd[i * K + i] += percdamp * mean_diag;

  // A = Hd^-1 through the Cholesky factor Hd = L L^T: A = L^-T L^-1.
  std::vector<double> L(KK, 0.0);
  for (int64_t j = 0; j < K; ++j) {
    double d = Hd[j * K + j];
    for (int64_t p = 0; p < j; ++p) d -= L[j * K + p] * L[j * K + p];
    if (!(d > 0.0)) return -2;
    const double ljj = std::sqrt(d);
    L[j * K + j] = ljj;
    for (int64_t i = j + 1; i < K; ++i) {
      double v = Hd[i * K + j];
      for (int64_t p = 0; p < j; ++p) v -= L[i * K + p] * L[j * K + p];
      L[i * K + j] = v / ljj;
    }
  }
  std::vector<double> Li(KK, 0.0);   // L^-1, lower triangular
  for (int64_t c = 0; c < K; ++c) {
    Li[c * K + c] = 1.0 / L[c * K + c];
    for (int64_t i = c + 1; i < K; ++i) {
      double v = 0.0;
      for (int64_t p = c; p < i; ++p) v -= L[i * K + p] * Li[p * K + c];
      Li[i * K + c] = v / L[i * K + i];
    }
  }
  std::vector<double> A(KK, 0.0);
  for (int64_t i = 0; i < K; ++i)
    for (int64_t j = 0; j < K; ++j) {
      double v = 0.0;
      for (int64_t p = std::max(i, j); p < K; ++p) v += Li[p * K + i] * Li[p * K + j];
      A[i * K + j] = v;
    }

  // O5: the pivot and the row of A each step uses; A then loses column k.
  // Every row of W meets the same sequence, so it is recorded once.
  std::vector<double> piv(static_cast<size_t>(K));
  std::vector<double> arow(KK, 0.0);   // arow[k*K + j] = A_kj at step k, j > k
  for (int64_t k = 0; k < K; ++k) {
    const double akk = A[k * K + k];
    piv[size_t(k)] = akk;
    for (int64_t j = k + 1; j < K; ++j) arow[k * K + j] = A[k * K + j];
    for (int64_t i = k + 1; i < K; ++i) {
      const double f = A[i * K + k] / akk;
      for (int64_t j = k + 1; j < K; ++j) A[i * K + j] -= f * A[k * K + j];
    }
  }

  parallel_rows(N, nthreads, [&](int64_t n) {
    std::vector<double> w(static_cast<size_t>(K));
    for (int64_t k = 0; k < K; ++k) w[size_t(k)] = f16(W[n * K + k]);
    double s = 1.0, z = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      if (k % g == 0) {
        // O3: the group's grid from its current (compensated) weights, R1-R5.
        const int64_t j = k / g;
        double lo = 0.0, hi = 0.0;
        for (int64_t c = k; c < k + g; ++c) {
          lo = std::min(lo, w[size_t(c)]);
          hi = std::max(hi, w[size_t(c)]);
        }
        s = f16(to_f16((hi - lo) / qmax));
        if (s == 0.0) {
          s = 1.0;
          z = 0.0;
        } else {
          z = std::nearbyint((0.0 - lo) / s);
        }
        scales[n * G + j] = to_f16(s);
        zeros[n * G + j] = to_f16(z);
      }
      const double wk = w[size_t(k)];
      if (u) u[n * K + k] = wk;
      double c = std::nearbyint(wk / s) + z;
      c = std::min(std::max(c, 0.0), qmax);
      q[n * K + k] = uint8_t(c);
      const double e = (wk - s * (c - z)) / piv[size_t(k)];
      for (int64_t j = k + 1; j < K; ++j) w[size_t(j)] -= e * arow[k * K + j];
    }
  });
  return 0;
}

// ------------------------------------------------ packing (R7)
int orc_pack(const uint8_t* q, int64_t N, int64_t K, int bits, uint32_t* words) {
  if (!q || !words || N < 1 || K < 1 || K % 32 != 0 || !valid_bits(bits)) return -1;
  const int64_t nw = words_per_row(K, bits);
  for (int64_t n = 0; n < N; ++n) pack_row(q + n * K, K, bits, words + n * nw);
  return 0;
}

int orc_unpack(const uint32_t* words, int64_t N, int64_t K, int bits, uint8_t* q) {
  if (!q || !words || N < 1 || K < 1 || K % 32 != 0 || !valid_bits(bits)) return -1;
  const int64_t nw = words_per_row(K, bits);
  for (int64_t n = 0; n < N; ++n) unpack_row(words + n * nw, K, bits, q + n * K);
  return 0;
}

// ------------------------------------------------ dequantise: w' = s (q - z)
int orc_dequant(const uint8_t* q, const uint16_t* scales, const uint16_t* zeros, int64_t N,
                int64_t K, int64_t group, double* wq) {
  if (!q || !scales || !zeros || !wq || N < 1 || K < 1) return -1;
  const int64_t g = effective_group(K, group);
  if (g < 0) return -1;
  const int64_t G = K / g;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      const int64_t j = k / g;
      wq[n * K + k] = f16(scales[n * G + j]) * (double(q[n * K + k]) - f16(zeros[n * G + j]));
    }
  return 0;
}

// ------------------------------------------------ y = x . W'^T in fp64
// x: bf16 bit patterns [M, K].  words/scales/zeros: packed codes and fp16
// parameters of all N rows.  cols: the output columns n to compute (NULL means
// all N, in order); y and bound are [M, ncols] fp64, bound = sum_k |x w'|.
int orc_gemm(const uint16_t* x, int64_t M, int64_t N, int64_t K, const uint32_t* words,
             const uint16_t* scales, const uint16_t* zeros, int bits, int64_t group,
             const int64_t* cols, int64_t ncols, double* y, double* bound, int nthreads) {
  if (!x || !words || !scales || !zeros || !y || M < 1 || N < 1 || K < 1 || K % 32 != 0 ||
      !valid_bits(bits))
    return -1;
  const int64_t g = effective_group(K, group);
  if (g < 0) return -1;
  if (!cols) ncols = N;
  for (int64_t i = 0; cols && i < ncols; ++i)
    if (cols[i] < 0 || cols[i] >= N) return -1;
  const int64_t G = K / g;
  const int64_t nw = words_per_row(K, bits);
  std::vector<double> xd(static_cast<size_t>(M * K));
  for (int64_t i = 0; i < M * K; ++i) xd[i] = bf16(x[i]);
  parallel_rows(ncols, nthreads, [&](int64_t c) {
    const int64_t n = cols ? cols[c] : c;
    std::vector<uint8_t> q(static_cast<size_t>(K));
    std::vector<double> w(static_cast<size_t>(K));
    unpack_row(words + n * nw, K, bits, q.data());
    for (int64_t k = 0; k < K; ++k) {
      const int64_t j = k / g;
      w[k] = f16(scales[n * G + j]) * (double(q[k]) - f16(zeros[n * G + j]));
    }
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0, b = 0.0;
      const double* xr = xd.data() + m * K;
      for (int64_t k = 0; k < K; ++k) {
        acc += xr[k] * w[k];
        b += std::fabs(xr[k] * w[k]);
      }
      y[m * ncols + c] = acc;
      if (bound) bound[m * ncols + c] = b;
    }
  });
  return 0;
}

}  // extern "C"
