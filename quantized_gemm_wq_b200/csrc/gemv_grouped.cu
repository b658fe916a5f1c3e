// gemv_grouped.cu -- decode y_l = x_l . W'_l^T for a list of linears l in one
// persistent launch (1 to 16 tokens), codes dequantised on the fly.
//
// Dequantise inside the matmul ("[Feature Request] 4bit and 2bit and 1bit
// quantization support": packed weights turn into floats on the GPU when
// used); decoding is bound by the bytes of packed weights read from GPU memory
// ("Platform For AI: BladeLLM model quantization", "Background information >
// Solutions" and "Quantization modes > weight_only_quant").  A decode step
// runs many small linears back to back; launched one by one, each pays a ramp
// (launch, first copies in flight, tail wave) that is as long as its transfer.
// Here every linear of the list is cut into tiles of 32 output rows, each tile
// into stages of 1024 codes of K, and the concatenated stage sequence is split
// into P equal contiguous ranges, one per persistent CTA (stream-K).  A CTA's
// TMA ring runs on across tile and linear boundaries, so the copies of the
// next tile are in flight while the current one is reduced.
//
// Stage contents (one ring slot), all completing on the slot's "full"
// mbarrier:
//   codes   TMA box of 32 rows x 32 units (BITS boxes of 32 rows x 128 bytes,
//           128-byte swizzle, rows past N / columns past K zero-filled);
//   x'      the stage's activations as MMA B fragments (bulk copy from the
//           workspace, written by xprep_kernel): for token m and code slot k,
//           x 2^(64 - b), b the code's bit offset in its 16-bit half;
//   sum x   per 128-code quad and token (bulk copy from the workspace);
//   (s, z)  the raw fp16 scales and zeros of the stage's groups for the 32
//           rows: each lane of the producer warp copies its row's window with
//           4-byte cp.async copies that arrive on the same barrier when they
//           land, so the producer never waits for them.
// Warp 8 is the producer; warps 0..7 consume, warp w quad w of every stage,
// exactly as in the 2..8-token GEMV (gemv_mma.cu): lane (g, t) unpacks unit
// 4w + t of rows g, g + 8, g + 16, g + 24 with one AND per two codes into the
// bf16 patterns q 2^(b-133) and issues mma.sync m16n8k16 against the tokens'
// x' (columns past the batch read a zero block; 16 tokens use two MMAs per A
// fragment).  Every product is q x 2^-69 exactly; per scale group the
// accumulators are folded into s (D 2^69 - z sum x).  At the end of a tile
// the warps' partial sums meet in shared memory (fixed order) and y is
// rounded once to bf16.  A tile cut between CTAs is finished by whichever of
// its CTAs arrives last on the tile's workspace counter: it adds the parked
// partial sums in CTA order (deterministic) and resets the counter.  No CTA
// ever waits for another.
#include <cuda.h>   // CUtensorMap

#include <atomic>

#include "grouped.h"
#include "stage_smem.cuh"
#include "unpack_tables.h"
#include "wq_internal.cuh"

namespace wq {

__device__ unsigned int g_gemv_grouped_timeout;

namespace {

using namespace stg;

constexpr int kNW = 8;                        // consumer warps
constexpr int kThreads = 32 * (kNW + 1);
// Words per row of an (s, z) slot: up to 9 halves of scales (8 groups and an
// odd start) in 5 words, then 5 words of zeros.  10 words apart, the rows
// g = 0..7 a consumer lane reads fall in distinct banks.
constexpr int kSzW = 5;
constexpr int kSzRow = 2 * kSzW;

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity) {
  return bw::pipe_wait(bar, parity, &g_gemv_grouped_timeout, nullptr);
}

template <int BITS>
__host__ __device__ constexpr const UnpackOp* unit_table() {
  if constexpr (BITS == 2) return kUnit2;
  else if constexpr (BITS == 3) return kUnit3;
  else if constexpr (BITS == 4) return kUnit4;
  else return kUnit8;
}

// AND T of the unit table applied to a unit's words: two bf16 code patterns.
template <int BITS, int T>
__device__ __forceinline__ uint32_t unit_pair(const uint32_t (&w)[BITS]) {
  constexpr UnpackOp op = unit_table<BITS>()[T];
  constexpr int k = op.s / 32, sh = op.s % 32;
  uint32_t win;
  if constexpr (sh == 0) {
    win = w[k];
  } else if constexpr (k + 1 < BITS) {
    win = __funnelshift_r(w[k], w[k + 1], sh);
  } else {
    win = w[k] >> sh;
  }
  return win & op.mask;
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same MMA with a zero accumulator input: D = A B.
__device__ __forceinline__ void mma_bf16_z(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
  const float z = 0.0f;
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%10, %10, %10, %10};"
      : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
}

// Accumulators of a lane for one quad: [tile][chain][4], tile 0 the rows of
// the lane's first A fragment pair (words w[0], w[1]), tile 1 the next
// (w[2], w[3]); chain J % 2, so consecutive MMAs of a tile do not wait for
// each other.  `h` selects the second 8-token half (16 tokens only).
struct QuadAcc {
  float c[2][2][4];
};

// MMA J..7 of 16-row tile T over a quad (A rows from the words wa, wb)
// against one 8-token B operand (xb); with TWO the same A fragments also meet
// the second 8-token operand (xb2).  FRESH: the first MMA of each chain
// starts from zero instead of adding to the accumulators.
template <int BITS, int T, int J, bool TWO, bool FRESH>
struct QuadMma {
  __device__ __forceinline__ static void run(QuadAcc& a, QuadAcc& a2, const uint32_t (&wa)[BITS],
                                             const uint32_t (&wb)[BITS], const uint32_t (&xb)[16],
                                             const uint32_t (&xb2)[16]) {
    const uint32_t a0 = unit_pair<BITS, 2 * J>(wa), a1 = unit_pair<BITS, 2 * J>(wb);
    const uint32_t a2r = unit_pair<BITS, 2 * J + 1>(wa), a3 = unit_pair<BITS, 2 * J + 1>(wb);
    if constexpr (FRESH && J < 2) {
      mma_bf16_z(a.c[T][J & 1], a0, a1, a2r, a3, xb[2 * J], xb[2 * J + 1]);
      if constexpr (TWO) mma_bf16_z(a2.c[T][J & 1], a0, a1, a2r, a3, xb2[2 * J], xb2[2 * J + 1]);
    } else {
      mma_bf16(a.c[T][J & 1], a0, a1, a2r, a3, xb[2 * J], xb[2 * J + 1]);
      if constexpr (TWO) mma_bf16(a2.c[T][J & 1], a0, a1, a2r, a3, xb2[2 * J], xb2[2 * J + 1]);
    }
    if constexpr (J + 1 < 8) QuadMma<BITS, T, J + 1, TWO, FRESH>::run(a, a2, wa, wb, xb, xb2);
  }
};

// Weight row (within an 8-row group) fed to MMA row g: an order in which the
// 8 lanes of each quarter-warp load 8 distinct 16-byte bank groups from the
// 128-byte-swizzled code boxes (2-bit and 4-bit units; 3-bit and 8-bit
// units are conflict-free in the plain order).
template <int BITS>
__host__ __device__ constexpr int mma_row(int g) {
  if constexpr (BITS == 4) return (g >> 1) | ((g & 1) << 2);
  else if constexpr (BITS == 2) return ((g & 1) << 2) | (g & 2) | ((g >> 2) & 1);
  else return g;
}

// The fields of the linear a CTA is working on, in registers.
struct LinRegs {
  const __half* scales;
  const __half* zeros;
  __nv_bfloat16* y;
  const uint32_t* xp;
  const float* sx;
  int64_t stage0;
  int N, K, G, TS, tiles;
  FastDiv upg;
  // Groups that tile a 1024-code stage (g = 128, 256, 512, 1024): a warp's
  // quad of every stage is in a new group, the group's index in the stage is
  // warp >> qshift, the stage's first group is 8 t >> qshift.
  bool tiles_stage;
  int qshift;
  __device__ __forceinline__ void load(const GLin& L) {
    scales = L.scales;
    zeros = L.zeros;
    y = L.y;
    xp = L.xp;
    sx = L.sx;
    stage0 = L.stage0;
    N = L.N;
    K = L.K;
    G = L.G;
    TS = L.TS;
    tiles = L.tiles;
    upg = L.upg;
    const int qpg = int(upg.d) >> 2;        // 128-code quads per group
    tiles_stage = qpg <= 8 && (8 % qpg) == 0;
    qshift = qpg >= 8 ? 3 : (qpg >= 4 ? 2 : (qpg >= 2 ? 1 : 0));
  }
};

// Code offsets (in the unit) and activation factors 2^(64 - b) of pair t of
// the unit table, for a pair index known only at run time.
template <int BITS, int T>
struct PairPick {
  __device__ __forceinline__ static void run(int t, int& lo, int& hi, float& flo, float& fhi) {
    constexpr UnpackOp op = unit_table<BITS>()[T];
    if (T == t) {
      lo = op.lo;
      hi = op.hi;
      flo = __int_as_float((127 + 64 - int(op.blo)) << 23);
      fhi = __int_as_float((127 + 64 - int(op.bhi)) << 23);
    }
    if constexpr (T + 1 < 16) PairPick<BITS, T + 1>::run(t, lo, hi, flo, fhi);
  }
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 16-byte chunk c of a quad's x' area (c = (token * 4 + unit) * 4 + i, chunk i
// holding pairs 4i..4i+3 of the unit) is stored at chunk position
// (c & ~7) | ((c ^ (c >> 3)) & 7): the 8 lanes of each quarter-warp then read
// 8 distinct 16-byte bank groups.
__host__ __device__ constexpr int xp_chunk_pos(int c) { return (c & ~7) | ((c ^ (c >> 3)) & 7); }

template <int MT>
struct Tok {
  static constexpr int SXW = MT < 4 ? 4 : MT;     // floats of sum x per quad (16-byte multiple)
  // accumulator columns per lane (column 2 tq + 1 never holds a token when MT = 1)
  static constexpr int NC = MT == 16 ? 4 : (MT == 1 ? 1 : 2);
};

// ---------------------------------------------------------------------------
// x' and the per-quad sums, once per call (every row tile reads them).
// One warp per (linear, quad, token); lane l covers unit l / 8 of the quad,
// pairs 2 (l % 8) and 2 (l % 8) + 1.
template <int BITS, int MT>
__global__ void __launch_bounds__(256) xprep_kernel(const __grid_constant__ PrepParams pp) {
  const int li = int(blockIdx.y);
  if (li >= pp.nlin) return;
  const PrepLin& L = pp.lin[li];
  const int wid = int(blockIdx.x) * 8 + int(threadIdx.x >> 5), lane = int(threadIdx.x & 31);
  const int nq = L.K / 128;
  if (wid >= nq * MT) return;
  const int q = wid / MT, m = wid % MT;
  const int tq = lane >> 3, p0 = 2 * (lane & 7);
  const bool live = m < pp.M;
  const __nv_bfloat16* xr = L.x + int64_t(live ? m : 0) * L.K + int64_t(q) * 128 + 32 * tq;
  uint32_t wv[2];
  float sum = 0.0f;
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    int lo = 0, hi = 0;
    float flo = 0.0f, fhi = 0.0f;
    PairPick<BITS, 0>::run(p0 + j, lo, hi, flo, fhi);
    const float xl = live ? __bfloat162float(xr[lo]) : 0.0f;
    const float xh = live ? __bfloat162float(xr[hi]) : 0.0f;
    wv[j] = pack_bf16x2(xl * flo, xh * fhi);
    sum += xl + xh;
  }
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
  // stage t = q / 8, quad w = q % 8 of that stage
  const int t = q >> 3, w = q & 7;
  const int c = (m * 4 + tq) * 4 + (p0 >> 2);
  uint32_t* dst = L.xp + int64_t(t) * MT * 512 + w * MT * 64 + xp_chunk_pos(c) * 4 + (p0 & 3);
  *reinterpret_cast<uint2*>(dst) = make_uint2(wv[0], wv[1]);
  if (lane == 0) L.sx[int64_t(q) * Tok<MT>::SXW + m] = sum;
}

// ---------------------------------------------------------------------------
template <int BITS, int MT, int D>
struct GCfg {
  static constexpr int SB = BITS * 4096;                  // codes: 32 rows x 32 units
  static constexpr int XB = MT * 2048;                    // x': 8 quads x MT tokens x 256 B
  static constexpr int SXB = 8 * Tok<MT>::SXW * 4;        // sums per quad and token
  static constexpr int SZB = 32 * kSzRow * 4;             // raw (s, z) of 32 rows x up to 8 groups
  // tile reduction buffers: with one or two tokens the warps meet through a
  // per-buffer counter instead of a barrier, and a warp may run D tiles ahead
  static constexpr int RB = MT <= 2 ? D + 1 : (MT <= 8 ? 2 : 1);
  static constexpr int REDB = RB * kNW * MT * 32 * 4;
  static constexpr int OFF_XP = D * SB;
  static constexpr int OFF_SX = OFF_XP + D * XB;
  static constexpr int OFF_SZ = OFF_SX + D * SXB;
  static constexpr int OFF_RED = OFF_SZ + D * SZB;
  static constexpr int OFF_ZERO = OFF_RED + REDB;         // 64 zero bytes: B of empty token columns
  static constexpr int OFF_BAR = OFF_ZERO + 64;           // full[D], empty[D]
  static constexpr int OFF_FLAG = OFF_BAR + 16 * D;
  static constexpr int OFF_TCNT = OFF_FLAG + 16;           // arrivals per reduction buffer
  static constexpr int BYTES = OFF_TCNT + 4 * RB + 1024;   // + alignment slack
};

// Position in a CTA's stage range: linear l, row tile r, stage t of the tile.
struct Pos {
  int l, t;
  int64_t r;
};

__device__ __forceinline__ Pos locate(const GParams& p, int64_t s) {
  int l = 0;
  while (l + 1 < p.nlin && p.lin[l + 1].stage0 <= s) ++l;
  const int64_t off = s - p.lin[l].stage0;
  const int TS = p.lin[l].TS;
  return Pos{l, int(off % TS), off / TS};
}
// First stage of CTA c's range.
__device__ __forceinline__ int64_t range_start(const GParams& p, int64_t c) { return p.total * c / p.P; }

template <int BITS, int MT, int D, int MINB>
__global__ void __launch_bounds__(kThreads, MINB) gemv_grouped_kernel(const __grid_constant__ GParams p) {
  using C = GCfg<BITS, MT, D>;
  constexpr int NC = Tok<MT>::NC, SXW = Tok<MT>::SXW;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (saddr(smem_raw) & 1023)) & 1023);
  const int warp = int(threadIdx.x >> 5), lane = int(threadIdx.x & 31);
  const uint32_t ring = saddr(smem);
  const uint32_t xps = ring + C::OFF_XP, sxs = ring + C::OFF_SX;
  const uint32_t full0 = ring + C::OFF_BAR, empty0 = full0 + 8 * D;
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  volatile int* flag = reinterpret_cast<volatile int*>(smem + C::OFF_FLAG);

  const int64_t cta = blockIdx.x;
  const int64_t sb = range_start(p, cta), se = range_start(p, cta + 1);
  const int T = int(se - sb);

  if (threadIdx.x == 0) {
    for (int s = 0; s < D; ++s) {
      // full: the producer's expect-tx arrive + one arrive per producer lane
      // (its scale/zero copies)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 33;" ::"r"(full0 + 8 * s));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty0 + 8 * s), "r"(kNW));
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (threadIdx.x < 16) reinterpret_cast<uint32_t*>(smem + C::OFF_ZERO)[threadIdx.x] = 0u;
  if (threadIdx.x < C::RB) reinterpret_cast<unsigned*>(smem + C::OFF_TCNT)[threadIdx.x] = 0u;
  __syncthreads();
  if (T <= 0) return;

  if (warp == kNW) {
    // ------------------------------------------------------------ producer
    Pos q = locate(p, sb);
    LinRegs L;
    L.load(p.lin[q.l]);
    // This lane's row of the stage's scales and zeros into the slot: the
    // halves [e0, e0 + gs) of each array, copied as the aligned 4-byte words
    // that hold them (word w at slot word w, zeros 5 words later).  A window
    // whose last word would pass the end of the arrays is read with plain
    // loads instead.  Every lane arrives on the stage's full barrier once.
    auto copy_sz = [&](const Pos& at, uint32_t full, uint32_t sz_slot) {
      const int64_t n = at.r * 32 + lane;
      if (n >= L.N) {
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(full) : "memory");
        return;
      }
      const int KU = L.K / 32;
      const uint32_t u0 = uint32_t(at.t) * 32, ul = uint32_t(min(at.t * 32 + 32, KU) - 1);
      const int64_t gfirst = L.upg.div(u0);
      const int gs = int(L.upg.div(ul) - gfirst) + 1;
      const int64_t e0 = n * L.G + gfirst, a0 = e0 & ~int64_t(1);
      const int nw = int((e0 + gs - a0 + 1) >> 1);
      const uint32_t sw = sz_slot + uint32_t(lane * kSzRow * 4);
      if (a0 + 2 * nw <= int64_t(L.N) * L.G) {
        const uint32_t* sg = reinterpret_cast<const uint32_t*>(L.scales + a0);
        const uint32_t* zg = L.zeros ? reinterpret_cast<const uint32_t*>(L.zeros + a0) : nullptr;
        for (int w = 0; w < nw; ++w) {
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sw + 4 * w), "l"(sg + w) : "memory");
          if (zg)
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(sw + 4 * (kSzW + w)), "l"(zg + w)
                         : "memory");
        }
        asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(full) : "memory");
      } else {
        const unsigned short* sh = reinterpret_cast<const unsigned short*>(L.scales);
        const unsigned short* zh = reinterpret_cast<const unsigned short*>(L.zeros);
        const int64_t end = int64_t(L.N) * L.G;
        for (int w = 0; w < nw; ++w) {
          const int64_t a = a0 + 2 * w;
          const uint32_t lo = a < end ? sh[a] : 0u, hi = a + 1 < end ? sh[a + 1] : 0u;
          asm volatile("st.shared.u32 [%0], %1;" ::"r"(sw + 4 * w), "r"(lo | (hi << 16)) : "memory");
          if (zh) {
            const uint32_t zl = a < end ? zh[a] : 0u, zu = a + 1 < end ? zh[a + 1] : 0u;
            asm volatile("st.shared.u32 [%0], %1;" ::"r"(sw + 4 * (kSzW + w)), "r"(zl | (zu << 16)) : "memory");
          }
        }
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(full) : "memory");
      }
    };
    bool ok = true;
    int ic = 0;
    for (int i = 0; i < T; ++i) {
      const int s = i % D;
      if (i >= D) {
        bool w = true;
        if (lane == 0) w = wait_bounded(empty0 + 8 * s, uint32_t(((i / D) - 1) & 1));
        ok = __shfl_sync(0xffffffffu, w ? 1 : 0, 0) != 0;
        if (!ok) break;
      }
      __syncwarp();
      if (lane == 0) {
        const int rem = L.K - q.t * 1024;
        const int nq = rem >= 1024 ? 8 : rem / 128;
        const uint32_t xb = uint32_t(nq * MT * 256), sxb = uint32_t(nq * SXW * 4);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full0 + 8 * s),
                     "r"(uint32_t(C::SB) + xb + sxb)
                     : "memory");
#pragma unroll
        for (int b = 0; b < BITS; ++b)
          asm volatile(
              "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
              " [%0], [%1, {%3, %4}], [%2];" ::"r"(ring + s * C::SB + b * 4096),
              "l"(&p.tm[q.l]), "r"(full0 + 8 * s), "r"(q.t * 32 * BITS + 32 * b), "r"(int(q.r * 32))
              : "memory");
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                xps + s * C::XB),
            "l"(L.xp + int64_t(q.t) * MT * 512), "r"(xb), "r"(full0 + 8 * s)
            : "memory");
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                sxs + s * C::SXB),
            "l"(L.sx + int64_t(q.t) * 8 * SXW), "r"(sxb), "r"(full0 + 8 * s)
            : "memory");
      }
      const uint32_t sz_slot_s = ring + C::OFF_SZ + s * C::SZB;
      copy_sz(q, full0 + 8 * s, sz_slot_s);
      ++ic;
      if (++q.t == L.TS) {
        q.t = 0;
        if (++q.r == L.tiles) {
          q.r = 0;
          if (++q.l < p.nlin && i + 1 < T) L.load(p.lin[q.l]);
        }
      }
    }
    if (!ok && lane == 0) {
      // Copies issued but not consumed must land before the CTA exits: only
      // the last D issued stages can still be in flight, each in phase t / D.
      for (int t = ic > D ? ic - D : 0; t < ic; ++t)
        bw::drain_wait(full0 + 8 * (t % D), uint32_t((t / D) & 1), &g_gemv_grouped_timeout);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int g = lane >> 2, tq = lane & 3;
  const int tid = int(threadIdx.x);
  // this lane's rows of the 32-row tile: the MMA rows g, g + 8 of tile 0 and
  // of tile 1 (rows 16..31) map to weight rows rw[0..3]
  int rw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) rw[i] = mma_row<BITS>(g) + 8 * i;
  // With one or two tokens only the lanes t = 0 hold real accumulator
  // columns; the fold then moves each row's dot product to a lane of its own
  // (lane l: MMA row l % 8 of quarter l / 8, i.e. weight row lrow).
  constexpr bool LR = MT <= 2;
  const int lrow = mma_row<BITS>(lane & 7) + 8 * (lane >> 3);
  uint32_t uoff[4][unit_pieces<BITS>()];
#pragma unroll
  for (int i = 0; i < 4; ++i) unit_offsets<BITS>(rw[i], 4 * warp + tq, uoff[i]);
  // B fragment chunk offsets in the quad's x' area: token g (and g + 8);
  // token columns past the batch tile read the zero block.
  uint32_t boffA[4], boffB[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    boffA[i] = g < MT ? uint32_t(warp * MT * 256 + xp_chunk_pos((g * 4 + tq) * 4 + i) * 16) : 0xffffffffu;
    boffB[i] = g + 8 < MT ? uint32_t(warp * MT * 256 + xp_chunk_pos(((g + 8) * 4 + tq) * 4 + i) * 16)
                          : 0xffffffffu;
  }
  const uint32_t zero_blk = ring + C::OFF_ZERO;
  // accumulator column c of this lane: token 2 tq + (c & 1) + 8 (c >> 1)
  auto tok_of = [&](int c) { return 2 * tq + (c & 1) + 8 * (c >> 1); };

  Pos q = locate(p, sb);
  LinRegs L;
  L.load(p.lin[q.l]);
  float acc[4][NC];
  QuadAcc qa, qa2;
  float sxg[NC];
  auto zero_quad = [&]() {
#pragma unroll
    for (int t = 0; t < 2; ++t)
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) qa.c[t][j][e] = qa2.c[t][j][e] = 0.0f;
#pragma unroll
    for (int c = 0; c < NC; ++c) sxg[c] = 0.0f;
  };
  zero_quad();
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < NC; ++c) acc[r][c] = 0.0f;
  bool ok = true;
  int tcount = 0;
  int64_t seg_start = sb;      // first stage of this CTA in the current tile
  const __half hz = __float2half_rn(float(1 << (BITS - 1)));

  for (int i = 0; i < T; ++i) {
    const int s = i % D;
    {
      const uint32_t par = uint32_t((i / D) & 1);
      if (ok) ok = __all_sync(0xffffffffu, mbar_try(full0 + 8 * s, par) || wait_bounded(full0 + 8 * s, par));
    }
    const int kq = q.t * 1024 + 128 * warp;              // first code of this warp's quad
    const bool seg_end = (i + 1 == T) || (q.t + 1 == L.TS);
    if (kq < L.K) {
      uint32_t xa[16], xb2[16];
      const uint32_t xbase = xps + s * C::XB;
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        const uint32_t a = boffA[i4] != 0xffffffffu ? xbase + boffA[i4] : zero_blk + 16 * i4;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(xa[4 * i4]), "=r"(xa[4 * i4 + 1]), "=r"(xa[4 * i4 + 2]), "=r"(xa[4 * i4 + 3])
                     : "r"(a));
        if constexpr (MT == 16) {
          const uint32_t b2 = xbase + boffB[i4];
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(xb2[4 * i4]), "=r"(xb2[4 * i4 + 1]), "=r"(xb2[4 * i4 + 2]), "=r"(xb2[4 * i4 + 3])
                       : "r"(b2));
        } else {
          xb2[4 * i4] = xb2[4 * i4 + 1] = xb2[4 * i4 + 2] = xb2[4 * i4 + 3] = 0u;
        }
      }
      // sum x of the quad for this lane's tokens
      const float* sxq = reinterpret_cast<const float*>(smem + C::OFF_SX + s * C::SXB) + warp * SXW;
      if constexpr (LR) {
#pragma unroll
        for (int c = 0; c < MT; ++c) sxg[c] += sxq[c];
      } else {
#pragma unroll
        for (int c = 0; c < NC; ++c)
          if (tok_of(c) < MT) sxg[c] += sxq[tok_of(c)];
      }
      const uint32_t stage = ring + uint32_t(s * C::SB);
      // Fold the quad's dot products D into y: acc += s (D 2^69 - z sum x),
      // (s, z) of row rw[r] at half h(r) of the row's window in the slot.
      auto fold = [&](int gfirst, int rel) {
        const __half* szs = reinterpret_cast<const __half*>(smem + C::OFF_SZ + s * C::SZB);
        // e0 = n G + gfirst has the parity of gfirst, plus that of n when G is odd
        const int gpar = L.G & 1;
        if constexpr (LR) {
          // lane l takes row lrow: quarter r = l / 8 of lane 4 (l % 8)'s rows
          const int h = ((gpar * (int(q.r) * 32 + lrow) + gfirst) & 1) + rel;
          const __half* rs = szs + lrow * (2 * kSzRow);
          const float sc = __half2float(rs[h]);
          const float zr = __half2float(L.zeros ? rs[2 * kSzW + h] : hz);
          const int src = 4 * (lane & 7), rq = lane >> 3;
#pragma unroll
          for (int c = 0; c < MT; ++c) {
            float mine = 0.0f;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const int t = r >> 1, ce = 2 * (r & 1) + c;
              const float d = __shfl_sync(0xffffffffu, qa.c[t][0][ce] + qa.c[t][1][ce], src);
              mine = rq == r ? d : mine;
            }
            acc[0][c] = fmaf(sc, fmaf(mine, 0x1p69f, -zr * sxg[c]), acc[0][c]);
          }
          return;
        }
        float2 zs[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int h = ((gpar * (int(q.r) * 32 + rw[r]) + gfirst) & 1) + rel;
          const __half* rs = szs + rw[r] * (2 * kSzRow);
          zs[r].x = __half2float(rs[h]);
          zs[r].y = __half2float(L.zeros ? rs[2 * kSzW + h] : hz);
        }
        // rows rw[0], rw[1] from tile 0 (MMA rows g, g + 8), rw[2], rw[3] from tile 1
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int t = r >> 1, e = 2 * (r & 1);
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            const QuadAcc& src = (c >> 1) ? qa2 : qa;
            const int ce = e + (c & 1);
            const float d = src.c[t][0][ce] + src.c[t][1][ce];
            acc[r][c] = fmaf(zs[r].x, fmaf(d, 0x1p69f, -zs[r].y * sxg[c]), acc[r][c]);
          }
        }
      };
      if (L.tiles_stage) {
        // every quad is a group of its own (or part of one inside this
        // stage): MMAs start from zero, the fold follows at once
        {
          uint32_t wa[BITS], wb[BITS];
          load_unit_at<BITS>(stage, uoff[0], wa);
          load_unit_at<BITS>(stage, uoff[1], wb);
          QuadMma<BITS, 0, 0, MT == 16, true>::run(qa, qa2, wa, wb, xa, xb2);
        }
        {
          uint32_t wa[BITS], wb[BITS];
          load_unit_at<BITS>(stage, uoff[2], wa);
          load_unit_at<BITS>(stage, uoff[3], wb);
          QuadMma<BITS, 1, 0, MT == 16, true>::run(qa, qa2, wa, wb, xa, xb2);
        }
        fold((q.t * 8) >> L.qshift, warp >> L.qshift);
#pragma unroll
        for (int c = 0; c < NC; ++c) sxg[c] = 0.0f;
      } else {
        {
          uint32_t wa[BITS], wb[BITS];
          load_unit_at<BITS>(stage, uoff[0], wa);
          load_unit_at<BITS>(stage, uoff[1], wb);
          QuadMma<BITS, 0, 0, MT == 16, false>::run(qa, qa2, wa, wb, xa, xb2);
        }
        {
          uint32_t wa[BITS], wb[BITS];
          load_unit_at<BITS>(stage, uoff[2], wa);
          load_unit_at<BITS>(stage, uoff[3], wb);
          QuadMma<BITS, 1, 0, MT == 16, false>::run(qa, qa2, wa, wb, xa, xb2);
        }
        // fold when the next quad of this warp is in another group, or absent
        const uint32_t uq = uint32_t(kq / 32);
        const int gq = int(L.upg.div(uq));
        const bool next_in = !seg_end && kq + 1024 < L.K;
        if (!next_in || int(L.upg.div(uq + 32)) != gq) {
          const int gfirst = int(L.upg.div(uint32_t(q.t) * 32));
          fold(gfirst, gq - gfirst);
          zero_quad();
        }
      }
    }
    __syncwarp();
    if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty0 + 8 * s) : "memory");

    if (seg_end) {
      // ---------------------------------------------------- tile epilogue
      const int64_t tb = L.stage0 + q.r * L.TS, te = tb + L.TS;
      const bool whole = seg_start <= tb && te <= se;
      const int64_t row0 = q.r * 32;
      // parked partials: slot 0 for a CTA's first tile, slot 1 for its last
      const int myslot = sb >= tb ? 0 : 1;
      // contributors of a cut tile: the CTAs whose ranges hold its first and last stage
      const int64_t ca = ((tb + 1) * p.P - 1) / p.total, cbk = (te * p.P - 1) / p.total;
      if constexpr (LR) {
        // Each warp parks its 32 row sums; the last warp to arrive on the
        // buffer's counter adds the eight in warp order and writes y (or the
        // CTA's partial of a cut tile).  No barrier: the others go on.
        const int slot = tcount % C::RB;
        float* rb = red + slot * (kNW * MT * 32);
        unsigned* tcnt = reinterpret_cast<unsigned*>(smem + C::OFF_TCNT) + slot;
#pragma unroll
        for (int c = 0; c < MT; ++c) rb[(warp * MT + c) * 32 + lrow] = acc[0][c];
        __syncwarp();
        unsigned arrived = 0;
        if (lane == 0) {
          __threadfence_block();
          arrived = atomicAdd(tcnt, 1u);
        }
        if (__shfl_sync(0xffffffffu, arrived, 0) == unsigned(kNW - 1)) {
          __threadfence_block();
#pragma unroll
          for (int m = 0; m < MT; ++m) {
            float v = 0.0f;
#pragma unroll
            for (int wv = 0; wv < kNW; ++wv) v += rb[(wv * MT + m) * 32 + lane];
            if (whole) {
              if (m < p.M && row0 + lane < L.N) L.y[int64_t(m) * L.N + row0 + lane] = __float2bfloat16_rn(v);
            } else {
              p.part[((cta * 2 + myslot) * MT + m) * 32 + lane] = v;
            }
          }
          if (!whole) {
            __threadfence();
            __syncwarp();
            unsigned old = 0;
            if (lane == 0) old = atomicAdd(p.cnt + ca, 1u);
            if (__shfl_sync(0xffffffffu, old, 0) == unsigned(cbk - ca)) {
              __threadfence();
              const int slot_a = range_start(p, ca) < tb ? 1 : 0;
#pragma unroll
              for (int m = 0; m < MT; ++m) {
                float v = 0.0f;
                for (int64_t cc = ca; cc <= cbk; ++cc)
                  v += __ldcg(p.part + ((cc * 2 + (cc == ca ? slot_a : 0)) * MT + m) * 32 + lane);
                if (m < p.M && row0 + lane < L.N) L.y[int64_t(m) * L.N + row0 + lane] = __float2bfloat16_rn(v);
              }
              __syncwarp();
              if (lane == 0) atomicExch(p.cnt + ca, 0u);
            }
          }
          __syncwarp();
          if (lane == 0) atomicExch(tcnt, 0u);     // the buffer is free again
        }
      } else {
      float* rb = red + (C::RB == 2 ? (tcount & 1) : 0) * (kNW * MT * 32);
#pragma unroll
      for (int c = 0; c < NC; ++c)
        if (tok_of(c) < MT) {
#pragma unroll
          for (int r = 0; r < 4; ++r) rb[(warp * MT + tok_of(c)) * 32 + rw[r]] = acc[r][c];
        }
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kNW) : "memory");
      // the summing threads rotate over the warps from tile to tile
      const int rt = (tid + 32 * (tcount & 7)) & (32 * kNW - 1);
      for (int idx = rt; idx < 32 * MT; idx += 32 * kNW) {
        const int m = idx >> 5, row = idx & 31;
        float v = 0.0f;
#pragma unroll
        for (int wv = 0; wv < kNW; ++wv) v += rb[(wv * MT + m) * 32 + row];
        if (whole) {
          if (m < p.M && row0 + row < L.N) L.y[int64_t(m) * L.N + row0 + row] = __float2bfloat16_rn(v);
        } else {
          p.part[((cta * 2 + myslot) * MT + m) * 32 + row] = v;
        }
      }
      if (!whole) {
        __threadfence();
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kNW) : "memory");
        if (tid == 0) {
          const unsigned old = atomicAdd(p.cnt + ca, 1u);
          *flag = old == unsigned(cbk - ca) ? 1 : 0;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(32 * kNW) : "memory");
        if (*flag) {
          __threadfence();
          const int slot_a = range_start(p, ca) < tb ? 1 : 0;
          for (int idx = tid; idx < 32 * MT; idx += 32 * kNW) {
            const int m = idx >> 5, row = idx & 31;
            float v = 0.0f;
            for (int64_t cc = ca; cc <= cbk; ++cc)
              v += __ldcg(p.part + ((cc * 2 + (cc == ca ? slot_a : 0)) * MT + m) * 32 + row);
            if (m < p.M && row0 + row < L.N) L.y[int64_t(m) * L.N + row0 + row] = __float2bfloat16_rn(v);
          }
          if (tid == 0) atomicExch(p.cnt + ca, 0u);
        }
      }
      if constexpr (C::RB == 1) asm volatile("bar.sync 1, %0;" ::"n"(32 * kNW) : "memory");
      }
      ++tcount;
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[r][c] = 0.0f;
      seg_start = sb + i + 1;
    }
    // next stage; a new linear's fields are read once, and its first
    // accumulating MMA must not add to what a fresh-start linear left behind
    if (++q.t == L.TS) {
      q.t = 0;
      if (++q.r == L.tiles) {
        q.r = 0;
        if (++q.l < p.nlin && i + 1 < T) {
          L.load(p.lin[q.l]);
          zero_quad();
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
struct DevInfo {
  std::atomic<int> sms{0};
};
DevInfo g_dev[64];

int device_sms(int dev) {
  if (dev < 0 || dev >= 64) return 0;
  int v = g_dev[dev].sms.load(std::memory_order_relaxed);
  if (v == 0) {
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    g_dev[dev].sms.store(v, std::memory_order_relaxed);
  }
  return v;
}

// Ring depth and resident CTAs per SM: as many stages as the shared memory
// of two CTAs per SM holds (one CTA for 16 tokens), because the achieved
// bandwidth follows the bytes each SM keeps in flight.
template <int BITS, int MT>
struct Shape {
  // per stage: codes, x', sums, (s, z), barriers (and a reduction buffer with <= 2 tokens)
  static constexpr int kPer = BITS * 4096 + MT * 2048 + 8 * Tok<MT>::SXW * 4 + 32 * kSzRow * 4 + 16 +
                              (MT <= 2 ? kNW * MT * 32 * 4 + 4 : 0);
  static constexpr int kRed = (MT <= 2 ? 1 : (MT <= 8 ? 2 : 1)) * kNW * MT * 32 * 4;
  static constexpr int kFixed = kRed + 64 + 16 + 64 + 1024;
  // two CTAs per SM when two stages each still fit in half the shared memory
  static constexpr int MINB = (MT <= 8 && 2 * kPer + kFixed <= 113 * 1024) ? 2 : 1;
  static constexpr int kFit = ((MINB == 2 ? 113 : 226) * 1024 - kFixed) / kPer;
  static constexpr int D = kFit < 2 ? 2 : (kFit > 12 ? 12 : kFit);
};

template <int BITS, int MT>
cudaError_t launch_mt(const GroupedLinear* lins, int count, int M, const WsLayout& ws, cudaStream_t st) {
  constexpr int D = Shape<BITS, MT>::D, MINB = Shape<BITS, MT>::MINB;
  static_assert(GCfg<BITS, MT, D>::BYTES <= (MINB == 2 ? 113 : 226) * 1024, "shared memory");
  using C = GCfg<BITS, MT, D>;
  auto kern = gemv_grouped_kernel<BITS, MT, D, MINB>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  static std::atomic<int> occ[64];
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  const int nsm = device_sms(dev);
  if (nsm <= 0) return cudaErrorInvalidDevice;
  int nb = occ[dev].load(std::memory_order_relaxed);
  if (nb == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kThreads, C::BYTES);
    if (e != cudaSuccess) return e;
    if (nb < 1) return cudaErrorInvalidConfiguration;
    occ[dev].store(nb, std::memory_order_relaxed);
  }

  // x' and sums of every linear
  for (int c0 = 0; c0 < count; c0 += kMaxPrepLinears) {
    const int n = count - c0 < kMaxPrepLinears ? count - c0 : kMaxPrepLinears;
    PrepParams pp{};
    pp.nlin = n;
    pp.M = M;
    int maxw = 1;
    for (int j = 0; j < n; ++j) {
      const GroupedLinear& g = lins[c0 + j];
      pp.lin[j] = PrepLin{g.x, int(g.K), ws.xp[c0 + j], ws.sx[c0 + j]};
      const int w = int(g.K / 128) * MT;
      maxw = w > maxw ? w : maxw;
    }
    xprep_kernel<BITS, MT><<<dim3(unsigned((maxw + 7) / 8), unsigned(n)), 256, 0, st>>>(pp);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }

  // the stage sequence, in launches of at most kMaxLinears linears
  for (int c0 = 0; c0 < count; c0 += kMaxLinears) {
    const int n = count - c0 < kMaxLinears ? count - c0 : kMaxLinears;
    GParams* gp = new (std::nothrow) GParams();
    if (!gp) return cudaErrorMemoryAllocation;
    int64_t total = 0;
    for (int j = 0; j < n; ++j) {
      const GroupedLinear& g = lins[c0 + j];
      if (!make_tensor_map_2d(&gp->tm[j], TmaType::kU32, g.codes, uint64_t(g.K * BITS / 32), uint64_t(g.N),
                              uint64_t(g.K * BITS / 8), 32, 32, 128)) {
        delete gp;
        return cudaErrorInvalidValue;
      }
      GLin& L = gp->lin[j];
      L.scales = g.scales;
      L.zeros = g.zeros;
      L.y = g.y;
      L.xp = ws.xp[c0 + j];
      L.sx = ws.sx[c0 + j];
      L.stage0 = total;
      L.N = int(g.N);
      L.K = int(g.K);
      L.G = int(g.K / g.group);
      L.TS = int((g.K + 1023) / 1024);
      L.tiles = int((g.N + 31) / 32);
      L.upg = FastDiv(uint32_t(g.group / 32));
      total += int64_t(L.TS) * L.tiles;
    }
    int64_t P = int64_t(nsm) * nb;
    P = P < total ? P : total;
    P = P < kMaxCtas ? P : kMaxCtas;
    gp->nlin = n;
    gp->M = M;
    gp->total = total;
    gp->P = int(P);
    gp->part = ws.part;
    gp->cnt = ws.cnt;
    kern<<<unsigned(P), kThreads, C::BYTES, st>>>(*gp);
    delete gp;
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int BITS>
cudaError_t launch_bits(const GroupedLinear* lins, int count, int M, const WsLayout& ws, cudaStream_t st) {
  switch (grouped_token_tile(M)) {
    case 1: return launch_mt<BITS, 1>(lins, count, M, ws, st);
    case 2: return launch_mt<BITS, 2>(lins, count, M, ws, st);
    case 4: return launch_mt<BITS, 4>(lins, count, M, ws, st);
    case 8: return launch_mt<BITS, 8>(lins, count, M, ws, st);
    default: return launch_mt<BITS, 16>(lins, count, M, ws, st);
  }
}

}  // namespace

int grouped_token_tile(int M) { return M <= 1 ? 1 : M <= 2 ? 2 : M <= 4 ? 4 : M <= 8 ? 8 : 16; }

bool grouped_supported(int64_t K, int64_t g) { return K % 128 == 0 && g % 128 == 0; }

size_t grouped_workspace_layout(const GroupedLinear* lins, int count, int M, uintptr_t base, WsLayout* out) {
  const int MT = grouped_token_tile(M);
  const size_t sxw = MT < 4 ? 4 : size_t(MT);
  auto up = [](size_t v) { return (v + 255) & ~size_t(255); };
  size_t off = 0;
  if (out) {
    out->xp.assign(size_t(count), nullptr);
    out->sx.assign(size_t(count), nullptr);
    out->cnt = reinterpret_cast<unsigned*>(base + off);
  }
  off = up(off + sizeof(unsigned) * kMaxCtas);
  if (out) out->part = reinterpret_cast<float*>(base + off);
  off = up(off + sizeof(float) * size_t(kMaxCtas) * 2 * MT * 32);
  for (int j = 0; j < count; ++j) {
    const size_t TS = size_t((lins[j].K + 1023) / 1024);
    if (out) out->xp[j] = reinterpret_cast<uint32_t*>(base + off);
    off = up(off + TS * size_t(MT) * 2048);
    if (out) out->sx[j] = reinterpret_cast<float*>(base + off);
    off = up(off + TS * 8 * sxw * sizeof(float));
  }
  return off;
}

cudaError_t launch_gemv_grouped(const GroupedLinear* lins, int count, int M, int bits, const WsLayout& ws,
                                cudaStream_t st) {
  switch (bits) {
    case 2: return launch_bits<2>(lins, count, M, ws, st);
    case 3: return launch_bits<3>(lins, count, M, ws, st);
    case 4: return launch_bits<4>(lins, count, M, ws, st);
    default: return launch_bits<8>(lins, count, M, ws, st);
  }
}

#ifdef WQ_TEST_HOOKS
// Test builds only: one thread waits, with the library's bounded pipeline
// wait, on a fresh mbarrier that nothing ever arrives on.  The wait runs out
// after the build's pipeline limit and raises this file's device flag, which
// wq_last_device_error reports; nothing faults and nothing is left running.
__global__ void wait_probe_kernel() {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = stg::saddr(&bar);
  if (threadIdx.x == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) wait_bounded(b, 0u);
  __syncthreads();
}
#endif

bool gemv_grouped_read_and_clear_timeout(cudaError_t* err) {
  unsigned int v = 0;
  const unsigned int zero = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&v, g_gemv_grouped_timeout, sizeof(v));
  if (e == cudaSuccess && v) e = cudaMemcpyToSymbol(g_gemv_grouped_timeout, &zero, sizeof(zero));
  *err = e;
  return v != 0;
}

}  // namespace wq

#ifdef WQ_TEST_HOOKS
// Test builds only: launch the wait probe on `stream`; 0 on success.
extern "C" int wq_test_expire_wait(void* stream) {
  wq::wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return cudaGetLastError() == cudaSuccess ? 0 : 7;
}
#endif
