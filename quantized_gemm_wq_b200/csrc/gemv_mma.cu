// gemv_mma.cu -- decode GEMV for 2..8 tokens with the multiply-adds on the
// tensor cores: y = x . W'^T, codes unpacked in registers straight into the A
// operand of warp-level MMAs (mma.sync m16n8k16, bf16 in, fp32 out); the
// tokens are the MMA's 8 columns, so up to 8 of them cost one MMA.
//
// Why the tensor cores here.  Decoding is bound by the bytes of packed codes
// read from memory ("Platform For AI: BladeLLM model quantization",
// "Quantization modes > weight_only_quant"); a CUDA-core dot product spends
// one FMA per code and token on top of the unpack, so its cost grows with the
// batch.  Here one AND yields two codes (one per 16-bit half, as bf16 bit
// patterns) for all tokens at once and the MMA does the multiply-adds.
//
// Unpacking.  A code q in bits [b, b + c) of a 16-bit half, every other bit of
// the half clear, is the bf16 pattern of q 2^(b-133) for b + c <= 8 (the
// subnormals and the first normal binade, where the encoding is linear).  A
// 32-code unit of one row (c 32-bit words) is covered by 16 ANDs of shifted
// windows of its bit stream (kUnit tables: window start, mask, and the code
// and bit offset of each half).  The activation multiplied with a code at
// offset b is stored as x 2^(64-b) (exact: a power of two), so every product
// is q x 2^-69 exactly and the fp32 sums are brought back by 2^69.
//
// Work split.  A CTA owns 32 output rows (two 16-row MMA tiles) over its
// share of K; a stage is 1024 codes of K (8 quads of 4 units).  Warp NW is the
// producer: one lane issues the TMA copy of the stage's codes (32 rows x 32
// units, 128-byte swizzle) and one bulk copy per token of its 1024 x values
// into a ring of D stages.  Consumer warp w takes quad w of every stage for
// all 32 rows: lane (g, t) = (l / 4, l % 4) supplies unit 4w + t of rows g,
// g + 8, g + 16, g + 24, so MMA j of a tile reduces over pairs 2j and 2j + 1
// of the quad's four units (one scale group: groups are whole quads).  The
// warp first writes the quad's x' operand of each token (64 words, two per
// lane) into its own shared buffer; lane (g, t) reads the B fragment of token
// g from there (token columns past MT read zeros).  Per scale group the
// accumulators (tokens 2t and 2t + 1 of the lane's rows) are folded into y as
// s (dot 2^69 - z sum x).  Partial sums meet across warps in shared memory and
// across a split-K cluster through distributed shared memory.
#include <cuda.h>   // CUtensorMap

#include <atomic>

#include "stage_smem.cuh"
#include "unpack_tables.h"
#include "wq_internal.cuh"

namespace wq {
namespace {

using namespace stg;

#ifndef WQ_GEMV_MMA_TARGET_CTAS
#define WQ_GEMV_MMA_TARGET_CTAS 444
#endif
#ifndef WQ_GEMV_MMA_MIN_STAGES
#define WQ_GEMV_MMA_MIN_STAGES 4
#endif
__device__ unsigned int g_gemv_mma_timeout;

__device__ __forceinline__ bool mma_wait_bounded(uint32_t bar, uint32_t parity) {
  return bw::pipe_wait(bar, parity, &g_gemv_mma_timeout, nullptr);
}

template <int BITS, int MT>
struct MmaCfg {
  static constexpr int NW = 8;                       // consumer warps, one quad of a stage each
  static constexpr int D = 3;                        // ring stages
  static constexpr int STAGE_WORDS = 32 * BITS;      // words of one row per stage
  static constexpr int BOX_BYTES = 32 * 128;
  static constexpr int STAGE_BYTES = BITS * BOX_BYTES;
  static constexpr int XRAW_BYTES = MT * 1024 * 2;   // the stage's x values of MT tokens, bf16
  static constexpr int XB = 20;                      // words per unit of x' (16 pairs + bank pad)
  static constexpr int XP_BYTES = NW * MT * 4 * XB * 4;   // per warp and token: x' of its quad
  static constexpr int ZERO_BYTES = 4 * XB * 4;      // B operand of the empty token columns
  static constexpr int FIXED = D * (STAGE_BYTES + XRAW_BYTES) + XP_BYTES + ZERO_BYTES + 2 * D * 8;
  static int smem(int gcap) { return FIXED + 32 * gcap * 8 + 1024; }
};

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

// Code offsets (in the unit) and x factors 2^(64 - b) of pair t, for a pair
// index known only at run time (once per lane).
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

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The 8 MMAs of one 16-row tile over a quad: rows g (words wa) and g + 8
// (words wb) of this lane's unit, B from xb.
template <int BITS, int J>
struct TileMma {
  __device__ __forceinline__ static void run(float (&c)[4], const uint32_t (&wa)[BITS],
                                             const uint32_t (&wb)[BITS], const uint32_t (&xb)[16]) {
    mma_bf16(c, unit_pair<BITS, 2 * J>(wa), unit_pair<BITS, 2 * J>(wb), unit_pair<BITS, 2 * J + 1>(wa),
             unit_pair<BITS, 2 * J + 1>(wb), xb[2 * J], xb[2 * J + 1]);
    if constexpr (J + 1 < 8) TileMma<BITS, J + 1>::run(c, wa, wb, xb);
  }
};

// Sums of MT per-token values over the warp, one token per lane: at each step
// lanes keep half of their tokens and add the partner's copy of that half, so
// after log2(MT) steps lane l holds a partial of token (l >> (5 - log2 MT)),
// completed by the remaining xor steps.  MT - 1 + 5 - log2(MT) shuffles
// instead of 5 MT.
template <int MT>
__device__ __forceinline__ float token_sums(float (&p)[MT], int lane) {
  constexpr int LG = MT == 2 ? 1 : (MT == 4 ? 2 : 3);
  static_assert(MT == (1 << LG), "MT must be 2, 4 or 8");
#pragma unroll
  for (int step = 0; step < LG; ++step) {
    const int d = 16 >> step, half = MT >> (step + 1);
    const bool hi = lane & d;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = hi ? p[half + i] : p[i], send = hi ? p[i] : p[half + i];
      p[i] = keep + __shfl_xor_sync(0xffffffffu, send, d);
    }
  }
  float r = p[0];
#pragma unroll
  for (int d = 16 >> LG; d >= 1; d >>= 1) r += __shfl_xor_sync(0xffffffffu, r, d);
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <int BITS, int MT, int MINB>
__global__ void __launch_bounds__(32 * (MmaCfg<BITS, MT>::NW + 1), MINB)
gemv_mma_kernel(const __grid_constant__ CUtensorMap tm_codes, const __nv_bfloat16* __restrict__ x,
                int M, int64_t N, int64_t K, const __half* __restrict__ scales,
                const __half* __restrict__ zeros, FastDiv units_per_group, int gcap,
                __nv_bfloat16* __restrict__ y) {
  using Cfg = MmaCfg<BITS, MT>;
  constexpr int NW = Cfg::NW, D = Cfg::D, XB = Cfg::XB;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ float red[NW][MT][32];
  uint8_t* smem = smem_raw + ((1024 - (saddr(smem_raw) & 1023)) & 1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ring = saddr(smem);
  const uint32_t xraw0 = ring + D * Cfg::STAGE_BYTES;
  uint8_t* xp_base = smem + D * (Cfg::STAGE_BYTES + Cfg::XRAW_BYTES);
  uint32_t* zero_blk = reinterpret_cast<uint32_t*>(xp_base + Cfg::XP_BYTES);
  const uint32_t full0 = saddr(xp_base + Cfg::XP_BYTES + Cfg::ZERO_BYTES);
  const uint32_t empty0 = full0 + 8 * D;
  float2* tbl = reinterpret_cast<float2*>(xp_base + Cfg::XP_BYTES + Cfg::ZERO_BYTES + 16 * D);

  const int64_t row0 = int64_t(blockIdx.x) * 32;
  const int64_t KU = K / 32;
  const int TT = int((KU + 31) / 32);
  const int ks = int(gridDim.y), kr = int(blockIdx.y);
  const int tb = int(int64_t(TT) * kr / ks), te = int(int64_t(TT) * (kr + 1) / ks);
  const int T = te - tb;
  const int64_t G = K / (int64_t(units_per_group.d) * 32);

  if (threadIdx.x == 0) {
    for (int s = 0; s < D; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full0 + 8 * s));
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(empty0 + 8 * s), "r"(NW));
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = threadIdx.x; i < 4 * XB; i += blockDim.x) zero_blk[i] = 0u;
  __syncthreads();

  if (warp == NW) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      bool ok = true;
      int ic = 0;                                   // stages issued
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % D;
        if (t >= D) ok = mma_wait_bounded(empty0 + 8 * s, uint32_t(((t / D) - 1) & 1));
        // the first stage goes out alone (see gemv_tma.cu)
        if (t == 1) ok = ok && mma_wait_bounded(full0, 0u);
        if (!ok) break;
        const int64_t k0 = int64_t(tb + t) * 1024;
        const uint32_t xbytes = uint32_t((K - k0 < 1024 ? K - k0 : 1024) * 2);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full0 + 8 * s),
                     "r"(uint32_t(Cfg::STAGE_BYTES) + uint32_t(M) * xbytes)
                     : "memory");
#pragma unroll
        for (int b = 0; b < BITS; ++b)
          asm volatile(
              "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
              " [%0], [%1, {%3, %4}], [%2];" ::"r"(ring + s * Cfg::STAGE_BYTES + b * Cfg::BOX_BYTES),
              "l"(&tm_codes), "r"(full0 + 8 * s), "r"((tb + t) * Cfg::STAGE_WORDS + 32 * b), "r"(int(row0))
              : "memory");
        for (int m = 0; m < M; ++m)
          asm volatile(
              "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                  xraw0 + s * Cfg::XRAW_BYTES + m * 2048),
              "l"(x + int64_t(m) * K + k0), "r"(xbytes), "r"(full0 + 8 * s)
              : "memory");
        ++ic;
      }
      if (!ok) {
        // Copies issued but not consumed must land before the CTA exits.  Only
        // the last D issued stages can still be in flight (a slot is re-armed
        // only by issuing the stage D later), each in phase t / D of its slot.
        for (int t = ic > D ? ic - D : 0; t < ic; ++t)
          bw::drain_wait(full0 + 8 * (t % D), uint32_t((t / D) & 1), &g_gemv_mma_timeout);
      }
    }
  } else {
    // ---------------------------------------------------------------- consumers
    const int g = lane >> 2, tq = lane & 3;
    // x' words this lane writes for every token: unit lane / 8 of the quad,
    // pairs 2 (lane % 8) and +1
    const int xu = lane >> 3, xpair = 2 * (lane & 7);
    int lo0 = 0, hi0 = 0, lo1 = 0, hi1 = 0;
    float flo0 = 0.0f, fhi0 = 0.0f, flo1 = 0.0f, fhi1 = 0.0f;
    PairPick<BITS, 0>::run(xpair, lo0, hi0, flo0, fhi0);
    PairPick<BITS, 0>::run(xpair + 1, lo1, hi1, flo1, fhi1);
    uint32_t* xpw = reinterpret_cast<uint32_t*>(xp_base) + warp * MT * 4 * XB;
    // B operand: token column g (columns past MT are empty)
    const uint4* xbsrc = reinterpret_cast<const uint4*>((g < MT ? xpw + g * 4 * XB : zero_blk) + tq * XB);

    const int trow = threadIdx.x >> 3, tj = threadIdx.x & 7;
    const bool trow_in = row0 + trow < N;
    const __half* srow = scales + (trow_in ? row0 + trow : 0) * G;
    const __half* zrow = zeros ? zeros + (trow_in ? row0 + trow : 0) * G : nullptr;
    auto load_table = [&](int64_t wg0) {
      float sv[16], zv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int j = tj + 8 * i;
        const bool in = trow_in && j < gcap && wg0 + j < G;
        sv[i] = in ? __half2float(srow[wg0 + j]) : 0.0f;
        zv[i] = in ? (zrow ? __half2float(zrow[wg0 + j]) : float(1 << (BITS - 1))) : 0.0f;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(32 * NW) : "memory");   // old table no longer read
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int j = tj + 8 * i;
        if (j < gcap) tbl[trow * gcap + j] = make_float2(sv[i], zv[i]);
      }
      asm volatile("bar.sync 1, %0;" ::"n"(32 * NW) : "memory");   // new table visible
    };
    const uint32_t ulast = uint32_t((int64_t(te) * 32 < KU ? int64_t(te) * 32 : KU) - 1);
    int64_t wg0 = units_per_group.div(uint32_t(tb) * 32);
    const bool one_window = int64_t(units_per_group.div(ulast)) < wg0 + gcap;
    load_table(wg0);

    uint32_t uoff[4][unit_pieces<BITS>()];
#pragma unroll
    for (int i = 0; i < 4; ++i) unit_offsets<BITS>(g + 8 * i, 4 * warp + tq, uoff[i]);
    // acc[r][c]: row g + 8 r, token 2 tq + c
    float acc[4][2] = {};
    float c0[4] = {0.0f, 0.0f, 0.0f, 0.0f}, c1[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    // sum x of the group so far, of token lane >> (5 - log2 MT) (see token_sums)
    constexpr int kTokShift = MT == 2 ? 4 : (MT == 4 ? 3 : 2);
    float sxg = 0.0f;
    int64_t cur = -1;                            // group of the accumulators
    auto flush = [&]() {
      int64_t gi = cur - wg0;
      gi = gi < gcap ? gi : gcap - 1;
      // sum x of tokens 2 tq and 2 tq + 1 (a token past MT reads some lane: unused)
      const float s0 = __shfl_sync(0xffffffffu, sxg, ((2 * tq) << kTokShift) & 31);
      const float s1 = __shfl_sync(0xffffffffu, sxg, ((2 * tq + 1) << kTokShift) & 31);
      const float2 sz[4] = {tbl[g * gcap + gi], tbl[(g + 8) * gcap + gi], tbl[(g + 16) * gcap + gi],
                            tbl[(g + 24) * gcap + gi]};
      const float cc[4][2] = {{c0[0], c0[1]}, {c0[2], c0[3]}, {c1[0], c1[1]}, {c1[2], c1[3]}};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        acc[r][0] = fmaf(sz[r].x, fmaf(cc[r][0], 0x1p69f, -sz[r].y * s0), acc[r][0]);
        acc[r][1] = fmaf(sz[r].x, fmaf(cc[r][1], 0x1p69f, -sz[r].y * s1), acc[r][1]);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) c0[i] = c1[i] = 0.0f;
      sxg = 0.0f;
    };
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int s = t % D;
      const int64_t u0 = int64_t(tb + t) * 32;         // first unit of the stage
      const int64_t q0 = u0 + 4 * warp;                 // first unit of this warp's quad
      const int64_t grp = int64_t(units_per_group.div(uint32_t(q0)));
      if (cur >= 0 && grp != cur) flush();              // before the table may move
      if (!one_window) {
        const int64_t ue = (u0 + 32 < KU ? u0 + 32 : KU) - 1;
        if (int64_t(units_per_group.div(uint32_t(ue))) >= wg0 + gcap) {
          wg0 = units_per_group.div(uint32_t(u0));
          load_table(wg0);
        }
      }
      cur = grp;
      {   // the common case (stage landed) without the call to the bounded wait
        const uint32_t par = uint32_t((t / D) & 1);
        if (ok) ok = __all_sync(0xffffffffu, mbar_try(full0 + 8 * s, par) || mma_wait_bounded(full0 + 8 * s, par));
      }
      // x' of the quad for every token: this lane's two words, and sum x over the quad
      const bool uin = q0 + xu < KU;
      float px[MT];
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const __nv_bfloat16* xr =
            reinterpret_cast<const __nv_bfloat16*>(smem + D * Cfg::STAGE_BYTES + s * Cfg::XRAW_BYTES) +
            m * 1024 + (4 * warp + xu) * 32;
        const bool in = uin && m < M;
        const float xl0 = in ? __bfloat162float(xr[lo0]) : 0.0f, xh0 = in ? __bfloat162float(xr[hi0]) : 0.0f;
        const float xl1 = in ? __bfloat162float(xr[lo1]) : 0.0f, xh1 = in ? __bfloat162float(xr[hi1]) : 0.0f;
        *reinterpret_cast<uint2*>(xpw + (m * 4 + xu) * XB + xpair) =
            make_uint2(pack_bf16x2(xl0 * flo0, xh0 * fhi0), pack_bf16x2(xl1 * flo1, xh1 * fhi1));
        px[m] = (xl0 + xh0) + (xl1 + xh1);
      }
      sxg += token_sums<MT>(px, lane);
      __syncwarp();                                     // x' visible to the warp
      uint32_t xb[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 v = xbsrc[i];
        xb[4 * i] = v.x; xb[4 * i + 1] = v.y; xb[4 * i + 2] = v.z; xb[4 * i + 3] = v.w;
      }
      const uint32_t stage = ring + uint32_t(s * Cfg::STAGE_BYTES);
      {
        uint32_t wa[BITS], wb[BITS];
        load_unit_at<BITS>(stage, uoff[0], wa);
        load_unit_at<BITS>(stage, uoff[1], wb);
        TileMma<BITS, 0>::run(c0, wa, wb, xb);
      }
      {
        uint32_t wa[BITS], wb[BITS];
        load_unit_at<BITS>(stage, uoff[2], wa);
        load_unit_at<BITS>(stage, uoff[3], wb);
        TileMma<BITS, 0>::run(c1, wa, wb, xb);
      }
      __syncwarp();                                     // done with stage s and the x' buffers
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty0 + 8 * s) : "memory");
    }
    if (cur >= 0) flush();
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const int m = 2 * tq + c;
      if (m < MT) {
#pragma unroll
        for (int r = 0; r < 4; ++r) red[warp][m][g + 8 * r] = acc[r][c];
      }
    }
  }
  __syncthreads();
  // thread i < 32 MT: token i / 32, row i % 32
  const int om = int(threadIdx.x) >> 5, orow = int(threadIdx.x) & 31;
  if (threadIdx.x < 32 * MT) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += red[w][om][orow];
    red[0][om][orow] = v;
  }
  if (ks > 1) {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (kr == 0 && threadIdx.x < 32 * MT) {
      float v = red[0][om][orow];
      const uint32_t mine = saddr(&red[0][om][orow]);
      for (int r = 1; r < ks; ++r) {
        uint32_t peer;
        float pv;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(peer) : "r"(mine), "r"(r));
        asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(pv) : "r"(peer) : "memory");
        v += pv;
      }
      red[0][om][orow] = v;
    }
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  } else {
    __syncthreads();
  }
  if (kr == 0 && threadIdx.x < 32 * MT && om < M) {
    const int64_t n = row0 + orow;
    if (n < N) y[int64_t(om) * N + n] = __float2bfloat16_rn(red[0][om][orow]);
  }
}

template <int BITS, int MT>
cudaError_t launch_mt(const __nv_bfloat16* x, int M, int64_t N, int64_t K, const uint32_t* codes,
                      const __half* scales, const __half* zeros, int64_t g, __nv_bfloat16* y,
                      cudaStream_t st) {
  using Cfg = MmaCfg<BITS, MT>;
  alignas(64) CUtensorMap tm;
  if (!make_tensor_map_2d(&tm, TmaType::kU32, codes, uint64_t(K * BITS / 32), uint64_t(N),
                          uint64_t(K * BITS / 8), 32, 32, 128))
    return cudaErrorInvalidValue;
  // per device, set once; concurrent first calls repeat idempotent queries
  static std::atomic<bool> attr_set[64];
  static std::atomic<int> sms[64];
  constexpr int kMaxGcap = 127;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(gemv_mma_kernel<BITS, MT, 2>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::smem(kMaxGcap));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemv_mma_kernel<BITS, MT, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::smem(kMaxGcap));
    int nsm_dev = 0;
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm_dev, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    sms[dev].store(nsm_dev, std::memory_order_relaxed);
    attr_set[dev].store(true, std::memory_order_release);
  }
  const int64_t tiles = (N + 31) / 32;
  const int64_t KU = K / 32, stages = (KU + 31) / 32;
  int ks = int((WQ_GEMV_MMA_TARGET_CTAS + tiles - 1) / tiles);
  ks = ks < 1 ? 1 : (ks > 8 ? 8 : ks);
  while (ks > 1 && stages / ks < WQ_GEMV_MMA_MIN_STAGES) --ks;
  const int64_t upg = g / 32;
  int64_t span = 1;
  for (int r = 0; r < ks; ++r) {
    const int64_t tb = stages * r / ks, te = stages * (r + 1) / ks;
    const int64_t ue = (te * 32 < KU ? te * 32 : KU) - 1;
    const int64_t sp = ue / upg - (tb * 32) / upg + 1;
    span = sp > span ? sp : span;
  }
  const int gcap = int(span < kMaxGcap ? span : kMaxGcap) | 1;
  const int smem = Cfg::smem(gcap);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(tiles), unsigned(ks), 1);
  cfg.blockDim = dim3(32 * (Cfg::NW + 1), 1, 1);
  cfg.dynamicSmemBytes = size_t(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = unsigned(ks);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const FastDiv fd{uint32_t(upg)};
  const int nsm_known = (dev >= 0 && dev < 64) ? sms[dev].load(std::memory_order_relaxed) : 0;
  const int64_t ctas = tiles * ks, nsm = nsm_known > 0 ? nsm_known : 1;
  constexpr int kRed = int(sizeof(float)) * Cfg::NW * MT * 32;   // static shared memory
  if ((ctas + 3 * nsm - 1) / (3 * nsm) < (ctas + 2 * nsm - 1) / (2 * nsm) &&
      3 * (smem + kRed + 1024) <= 228 * 1024)
    return cudaLaunchKernelEx(&cfg, gemv_mma_kernel<BITS, MT, 3>, tm, x, M, N, K, scales, zeros, fd, gcap, y);
  return cudaLaunchKernelEx(&cfg, gemv_mma_kernel<BITS, MT, 2>, tm, x, M, N, K, scales, zeros, fd, gcap, y);
}

template <int BITS>
cudaError_t launch_bits(const __nv_bfloat16* x, int M, int64_t N, int64_t K, const uint32_t* codes,
                        const __half* scales, const __half* zeros, int64_t g, __nv_bfloat16* y,
                        cudaStream_t st) {
  if (M <= 2) return launch_mt<BITS, 2>(x, M, N, K, codes, scales, zeros, g, y, st);
  if (M <= 4) return launch_mt<BITS, 4>(x, M, N, K, codes, scales, zeros, g, y, st);
  return launch_mt<BITS, 8>(x, M, N, K, codes, scales, zeros, g, y, st);
}

}  // namespace

bool gemv_mma_supported(int M, const void* x, const void* codes, int64_t K, int64_t g) {
  // 2..8 tokens, whole 128-code quads per scale group, TMA-aligned code rows and x rows
  return M >= 2 && M <= 8 && K % 128 == 0 && g % 128 == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(codes) & 15) == 0;
}

cudaError_t launch_gemv_mma(const __nv_bfloat16* x, int M, int64_t N, int64_t K, const uint32_t* codes,
                            const __half* scales, const __half* zeros, int bits, int64_t g,
                            __nv_bfloat16* y, cudaStream_t st) {
  switch (bits) {
    case 2: return launch_bits<2>(x, M, N, K, codes, scales, zeros, g, y, st);
    case 3: return launch_bits<3>(x, M, N, K, codes, scales, zeros, g, y, st);
    case 4: return launch_bits<4>(x, M, N, K, codes, scales, zeros, g, y, st);
    default: return launch_bits<8>(x, M, N, K, codes, scales, zeros, g, y, st);
  }
}

bool gemv_mma_read_and_clear_timeout(cudaError_t* err) {
  unsigned int v = 0;
  const unsigned int zero = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&v, g_gemv_mma_timeout, sizeof(v));
  if (e == cudaSuccess && v) e = cudaMemcpyToSymbol(g_gemv_mma_timeout, &zero, sizeof(zero));
  *err = e;
  return v != 0;
}

}  // namespace wq
