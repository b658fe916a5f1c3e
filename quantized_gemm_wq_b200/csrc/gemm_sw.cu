// gemm_sw.cu -- y = x . W'^T for batches of 17..255 rows on the Blackwell
// tensor cores (tcgen05), with the weight rows on the MMA's M side.
//
// Dequantise inside the matmul ("[Feature Request] 4bit and 2bit and 1bit
// quantization support": the weights stay packed and become floats on the
// GPU; "Platform For AI: BladeLLM model quantization", "Background
// information > Solutions": batching requests raises throughput).  A batch of
// a few dozen rows is still bound by the bytes of packed weights, but a
// CUDA-core or warp-MMA GEMV pays per token, and a 256-row batch tile wastes
// most of its MMA rows.  So the roles swap: 128 weight rows are the MMA's M
// side, the batch (padded to MT = 32, 64, 128 or 256 columns, rows past the
// batch zero-filled by TMA) its N side, and one tcgen05.mma M = 128, N = MT,
// K = 16 per 16 inputs covers the whole batch.
//
// One CTA computes 128 outputs for the whole batch over its share of K, in
// 64-wide K steps:
//   warp 0      TMA producer of the packed code tiles (128 rows x 128 codes,
//               unswizzled), as far ahead as the code ring allows;
//   warp 10     TMA producer of the x tiles (bf16, 128-byte swizzled,
//               MT x 64), which wait for the MMAs: kept apart so that the
//               code stream (the HBM traffic) never waits on them;
//   warp 1      owns tensor memory (MT fp32 columns x 128 lanes) and one lane
//               issues the MMAs, A = W' from shared memory, B = x;
//   warps 2..9  dequantise codes -> w' = bf16_rne(scale * (q - zero)) (exact
//               in fp32, rounded once) into the canonical K-major 128-byte
//               swizzled layout, then the epilogue: tcgen05.ld -> bf16 -> y.
// With one grid per row the MMA gets the exact integers q - zero and the fp32
// scale of each row (tensor-memory lane) is applied in the epilogue.
// One linear (gemm_sw_kernel): K is split over a thread-block cluster when
// the 128-row tiles leave SMs idle; every rank parks its fp32 partial tile in
// its own shared memory and each rank sums a share of the columns over all
// ranks through distributed shared memory.  Many linears
// (gemm_sw_grouped_kernel): one launch over all their row tiles, K not split.
// Every wait is bounded (bounded_wait.cuh): an expired wait raises this file's
// device flag, the CTA drains its copies and MMAs and frees its tensor memory.
#include <cuda.h>

#include <atomic>

#include "bounded_wait.cuh"
#include "grouped.h"
#include "wq_internal.cuh"

namespace wq {

__device__ unsigned int g_gemm_sw_timeout;

namespace {

constexpr int BN = 128, BK = 64, CK = 128;
constexpr int kDqWarps = 8;
constexpr int kXWarp = 2 + kDqWarps;                       // the x producer
constexpr int kThreads = 32 * (kXWarp + 1);
constexpr uint32_t kWBytes = uint32_t(BN) * BK * 2;       // one W' stage

#ifndef WQ_GEMM_SW_MAX_SPLIT
#define WQ_GEMM_SW_MAX_SPLIT 8
#endif
#ifndef WQ_GEMM_SW_MIN_STAGES
#define WQ_GEMM_SW_MIN_STAGES 4   // 128-wide code stages each split keeps at least
#endif

// Scales and zeros reach the dequantising warps in chunks of kChG groups:
// each warp copies its own 16 rows' windows (kChG halves plus an odd start,
// kChW words per row and array) one chunk ahead into a double buffer.
constexpr int kMaxSwLinears = 64;   // linears per grouped launch (kernel parameter space)
constexpr int kChG = 8;
constexpr int kChW = kChG / 2 + 1;
constexpr uint32_t kChWarpWords = 2u * 16 * 2 * kChW;              // [buffer][row][array][word]
constexpr uint32_t kChBytes = kDqWarps * kChWarpWords * 4;

template <int BITS, int MT>
struct SwCfg {
  static constexpr uint32_t kXBytes = uint32_t(MT) * BK * 2;          // one x stage
  static constexpr uint32_t kCBytes = uint32_t(BN) * CK * BITS / 8;   // one code stage
  static constexpr uint32_t kMisc = 1024 /* align */ + 512 /* barriers */ + 4 * BN /* row scales */ + kChBytes;
  // Two CTAs per SM when 3 W' stages, 3 x stages and 3 code stages fit in
  // half the shared memory, or else 2, 2 and 3; otherwise one CTA with
  // deeper rings.  The code ring (the HBM stream) takes what is left: the
  // bandwidth an SM draws follows the bytes it keeps in flight.
  static constexpr bool kTwo3 = MT <= 128 && 3 * kWBytes + 3 * kXBytes + 3 * kCBytes + kMisc <= 112 * 1024;
  static constexpr bool kTwo2 = MT <= 128 && 2 * kWBytes + 2 * kXBytes + 3 * kCBytes + kMisc <= 112 * 1024;
  static constexpr bool kTwo = kTwo3 || kTwo2;
  static constexpr uint32_t kBudget = kTwo ? 112 * 1024 : 226 * 1024;
  static constexpr int SW = kTwo3 ? 3 : (kTwo2 ? 2 : 4);
  static constexpr int SX = kTwo3 ? 3 : (kTwo2 ? 2 : (MT <= 128 ? 4 : 2));
  static constexpr int SCf = int((kBudget - kMisc - SW * kWBytes - SX * kXBytes) / kCBytes);
  static constexpr int SC = SCf > 8 ? 8 : SCf;
  static_assert(SC >= 3, "code ring");
  static constexpr uint32_t kRing = SX * kXBytes + SW * kWBytes + SC * kCBytes;
  static constexpr uint32_t kSmem = kRing + kMisc;
  static constexpr uint32_t kPartBytes = uint32_t(BN) * MT * 4;        // split-K partial tile
  static constexpr uint32_t kTmemCols = MT < 32 ? 32 : MT;
  // kind::f16: fp32 accumulator, bf16 A and B, both K-major, N = MT, M = 128
  static constexpr uint32_t kIdesc =
      (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(MT >> 3) << 17) | (uint32_t(BN >> 4) << 24);
  static_assert(kPartBytes <= kRing, "the partial tile is parked in the ring");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

// One linear of a grouped launch (tensor maps first: they need 64-byte alignment).
struct alignas(64) SwLin {
  CUtensorMap tm_x, tm_c;
  const __half* scales;
  const __half* zeros;
  __nv_bfloat16* y;
  int64_t N, K, g;
  FastDiv upg;
  int tile0;        // first CTA of this linear's row tiles
};
struct SwGroup {
  SwLin lin[kMaxSwLinears];
  int nlin;
  int64_t M;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile uint32_t* abort) {
  const uint32_t a = smem_u32(b);
  return bw::try_parity(a, parity) || bw::pipe_wait(a, parity, &g_gemm_sw_timeout, abort);
}
__device__ __forceinline__ void mbar_drain(uint64_t* b, uint32_t parity) {
  bw::drain_wait(smem_u32(b), parity, &g_gemm_sw_timeout);
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart, sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t(16u >> 4) << 16;
  d |= uint64_t(1024u >> 4) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float4 ld_peer_f4(const void* p, int rank) {
  uint32_t peer;
  float4 v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(peer) : "r"(smem_u32(p)), "r"(rank));
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(peer)
               : "memory");
  return v;
}
// 16 consecutive tensor-memory columns of this warp's 32 lanes -> registers.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

constexpr float pow2f(int e) {
  float r = 1.0f;
  for (int i = 0; i < e; ++i) r *= 2.0f;
  return r;
}
__device__ __forceinline__ uint32_t bf162_bits(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);   // a -> low half (lower address)
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
// bf16 pairs (codes 2j, 2j+1 of a unit) of w' = fma(q 2^-30, A, B), j = J..15,
// two lanes of fp32 per packed multiply and FMA: the code from one AND is the
// subnormal q 2^(p-149); times 2^(119-p) it is q 2^-30 exactly, and the FMA
// with A = s 2^30, B = -s z is exact (s q and s z have at most 20 significant
// bits), so the bf16 conversion is the only rounding.
template <int BITS, int J>
struct SwDq {
  __device__ __forceinline__ static void run(const uint32_t (&w)[BITS], uint64_t AA, uint64_t BB,
                                             uint32_t (&out)[16]) {
    constexpr float F0 = pow2f(119 - code_p<BITS>(2 * J));
    constexpr float F1 = pow2f(119 - code_p<BITS>(2 * J + 1));
    const uint64_t q2 = f32x2(code_subnormal<BITS, 2 * J>(w), code_subnormal<BITS, 2 * J + 1>(w));
    uint64_t v;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(v) : "l"(q2), "l"(f32x2(F0, F1)));
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(v) : "l"(v), "l"(AA), "l"(BB));
    uint32_t o;
    asm("{\n\t.reg .f32 lo, hi;\n\t"
        "mov.b64 {lo, hi}, %1;\n\t"
        "cvt.rn.bf16x2.f32 %0, hi, lo;\n\t}"
        : "=r"(o)
        : "l"(v));
    out[J] = o;                                          // code 2j in the low half
    if constexpr (J + 1 < 16) SwDq<BITS, J + 1>::run(w, AA, BB, out);
  }
};
template <int BITS>
__device__ __forceinline__ void lds_unit(const uint8_t* p, uint32_t (&w)[BITS]) {
  if constexpr (BITS == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x; w[1] = v.y;
  } else if constexpr (BITS == 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
  } else if constexpr (BITS == 8) {
    const uint4 a = reinterpret_cast<const uint4*>(p)[0];
    const uint4 b = reinterpret_cast<const uint4*>(p)[1];
    w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
    w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
  } else {
    const uint32_t* q = reinterpret_cast<const uint32_t*>(p);
    w[0] = q[0]; w[1] = q[1]; w[2] = q[2];
  }
}

// One CTA's work: output rows n0 .. n0 + 127 of one linear over split kr of
// ks along K (the tensor maps live in kernel parameter space).
template <int BITS, int MT>
__device__ __forceinline__ void sw_tile(const CUtensorMap* tm_x, const CUtensorMap* tm_c,
                                        const __half* __restrict__ scales, const __half* __restrict__ zeros,
                                        int64_t M, int64_t N, int64_t K, int64_t g, FastDiv units_per_group,
                                        __nv_bfloat16* __restrict__ y, int64_t n0, int ks, int kr) {
  using Cfg = SwCfg<BITS, MT>;
  constexpr int SX = Cfg::SX, SW = Cfg::SW, SC = Cfg::SC;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = base;                                   // [SX][MT x 64 bf16], swizzled
  uint8_t* sW = sX + SX * Cfg::kXBytes;                 // [SW][128 x 64 bf16], swizzled
  uint8_t* sC = sW + SW * kWBytes;                      // [SC][128 rows x 128 codes]
  uint32_t* sCh = reinterpret_cast<uint32_t*>(sC + SC * Cfg::kCBytes);   // [kDqWarps][kChWarpWords]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sCh + kDqWarps * kChWarpWords);
  uint64_t* full_x = bars;             // TMA x landed             (1 arrival + bytes)
  uint64_t* empty_x = full_x + SX;     // MMAs done with the x slot (commit)
  uint64_t* full_w = empty_x + SX;     // W' written              (kDqWarps arrivals)
  uint64_t* empty_w = full_w + SW;     // MMAs done with W'        (commit)
  uint64_t* full_c = empty_w + SW;     // TMA codes landed         (1 arrival + bytes)
  uint64_t* empty_c = full_c + SC;     // codes consumed           (kDqWarps arrivals)
  uint64_t* tmem_full = empty_c + SC;  // accumulators final       (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_full + 1);
  volatile uint32_t* abort = tmem_slot + 1;
  float* row_scale = reinterpret_cast<float*>(bars + 64);   // [128], per-row grids

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KT = int((K + BK - 1) / BK);
  const int KC = (KT + 1) / 2;
  const int kt0 = 2 * int(int64_t(KC) * kr / ks);
  const int kt1 = min(KT, 2 * int(int64_t(KC) * (kr + 1) / ks));
  const bool rowwise = (g == K);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) {
      mbar_init(&full_x[s], 1);
      mbar_init(&empty_x[s], 1);
    }
    for (int s = 0; s < SW; ++s) {
      mbar_init(&full_w[s], kDqWarps);
      mbar_init(&empty_w[s], 1);
    }
    for (int s = 0; s < SC; ++s) {
      mbar_init(&full_c[s], 1);
      mbar_init(&empty_c[s], kDqWarps);
    }
    mbar_init(tmem_full, 1);
    *abort = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(Cfg::kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ep_ok = false;

  if (warp == 0) {
    // ------------------------------------------------------------ code producer
    if (lane == 0) {
      const int nc = (kt1 - kt0 + 1) / 2;              // 128-wide code stages of this split
      int issued = 0;
      bool ok = true;
      for (int c = 0; c < nc && ok; ++c) {
        const int cs = c % SC;
        if (c >= SC) ok = mbar_wait(&empty_c[cs], ((c / SC) - 1) & 1, abort);
        if (!ok) break;
        mbar_expect_tx(&full_c[cs], Cfg::kCBytes);
        tma_load_2d(sC + cs * Cfg::kCBytes, tm_c, &full_c[cs], ((kt0 >> 1) + c) * (CK * BITS / 32), int(n0));
        ++issued;
      }
      if (!ok)   // copies in flight land before shared memory goes away
        for (int c = (issued > SC ? issued - SC : 0); c < issued; ++c) mbar_drain(&full_c[c % SC], (c / SC) & 1);
    }
  } else if (warp == kXWarp) {
    // ------------------------------------------------------------ x producer
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int kt = kt0; kt < kt1 && ok; ++kt) {
        const int j = kt - kt0, s = j % SX;
        if (j >= SX) ok = mbar_wait(&empty_x[s], ((j / SX) - 1) & 1, abort);
        if (!ok) break;
        mbar_expect_tx(&full_x[s], Cfg::kXBytes);
        tma_load_2d(sX + s * Cfg::kXBytes, tm_x, &full_x[s], kt * BK, 0);
        ++issued;
      }
      if (!ok)
        for (int j = (issued > SX ? issued - SX : 0); j < issued; ++j) mbar_drain(&full_x[j % SX], (j / SX) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int kt = kt0; kt < kt1 && ok; ++kt) {
        const int j = kt - kt0;
        const int sx = j % SX, sw = j % SW;
        ok = mbar_wait(&full_x[sx], (j / SX) & 1, abort) && mbar_wait(&full_w[sw], (j / SW) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sW + sw * kWBytes);
        const uint32_t b0 = smem_u32(sX + sx * Cfg::kXBytes);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          umma(tmem, sw128_desc(a0 + kk * 32), sw128_desc(b0 + kk * 32), Cfg::kIdesc,
               (kt > kt0 || kk > 0) ? 1u : 0u);
        umma_commit(&empty_x[sx]);
        umma_commit(&empty_w[sw]);
      }
      umma_commit(tmem_full);      // always: the teardown waits on it before freeing tensor memory
    }
  } else if (warp < kXWarp) {
    // ------------------------------------------------------------ dequantise
    const int td = threadIdx.x - 64;                 // 0..255
    const int r = td >> 1, cu = td & 1;              // tile row, 32-code unit of the 64-wide step
    const int64_t n = n0 + r;
    const int64_t G = K / g;
    if (rowwise) {                                   // epilogue scale of each row
      if (cu == 0) row_scale[r] = n < N ? __half2float(scales[n * G]) : 0.0f;
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kDqWarps) : "memory");
    }
    // per-row grids: the zero of the row, once (the scale goes to the epilogue)
    const uint16_t zsym = uint16_t((BITS - 1 + 15) << 10);   // fp16 2^(b-1): the symmetric grid's zero
    uint16_t rz2 = zsym;
    if (rowwise && zeros && n < N) rz2 = __ldg(reinterpret_cast<const unsigned short*>(zeros) + n * G);
    // grouped grids: chunk q holds groups [grp0 + 8 q, grp0 + 8 q + 8) of the
    // warp's rows; lane l copies array l & 1 (scales, zeros) of row l / 2
    const int dw = warp - 2;
    uint32_t* chw = sCh + dw * kChWarpWords;
    const uint32_t grp0 = rowwise ? 0u : units_per_group.div(uint32_t((kt0 * BK) >> 5));
    const uint32_t gend = rowwise ? 0u : units_per_group.div(uint32_t((kt1 * BK - 1) >> 5)) + 1u;
    auto load_chunk = [&](int qc) {
      const int rr = 16 * dw + (lane >> 1), arr = lane & 1;
      const int64_t nn = n0 + rr;
      const __half* src = arr ? zeros : scales;
      const uint32_t ga = grp0 + uint32_t(qc) * kChG;
      const uint32_t gb = min(ga + uint32_t(kChG), gend);
      if (src != nullptr && nn < N && ga < gb) {
        const int64_t e0 = nn * G + ga, a0 = e0 & ~int64_t(1), end = N * G;
        const int nw = int((e0 + (gb - ga) - a0 + 1) >> 1);
        const uint32_t dst = smem_u32(chw + (((qc & 1) * 16 + (lane >> 1)) * 2 + arr) * kChW);
        for (int w = 0; w < nw; ++w) {
          const int64_t a = a0 + 2 * w;                  // a < end: the window ends at a needed group
          const uint32_t bytes = a + 2 <= end ? 4u : 2u;
          asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst + 4 * w), "l"(src + a), "r"(bytes)
                       : "memory");
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    if (!rowwise) load_chunk(0);
    int qcur = -1;
    bool ok = true;
    for (int kt = kt0; kt < kt1 && ok; ++kt) {
      const int j = kt - kt0;
      const int c = j >> 1, cs = c % SC, s = j % SW;
      ok = mbar_wait(&full_c[cs], (c / SC) & 1, abort);
      if (ok && j >= SW) ok = mbar_wait(&empty_w[s], ((j / SW) - 1) & 1, abort);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      // scale and zero of this thread's 32 codes as raw fp16 bits: element h
      // of the row's window in the chunk (h = the parity of the window's first
      // element + the group's offset in the chunk)
      uint16_t s2 = 0x3C00, z2 = rz2;                   // 0x3C00: fp16 1.0
      if (!rowwise) {
        const int q = int((units_per_group.div(uint32_t((kt * BK) >> 5)) - grp0) / kChG);   // warp-uniform
        if (q != qcur) {
          __syncwarp();                                  // every lane is done with chunk q - 1's buffer
          if (grp0 + uint32_t(q + 1) * kChG < gend) load_chunk(q + 1);
          else asm volatile("cp.async.commit_group;" ::: "memory");
          asm volatile("cp.async.wait_group 1;" ::: "memory");   // chunk q has landed (this lane's part)
          __syncwarp();                                  // ... and every lane's
          qcur = q;
        }
        const uint32_t ga = grp0 + uint32_t(q) * kChG;
        const uint32_t h = uint32_t((n * G + ga) & 1) + units_per_group.div(uint32_t((kt * BK + 32 * cu) >> 5)) - ga;
        const unsigned short* ch =
            reinterpret_cast<const unsigned short*>(chw + (((q & 1) * 16 + (lane >> 1)) * 2) * kChW);
        s2 = ch[h];
        z2 = zeros ? ch[2 * kChW + h] : zsym;
      }
      const float sc = __half2float(__ushort_as_half(s2));
      const float A = sc * 0x1p30f, B = -sc * __half2float(__ushort_as_half(z2));
      const uint64_t AA = f32x2(A, A), BB = f32x2(B, B);
      const uint8_t* ctile = sC + cs * Cfg::kCBytes;
      uint8_t* wtile = sW + s * kWBytes;
      const int ucode = (kt & 1) * 2 + cu;           // unit within the 128-code stage
      uint32_t w[BITS];
      lds_unit<BITS>(ctile + r * (CK * BITS / 8) + ucode * (4 * BITS), w);
      uint32_t p[16];
      SwDq<BITS, 0>::run(w, AA, BB, p);
      uint8_t* wrow = wtile + r * 128;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int chunk = (cu * 4 + jj) ^ (r & 7);
        *reinterpret_cast<uint4*>(wrow + chunk * 16) = make_uint4(p[4 * jj], p[4 * jj + 1], p[4 * jj + 2], p[4 * jj + 3]);
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&full_w[s]);
        if ((j & 1) || kt == kt1 - 1) mbar_arrive(&empty_c[cs]);
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");   // no copy may land after the CTA exits
    if (ok) ok = mbar_wait(tmem_full, 0, abort);
    ep_ok = __all_sync(0xffffffffu, ok);             // tcgen05.ld needs the whole warp
  }

  // ------------------------------------------------------------ epilogue
  // Warp w (2..9) reads tensor-memory lane quarter w % 4 (rows 32 (w % 4) ..)
  // and column half (w - 2) / 4.  Without split-K it converts its columns to
  // bf16 and stores them.  With split-K every rank parks its fp32 partial tile
  // in its own (now idle) shared memory as [column / 4][row][4] floats; then
  // rank r sums the 4-column groups u = r, r + ks, ... over all ranks (in
  // rank order, through distributed shared memory) and stores them, so the
  // reduction is spread over the cluster.  Every thread takes part in the
  // cluster barriers.
  const bool dq = warp >= 2 && warp < kXWarp;
  const int q = warp & 3, ch = (warp - 2) >> 2;
  const int row = 32 * q + lane;
  const int64_t n = n0 + row;
  float4* part = reinterpret_cast<float4*>(sX);
  const uint32_t tbase = tmem + (uint32_t(32 * q) << 16);
  constexpr int HALF = MT / 2;
  if (ks == 1) {
    if (dq && ep_ok) {
      tc_fence_after();
      const float rs = rowwise ? row_scale[row] : 1.0f;
#pragma unroll 1
      for (int c0 = ch * HALF; c0 < (ch + 1) * HALF; c0 += 16) {
        float v[16];
        tmem_ld16(tbase + uint32_t(c0), v);
        if (n < N) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int64_t m = c0 + i;
            if (m < M) y[m * N + n] = __float2bfloat16_rn(rowwise ? v[i] * rs : v[i]);
          }
        }
      }
    }
  } else {
    if (dq && ep_ok) {
      tc_fence_after();
#pragma unroll 1
      for (int c0 = ch * HALF; c0 < (ch + 1) * HALF; c0 += 16) {
        float v[16];
        tmem_ld16(tbase + uint32_t(c0), v);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          part[((c0 >> 2) + u) * BN + row] = make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
      }
    }
    cluster_sync();
    if (dq) {
      const float rs = rowwise ? row_scale[row] : 1.0f;
#pragma unroll 1
      for (int u = kr + ks * ch; u < MT / 4; u += 2 * ks) {
        float4 pv[WQ_GEMM_SW_MAX_SPLIT];
#pragma unroll
        for (int pr = 0; pr < WQ_GEMM_SW_MAX_SPLIT; ++pr)
          if (pr < ks) pv[pr] = ld_peer_f4(&part[u * BN + row], pr);   // all loads in flight at once
        float4 v = pv[0];
#pragma unroll
        for (int pr = 1; pr < WQ_GEMM_SW_MAX_SPLIT; ++pr)
          if (pr < ks) {
            v.x += pv[pr].x;
            v.y += pv[pr].y;
            v.z += pv[pr].z;
            v.w += pv[pr].w;
          }
        if (n < N) {
          const float o[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int64_t m = 4 * u + i;
            if (m < M) y[m * N + n] = __float2bfloat16_rn(rowwise ? o[i] * rs : o[i]);
          }
        }
      }
    }
    cluster_sync();                                  // peers keep their partials until read
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*abort) {
      if (lane == 0) mbar_drain(tmem_full, 0);       // MMAs issued finish before tensor memory is freed
      __syncwarp();
    }
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Cfg::kTmemCols));
  }
}

// Two resident CTAs of 11 warps put up to 6 warps on one of the SM's four
// schedulers, whose register file holds 16K registers: 80 per thread at most
// (declared as a 384-thread bound for two CTAs).
#define WQ_SW_BOUNDS __launch_bounds__(SwCfg<BITS, MT>::kTwo ? 384 : kThreads, SwCfg<BITS, MT>::kTwo ? 2 : 1)

// One linear: blockIdx.x the 128-row tile, blockIdx.z the split of K (a
// cluster of gridDim.z CTAs along K).
template <int BITS, int MT>
__global__ void WQ_SW_BOUNDS gemm_sw_kernel(const __grid_constant__ CUtensorMap tm_x,
                                            const __grid_constant__ CUtensorMap tm_c,
                                            const __half* __restrict__ scales, const __half* __restrict__ zeros,
                                            int64_t M, int64_t N, int64_t K, int64_t g, FastDiv units_per_group,
                                            __nv_bfloat16* __restrict__ y) {
  sw_tile<BITS, MT>(&tm_x, &tm_c, scales, zeros, M, N, K, g, units_per_group, y, int64_t(blockIdx.x) * BN,
                    int(gridDim.z), int(blockIdx.z));
}

// Many linears in one launch: CTA b takes row tile b - tile0 of the linear
// whose tiles hold b, over the whole of K (with thousands of tiles in a
// decode step the SMs stay busy without splitting K).
template <int BITS, int MT>
__global__ void WQ_SW_BOUNDS gemm_sw_grouped_kernel(const __grid_constant__ SwGroup p) {
  const int b = int(blockIdx.x);
  int l = 0;
  while (l + 1 < p.nlin && p.lin[l + 1].tile0 <= b) ++l;
  const SwLin& L = p.lin[l];
  sw_tile<BITS, MT>(&L.tm_x, &L.tm_c, L.scales, L.zeros, p.M, L.N, L.K, L.g, L.upg, L.y,
                    int64_t(b - L.tile0) * BN, 1, 0);
}

// ------------------------------------------------------------------ host
#ifndef WQ_GEMM_SW_SPLIT_STAGES
#define WQ_GEMM_SW_SPLIT_STAGES 1.0
#endif
constexpr double kWaveStages = 4.0;    // prologue + epilogue of one CTA, in code stages
constexpr double kSplitStages = WQ_GEMM_SW_SPLIT_STAGES;   // partial-tile exchange per extra split
constexpr double kPairGain = 1.35;     // throughput of an SM running two CTAs, relative to one

template <int BITS, int MT>
cudaError_t launch_mt(const __nv_bfloat16* x, int64_t M, int64_t N, int64_t K, const uint32_t* codes,
                      const __half* scales, const __half* zeros, int64_t g, __nv_bfloat16* y, cudaStream_t st) {
  using Cfg = SwCfg<BITS, MT>;
  alignas(64) CUtensorMap tx, tc;
  if (!make_tensor_map_2d(&tx, TmaType::kBF16, x, uint64_t(K), uint64_t(M), uint64_t(K) * 2, BK, MT, 128) ||
      !make_tensor_map_2d(&tc, TmaType::kU32, codes, uint64_t(K * BITS / 32), uint64_t(N), uint64_t(K * BITS / 8),
                          CK * BITS / 32, BN, 0))
    return cudaErrorInvalidValue;
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_sw_kernel<BITS, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(Cfg::kSmem));
    // all of the unified L1 as shared memory: the two-CTA builds need it
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_sw_kernel<BITS, MT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               int(cudaSharedmemCarveoutMaxShared));
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  // Split K over a cluster when the 128-row tiles alone fill the SMs badly.
  // Cost in units of one 128-wide code stage: a CTA takes its share of K
  // plus a fixed prologue/epilogue and an exchange cost per extra split; an
  // SM that holds two CTAs (the two-CTA builds) runs each at kPairGain / 2
  // of the speed of one.  The resident CTAs per SM come from the build (the
  // runtime's occupancy query reports one CTA per SM for the two-CTA
  // builds, which ncu and the launches show resident in pairs).
  const int64_t tiles = (N + BN - 1) / BN;
  const int64_t kc = K / CK;
  int nsm = 0;
  if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm < 1) nsm = 1;
  int ks = 1;
  double best = 1e300;
  for (int c = 1; c <= WQ_GEMM_SW_MAX_SPLIT; ++c) {
    if (c > 1 && kc / c < WQ_GEMM_SW_MIN_STAGES) break;
    const int64_t n = tiles * c;
    const double per_cta = double(kc) / c + kWaveStages + kSplitStages * (c - 1);
    double t;
    if (Cfg::kTwo && n > nsm)
      t = double((n + 2 * nsm - 1) / (2 * nsm)) * 2.0 * per_cta / kPairGain;
    else
      t = double((n + nsm - 1) / nsm) * per_cta;
    if (t < best - 1e-9) {
      best = t;
      ks = c;
    }
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(tiles), 1, unsigned(ks));
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cfg::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = unsigned(ks);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_sw_kernel<BITS, MT>, tx, tc, scales, zeros, M, N, K, g,
                            FastDiv(uint32_t(g / 32)), y);
}

template <int BITS>
cudaError_t launch_bits(const __nv_bfloat16* x, int64_t M, int64_t N, int64_t K, const uint32_t* codes,
                        const __half* scales, const __half* zeros, int64_t g, __nv_bfloat16* y, cudaStream_t st) {
  if (M <= 32) return launch_mt<BITS, 32>(x, M, N, K, codes, scales, zeros, g, y, st);
  if (M <= 64) return launch_mt<BITS, 64>(x, M, N, K, codes, scales, zeros, g, y, st);
  if (M <= 128) return launch_mt<BITS, 128>(x, M, N, K, codes, scales, zeros, g, y, st);
  return launch_mt<BITS, 256>(x, M, N, K, codes, scales, zeros, g, y, st);
}

template <int BITS, int MT>
cudaError_t launch_grouped_mt(const GroupedLinear* lins, int count, int64_t M, cudaStream_t st) {
  using Cfg = SwCfg<BITS, MT>;
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_sw_grouped_kernel<BITS, MT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(Cfg::kSmem));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemm_sw_grouped_kernel<BITS, MT>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               int(cudaSharedmemCarveoutMaxShared));
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  SwGroup p;
  for (int c0 = 0; c0 < count; c0 += kMaxSwLinears) {
    const int n = count - c0 < kMaxSwLinears ? count - c0 : kMaxSwLinears;
    p.nlin = n;
    p.M = M;
    int tiles = 0;
    for (int j = 0; j < n; ++j) {
      const GroupedLinear& L = lins[c0 + j];
      SwLin& d = p.lin[j];
      if (!make_tensor_map_2d(&d.tm_x, TmaType::kBF16, L.x, uint64_t(L.K), uint64_t(M), uint64_t(L.K) * 2, BK, MT,
                              128) ||
          !make_tensor_map_2d(&d.tm_c, TmaType::kU32, L.codes, uint64_t(L.K * BITS / 32), uint64_t(L.N),
                              uint64_t(L.K * BITS / 8), CK * BITS / 32, BN, 0))
        return cudaErrorInvalidValue;
      d.scales = L.scales;
      d.zeros = L.zeros;
      d.y = L.y;
      d.N = L.N;
      d.K = L.K;
      d.g = L.group;
      d.upg = FastDiv(uint32_t(L.group / 32));
      d.tile0 = tiles;
      tiles += int((L.N + BN - 1) / BN);
    }
    gemm_sw_grouped_kernel<BITS, MT><<<dim3(unsigned(tiles)), dim3(kThreads), Cfg::kSmem, st>>>(p);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

template <int BITS>
cudaError_t launch_grouped_bits(const GroupedLinear* lins, int count, int64_t M, cudaStream_t st) {
  if (M <= 32) return launch_grouped_mt<BITS, 32>(lins, count, M, st);
  if (M <= 64) return launch_grouped_mt<BITS, 64>(lins, count, M, st);
  if (M <= 128) return launch_grouped_mt<BITS, 128>(lins, count, M, st);
  return launch_grouped_mt<BITS, 256>(lins, count, M, st);
}

}  // namespace

bool gemm_sw_supported(int64_t M, int64_t K) { return M > 16 && M < 256 && K % CK == 0; }

cudaError_t launch_gemm_sw_grouped(const GroupedLinear* lins, int count, int64_t M, int bits, cudaStream_t st) {
  switch (bits) {
    case 2: return launch_grouped_bits<2>(lins, count, M, st);
    case 3: return launch_grouped_bits<3>(lins, count, M, st);
    case 4: return launch_grouped_bits<4>(lins, count, M, st);
    default: return launch_grouped_bits<8>(lins, count, M, st);
  }
}

cudaError_t launch_gemm_sw(const __nv_bfloat16* x, int64_t M, int64_t N, int64_t K, const uint32_t* codes,
                           const __half* scales, const __half* zeros, int bits, int64_t g, __nv_bfloat16* y,
                           cudaStream_t st) {
  switch (bits) {
    case 2: return launch_bits<2>(x, M, N, K, codes, scales, zeros, g, y, st);
    case 3: return launch_bits<3>(x, M, N, K, codes, scales, zeros, g, y, st);
    case 4: return launch_bits<4>(x, M, N, K, codes, scales, zeros, g, y, st);
    default: return launch_bits<8>(x, M, N, K, codes, scales, zeros, g, y, st);
  }
}

bool gemm_sw_read_and_clear_timeout(cudaError_t* err) {
  unsigned int v = 0;
  const unsigned int zero = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&v, g_gemm_sw_timeout, sizeof(v));
  if (e == cudaSuccess && v) e = cudaMemcpyToSymbol(g_gemm_sw_timeout, &zero, sizeof(zero));
  *err = e;
  return v != 0;
}

}  // namespace wq
