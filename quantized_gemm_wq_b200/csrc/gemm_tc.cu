// gemm_tc.cu -- prefill y = x . W'^T on the Blackwell tensor cores (tcgen05).
//
// Dequantise inside the matmul ("[Feature Request] 4bit and 2bit and 1bit
// quantization support": weights stay packed and become floats on the GPU;
// "Platform For AI: BladeLLM model quantization", "Background information >
// Solutions").  For a batch of hundreds of rows the product is a dense
// contraction, so it runs on the tensor cores with W' rebuilt in bf16 on chip.
//
// One CTA computes a 256 x 256 tile of y (256 batch rows x 256 output
// features) over its share of K, in 64-wide K steps (the whole K, or a share
// of it when K is split over a thread-block cluster: the ranks' partial
// tiles meet through distributed shared memory, each rank summing a share of
// the columns; whole waves of tiles and the leftover tiles may go to two
// launches, the leftovers split, the second a programmatic dependent of the
// first so that it fills SMs as they free up):
//   warp 0      TMA producer: x tiles (bf16, 128-byte swizzled, 256 x 64) and
//               packed code tiles (256 rows x 128 codes, unswizzled) into two
//               shared-memory rings (W' has a third, written by warps 2..9);
//   warp 1      owns tensor memory (512 columns: two 128 x 256 fp32
//               accumulators) and one lane issues the MMAs:
//               tcgen05.mma.cta_group::1.kind::f16, M = 128, N = 256, K = 16,
//               bf16 x bf16 -> fp32, A = x (two 128-row halves), B = W';
//   warps 2..9  dequantise: codes -> w' = bf16_rne(scale * (q - zero)) (the
//               product is exact in fp32, so w' is rounded once) written in the
//               canonical K-major 128-byte-swizzled layout the MMA reads, then
//               the epilogue: tcgen05.ld of the accumulators -> bf16 -> y.
// With one grid per row the scale is constant along K, so the MMA is fed the
// exact integers q - zero (exact in bf16 up to 256 in magnitude) and the fp32
// scale of each output column is applied in the epilogue: the products are
// then exact, as in the GEMV.  (Rounding scale * (q - zero) to bf16 would give
// every weight of a row the same relative error, which does not average out.)
// Stage hand-offs use mbarriers; tcgen05.commit frees a stage when the MMAs
// that read it have completed.  Every wait is bounded in time: a wait that
// expires raises a device flag (read by wq_last_device_error), makes the CTA
// stop, drain its copies in flight and free its tensor memory.
#include <cuda.h>   // CUtensorMap types only; the driver entry point is fetched at run time

#include <atomic>

#include "bounded_wait.cuh"
#include "wq_internal.cuh"

namespace wq {

// Set by a kernel that gave up a bounded wait; read and cleared by the host.
__device__ unsigned int g_timeout_flag;

namespace {

constexpr int BM = 256, BN = 256, BK = 64, CK = 128;

#ifndef WQ_GEMM_MAX_SPLIT
#define WQ_GEMM_MAX_SPLIT 8   // largest split-K cluster
#endif
#ifndef WQ_GEMM_MIN_STAGES
#define WQ_GEMM_MIN_STAGES 8  // 128-wide code stages each split keeps at least
#endif
constexpr int kMmaM = 128, kMmaN = 256, kMmaK = 16;
#ifndef WQ_GEMM_DQ_WARPS
#define WQ_GEMM_DQ_WARPS 8
#endif
constexpr int kDqWarps = WQ_GEMM_DQ_WARPS;                 // 8 or 16
constexpr int kRowsPerThread = BN / (16 * kDqWarps);       // W' rows each dequantising thread writes
constexpr int kColGroups = kDqWarps / 4;                   // epilogue column groups per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kDqWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kABytes = BM * BK * 2;
constexpr uint32_t kBBytes = BN * BK * 2;

template <int BITS>
struct TcCfg {
  // One more W' stage than codes lets the dequantising warps run a full
  // k-block ahead of the MMAs; the x ring keeps three TMA loads in flight.
  // (4 x / 2 W' stages measured 3% slower on the K = 13824 down projection,
  // 3 x / 4 code stages no faster than 4 / 2 / 2.) 8-bit codes are twice as
  // large, so their rings stay at 3 / 2 / 2.
  static constexpr int kXStages = 3;                       // x ring (64 K each)
  static constexpr int kWStages = BITS == 8 ? 2 : 3;       // W' ring (64 K each)
  static constexpr int kCStages = 2;                       // codes ring (128 K each)
  static constexpr uint32_t kCBytes = uint32_t(BN) * CK * BITS / 8;
  static constexpr uint32_t kRingBytes =
      kXStages * kABytes + kWStages * kBBytes + kCStages * kCBytes;
  static constexpr uint32_t kSmem = kRingBytes + 1024 + 256 + 4 * BN;
};
static_assert(TcCfg<4>::kSmem <= 232448, "shared memory");
static_assert(TcCfg<8>::kSmem <= 232448, "shared memory");
static_assert(TcCfg<3>::kSmem <= 232448, "shared memory");

// ------------------------------------------------------------------ PTX
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
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)),
               "r"(bytes)
               : "memory");
}
// Waits: bounded_wait.cuh (pipeline waits give up after its limit, raising
// the CTA abort word and g_timeout_flag; exit-path drains ignore the abort).
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile uint32_t* abort) {
  const uint32_t a = smem_u32(b);
  return bw::try_parity(a, parity) || bw::pipe_wait(a, parity, &g_timeout_flag, abort);
}
__device__ __forceinline__ void mbar_drain(uint64_t* b, uint32_t parity) {
  bw::drain_wait(smem_u32(b), parity, &g_timeout_flag);
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (SBO), sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t(16u >> 4) << 16;
  d |= uint64_t(1024u >> 4) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kMmaN >> 3) << 17) |
                            (uint32_t(kMmaM >> 4) << 24);

__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(kIdesc), "r"(accum));
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 16-byte load from the same shared-memory offset in cluster rank `rank`.
__device__ __forceinline__ float4 ld_peer_f4(const void* p, int rank) {
  uint32_t peer;
  float4 v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(peer) : "r"(smem_u32(p)), "r"(rank));
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(peer) : "memory");
  return v;
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

constexpr float pow2f(int e) {
  float r = 1.0f;
  for (int i = 0; i < e; ++i) r *= 2.0f;
  return r;
}

__device__ __forceinline__ uint32_t bf162_bits(float a, float b);

__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

// bf16 pairs (codes 2j, 2j+1 of a unit) of w' = fma(q 2^-30, A, B), j = J..15,
// two codes per packed fp32 multiply and FMA (the same IEEE operations as
// two scalar ones); AA, BB hold A and B in both lanes.
template <int BITS, int J>
struct DqPairs {
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
    if constexpr (J + 1 < 16) DqPairs<BITS, J + 1>::run(w, AA, BB, out);
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

__device__ __forceinline__ uint32_t bf162_bits(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);   // a -> low half (lower address)
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_c,
               const __half* __restrict__ scales, const __half* __restrict__ zeros, int64_t M,
               int64_t N, int64_t K, int64_t g, FastDiv units_per_group,
               __nv_bfloat16* __restrict__ y, int tile0, int ntn) {
  using Cfg = TcCfg<BITS>;
  constexpr int SX = Cfg::kXStages, SW = Cfg::kWStages, SC = Cfg::kCStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = base;                                   // [SX][256 x 64 bf16], swizzled
  uint8_t* sB = sA + SX * kABytes;                      // [SW][256 x 64 bf16], swizzled
  uint8_t* sC = sB + SW * kBBytes;                      // [SC][256 x 128 codes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sC + SC * Cfg::kCBytes);
  uint64_t* full_a = bars;             // TMA x landed            (1 arrival + bytes)
  uint64_t* empty_a = full_a + SX;     // MMAs done with x slot   (commit)
  uint64_t* full_b = empty_a + SX;     // W' written             (kDqWarps arrivals)
  uint64_t* empty_b = full_b + SW;     // MMAs done with W' slot (commit)
  uint64_t* full_c = empty_b + SW;     // TMA codes landed       (1 arrival + bytes)
  uint64_t* empty_c = full_c + SC;     // codes consumed         (kDqWarps arrivals)
  uint64_t* tmem_full = empty_c + SC;  // accumulators final     (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_full + 1);
  volatile uint32_t* abort = tmem_slot + 1;

  float* col_scale = reinterpret_cast<float*>(tmem_slot + 2);   // [BN], per-row grids only

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // output tile t = tile0 + blockIdx.x, row-major over (M tiles, N tiles)
  const int t = tile0 + int(blockIdx.x);
  const int64_t n0 = int64_t(t % ntn) * BN, m0 = int64_t(t / ntn) * BM;
  const int KT = int((K + BK - 1) / BK);
  // Split-K over the CTAs of a cluster (gridDim.z of them): this CTA takes the
  // 128-wide code stages [cb, ce), i.e. K steps [kt0, kt1); the partial tiles
  // are added in cluster rank 0 through distributed shared memory.
  const int ks = int(gridDim.z), kr = int(blockIdx.z);
  const int KC = (KT + 1) / 2;
  const int kt0 = 2 * int(int64_t(KC) * kr / ks);
  const int kt1 = min(KT, 2 * int(int64_t(KC) * (kr + 1) / ks));
  const bool rowwise = (g == K);

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) {
      mbar_init(&full_a[s], 1);
      mbar_init(&empty_a[s], 1);
    }
    for (int s = 0; s < SW; ++s) {
      mbar_init(&full_b[s], kDqWarps);
      mbar_init(&empty_b[s], 1);
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
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ep_ok = false;                         // dequant warps: accumulators are final
  // A second launch of this kernel over other tiles of the same y (the
  // leftover tiles of a two-launch plan) may take SMs as this one frees them.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued_a = 0, issued_c = 0;
      bool ok = true;
      for (int kt = kt0; kt < kt1 && ok; ++kt) {
        const int j = kt - kt0;                         // local step (ring phase)
        if ((j & 1) == 0) {                             // codes for K [kt*64, kt*64 + 128)
          const int c = j >> 1, cs = c % SC;
          if (c >= SC) ok = mbar_wait(&empty_c[cs], ((c / SC) - 1) & 1, abort);
          if (!ok) break;
          mbar_expect_tx(&full_c[cs], Cfg::kCBytes);
          tma_load_2d(sC + cs * Cfg::kCBytes, &tm_c, &full_c[cs], (kt >> 1) * (CK * BITS / 32), int(n0));
          ++issued_c;
        }
        const int s = j % SX;
        if (j >= SX) ok = mbar_wait(&empty_a[s], ((j / SX) - 1) & 1, abort);
        if (!ok) break;
        mbar_expect_tx(&full_a[s], kABytes);
        tma_load_2d(sA + s * kABytes, &tm_x, &full_a[s], kt * BK, int(m0));
        ++issued_a;
      }
      if (!ok) {   // let the copies still in flight land before shared memory goes away
        for (int kt = (issued_a > SX ? issued_a - SX : 0); kt < issued_a; ++kt)
          mbar_drain(&full_a[kt % SX], (kt / SX) & 1);
        for (int c = (issued_c > SC ? issued_c - SC : 0); c < issued_c; ++c)
          mbar_drain(&full_c[c % SC], (c / SC) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int kt = kt0; kt < kt1 && ok; ++kt) {
        const int j = kt - kt0;
        const int sx = j % SX, sw = j % SW;
        ok = mbar_wait(&full_a[sx], (j / SX) & 1, abort) && mbar_wait(&full_b[sw], (j / SW) & 1, abort);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA + sx * kABytes);
        const uint32_t b0 = smem_u32(sB + sw * kBBytes);
#pragma unroll
        for (int kk = 0; kk < BK / kMmaK; ++kk) {
          const uint64_t bd = sw128_desc(b0 + kk * kMmaK * 2);
#pragma unroll
          for (int mt = 0; mt < BM / kMmaM; ++mt) {
            const uint64_t ad = sw128_desc(a0 + mt * (kMmaM * 128) + kk * kMmaK * 2);
            umma(tmem + uint32_t(mt * kMmaN), ad, bd, (kt > kt0 || kk > 0) ? 1u : 0u);
          }
        }
        umma_commit(&empty_a[sx]);
        umma_commit(&empty_b[sw]);
      }
      umma_commit(tmem_full);      // always: the teardown waits on it before freeing TMEM
    }
  } else {
    // ------------------------------------------------------------ dequantise
    const int dw = warp - 2;
    const int cu = lane & 1;                 // 32-code unit within the 64-wide K step
    const int64_t G = K / g;
    if (rowwise) {                           // epilogue scale of each output column
      const int c = threadIdx.x - 64;
      if (c < BN) col_scale[c] = (n0 + c < N) ? __half2float(scales[(n0 + c) * G]) : 0.0f;
      asm volatile("bar.sync 1, %0;" ::"n"(32 * kDqWarps) : "memory");
    }
    // Per thread: rows 16 (dw + kDqWarps i) + lane / 2 of the tile
    // (i < kRowsPerThread), unit cu of every 64-wide K step.  w' = s (q - z) = fma(q 2^-30, s 2^30, -s z): the
    // code comes out of one AND as the subnormal float q 2^(p-149), one FMUL by
    // 2^(119-p) (exact) gives q 2^-30, and the FMA is exact (s q and s z have at
    // most 20 significant bits); the bf16 conversion is the only rounding.
    // Scale and zero of the next step are loaded one step ahead as raw fp16
    // bits; nothing reads those registers until that step (a use right after
    // the load would stall the warp for the whole load latency), so the loop
    // runs two steps per iteration with two register sets.
    const int r0 = 16 * dw + (lane >> 1);
    // This thread's two rows of the scale and zero arrays (row n >= N: none).
    const unsigned short* srow[kRowsPerThread];
    const unsigned short* zrow[kRowsPerThread];
#pragma unroll
    for (int i = 0; i < kRowsPerThread; ++i) {
      const int64_t n = n0 + r0 + 16 * kDqWarps * i;
      srow[i] = n < N ? reinterpret_cast<const unsigned short*>(scales) + n * G : nullptr;
      zrow[i] = n < N && zeros ? reinterpret_cast<const unsigned short*>(zeros) + n * G : nullptr;
    }
    auto load_raw = [&](int kt, uint16_t (&s2)[kRowsPerThread], uint16_t (&z2)[kRowsPerThread]) {
      const int k = kt * BK + 32 * cu;
      const uint32_t grp = units_per_group.div(uint32_t(k < K ? k >> 5 : 0));
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        s2[i] = 0;
        z2[i] = 0;
        if (kt < kt1 && srow[i] != nullptr && k < K) {
          s2[i] = rowwise ? uint16_t(0x3C00) : __ldg(srow[i] + grp);   // 0x3C00: fp16 1.0
          // no zeros array: the symmetric grid's zero 2^(b-1) as fp16 bits
          z2[i] = zrow[i] ? __ldg(zrow[i] + grp) : uint16_t((BITS - 1 + 15) << 10);
        }
      }
    };
    // With groups that are whole multiples of 128 the two K steps of a pair
    // (kt - kt0 even, and kt + 1) use one group, so a pair loads its scale and
    // zero once, during its second step, for the next pair.
    const bool pair_group = (g % (2 * BK)) == 0;
    bool ok = true;
    // One K step with the step's raw scale/zero (cs, cz); the next step's are
    // requested into (ns, nz).
    auto step = [&](int kt, const uint16_t (&cs2)[kRowsPerThread], const uint16_t (&cz2)[kRowsPerThread],
                    uint16_t (&ns2)[kRowsPerThread], uint16_t (&nz2)[kRowsPerThread], bool load_next) {
      if (load_next) load_raw(kt + 1, ns2, nz2);
      float A[kRowsPerThread], B[kRowsPerThread];
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const float sc = __half2float(__ushort_as_half(cs2[i]));
        A[i] = sc * 0x1p30f;
        B[i] = -sc * __half2float(__ushort_as_half(cz2[i]));
      }
      const int j = kt - kt0;
      const int c = j >> 1, cs = c % SC, s = j % SW;
      ok = mbar_wait(&full_c[cs], (c / SC) & 1, abort);
      if (ok && j >= SW) ok = mbar_wait(&empty_b[s], ((j / SW) - 1) & 1, abort);
      ok = __all_sync(0xffffffffu, ok);      // the warp leaves the loop together
      if (!ok) return;
      const uint8_t* ctile = sC + cs * Cfg::kCBytes;
      uint8_t* btile = sB + s * kBBytes;
      const int ucode = (kt & 1) * 2 + cu;   // unit index within the 128-code stage
#pragma unroll
      for (int i = 0; i < kRowsPerThread; ++i) {
        const int r = r0 + 16 * kDqWarps * i;
        uint32_t w[BITS];
        lds_unit<BITS>(ctile + r * (CK * BITS / 8) + ucode * (4 * BITS), w);
        uint32_t p[16];
        DqPairs<BITS, 0>::run(w, f32x2(A[i], A[i]), f32x2(B[i], B[i]), p);
        uint8_t* brow = btile + r * 128;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const int chunk = (cu * 4 + jj) ^ (r & 7);
          *reinterpret_cast<uint4*>(brow + chunk * 16) = make_uint4(p[4 * jj], p[4 * jj + 1], p[4 * jj + 2], p[4 * jj + 3]);
        }
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&full_b[s]);
        if ((j & 1) || kt == kt1 - 1) mbar_arrive(&empty_c[cs]);
      }
    };
    uint16_t s0r[kRowsPerThread], z0r[kRowsPerThread], s1r[kRowsPerThread], z1r[kRowsPerThread];
    load_raw(kt0, s0r, z0r);
    if (pair_group) {
      for (int kt = kt0; kt < kt1 && ok; kt += 4) {   // two pairs: register sets 0 then 1
        step(kt, s0r, z0r, s1r, z1r, false);
        if (ok && kt + 1 < kt1) step(kt + 1, s0r, z0r, s1r, z1r, true);
        if (ok && kt + 2 < kt1) step(kt + 2, s1r, z1r, s0r, z0r, false);
        if (ok && kt + 3 < kt1) step(kt + 3, s1r, z1r, s0r, z0r, true);
      }
    } else {
      for (int kt = kt0; kt < kt1 && ok; kt += 2) {
        step(kt, s0r, z0r, s1r, z1r, true);
        if (ok && kt + 1 < kt1) step(kt + 1, s1r, z1r, s0r, z0r, true);
      }
    }
    if (ok) ok = mbar_wait(tmem_full, 0, abort);
    ep_ok = __all_sync(0xffffffffu, ok);     // tcgen05.ld needs the whole warp
  }

  // ------------------------------------------------------------ epilogue
  // Accumulator mt (rows 128 mt .. 128 mt + 127 of the tile) is written out by
  // the 8 dequant warps: warp w reads TMEM lane quarter w % 4.  Without
  // split-K, warp w converts 128 of the 256 columns and stores them.  With
  // split-K every rank parks its partial tile in its own (now idle) shared
  // memory as [column / 4][row][4] floats; then rank r sums the 32-column
  // blocks b = r, r + ks, ... over all ranks (in rank order, through
  // distributed shared memory) and stores them, so the reduction is spread
  // over the cluster.  Every thread takes part in the cluster barriers.
  const bool dq = warp >= 2;
  const int q = warp & 3;                    // TMEM lane quarter this warp may access
  const int ch = (warp - 2) >> 2;            // column group (kColGroups of them)
  float4* part = reinterpret_cast<float4*>(sA);
  const bool vec = (N % 8) == 0;
  // bf16 of 32 columns of row m from column n, scaled per column for per-row grids
  auto store32 = [&](int64_t m, int col0, uint32_t (&r)[32]) {
    if (rowwise) {
#pragma unroll
      for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * col_scale[col0 + j]);
    }
    const int64_t n = n0 + col0;
    if (m < M && n < N) {
      __nv_bfloat16* dst = y + m * N + n;
      if (vec && n + 32 <= N) {
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 o;
          o.x = bf162_bits(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
          o.y = bf162_bits(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
          o.z = bf162_bits(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
          o.w = bf162_bits(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
          reinterpret_cast<uint4*>(dst)[v] = o;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (n + j < N) dst[j] = __float2bfloat16_rn(__uint_as_float(r[j]));
      }
    }
  };
  for (int mt = 0; mt < BM / kMmaM; ++mt) {
    const int row = 32 * q + lane;           // row within accumulator mt
    const int64_t m = m0 + mt * kMmaM + row;
    const uint32_t tbase = tmem + (uint32_t(32 * q) << 16) + uint32_t(mt * kMmaN);
    if (ks == 1) {
      if (dq && ep_ok) {
        tc_fence_after();
        for (int cb = 0; cb < 8 / kColGroups; ++cb) {
          const int col0 = (256 / kColGroups) * ch + 32 * cb;
          uint32_t r[32];
          tmem_ld32(tbase + uint32_t(col0), r);
          store32(m, col0, r);
        }
      }
      continue;
    }
    if (dq && ep_ok) {
      tc_fence_after();
      for (int cb = 0; cb < 8 / kColGroups; ++cb) {
        const int col0 = (256 / kColGroups) * ch + 32 * cb;
        uint32_t r[32];
        tmem_ld32(tbase + uint32_t(col0), r);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          part[((col0 >> 2) + v) * 128 + row] =
              make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                          __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
      }
    }
    cluster_sync();
    if (dq) {
      for (int blk = kr + ks * ch; blk < kMmaN / 32; blk += kColGroups * ks) {
        const int col0 = 32 * blk;
        float4 acc[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) acc[v] = ld_peer_f4(&part[((col0 >> 2) + v) * 128 + row], 0);
        for (int pr = 1; pr < ks; ++pr) {
          float4 pv[8];
#pragma unroll
          for (int v = 0; v < 8; ++v) pv[v] = ld_peer_f4(&part[((col0 >> 2) + v) * 128 + row], pr);
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            acc[v].x += pv[v].x;
            acc[v].y += pv[v].y;
            acc[v].z += pv[v].z;
            acc[v].w += pv[v].w;
          }
        }
        uint32_t r[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          r[4 * v] = __float_as_uint(acc[v].x);
          r[4 * v + 1] = __float_as_uint(acc[v].y);
          r[4 * v + 2] = __float_as_uint(acc[v].z);
          r[4 * v + 3] = __float_as_uint(acc[v].w);
        }
        store32(m, col0, r);
      }
    }
    cluster_sync();                          // peers keep their partials until read
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (*abort) {
      if (lane == 0) mbar_drain(tmem_full, 0);   // MMAs issued must finish before TMEM is freed
      __syncwarp();
    }
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
  // Such a second launch ends only after the first has (a no-op otherwise),
  // so work queued behind it on the stream sees every tile of y.
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ------------------------------------------------------------------ host
constexpr double kWaveStages = 5.0;    // prologue + epilogue of one wave, in code stages
#ifndef WQ_GEMM_SPLIT_STAGES
#define WQ_GEMM_SPLIT_STAGES 1.5
#endif
constexpr double kSplitStages = WQ_GEMM_SPLIT_STAGES;   // partial-tile exchange per extra split

// Clusters of c CTAs (one per SM, `smem` bytes each) resident at once; cached
// per device and cluster size.  0 if the query fails.
template <int BITS>
int cluster_slots(int dev, int c, uint32_t smem) {
  static std::atomic<int> cache[64][WQ_GEMM_MAX_SPLIT + 1];   // 0 unknown, -1 query failed
  const int ci = c;
  if (dev < 0 || dev >= 64 || ci < 1 || ci > WQ_GEMM_MAX_SPLIT) return 0;
  const int known = cache[dev][ci].load(std::memory_order_relaxed);
  if (known != 0) return known > 0 ? known : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, unsigned(c));
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = unsigned(c);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<BITS>, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    cache[dev][ci].store(-1, std::memory_order_relaxed);
    return 0;
  }
  cache[dev][ci].store(n, std::memory_order_relaxed);
  return n;
}

template <int BITS>
cudaError_t launch_bits(const __nv_bfloat16* x, int64_t M, int64_t N, int64_t K,
                        const uint32_t* codes, const __half* scales, const __half* zeros,
                        int64_t g, __nv_bfloat16* y, cudaStream_t st) {
  alignas(64) CUtensorMap tx, tc;
  if (!make_tensor_map_2d(&tx, TmaType::kBF16, x, uint64_t(K), uint64_t(M), uint64_t(K) * 2, BK, BM,
                          128) ||
      !make_tensor_map_2d(&tc, TmaType::kU32, codes, uint64_t(K * BITS / 32), uint64_t(N),
                          uint64_t(K * BITS / 8), CK * BITS / 32, BN, 0))
    return cudaErrorInvalidValue;
  constexpr uint32_t smem = TcCfg<BITS>::kSmem;
  // per device, set once; concurrent first calls repeat an idempotent call
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BITS>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  // Split K over a cluster when the output tiles alone fill the SMs badly.
  // Cost model in units of one 128-wide code stage: every wave of clusters
  // takes its share of K plus a fixed prologue/epilogue and a reduction cost
  // per extra split; the cluster slots per wave come from the occupancy API
  // (clusters of c CTAs of this size do not always pack the SMs fully).
  // Besides one launch for all tiles, the model weighs two: the whole waves
  // of tiles without a split, then the few tiles left over split over
  // clusters (so that a last, nearly empty wave of whole tiles does not set
  // the time).
  const int ntn = int((N + BN - 1) / BN);
  const int tiles = ntn * int((M + BM - 1) / BM);
  const int64_t kc = K / CK;
  auto cost = [&](int ntiles, int c) -> double {
    const int slots = cluster_slots<BITS>(dev, c, smem);
    if (slots <= 0) return 1e300;
    const double waves = double((ntiles + slots - 1) / slots);
    return waves * (double(kc) / c + kWaveStages + kSplitStages * (c - 1));
  };
  auto best_split = [&](int ntiles, double* t_out) -> int {
    int bc = 1;
    double bt = 1e300;
    for (int c = 1; c <= WQ_GEMM_MAX_SPLIT; ++c) {
      if (c > 1 && kc / c < WQ_GEMM_MIN_STAGES) break;
      const double t = cost(ntiles, c);
      if (t < bt - 1e-9) {
        bt = t;
        bc = c;
      }
    }
    *t_out = bt;
    return bc;
  };
  double t_one = 0.0;
  const int ks_one = best_split(tiles, &t_one);
  const int slots1 = cluster_slots<BITS>(dev, 1, smem);
  int whole = 0, ks_rest = 1;
  if (slots1 > 0 && tiles > slots1 && tiles % slots1 != 0) {
    const int w = (tiles / slots1) * slots1;
    double t_rest = 0.0;
    const int c = best_split(tiles - w, &t_rest);
    if (double(w / slots1) * (double(kc) + kWaveStages) + t_rest < t_one - 1e-9) {
      whole = w;
      ks_rest = c;
    }
  }
  // The second of two launches is a programmatic dependent of the first: it
  // reads only x and the codes and writes other tiles of y, so its CTAs may
  // start on SMs that the first launch's CTAs leave, and its prologue and
  // launch latency overlap the first launch's last tiles.
  auto launch = [&](int tile0, int count, int ks, bool overlap) -> cudaError_t {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(count), 1, unsigned(ks));
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = unsigned(ks);
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = overlap ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BITS>, tx, tc, scales, zeros, M, N, K, g,
                              FastDiv(uint32_t(g / 32)), y, tile0, ntn);
  };
  if (whole == 0) return launch(0, tiles, ks_one, false);
  cudaError_t e = launch(0, whole, 1, false);
  if (e == cudaSuccess) e = launch(whole, tiles - whole, ks_rest, true);
  return e;
}

}  // namespace

bool gemm_tc_supported(int64_t K, int bits) {
  (void)bits;
  return K % CK == 0;
}

cudaError_t launch_gemm_tc(const __nv_bfloat16* x, int64_t M, int64_t N, int64_t K,
                           const uint32_t* codes, const __half* scales, const __half* zeros,
                           int bits, int64_t g, __nv_bfloat16* y, cudaStream_t st) {
  switch (bits) {
    case 2: return launch_bits<2>(x, M, N, K, codes, scales, zeros, g, y, st);
    case 3: return launch_bits<3>(x, M, N, K, codes, scales, zeros, g, y, st);
    case 4: return launch_bits<4>(x, M, N, K, codes, scales, zeros, g, y, st);
    default: return launch_bits<8>(x, M, N, K, codes, scales, zeros, g, y, st);
  }
}

bool gemm_tc_read_and_clear_timeout(cudaError_t* err) {
  unsigned int v = 0;
  const unsigned int zero = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&v, g_timeout_flag, sizeof(v));
  if (e == cudaSuccess && v) e = cudaMemcpyToSymbol(g_timeout_flag, &zero, sizeof(zero));
  *err = e;
  return v != 0;
}

}  // namespace wq
