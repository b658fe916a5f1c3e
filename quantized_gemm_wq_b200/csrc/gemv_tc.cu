// gemv_tc.cu -- decode y = x . W'^T for 2 to 16 batch rows on the Blackwell
// tensor cores, with the weights dequantised on the fly ("[Feature Request]
// 4bit and 2bit and 1bit quantization support": the packed weights stay in
// memory and become floats on the GPU; "Platform For AI: BladeLLM model
// quantization", "Background information > Solutions").
//
// The arithmetic: for one row and one quantisation group, y gets
// s * (sum_k q_k x_k - z * sum_k x_k) (OPTQ's asymmetric min-max grid,
// w' = s (q - z)).  The sum of q_k x_k is a dot product of small integers
// with activations, which the tensor cores do exactly if q_k reaches them as
// a bf16: a code q in bits [b, b + c) of a 16-bit half with all other bits
// clear is the bf16 bit pattern of q 2^(b-133) whenever b + c <= 8 (patterns
// below 0x100 are the subnormals and the first normal binade, where the
// encoding is linear).  So one AND of a 32-bit window of a row's code stream
// yields two weights for the MMA; unpack_tables.h lists the 64 ANDs per
// 128-code segment and the activation slot each value meets, pre-multiplied
// by 2^(64 - b), so every product is q x 2^-69 exactly.
//
// One CTA owns 128 weight rows (the 128 lanes of tensor memory) and a run of
// J 128-code segments of K; a cluster of CTAs along grid.y splits K and adds
// its partial sums through distributed shared memory.  Warps:
//   0      TMA producer: per segment the 128-row box of packed codes, swizzled
//          so that one row per thread reads without bank conflicts;
//   1      owns tensor memory; one elected lane issues
//          tcgen05.mma.cta_group::1.kind::f16, M = 128 rows, N = 16 batch
//          columns, K = 16, A (the bf16 code patterns) from tensor memory, B
//          (activations) from shared memory, fp32 accumulators per
//          accumulation unit (AU: 32, 64 or 128 codes, inside one group);
//   2..9   first, together: the CTA's scales and zeros into shared memory
//          (cp.async), the B operand of all J segments (slot order and
//          2^(64 - b) factors of the unpack table) and 2^-69 sum(x) per AU;
//          then one warp per tensor-memory lane quarter and segment parity:
//          each thread unpacks its row's 128 codes into 64 bf16 pairs and
//          stores them into tensor memory, and two of its segments later
//          reads the AU accumulators D = 2^-69 sum q x of that segment and adds
//          s 2^69 (D - z 2^-69 sum x).
// The B operand is stored densely: per 8-slot chunk the MP batch rows of 16
// bytes follow each other, and the descriptor steps MP * 16 bytes per chunk;
// for MP < 8 the MMA's rows MP..15 then read neighbouring chunks, which only
// feeds accumulator columns that are never read.  (One batch row runs the
// CUDA-core GEMV in gemv_tma.cu, whose shorter pipeline is faster there.)
// Every wait is bounded in time (1 s): an expired wait raises a device flag,
// read by wq_last_device_error, and the CTA drains and leaves.
#include <cuda.h>

#include <atomic>
#include <algorithm>

#include "tc_unpack.cuh"
#include "wq_internal.cuh"
#include "wq_ptx.cuh"

namespace wq {

// Set by a kernel that gave up a bounded wait; read and cleared by the host.
__device__ unsigned int g_gemv_tc_timeout;

namespace {

using namespace ptx;
using namespace tcu;

constexpr int kRows = 128;                  // weight rows per CTA (tensor-memory lanes)
constexpr int kSeg = 128;                   // codes per segment
constexpr int kDqWarps = 8;
constexpr int kThreads = 32 * (2 + kDqWarps);
constexpr uint32_t kTmemCols = 256;         // two CTAs per SM share the 512 columns
constexpr int kMaxRA = 3, kMaxRD = 4;
constexpr int kMmaN = 16;
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(kMmaN >> 3) << 17) |
                            (uint32_t(kRows >> 4) << 24);   // bf16 x bf16 -> fp32, K-major
constexpr float kTwo69 = 590295810358705651712.0f;          // 2^69
constexpr float kTwoM69 = 1.6940658945086007e-21f;          // 2^-69

constexpr int kMaxGroups = 32;              // quantisation groups a CTA's K-run may touch
constexpr int kMaxSplit = 8;                // CTAs of a split-K cluster
constexpr int kSPitch = 19;                 // words per row of staged scales (odd: no bank conflicts)
constexpr uint32_t kSmemBudget = 112 * 1024;

template <int BITS, int MP>
struct TcvM {
  static constexpr uint32_t kChunk = uint32_t(MP) * 16;     // B bytes per 8-slot chunk
  static constexpr uint32_t kSegB = 16 * kChunk;            // B bytes per segment
  // Segments a CTA may own (its B operand stays resident); 8-bit code boxes
  // are twice as large, so they leave less room.
  static constexpr int kMaxJ = MP == 4 ? (BITS == 8 ? 16 : 32) : (BITS == 8 ? 4 : 11);
  static constexpr uint32_t kBBytes = kMaxJ * kSegB + 256;  // + what rows past MP may read
  static constexpr uint32_t kXsBytes = kMaxJ * 4 * MP * 4;  // 2^-69 sum(x) per segment, AU, row
};

template <int BITS, int MP>
struct TcvCfg {
  static constexpr int kWords = 4 * BITS;                   // code words of a row per segment
  static constexpr uint32_t kBox = uint32_t(kRows) * kWords * 4;
  // Box swizzle: the box row is 16 * BITS bytes; 32/64/128-byte swizzles for
  // 2/4/8 bits, none for 3 bits (48-byte rows already spread over all banks).
  static constexpr int kSwzBytes = BITS == 2 ? 32 : BITS == 4 ? 64 : BITS == 8 ? 128 : 0;
  static constexpr uint32_t kSwzMask = BITS == 2 ? 1u : BITS == 4 ? 3u : BITS == 8 ? 7u : 0u;
  static constexpr uint32_t kOther = TcvM<BITS, MP>::kBBytes + TcvM<BITS, MP>::kXsBytes + kRows * MP * 4 +
                                     2 * kRows * kSPitch * 4 + 1024 /* barriers */ + 1024 /* align */;
  static constexpr uint32_t kRingMax = kSmemBudget - kOther < 65536u ? kSmemBudget - kOther : 65536u;
  static constexpr int RC = int(kRingMax / kBox);          // codes ring
  static_assert(RC >= 4, "codes ring");
};

template <int BITS, int MP>
struct TcvSmem {
  static constexpr uint32_t kC = 0;
  static constexpr uint32_t kB = kC + TcvCfg<BITS, MP>::RC * TcvCfg<BITS, MP>::kBox;
  static constexpr uint32_t kXs = kB + TcvM<BITS, MP>::kBBytes;
  static constexpr uint32_t kPart = kXs + TcvM<BITS, MP>::kXsBytes;
  static constexpr uint32_t kScale = kPart + kRows * MP * 4;      // [2][128][kSPitch] words
  static constexpr uint32_t kBars = kScale + 2 * kRows * kSPitch * 4;
  static constexpr int kNumBars = 2 * TcvCfg<BITS, MP>::RC + 2 * kMaxRA + 2 * kMaxRD + 1;
  static constexpr uint32_t kMisc = kBars + kNumBars * 8;
  static constexpr uint32_t kTotal = kMisc + 16 + 1024;     // + alignment slack
};
static_assert(TcvSmem<2, 16>::kTotal <= 113 * 1024, "two CTAs per SM");
static_assert(TcvSmem<3, 16>::kTotal <= 113 * 1024, "two CTAs per SM");
static_assert(TcvSmem<4, 16>::kTotal <= 113 * 1024, "two CTAs per SM");
static_assert(TcvSmem<8, 16>::kTotal <= 113 * 1024, "two CTAs per SM");
static_assert(TcvSmem<8, 4>::kTotal <= 113 * 1024, "two CTAs per SM");

template <int BITS, int MP>
__global__ void __launch_bounds__(kThreads, 2)
gemv_tc_kernel(const __grid_constant__ CUtensorMap tm_c, const __nv_bfloat16* __restrict__ x,
               const __half* __restrict__ scales, const __half* __restrict__ zeros, int M,
               int64_t N, int64_t K, int64_t g, int64_t G, FastDiv units_per_group, int nau,
               __nv_bfloat16* __restrict__ y) {
  using C = TcvCfg<BITS, MP>;
  using MC = TcvM<BITS, MP>;
  using L = TcvSmem<BITS, MP>;
  constexpr int RC = C::RC;
  unsigned int* const flag = &g_gemv_tc_timeout;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sC = base + L::kC;
  uint8_t* sB = base + L::kB;
  float* xsum = reinterpret_cast<float*>(base + L::kXs);       // [J][4 AU][MP]
  float* part = reinterpret_cast<float*>(base + L::kPart);     // [128][MP]
  uint32_t* sstage = reinterpret_cast<uint32_t*>(base + L::kScale);
  uint64_t* c_full = reinterpret_cast<uint64_t*>(base + L::kBars);
  uint64_t* c_empty = c_full + RC;
  uint64_t* a_full = c_empty + RC;
  uint64_t* a_empty = a_full + kMaxRA;
  uint64_t* d_full = a_empty + kMaxRA;
  uint64_t* d_empty = d_full + kMaxRD;
  uint64_t* mma_done = d_empty + kMaxRD;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L::kMisc);
  volatile uint32_t* abort = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n0 = int64_t(blockIdx.x) * kRows;
  const int nseg = int(K / kSeg);
  const int ks = int(gridDim.y), kr = int(blockIdx.y);
  const int s0 = int(int64_t(nseg) * kr / ks);
  const int J = int(int64_t(nseg) * (kr + 1) / ks) - s0;     // segments of this CTA (<= kMaxJ)
  const int RA = nau == 4 ? 2 : 3;                            // A ring (64 columns each)
  const int RD = (int(kTmemCols) - 64 * RA) / (16 * nau);     // D slots (segments): 4, 2, 2
  const int lag = RD >= 4 ? 4 : 2;                            // epilogue lag, in segments
  const int aus = 8 / nau;                                    // MMAs per AU

  if (threadIdx.x == 0) {
    for (int i = 0; i < RC; ++i) {
      mbar_init(&c_full[i], 1);
      mbar_init(&c_empty[i], 4);
    }
    for (int i = 0; i < kMaxRA; ++i) {
      mbar_init(&a_full[i], 4);
      mbar_init(&a_empty[i], 1);
    }
    for (int i = 0; i < kMaxRD; ++i) {
      mbar_init(&d_full[i], 1);
      mbar_init(&d_empty[i], 4);
    }
    mbar_init(mma_done, 1);
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
  const uint32_t dcol0 = uint32_t(64 * RA);

  float acc[MP];
#pragma unroll
  for (int m = 0; m < MP; ++m) acc[m] = 0.0f;
  const int dw = warp - 2, q = warp & 3, h = dw >> 2;
  const int row = 32 * q + lane;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int ic = 0;
      bool ok = true;
      for (int j = 0; j < J && ok; ++j) {
        const int cs = j % RC;
        if (j >= RC) ok = mbar_wait(&c_empty[cs], ((j / RC) - 1) & 1, abort, flag);
        if (!ok) break;
        mbar_expect_tx(&c_full[cs], C::kBox);
        tma_load_2d(sC + cs * C::kBox, &tm_c, &c_full[cs], (s0 + j) * C::kWords, int(n0));
        ++ic;
      }
      if (!ok)   // copies in flight must land before shared memory goes away
        for (int j = (ic > RC ? ic - RC : 0); j < ic; ++j) mbar_drain(&c_full[j % RC], (j / RC) & 1, flag);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    const uint32_t bbase = smem_u32(sB);
    Ring ra, rd;
    bool ok = true;
    for (int j = 0; j < J; ++j) {
      ok = mbar_wait(&a_full[ra.slot], ra.phase, abort, flag);   // A of segment j in TMEM
      if (ok && j >= RD) ok = mbar_wait(&d_empty[rd.slot], rd.phase ^ 1u, abort, flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t acol = tmem + uint32_t(64 * ra.slot);
      const uint32_t bseg = bbase + uint32_t(j) * MC::kSegB;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const int au = kk / aus;
        const uint32_t d = tmem + dcol0 + uint32_t((rd.slot * nau + au) * 16);
        const uint64_t bd = desc_noswz(bseg + uint32_t(kk) * 2 * MC::kChunk, MC::kChunk, MP > 8 ? 128 : 0);
        mma_elect(d, acol + uint32_t(8 * kk), bd, kIdesc, (kk % aus) != 0 ? 1u : 0u);
      }
      commit_elect(&a_empty[ra.slot]);
      commit_elect(&d_full[rd.slot]);
      ra.advance(1, RA);
      rd.advance(1, RD);
    }
    commit_elect(mma_done);     // the teardown waits on it before freeing tensor memory
  } else {
    // ------------------------------------------------------------ dequant warps
    const int64_t n = n0 + row;
    const int td = threadIdx.x - 64;                 // 0..255 over the 8 warps
    const uint32_t lanes = tmem + (uint32_t(32 * q) << 16);
    const int auc = 128 / nau;                       // codes per AU
    // (1) this row's scales and zeros for the CTA's groups [gA, gB] into
    // shared memory: 4-byte asynchronous copies of aligned half pairs (parity
    // 0 copies the scales, parity 1 the zeros).  off: where group gA sits.
    const int gA = int(int64_t(s0) * kSeg / g);
    const int gB = int((int64_t(s0 + J) * kSeg - 1) / g);
    const int64_t e0 = n * G + gA;
    const int off = int(e0 & 1);
    {
      const __half* src = h ? zeros : scales;
      uint32_t* dst = sstage + (h * kRows + row) * kSPitch;
      if (n < N && src == nullptr) {
        // no zeros array (symmetric grid): every zero is 2^(b-1)
        constexpr uint32_t zh = uint32_t(BITS - 1 + 15) << 10;
        int wi = 0;
        for (int64_t a = e0 - off; a <= n * G + gB; a += 2, ++wi) dst[wi] = zh | (zh << 16);
      } else if (n < N) {
        const int64_t total = N * G;
        int wi = 0;
        for (int64_t a = e0 - off; a <= n * G + gB; a += 2, ++wi) {
          if (a + 1 < total) {
            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst + wi)),
                         "l"(src + a)
                         : "memory");
          } else {          // the array's last element, alone in its pair
            dst[wi] = uint32_t(__half_as_ushort(src[a]));
          }
        }
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    // (2) the B operand of all J segments: slot pair t of segment j, batch
    // row m, at j * kSegB + (t / 4) * kChunk + m * 16 + (t % 4) * 4.  Thread
    // td keeps one pair t = td % 64 and walks (j, m); loads go out 8 at a time.
    {
      const int t = td & 63;
      int olo, ohi;
      float oflo, ofhi;
      OpPick<BITS, 0>::run(t, olo, ohi, oflo, ofhi);
      const __nv_bfloat16* xc = x + int64_t(s0) * kSeg;
      uint8_t* bcol = sB + (t >> 2) * MC::kChunk + (t & 3) * 4;
      const int JM = J * MP;
      for (int jm0 = td >> 6; jm0 < JM; jm0 += 4 * 8) {
        float a[8], b[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int jm = jm0 + 4 * u, j = jm / MP, m = jm % MP;
          a[u] = 0.0f;
          b[u] = 0.0f;
          if (jm < JM && m < M) {
            const __nv_bfloat16* xr = xc + int64_t(m) * K + j * kSeg;
            a[u] = __bfloat162float(xr[olo]);
            b[u] = __bfloat162float(xr[ohi]);
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int jm = jm0 + 4 * u, j = jm / MP, m = jm % MP;
          if (jm < JM)       // exact: power-of-two multiples of bf16 values
            *reinterpret_cast<uint32_t*>(bcol + j * MC::kSegB + m * 16) = bf162_bits(a[u] * oflo, b[u] * ofhi);
        }
      }
      for (int i = td; i < 256 / 16; i += 32 * kDqWarps)   // what rows past MP may read
        reinterpret_cast<uint4*>(sB + J * MC::kSegB)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    // (3) 2^-69 sum(x) per segment, AU and batch row: 8 threads per item, each
    // summing auc / 8 activations (loaded 4 at a time), then a shuffle tree.
    {
      const int items = J * nau * MP;
      for (int base_it = 0; base_it < items; base_it += (32 * kDqWarps) / 8) {
        const int it = base_it + td / 8, part8 = td & 7;
        float sx = 0.0f;
        if (it < items) {
          const int m = it % MP, au = (it / MP) % nau, j = it / (MP * nau);
          if (m < M) {
            const uint2* xr = reinterpret_cast<const uint2*>(
                x + int64_t(m) * K + int64_t(s0 + j) * kSeg + au * auc + part8 * (auc / 8));
            uint2 v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = (e < auc / 32) ? xr[e] : make_uint2(0u, 0u);
#pragma unroll
            for (int e = 0; e < 4; ++e)
              sx += (__uint_as_float(v[e].x << 16) + __uint_as_float(v[e].x & 0xFFFF0000u)) +
                    (__uint_as_float(v[e].y << 16) + __uint_as_float(v[e].y & 0xFFFF0000u));
          }
        }
        sx += __shfl_xor_sync(0xffffffffu, sx, 1);
        sx += __shfl_xor_sync(0xffffffffu, sx, 2);
        sx += __shfl_xor_sync(0xffffffffu, sx, 4);
        if (it < items && part8 == 0) xsum[it] = sx * kTwoM69;
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    fence_async_smem();                              // B: generic stores -> the MMA's reads
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kDqWarps) : "memory");

    const __half* hs = reinterpret_cast<const __half*>(sstage + row * kSPitch);
    const __half* hz = reinterpret_cast<const __half*>(sstage + (kRows + row) * kSPitch);
    auto epilogue = [&](int j) -> bool {
      const int sd = j % RD;
      bool ok = mbar_wait(&d_full[sd], (j / RD) & 1, abort, flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) return false;
      tc_fence_after();
      const float* X = xsum + j * nau * MP;
#pragma unroll
      for (int au = 0; au < 4; ++au) {
        if (au < nau) {
          float ps = 0.0f, pz = 0.0f;
          if (n < N) {
            const uint32_t unit = uint32_t(((s0 + j) * kSeg + au * auc) >> 5);
            const int i = int(units_per_group.div(unit)) - gA + off;
            ps = __half2float(hs[i]) * kTwo69;
            pz = __half2float(hz[i]);
          }
          float v[MP];
          tmem_ld<MP>(lanes + dcol0 + uint32_t((sd * nau + au) * 16), v);
#pragma unroll
          for (int m = 0; m < MP; ++m) acc[m] = fmaf(ps, fmaf(-pz, X[au * MP + m], v[m]), acc[m]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[sd]);
      return true;
    };
    bool ok = true;
    int next_ep = h;                                 // next own segment awaiting its epilogue
    for (int j = h; j < J; j += 2) {
      const int cs = j % RC, sa = j % RA;
      ok = mbar_wait(&c_full[cs], (j / RC) & 1, abort, flag);
      if (ok && j >= RA) ok = mbar_wait(&a_empty[sa], ((j / RA) - 1) & 1, abort, flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      uint32_t w[4 * BITS];
      {
        const uint8_t* box = sC + cs * C::kBox;
#pragma unroll
        for (int c = 0; c < BITS; ++c) {
          const uint32_t lin = uint32_t(row * 16 * BITS + 16 * c);
          const uint32_t phys = lin ^ (((lin >> 7) & C::kSwzMask) << 4);
          uint4 v;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(smem_u32(box) + phys));
          w[4 * c] = v.x;
          w[4 * c + 1] = v.y;
          w[4 * c + 2] = v.z;
          w[4 * c + 3] = v.w;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&c_empty[cs]);     // the codes are in registers
      {
        uint32_t o[32];
        UnpackRun<BITS, 0, 0>::run(w, o);
        tmem_st32(lanes + uint32_t(64 * sa), o);
        UnpackRun<BITS, 32, 32>::run(w, o);
        tmem_st32(lanes + uint32_t(64 * sa + 32), o);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[sa]);
      if (j - next_ep >= lag) {                      // the epilogue `lag` segments back
        ok = epilogue(next_ep);
        if (!ok) break;
        next_ep += 2;
      }
    }
    for (; ok && next_ep < J; next_ep += 2) ok = epilogue(next_ep);
  }

  // ------------------------------------------------------------ reduction
  // The two parities' partial sums meet in `part`, then the cluster's CTAs
  // add theirs: rank kr writes rows r with r % ks == kr.
  if (warp >= 2 && h == 1) {
#pragma unroll
    for (int m = 0; m < MP; ++m) part[row * MP + m] = acc[m];
  }
  __syncthreads();
  if (warp >= 2 && h == 0) {
#pragma unroll
    for (int m = 0; m < MP; ++m) part[row * MP + m] += acc[m];
  }
  __syncthreads();
  if (ks > 1) cluster_sync();
  for (int f = threadIdx.x; f < kRows * MP; f += kThreads) {
    const int rr = f / MP, m = f % MP;
    if (rr % ks != kr || m >= M || n0 + rr >= N) continue;
    float v[kMaxSplit];
#pragma unroll
    for (int p = 0; p < kMaxSplit; ++p)        // all peer loads in flight at once
      v[p] = (p >= ks) ? 0.0f : (p == kr) ? part[f] : ld_peer_f32(&part[f], p);
    float sum = 0.0f;
#pragma unroll
    for (int p = 0; p < kMaxSplit; ++p) sum += v[p];
    y[int64_t(m) * N + n0 + rr] = __float2bfloat16_rn(sum);
  }
  if (ks > 1) cluster_sync();          // peers keep their partials until read

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) mbar_drain(mma_done, 0, flag);     // issued MMAs finish before TMEM is freed
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// ------------------------------------------------------------------ host
constexpr double kFixedSegs = 3.0;     // prologue, pipeline fill and epilogue, in segments
constexpr double kSplitSegs = 1.0;     // cluster reduction

template <int BITS, int MP>
int cluster_slots(int dev, int c, uint32_t smem) {
  static std::atomic<int> cache[64][kMaxSplit + 1];   // 0 unknown, -1 query failed
  if (dev < 0 || dev >= 64 || c < 1 || c > kMaxSplit) return 0;
  const int known = cache[dev][c].load(std::memory_order_relaxed);
  if (known != 0) return known > 0 ? known : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, unsigned(c), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = unsigned(c);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemv_tc_kernel<BITS, MP>, &cfg) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    cache[dev][c].store(-1, std::memory_order_relaxed);
    return 0;
  }
  cache[dev][c].store(n, std::memory_order_relaxed);
  return n;
}

int gcd_int(int a, int b) { return b == 0 ? a : gcd_int(b, a % b); }

template <int BITS>
int max_segs_bits(int M) {
  return M <= 4 ? TcvM<BITS, 4>::kMaxJ : TcvM<BITS, 16>::kMaxJ;
}
int max_segs_for(int M, int bits) {
  switch (bits) {
    case 2: return max_segs_bits<2>(M);
    case 3: return max_segs_bits<3>(M);
    case 4: return max_segs_bits<4>(M);
    default: return max_segs_bits<8>(M);
  }
}

// Largest number of quantisation groups one CTA's run of segments touches
// when nseg segments are split over ks CTAs (the kernel stages them).
int group_span(int nseg, int ks, int64_t g) {
  int span = 0;
  for (int r = 0; r < ks; ++r) {
    const int64_t a = int64_t(nseg) * r / ks, b = int64_t(nseg) * (r + 1) / ks;
    const int64_t ga = a * kSeg / g, gb = (b * kSeg - 1) / g;
    span = std::max(span, int(gb - ga + 1));
  }
  return span;
}

template <int BITS, int MP>
cudaError_t launch_tc(const __nv_bfloat16* x, int M, int64_t N, int64_t K, const uint32_t* codes,
                      const __half* scales, const __half* zeros, int64_t g, __nv_bfloat16* y,
                      cudaStream_t st) {
  using C = TcvCfg<BITS, MP>;
  alignas(64) CUtensorMap tc;
  if (!make_tensor_map_2d(&tc, TmaType::kU32, codes, uint64_t(K * BITS / 32), uint64_t(N),
                          uint64_t(K * BITS / 8), uint32_t(C::kWords), kRows, C::kSwzBytes))
    return cudaErrorInvalidValue;
  constexpr uint32_t smem = TcvSmem<BITS, MP>::kTotal;
  // per device, set once; concurrent first calls repeat an idempotent call
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(gemv_tc_kernel<BITS, MP>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  const int nseg = int(K / kSeg);
  const int64_t tiles = (N + kRows - 1) / kRows;
  // Split K over a cluster: each wave of clusters takes its share of the
  // segments plus a fixed cost; cluster slots per wave from the occupancy API.
  int ks = 1;
  double best = 1e300;
  auto fits = [&](int c) {
    return group_span(nseg, c, g) <= kMaxGroups && (nseg + c - 1) / c <= TcvM<BITS, MP>::kMaxJ;
  };
  for (int c = 1; c <= kMaxSplit && c <= nseg; ++c) {
    if (!fits(c)) continue;
    const int slots = cluster_slots<BITS, MP>(dev, c, smem);
    if (slots <= 0) break;
    const double waves = double((tiles + slots - 1) / slots);
    const double t = waves * (double((nseg + c - 1) / c) + kFixedSegs) + (c > 1 ? kSplitSegs : 0.0);
    if (t < best - 1e-9) {
      best = t;
      ks = c;
    }
  }
#ifdef WQ_GEMV_TC_SPLIT
  for (int c = std::min(nseg, WQ_GEMV_TC_SPLIT); c >= 1; --c)
    if (fits(c)) { ks = c; break; }
#endif
  if (!fits(ks)) return cudaErrorInvalidValue;
  const int au = 32 * gcd_int(int(g / 32), 4);
  const int nau = kSeg / au;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(tiles), unsigned(ks), 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = unsigned(ks);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemv_tc_kernel<BITS, MP>, tc, x, scales, zeros, M, N, K, g,
                            K / g, FastDiv(uint32_t(g / 32)), nau, y);
}

template <int BITS>
cudaError_t launch_mp(const __nv_bfloat16* x, int M, int64_t N, int64_t K, const uint32_t* codes,
                      const __half* s, const __half* z, int64_t g, __nv_bfloat16* y, cudaStream_t st) {
  if (M <= 4) return launch_tc<BITS, 4>(x, M, N, K, codes, s, z, g, y, st);
  return launch_tc<BITS, 16>(x, M, N, K, codes, s, z, g, y, st);
}

}  // namespace

bool gemv_tc_supported(int M, int64_t K, int bits, int64_t g) {
  if (M < 2 || M > 16 || K % kSeg != 0 || g % 32 != 0) return false;
  if (bits == 3 && g % kSeg != 0) return false;   // the 3-bit unpack table spans whole segments
  const int nseg = int(K / kSeg);
  const int ks = std::min(nseg, kMaxSplit);
  return group_span(nseg, ks, g) <= kMaxGroups && (nseg + ks - 1) / ks <= max_segs_for(M, bits);
}

cudaError_t launch_gemv_tc(const __nv_bfloat16* x, int M, int64_t N, int64_t K,
                           const uint32_t* codes, const __half* scales, const __half* zeros,
                           int bits, int64_t g, __nv_bfloat16* y, cudaStream_t st) {
  switch (bits) {
    case 2: return launch_mp<2>(x, M, N, K, codes, scales, zeros, g, y, st);
    case 3: return launch_mp<3>(x, M, N, K, codes, scales, zeros, g, y, st);
    case 4: return launch_mp<4>(x, M, N, K, codes, scales, zeros, g, y, st);
    default: return launch_mp<8>(x, M, N, K, codes, scales, zeros, g, y, st);
  }
}

bool gemv_tc_read_and_clear_timeout(cudaError_t* err) {
  unsigned int v = 0;
  const unsigned int zero = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(&v, g_gemv_tc_timeout, sizeof(v));
  if (e == cudaSuccess && v) e = cudaMemcpyToSymbol(g_gemv_tc_timeout, &zero, sizeof(zero));
  *err = e;
  return v != 0;
}

}  // namespace wq
