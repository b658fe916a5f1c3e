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

#include <atomic>

#include "stage_smem.cuh"
#include "wq_internal.cuh"

namespace wq {
namespace {

using namespace stg;

constexpr int kScaleS = 64;

// The kernel is compiled for 2 resident CTAs per SM, and for 3 for grids that
// need fewer waves of 3 than of 2.
// Split-K heuristic: CTAs wanted in total, and K stages kept per CTA.
#ifndef WQ_GEMV_M1_TARGET_CTAS
#define WQ_GEMV_M1_TARGET_CTAS 444
#endif
#ifndef WQ_GEMV_M1_MIN_STAGES
#define WQ_GEMV_M1_MIN_STAGES 4
#endif
__device__ unsigned int g_gemv_tma_timeout;

// d[I % 4] += x'[I] * f_I for I = I0..31 (four independent chains).
template <int BITS, int I>
struct Dot {
  __device__ __forceinline__ static void run(const uint32_t (&w)[BITS], const float (&xp)[32],
                                             float (&d)[4]) {
    d[I & 3] = fmaf(xp[I], code_subnormal<BITS, I>(w), d[I & 3]);
    if constexpr (I + 1 < 32) Dot<BITS, I + 1>::run(w, xp, d);
  }
};
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  return bw::pipe_wait(bar, parity, &g_gemv_tma_timeout, nullptr);
}

template <int BITS>
struct M1Cfg {
  static constexpr int NW = 8;                       // consumer warps (4 units of a stage each)
  static constexpr int D = 3;                        // ring stages
  static constexpr int STAGE_WORDS = 32 * BITS;      // 32 units of one row
  static constexpr int BOX_BYTES = 32 * 128;         // one TMA box: 32 rows x 128 bytes, swizzled
  static constexpr int STAGE_BYTES = BITS * BOX_BYTES;
  static constexpr int XRAW_BYTES = 1024 * 2;        // the stage's 1024 x values, bf16, as copied
  static constexpr int XU = 36;                      // floats per staged unit of x' (32 + bank pad)
  static constexpr int XS_BYTES = NW * 4 * XU * 4;   // per warp: x' of its 4 units
  // ring, raw x slots, x' buffers and barriers; the scale table follows
  static constexpr int FIXED = D * (STAGE_BYTES + XRAW_BYTES) + XS_BYTES + 2 * D * 8;
  static int smem(int gcap) { return FIXED + 32 * gcap * 8 + 1024; }
};

// One CTA: 32 output rows over its share of K.  Warp NW is the producer: one
// lane issues, per stage, the TMA copy of the 32-row x 32-unit box of codes and
// a bulk copy of the stage's 1024 x values (bf16) into a ring of D stages,
// both completing on the stage's "full" barrier.  Warps 0..NW-1 consume: warp
// w takes units 4w..4w+3 of every box, lane l rows lr, lr+8, lr+16, lr+24
// (lr = l % 8) of unit 4w + l / 8.  A stage is released when every consumer
// warp has arrived on its "empty" barrier.  The scales and zeros of the CTA's
// rows are read from global memory once, into a shared table of (s, z) pairs
// covering up to gcap groups, while the first codes are in flight; a CTA whose
// K range spans more groups reloads the table between stages.  The consumers
// therefore wait on nothing but the ring.
template <int BITS, int MINB>
__global__ void __launch_bounds__(32 * (M1Cfg<BITS>::NW + 1), MINB)
gemv_m1_tma_kernel(const __grid_constant__ CUtensorMap tm_codes, const __nv_bfloat16* __restrict__ x,
                   int64_t N, int64_t K, const __half* __restrict__ scales,
                   const __half* __restrict__ zeros, FastDiv units_per_group, int gcap,
                   __nv_bfloat16* __restrict__ y) {
  using Cfg = M1Cfg<BITS>;
  constexpr int NW = Cfg::NW, D = Cfg::D, XU = Cfg::XU;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ float red[NW][32];
  // the swizzle pattern repeats every 1024 bytes: align the ring to it
  uint8_t* smem = smem_raw + ((1024 - (saddr(smem_raw) & 1023)) & 1023);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t ring = saddr(smem);
  const uint32_t xraw0 = ring + D * Cfg::STAGE_BYTES;
  uint8_t* xs_base = smem + D * (Cfg::STAGE_BYTES + Cfg::XRAW_BYTES);
  const uint32_t full0 = saddr(xs_base + Cfg::XS_BYTES);
  const uint32_t empty0 = full0 + 8 * D;
  float2* tbl = reinterpret_cast<float2*>(xs_base + Cfg::XS_BYTES + 16 * D);

  const int64_t row0 = int64_t(blockIdx.x) * 32;
  const int64_t KU = K / 32;
  const int TT = int((KU + 31) / 32);                // stages along the whole K
  // split-K over the CTAs of a cluster (gridDim.y = cluster size): this CTA
  // takes stages [tb, te) and the partial sums meet in cluster rank 0
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
  __syncthreads();

  if (warp == NW) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      bool ok = true;
      int ic = 0;                                   // stages issued
      for (int t = 0; t < T && ok; ++t) {
        const int s = t % D;
        if (t >= D) ok = mbar_wait_bounded(empty0 + 8 * s, uint32_t(((t / D) - 1) & 1));
        // the first stage goes out alone: with every CTA's whole ring in flight at once
        // the memory system returns the first stages late
        if (t == 1) ok = ok && mbar_wait_bounded(full0, 0u);
        if (!ok) break;
        const int64_t k0 = int64_t(tb + t) * 1024;
        const uint32_t xbytes = uint32_t((K - k0 < 1024 ? K - k0 : 1024) * 2);
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(full0 + 8 * s),
                     "r"(uint32_t(Cfg::STAGE_BYTES) + xbytes)
                     : "memory");
#pragma unroll
        for (int b = 0; b < BITS; ++b)
          asm volatile(
              "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
              " [%0], [%1, {%3, %4}], [%2];" ::"r"(ring + s * Cfg::STAGE_BYTES + b * Cfg::BOX_BYTES),
              "l"(&tm_codes), "r"(full0 + 8 * s), "r"((tb + t) * Cfg::STAGE_WORDS + 32 * b), "r"(int(row0))
              : "memory");
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                xraw0 + s * Cfg::XRAW_BYTES),
            "l"(x + k0), "r"(xbytes), "r"(full0 + 8 * s)
            : "memory");
        ++ic;
      }
      if (!ok) {
        // Copies issued but not consumed must land before the CTA exits.  Only
        // the last D issued stages can still be in flight (a slot is re-armed
        // only by issuing the stage D later), each in phase t / D of its slot.
        for (int t = ic > D ? ic - D : 0; t < ic; ++t)
          bw::drain_wait(full0 + 8 * (t % D), uint32_t((t / D) & 1), &g_gemv_tma_timeout);
      }
    }
  } else {
    // ---------------------------------------------------------------- consumers
    const int lr = lane & 7, kq = lane >> 3;
    float* xs = reinterpret_cast<float*>(xs_base) + warp * 4 * XU;
    const float xscale = __uint_as_float(uint32_t(127 + kScaleS - code_p<BITS>(lane)) << 23);
    const int ub = 4 * warp;                           // this warp's first unit in a box

    // (s, z) of rows row0..row0+31, groups [wg0, wg0 + gcap): thread c of the
    // 256 consumers reads groups c % 8, c % 8 + 8, ... of row c / 8.  Every
    // consumer passes both barriers, also after a timed-out wait.
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
    for (int i = 0; i < 4; ++i) unit_offsets<BITS>(lr + 8 * i, ub + kq, uoff[i]);
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int s = t % D;
      const int64_t u0 = int64_t(tb + t) * 32;         // first unit of the stage
      if (!one_window) {
        const int64_t ue = (u0 + 32 < KU ? u0 + 32 : KU) - 1;
        if (int64_t(units_per_group.div(uint32_t(ue))) >= wg0 + gcap) {
          wg0 = units_per_group.div(uint32_t(u0));
          load_table(wg0);
        }
      }
      {   // the common case (stage landed) without the call to the bounded wait
        const uint32_t par = uint32_t((t / D) & 1);
        if (ok) ok = __all_sync(0xffffffffu, mbar_try(full0 + 8 * s, par) || mbar_wait_bounded(full0 + 8 * s, par));
      }
      // x' of this warp's 4 units (zero past K) and sum x of the lane's unit kq
      const __nv_bfloat16* xr =
          reinterpret_cast<const __nv_bfloat16*>(smem + D * Cfg::STAGE_BYTES + s * Cfg::XRAW_BYTES) +
          ub * 32 + lane;
      float xv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        xv[u] = (u0 + ub + u < KU) ? __bfloat162float(xr[32 * u]) : 0.0f;
        xs[u * XU + lane] = xv[u] * xscale;
      }
      float sx;
      {
        const bool h16 = lane & 16, h8 = lane & 8;
        float a = (h16 ? xv[2] : xv[0]) + __shfl_xor_sync(0xffffffffu, h16 ? xv[0] : xv[2], 16);
        float b = (h16 ? xv[3] : xv[1]) + __shfl_xor_sync(0xffffffffu, h16 ? xv[1] : xv[3], 16);
        sx = (h8 ? b : a) + __shfl_xor_sync(0xffffffffu, h8 ? a : b, 8);
        sx += __shfl_xor_sync(0xffffffffu, sx, 4);
        sx += __shfl_xor_sync(0xffffffffu, sx, 2);
        sx += __shfl_xor_sync(0xffffffffu, sx, 1);
      }
      __syncwarp();                      // x' is visible to every lane
      const uint32_t stage = ring + uint32_t(s * Cfg::STAGE_BYTES);
      float xp[32];
      const float4* xq = reinterpret_cast<const float4*>(xs + kq * XU);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 v = xq[j];
        xp[4 * j] = v.x; xp[4 * j + 1] = v.y; xp[4 * j + 2] = v.z; xp[4 * j + 3] = v.w;
      }
      // past K the unit's x' and sum are zero, so any table entry will do
      int64_t grp = int64_t(units_per_group.div(uint32_t(u0 + ub + kq))) - wg0;
      grp = grp < gcap ? grp : gcap - 1;
      const float2* tz = tbl + lr * gcap + grp;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t w[BITS];
        load_unit_at<BITS>(stage, uoff[i], w);
        float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
        Dot<BITS, 0>::run(w, xp, d);
        const float dot = (d[0] + d[1]) + (d[2] + d[3]);
        const float2 sz = tz[8 * i * gcap];
        acc[i] = fmaf(sz.x, fmaf(dot, 0x1p85f, -sz.y * sx), acc[i]);
      }
      __syncwarp();                      // this warp is done with stage s and its x' buffer
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(empty0 + 8 * s) : "memory");
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v = acc[i];
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      if (kq == 0) red[warp][lr + 8 * i] = v;
    }
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = 0.0f;
#pragma unroll
    for (int w = 0; w < NW; ++w) v += red[w][threadIdx.x];
    red[0][threadIdx.x] = v;                        // this CTA's partial sums
  }
  if (ks > 1) {
    // every CTA of the cluster has its partials in red[0]; rank 0 adds them
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (kr == 0 && threadIdx.x < 32) {
      float v = red[0][threadIdx.x];
      const uint32_t mine = saddr(&red[0][threadIdx.x]);
      for (int r = 1; r < ks; ++r) {
        uint32_t peer;
        float pv;
        asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(peer) : "r"(mine), "r"(r));
        asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(pv) : "r"(peer) : "memory");
        v += pv;
      }
      red[0][threadIdx.x] = v;
    }
    // peers keep their shared memory until rank 0 has read it
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
  } else {
    __syncthreads();
  }
  if (kr == 0 && threadIdx.x < 32) {
    const int64_t n = row0 + threadIdx.x;
    if (n < N) y[n] = __float2bfloat16_rn(red[0][threadIdx.x]);
  }
}

template <int BITS>
cudaError_t launch_bits(const __nv_bfloat16* x, int64_t N, int64_t K, const uint32_t* codes,
                        const __half* scales, const __half* zeros, int64_t g, __nv_bfloat16* y,
                        cudaStream_t st) {
  using Cfg = M1Cfg<BITS>;
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
    cudaError_t e = cudaFuncSetAttribute(gemv_m1_tma_kernel<BITS, 2>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::smem(kMaxGcap));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gemv_m1_tma_kernel<BITS, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cfg::smem(kMaxGcap));
    int nsm_dev = 0;
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&nsm_dev, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    sms[dev].store(nsm_dev, std::memory_order_relaxed);
    attr_set[dev].store(true, std::memory_order_release);
  }
  // Split K over a cluster of ks CTAs (at most 8) when the row tiles alone
  // would leave SMs idle or run in a ragged second wave; every CTA keeps at
  // least WQ_GEMV_M1_MIN_STAGES stages of K so its TMA ring still pipelines.
  const int64_t tiles = (N + 31) / 32;
  const int64_t KU = K / 32, stages = (KU + 31) / 32;
  int ks = int((WQ_GEMV_M1_TARGET_CTAS + tiles - 1) / tiles);
  ks = ks < 1 ? 1 : (ks > 8 ? 8 : ks);
  while (ks > 1 && stages / ks < WQ_GEMV_M1_MIN_STAGES) --ks;
  // Scale table: the most groups one CTA's K range spans, odd (bank-conflict
  // free rows), at most kMaxGcap (longer ranges reload the table).
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
  // The variant sized for three CTAs per SM, when three fit in shared memory
  // and the grid then runs in fewer waves.
  const int nsm_known = (dev >= 0 && dev < 64) ? sms[dev].load(std::memory_order_relaxed) : 0;
  const int64_t ctas = tiles * ks, nsm = nsm_known > 0 ? nsm_known : 1;
  if ((ctas + 3 * nsm - 1) / (3 * nsm) < (ctas + 2 * nsm - 1) / (2 * nsm) && 3 * (smem + 1024) <= 228 * 1024)
    return cudaLaunchKernelEx(&cfg, gemv_m1_tma_kernel<BITS, 3>, tm, x, N, K, scales, zeros, fd, gcap, y);
  return cudaLaunchKernelEx(&cfg, gemv_m1_tma_kernel<BITS, 2>, tm, x, N, K, scales, zeros, fd, gcap, y);
}

}  // namespace

bool gemv_m1_tma_supported(const void* x, const void* codes, int64_t K, int bits) {
  // code rows and x start on 16 bytes: TMA box copies and bulk copies of x
  return (K * bits) % 128 == 0 && (reinterpret_cast<uintptr_t>(x) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(codes) & 15) == 0;
}

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
