// tc_unpack.cuh -- pieces shared by the tensor-core GEMVs: the per-segment
// unpack of packed codes into bf16 patterns (tables in unpack_tables.h), the
// activation slot factors, the no-swizzle shared-memory descriptor and the
// elected-lane MMA / commit.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

#include "unpack_tables.h"
#include "wq_ptx.cuh"

namespace wq {
namespace tcu {

using ptx::smem_u32;

template <int BITS>
__host__ __device__ constexpr const UnpackOp* unpack_table() {
  if constexpr (BITS == 2) return kUnpack2;
  else if constexpr (BITS == 3) return kUnpack3;
  else if constexpr (BITS == 4) return kUnpack4;
  else return kUnpack8;
}

// Window of the row's code stream starting at bit s, ANDed with the mask.
template <int BITS, int T>
__device__ __forceinline__ uint32_t unpack_op(const uint32_t (&w)[4 * BITS]) {
  constexpr UnpackOp op = unpack_table<BITS>()[T];
  constexpr int k = op.s / 32, sh = op.s % 32;
  uint32_t win;
  if constexpr (sh == 0) {
    win = w[k];
  } else if constexpr (k + 1 < 4 * BITS) {
    win = __funnelshift_r(w[k], w[k + 1], sh);
  } else {
    win = w[k] >> sh;
  }
  return win & op.mask;
}

template <int BITS, int T0, int T>
struct UnpackRun {
  __device__ __forceinline__ static void run(const uint32_t (&w)[4 * BITS], uint32_t (&o)[32]) {
    o[T - T0] = unpack_op<BITS, T>(w);
    if constexpr (T + 1 < T0 + 32) UnpackRun<BITS, T0, T + 1>::run(w, o);
  }
};

// Op t of the table: the codes its slot pair holds and the activation factors
// 2^(64 - b).
template <int BITS, int T>
struct OpPick {
  __device__ __forceinline__ static void run(int t, int& lo, int& hi, float& flo, float& fhi) {
    constexpr UnpackOp op = unpack_table<BITS>()[T];
    if (T == t) {
      lo = op.lo;
      hi = op.hi;
      flo = __int_as_float((127 + 64 - int(op.blo)) << 23);
      fhi = __int_as_float((127 + 64 - int(op.bhi)) << 23);
    }
    if constexpr (T + 1 < 64) OpPick<BITS, T + 1>::run(t, lo, hi, flo, fhi);
  }
};

__device__ __forceinline__ uint32_t bf162_bits(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);   // a -> low half
  return *reinterpret_cast<uint32_t*>(&h);
}

// Shared-memory descriptor, K-major, no swizzle: core matrices of 8 rows x 16
// bytes; lbo = byte step between core matrices along K, sbo = along N.
__device__ __forceinline__ uint64_t desc_noswz(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  return d;
}

// One elected lane of the (converged) warp issues the MMA / commit.
__device__ __forceinline__ void mma_elect(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred P, Q;\n\t"
      "elect.sync _|P, 0xffffffff;\n\t"
      "setp.ne.b32 Q, %3, 0;\n\t"
      "@P tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, Q;\n\t}" ::"r"(d),
      "r"(a), "l"(b), "r"(accum), "r"(idesc));
}
__device__ __forceinline__ void commit_elect(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred P;\n\t"
      "elect.sync _|P, 0xffffffff;\n\t"
      "@P tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Ring position: slot and phase parity of use j, advanced by `step` per call.
struct Ring {
  int slot = 0;
  uint32_t phase = 0;
  __device__ __forceinline__ void advance(int step, int size) {
    slot += step;
    while (slot >= size) {
      slot -= size;
      phase ^= 1u;
    }
  }
};

}  // namespace tcu
}  // namespace wq
