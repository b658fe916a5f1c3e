// stage_smem.cuh -- shared-memory helpers of the TMA-staged decode GEMVs: a
// stage holds, for 32 rows, BITS boxes of 32 words per row as the 128-byte
// swizzled TMA copy lays them out; mbarrier polling and the global timer.
#pragma once
#include <cstdint>

#include "bounded_wait.cuh"

namespace wq {
namespace stg {

__device__ __forceinline__ uint32_t saddr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) { return bw::try_parity(bar, parity); }
__device__ __forceinline__ uint64_t now_ns() { return bw::now_ns(); }
// Shared-memory byte offset of word wi (0 .. 32*BITS-1) of row r in a stage:
// the stage holds BITS boxes of 32 words per row; inside a box, rows are 128
// bytes apart and the 16-byte chunk index is XOR-ed with r % 8 (128B swizzle).
__device__ __forceinline__ uint32_t swz_word(int r, int wi) {
  const int box = wi >> 5, c = (wi >> 2) & 7, e = wi & 3;
  return uint32_t(box * 4096 + r * 128 + ((c ^ (r & 7)) << 4) + (e << 2));
}

// Shared-memory offsets of the pieces of unit u of row r in a stage: one
// vector per 16-byte chunk (b = 2, 4, 8: 1, 1, 2 pieces) or one per word
// (b = 3: 3 pieces).  They do not depend on the stage, so each lane computes
// them once.
template <int BITS>
constexpr int unit_pieces() { return BITS == 3 ? 3 : (BITS == 8 ? 2 : 1); }

template <int BITS>
__device__ __forceinline__ void unit_offsets(int r, int u, uint32_t (&o)[unit_pieces<BITS>()]) {
  if constexpr (BITS == 3) {
#pragma unroll
    for (int j = 0; j < 3; ++j) o[j] = swz_word(r, 3 * u + j);
  } else if constexpr (BITS == 8) {
    o[0] = swz_word(r, 8 * u);
    o[1] = swz_word(r, 8 * u + 4);
  } else {
    o[0] = swz_word(r, BITS * u);
  }
}

template <int BITS>
__device__ __forceinline__ void load_unit_at(uint32_t stage, const uint32_t (&o)[unit_pieces<BITS>()],
                                             uint32_t (&w)[BITS]) {
  if constexpr (BITS == 4) {
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(stage + o[0]));
  } else if constexpr (BITS == 2) {
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(stage + o[0]));
  } else if constexpr (BITS == 8) {
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(stage + o[0]));
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7]) : "r"(stage + o[1]));
  } else {
#pragma unroll
    for (int j = 0; j < 3; ++j)
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(w[j]) : "r"(stage + o[j]));
  }
}

}  // namespace stg
}  // namespace wq
