// grouped.h -- structures shared by the C ABI layer (wq_api.cu) and the
// grouped decode GEMV (gemv_grouped.cu).
#pragma once
#include <cuda.h>   // CUtensorMap
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#include "wq_internal.cuh"

namespace wq {

constexpr int kMaxLinears = 128;      // linears per persistent launch (kernel parameter space)
constexpr int kMaxPrepLinears = 512;  // linears per activation-preparation launch
constexpr int kMaxCtas = 1024;        // persistent CTAs per launch (workspace sizing)

// One linear of a grouped call, after validation (group already effective).
struct GroupedLinear {
  const __nv_bfloat16* x;
  const uint32_t* codes;
  const __half* scales;
  const __half* zeros;   // null: symmetric grid, zero 2^(bits-1)
  __nv_bfloat16* y;
  int64_t N, K, group;
};

// Workspace carve-up: counters, parked partial sums, then per linear the
// prepared activations x' and the per-quad sums of x.
struct WsLayout {
  unsigned* cnt = nullptr;
  float* part = nullptr;
  std::vector<uint32_t*> xp;
  std::vector<float*> sx;
};

// Kernel-side description of one linear.
struct GLin {
  const __half* scales;
  const __half* zeros;
  __nv_bfloat16* y;
  uint32_t* xp;
  float* sx;
  int64_t stage0;   // first index of this linear's stages in the launch's sequence
  int N, K, G, TS, tiles;
  FastDiv upg;      // 32-code units per scale group
};

struct GParams {
  CUtensorMap tm[kMaxLinears];
  GLin lin[kMaxLinears];
  int nlin, M;
  int64_t total;    // stages of the launch
  int P;            // persistent CTAs
  float* part;
  unsigned* cnt;
};

struct PrepLin {
  const __nv_bfloat16* x;
  int K;
  uint32_t* xp;
  float* sx;
};

struct PrepParams {
  PrepLin lin[kMaxPrepLinears];
  int nlin, M;
};

// Token tile of the grouped kernel for a batch of M (1, 2, 4, 8 or 16).
int grouped_token_tile(int M);
// True when the grouped kernel takes this shape (K and group multiples of 128).
bool grouped_supported(int64_t K, int64_t g);
// Bytes of workspace a grouped call needs; with `out`, also the carve-up of
// the workspace starting at `base`.
size_t grouped_workspace_layout(const GroupedLinear* lins, int count, int M, uintptr_t base, WsLayout* out);
cudaError_t launch_gemv_grouped(const GroupedLinear* lins, int count, int M, int bits, const WsLayout& ws,
                                cudaStream_t st);
bool gemv_grouped_read_and_clear_timeout(cudaError_t* err);

// 17 <= M <= 255 (gemm_sw_supported): the swap-AB tensor-core GEMM over many
// linears in one launch per 64 linears, one CTA per 128-row tile over all of K
// (gemm_sw.cu).  No workspace.
cudaError_t launch_gemm_sw_grouped(const GroupedLinear* lins, int count, int64_t M, int bits, cudaStream_t st);

// The built-in workspace of wq_gemm_grouped_noalloc (noalloc.cu): its size,
// and its device address on the current device (looked up on first use).
size_t static_workspace_bytes();
cudaError_t static_workspace(void** addr);

}  // namespace wq
