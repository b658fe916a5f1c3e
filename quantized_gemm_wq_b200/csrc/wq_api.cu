// wq_api.cu -- the C ABI of libwq.so (include/wq.h): argument checks, device
// check, dispatch on the batch size, status strings.
//
// Every check runs before any launch, so a failing call writes nothing.
#include <mutex>
#include <vector>

#include "../../include/wq.h"
#include "grouped.h"
#include "wq_internal.cuh"

namespace {

bool valid_bits(int b) { return b == 2 || b == 3 || b == 4 || b == 8; }

// K is assumed already checked (>= 32, multiple of 32).
bool valid_group(int64_t K, int64_t group) {
  if (group == 0 || group == K) return true;
  return group > 0 && group % 32 == 0 && K % group == 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kMaxDim = int64_t(1) << 31;

// Compute capability of every device, checked once per device.
wq_status check_device() {
  static std::mutex mu;
  static int verdict[64];   // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return WQ_ERR_CUDA;
  if (dev < 0 || dev >= 64) return WQ_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(mu);
  if (verdict[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return WQ_ERR_CUDA;
    verdict[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return verdict[dev] == 1 ? WQ_OK : WQ_ERR_UNSUPPORTED_DEVICE;
}

wq_status check_common(int64_t N, int64_t K, int bits, int64_t group) {
  if (!valid_bits(bits)) return WQ_ERR_BITS;
  if (N < 1 || K < 1 || K % 32 != 0 || N >= kMaxDim || K >= kMaxDim) return WQ_ERR_SHAPE;
  if (!valid_group(K, group)) return WQ_ERR_GROUP;
  return WQ_OK;
}

// One linear, arguments already checked: the kernel by batch size (see wq.h).
cudaError_t dispatch_one(const __nv_bfloat16* x, int64_t M, int64_t N, int64_t K, const uint32_t* codes,
                         const __half* s, const __half* z, int bits, int64_t g, __nv_bfloat16* y,
                         cudaStream_t strm) {
  cudaError_t e;
  if (M > wq::kGemvMaxM && wq::gemm_sw_supported(M, K)) {
    e = wq::launch_gemm_sw(x, M, N, K, codes, s, z, bits, g, y, strm);
  } else if (M > wq::kGemvMaxM && wq::gemm_tc_supported(K, bits)) {
    e = wq::launch_gemm_tc(x, M, N, K, codes, s, z, bits, g, y, strm);
  } else {
    // Small batches, and K that the tensor-core GEMM cannot stage with TMA
    // (K not a multiple of 128): 16 batch rows per launch.  One row runs the
    // CUDA-core GEMV (its short pipeline wins at one row); 2..16 rows the
    // tensor-core GEMVs where their shape rules allow, else the CUDA-core GEMV.
    e = cudaSuccess;
    for (int64_t m0 = 0; m0 < M && e == cudaSuccess; m0 += wq::kGemvMaxM) {
      const int mc = int(M - m0 < wq::kGemvMaxM ? M - m0 : wq::kGemvMaxM);
      if (wq::gemv_mma_supported(mc, x + m0 * K, codes, K, g))
        e = wq::launch_gemv_mma(x + m0 * K, mc, N, K, codes, s, z, bits, g, y + m0 * N, strm);
      else if (wq::gemv_tc_supported(mc, K, bits, g))
        e = wq::launch_gemv_tc(x + m0 * K, mc, N, K, codes, s, z, bits, g, y + m0 * N, strm);
      else
        e = wq::launch_gemv(x + m0 * K, mc, N, K, codes, s, z, bits, g, y + m0 * N, strm);
    }
  }
  return e;
}

// Checks of one grouped linear (same rules as wq_gemm).
wq_status check_linear(const wq_linear& L, int64_t M, int bits) {
  if (!L.x_bf16 || !L.codes || !L.scales_f16 || !L.y_bf16) return WQ_ERR_NULL;   // zeros NULL: symmetric
  wq_status st = check_common(L.N, L.K, bits, L.group);
  if (st != WQ_OK) return st;
  if (M < 1 || M >= kMaxDim) return WQ_ERR_SHAPE;
  if (!aligned16(L.x_bf16) || !aligned16(L.codes) || !aligned16(L.scales_f16) ||
      (L.zeros_f16 && !aligned16(L.zeros_f16)) || !aligned16(L.y_bf16))
    return WQ_ERR_ALIGN;
  return WQ_OK;
}

wq::GroupedLinear to_grouped(const wq_linear& L) {
  return wq::GroupedLinear{static_cast<const __nv_bfloat16*>(L.x_bf16), L.codes,
                           static_cast<const __half*>(L.scales_f16), static_cast<const __half*>(L.zeros_f16),
                           static_cast<__nv_bfloat16*>(L.y_bf16), L.N, L.K, wq::effective_group(L.K, L.group)};
}

// The linears of a grouped call that the swap-AB GEMM takes in grouped
// launches (17 <= M <= 255, K a multiple of 128).
std::vector<wq::GroupedLinear> grouped_sw_list(const wq_linear* lins, int count, int64_t M) {
  std::vector<wq::GroupedLinear> v;
  if (M <= wq::kGemvMaxM) return v;
  for (int i = 0; i < count; ++i) {
    const wq::GroupedLinear g = to_grouped(lins[i]);
    if (wq::gemm_sw_supported(M, g.K)) v.push_back(g);
  }
  return v;
}

// True when linear L of a grouped call runs in one of the grouped launches.
bool grouped_launch_takes(const wq::GroupedLinear& g, int64_t M) {
  return M <= wq::kGemvMaxM ? wq::grouped_supported(g.K, g.group) : wq::gemm_sw_supported(M, g.K);
}

// The linears of a grouped call that the persistent kernel takes.
std::vector<wq::GroupedLinear> grouped_fast_list(const wq_linear* lins, int count, int64_t M) {
  std::vector<wq::GroupedLinear> v;
  if (M > wq::kGemvMaxM) return v;
  for (int i = 0; i < count; ++i) {
    const wq::GroupedLinear g = to_grouped(lins[i]);
    if (wq::grouped_supported(g.K, g.group)) v.push_back(g);
  }
  return v;
}

}  // namespace

extern "C" {

size_t wq_codes_words(int64_t N, int64_t K, int bits) {
  if (!valid_bits(bits) || N < 1 || K < 1 || K % 32 != 0) return 0;
  return size_t(N) * size_t(K / 32) * size_t(bits);
}

size_t wq_params_count(int64_t N, int64_t K, int64_t group) {
  if (N < 1 || K < 1 || K % 32 != 0 || !valid_group(K, group)) return 0;
  return size_t(N) * size_t(K / wq::effective_group(K, group));
}

const char* wq_status_string(wq_status s) {
  switch (s) {
    case WQ_OK: return "ok";
    case WQ_ERR_NULL: return "a required pointer is NULL";
    case WQ_ERR_BITS: return "bits must be 2, 3, 4 or 8";
    case WQ_ERR_GROUP: return "group must be 0, K, or a multiple of 32 that divides K";
    case WQ_ERR_SHAPE: return "M, N, K must be >= 1 and < 2^31, K a multiple of 32";
    case WQ_ERR_ALIGN: return "every pointer must be 16-byte aligned";
    case WQ_ERR_UNSUPPORTED_DEVICE: return "the current device is not compute capability 10.0 (B200)";
    case WQ_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case WQ_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait expired";
    case WQ_ERR_WORKSPACE: return "the workspace is NULL or smaller than the call needs";
  }
  return "unknown status";
}

wq_status wq_quantize_rtn(const void* W_f16, int64_t N, int64_t K, int bits, int64_t group,
                          uint32_t* codes, void* scales_f16, void* zeros_f16, void* stream) {
  if (!W_f16 || !codes || !scales_f16 || !zeros_f16) return WQ_ERR_NULL;
  wq_status st = check_common(N, K, bits, group);
  if (st != WQ_OK) return st;
  if (!aligned16(W_f16) || !aligned16(codes) || !aligned16(scales_f16) || !aligned16(zeros_f16))
    return WQ_ERR_ALIGN;
  if ((st = check_device()) != WQ_OK) return st;
  cudaError_t e = wq::launch_quantize(static_cast<const __half*>(W_f16), N, K, bits,
                                      wq::effective_group(K, group), codes,
                                      static_cast<__half*>(scales_f16),
                                      static_cast<__half*>(zeros_f16),
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status wq_quantize_rtn_sym(const void* W_f16, int64_t N, int64_t K, int bits, int64_t group,
                              uint32_t* codes, void* scales_f16, void* stream) {
  if (!W_f16 || !codes || !scales_f16) return WQ_ERR_NULL;
  wq_status st = check_common(N, K, bits, group);
  if (st != WQ_OK) return st;
  if (!aligned16(W_f16) || !aligned16(codes) || !aligned16(scales_f16)) return WQ_ERR_ALIGN;
  if ((st = check_device()) != WQ_OK) return st;
  // a null zeros array selects the symmetric grid in the quantiser
  cudaError_t e = wq::launch_quantize(static_cast<const __half*>(W_f16), N, K, bits,
                                      wq::effective_group(K, group), codes,
                                      static_cast<__half*>(scales_f16), nullptr,
                                      static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status wq_gemm(const void* x_bf16, int64_t M, int64_t N, int64_t K, const uint32_t* codes,
                  const void* scales_f16, const void* zeros_f16, int bits, int64_t group,
                  void* y_bf16, void* stream) {
  if (!x_bf16 || !codes || !scales_f16 || !y_bf16) return WQ_ERR_NULL;   // zeros NULL: symmetric grid
  wq_status st = check_common(N, K, bits, group);
  if (st != WQ_OK) return st;
  if (M < 1 || M >= kMaxDim) return WQ_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scales_f16) ||
      (zeros_f16 && !aligned16(zeros_f16)) || !aligned16(y_bf16))
    return WQ_ERR_ALIGN;
  if ((st = check_device()) != WQ_OK) return st;
  const int64_t g = wq::effective_group(K, group);
  const cudaError_t e = dispatch_one(static_cast<const __nv_bfloat16*>(x_bf16), M, N, K, codes,
                                     static_cast<const __half*>(scales_f16),
                                     static_cast<const __half*>(zeros_f16), bits, g,
                                     static_cast<__nv_bfloat16*>(y_bf16), static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

size_t wq_gemm_grouped_workspace_size(const wq_linear* linears, int count, int64_t M, int bits) {
  if (!linears || count < 1 || !valid_bits(bits)) return 0;
  for (int i = 0; i < count; ++i)
    if (check_linear(linears[i], M, bits) != WQ_OK) return 0;
  const std::vector<wq::GroupedLinear> fast = grouped_fast_list(linears, count, M);
  if (fast.empty()) return 0;
  return wq::grouped_workspace_layout(fast.data(), int(fast.size()), int(M), 0, nullptr);
}

wq_status wq_gemm_grouped(const wq_linear* linears, int count, int64_t M, int bits, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (!linears) return WQ_ERR_NULL;
  if (count < 1) return WQ_ERR_SHAPE;
  if (!valid_bits(bits)) return WQ_ERR_BITS;
  for (int i = 0; i < count; ++i) {
    const wq_status st = check_linear(linears[i], M, bits);
    if (st != WQ_OK) return st;
  }
  const std::vector<wq::GroupedLinear> fast = grouped_fast_list(linears, count, M);
  wq::WsLayout ws;
  if (!fast.empty()) {
    const size_t need = wq::grouped_workspace_layout(fast.data(), int(fast.size()), int(M), 0, nullptr);
    if (!workspace || workspace_bytes < need) return WQ_ERR_WORKSPACE;
    if (!aligned16(workspace)) return WQ_ERR_ALIGN;
    wq::grouped_workspace_layout(fast.data(), int(fast.size()), int(M), reinterpret_cast<uintptr_t>(workspace),
                                 &ws);
  }
  wq_status st = check_device();
  if (st != WQ_OK) return st;
  const auto strm = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (!fast.empty()) e = wq::launch_gemv_grouped(fast.data(), int(fast.size()), int(M), bits, ws, strm);
  const std::vector<wq::GroupedLinear> sw = grouped_sw_list(linears, count, M);
  if (e == cudaSuccess && !sw.empty()) e = wq::launch_gemm_sw_grouped(sw.data(), int(sw.size()), M, bits, strm);
  for (int i = 0; i < count && e == cudaSuccess; ++i) {
    const wq::GroupedLinear g = to_grouped(linears[i]);
    if (grouped_launch_takes(g, M)) continue;
    e = dispatch_one(g.x, M, g.N, g.K, g.codes, g.scales, g.zeros, bits, g.group, g.y, strm);
  }
  return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status wq_gemm_grouped_noalloc(const wq_linear* linears, int count, int64_t M, int bits, void* stream) {
  if (!linears) return WQ_ERR_NULL;
  if (count < 1) return WQ_ERR_SHAPE;
  if (!valid_bits(bits)) return WQ_ERR_BITS;
  for (int i = 0; i < count; ++i) {
    const wq_status st = check_linear(linears[i], M, bits);
    if (st != WQ_OK) return st;
  }
  const std::vector<wq::GroupedLinear> fast = grouped_fast_list(linears, count, M);
  const size_t need =
      fast.empty() ? 0 : wq::grouped_workspace_layout(fast.data(), int(fast.size()), int(M), 0, nullptr);
  if (need > wq::static_workspace_bytes()) return WQ_ERR_WORKSPACE;
  wq_status st = check_device();
  if (st != WQ_OK) return st;
  const auto strm = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (!fast.empty()) {
    void* base = nullptr;
    e = wq::static_workspace(&base);
    if (e != cudaSuccess) return WQ_ERR_CUDA;
    wq::WsLayout ws;
    wq::grouped_workspace_layout(fast.data(), int(fast.size()), int(M), reinterpret_cast<uintptr_t>(base), &ws);
    // Every call shares the array: the tile counters must start at zero, and a
    // call that gave up a bounded wait may have left some set.
    e = cudaMemsetAsync(ws.cnt, 0, sizeof(unsigned) * wq::kMaxCtas, strm);
    if (e == cudaSuccess) e = wq::launch_gemv_grouped(fast.data(), int(fast.size()), int(M), bits, ws, strm);
  }
  const std::vector<wq::GroupedLinear> sw = grouped_sw_list(linears, count, M);
  if (e == cudaSuccess && !sw.empty()) e = wq::launch_gemm_sw_grouped(sw.data(), int(sw.size()), M, bits, strm);
  for (int i = 0; i < count && e == cudaSuccess; ++i) {
    const wq::GroupedLinear g = to_grouped(linears[i]);
    if (grouped_launch_takes(g, M)) continue;
    e = dispatch_one(g.x, M, g.N, g.K, g.codes, g.scales, g.zeros, bits, g.group, g.y, strm);
  }
  return e == cudaSuccess ? WQ_OK : WQ_ERR_CUDA;
}

wq_status wq_last_device_error(void) {
  cudaError_t e[6] = {cudaSuccess, cudaSuccess, cudaSuccess, cudaSuccess, cudaSuccess, cudaSuccess};
  const bool hit = wq::gemm_tc_read_and_clear_timeout(&e[0]) | wq::gemv_m1_tma_read_and_clear_timeout(&e[1]) |
                   wq::gemv_tc_read_and_clear_timeout(&e[2]) | wq::gemv_mma_read_and_clear_timeout(&e[3]) |
                   wq::gemv_grouped_read_and_clear_timeout(&e[4]) | wq::gemm_sw_read_and_clear_timeout(&e[5]);
  for (cudaError_t x : e)
    if (x != cudaSuccess) return WQ_ERR_CUDA;
  return hit ? WQ_ERR_DEVICE_TIMEOUT : WQ_OK;
}

}  // extern "C"
