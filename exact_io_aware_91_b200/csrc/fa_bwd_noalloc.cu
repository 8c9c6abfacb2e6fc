// fa_bwd_noalloc: the backward pass (fa_bwd_gqa with H_kv = H) with its workspace taken from
// a scratch array compiled into the library, for callers that cannot allocate device memory
// (see fa.h).
// The array is a file-scope __device__ variable; host code cannot use its name as
// a device address, so the address is looked up once per device with
// cudaGetSymbolAddress while that device is current, and handed to fa_bwd_gqa.
#include <cmath>
#include <cstddef>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/fa.h"

namespace {

constexpr size_t kScratchBytes = FA_BWD_NOALLOC_MAX_WORKSPACE;
static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];  // device address of g_bwd_scratch, per device
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (nullptr on failure).
void* scratch_address() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_bwd_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                                    const void* o_resid, const void* dout, const float* lse, float* dq, float* dk,
                                    float* dv, int B, int H, int N, int d, float scale, int causal,
                                    fa_stream_t stream) {
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need == 0)  // empty or invalid problem: fa_bwd_gqa returns FA_OK or the argument error
    return fa_bwd_gqa(q, k, v, o, o_resid, dout, lse, dq, dk, dv, B, H, H, N, d, scale, causal, nullptr, 0, stream);
  // argument errors are reported before any CUDA call, as fa_bwd_gqa does
  if (!(std::isfinite(scale) && scale > 0.f) || (causal != 0 && causal != 1)) return FA_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (need > kScratchBytes) return FA_ERR_UNSUPPORTED;
  void* scratch = scratch_address();
  if (scratch == nullptr) return FA_ERR_CUDA;
  return fa_bwd_gqa(q, k, v, o, o_resid, dout, lse, dq, dk, dv, B, H, H, N, d, scale, causal, scratch,
                    kScratchBytes, stream);
}
