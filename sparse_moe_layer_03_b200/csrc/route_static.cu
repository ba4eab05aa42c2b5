// moe_route_static: the router (moe_route) for callers that cannot allocate
// device memory.
//
// Some callers cannot call cudaMalloc or hand over a workspace: plugins whose
// host framework owns every device allocation and exposes no allocator to
// them; serving runtimes that fix their device memory at start-up and forbid
// allocation afterwards; and latency-critical paths that cannot afford
// cudaMalloc's implicit device-wide synchronisation.  For them this entry point
// takes the router's scratch from a fixed array that lives in this library's
// device image instead of a caller-provided workspace.
//
// The array is kStaticScratchBytes (4 MiB) per GPU, reserved on every GPU that
// loads the library and held until the process exits.  Its device address is
// looked up once per device (cudaGetSymbolAddress, with that device current)
// on the first call made on that device.  Every call shares the array: calls
// that may run at the same time on the GPU (different streams, or threads) race
// and must be serialised by the caller.  The array keeps the last call's
// contents; the counters that must start at zero are cleared by each call.
// The status word is not: like a workspace's, it keeps the first error a
// kernel found until moe_route_static_check_status reads and clears it.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "../../include/moe.h"
#include "kernels.h"

namespace {

constexpr size_t kStaticScratchBytes = 4u << 20;

// The scratch array.  Host code must not use `g_route_scratch` as a device
// address: on the host it is only a stand-in symbol; the real address comes
// from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_route_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

int scratch_for_current_device(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    char msg[160];
    snprintf(msg, sizeof(msg), "moe_route_static: no usable current device (%s)", cudaGetErrorString(e));
    moe::set_last_error_message(msg);
    return MOE_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_route_scratch);     // device `dev` is current here
    if (e != cudaSuccess || p == nullptr) {
      char msg[160];
      snprintf(msg, sizeof(msg), "moe_route_static: cudaGetSymbolAddress failed on device %d (%s)", dev,
               cudaGetErrorString(e));
      moe::set_last_error_message(msg);
      return MOE_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" int moe_route_static(const moe_config_t* cfg, const void* x, const void* wg, const float* router_bias,
                                int32_t* topk_idx, float* topk_w, int32_t* n_sel, int32_t* counts,
                                float* aux_loss, void* stream) {
  const size_t need = moe_workspace_size(cfg);
  if (need == 0)   // invalid configuration: moe_route reports the same code and message, launching nothing
    return moe_route(cfg, x, wg, router_bias, topk_idx, topk_w, n_sel, counts, aux_loss, nullptr, nullptr, 0, stream);
  if (need > kStaticScratchBytes) {
    char msg[200];
    snprintf(msg, sizeof(msg),
             "moe_route_static: this configuration needs %zu bytes of scratch, above the built-in %zu; "
             "use moe_route with a caller workspace",
             need, kStaticScratchBytes);
    moe::set_last_error_message(msg);
    return MOE_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  int rc = scratch_for_current_device(&ws);
  if (rc != MOE_OK) return rc;
  // the counters after the status word (and its error site) start at zero on every call; the
  // status word itself keeps an earlier call's error until it is read
  cudaError_t e = cudaMemsetAsync(static_cast<unsigned char*>(ws) + 8, 0, 248, (cudaStream_t)stream);
  if (e != cudaSuccess) {
    char msg[160];
    snprintf(msg, sizeof(msg), "moe_route_static: clearing the counters failed (%s)", cudaGetErrorString(e));
    moe::set_last_error_message(msg);
    return MOE_ERR_CUDA;
  }
  return moe_route(cfg, x, wg, router_bias, topk_idx, topk_w, n_sel, counts, aux_loss, nullptr, ws,
                   kStaticScratchBytes, stream);
}

extern "C" int moe_route_static_check_status(void* stream) {
  void* ws = nullptr;
  const int rc = scratch_for_current_device(&ws);
  if (rc != MOE_OK) return rc;
  return moe_check_status(ws, stream);
}
