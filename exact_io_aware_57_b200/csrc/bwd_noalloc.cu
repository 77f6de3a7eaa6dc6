// attn_bwd_noalloc: the backward without a caller-provided workspace.
//
// Some callers cannot call cudaMalloc at the point where they run the backward:
// code embedded in a framework that owns every byte of device memory (an extra
// allocation would fail or break its accounting), or latency-critical loops
// where cudaMalloc's implicit device synchronisation is not acceptable.  For
// them this entry point takes its scratch (the fp32 dQ accumulator and the
// D_i = dO_i . O_i row terms) from a fixed array that is part of the library
// image, so it allocates nothing.
//
// Costs and rules:
//   * every GPU that loads the library holds kScratchBytes of device memory for
//     that array until the process exits;
//   * problems whose scratch exceeds kScratchBytes are rejected;
//   * all calls share the one array per device, so calls that overlap on the
//     GPU (different streams, or different host threads without ordering) race;
//     the kernels zero what must start at zero on every call, so the contents a
//     previous call left behind do not matter;
//   * the first call on a device looks up the array's device address
//     (cudaGetSymbolAddress) with that device current and keeps it; make that
//     first call before any stream capture.  A cudaDeviceReset after it is not
//     supported (the array may then sit at another address).
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace attn {
namespace {

constexpr size_t kScratchBytes = ATTN_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_bwd_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device (looked up once
// per device).  In host code `g_bwd_scratch` is only a stand-in symbol, never a
// device address, so it must not be passed to a kernel directly.
void* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_bwd_scratch) != cudaSuccess || ptr == nullptr) return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace attn

extern "C" int attn_bwd_noalloc(const void* q, const void* k, const void* v, const float* bias,
                                long long bias_batch_stride, const void* o, const float* lse, const void* dout,
                                void* dq, void* dk, void* dv, int batch, int h_q, int h_kv, int n_q, int n_k, int d,
                                float scale, int causal, int dtype, void* stream) {
  using namespace attn;
  if (batch <= 0 || h_q <= 0 || n_q <= 0 || d <= 0) return ATTN_ERR_INVALID;
  const size_t need = attn_bwd_workspace_size(batch, h_q, n_q, d);
  if (need == 0 || need > kScratchBytes) return ATTN_ERR_WORKSPACE;  // larger than the built-in scratch
  // the array serves as attn_bwd's workspace (accumulator first, then D)
  void* scratch = scratch_on_current_device();
  if (!scratch) return ATTN_ERR_CUDA;
  return attn_bwd(q, k, v, bias, bias_batch_stride, o, lse, dout, dq, dk, dv, scratch, kScratchBytes, batch, h_q, h_kv,
                  n_q, n_k, d, scale, causal, dtype, stream);
}
