// moe_noalloc.cu -- moe_forward for callers that cannot allocate device memory.
//
// Some callers of this library have no way to obtain a workspace: a plugin hosted by an
// application that owns every device allocation through its own pool and forbids outside
// cudaMalloc calls, or a latency-critical loop that must never allocate because cudaMalloc
// can synchronise the device.  moe_forward_noalloc serves them with a workspace that lives
// in this file's fixed-size device array instead of caller memory.
//
// The array below is part of the library's device image: every GPU that loads it holds
// MOE_NOALLOC_WORKSPACE_BYTES of device memory until the process exits.
#include <mutex>

#include "../../include/moe.h"
#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_workspace[MOE_NOALLOC_WORKSPACE_BYTES];

std::mutex g_setup_mu;
void* g_workspace_addr[64] = {};  // device address of g_noalloc_workspace, per device

// Once per device, with that device current: look up the array's device address (in host
// code the array's name is only a stand-in, not an address a kernel may use) and zero the
// status word at its start, which is the only part of a workspace that must begin at zero.
moe_status noalloc_workspace(void** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (!g_workspace_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_workspace) != cudaSuccess || p == nullptr)
      return MOE_ERR_CUDA;
    if (cudaMemset(p, 0, 256) != cudaSuccess) return MOE_ERR_CUDA;
    g_workspace_addr[dev] = p;
  }
  *addr = g_workspace_addr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_forward_noalloc(const void* x, const float* W_g, const void* W1,
                                          const void* W3, const void* W2, int64_t T, int64_t d,
                                          int64_t F, int n, int K, moe_dtype dt, void* out,
                                          void* stream) {
  const size_t need = moe_workspace_bytes(T, d, F, n, K, dt);
  if (need == 0)  // unsupported or invalid shape: moe_forward reports which, before any use
    return moe_forward(x, W_g, W1, W3, W2, T, d, F, n, K, dt, out, nullptr, 0, stream);
  if (T == 0) return MOE_OK;
  if (need > (size_t)MOE_NOALLOC_WORKSPACE_BYTES) return MOE_ERR_WORKSPACE;
  void* ws = nullptr;
  const moe_status st = noalloc_workspace(&ws);
  if (st != MOE_OK) return st;
  return moe_forward(x, W_g, W1, W3, W2, T, d, F, n, K, dt, out, ws,
                     (size_t)MOE_NOALLOC_WORKSPACE_BYTES, stream);
}
