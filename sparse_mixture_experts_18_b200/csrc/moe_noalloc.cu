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

// Device address of the array on the current device.  In host code the array's name is only
// a stand-in, not an address a kernel may use, so it is looked up with cudaGetSymbolAddress
// on every call (cheap; a context re-created after cudaDeviceReset gets a new address).  When
// the address is new for this device (the first call, or a new context), the 256-byte header
// at its start -- the status word and the routing tickets, the only part of a workspace that
// must begin at zero -- is zeroed with cudaMemsetAsync on the caller's stream, so that it is
// ordered before the kernels this call then enqueues on that stream.
moe_status noalloc_workspace(cudaStream_t stream, void** addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MOE_ERR_CUDA;
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_workspace) != cudaSuccess || p == nullptr)
    return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  if (g_workspace_addr[dev] != p) {
    if (cudaMemsetAsync(p, 0, 256, stream) != cudaSuccess) return MOE_ERR_CUDA;
    g_workspace_addr[dev] = p;
  }
  *addr = p;
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
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  const moe_status st = noalloc_workspace(s, &ws);
  if (st != MOE_OK) return st;
  return moe_forward(x, W_g, W1, W3, W2, T, d, F, n, K, dt, out, ws,
                     (size_t)MOE_NOALLOC_WORKSPACE_BYTES, stream);
}

extern "C" moe_status moe_noalloc_status(void* stream, uint32_t* raw) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  void* ws = nullptr;
  moe_status st = noalloc_workspace(s, &ws);
  if (st != MOE_OK) return st;
  st = moe_workspace_status(ws, stream, raw);
  if (st == MOE_OK) return st;
  // an interrupted call can leave the routing tickets mid-count: start the next one afresh
  if (cudaMemsetAsync(ws, 0, 256, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return st;
}
