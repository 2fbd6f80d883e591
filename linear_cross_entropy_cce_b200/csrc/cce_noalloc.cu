// cce_fwd_noalloc: the forward pass with its scratch in a fixed file-scope
// device array instead of a caller-provided workspace, for callers that
// cannot allocate device memory (see include/cce.h).  No cudaMalloc,
// cudaFree or allocating library routine is called here.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/cce.h"

namespace {

// The scratch itself.  In host code this name is only a stand-in for the
// device symbol: its device address comes from cudaGetSymbolAddress below
// and is what the kernels receive.
static __device__ __align__(256) unsigned char g_fwd_scratch[CCE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_dev_addr[kMaxDevices] = {};  // device address of g_fwd_scratch, per device

// Once per device, with that device current: look up the array's address.
void* scratch_on_current_device(int* rc) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *rc = CCE_EDEVICE;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_dev_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fwd_scratch) != cudaSuccess || p == nullptr) {
      *rc = CCE_EDEVICE;
      return nullptr;
    }
    g_dev_addr[dev] = p;
  }
  *rc = CCE_OK;
  return g_dev_addr[dev];
}

}  // namespace

extern "C" int cce_fwd_noalloc(const void* H, const void* E, const int32_t* y, int64_t N,
                               int64_t D, int64_t V, int32_t ignore_index,
                               const cce_segment* segs, int32_t n_segs, float* loss, float* lse,
                               float* colmax, int32_t* status, void* stream) {
  const size_t need = cce_fwd_workspace_size(N, D, V, segs ? n_segs : 0);
  if (need == 0) return CCE_EINVAL;
  if (need > (size_t)CCE_NOALLOC_SCRATCH_BYTES) return CCE_EWORKSPACE;  // beyond the fixed size
  if (N == 0) return cce_fwd(H, E, y, N, D, V, ignore_index, segs, n_segs, loss, lse, colmax,
                             nullptr, 0, status, stream);
  int rc = CCE_OK;
  void* scratch = scratch_on_current_device(&rc);
  if (rc != CCE_OK) return rc;
  return cce_fwd(H, E, y, N, D, V, ignore_index, segs, n_segs, loss, lse, colmax, scratch,
                 (size_t)CCE_NOALLOC_SCRATCH_BYTES, status, stream);
}
