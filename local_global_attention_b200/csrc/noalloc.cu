// Backward that uses a static device scratch array instead of a
// caller-allocated workspace, for callers that cannot allocate device memory.
// It runs the same kernels as pack3d_backward; only where the workspace comes
// from differs.
#include <mutex>

#include "pack3d_internal.cuh"

namespace {

constexpr int kMaxDevices = 64;

// The scratch the backward needs (row statistics, recomputed summaries and
// their gradients), shared by every call on a device.
__device__ __align__(256) unsigned char g_backward_scratch[PACK3D_NOALLOC_SCRATCH_BYTES];

std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices];  // device address of g_backward_scratch per device

// Device address of the scratch array on the current device, looked up once
// per device (the host-side symbol is a stand-in, not a device address).
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PACK3D_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return PACK3D_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_backward_scratch) != cudaSuccess || !ptr)
      return PACK3D_ERR_CUDA;
    g_scratch_addr[dev] = ptr;
  }
  *out = g_scratch_addr[dev];
  return PACK3D_OK;
}

}  // namespace

extern "C" int pack3d_backward_noalloc(const pack3d_params* p, const pack3d_index* idx,
                                       const void* q, const void* k, const void* v,
                                       const void* out, const float* lse, const void* dout,
                                       void* dq, void* dk, void* dv, pack3d_stream_t stream) {
  p3d::Geo g;
  int rc = p3d::make_geo(p, &g);
  if (rc) return rc;
  if (p3d::backward_workspace_bytes(g) > PACK3D_NOALLOC_SCRATCH_BYTES)
    return PACK3D_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if ((rc = scratch_for_current_device(&scratch))) return rc;
  return pack3d_backward(p, idx, q, k, v, out, lse, dout, dq, dk, dv, scratch,
                         PACK3D_NOALLOC_SCRATCH_BYTES, stream);
}
