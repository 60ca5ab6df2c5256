// Backward that uses a static device scratch array instead of a
// caller-allocated workspace, for callers that cannot allocate device memory.
// It runs the CUDA-core backward kernels (fp32 arithmetic), whose workspace -
// row statistics, the recomputed summaries and their gradients - fits a
// modest static array; the tensor-core backward of pack3d_backward stages
// grid-order copies of q, k, v and dO (hundreds of MB at the 65k shape),
// which no static array of a stated modest size holds.
#include "pack3d_internal.cuh"

namespace {

// The scratch the backward needs (row statistics, recomputed summaries and
// their gradients), shared by every call on a device.
__device__ __align__(256) unsigned char g_backward_scratch[PACK3D_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch array on the current device (the host-side
// symbol is a stand-in, not a device address).  Looked up on every call: the
// lookup is not a stream operation and costs little, and an address cached
// across calls would go stale if the device's primary context were destroyed
// and created again.
int scratch_for_current_device(void** out) {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_backward_scratch) != cudaSuccess || !ptr)
    return PACK3D_ERR_CUDA;
  *out = ptr;
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
  if ((rc = p3d::backward_simt_supported(g))) return rc;
  if (p3d::backward_workspace_bytes(g, true) > PACK3D_NOALLOC_SCRATCH_BYTES)
    return PACK3D_ERR_UNSUPPORTED;
  if (!idx || !q || !k || !v || !out || !lse || !dout || !dq || !dk || !dv) return PACK3D_ERR_ARG;
  void* scratch = nullptr;
  if ((rc = scratch_for_current_device(&scratch))) return rc;
  return p3d::backward_call(p, idx, q, k, v, out, lse, dout, dq, dk, dv, scratch,
                            PACK3D_NOALLOC_SCRATCH_BYTES, true, (cudaStream_t)stream);
}
