// Diagnostic of the bounded device-side waits.  Every wait of the library's
// kernels polls an mbarrier a bounded number of times; a CTA whose wait runs
// out sets the timeout bit of the index error word, drains what it has in
// flight and returns, so the context stays usable.  This entry point runs the
// same wait on a barrier phase that nothing completes and reports the result.
#include "pack3d_internal.cuh"
#include "tc_primitives.cuh"

namespace p3d {
namespace {

__device__ int32_t g_selftest_word;

// One warp: a barrier expecting one arrival that never comes.
__global__ void k_wait_selftest(uint32_t polls) {
  using namespace tc;
  __shared__ uint64_t bar;
  __shared__ int32_t abort_word;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_word = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const bool ok = __all_sync(0xffffffffu, mbar_wait_or_abort(&bar, 0, polls, &abort_word));
  if (threadIdx.x == 0) g_selftest_word = ok ? 0 : 4;
}

}  // namespace
}  // namespace p3d

extern "C" int pack3d_wait_selftest(uint32_t polls, pack3d_stream_t stream) {
  if (polls == 0 || polls > (1u << 24)) return PACK3D_ERR_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  p3d::k_wait_selftest<<<1, 32, 0, s>>>(polls);
  p3d::count_launches(1);
  if (cudaGetLastError() != cudaSuccess) return PACK3D_ERR_CUDA;
  int32_t word = -1;
  if (cudaMemcpyFromSymbolAsync(&word, p3d::g_selftest_word, sizeof(word), 0,
                                cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return PACK3D_ERR_CUDA;
  return word == 4 ? PACK3D_ERR_TIMEOUT : (word == 0 ? PACK3D_OK : PACK3D_ERR_CUDA);
}
