// Self-test of failure detection without a GPU fault: one CTA waits on an
// mbarrier through the same bounded wait every tensor-core kernel uses.
// Armed, nothing completes the barrier's phase, so the wait gives up after
// its limit, records BB_ERR_TIMEOUT in the status word and returns; the
// kernel then exits normally and the context stays usable.  Unarmed, the
// waiting thread arrives first and the wait succeeds at once.
#include "sm100.cuh"

namespace bb {
namespace {

using namespace sm100;

__global__ void wait_probe_kernel(int* status, int armed) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!armed) mbar_arrive(&bar);  // completes phase 0
    mbar_wait(&bar, 0, &abort_flag, status);
  }
}

}  // namespace
}  // namespace bb

extern "C" int bb_debug_wait_probe(void* workspace, size_t ws_bytes, int armed,
                                   void* stream) {
  if (!workspace || ((uintptr_t)workspace & 15u) || ws_bytes < 256 ||
      (armed != 0 && armed != 1))
    return BB_ERR_INVALID;
  cudaStream_t s = (cudaStream_t)stream;
  int* status = (int*)workspace;  // the status word of a call's workspace
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess) return BB_ERR_CUDA;
  bb::wait_probe_kernel<<<1, 32, 0, s>>>(status, armed);
  return cudaGetLastError() == cudaSuccess ? BB_OK : BB_ERR_CUDA;
}
