// kvq_selftest.cu -- a self-test of the bounded mbarrier wait every kernel of
// the library uses, so that the timeout path can be run on a GPU without a
// fault: one warp waits on an mbarrier phase that is either completed first
// (arrive = 1: the wait must succeed, no error) or never completed (arrive =
// 0: the wait gives up after about two seconds and KVQ_DERR_TIMEOUT is set).
#include "kvq.h"
#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

__global__ void bounded_wait_kernel(int* d_err, int arrive) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_init_fence();
  }
  __syncwarp();
  if (arrive && threadIdx.x == 0) mbar_arrive(&bar);
  __syncwarp();
  const bool done = mbar_wait_bounded(&bar, 0);
  if (__any_sync(0xffffffffu, !done) && threadIdx.x == 0) set_err(d_err, kErrTimeout);
}

}  // namespace
}  // namespace kvq

extern "C" kvq_status kvq_selftest_bounded_wait(int32_t* d_err, int32_t arrive,
                                                kvq_stream stream) {
  if (!d_err) return KVQ_ERR_INVALID_ARG;
  kvq::bounded_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(d_err, arrive != 0);
  return cudaGetLastError() == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA;
}
