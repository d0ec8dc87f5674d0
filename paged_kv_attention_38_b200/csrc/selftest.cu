// Self-test of the bounded device-side waits every kernel of the library uses.
//
// One CTA waits on an mbarrier that nothing ever arrives on, through the same
// mbar_wait the attention kernels call. The wait must give up after its time
// limit, record the timeout in the status word, raise the CTA's abort flag,
// and let the kernel return normally (the CUDA context stays usable); a
// second wait after the abort must return at once. No fault, trap or hang is
// involved: the kernel ends by itself after about two seconds.
#include <cuda_runtime.h>

#include <cstdint>
#include <string>

#include "pkv.h"
#include "sm100_ptx.cuh"

namespace pkv {
void set_last_error(const std::string& msg);

namespace {

__global__ void wait_timeout_kernel(int32_t* status, int64_t* times) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x != 0) return;
  WaitCtx wc{&abort_flag, status};
  const uint64_t t0 = globaltimer_ns();
  const bool first = mbar_wait(&bar, 0, wc);  // never completes: times out
  const uint64_t t1 = globaltimer_ns();
  const bool second = mbar_wait(&bar, 0, wc);  // the CTA is aborting: returns at once
  const uint64_t t2 = globaltimer_ns();
  times[0] = first ? -1 : (int64_t)(t1 - t0);
  times[1] = second ? -1 : (int64_t)(t2 - t1);
}

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_selftest_wait_timeout(int32_t* status, int64_t* times, void* stream) {
  using namespace pkv;
  if (!status || !times) {
    set_last_error("NULL pointer");
    return PKV_EINVAL;
  }
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status, times);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error(std::string("selftest: ") + cudaGetErrorString(e));
    return PKV_ECUDA;
  }
  return PKV_OK;
}
