// Host-side launch helpers shared by the kernel launchers.
#pragma once
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

namespace pkv {

// Kernel attributes are per device: a kernel's dynamic shared-memory limit
// (and, with `max_carveout`, the preference for the whole unified L1 / shared
// array as shared memory) must be raised on every device that launches it.
// `done` keeps one bit per device ordinal below 64, so each device pays for the
// two driver calls once; on ordinals >= 64 the attributes are set on every
// call. Threads that race on a first launch both set the same values, which is
// harmless.
inline cudaError_t set_smem_attrs_once(const void* kernel, int smem_bytes, std::atomic<uint64_t>& done,
                                       bool max_carveout) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = (dev >= 0 && dev < 64) ? (uint64_t(1) << dev) : 0;
  if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e == cudaSuccess && max_carveout)
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && bit != 0) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

}  // namespace pkv
