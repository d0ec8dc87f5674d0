// Absorbed-MLA paged prefill (placeholder until the tcgen05 kernel lands).
#include <cuda_runtime.h>

#include "pkv_internal.h"

namespace pkv {

cudaError_t launch_mla(const LaunchGeom&, const DeviceView&, const int32_t*, const void*, const void*,
                       const void*, const void*, void*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace pkv
