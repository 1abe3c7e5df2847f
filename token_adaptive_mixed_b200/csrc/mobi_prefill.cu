// mobi_prefill.cu — prefill GEMM (T > 16) of the token-routed mixed-bit layer.
// The tcgen05 kernel is not in this file yet; the launcher reports "not supported".
#include <cstdint>

#include "mobi_device.cuh"
#include "mobi_host.h"

namespace mobi {

size_t prefill_ws_bytes(int64_t T, int64_t N, int64_t K) { return 0; }

cudaError_t launch_prefill(const void*, int64_t, int64_t, const int32_t*, const int32_t*, const int32_t*,
                           const uint32_t*, const uint32_t*, int64_t, int, float*, void*, cudaStream_t,
                           DeviceStatus*) {
  return cudaErrorNotSupported;
}

}  // namespace mobi
