// Launchers of kernels not built yet: they report "not supported".
#include "rrq_params.h"

namespace rrq {
cudaError_t launch_q4_0(const void*, int, int64_t, int, uint64_t, int, float, void*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_q4_0_decode(const void*, int64_t, int, uint64_t, int, float, void*, int,
                               cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_encode_qjl(const void*, int, int64_t, int, const QuantParams&, const uint16_t*,
                              uint8_t*, float*, uint8_t*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace rrq
