// Launchers of kernels not built yet: they report "not supported".
#include "rrq_params.h"

namespace rrq {
cudaError_t launch_encode_qjl(const void*, int, int64_t, int, const QuantParams&, const uint16_t*,
                              uint8_t*, float*, uint8_t*, float*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace rrq
