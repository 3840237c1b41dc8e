// fp32 SIMT path (placeholder).
#include <cuda_runtime.h>
#include "mala.h"
namespace mala {
mala_status fp32_fwd(const float*, const float*, const float*, float*, float*, int, int, int, int,
                     int, float, float, bool, uint8_t*, cudaStream_t) {
  return MALA_ERR_UNSUPPORTED;
}
}  // namespace mala
namespace mala {
mala_status fp32_decode(const float*, const float*, const float*, float*, float*, int, int, int,
                        int, int, float, float, int, bool, uint8_t*, uint8_t*, cudaStream_t) {
  return MALA_ERR_UNSUPPORTED;
}
}  // namespace mala
namespace mala {
mala_status fp32_bwd(const float*, const float*, const float*, const float*, const float*,
                     const float*, float*, float*, float*, int, int, int, int, int, float, float,
                     bool, uint8_t*, uint8_t*, cudaStream_t) {
  return MALA_ERR_UNSUPPORTED;
}
}  // namespace mala
