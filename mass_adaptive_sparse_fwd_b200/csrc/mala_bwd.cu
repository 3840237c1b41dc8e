// MALA backward (placeholder until the sm_100a kernel lands).
#include <cuda_runtime.h>
#include "mala.h"
#include "mala_common.cuh"
namespace mala {
size_t bwd_workspace_bytes(int B, int H, int Hkv, int L, int d, int dtype) {
  (void)Hkv; (void)dtype;
  return kWorkspaceHeader + (size_t)B * L * H * d * 4 + (size_t)B * H * L * 4;
}
mala_status bwd_dispatch(const void*, const void*, const void*, const void*, const float*,
                         const void*, void*, void*, void*, int, int, int, int, int, int, float,
                         float, unsigned, uint8_t*, uint8_t*, uint64_t, cudaStream_t) {
  return MALA_ERR_UNSUPPORTED;
}
}  // namespace mala
