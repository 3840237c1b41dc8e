// MALA split-KV decode (placeholder until the sm_100a kernel lands).
#include <cuda_runtime.h>
#include "mala.h"
#include "mala_common.cuh"
namespace mala {
int decode_auto_splits(int B, int Hkv, int Nk) {
  const int T = (Nk + kTile - 1) / kTile;
  int s = (2 * 148 + B * Hkv - 1) / (B * Hkv);
  return s < 1 ? 1 : (s > T ? T : s);
}
size_t decode_workspace_bytes(int B, int H, int Hkv, int Nk, int d, int dtype, int S) {
  (void)Hkv; (void)Nk; (void)dtype;
  return kWorkspaceHeader + (size_t)B * H * S * (d + 1) * 4;
}
mala_status decode_dispatch(const void*, const void*, const void*, void*, float*, int, int, int,
                            int, int, int, float, float, int, unsigned, uint8_t*, uint8_t*,
                            uint64_t, cudaStream_t) {
  return MALA_ERR_UNSUPPORTED;
}
}  // namespace mala
