// mala_decode_noalloc: split-KV decode that allocates no device memory.
//
// mala_decode needs a few megabytes of scratch for its split partials and merge
// tickets, which it takes from a caller workspace or allocates stream-ordered.  Some
// callers can do neither: a serving runtime that forbids allocation once its memory
// plan is fixed, a plugin running inside another framework that owns the device
// allocator, or code that must not call cudaMalloc / cudaMallocAsync on its hot path.
// This entry point serves them from a fixed array compiled into the library instead.
//
// The array has static storage on every GPU that loads the library and stays allocated
// until the process exits.  All calls on a device share it and it keeps the previous
// call's contents, so the parts that must start at zero (error word, merge tickets) are
// cleared on the stream at the start of every call; two calls whose work overlaps on
// the GPU (for example on two streams at once) race on it and must be serialised.

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "mala.h"
#include "mala_common.cuh"

namespace mala {

mala_status decode_dispatch(const void* q, const void* K, const void* V, void* O, float* LSE,
                            int B, int H, int Hkv, int Nk, int d, int dtype, float scale,
                            float tau, int num_splits, unsigned flags, uint8_t* ws,
                            uint8_t* tile_mask, float* tile_margin, uint64_t budget_ns,
                            cudaStream_t stream);
size_t decode_workspace_bytes(int B, int H, int Hkv, int Nk, int d, int dtype, int num_splits);
int decode_auto_splits(int B, int Hkv, int Nk);
bool common_args_ok(int B, int H, int Hkv, int L, int d, int dtype, float scale, float tau);
bool aligned16(const void* p);
uint64_t wait_budget_ns();

namespace {

// The scratch itself.  In host code `g_noalloc_scratch` is only a stand-in symbol, not
// a device address: the kernels get the address from cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MALA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};
void* g_scratch_ctx[kMaxDevices] = {};  // context the cached address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The current driver context (null if it cannot be queried).
void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  CUcontext ctx = nullptr;
  if (!fn || fn(&ctx) != CUDA_SUCCESS) return nullptr;
  return ctx;
}

// Device address of the scratch on the current device.  It is looked up once per device
// and context: after the primary context of a device has been destroyed and recreated
// (cudaDeviceReset) the module is loaded again, possibly elsewhere, so a cached address
// from the old context is looked up afresh.
mala_status scratch_for_current_device(uint8_t** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MALA_ERR_CUDA;
  // (before the runtime's first call on this thread no context may be current yet: the
  // lookup below then runs, and it makes the device's primary context current)
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (!g_scratch_ptr[dev] || !ctx || g_scratch_ctx[dev] != ctx) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
      return MALA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
    g_scratch_ctx[dev] = current_context();
  }
  *out = static_cast<uint8_t*>(g_scratch_ptr[dev]);
  return MALA_OK;
}

}  // namespace
}  // namespace mala

using namespace mala;

extern "C" mala_status mala_decode_noalloc(const void* q, const void* Kc, const void* Vc,
                                           void* O, float* LSE, int B, int H, int H_kv, int Nk,
                                           int d, int dtype, float scale, float tau,
                                           int num_splits, unsigned flags, uint8_t* tile_mask,
                                           void* stream) {
  if (!common_args_ok(B, H, H_kv, Nk, d, dtype, scale, tau)) return MALA_ERR_INVALID_ARG;
  if (!q || !Kc || !Vc || !O || !LSE) return MALA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(Kc) || !aligned16(Vc) || !aligned16(O))
    return MALA_ERR_INVALID_ARG;
  const int T = (Nk + kTile - 1) / kTile;
  if (num_splits == 0) num_splits = decode_auto_splits(B, H_kv, Nk);
  if (num_splits < 1 || num_splits > T) return MALA_ERR_INVALID_ARG;
  if (dtype == MALA_BF16 && d != 64 && d != 128) return MALA_ERR_UNSUPPORTED;
  if (dtype == MALA_BF16 && H / H_kv > 8) return MALA_ERR_UNSUPPORTED;  // up to 8 per group
  if (dtype == MALA_FP32 && d > 128) return MALA_ERR_UNSUPPORTED;
  const size_t need = decode_workspace_bytes(B, H, H_kv, Nk, d, dtype, num_splits);
  if (need > MALA_DECODE_NOALLOC_SCRATCH_BYTES) return MALA_ERR_WORKSPACE;
  uint8_t* ws = nullptr;
  mala_status st = scratch_for_current_device(&ws);
  if (st != MALA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the error word and counters must start at zero; the launcher clears the tickets
  if (cudaMemsetAsync(ws, 0, kWorkspaceHeader, s) != cudaSuccess) return MALA_ERR_CUDA;
  return decode_dispatch(q, Kc, Vc, O, LSE, B, H, H_kv, Nk, d, dtype, scale, tau, num_splits,
                         flags, ws, tile_mask, nullptr, wait_budget_ns(), s);
}
