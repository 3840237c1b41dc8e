// C-ABI entry points of the MALA library: argument validation, TMA descriptor
// construction, workspace handling and kernel launches.  See include/mala.h.

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <vector>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "mala.h"
#include "mala_common.cuh"
#include "sm100.cuh"

namespace mala {
cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, int d, bool screen, int grid, cudaStream_t stream);
mala_status bwd_dispatch(const void* Q, const void* K, const void* V, const void* O,
                         const float* LSE, const void* dO, void* dQ, void* dK, void* dV, int B,
                         int H, int Hkv, int L, int d, int dtype, float scale, float tau,
                         unsigned flags, uint8_t* ws, uint8_t* tile_mask, float* tile_margin,
                         uint64_t budget_ns, cudaStream_t stream);
size_t bwd_workspace_bytes(int B, int H, int Hkv, int L, int d, int dtype);
mala_status decode_dispatch(const void* q, const void* K, const void* V, void* O, float* LSE,
                            int B, int H, int Hkv, int Nk, int d, int dtype, float scale,
                            float tau, int num_splits, unsigned flags, uint8_t* ws,
                            uint8_t* tile_mask, float* tile_margin, uint64_t budget_ns,
                            cudaStream_t stream);
size_t decode_workspace_bytes(int B, int H, int Hkv, int Nk, int d, int dtype, int num_splits);
int decode_auto_splits(int B, int Hkv, int Nk);
mala_status fp32_fwd(const float* Q, const float* K, const float* V, float* O, float* LSE, int B,
                     int H, int Hkv, int L, int Lk, int d, float scale, float tau, bool screen,
                     uint8_t* ws, uint8_t* tile_mask, float* tile_margin, cudaStream_t stream);

// ---------------------------------------------------------------------------- shared host helpers

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// 4-D bf16 tensor [n3][n2][n1][n0] (n0 fastest), box {64, 1, 128, 1}, 128-byte swizzle.
bool make_tile_map(CUtensorMap* m, const void* base, int n0, int n1, int n2, int n3) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {(cuuint64_t)n0, (cuuint64_t)n1, (cuuint64_t)n2, (cuuint64_t)n3};
  cuuint64_t strides[3] = {(cuuint64_t)n0 * 2, (cuuint64_t)n0 * n1 * 2,
                           (cuuint64_t)n0 * n1 * n2 * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n > 0 ? n : 148;
}

static uint64_t g_budget_ns = 2000000000ull;

uint64_t wait_budget_ns() { return g_budget_ns; }

// Debug margin buffer of the calling host thread (mala_set_debug).
static thread_local float* t_margin = nullptr;
static thread_local size_t t_margin_count = 0;

// The margin buffer for a call that tests `entries` tiles: null when debugging is off.
// `ok` turns false when the registered buffer is too small for the call.
float* debug_margin(size_t entries, bool& ok) {
  ok = true;
  if (!t_margin) return nullptr;
  if (t_margin_count < entries) {
    ok = false;
    return nullptr;
  }
  return t_margin;
}

// Fills the first `entries` margins with the all-ones bit pattern (a NaN): entries of
// tiles that are not tested keep it, and the kernels' float max starts from it.
bool debug_margin_clear(float* margin, size_t entries, cudaStream_t stream) {
  return !margin || cudaMemsetAsync(margin, 0xff, entries * sizeof(float), stream) == cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool common_args_ok(int B, int H, int Hkv, int L, int d, int dtype, float scale, float tau) {
  if (B <= 0 || H <= 0 || Hkv <= 0 || L <= 0 || d <= 0) return false;
  if (H % Hkv != 0) return false;
  if (!(std::isfinite(scale) && scale > 0.f)) return false;
  if (!(std::isfinite(tau) && tau >= 0.f)) return false;
  if (dtype != MALA_BF16 && dtype != MALA_FP32) return false;
  return true;
}

// Runs `body(ws)` with either the caller's workspace or a stream-ordered allocation.
template <class F>
mala_status with_workspace(void* workspace, size_t ws_bytes, size_t need, cudaStream_t stream,
                           F body) {
  if (workspace) {
    if (ws_bytes < need) return MALA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return MALA_ERR_INVALID_ARG;
    return body(static_cast<uint8_t*>(workspace));
  }
  void* ws = nullptr;
  if (cudaMallocAsync(&ws, need, stream) != cudaSuccess) return MALA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, kWorkspaceHeader, stream) != cudaSuccess) {
    cudaFreeAsync(ws, stream);
    return MALA_ERR_CUDA;
  }
  mala_status st = body(static_cast<uint8_t*>(ws));
  if (cudaFreeAsync(ws, stream) != cudaSuccess && st == MALA_OK) st = MALA_ERR_CUDA;
  return st;
}

// Self-test of the bounded waits: one thread waits on an mbarrier that nothing arrives
// on, so the wait runs out after `budget_ns` and records MALA_ERR_TIMEOUT in `err`.
__global__ void selftest_wait_kernel(uint32_t* err, uint64_t budget_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const AbortState st{&flag, err, budget_ns, 0xF00u};
    (void)mbar_wait(&bar, 0, st, 1);
  }
  __syncthreads();
}

}  // namespace mala

using namespace mala;

extern "C" {

int mala_version(void) { return 203; }

const char* mala_status_string(mala_status s) {
  switch (s) {
    case MALA_OK: return "ok";
    case MALA_ERR_INVALID_ARG: return "invalid argument";
    case MALA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MALA_ERR_CUDA: return "CUDA error";
    case MALA_ERR_TIMEOUT: return "device wait timed out";
    case MALA_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

mala_status mala_set_wait_budget_ns(uint64_t ns) {
  if (ns == 0) return MALA_ERR_INVALID_ARG;
  g_budget_ns = ns;
  return MALA_OK;
}

mala_status mala_set_debug(const mala_debug* dbg) {
  if (!dbg || !dbg->tile_margin) {
    t_margin = nullptr;
    t_margin_count = 0;
    return MALA_OK;
  }
  if ((reinterpret_cast<uintptr_t>(dbg->tile_margin) & 3u) != 0 || dbg->tile_margin_count == 0)
    return MALA_ERR_INVALID_ARG;
  t_margin = dbg->tile_margin;
  t_margin_count = dbg->tile_margin_count;
  return MALA_OK;
}

mala_status mala_read_device_error(const void* workspace, void* stream, uint32_t* out,
                                   int clear) {
  if (!workspace || !out) return MALA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MALA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MALA_ERR_CUDA;
  *out = v;
  if (clear && cudaMemsetAsync(const_cast<void*>(workspace), 0, 4, s) != cudaSuccess)
    return MALA_ERR_CUDA;
  return MALA_OK;
}

mala_status mala_selftest_wait_timeout(void* workspace, uint64_t budget_ns, void* stream) {
  if (!workspace || budget_ns == 0 || budget_ns > 10000000000ull) return MALA_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return MALA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* hdr = static_cast<uint32_t*>(workspace);
  if (cudaMemsetAsync(hdr + kHdrError, 0, sizeof(uint32_t), s) != cudaSuccess)
    return MALA_ERR_CUDA;
  selftest_wait_kernel<<<1, 32, 0, s>>>(hdr + kHdrError, budget_ns);
  return cudaGetLastError() == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}

mala_status mala_get_stats(const void* workspace, void* stream, mala_stats* out) {
  if (!workspace || !out) return MALA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned long long v[3] = {0, 0, 0};
  if (cudaMemcpyAsync(v, static_cast<const uint8_t*>(workspace) + kStatsOffset, sizeof(v),
                      cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MALA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MALA_ERR_CUDA;
  out->legal_tiles = v[0];
  out->retained_tiles = v[1];
  out->v_tiles_loaded = v[2];
  return MALA_OK;
}

size_t mala_fwd_workspace_bytes(int B, int H, int H_kv, int L, int d, int dtype) {
  if (!common_args_ok(B, H, H_kv, L, d, dtype, 1.f, 0.f)) return 0;
  return kWorkspaceHeader;
}

}  // extern "C"

namespace mala {
namespace {

// The forward for L query rows that are the last L of Lk key positions (Lk == L: the
// ordinary causal forward; Lk > L: a prefill chunk with causal offset Lk - L).
mala_status run_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                    int H, int H_kv, int L, int Lk, int d, int dtype, float scale, float tau,
                    unsigned flags, void* workspace, size_t workspace_bytes, uint8_t* tile_mask,
                    void* stream) {
  if (!common_args_ok(B, H, H_kv, L, d, dtype, scale, tau)) return MALA_ERR_INVALID_ARG;
  if (Lk < L) return MALA_ERR_INVALID_ARG;
  if (!Q || !K || !V || !O || !LSE) return MALA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return MALA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool screen = (tau > 0.f) || (flags & MALA_FLAG_ALWAYS_TEST);
  const int T = (L + kTile - 1) / kTile;
  const int Tk = (Lk + kTile - 1) / kTile;
  bool margin_ok = true;
  float* margin = debug_margin(static_cast<size_t>(B) * H * T * Tk, margin_ok);
  if (!margin_ok) return MALA_ERR_INVALID_ARG;
  if (dtype == MALA_FP32) {
    if (d > 128) return MALA_ERR_UNSUPPORTED;
    // this path needs no scratch; a caller's workspace only receives the call statistics
    uint8_t* ws = nullptr;
    if (workspace) {
      if (workspace_bytes < kWorkspaceHeader) return MALA_ERR_WORKSPACE;
      if (!aligned16(workspace)) return MALA_ERR_INVALID_ARG;
      ws = static_cast<uint8_t*>(workspace);
      if (cudaMemsetAsync(ws + kStatsOffset, 0, 3 * sizeof(unsigned long long), st) !=
          cudaSuccess)
        return MALA_ERR_CUDA;
    }
    if (!debug_margin_clear(margin, static_cast<size_t>(B) * H * T * Tk, st)) return MALA_ERR_CUDA;
    return fp32_fwd(static_cast<const float*>(Q), static_cast<const float*>(K),
                    static_cast<const float*>(V), static_cast<float*>(O), LSE, B, H, H_kv, L, Lk,
                    d, scale, tau, screen, ws, tile_mask, margin, st);
  }
  if (d != 64 && d != 128) return MALA_ERR_UNSUPPORTED;
  if ((long long)B * Lk > (1ll << 31) || (long long)B * H * T > (1ll << 30))
    return MALA_ERR_UNSUPPORTED;
  if (workspace && workspace_bytes < mala_fwd_workspace_bytes(B, H, H_kv, L, d, dtype))
    return MALA_ERR_WORKSPACE;
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, Q, d, H, L, B) || !make_tile_map(&tk, K, d, H_kv, Lk, B) ||
      !make_tile_map(&tv, V, d, H_kv, Lk, B))
    return MALA_ERR_CUDA;
  const size_t need = mala_fwd_workspace_bytes(B, H, H_kv, L, d, dtype);
  return with_workspace(workspace, workspace_bytes, need, st, [&](uint8_t* ws) -> mala_status {
    uint32_t* hdr = reinterpret_cast<uint32_t*>(ws);
    if (cudaMemsetAsync(hdr + kHdrSched0, 0, 3 * sizeof(uint32_t), st) != cudaSuccess ||
        cudaMemsetAsync(ws + kStatsOffset, 0, 3 * sizeof(unsigned long long), st) != cudaSuccess ||
        !debug_margin_clear(margin, static_cast<size_t>(B) * H * T * Tk, st))
      return MALA_ERR_CUDA;
    FwdParams p;
    p.B = B; p.H = H; p.Hkv = H_kv; p.L = L; p.T = T; p.G = H / H_kv;
    p.Lk = Lk; p.Tk = Tk; p.off = Lk - L;
    p.Lrows = L;
    p.vtab = nullptr;
    p.npairs = (p.G + 1) / 2;
    p.n_units = T * B * H_kv * p.npairs;
    p.scale_log2 = scale * kLog2e;
    p.log2_tau = (tau > 0.f) ? std::log2(tau) : -INFINITY;
    p.O = O; p.LSE = LSE; p.tile_mask = tile_mask;
    p.tile_margin = margin;
    p.err = hdr + kHdrError;
    p.sched = hdr + kHdrSched0;
    p.budget_ns = wait_budget_ns();
    p.stats = reinterpret_cast<unsigned long long*>(ws + kStatsOffset);
    const int grid = p.n_units < sm_count() ? p.n_units : sm_count();
    cudaError_t e = launch_fwd_bf16(tq, tk, tv, p, d, screen, grid, st);
    return e == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
  });
}

}  // namespace
}  // namespace mala

extern "C" {

mala_status mala_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                     int H, int H_kv, int L, int d, int dtype, float scale, float tau,
                     unsigned flags, void* workspace, size_t workspace_bytes,
                     uint8_t* tile_mask, void* stream) {
  return run_fwd(Q, K, V, O, LSE, B, H, H_kv, L, L, d, dtype, scale, tau, flags, workspace,
                 workspace_bytes, tile_mask, stream);
}

size_t mala_fwd_varlen_workspace_bytes(const int* cu_seqlens_q, int n_seqs, int H, int H_kv,
                                       int d, int dtype) {
  if (!cu_seqlens_q || n_seqs <= 0 || H <= 0 || H_kv <= 0 || H % H_kv || dtype != MALA_BF16 ||
      (d != 64 && d != 128))
    return 0;
  long long blocks = 0;
  for (int s = 0; s < n_seqs; ++s) {
    const int Lq = cu_seqlens_q[s + 1] - cu_seqlens_q[s];
    if (Lq < 0) return 0;
    blocks += (Lq + kTile - 1) / kTile;
  }
  return kWorkspaceHeader + static_cast<size_t>(blocks) * sizeof(VarlenBlock);
}

mala_status mala_fwd_varlen(const void* Q, const void* K, const void* V, void* O, float* LSE,
                            const int* cu_seqlens_q, const int* cu_seqlens_k, int n_seqs, int H,
                            int H_kv, int d, int dtype, float scale, float tau, unsigned flags,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (!cu_seqlens_q || !cu_seqlens_k || n_seqs <= 0) return MALA_ERR_INVALID_ARG;
  if (cu_seqlens_q[0] != 0 || cu_seqlens_k[0] != 0) return MALA_ERR_INVALID_ARG;
  std::vector<VarlenBlock> tab;
  for (int s = 0; s < n_seqs; ++s) {
    const int Lq = cu_seqlens_q[s + 1] - cu_seqlens_q[s];
    const int Lk = cu_seqlens_k[s + 1] - cu_seqlens_k[s];
    if (Lq < 0 || Lk < Lq) return MALA_ERR_INVALID_ARG;
    for (int i = 0; i < (Lq + kTile - 1) / kTile; ++i) {
      VarlenBlock e{};
      e.qrow0 = cu_seqlens_q[s];
      e.krow0 = cu_seqlens_k[s];
      e.L = Lq;
      e.off = Lk - Lq;
      e.i = i;
      tab.push_back(e);
    }
  }
  const int total_q = cu_seqlens_q[n_seqs], total_k = cu_seqlens_k[n_seqs];
  if (tab.empty()) return MALA_OK;  // no query rows: nothing to do
  if (!common_args_ok(1, H, H_kv, total_q, d, dtype, scale, tau)) return MALA_ERR_INVALID_ARG;
  if (dtype != MALA_BF16) return MALA_ERR_UNSUPPORTED;  // packed batches: tensor-core path only
  if (d != 64 && d != 128) return MALA_ERR_UNSUPPORTED;
  if (!Q || !K || !V || !O || !LSE || !workspace) return MALA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(workspace))
    return MALA_ERR_INVALID_ARG;
  const size_t need = mala_fwd_varlen_workspace_bytes(cu_seqlens_q, n_seqs, H, H_kv, d, dtype);
  if (workspace_bytes < need) return MALA_ERR_WORKSPACE;
  if (static_cast<long long>(tab.size()) * H_kv * ((H / H_kv + 1) / 2) > (1ll << 30))
    return MALA_ERR_UNSUPPORTED;  // unit count must fit the scheduler's 32-bit counter
  // heaviest first: the blocks with the most key tiles
  auto weight = [](const VarlenBlock& e) {
    return (e.off + std::min(e.i * kTile + kTile - 1, e.L - 1)) / kTile + 1;
  };
  std::stable_sort(tab.begin(), tab.end(), [&](const VarlenBlock& a, const VarlenBlock& b) {
    return weight(a) > weight(b);
  });
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool screen = (tau > 0.f) || (flags & MALA_FLAG_ALWAYS_TEST);
  CUtensorMap tq, tk, tv;
  if (!make_tile_map(&tq, Q, d, H, total_q, 1) || !make_tile_map(&tk, K, d, H_kv, total_k, 1) ||
      !make_tile_map(&tv, V, d, H_kv, total_k, 1))
    return MALA_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* hdr = reinterpret_cast<uint32_t*>(ws);
  VarlenBlock* dtab = reinterpret_cast<VarlenBlock*>(ws + kWorkspaceHeader);
  // the table comes from pageable host memory: the copy is staged before the call returns
  if (cudaMemcpyAsync(dtab, tab.data(), tab.size() * sizeof(VarlenBlock), cudaMemcpyHostToDevice,
                      st) != cudaSuccess ||
      cudaMemsetAsync(hdr + kHdrSched0, 0, 3 * sizeof(uint32_t), st) != cudaSuccess ||
      cudaMemsetAsync(ws + kStatsOffset, 0, 3 * sizeof(unsigned long long), st) != cudaSuccess)
    return MALA_ERR_CUDA;
  FwdParams p;
  p.B = 1; p.H = H; p.Hkv = H_kv; p.G = H / H_kv;
  p.L = total_q; p.T = 0; p.Lk = total_k; p.Tk = 0; p.off = 0;
  p.Lrows = total_q;
  p.vtab = dtab;
  p.npairs = (p.G + 1) / 2;
  p.n_units = static_cast<int>(tab.size()) * H_kv * p.npairs;
  p.scale_log2 = scale * kLog2e;
  p.log2_tau = (tau > 0.f) ? std::log2(tau) : -INFINITY;
  p.O = O; p.LSE = LSE; p.tile_mask = nullptr;
  p.tile_margin = nullptr;
  p.err = hdr + kHdrError;
  p.sched = hdr + kHdrSched0;
  p.budget_ns = wait_budget_ns();
  p.stats = reinterpret_cast<unsigned long long*>(ws + kStatsOffset);
  const int grid = p.n_units < sm_count() ? p.n_units : sm_count();
  return launch_fwd_bf16(tq, tk, tv, p, d, screen, grid, st) == cudaSuccess ? MALA_OK
                                                                            : MALA_ERR_CUDA;
}

mala_status mala_fwd_prefill(const void* Q, const void* K, const void* V, void* O, float* LSE,
                             int B, int H, int H_kv, int N_q, int N_k, int d, int dtype,
                             float scale, float tau, unsigned flags, void* workspace,
                             size_t workspace_bytes, uint8_t* tile_mask, void* stream) {
  if (N_k <= 0 || N_q > N_k) return MALA_ERR_INVALID_ARG;
  return run_fwd(Q, K, V, O, LSE, B, H, H_kv, N_q, N_k, d, dtype, scale, tau, flags, workspace,
                 workspace_bytes, tile_mask, stream);
}

size_t mala_bwd_workspace_bytes(int B, int H, int H_kv, int L, int d, int dtype) {
  if (!common_args_ok(B, H, H_kv, L, d, dtype, 1.f, 0.f)) return 0;
  return bwd_workspace_bytes(B, H, H_kv, L, d, dtype);
}

mala_status mala_bwd(const void* Q, const void* K, const void* V, const void* O,
                     const float* LSE, const void* dO, void* dQ, void* dK, void* dV, int B,
                     int H, int H_kv, int L, int d, int dtype, float scale, float tau,
                     unsigned flags, void* workspace, size_t workspace_bytes,
                     uint8_t* tile_mask, void* stream) {
  if (!common_args_ok(B, H, H_kv, L, d, dtype, scale, tau)) return MALA_ERR_INVALID_ARG;
  if (!Q || !K || !V || !O || !LSE || !dO || !dQ || !dK || !dV) return MALA_ERR_INVALID_ARG;
  for (const void* ptr : {Q, K, V, O, dO, static_cast<const void*>(dQ),
                          static_cast<const void*>(dK), static_cast<const void*>(dV)})
    if (!aligned16(ptr)) return MALA_ERR_INVALID_ARG;
  if (dtype == MALA_BF16 && d != 64 && d != 128) return MALA_ERR_UNSUPPORTED;
  if (dtype == MALA_FP32 && d > 128) return MALA_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t T = (static_cast<size_t>(L) + kTile - 1) / kTile;
  bool margin_ok = true;
  float* margin = debug_margin(static_cast<size_t>(B) * H * T * T, margin_ok);
  if (!margin_ok) return MALA_ERR_INVALID_ARG;
  const size_t need = bwd_workspace_bytes(B, H, H_kv, L, d, dtype);
  return with_workspace(workspace, workspace_bytes, need, st, [&](uint8_t* ws) -> mala_status {
    if (!debug_margin_clear(margin, static_cast<size_t>(B) * H * T * T, st)) return MALA_ERR_CUDA;
    return bwd_dispatch(Q, K, V, O, LSE, dO, dQ, dK, dV, B, H, H_kv, L, d, dtype, scale, tau,
                        flags, ws, tile_mask, margin, wait_budget_ns(), st);
  });
}

int mala_decode_num_splits(int B, int H, int H_kv, int Nk) {
  if (B <= 0 || H <= 0 || H_kv <= 0 || Nk <= 0 || H % H_kv) return 0;
  return decode_auto_splits(B, H_kv, Nk);
}

size_t mala_decode_workspace_bytes(int B, int H, int H_kv, int Nk, int d, int dtype,
                                   int num_splits) {
  if (!common_args_ok(B, H, H_kv, Nk, d, dtype, 1.f, 0.f)) return 0;
  if (num_splits == 0) num_splits = decode_auto_splits(B, H_kv, Nk);
  const int T = (Nk + kTile - 1) / kTile;
  if (num_splits < 1 || num_splits > T) return 0;
  return decode_workspace_bytes(B, H, H_kv, Nk, d, dtype, num_splits);
}

mala_status mala_decode(const void* q, const void* Kc, const void* Vc, void* O, float* LSE,
                        int B, int H, int H_kv, int Nk, int d, int dtype, float scale,
                        float tau, int num_splits, unsigned flags, void* workspace,
                        size_t workspace_bytes, uint8_t* tile_mask, void* stream) {
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
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  bool margin_ok = true;
  float* margin = debug_margin(static_cast<size_t>(B) * H * T, margin_ok);
  if (!margin_ok) return MALA_ERR_INVALID_ARG;
  const size_t need = decode_workspace_bytes(B, H, H_kv, Nk, d, dtype, num_splits);
  return with_workspace(workspace, workspace_bytes, need, st, [&](uint8_t* ws) -> mala_status {
    if (!debug_margin_clear(margin, static_cast<size_t>(B) * H * T, st)) return MALA_ERR_CUDA;
    return decode_dispatch(q, Kc, Vc, O, LSE, B, H, H_kv, Nk, d, dtype, scale, tau, num_splits,
                           flags, ws, tile_mask, margin, wait_budget_ns(), st);
  });
}

}  // extern "C"
