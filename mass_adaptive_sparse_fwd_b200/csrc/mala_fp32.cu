// fp32 MALA path (small problems): forward, backward and split-KV decode with fp32
// inputs and outputs and fp32 CUDA-core arithmetic (no tensor cores, so no tf32
// rounding of the scores).  Same tiling, traversal and retention rules as the bf16
// tensor-core kernels:
//   "MassAlloc Attention: Let Attention Allocate Its Own Compute", §2.2 Eq. (3) (online
//   forward test), Eq. (4) (offline backward test), §2.4 (split-KV decoding),
//   App. A Algorithms 1 and 2.
// One CTA of 128 threads works on one 128-row block; thread t owns row t of it.  The
// tile decision is a block-wide OR (__syncthreads_or), so it is uniform by construction.

#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "mala.h"
#include "mala_common.cuh"

namespace mala {

namespace {

constexpr int kF32Threads = 128;

__device__ __forceinline__ float dot_rows(const float* a, const float* b, int d) {
  float s = 0.f;
  for (int c = 0; c < d; ++c) s = fmaf(a[c], b[c], s);
  return s;
}

// log(tau / L_q) (natural log); -inf when the test is off (tau == 0).
__device__ __forceinline__ float log_thr(float tau, int Lq, bool screen) {
  if (!screen || tau == 0.f) return -INFINITY;
  return logf(tau) - logf(static_cast<float>(Lq));
}

// Forward: one CTA per (b, h, query block i); K_j, V_j staged in shared memory.  The L
// query rows are the last L of Lk key positions (row q at position off + q, off = Lk - L;
// off = 0 for the ordinary forward, > 0 for a prefill chunk).
__global__ void __launch_bounds__(kF32Threads)
    fp32_fwd_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                    const float* __restrict__ V, float* __restrict__ O, float* __restrict__ LSE,
                    int B, int H, int Hkv, int L, int Lk, int d, float scale, float tau,
                    bool screen, uint8_t* tile_mask, float* tile_margin,
                    unsigned long long* stats) {
  extern __shared__ float fsm[];
  float* sK = fsm;             // [128][d]
  float* sV = fsm + kTile * d;  // [128][d]
  const int T = (L + kTile - 1) / kTile;
  const int Tk = (Lk + kTile - 1) / kTile;
  const int off = Lk - L;
  const int i = blockIdx.x % T;
  const int h = (blockIdx.x / T) % H;
  const int b = blockIdx.x / (T * H);
  const int g = h / (H / Hkv);
  const int r = threadIdx.x;
  const int q = i * kTile + r;
  const bool valid = q < L;
  const int pos = off + q;
  float qv[128], acc[128], s[kTile];
  for (int c = 0; c < d; ++c) {
    qv[c] = valid ? Q[((static_cast<size_t>(b) * L + q) * H + h) * d + c] : 0.f;
    acc[c] = 0.f;
  }
  const float theta = log_thr(tau, pos + 1, screen);
  float m = -INFINITY, l = 0.f;
  const int j_last = (off + min(i * kTile + kTile - 1, L - 1)) / kTile;
  for (int j = j_last; j >= 0; --j) {  // diagonal first
    __syncthreads();
    for (int e = r; e < kTile * d; e += kF32Threads) {
      const int k = j * kTile + e / d, c = e % d;
      const size_t src = ((static_cast<size_t>(b) * Lk + k) * Hkv + g) * d + c;
      sK[e] = k < Lk ? K[src] : 0.f;
      sV[e] = k < Lk ? V[src] : 0.f;
    }
    __syncthreads();
    float rmax = -INFINITY;
    bool has = false;
    for (int kk = 0; kk < kTile; ++kk) {
      const int k = j * kTile + kk;
      const bool legal = valid && k <= pos;
      s[kk] = legal ? scale * dot_rows(qv, sK + kk * d, d) : -INFINITY;
      if (legal) { has = true; rmax = fmaxf(rmax, s[kk]); }
    }
    bool mine = has;
    const float x = (l > 0.f) ? rmax - m - logf(l) - theta : INFINITY;
    if (screen && has && l > 0.f) mine = x >= 0.f;
    // debug: the tile's margin, max over rows with a legal key (natural-log units)
    if (screen && has && tile_margin)
      atomic_max_f32(tile_margin + ((static_cast<size_t>(b) * H + h) * T + i) * Tk + j, x);
    const bool keep = __syncthreads_or(mine) != 0;
    if (r == 0) {
      stats_add(stats, 1, keep ? 1 : 0, 0);
      if (tile_mask) tile_mask[((static_cast<size_t>(b) * H + h) * T + i) * Tk + j] = keep ? 1 : 0;
    }
    if (!keep || !has) continue;
    const float mn = fmaxf(m, rmax);
    const float alpha = expf(m - mn);
    float psum = 0.f;
    for (int c = 0; c < d; ++c) acc[c] *= alpha;
    for (int kk = 0; kk < kTile; ++kk) {
      if (s[kk] == -INFINITY) continue;
      const float p = expf(s[kk] - mn);
      psum += p;
      for (int c = 0; c < d; ++c) acc[c] = fmaf(p, sV[kk * d + c], acc[c]);
    }
    l = l * alpha + psum;
    m = mn;
  }
  if (valid) {
    for (int c = 0; c < d; ++c) O[((static_cast<size_t>(b) * L + q) * H + h) * d + c] = acc[c] / l;
    LSE[(static_cast<size_t>(b) * H + h) * L + q] = m + logf(l);
  }
}

// D_q = <O_q, dO_q>, one thread per (b, q, h) row.
__global__ void fp32_dsum_kernel(const float* __restrict__ O, const float* __restrict__ dO,
                                 float* __restrict__ Dsum, int B, int L, int H, int d) {
  const long long row = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (row >= static_cast<long long>(B) * L * H) return;
  const int h = static_cast<int>(row % H);
  const int q = static_cast<int>((row / H) % L);
  const int b = static_cast<int>(row / (static_cast<long long>(H) * L));
  Dsum[(static_cast<size_t>(b) * H + h) * L + q] = dot_rows(O + row * d, dO + row * d, d);
}

// Backward, key-major pass: one CTA per (b, KV head g, key block j); thread = key row.
// Produces dK, dV and the tile decisions.
__global__ void __launch_bounds__(kF32Threads)
    fp32_bwd_kv_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                       const float* __restrict__ V, const float* __restrict__ LSE,
                       const float* __restrict__ dO, const float* __restrict__ Dsum,
                       float* __restrict__ dK, float* __restrict__ dV, int B, int H, int Hkv,
                       int L, int d, float scale, float tau, bool screen, uint8_t* tile_mask,
                       float* tile_margin, unsigned long long* stats) {
  extern __shared__ float fsm[];
  float* sQ = fsm;               // [128][d]
  float* sdO = fsm + kTile * d;  // [128][d]
  float* sL = sdO + kTile * d;   // [128] LSE
  float* sD = sL + kTile;        // [128] D
  float* sT = sD + kTile;        // [128] log(tau / L_q)
  const int T = (L + kTile - 1) / kTile;
  const int G = H / Hkv;
  const int j = blockIdx.x % T;
  const int g = (blockIdx.x / T) % Hkv;
  const int b = blockIdx.x / (T * Hkv);
  const int r = threadIdx.x;
  const int k = j * kTile + r;
  const bool kvalid = k < L;
  float kv[128], vv[128], gk[128], gv[128];
  for (int c = 0; c < d; ++c) {
    const size_t src = ((static_cast<size_t>(b) * L + k) * Hkv + g) * d + c;
    kv[c] = kvalid ? K[src] : 0.f;
    vv[c] = kvalid ? V[src] : 0.f;
    gk[c] = gv[c] = 0.f;
  }
  for (int h = g * G; h < (g + 1) * G; ++h) {
    for (int i = j; i < T; ++i) {  // query blocks ascending from the diagonal
      __syncthreads();
      for (int e = r; e < kTile * d; e += kF32Threads) {
        const int q = i * kTile + e / d, c = e % d;
        const size_t src = ((static_cast<size_t>(b) * L + q) * H + h) * d + c;
        sQ[e] = q < L ? Q[src] : 0.f;
        sdO[e] = q < L ? dO[src] : 0.f;
      }
      {
        const int q = i * kTile + r;
        const size_t li = (static_cast<size_t>(b) * H + h) * L + q;
        sL[r] = q < L ? LSE[li] : 0.f;
        sD[r] = q < L ? Dsum[li] : 0.f;
        sT[r] = log_thr(tau, q + 1, screen);
      }
      __syncthreads();
      bool mine = false;
      float ymax = -INFINITY;  // this key's largest log P - log(tau / L_q) in the tile
      for (int qq = 0; qq < kTile; ++qq) {
        const int q = i * kTile + qq;
        if (!kvalid || q >= L || q < k) continue;
        const float s = scale * dot_rows(sQ + qq * d, kv, d);
        const float y = s - sL[qq] - sT[qq];
        ymax = fmaxf(ymax, y);
        if (!screen || y >= 0.f) mine = true;
      }
      if (screen && tile_margin && ymax != -INFINITY)
        atomic_max_f32(tile_margin + ((static_cast<size_t>(b) * H + h) * T + i) * T + j, ymax);
      const bool keep = __syncthreads_or(mine) != 0;
      if (r == 0) {
        stats_add(stats, 1, keep ? 1 : 0, 0);
        if (tile_mask) tile_mask[((static_cast<size_t>(b) * H + h) * T + i) * T + j] = keep ? 1 : 0;
      }
      if (!keep || !kvalid) continue;
      for (int qq = 0; qq < kTile; ++qq) {
        const int q = i * kTile + qq;
        if (q >= L || q < k) continue;
        const float s = scale * dot_rows(sQ + qq * d, kv, d);
        const float p = expf(s - sL[qq]);
        const float dp = dot_rows(sdO + qq * d, vv, d);
        const float ds = p * (dp - sD[qq]);
        for (int c = 0; c < d; ++c) {
          gv[c] = fmaf(p, sdO[qq * d + c], gv[c]);
          gk[c] = fmaf(scale * ds, sQ[qq * d + c], gk[c]);
        }
      }
    }
  }
  if (kvalid)
    for (int c = 0; c < d; ++c) {
      const size_t dst = ((static_cast<size_t>(b) * L + k) * Hkv + g) * d + c;
      dK[dst] = gk[c];
      dV[dst] = gv[c];
    }
}

// Backward, query-major pass: one CTA per (b, h, query block i); thread = query row.
// Re-evaluates the same tile test (identical fp32 score arithmetic) and forms dQ.
__global__ void __launch_bounds__(kF32Threads)
    fp32_bwd_q_kernel(const float* __restrict__ Q, const float* __restrict__ K,
                      const float* __restrict__ V, const float* __restrict__ LSE,
                      const float* __restrict__ dO, const float* __restrict__ Dsum,
                      float* __restrict__ dQ, int B, int H, int Hkv, int L, int d, float scale,
                      float tau, bool screen) {
  extern __shared__ float fsm[];
  float* sK = fsm;             // [128][d]
  float* sV = fsm + kTile * d;  // [128][d]
  const int T = (L + kTile - 1) / kTile;
  const int i = blockIdx.x % T;
  const int h = (blockIdx.x / T) % H;
  const int b = blockIdx.x / (T * H);
  const int g = h / (H / Hkv);
  const int r = threadIdx.x;
  const int q = i * kTile + r;
  const bool valid = q < L;
  float qv[128], gv[128], gq[128];
  for (int c = 0; c < d; ++c) {
    const size_t src = ((static_cast<size_t>(b) * L + q) * H + h) * d + c;
    qv[c] = valid ? Q[src] : 0.f;
    gv[c] = valid ? dO[src] : 0.f;
    gq[c] = 0.f;
  }
  const size_t li = (static_cast<size_t>(b) * H + h) * L + q;
  const float lse = valid ? LSE[li] : 0.f;
  const float Dq = valid ? Dsum[li] : 0.f;
  const float theta = log_thr(tau, q + 1, screen);
  for (int j = 0; j <= i; ++j) {
    __syncthreads();
    for (int e = r; e < kTile * d; e += kF32Threads) {
      const int k = j * kTile + e / d, c = e % d;
      const size_t src = ((static_cast<size_t>(b) * L + k) * Hkv + g) * d + c;
      sK[e] = k < L ? K[src] : 0.f;
      sV[e] = k < L ? V[src] : 0.f;
    }
    __syncthreads();
    bool mine = false;
    for (int kk = 0; kk < kTile; ++kk) {
      const int k = j * kTile + kk;
      if (!valid || k > q) continue;
      const float s = scale * dot_rows(qv, sK + kk * d, d);
      if (!screen || s - lse - theta >= 0.f) mine = true;
    }
    if (!__syncthreads_or(mine) || !valid) continue;
    for (int kk = 0; kk < kTile; ++kk) {
      const int k = j * kTile + kk;
      if (k > q) continue;
      const float s = scale * dot_rows(qv, sK + kk * d, d);
      const float p = expf(s - lse);
      const float dp = dot_rows(gv, sV + kk * d, d);
      const float ds = p * (dp - Dq);
      for (int c = 0; c < d; ++c) gq[c] = fmaf(scale * ds, sK[kk * d + c], gq[c]);
    }
  }
  if (valid)
    for (int c = 0; c < d; ++c) dQ[((static_cast<size_t>(b) * L + q) * H + h) * d + c] = gq[c];
}

// Decode: one CTA per (b, h, split); thread = key of the current tile.
__global__ void __launch_bounds__(kF32Threads)
    fp32_decode_split_kernel(const float* __restrict__ q, const float* __restrict__ K,
                             const float* __restrict__ V, float* __restrict__ part_o,
                             float* __restrict__ part_z, int B, int H, int Hkv, int Nk, int d,
                             int S, float scale, float tau, bool screen, uint8_t* tile_mask,
                             float* tile_margin, unsigned long long* stats) {
  __shared__ float sq[128], sp[kTile], red[kTile];
  const int T = (Nk + kTile - 1) / kTile;
  const int s = blockIdx.x % S;
  const int h = (blockIdx.x / S) % H;
  const int b = blockIdx.x / (S * H);
  const int g = h / (H / Hkv);
  const int r = threadIdx.x;
  if (r < d) sq[r] = q[(static_cast<size_t>(b) * H + h) * d + r];
  __syncthreads();
  const int t_lo = static_cast<int>(static_cast<long long>(s) * T / S);
  const int t_hi = static_cast<int>(static_cast<long long>(s + 1) * T / S);
  const float theta = log_thr(tau, Nk, screen);
  float m = -INFINITY, l = 0.f, acc = 0.f;  // acc: head-dim column r (r < d)
  for (int t = t_hi - 1; t >= t_lo; --t) {
    const int k = t * kTile + r;
    const bool kv = k < Nk;
    float sc = -INFINITY;
    if (kv) sc = scale * dot_rows(sq, K + ((static_cast<size_t>(b) * Nk + k) * Hkv + g) * d, d);
    red[r] = sc;
    __syncthreads();
    for (int o = kTile / 2; o > 0; o >>= 1) {
      if (r < o) red[r] = fmaxf(red[r], red[r + o]);
      __syncthreads();
    }
    const float rmax = red[0];
    __syncthreads();
    bool keep = true;
    const float x = (l > 0.f) ? rmax - m - logf(l) - theta : INFINITY;
    if (screen && l > 0.f) keep = x >= 0.f;
    if (r == 0 && screen && tile_margin)
      tile_margin[(static_cast<size_t>(b) * H + h) * T + t] = x;  // debug margin
    if (r == 0) {
      // this path loads V per head: one V tile per retained (head, tile)
      stats_add(stats, 1, keep ? 1 : 0, keep ? 1 : 0);
      if (tile_mask) tile_mask[(static_cast<size_t>(b) * H + h) * T + t] = keep ? 1 : 0;
    }
    if (!keep) continue;  // uniform: every thread computed the same values
    const float mn = fmaxf(m, rmax);
    const float alpha = expf(m - mn);
    const float p = kv ? expf(sc - mn) : 0.f;
    sp[r] = p;
    red[r] = p;
    __syncthreads();
    for (int o = kTile / 2; o > 0; o >>= 1) {
      if (r < o) red[r] += red[r + o];
      __syncthreads();
    }
    const float psum = red[0];
    if (r < d) {
      acc *= alpha;
      for (int kk = 0; kk < kTile; ++kk) {
        const int kx = t * kTile + kk;
        if (kx < Nk) acc = fmaf(sp[kk], V[((static_cast<size_t>(b) * Nk + kx) * Hkv + g) * d + r], acc);
      }
    }
    l = l * alpha + psum;
    m = mn;
    __syncthreads();
  }
  const size_t row = (static_cast<size_t>(b) * H + h) * S + s;
  if (r < d) part_o[row * d + r] = acc / l;
  if (r == 0) part_z[row] = m + logf(l);
}

__global__ void fp32_decode_merge_kernel(const float* __restrict__ part_o,
                                         const float* __restrict__ part_z,
                                         float* __restrict__ O, float* __restrict__ LSE, int BH,
                                         int S, int d) {
  const int row = blockIdx.x;
  const int c = threadIdx.x;
  if (row >= BH) return;
  float zmax = -INFINITY;
  for (int s = 0; s < S; ++s) zmax = fmaxf(zmax, part_z[row * S + s]);
  float w = 0.f, o = 0.f;
  for (int s = 0; s < S; ++s) {
    const float e = expf(part_z[row * S + s] - zmax);
    w += e;
    if (c < d) o += e * part_o[(static_cast<size_t>(row) * S + s) * d + c];
  }
  if (c < d) O[static_cast<size_t>(row) * d + c] = o / w;
  if (c == 0) LSE[row] = zmax + logf(w);
}

cudaError_t set_smem(const void* fn, int bytes) {
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

mala_status fp32_fwd(const float* Q, const float* K, const float* V, float* O, float* LSE, int B,
                     int H, int Hkv, int L, int Lk, int d, float scale, float tau, bool screen,
                     uint8_t* ws, uint8_t* tile_mask, float* tile_margin, cudaStream_t stream) {
  const int T = (L + kTile - 1) / kTile;
  const int smem = 2 * kTile * d * static_cast<int>(sizeof(float));
  unsigned long long* stats =
      ws ? reinterpret_cast<unsigned long long*>(ws + kStatsOffset) : nullptr;
  if (set_smem(reinterpret_cast<const void*>(fp32_fwd_kernel), smem) != cudaSuccess)
    return MALA_ERR_CUDA;
  fp32_fwd_kernel<<<B * H * T, kF32Threads, smem, stream>>>(
      Q, K, V, O, LSE, B, H, Hkv, L, Lk, d, scale, tau, screen, tile_mask, tile_margin, stats);
  return cudaGetLastError() == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}

mala_status fp32_bwd(const float* Q, const float* K, const float* V, const float* O,
                     const float* LSE, const float* dO, float* dQ, float* dK, float* dV, int B,
                     int H, int Hkv, int L, int d, float scale, float tau, bool screen,
                     uint8_t* ws, uint8_t* tile_mask, float* tile_margin, cudaStream_t stream) {
  const int T = (L + kTile - 1) / kTile;
  float* Dsum = reinterpret_cast<float*>(ws + kWorkspaceHeader);
  const long long rows = static_cast<long long>(B) * L * H;
  fp32_dsum_kernel<<<static_cast<unsigned>((rows + 127) / 128), 128, 0, stream>>>(O, dO, Dsum, B,
                                                                                  L, H, d);
  const int smem_kv = (2 * kTile * d + 3 * kTile) * static_cast<int>(sizeof(float));
  const int smem_q = 2 * kTile * d * static_cast<int>(sizeof(float));
  if (set_smem(reinterpret_cast<const void*>(fp32_bwd_kv_kernel), smem_kv) != cudaSuccess ||
      set_smem(reinterpret_cast<const void*>(fp32_bwd_q_kernel), smem_q) != cudaSuccess)
    return MALA_ERR_CUDA;
  fp32_bwd_kv_kernel<<<B * Hkv * T, kF32Threads, smem_kv, stream>>>(
      Q, K, V, LSE, dO, Dsum, dK, dV, B, H, Hkv, L, d, scale, tau, screen, tile_mask, tile_margin,
      reinterpret_cast<unsigned long long*>(ws + kStatsOffset));
  fp32_bwd_q_kernel<<<B * H * T, kF32Threads, smem_q, stream>>>(Q, K, V, LSE, dO, Dsum, dQ, B, H,
                                                                Hkv, L, d, scale, tau, screen);
  return cudaGetLastError() == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}

mala_status fp32_decode(const float* q, const float* K, const float* V, float* O, float* LSE,
                        int B, int H, int Hkv, int Nk, int d, float scale, float tau, int S,
                        bool screen, uint8_t* ws, uint8_t* tile_mask, float* tile_margin,
                        cudaStream_t stream) {
  float* part_o = reinterpret_cast<float*>(ws + kWorkspaceHeader);
  float* part_z = part_o + static_cast<size_t>(B) * H * S * d;
  fp32_decode_split_kernel<<<B * H * S, kF32Threads, 0, stream>>>(
      q, K, V, part_o, part_z, B, H, Hkv, Nk, d, S, scale, tau, screen, tile_mask, tile_margin,
      reinterpret_cast<unsigned long long*>(ws + kStatsOffset));
  fp32_decode_merge_kernel<<<B * H, 128, 0, stream>>>(part_o, part_z, O, LSE, B * H, S, d);
  return cudaGetLastError() == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}

}  // namespace mala
