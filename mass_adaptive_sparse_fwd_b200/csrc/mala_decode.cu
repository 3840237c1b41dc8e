// MALA split-KV decode kernel for sm_100a (bf16, head dim 64 or 128).
//
// "MassAlloc Attention: Let Attention Allocate Its Own Compute", §2.1 (L_0 = N_k in
// decoding), §2.4 and A.1 (fused decoding: every cached key is scored, V is loaded and
// P.V executed only for retained tiles; each split tests against its own partial
// normaliser; the partial outputs are merged by the normaliser-aware reduction).
//
// Work unit = (batch b, KV head g, split s): the G = H / H_kv query heads of group g
// against the split's key tiles, newest first.  Persistent CTAs walk the units
// round-robin; the last CTA to finish a (b, g) merges its splits (atomic ticket).
//
// Decode is bound by HBM bandwidth: every K byte must be read, and V bytes only for
// retained tiles.  The retention decisions depend on Q and K alone, so the kernel
// decides ahead of the P.V work and gates each V load on the decision:
//   warp CW     K producer: streams K tiles of the CTA's units into a ring (TMA).
//   warp CW+1   V producer: waits for the decision of each tile and loads V only when
//               at least one head of the group retains it.
//   warps 0..CW-1  consumers (CW = 8 for d = 128, two per SM sub-partition, so one
//               warp's dependent mma / shuffle / barrier chain hides another's):
//               scores S = K_t q_g^T (mma.sync m16n8k16, heads padded to 8 as the
//               N dimension) and per-warp maxima; one barrier per tile; then every
//               warp takes the same per-head decision, lane-distributed, forms P_t
//               against its own maxima only for kept tiles, and does the P.V product
//               of tile t kLag tiles later, when its V has had time to arrive.  The
//               row sums of a tile ride on the next tile's barrier, where they close
//               its normaliser update before the next test.
// Groups of up to 4 query heads run with one head slot per decision lane, groups of
// 5..8 with two (template parameter HS).
// The contraction per tile is tiny (128 keys x 128 dims x G heads) and the kernel is
// bandwidth bound, so it uses warp-level mma.sync rather than tcgen05 / TMEM.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "mala.h"
#include "mala_common.cuh"
#include "sm100.cuh"

namespace mala {

bool make_tile_map(CUtensorMap* m, const void* base, int n0, int n1, int n2, int n3);
int sm_count();

namespace {

constexpr int kLag = 2;        // tiles between a decision and its P.V
// P / decision ring depth: P of tile n is written before tile n's barrier, while a slower
// warp may still be in the P.V of tile n - kLag - 1 (before that barrier); slot n was last
// read by the P.V of tile n - kLag - 2, which every warp finished before barrier n - 1
constexpr int kPR = kLag + 2;

template <int D>
struct DecCfg {
  static constexpr int TILE_BYTES = kTile * D * 2;
  static constexpr int BOXES = D / 64;
  // consumer warps: warp w scores keys [16 KB w, 16 KB (w+1)) of a tile and owns
  // head-dim rows [16 MB w, 16 MB (w+1)) of O^T
  static constexpr int CW = (D == 128) ? 8 : 4;
  static constexpr int KB = kTile / (16 * CW);
  static constexpr int MB = D / (16 * CW);
  static constexpr int NT = 32 * CW;            // consumer threads
  static constexpr int THREADS = NT + 64;       // + K producer warp + V producer warp
  static constexpr int NK = (D == 128) ? 3 : 6;
  static constexpr int NV = (D == 128) ? 3 : 6;
  static constexpr int SMEM = (NK + NV) * TILE_BYTES + 1024;
};

struct DecParams {
  int B, H, Hkv, Nk, T, G, S, n_units;
  float scale_log2, thr2;  // thr2 = log2(tau / N_k), -inf when tau == 0
  const __nv_bfloat16* q;  // [B, H, D]
  __nv_bfloat16* O;        // [B, H, D]
  float* LSE;              // [B, H]
  float* part_o;           // [B, H, S, D]
  float* part_z;           // [B, H, S] (natural log)
  uint32_t* tickets;       // [B * Hkv]
  uint8_t* tile_mask;      // [B, H, T] or null
  float* tile_margin;      // [B, H, T] debug margins (natural log) or null
  unsigned long long* stats;  // call statistics (kStatsOffset) or null
  uint32_t* err;
  uint64_t budget_ns;
};

struct DecShared {
  uint64_t k_full[6], k_empty[6], v_full[6], v_empty[6];
  uint64_t dec_full[kPR], dec_empty[kPR];
  __nv_bfloat16 qs[8][128];           // query rows of the group, heads >= G are zero
  // P_t in fp32, rows = heads (>= G zero), each warp's keys relative to that warp's own
  // maximum; rows padded by 8 keys (bank spread of the P.V fragment loads)
  alignas(16) float P[kPR][8][kTile + 8];
  float beta[kPR][8][8];              // [key segment][head]: 2^(segment max - new max)
  float alpha[kPR][8];                // rescale of O at tile t, per head
  uint32_t keep[kPR];                 // bit h: head h retained tile t
  // per-warp tile maxima and row sums, [warp][head], double-buffered by tile parity
  float rmax[2][8][8];
  float rsum[2][8][8];
  float mz[8], mw[8];                 // merge: per head max_s z_s and sum_s e^(z_s - max)
  uint32_t last_flag;
  uint32_t abort_flag;
};

static_assert(DecCfg<128>::SMEM + sizeof(DecShared) <= 232448, "decode smem budget");
static_assert(DecCfg<64>::SMEM + sizeof(DecShared) <= 232448, "decode smem budget");

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                            uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte address of 16-byte chunk `c` (of 8 bf16 along the head dim) of key row `r` in
// a tile loaded by TMA as D/64 boxes of [128 rows x 128 bytes] with 128-byte swizzle.
__device__ __forceinline__ uint32_t tile_chunk_addr(uint32_t base, int r, int c) {
  return base + (c >> 3) * 16384 + sw128_offset(r, c & 7);
}

// Units are numbered KV head fastest: CTAs that run side by side stream the same key
// range of all H_kv heads, i.e. whole [H_kv, d] rows of the cache, which keeps DRAM
// pages fully used (one head's keys are 2*d-byte pieces at a 2*H_kv*d-byte stride).
__device__ __forceinline__ void unit_coords(const DecParams& p, int u, int& b, int& g, int& s,
                                            int& t_lo, int& t_hi) {
  g = u % p.Hkv;
  s = (u / p.Hkv) % p.S;
  b = u / (p.Hkv * p.S);
  t_lo = static_cast<int>(static_cast<long long>(s) * p.T / p.S);
  t_hi = static_cast<int>(static_cast<long long>(s + 1) * p.T / p.S);
}

// Applies the previous tile's decision of head hd to the normaliser once that tile's
// per-warp row sums are published: l = l alpha + sum_w rowsum_w beta_w (lane (dw, hd) holds
// segment dw's beta; the 8 segment lanes of a head reduce by shuffles).  Warp-collective.
template <int CW>
__device__ __forceinline__ void close_prev(const float (&rsum)[8][8], int dw, int hd,
                                           float mnew_prev, float alpha_prev, float beta_prev,
                                           bool& k_prev, float& m_h, float& l_h) {
  const float sv = (dw < CW) ? rsum[dw][hd] : 0.f;
  float sum = k_prev ? sv * beta_prev : 0.f;
  sum += __shfl_xor_sync(0xffffffffu, sum, 1);
  sum += __shfl_xor_sync(0xffffffffu, sum, 2);
  sum += __shfl_xor_sync(0xffffffffu, sum, 4);
  if (k_prev) {
    l_h = l_h * alpha_prev + sum;
    m_h = mnew_prev;
  }
  k_prev = false;
}

// HS = head slots per decision lane: 1 for groups of up to 4 query heads, 2 for up to 8.
template <int D, bool kScreen, int HS>
__global__ void __launch_bounds__(DecCfg<D>::THREADS, 1)
    mala_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const DecParams p) {
  using C = DecCfg<D>;
  constexpr int NK = C::NK, NV = C::NV;
  constexpr int CW = C::CW, KB = C::KB, MB = C::MB, NT = C::NT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + NK * C::TILE_BYTES;
  __shared__ DecShared sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < NK; ++i) {
      mbar_init(&sh.k_full[i], 1);
      mbar_init(&sh.k_empty[i], CW);
    }
    for (int i = 0; i < NV; ++i) {
      mbar_init(&sh.v_full[i], 1);
      mbar_init(&sh.v_empty[i], CW);
    }
    for (int i = 0; i < kPR; ++i) {
      mbar_init(&sh.dec_full[i], 1);
      mbar_init(&sh.dec_empty[i], 1);
    }
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const AbortState ast{&sh.abort_flag, p.err, p.budget_ns, 0x300u};

  if (warp == CW) {
    // ------------------------------------------------------------------ K producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      uint32_t c = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
        int b, g, s, t_lo, t_hi;
        unit_coords(p, u, b, g, s, t_lo, t_hi);
        for (int t = t_hi - 1; t >= t_lo && ok; --t, ++c) {
          const int st = c % NK;
          if (c >= NK && !(ok = mbar_wait(&sh.k_empty[st], ((c / NK) - 1) & 1, ast, 1))) break;
          mbar_arrive_expect_tx(&sh.k_full[st], C::TILE_BYTES);
          for (int x = 0; x < C::BOXES; ++x)
            tma_load_4d(sK + st * C::TILE_BYTES + x * 16384, &tmK, &sh.k_full[st], x * 64, g,
                        t * kTile, b);
        }
      }
      if (!ok) {
        AbortState drain = ast;
        uint32_t zero = 0;
        drain.flag = &zero;
        drain.budget_ns = kTeardownBudgetNs;
        for (uint32_t cc = (c > NK ? c - NK : 0); cc < c; ++cc)
          mbar_wait(&sh.k_full[cc % NK], (cc / NK) & 1, drain, 2);
      }
    }
  } else if (warp == CW + 1) {
    // ------------------------------------------------------------------ V producer
    if (lane == 0) {
      tma_prefetch_desc(&tmV);
      uint32_t n = 0, c = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
        int b, g, s, t_lo, t_hi;
        unit_coords(p, u, b, g, s, t_lo, t_hi);
        for (int t = t_hi - 1; t >= t_lo && ok; --t, ++n) {
          const int slot = n % kPR;
          if (!(ok = mbar_wait(&sh.dec_full[slot], (n / kPR) & 1, ast, 3))) break;
          const uint32_t keep = sh.keep[slot];
          mbar_arrive(&sh.dec_empty[slot]);
          if (!keep) continue;
          const int st = c % NV;
          if (c >= NV && !(ok = mbar_wait(&sh.v_empty[st], ((c / NV) - 1) & 1, ast, 4))) break;
          mbar_arrive_expect_tx(&sh.v_full[st], C::TILE_BYTES);
          for (int x = 0; x < C::BOXES; ++x)
            tma_load_4d(sV + st * C::TILE_BYTES + x * 16384, &tmV, &sh.v_full[st], x * 64, g,
                        t * kTile, b);
          ++c;
        }
      }
      if (!ok) {
        AbortState drain = ast;
        uint32_t zero = 0;
        drain.flag = &zero;
        drain.budget_ns = kTeardownBudgetNs;
        for (uint32_t cc = (c > NV ? c - NV : 0); cc < c; ++cc)
          mbar_wait(&sh.v_full[cc % NV], (cc / NV) & 1, drain, 5);
      }
      stats_add(p.stats, 0, 0, c);
    }
  } else {
    // ------------------------------------------------------------------ consumers
    const int G = p.G;
    const float NEG_INF = -INFINITY;
    const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
    uint32_t kc = 0, vc = 0, n_glob = 0;
    uint32_t st_legal = 0, st_ret = 0;  // call statistics (thread 0)
    bool ok = true;
    // zero the padded heads of P once (rows >= G are never written again)
    for (int i = tid; i < kPR * 8 * (kTile + 8); i += NT) {
      const int row = (i / (kTile + 8)) % 8;
      if (row >= G) (&sh.P[0][0][0])[i] = 0.f;
    }
    // scale factors of heads without a decision (padding, or heads 4..7 of a group of at
    // most 4, whose slots are never written) stay finite: beta 0, alpha 1
    for (int i = tid; i < kPR * 8 * 8; i += NT) (&sh.beta[0][0][0])[i] = 0.f;
    for (int i = tid; i < kPR * 8; i += NT) (&sh.alpha[0][0])[i] = 1.f;
    // decision lanes: lane L of every consumer warp handles key segment (warp) dw and
    // heads dh and dh + 4 (a group has up to 8 heads); the per-head state m, l lives in
    // the lanes of that head (replicated over the 8 segment lanes, and over warps: every
    // warp takes the same decisions)
    const int dw = lane & 7, dh = lane >> 3;
    for (int u = blockIdx.x; u < p.n_units && ok; u += gridDim.x) {
      int b, g, s, t_lo, t_hi;
      unit_coords(p, u, b, g, s, t_lo, t_hi);
      const int nt = t_hi - t_lo;
      // query rows of the group -> shared, then the B fragments of S = K q^T
      named_bar_sync(1, NT);
      for (int i = tid; i < 8 * D; i += NT) {
        const int hh = i / D, c = i % D;
        sh.qs[hh][c] = (hh < G) ? p.q[(static_cast<size_t>(b) * p.H + g * G + hh) * D + c]
                                : __float2bfloat16(0.f);
      }
      named_bar_sync(1, NT);
      uint32_t qb[D / 16][2];
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        const int hh = lane >> 2, c0 = ks * 16 + (lane & 3) * 2;
        qb[ks][0] = *reinterpret_cast<const uint32_t*>(&sh.qs[hh][c0]);
        qb[ks][1] = *reinterpret_cast<const uint32_t*>(&sh.qs[hh][c0 + 8]);
      }
      // running state (online, log2 units) of heads dh and dh + 4 (slots 0 and 1), and
      // the previous tile's decision for them, applied to l once its row sums arrive
      float m_h[2] = {NEG_INF, NEG_INF}, l_h[2] = {0.f, 0.f};  // slots [0, HS) used
      bool k_prev[2] = {false, false};
      float mnew_prev[2] = {NEG_INF, NEG_INF}, alpha_prev[2] = {1.f, 1.f};
      float beta_prev[2] = {0.f, 0.f};
      float ps_prev[2] = {0.f, 0.f};  // this warp's row sums of the previous tile
      // O^T accumulators: warp owns head-dim rows [16 MB w, 16 MB (w+1))
      float acc[MB][4];
#pragma unroll
      for (int mb = 0; mb < MB; ++mb)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mb][e] = 0.f;

      for (int n = 0; n < nt + kLag && ok; ++n) {
        if (n < nt) {
          const int t = t_hi - 1 - n;
          const uint32_t slot = (n_glob + n) % kPR;
          const int kst = kc % NK;
          // A failed wait only raises the abort flag; the consumers leave the loop
          // together, right after their next named barrier.
          const bool got = mbar_wait_warp(&sh.k_full[kst], (kc / NK) & 1, ast, 10);
          // scores of this warp's keys x 8 (padded) heads
          float sc[KB][4];
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[kb][e] = 0.f;
            const int row0 = warp * (16 * KB) + kb * 16;
            if (got) {
#pragma unroll
              for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t a0, a1, a2, a3;
                ldmatrix_x4(tile_chunk_addr(sKa + kst * C::TILE_BYTES, row0 + (lane & 15),
                                            ks * 2 + (lane >> 4)),
                            a0, a1, a2, a3);
                mma_bf16(sc[kb], a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
              }
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sh.k_empty[kst]);
          ++kc;
          // log2-domain scores (keys past the end masked) and this warp's maxima: thread
          // columns are heads h0 and h0 + 1, rows are keys
          const int h0 = (lane & 3) * 2;
          float mx[2] = {NEG_INF, NEG_INF};
#pragma unroll
          for (int kb = 0; kb < KB; ++kb)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int key = t * kTile + warp * (16 * KB) + kb * 16 + (lane >> 2) + (e >> 1) * 8;
              float x = sc[kb][e] * p.scale_log2;
              x = (key < p.Nk) ? x : NEG_INF;
              sc[kb][e] = x;
              mx[e & 1] = fmaxf(mx[e & 1], x);
            }
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) {
            mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], o));
            mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xffffffffu, mx[1], o));
          }
          // the tile's only barrier publishes this tile's per-warp maxima together with
          // the previous tile's per-warp row sums; it also orders the P, beta and alpha of
          // older tiles before their P.V below
          const int rb = n & 1;
          if (lane < 2 * HS) {  // lane c holds heads 2c and 2c + 1
            sh.rmax[rb][warp][lane * 2] = mx[0];
            sh.rmax[rb][warp][lane * 2 + 1] = mx[1];
            sh.rsum[rb][warp][lane * 2] = ps_prev[0];
            sh.rsum[rb][warp][lane * 2 + 1] = ps_prev[1];
          }
          if (named_bar_or(1, NT, *ast.flag != 0)) { ok = false; break; }  // uniform exit
          #pragma unroll
          for (int hs = 0; hs < HS; ++hs)
            close_prev<CW>(sh.rsum[rb], dw, dh + 4 * hs, mnew_prev[hs], alpha_prev[hs],
                           beta_prev[hs], k_prev[hs], m_h[hs], l_h[hs]);
          // retention test (Eq. 3 with L_0 = N_k) of heads dh and dh + 4 on the tile maxima
          uint32_t keep = 0;
#pragma unroll
          for (int hs = 0; hs < HS; ++hs) {
            const int hd = dh + 4 * hs;
            const float mv = (dw < CW) ? sh.rmax[rb][dw][hd] : NEG_INF;
            float tmax = mv;
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
            tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 4));
            bool k = hd < G;
            const float cut = m_h[hs] + __log2f(l_h[hs]) + p.thr2;
            if (kScreen && k) k = (l_h[hs] == 0.f) || (tmax >= cut);
            const uint32_t bal = __ballot_sync(0xffffffffu, k);
            keep |= ((bal & 1u) | ((bal >> 7) & 2u) | ((bal >> 14) & 4u) | ((bal >> 21) & 8u))
                    << (4 * hs);
            k_prev[hs] = k;
            if (k) {  // the normaliser update itself waits for the row sums (next barrier)
              mnew_prev[hs] = m_h[hs];
              alpha_prev[hs] = 1.f;
              if (tmax > m_h[hs] + 8.0f) {
                mnew_prev[hs] = tmax;
                alpha_prev[hs] = fast_exp2(m_h[hs] - tmax);  // 0 on the first retained tile
              }
              beta_prev[hs] = fast_exp2(mv - mnew_prev[hs]);  // 0 for a segment with no key
            }
            if (warp == 0) {
              if (dw < CW) sh.beta[slot][dw][hd] = k ? beta_prev[hs] : 0.f;
              if (dw == 0) sh.alpha[slot][hd] = k ? alpha_prev[hs] : 1.f;
              if (p.tile_mask && dw == 0 && hd < G)
                p.tile_mask[(static_cast<size_t>(b) * p.H + g * G + hd) * p.T + t] = k ? 1 : 0;
              // debug: the margin of the test in natural-log units (+inf on a split's
              // first tile)
              if (kScreen && p.tile_margin && dw == 0 && hd < G)
                p.tile_margin[(static_cast<size_t>(b) * p.H + g * G + hd) * p.T + t] =
                    (l_h[hs] == 0.f) ? INFINITY : (tmax - cut) * kLn2;
            }
          }
          const uint32_t bal = keep;  // nonzero: some head keeps the tile (warp-uniform)
          // hand the decision to the V producer (ring slot must be free)
          if (tid == 0) {
            st_legal += static_cast<uint32_t>(G);
            st_ret += __popc(keep);
            bool free_slot = true;
            if (n_glob + n >= kPR)
              free_slot = mbar_wait(&sh.dec_empty[slot], (((n_glob + n) / kPR) - 1) & 1, ast, 11);
            sh.keep[slot] = keep;
            if (free_slot) mbar_arrive(&sh.dec_full[slot]);
          }
          // P of a kept tile, relative to this warp's own maxima (a head that skips the
          // tile gets beta = 0), and this warp's row sums for the next barrier
          ps_prev[0] = 0.f;
          ps_prev[1] = 0.f;
          if (bal) {
#pragma unroll
            for (int kb = 0; kb < KB; ++kb)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c = e & 1, hh = h0 + c;
                const float mu = (mx[c] == NEG_INF) ? 0.f : mx[c];
                const float pv = fast_exp2(sc[kb][e] - mu);
                ps_prev[c] += pv;
                if (hh < G)
                  sh.P[slot][hh][warp * (16 * KB) + kb * 16 + (lane >> 2) + (e >> 1) * 8] = pv;
              }
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
              ps_prev[0] += __shfl_xor_sync(0xffffffffu, ps_prev[0], o);
              ps_prev[1] += __shfl_xor_sync(0xffffffffu, ps_prev[1], o);
            }
          }
        } else if (n == nt) {
          // publish the last tile's row sums and close it; this barrier also orders its P,
          // beta, alpha and keep before the P.V that follow
          const int rb = n & 1;
          if (lane < 2 * HS) {
            sh.rsum[rb][warp][lane * 2] = ps_prev[0];
            sh.rsum[rb][warp][lane * 2 + 1] = ps_prev[1];
          }
          if (named_bar_or(1, NT, *ast.flag != 0)) { ok = false; break; }  // uniform exit
          #pragma unroll
          for (int hs = 0; hs < HS; ++hs)
            close_prev<CW>(sh.rsum[rb], dw, dh + 4 * hs, mnew_prev[hs], alpha_prev[hs],
                           beta_prev[hs], k_prev[hs], m_h[hs], l_h[hs]);
        }
        // P.V of the tile decided kLag iterations ago
        if (n >= kLag) {
          const int n2 = n - kLag;
          const uint32_t slot2 = (n_glob + n2) % kPR;
          const uint32_t keep2 = sh.keep[slot2];
          if (keep2) {
            const int vst = vc % NV;
            const bool vgot = mbar_wait_warp(&sh.v_full[vst], (vc / NV) & 1, ast, 12);
            // rescale: thread's accumulator columns are heads (lane&3)*2 + {0,1}
            const int h0 = (lane & 3) * 2;
            // (one head slot: heads 4..7 are padding, alpha 1 and beta 0)
            const float a0 = (HS == 1 && h0 >= 4) ? 1.f : sh.alpha[slot2][h0];
            const float a1 = (HS == 1 && h0 + 1 >= 4) ? 1.f : sh.alpha[slot2][h0 + 1];
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) {
              acc[mb][0] *= a0; acc[mb][1] *= a1; acc[mb][2] *= a0; acc[mb][3] *= a1;
            }
            const uint32_t vbase = sVa + vst * C::TILE_BYTES;
            const int hh = lane >> 2;  // B-fragment column (head) of this thread
#pragma unroll
            for (int ks = 0; ks < (vgot ? kTile / 16 : 0); ++ks) {
              // P of key segment ks / KB, scaled to the tile's new maximum
              const float bt = (HS == 1 && hh >= 4) ? 0.f : sh.beta[slot2][ks / KB][hh];
              const int kk = ks * 16 + (lane & 3) * 2;
              const float2 p0 = *reinterpret_cast<const float2*>(&sh.P[slot2][hh][kk]);
              const float2 p1 = *reinterpret_cast<const float2*>(&sh.P[slot2][hh][kk + 8]);
              const uint32_t b0 = pack_bf16(p0.x * bt, p0.y * bt);
              const uint32_t b1 = pack_bf16(p1.x * bt, p1.y * bt);
#pragma unroll
              for (int mb = 0; mb < MB; ++mb) {
                const int d0 = warp * (16 * MB) + mb * 16;
                const int mi = lane >> 3;
                uint32_t r0, r1, r2, r3;
                ldmatrix_x4_trans(
                    tile_chunk_addr(vbase, ks * 16 + (lane & 7) + (mi >> 1) * 8, (d0 >> 3) + (mi & 1)),
                    r0, r1, r2, r3);
                mma_bf16(acc[mb], r0, r1, r2, r3, b0, b1);
              }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.v_empty[vst]);
            ++vc;
          }
        }
      }
      if (!ok) break;
      n_glob += nt;
      if (named_bar_or(1, NT, *ast.flag != 0)) { ok = false; break; }  // uniform exit
      // this split's normalised output o_s = acc / l and z_s = (m + log2 l) ln 2
      {
        const int h0 = (lane & 3) * 2;
        // head h's state sits in slot h / 4 of lanes 8 (h % 4) .. 8 (h % 4) + 7
        const float l0a = __shfl_sync(0xffffffffu, l_h[0], (h0 & 3) * 8);
        const float l1a = __shfl_sync(0xffffffffu, l_h[1], (h0 & 3) * 8);
        const float l0b = __shfl_sync(0xffffffffu, l_h[0], ((h0 + 1) & 3) * 8);
        const float l1b = __shfl_sync(0xffffffffu, l_h[1], ((h0 + 1) & 3) * 8);
        const float la = (HS == 1 || h0 < 4) ? l0a : l1a;
        const float lb = (HS == 1 || h0 + 1 < 4) ? l0b : l1b;
#pragma unroll
        for (int mb = 0; mb < MB; ++mb)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int hh = h0 + (e & 1);
            const int dd = warp * (16 * MB) + mb * 16 + (lane >> 2) + (e >> 1) * 8;
            if (hh < G)
              p.part_o[((static_cast<size_t>(b) * p.H + g * G + hh) * p.S + s) * D + dd] =
                  acc[mb][e] / ((e & 1) ? lb : la);
          }
#pragma unroll
        for (int hs = 0; hs < HS; ++hs)
          if (warp == 0 && dw == 0 && dh + 4 * hs < G)
            p.part_z[(static_cast<size_t>(b) * p.H + g * G + dh + 4 * hs) * p.S + s] =
                (m_h[hs] + __log2f(l_h[hs])) * kLn2;
      }
      // last CTA of this (b, g) merges the splits
      named_bar_sync(1, NT);
      if (tid == 0) {
        __threadfence();
        const uint32_t prev = atomicAdd(&p.tickets[b * p.Hkv + g], 1u);
        sh.last_flag = (prev == static_cast<uint32_t>(p.S - 1)) ? 1u : 0u;
      }
      named_bar_sync(1, NT);
      if (sh.last_flag) {
        __threadfence();
        // The other CTAs' partials are read from L2 (ld.global.cg).  First one warp per
        // head: z = log sum_s e^(z_s), from lane-strided loads and shuffles.
        for (int hh = warp; hh < G; hh += CW) {
          const size_t row = static_cast<size_t>(b) * p.H + g * G + hh;
          const float* pz = p.part_z + row * p.S;
          float zmax = NEG_INF;
          for (int ss = lane; ss < p.S; ss += 32) zmax = fmaxf(zmax, __ldcg(pz + ss));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1)
            zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));
          float wsum = 0.f;
          for (int ss = lane; ss < p.S; ss += 32) wsum += __expf(__ldcg(pz + ss) - zmax);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
          if (lane == 0) {
            sh.mz[hh] = zmax;
            sh.mw[hh] = wsum;
            p.LSE[row] = zmax + __logf(wsum);
          }
        }
        named_bar_sync(1, NT);
        // then o = sum_s e^(z_s - z) o_s, one output element per thread and pass; the
        // split loop's loads are independent, so several are in flight at once
        for (int i = tid; i < G * D; i += NT) {
          const int hh = i / D, dd = i % D;
          const size_t row = static_cast<size_t>(b) * p.H + g * G + hh;
          const float* pz = p.part_z + row * p.S;
          const float* po = p.part_o + row * p.S * D + dd;
          const float zmax = sh.mz[hh];
          float o0 = 0.f, o1 = 0.f;
          int ss = 0;
          for (; ss + 8 <= p.S; ss += 8) {
            float zv[8], ov[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              zv[e] = __ldcg(pz + ss + e);
              ov[e] = __ldcg(po + static_cast<size_t>(ss + e) * D);
            }
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              o0 += __expf(zv[e] - zmax) * ov[e];
              o1 += __expf(zv[e + 1] - zmax) * ov[e + 1];
            }
          }
          for (; ss < p.S; ++ss) o0 += __expf(__ldcg(pz + ss) - zmax) * __ldcg(po + static_cast<size_t>(ss) * D);
          p.O[row * D + dd] = __float2bfloat16((o0 + o1) / sh.mw[hh]);
        }
      }
    }
    if (tid == 0) stats_add(p.stats, st_legal, st_ret, 0);
  }
  __syncthreads();
}

}  // namespace

int decode_auto_splits(int B, int Hkv, int Nk) {
  // A persistent CTA (one per SM of a 148-SM B200) takes units (b, g, split) round-robin,
  // so its time is about waves x (key tiles per split + a fixed cost per unit: the q load,
  // the pipeline fill and drain, the partial write and the ticket), the fixed cost being
  // worth about 10 tiles at the HBM rate.  One SM alone streams K and V at about 1/148 of
  // the HBM rate, so a single wave of fewer CTAs is not bandwidth-starved beyond its tile
  // count.  The last CTA of each (b, g) then merges its S partials, which adds about S / 9
  // tiles (measured: with one KV head at batch 1 the best S grows as about 3 sqrt(T)).
  // The rule takes the split count S <= T of at most two waves that minimises
  // ceil(B Hkv S / 148) (ceil(T / S) + 10) + S / 9; ties go to fewer splits.
  constexpr int kSMs = 148, kUnitCostTiles = 10, kSplitsPerMergeTile = 9;
  const int T = (Nk + kTile - 1) / kTile;
  const int bg = B * Hkv;
  int smax = (2 * kSMs) / bg;
  if (smax > T) smax = T;
  if (smax < 1) smax = 1;
  int best_s = 1;
  long long best_cost = -1;
  for (int s = 1; s <= smax; ++s) {
    const long long waves = (static_cast<long long>(bg) * s + kSMs - 1) / kSMs;
    // in units of 1/9 tile
    const long long cost =
        kSplitsPerMergeTile * waves * ((T + s - 1) / s + kUnitCostTiles) + s;
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best_s = s;
    }
  }
  return best_s;
}

size_t decode_workspace_bytes(int B, int H, int Hkv, int Nk, int d, int dtype, int S) {
  (void)Nk; (void)dtype;
  const size_t part = static_cast<size_t>(B) * H * S * (d + 1) * sizeof(float);
  const size_t tick = static_cast<size_t>(B) * Hkv * sizeof(uint32_t);
  return kWorkspaceHeader + ((part + 255) / 256) * 256 + ((tick + 255) / 256) * 256;
}

mala_status fp32_decode(const float* q, const float* K, const float* V, float* O, float* LSE,
                        int B, int H, int Hkv, int Nk, int d, float scale, float tau, int S,
                        bool screen, uint8_t* ws, uint8_t* tile_mask, float* tile_margin,
                        cudaStream_t stream);

template <int D, bool kScreen, int HS>
static cudaError_t launch_decode(const CUtensorMap& tk, const CUtensorMap& tv,
                                 const DecParams& p, int grid, cudaStream_t stream) {
  auto kern = mala_decode_kernel<D, kScreen, HS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       DecCfg<D>::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<grid, DecCfg<D>::THREADS, DecCfg<D>::SMEM, stream>>>(tk, tv, p);
  return cudaGetLastError();
}

mala_status decode_dispatch(const void* q, const void* K, const void* V, void* O, float* LSE,
                            int B, int H, int Hkv, int Nk, int d, int dtype, float scale,
                            float tau, int num_splits, unsigned flags, uint8_t* ws,
                            uint8_t* tile_mask, float* tile_margin, uint64_t budget_ns,
                            cudaStream_t stream) {
  const bool screen = (tau > 0.f) || (flags & MALA_FLAG_ALWAYS_TEST);
  if (cudaMemsetAsync(ws + kStatsOffset, 0, 3 * sizeof(unsigned long long), stream) !=
      cudaSuccess)
    return MALA_ERR_CUDA;
  if (dtype == MALA_FP32)
    return fp32_decode(static_cast<const float*>(q), static_cast<const float*>(K),
                       static_cast<const float*>(V), static_cast<float*>(O), LSE, B, H, Hkv, Nk,
                       d, scale, tau, num_splits, screen, ws, tile_mask, tile_margin, stream);
  if (H / Hkv > 8) return MALA_ERR_UNSUPPORTED;  // the kernel packs up to 8 heads per group
  CUtensorMap tk, tv;
  if (!make_tile_map(&tk, K, d, Hkv, Nk, B) || !make_tile_map(&tv, V, d, Hkv, Nk, B))
    return MALA_ERR_CUDA;
  DecParams p;
  p.B = B; p.H = H; p.Hkv = Hkv; p.Nk = Nk; p.T = (Nk + kTile - 1) / kTile; p.G = H / Hkv;
  p.S = num_splits;
  p.n_units = B * Hkv * num_splits;
  p.scale_log2 = scale * kLog2e;
  p.thr2 = (tau > 0.f) ? std::log2(tau) - std::log2(static_cast<float>(Nk)) : -INFINITY;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.O = static_cast<__nv_bfloat16*>(O);
  p.LSE = LSE;
  uint8_t* part = ws + kWorkspaceHeader;
  const size_t part_bytes = static_cast<size_t>(B) * H * num_splits * (d + 1) * sizeof(float);
  p.part_o = reinterpret_cast<float*>(part);
  p.part_z = p.part_o + static_cast<size_t>(B) * H * num_splits * d;
  p.tickets = reinterpret_cast<uint32_t*>(part + ((part_bytes + 255) / 256) * 256);
  p.tile_mask = tile_mask;
  p.tile_margin = tile_margin;
  p.stats = reinterpret_cast<unsigned long long*>(ws + kStatsOffset);
  p.err = reinterpret_cast<uint32_t*>(ws) + kHdrError;
  p.budget_ns = budget_ns;
  if (cudaMemsetAsync(p.tickets, 0, static_cast<size_t>(B) * Hkv * sizeof(uint32_t), stream) !=
      cudaSuccess)
    return MALA_ERR_CUDA;
  const int grid = p.n_units < sm_count() ? p.n_units : sm_count();
  cudaError_t e;
  const bool wide = p.G > 4;
  if (d == 128)
    e = screen ? (wide ? launch_decode<128, true, 2>(tk, tv, p, grid, stream)
                       : launch_decode<128, true, 1>(tk, tv, p, grid, stream))
               : (wide ? launch_decode<128, false, 2>(tk, tv, p, grid, stream)
                       : launch_decode<128, false, 1>(tk, tv, p, grid, stream));
  else
    e = screen ? (wide ? launch_decode<64, true, 2>(tk, tv, p, grid, stream)
                       : launch_decode<64, true, 1>(tk, tv, p, grid, stream))
               : (wide ? launch_decode<64, false, 2>(tk, tv, p, grid, stream)
                       : launch_decode<64, false, 1>(tk, tv, p, grid, stream));
  return e == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}

}  // namespace mala
