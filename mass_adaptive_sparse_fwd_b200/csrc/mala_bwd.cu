// MALA backward for sm_100a (bf16, head dim 64 or 128).
//
// "MassAlloc Attention: Let Attention Allocate Its Own Compute", §2.2 (offline sparse
// probability, Eq. (4)), App. A Algorithm 2 and A.1 (fused backward execution).
//
// Three launches:
//   1. mala_bwd_prep:  D_q = rowsum(O_q * dO_q) (fp32) and zeroing of the fp32 dQ
//                      accumulator (the softmax-backward term of Algorithm 2).
//   2. mala_bwd_kernel (below): key-major, one persistent CTA per SM pulling units
//                      (b, KV head g, key block j, head part), KV head slowest and
//                      heaviest first (small j) within a head, so that the CTAs running
//                      together share one group's Q, dO and dQ accumulator in L2;
//                      within a unit the part's query heads of the group and the query
//                      blocks i = j, j+1, ... are visited in ascending order (A.1).
//   3. mala_bwd_dq:    dQ = bf16(dQ accumulator) (and dK, dV likewise when split).
//
// Head parts: a unit normally carries all G query heads of its KV head and stores dK_j
// and dV_j itself.  When a problem has few units (few KV heads and short sequences: the
// j = 0 unit holds G T tiles and alone sets the kernel's length), the G heads are split
// into P parts (P a power of two dividing G, chosen from the shape alone); each part's
// unit adds its dK_j / dV_j share into fp32 accumulators, converted to bf16 at the end.
//
// Per tile (key block j, query block i of head h) the score tile S^T = K_j Q_i^T is
// always recomputed.  The offline test of Eq. (4): the tile is retained iff some legal
// entry has s_kq * scale - LSE_q >= log(tau / L_q) (L_q = q + 1), evaluated in log2
// units.  Only a retained tile runs the post-score work:
//   P^T = exp(S^T - LSE),  dP^T = V_j dO_i^T,  dS^T = P^T o (dP^T - D),
//   dV += P^T dO_i,  dK += scale dS^T Q_i,  dQ_i += scale dS K_j  (fp32 reduction into
//   global; the scale is applied when dK is stored and when dQ is converted).
//
// Warp roles (512 threads):
//   warp 0       TMA producer: K_j and V_j once per unit; Q_i (2-stage ring) and dO_i
//                (1 stage) per tile.  dO is fetched ahead of the decision, like V in the
//                forward.
//   warp 1       TMEM owner and UMMA issuer.
//   warps 4-11   two softmax warpgroups: thread = key row (TMEM lane); warpgroup w
//                owns query columns [64 w, 64 w + 64).  They evaluate the test (one
//                bar.red.or over both groups), write P^T into TMEM and dS^T into shared
//                memory.
//   warps 12-15  dQ drain and the per-unit dK / dV epilogue.  The dQ tile is copied
//                from TMEM into a 128-byte-swizzled fp32 staging buffer (64 columns at a
//                time) and added into the global fp32 accumulator with TMA bulk
//                reductions (cp.reduce.async.bulk.tensor .add); its TMEM columns are
//                released as soon as they have been read.
// TMEM columns: S^T [0,128) (P^T bf16 overwrites [0,64)), dP^T [128,256) (the dQ tile
// of the same step overwrites it once dS^T has been formed), dV [256, 256+D),
// dK [256+D, 256+2D).

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

constexpr int kBwdThreads = 512;

template <int D>
struct BwdCfg {
  static constexpr int TILE_BYTES = kTile * D * 2;
  static constexpr int BOXES = D / 64;
  static constexpr int NQ = 2;  // Q ring stages (dO has one)
  static constexpr int STAGE_BYTES = 2 * 16384;  // dQ staging: two [128 x 32] fp32 boxes
  // K, V, NQ x Q, dO, dS^T (128 x 128 bf16), dQ staging
  static constexpr int SMEM =
      2 * TILE_BYTES + NQ * TILE_BYTES + TILE_BYTES + kTile * kTile * 2 + STAGE_BYTES;
};

struct BwdParams {
  int B, H, Hkv, L, T, G, n_units;
  int P, Gp;             // head parts per (b, g, j) and query heads per part (G = P Gp)
  float scale, scale_log2, log2_tau;
  const float* LSE;      // [B, H, L] natural log
  const float* Dsum;     // [B, H, L]
  float* dQacc;          // [B, L, H, D] fp32
  __nv_bfloat16* dK;     // [B, L, Hkv, D]
  __nv_bfloat16* dV;
  float* dKacc;          // [B, L, Hkv, D] fp32 accumulators when P > 1 (scaled), else null
  float* dVacc;
  uint8_t* tile_mask;    // [B, H, T, T] or null
  float* tile_margin;    // [B, H, T, T] debug margins (natural log) or null
  unsigned long long* stats;  // call statistics (kStatsOffset) or null
  uint32_t* err;
  uint32_t* sched;
  uint64_t budget_ns;
};

struct BwdShared {
  uint64_t kv_full, kv_empty;
  uint64_t q_full[2], q_empty[2];
  uint64_t do_full, do_empty;
  uint64_t s_full, p_full, dp_full, ds_full, dq_full, dq_empty, acc_full, acc_empty;
  uint64_t sched_full[2], sched_empty[2];
  uint64_t final_bar;
  // per softmax warpgroup and query column: LSE_q in log2 units (+inf past L, so the
  // probability is 0 there), the threshold log2(tau / L_q) and D_q
  alignas(16) float lse2[2][64];
  alignas(16) float cut2[2][64];  // LSE2_q + log2(tau / L_q): the screen's cut
  alignas(16) float dsum[2][64];
  int sched_ring[2];
  uint32_t dec;      // decision of the current tile (1 = retained)
  uint32_t abort_seen[2];  // the abort flag as seen before a tile's vote (by tile parity)
  uint32_t dq_flag[2];
  uint32_t acc_valid;  // the unit retained at least one tile (dK / dV were written)
  uint32_t tmem_base;
  uint32_t abort_flag;
};

// dynamic + static shared memory must fit the 227 KB per-block limit of sm_100
static_assert(BwdCfg<128>::SMEM + sizeof(BwdShared) <= 232448, "backward smem budget");
static_assert(BwdCfg<64>::SMEM + sizeof(BwdShared) <= 232448, "backward smem budget");

struct BUnit {
  int b, g, j, part, ntiles;  // tiles = Gp heads x (T - j) query blocks
};

__device__ __forceinline__ BUnit decode_bunit(const BwdParams& p, int u) {
  BUnit w;
  // KV head slowest, heaviest first (small j) within a head
  const int nbp = p.B * p.P;
  const int upg = nbp * p.T;
  w.g = u / upg;
  const int r = u % upg;
  w.j = r / nbp;
  w.b = (r % nbp) / p.P;
  w.part = r % p.P;
  w.ntiles = p.Gp * (p.T - w.j);
  return w;
}

// tile n of a unit -> (head h, query block i)
__device__ __forceinline__ void tile_hi(const BwdParams& p, const BUnit& w, int n, int& h,
                                        int& i) {
  const int per = p.T - w.j;
  h = w.g * p.G + w.part * p.Gp + n / per;
  i = w.j + n % per;
}

template <int D, bool kScreen>
__global__ void __launch_bounds__(kBwdThreads, 1)
    mala_bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmdQ, const BwdParams p) {
  using C = BwdCfg<D>;
  constexpr int NQ = C::NQ;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint8_t* sK = smem;
  uint8_t* sV = sK + C::TILE_BYTES;
  uint8_t* sQ = sV + C::TILE_BYTES;                 // NQ tiles
  uint8_t* sdO = sQ + NQ * C::TILE_BYTES;           // 1 tile
  uint8_t* sdS = sdO + C::TILE_BYTES;               // 128 x 128 bf16, two 64-column atoms
  uint8_t* sdQ = sdS + kTile * kTile * 2;           // dQ staging, two [128 x 32] fp32 boxes
  __shared__ BwdShared sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // the 128-byte-swizzled operand tiles need 1024-byte aligned shared memory
  if (smem_u32(smem) & 1023u) {
    if (tid == 0 && p.err) atomicCAS(p.err, 0u, static_cast<uint32_t>(MALA_ERR_UNSUPPORTED));
    return;
  }
  if (tid == 0) {
    mbar_init(&sh.kv_full, 1);
    mbar_init(&sh.kv_empty, 1);
    for (int s = 0; s < NQ; ++s) {
      mbar_init(&sh.q_full[s], 1);
      mbar_init(&sh.q_empty[s], 1);
    }
    mbar_init(&sh.do_full, 1);
    mbar_init(&sh.do_empty, 1);
    mbar_init(&sh.s_full, 1);
    mbar_init(&sh.p_full, 8);   // one arrival per softmax warp
    mbar_init(&sh.dp_full, 1);
    mbar_init(&sh.ds_full, 8);
    mbar_init(&sh.dq_full, 1);
    mbar_init(&sh.dq_empty, 4);  // one arrival per drain warp
    mbar_init(&sh.acc_full, 1);
    mbar_init(&sh.acc_empty, 128);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sh.sched_full[s], 1);
      mbar_init(&sh.sched_empty[s], 1 + 256 + 128);
    }
    mbar_init(&sh.final_bar, 1);
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tb = sh.tmem_base;
  const uint32_t tS = tb, tdP = tb + 128, tdV = tb + 256, tdK = tb + 256 + D;
  const AbortState ast{&sh.abort_flag, p.err, p.budget_ns, 0x200u};

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmdO);
      tma_prefetch_desc(&tmdQ);
      uint32_t c = 0, nu = 0, ndo = 0;
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int ring = k & 1;
        if (k >= 2 && !(ok = mbar_wait(&sh.sched_empty[ring], ((k >> 1) - 1) & 1, ast, 1))) break;
        const int u = static_cast<int>(atomicAdd(p.sched, 1u));
        sh.sched_ring[ring] = u;
        mbar_arrive(&sh.sched_full[ring]);
        if (u >= p.n_units) break;
        const BUnit w = decode_bunit(p, u);
        if (nu > 0 && !(ok = mbar_wait(&sh.kv_empty, (nu - 1) & 1, ast, 2))) break;
        mbar_arrive_expect_tx(&sh.kv_full, 2 * C::TILE_BYTES);
        for (int x = 0; x < C::BOXES; ++x) {
          tma_load_4d(sK + x * 16384, &tmK, &sh.kv_full, x * 64, w.g, w.j * kTile, w.b);
          tma_load_4d(sV + x * 16384, &tmV, &sh.kv_full, x * 64, w.g, w.j * kTile, w.b);
        }
        ++nu;
        for (int n = 0; n < w.ntiles && ok; ++n, ++c) {
          int h, i;
          tile_hi(p, w, n, h, i);
          const int st = c % NQ;
          if (c >= NQ && !(ok = mbar_wait(&sh.q_empty[st], ((c / NQ) - 1) & 1, ast, 3))) break;
          mbar_arrive_expect_tx(&sh.q_full[st], C::TILE_BYTES);
          for (int x = 0; x < C::BOXES; ++x)
            tma_load_4d(sQ + st * C::TILE_BYTES + x * 16384, &tmQ, &sh.q_full[st], x * 64, h,
                        i * kTile, w.b);
          // dO has a single stage: released by the MMA once dP^T and dV of tile c-1 are done
          if (c >= 1 && !(ok = mbar_wait(&sh.do_empty, (c - 1) & 1, ast, 5))) break;
          mbar_arrive_expect_tx(&sh.do_full, C::TILE_BYTES);
          for (int x = 0; x < C::BOXES; ++x)
            tma_load_4d(sdO + x * 16384, &tmdO, &sh.do_full, x * 64, h, i * kTile, w.b);
          ndo = c + 1;
        }
      }
      if (!ok) {
        AbortState drain = ast;
        uint32_t zero = 0;
        drain.flag = &zero;
        drain.budget_ns = kTeardownBudgetNs;
        if (nu > 0) mbar_wait(&sh.kv_full, (nu - 1) & 1, drain, 4);
        for (uint32_t cc = (c > NQ ? c - NQ : 0); cc < c; ++cc)
          mbar_wait(&sh.q_full[cc % NQ], (cc / NQ) & 1, drain, 4);
        if (ndo > 0) mbar_wait(&sh.do_full, (ndo - 1) & 1, drain, 4);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16(128, 128, 0, 0);    // S^T, dP^T
      constexpr uint32_t id_acc = idesc_bf16(128, D, 0, 1);    // dV (TS), dK (SS)
      constexpr uint32_t id_dq = idesc_bf16(128, D, 1, 1);     // dQ = dS K_j
      const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), adS = smem_u32(sdS);
      uint32_t c = 0, nu = 0, ntile = 0, nret = 0;  // tiles / retained tiles (all units)
      bool acc_waited = true;  // acc_empty of the previous unit already observed
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int ring = k & 1;
        if (!(ok = mbar_wait(&sh.sched_full[ring], (k >> 1) & 1, ast, 10))) break;
        const int u = sh.sched_ring[ring];
        mbar_arrive(&sh.sched_empty[ring]);
        if (u >= p.n_units) break;
        const BUnit w = decode_bunit(p, u);
        if (!(ok = mbar_wait(&sh.kv_full, nu & 1, ast, 11))) break;
        bool acc_started = false;
        acc_waited = (nu == 0);
        auto issue_s = [&](uint32_t cc) {
          const uint32_t aQ = smem_u32(sQ + (cc % NQ) * C::TILE_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_ss(tS, sdesc_sw128(aK + off, 16, 1024), sdesc_sw128(aQ + off, 16, 1024), id_s,
                    kk > 0);
          }
          umma_commit(&sh.s_full);
        };
        // prologue: S^T of the first tile
        if (!(ok = mbar_wait(&sh.q_full[c % NQ], (c / NQ) & 1, ast, 12))) break;
        tc_fence_after();
        issue_s(c);
        for (int n = 0; n < w.ntiles && ok; ++n, ++c, ++ntile) {
          const int st = c % NQ;
          const uint32_t aQ = smem_u32(sQ + st * C::TILE_BYTES);
          const uint32_t adO = smem_u32(sdO);
          if (!(ok = mbar_wait(&sh.p_full, ntile & 1, ast, 13))) break;
          tc_fence_after();
          const bool keep = sh.dec != 0;
          if (!keep) {
            // Skipped tile: its Q stage was read only by its own S^T MMA, which completed
            // before the decision, and its dO by no MMA, so both stages go back at once
            // with plain arrivals (no tensor-core work of this tile is pending on them);
            // dO is released before the next S^T issue so the single-stage dO ring's next
            // load starts as early as possible.
            mbar_arrive(&sh.q_empty[st]);
            // the dO load of this tile must have landed before its stage is handed back
            if (!(ok = mbar_wait(&sh.do_full, c & 1, ast, 20))) break;
            mbar_arrive(&sh.do_empty);
            if (n + 1 < w.ntiles) {
              const uint32_t c1 = c + 1;
              if (!(ok = mbar_wait(&sh.q_full[c1 % NQ], (c1 / NQ) & 1, ast, 16))) break;
              tc_fence_after();
              issue_s(c1);
            }
          } else {
            if (!(ok = mbar_wait(&sh.do_full, c & 1, ast, 20))) break;
            // dP^T reuses the columns of the previous dQ tile: wait for its drain
            if (ntile > 0 && !(ok = mbar_wait(&sh.dq_empty, (ntile - 1) & 1, ast, 14))) break;
            // first accumulation of the unit overwrites dK / dV: previous epilogue done
            if (!acc_waited && !(ok = acc_waited = mbar_wait(&sh.acc_empty, (nu - 1) & 1, ast, 15)))
              break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
              umma_ss(tdP, sdesc_sw128(aV + off, 16, 1024), sdesc_sw128(adO + off, 16, 1024),
                      id_s, kk > 0);
            }
            umma_commit(&sh.dp_full);
            // dV += P^T dO (P^T bf16 in TMEM columns [0, 64))
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ts(tdV, tS + kk * 8, sdesc_sw128(adO + kk * 2048, 16384, 1024), id_acc,
                      (acc_started || kk > 0) ? 1u : 0u);
            umma_commit(&sh.do_empty);  // after dP^T and dV have read dO
            // next tile's S^T (after dV has consumed P^T from the same columns)
            if (n + 1 < w.ntiles) {
              const uint32_t c1 = c + 1;
              if (!(ok = mbar_wait(&sh.q_full[c1 % NQ], (c1 / NQ) & 1, ast, 16))) break;
              tc_fence_after();
              issue_s(c1);
            }
          }
          if (keep) {
            if (!(ok = mbar_wait(&sh.ds_full, nret & 1, ast, 17))) break;
            tc_fence_after();
            // dK += dS^T Q_i  (A = dS^T K-major, B = Q_i MN-major)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
              umma_ss(tdK, sdesc_sw128(adS + off, 16, 1024),
                      sdesc_sw128(aQ + kk * 2048, 16384, 1024), id_acc,
                      (acc_started || kk > 0) ? 1u : 0u);
            }
            // dQ_i = dS K_j  (A = dS^T read MN-major, B = K_j MN-major) into dP^T columns
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_ss(tdP, sdesc_sw128(adS + kk * 2048, 16384, 1024),
                      sdesc_sw128(aK + kk * 2048, 16384, 1024), id_dq, kk > 0);
            acc_started = true;
            ++nret;
          }
          // keep dq_full in lockstep with the drain (at most one phase ahead of it)
          if (ntile > 0 && !(ok = mbar_wait(&sh.dq_empty, (ntile - 1) & 1, ast, 19))) break;
          sh.dq_flag[ntile & 1] = keep ? 1u : 0u;
          umma_commit(&sh.dq_full);
          if (keep) umma_commit(&sh.q_empty[st]);  // after dK has read Q_i
        }
        if (!ok) break;
        if (!acc_waited && !(ok = acc_waited = mbar_wait(&sh.acc_empty, (nu - 1) & 1, ast, 15)))
          break;
        sh.acc_valid = acc_started ? 1u : 0u;
        umma_commit(&sh.acc_full);
        umma_commit(&sh.kv_empty);
        ++nu;
      }
      umma_commit(&sh.final_bar);
      AbortState fin = ast;
      uint32_t zero = 0;
      fin.flag = &zero;
      fin.budget_ns = kTeardownBudgetNs;
      mbar_wait(&sh.final_bar, 0, fin, 18);
    }
  } else if (warp >= 4 && warp < 12) {
    // ------------------------------------------------------------------ softmax
    const int wg = (warp - 4) >> 2;         // query-column half
    const int wq = warp & 3;
    const int r = wq * 32 + lane;           // key row within the tile / TMEM lane
    const int tw = tid - 128 - 128 * wg;    // 0..127 within the warpgroup
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const float NEG_INF = -INFINITY;
    uint32_t ntile = 0, nret = 0;  // tiles tested / retained by this CTA (also the stats)
    bool ok = true;
    uint8_t* dsrow_base = sdS + wg * 16384;  // this warpgroup's 64-column atom
    for (uint32_t k = 0; ok; ++k) {
      const int ring = k & 1;
      const bool got = mbar_wait(&sh.sched_full[ring], (k >> 1) & 1, ast, 20);
      // exits are decided by barrier reductions, so both softmax warpgroups leave together
      if (named_bar_or(1, 256, !got || *ast.flag)) { ok = false; break; }
      const int u = sh.sched_ring[ring];
      mbar_arrive(&sh.sched_empty[ring]);
      if (u >= p.n_units) break;
      const BUnit w = decode_bunit(p, u);
      const int krow = w.j * kTile + r;
      const bool kvalid = krow < p.L;
      // per-column constants (LSE in log2 units, the screen's cut LSE2 + log2(tau / L_q),
      // D) of tile n, loaded one tile ahead into registers by threads tw < 64 and
      // published through shared memory
      auto load_cols = [&](int n, float& l2, float& c2, float& ds) {
        int h, i;
        tile_hi(p, w, n, h, i);
        const int q = i * kTile + wg * 64 + tw;
        l2 = INFINITY; c2 = INFINITY; ds = 0.f;
        if (tw < 64 && q < p.L) {
          const size_t idx = (static_cast<size_t>(w.b) * p.H + h) * p.L + q;
          l2 = p.LSE[idx] * kLog2e;
          ds = p.Dsum[idx];
          if (kScreen) c2 = l2 + (p.log2_tau - __log2f(static_cast<float>(q + 1)));
        }
      };
      float nl2, nc2, nds;
      load_cols(0, nl2, nc2, nds);
      for (int n = 0; n < w.ntiles; ++n, ++ntile) {
        int h, i;
        tile_hi(p, w, n, h, i);
        named_bar_sync(2 + wg, 128);  // previous tile's readers are done
        if (tw < 64) {
          sh.lse2[wg][tw] = nl2;
          sh.cut2[wg][tw] = nc2;
          sh.dsum[wg][tw] = nds;
        }
        named_bar_sync(2 + wg, 128);
        if (n + 1 < w.ntiles) load_cols(n + 1, nl2, nc2, nds);
        const bool got = mbar_wait_warp(&sh.s_full, ntile & 1, ast, 21);
        tc_fence_after();
        uint32_t v[2][32];
        if (got) {
          tmem_ld32(tS + lane_off + wg * 64, v[0]);
          tmem_ld32(tS + lane_off + wg * 64 + 32, v[1]);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int e = 0; e < 32; ++e) v[a][e] = 0xff800000u;
        }
        // log2 P = s * scale * log2(e) - LSE2_q (-inf past L through LSE2 = +inf); the
        // tile is kept if some legal entry has log2 P >= log2(tau / L_q) (Eq. 4), i.e.
        // s * scale * log2(e) - cut2_q >= 0 with cut2_q = LSE2_q + log2(tau / L_q).
        // Causal masking is needed only on the diagonal block and past the last key:
        // the local column must be >= qlo (-1 off the diagonal, 64 for rows past L).
        const int qlo = !kvalid ? 64 : (i == w.j ? r - wg * 64 : -1);
        bool keep = true;
        if (kScreen) {
          const float4* c4 = reinterpret_cast<const float4*>(sh.cut2[wg]);
          float ymax = NEG_INF;
          if (qlo < 0) {
            // four independent three-input max chains
            float y4[4] = {NEG_INF, NEG_INF, NEG_INF, NEG_INF};
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
              for (int e4 = 0; e4 < 8; ++e4) {
                const float4 cv = c4[a * 8 + e4];
                const uint32_t* sv = &v[a][e4 * 4];
                const float y0 = fmaf(__uint_as_float(sv[0]), p.scale_log2, -cv.x);
                const float y1 = fmaf(__uint_as_float(sv[1]), p.scale_log2, -cv.y);
                const float y2 = fmaf(__uint_as_float(sv[2]), p.scale_log2, -cv.z);
                const float y3 = fmaf(__uint_as_float(sv[3]), p.scale_log2, -cv.w);
                y4[(e4 & 1) * 2] = fmax3(y4[(e4 & 1) * 2], y0, y1);
                y4[(e4 & 1) * 2 + 1] = fmax3(y4[(e4 & 1) * 2 + 1], y2, y3);
              }
            ymax = fmaxf(fmaxf(y4[0], y4[1]), fmaxf(y4[2], y4[3]));
          } else {
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
              for (int e4 = 0; e4 < 8; ++e4) {
                const float4 cv = c4[a * 8 + e4];
                const float cq[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                  const float y = fmaf(__uint_as_float(v[a][e4 * 4 + c]), p.scale_log2, -cq[c]);
                  ymax = (a * 32 + e4 * 4 + c >= qlo) ? fmaxf(ymax, y) : ymax;
                }
              }
          }
          // the abort flag as one thread saw it before the vote: every thread reads the same
          // copy after the barrier, so the exit below is uniform (the slot is rewritten two
          // tiles later, after every reader has passed the next vote)
          if (tid == 128) sh.abort_seen[ntile & 1] = *ast.flag;
          keep = named_bar_or(1, 256, ymax >= 0.f);
          if (p.tile_margin) {
            // debug: the tile's margin max over legal entries of log P - log(tau / L_q),
            // natural-log units
            const float x = warp_max_f32(ymax);
            if (lane == 0)
              atomic_max_f32(p.tile_margin + ((static_cast<size_t>(w.b) * p.H + h) * p.T + i) * p.T +
                                 w.j,
                             x * kLn2);
          }
          if (sh.abort_seen[ntile & 1]) { ok = false; break; }
        } else {
          // every S^T load done before P overwrites it; the reduction decides the exit
          if (named_bar_or(1, 256, *ast.flag != 0)) { ok = false; break; }
        }
        if (p.tile_mask && tid == 128)
          p.tile_mask[((static_cast<size_t>(w.b) * p.H + h) * p.T + i) * p.T + w.j] = keep ? 1 : 0;
        if (!keep) {
          if (tid == 128) sh.dec = 0;
          tc_fence_before();
          warp_arrive(&sh.p_full);
          continue;
        }
        // P^T = exp2(log2 P) -> bf16 pairs into TMEM columns [32 wg, 32 wg + 32)
        float pf[64];
        const float4* l4 = reinterpret_cast<const float4*>(sh.lse2[wg]);
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c0 = a * 32 + 2 * e;
            const float4 lv = l4[c0 >> 2];
            const float la = (e & 1) ? lv.z : lv.x, lb = (e & 1) ? lv.w : lv.y;
            float x0 = fmaf(__uint_as_float(v[a][2 * e]), p.scale_log2, -la);
            float x1 = fmaf(__uint_as_float(v[a][2 * e + 1]), p.scale_log2, -lb);
            x0 = (c0 >= qlo) ? x0 : NEG_INF;
            x1 = (c0 + 1 >= qlo) ? x1 : NEG_INF;
            const float p0 = fast_exp2(x0);
            const float p1 = fast_exp2(x1);
            pf[c0] = p0;
            pf[c0 + 1] = p1;
            pk[e] = pack_bf16(p0, p1);
          }
          tmem_st16(tS + lane_off + wg * 32 + a * 16, pk);
        }
        tmem_wait_st();
        if (tid == 128) sh.dec = 1;
        tc_fence_before();
        warp_arrive(&sh.p_full);
        // dS^T = P^T o (dP^T - D) -> bf16, swizzled K-major rows in shared memory (the
        // softmax scale is applied to dK in the epilogue and to dQ in the final convert)
        // dP^T of this tile was issued after the previous tile's dK / dQ MMAs, and MMAs
        // complete in issue order, so its completion also frees the dS^T buffer
        const bool dp_ok = mbar_wait_warp(&sh.dp_full, nret & 1, ast, 22);
        ++nret;
        tc_fence_after();
        if (dp_ok) {
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            uint32_t dp[32];
            tmem_ld32(tdP + lane_off + wg * 64 + a * 32, dp);
            tmem_wait_ld();
            const float4* d4 = reinterpret_cast<const float4*>(sh.dsum[wg]);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {  // 4 chunks of 8 columns = 16 bytes
              const float4 da = d4[a * 8 + ch * 2], db = d4[a * 8 + ch * 2 + 1];
              const float dq[8] = {da.x, da.y, da.z, da.w, db.x, db.y, db.z, db.w};
              uint32_t pk[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int c0 = a * 32 + ch * 8 + 2 * e;
                const float d0 = pf[c0] * (__uint_as_float(dp[ch * 8 + 2 * e]) - dq[2 * e]);
                const float d1 = pf[c0 + 1] * (__uint_as_float(dp[ch * 8 + 2 * e + 1]) - dq[2 * e + 1]);
                pk[e] = pack_bf16(d0, d1);
              }
              *reinterpret_cast<uint4*>(dsrow_base + sw128_offset(r, a * 4 + ch)) =
                  make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        warp_arrive(&sh.ds_full);
      }
    }
    if (tid == 128) stats_add(p.stats, ntile, nret, 0);
  } else if (warp >= 12) {
    // ------------------------------------------------------------------ dQ drain + dK/dV epilogue
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    uint32_t ntile = 0, nu = 0;
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int ring = k & 1;
      const bool got = mbar_wait(&sh.sched_full[ring], (k >> 1) & 1, ast, 30);
      if (named_bar_or(4, 128, !got || *ast.flag)) { ok = false; break; }
      const int u = sh.sched_ring[ring];
      mbar_arrive(&sh.sched_empty[ring]);
      if (u >= p.n_units) break;
      const BUnit w = decode_bunit(p, u);
      for (int n = 0; n < w.ntiles; ++n, ++ntile) {
        int h, i;
        tile_hi(p, w, n, h, i);
        const bool got_dq = mbar_wait_warp(&sh.dq_full, ntile & 1, ast, 31);
        tc_fence_after();
        // the drain below holds named barriers: decide it uniformly for the 128 threads
        const bool drain = named_bar_or(5, 128, got_dq && sh.dq_flag[ntile & 1] != 0);
        if (!drain) {
          tc_fence_before();
          warp_arrive(&sh.dq_empty);
          continue;
        }
        // dQ tile (row r of query block i): 64 columns per round through the staging
        // buffer, TMA bulk add into the fp32 accumulator.  The TMEM columns are released
        // right after the last round has been loaded into registers.
#pragma unroll
        for (int half = 0; half < D / 64; ++half) {
          uint32_t o[2][32];
          tmem_ld32(tdP + lane_off + half * 64, o[0]);
          tmem_ld32(tdP + lane_off + half * 64 + 32, o[1]);
          tmem_wait_ld();
          if (half == D / 64 - 1) {
            tc_fence_before();
            warp_arrive(&sh.dq_empty);
          }
          // staging buffer free: the previous round's bulk reads have completed
          if (tid == 384) bulk_wait_read_all();
          named_bar_sync(5, 128);
#pragma unroll
          for (int box = 0; box < 2; ++box)
#pragma unroll
            for (int ch = 0; ch < 8; ++ch)
              *reinterpret_cast<uint4*>(sdQ + box * 16384 + sw128_offset(r, ch)) =
                  make_uint4(o[box][4 * ch], o[box][4 * ch + 1], o[box][4 * ch + 2],
                             o[box][4 * ch + 3]);
          fence_proxy_async_smem();
          named_bar_sync(5, 128);
          if (tid == 384) {
#pragma unroll
            for (int box = 0; box < 2; ++box)
              tma_reduce_add_4d(&tmdQ, sdQ + box * 16384, half * 64 + box * 32, h, i * kTile,
                                w.b);
            bulk_commit_group();
          }
        }
      }
      // unit epilogue: dK, dV of key block j
      const bool got_acc = mbar_wait_warp(&sh.acc_full, nu & 1, ast, 32);
      tc_fence_after();
      const bool valid_acc = sh.acc_valid != 0;
      const int krow = w.j * kTile + r;
      // tcgen05.ld is warp-collective: every lane loads, only rows < L are stored
      if (got_acc) {
        const bool store = krow < p.L;
        const size_t base = ((static_cast<size_t>(w.b) * p.L + (store ? krow : 0)) * p.Hkv + w.g) * D;
        const bool split = p.dKacc != nullptr;  // head parts: add this part's share
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          __nv_bfloat16* dst = (which == 0 ? p.dV : p.dK) + base;
          float* accd = split ? (which == 0 ? p.dVacc : p.dKacc) + base : nullptr;
          const uint32_t src = (which == 0 ? tdV : tdK) + lane_off;
          const float sc = (which == 1) ? p.scale : 1.f;  // dK = scale * dS^T Q
#pragma unroll
          for (int a = 0; a < D / 32; ++a) {
            uint32_t o[32];
            tmem_ld32(src + a * 32, o);
            tmem_wait_ld();
            if (split) {
              if (store && valid_acc) {
#pragma unroll
                for (int e4 = 0; e4 < 8; ++e4) {
                  const float* f = reinterpret_cast<const float*>(o) + e4 * 4;
                  atomicAdd(reinterpret_cast<float4*>(accd + a * 32 + e4 * 4),
                            make_float4(f[0] * sc, f[1] * sc, f[2] * sc, f[3] * sc));
                }
              }
              continue;
            }
#pragma unroll
            for (int e8 = 0; e8 < 4; ++e8) {
              uint4 pk;
              const float* f = reinterpret_cast<const float*>(o) + e8 * 8;
              if (valid_acc) {
                pk.x = pack_bf16(f[0] * sc, f[1] * sc);
                pk.y = pack_bf16(f[2] * sc, f[3] * sc);
                pk.z = pack_bf16(f[4] * sc, f[5] * sc);
                pk.w = pack_bf16(f[6] * sc, f[7] * sc);
              } else {
                pk = make_uint4(0u, 0u, 0u, 0u);
              }
              if (store) *reinterpret_cast<uint4*>(dst + a * 32 + e8 * 8) = pk;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.acc_empty);
      ++nu;
    }
    // every dQ reduction of this CTA must have landed before the kernel ends
    if (tid == 384) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tb, 512);
}

// D_q = <O_q, dO_q> and zeroing of the dQ accumulator; one warp per (b, q, h) row.
template <int D>
__global__ void __launch_bounds__(256) mala_bwd_prep(const __nv_bfloat16* __restrict__ O,
                                                     const __nv_bfloat16* __restrict__ dO,
                                                     float* __restrict__ Dsum,
                                                     float* __restrict__ dQacc, int B, int L,
                                                     int H) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(B) * L * H) return;
  constexpr int PER = D / 32;  // elements per lane (2 or 4)
  const __nv_bfloat16* o = O + row * D + lane * PER;
  const __nv_bfloat16* g = dO + row * D + lane * PER;
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < PER; e += 2) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(o + e));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(g + e));
    s += a.x * b.x + a.y * b.y;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  float* z = dQacc + row * D + lane * PER;
#pragma unroll
  for (int e = 0; e < PER; ++e) z[e] = 0.f;
  if (lane == 0) {
    const int h = static_cast<int>(row % H);
    const long long bq = row / H;
    const int q = static_cast<int>(bq % L);
    const int b = static_cast<int>(bq / L);
    Dsum[(static_cast<long long>(b) * H + h) * L + q] = s;
  }
}

// dQ = bf16(scale * accumulator): the accumulator holds dS K without the softmax scale.
__global__ void __launch_bounds__(256) mala_bwd_dq(const float* __restrict__ acc,
                                                   __nv_bfloat16* __restrict__ dQ, long long n4,
                                                   float scale) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 v = reinterpret_cast<const float4*>(acc)[i];
  uint2 pk;
  pk.x = pack_bf16(v.x * scale, v.y * scale);
  pk.y = pack_bf16(v.z * scale, v.w * scale);
  reinterpret_cast<uint2*>(dQ)[i] = pk;
}

}  // namespace

// Head parts of a backward unit (a function of the shape alone, so that the workspace
// query and the launch agree): the G heads are halved while the problem has fewer than
// kPartsTarget (b, g, part) x (T + 1) work units, i.e. while the heaviest unit (key block 0,
// Gp T tiles) would exceed about half of a 148-SM share of the legal tiles.
constexpr long long kPartsTarget = 4 * 148;

int bwd_head_parts(int B, int H, int Hkv, int L) {
  const int G = H / Hkv;
  const long long T = (L + kTile - 1) / kTile;
  int P = 1;
  while (P < G && G % (2 * P) == 0 &&
         static_cast<long long>(B) * Hkv * (T + 1) * P < kPartsTarget)
    P *= 2;
  return P;
}

size_t bwd_workspace_bytes(int B, int H, int Hkv, int L, int d, int dtype) {
  const size_t acc = static_cast<size_t>(B) * L * H * d * sizeof(float);
  const size_t dsum = static_cast<size_t>(B) * H * L * sizeof(float);
  size_t bytes = kWorkspaceHeader + ((acc + 255) / 256) * 256 + ((dsum + 255) / 256) * 256;
  if (dtype != MALA_FP32 && bwd_head_parts(B, H, Hkv, L) > 1) {
    const size_t kv = static_cast<size_t>(B) * L * Hkv * d * sizeof(float);
    bytes += 2 * ((kv + 255) / 256) * 256;  // dK, dV accumulators
  }
  return bytes;
}

mala_status fp32_bwd(const float* Q, const float* K, const float* V, const float* O,
                     const float* LSE, const float* dO, float* dQ, float* dK, float* dV, int B,
                     int H, int Hkv, int L, int d, float scale, float tau, bool screen,
                     uint8_t* ws, uint8_t* tile_mask, float* tile_margin, cudaStream_t stream);

template <int D, bool kScreen>
static cudaError_t launch_bwd_main(const CUtensorMap& tq, const CUtensorMap& tk,
                                   const CUtensorMap& tv, const CUtensorMap& tdo,
                                   const CUtensorMap& tdq, const BwdParams& p, int grid,
                                   cudaStream_t stream) {
  auto kern = mala_bwd_kernel<D, kScreen>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       BwdCfg<D>::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<grid, kBwdThreads, BwdCfg<D>::SMEM, stream>>>(tq, tk, tv, tdo, tdq, p);
  return cudaGetLastError();
}

// fp32 [n3][n2][n1][n0] tensor, box {32, 1, 128, 1} (128-byte rows), 128-byte swizzle.
static bool make_f32_reduce_map(CUtensorMap* m, void* base, int n0, int n1, int n2, int n3) {
  typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                               const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                               const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                               CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
  void* f = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return false;
  cuuint64_t dims[4] = {(cuuint64_t)n0, (cuuint64_t)n1, (cuuint64_t)n2, (cuuint64_t)n3};
  cuuint64_t strides[3] = {(cuuint64_t)n0 * 4, (cuuint64_t)n0 * n1 * 4,
                           (cuuint64_t)n0 * n1 * n2 * 4};
  cuuint32_t box[4] = {32, 1, 128, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  return reinterpret_cast<EncodeFn>(f)(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides,
                                       box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                                       CU_TENSOR_MAP_SWIZZLE_128B,
                                       CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                       CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

mala_status bwd_dispatch(const void* Q, const void* K, const void* V, const void* O,
                         const float* LSE, const void* dO, void* dQ, void* dK, void* dV, int B,
                         int H, int Hkv, int L, int d, int dtype, float scale, float tau,
                         unsigned flags, uint8_t* ws, uint8_t* tile_mask, float* tile_margin,
                         uint64_t budget_ns, cudaStream_t stream) {
  const bool screen = (tau > 0.f) || (flags & MALA_FLAG_ALWAYS_TEST);
  if (cudaMemsetAsync(ws + kStatsOffset, 0, 3 * sizeof(unsigned long long), stream) !=
      cudaSuccess)
    return MALA_ERR_CUDA;
  if (dtype == MALA_FP32)
    return fp32_bwd(static_cast<const float*>(Q), static_cast<const float*>(K),
                    static_cast<const float*>(V), static_cast<const float*>(O), LSE,
                    static_cast<const float*>(dO), static_cast<float*>(dQ),
                    static_cast<float*>(dK), static_cast<float*>(dV), B, H, Hkv, L, d, scale,
                    tau, screen, ws, tile_mask, tile_margin, stream);
  const int T = (L + kTile - 1) / kTile;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_tile_map(&tq, Q, d, H, L, B) || !make_tile_map(&tk, K, d, Hkv, L, B) ||
      !make_tile_map(&tv, V, d, Hkv, L, B) || !make_tile_map(&tdo, dO, d, H, L, B))
    return MALA_ERR_CUDA;
  uint32_t* hdr = reinterpret_cast<uint32_t*>(ws);
  const size_t acc_bytes = static_cast<size_t>(B) * L * H * d * sizeof(float);
  const size_t dsum_bytes = static_cast<size_t>(B) * H * L * sizeof(float);
  float* dQacc = reinterpret_cast<float*>(ws + kWorkspaceHeader);
  float* Dsum = reinterpret_cast<float*>(ws + kWorkspaceHeader + ((acc_bytes + 255) / 256) * 256);
  const int P = bwd_head_parts(B, H, Hkv, L);
  const size_t kv_bytes = static_cast<size_t>(B) * L * Hkv * d * sizeof(float);
  float* dKacc = nullptr;
  float* dVacc = nullptr;
  if (P > 1) {
    uint8_t* kv0 = ws + kWorkspaceHeader + ((acc_bytes + 255) / 256) * 256 +
                   ((dsum_bytes + 255) / 256) * 256;
    dKacc = reinterpret_cast<float*>(kv0);
    dVacc = reinterpret_cast<float*>(kv0 + ((kv_bytes + 255) / 256) * 256);
    if (cudaMemsetAsync(kv0, 0, 2 * ((kv_bytes + 255) / 256) * 256, stream) != cudaSuccess)
      return MALA_ERR_CUDA;
  }
  CUtensorMap tdq;
  if (!make_f32_reduce_map(&tdq, dQacc, d, H, L, B)) return MALA_ERR_CUDA;
  if (cudaMemsetAsync(hdr + kHdrSched0, 0, 3 * sizeof(uint32_t), stream) != cudaSuccess)
    return MALA_ERR_CUDA;
  const long long rows = static_cast<long long>(B) * L * H;
  const unsigned prep_blocks = static_cast<unsigned>((rows + 7) / 8);
  if (d == 128)
    mala_bwd_prep<128><<<prep_blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO), Dsum, dQacc,
        B, L, H);
  else
    mala_bwd_prep<64><<<prep_blocks, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO), Dsum, dQacc,
        B, L, H);
  if (cudaGetLastError() != cudaSuccess) return MALA_ERR_CUDA;
  BwdParams p;
  p.B = B; p.H = H; p.Hkv = Hkv; p.L = L; p.T = T; p.G = H / Hkv;
  p.P = P; p.Gp = p.G / P;
  p.n_units = T * B * Hkv * P;
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.log2_tau = (tau > 0.f) ? std::log2(tau) : -INFINITY;
  p.LSE = LSE; p.Dsum = Dsum; p.dQacc = dQacc;
  p.dK = static_cast<__nv_bfloat16*>(dK);
  p.dV = static_cast<__nv_bfloat16*>(dV);
  p.dKacc = dKacc;
  p.dVacc = dVacc;
  p.tile_mask = tile_mask;
  p.tile_margin = tile_margin;
  p.stats = reinterpret_cast<unsigned long long*>(ws + kStatsOffset);
  p.err = hdr + kHdrError;
  p.sched = hdr + kHdrSched0;
  p.budget_ns = budget_ns;
  const int grid = p.n_units < sm_count() ? p.n_units : sm_count();
  cudaError_t e;
  if (d == 128)
    e = screen ? launch_bwd_main<128, true>(tq, tk, tv, tdo, tdq, p, grid, stream)
               : launch_bwd_main<128, false>(tq, tk, tv, tdo, tdq, p, grid, stream);
  else
    e = screen ? launch_bwd_main<64, true>(tq, tk, tv, tdo, tdq, p, grid, stream)
               : launch_bwd_main<64, false>(tq, tk, tv, tdo, tdq, p, grid, stream);
  if (e != cudaSuccess) return MALA_ERR_CUDA;
  const long long n4 = rows * d / 4;
  mala_bwd_dq<<<static_cast<unsigned>((n4 + 255) / 256), 256, 0, stream>>>(
      dQacc, static_cast<__nv_bfloat16*>(dQ), n4, scale);
  if (P > 1) {
    // the dK accumulator already holds the scale
    const long long kv4 = static_cast<long long>(B) * L * Hkv * d / 4;
    mala_bwd_dq<<<static_cast<unsigned>((kv4 + 255) / 256), 256, 0, stream>>>(
        dKacc, static_cast<__nv_bfloat16*>(dK), kv4, 1.f);
    mala_bwd_dq<<<static_cast<unsigned>((kv4 + 255) / 256), 256, 0, stream>>>(
        dVacc, static_cast<__nv_bfloat16*>(dV), kv4, 1.f);
  }
  return cudaGetLastError() == cudaSuccess ? MALA_OK : MALA_ERR_CUDA;
}

}  // namespace mala
