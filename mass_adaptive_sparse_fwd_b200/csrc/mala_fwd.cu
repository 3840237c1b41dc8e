// MALA forward kernel for sm_100a (bf16, head dim 64 or 128).
//
// "MassAlloc Attention: Let Attention Allocate Its Own Compute", §2.2 (online sparse
// softmax, Eq. (1)-(3)), App. A Algorithm 1 and A.1 (fused forward execution).
//
// One persistent CTA per SM pulls work units from an atomic counter.  A unit is one
// 128-row query block i of two query heads that share a KV head (two "slots"), so both
// slots stream the same K_j / V_j tiles; units are numbered heaviest first (largest i)
// within a KV head.
// Within a unit the key blocks are visited from the block of the unit's last query
// position down to 0 (diagonal first).  For chunked prefill (§2.3: the forward serves
// inference prefill) the L query rows are the last L of Lk key positions: row q sits at
// position off + q, off = Lk - L, attends to keys <= its position and has L_q = off + q + 1;
// with off = 0 this is the ordinary causal forward.  A packed batch of sequences of
// different lengths (varlen) gives every unit its own sequence's row bases, length and
// offset through a host-built table (FwdParams::vtab).
//
// Warp roles (576 threads):
//   warp 0       TMA producer: Q of both slots, then K_j and V_j per key block into a
//                ring of NS stages.  V is fetched together with K (see below).
//   warp 1       TMEM owner and UMMA issuer: S_s = Q_s K_j^T (SS, both K-major) into
//                TMEM, and O_s += P_s V_j (TS: P in TMEM, V MN-major) for retained tiles.
//   warps 2-9    softmax / retention test for slot 0: thread = query row = TMEM lane,
//                warps 2-5 on keys 0..63 of the tile and warps 6-9 on keys 64..127; the
//                two halves exchange their row maxima and shares of the row sum through
//                shared memory once per tile
//   warps 10-17  same for slot 1
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,256+D), O_1 [256+D, 256+2D).
// P_s (bf16, packed in pairs) overwrites, in each half, the first 32 of its 64 columns of
// S_s: keys 0..63 in columns [0, 32), keys 64..127 in columns [64, 96).
//
// Retention test (Eq. 3) per row q in the log2 domain: with the running state
// (m, l) of retained tiles, log2 Z = m + log2 l.  A row keeps the tile if l == 0
// (its first legal tile) or rowmax(S) * scale * log2(e) >= m + log2(l) + log2(tau/L_q),
// L_q = position + 1; rows with no legal key in the tile (above the diagonal, or q >= L) do
// not vote.  The tile is retained if any row keeps it (bar.red.or over the slot's 256
// threads).  A skipped tile leaves m, l and O untouched and costs only the QK^T MMA,
// the TMEM load of S and the row maxima: no exponentials, no P store, no PV MMA.
//
// The running max used for P is updated lazily (only when a row max exceeds it by
// more than 8 in log2 units), so O is rescaled in TMEM only on such jumps; log Z is
// m + log2 l for any m, so the test is unaffected.
//
// V loading: K_j and V_j are fetched together, before the decision for tile j exists.
// The forward is tensor-core bound and deciding first would put the V latency on the
// critical path of every retained tile; the skipped work is the exponentials and the
// PV MMA.  (Decode, which is bandwidth bound, gates its V loads on the decision.)
//
// Units are numbered KV head slowest and heaviest first within a head, so that the CTAs
// running together share one head's K and V in L2 (on skipped tiles the forward waits on
// K/V loads through the two-stage ring, and L2 hits shorten them).

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "mala_common.cuh"
#include "sm100.cuh"

namespace mala {

namespace {

template <int D>
struct FwdCfg {
  static constexpr int NS = (D == 128) ? 2 : 4;          // K/V ring stages (K and V tiles each)
  static constexpr int TILE_BYTES = kTile * D * 2;       // one 128 x D bf16 tile
  static constexpr int BOXES = D / 64;                   // 64-column TMA boxes per tile
  static constexpr int SMEM = 2 * TILE_BYTES + 2 * NS * TILE_BYTES + 1024;
  static constexpr int THREADS = 576;  // warps 0-1 TMA / MMA, warps 2-17 softmax
};

struct FwdShared {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[4], v_full[4], kv_empty[4];
  uint64_t s_full[2], p_full[2], o_done[2];
  uint64_t sched_full[2], sched_empty[2];
  uint64_t final_bar;
  int sched_ring[2];
  uint32_t dec[2];
  uint32_t tmem_base;
  uint32_t abort_flag;
  // per slot and key-column half: the half's raw row maximum of the current tile and its
  // share of the running row sum, exchanged once per tile
  float xmax[2][2][128];
  float xsum[2][2][128];
};

static_assert(FwdCfg<128>::SMEM + sizeof(FwdShared) <= 232448, "forward smem budget");
static_assert(FwdCfg<64>::SMEM + sizeof(FwdShared) <= 232448, "forward smem budget");

struct Unit {
  int b, g, i, h0;
  bool active[2];
  int qrow0, krow0;  // first row of the sequence in Q / K (packed varlen batch), else 0
  int L, off;        // the sequence's query rows and causal offset
};

// Whether slot s of the unit holds a head (constant-index access keeps Unit in registers).
__device__ __forceinline__ bool slot_active(const Unit& w, int s) {
  return s == 0 ? w.active[0] : w.active[1];
}

// Last key block holding a legal key of the unit's query block (its last row's position).
__device__ __forceinline__ int last_key_tile(const Unit& w) {
  const int q_last = min(w.i * kTile + kTile - 1, w.L - 1);
  return (w.off + q_last) / kTile;
}

__device__ __forceinline__ Unit decode_unit(const FwdParams& p, int u) {
  Unit w;
  int r, hp;
  if (p.vtab) {  // packed batch: the table lists (sequence, query block), heaviest first
    const int nbg = p.Hkv * p.npairs;
    const VarlenBlock e = p.vtab[u / nbg];
    r = u % nbg;
    w.b = 0;
    w.g = r / p.npairs;
    hp = r % p.npairs;
    w.i = e.i;
    w.qrow0 = e.qrow0;
    w.krow0 = e.krow0;
    w.L = e.L;
    w.off = e.off;
  } else {
    // KV head slowest: the CTAs that run together share one head's K and V in L2;
    // heaviest first (largest i) within a head
    const int nbp = p.B * p.npairs;
    const int upg = nbp * p.T;
    w.g = u / upg;
    r = u % upg;
    w.i = p.T - 1 - r / nbp;
    w.b = (r % nbp) / p.npairs;
    hp = r % p.npairs;
    w.qrow0 = 0;
    w.krow0 = 0;
    w.L = p.L;
    w.off = p.off;
  }
  w.h0 = w.g * p.G + 2 * hp;
  w.active[0] = true;
  w.active[1] = (2 * hp + 1) < p.G;
  return w;
}

template <int D, bool kScreen>
__global__ void __launch_bounds__(576, 1)
    mala_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using C = FwdCfg<D>;
  constexpr int NS = C::NS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sQ = smem;                                  // 2 tiles
  uint8_t* sK = smem + 2 * C::TILE_BYTES;              // NS tiles
  uint8_t* sV = sK + NS * C::TILE_BYTES;               // NS tiles
  __shared__ FwdShared sh;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sh.q_full[s], 1);
      mbar_init(&sh.q_empty[s], 1);
      mbar_init(&sh.s_full[s], 1);
      mbar_init(&sh.p_full[s], 8);  // one arrival per softmax warp of the slot
      mbar_init(&sh.o_done[s], 1);
      mbar_init(&sh.sched_full[s], 1);
      mbar_init(&sh.sched_empty[s], 1 + 512);
    }
    for (int st = 0; st < NS; ++st) {
      mbar_init(&sh.k_full[st], 1);
      mbar_init(&sh.v_full[st], 1);
      mbar_init(&sh.kv_empty[st], 1);
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
  const AbortState ast{&sh.abort_flag, p.err, p.budget_ns, 0x100u};

  if (warp == 0) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      uint32_t c = 0;                  // K/V tiles issued (all units)
      uint32_t nq[2] = {0, 0};         // Q loads issued per slot
      bool ok = true;
      for (uint32_t k = 0; ok; ++k) {
        const int ring = k & 1;
        if (k >= 2 && !(ok = mbar_wait(&sh.sched_empty[ring], ((k >> 1) - 1) & 1, ast, 1))) break;
        const int u = static_cast<int>(atomicAdd(p.sched, 1u));
        sh.sched_ring[ring] = u;
        mbar_arrive(&sh.sched_full[ring]);
        if (u >= p.n_units) break;
        const Unit w = decode_unit(p, u);
        for (int s = 0; s < 2 && ok; ++s) {
          if (!slot_active(w, s)) continue;
          if (nq[s] > 0 && !(ok = mbar_wait(&sh.q_empty[s], (nq[s] - 1) & 1, ast, 2))) break;
          mbar_arrive_expect_tx(&sh.q_full[s], C::TILE_BYTES);
          for (int x = 0; x < C::BOXES; ++x)
            tma_load_4d(sQ + s * C::TILE_BYTES + x * 16384, &tmQ, &sh.q_full[s], x * 64,
                        w.h0 + s, w.qrow0 + w.i * kTile, w.b);
          ++nq[s];
        }
        const int jl = last_key_tile(w);
        for (int t = 0; t <= jl && ok; ++t, ++c) {
          const int j = jl - t;
          const int st = c % NS;
          if (c >= NS && !(ok = mbar_wait(&sh.kv_empty[st], ((c / NS) - 1) & 1, ast, 3))) break;
          mbar_arrive_expect_tx(&sh.k_full[st], C::TILE_BYTES);
          for (int x = 0; x < C::BOXES; ++x)
            tma_load_4d(sK + st * C::TILE_BYTES + x * 16384, &tmK, &sh.k_full[st], x * 64, w.g,
                        w.krow0 + j * kTile, w.b);
          mbar_arrive_expect_tx(&sh.v_full[st], C::TILE_BYTES);
          for (int x = 0; x < C::BOXES; ++x)
            tma_load_4d(sV + st * C::TILE_BYTES + x * 16384, &tmV, &sh.v_full[st], x * 64, w.g,
                        w.krow0 + j * kTile, w.b);
        }
      }
      if (!ok) {
        // drain: wait (bounded) for the loads this CTA still has in flight
        AbortState drain = ast;
        uint32_t zero = 0;
        drain.flag = &zero;
        drain.budget_ns = kTeardownBudgetNs;
        for (uint32_t cc = (c > NS ? c - NS : 0); cc < c; ++cc) {
          mbar_wait(&sh.k_full[cc % NS], (cc / NS) & 1, drain, 4);
          mbar_wait(&sh.v_full[cc % NS], (cc / NS) & 1, drain, 4);
        }
        for (int s = 0; s < 2; ++s)
          if (nq[s] > 0) mbar_wait(&sh.q_full[s], (nq[s] - 1) & 1, drain, 4);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t id_pv = idesc_bf16(128, D, 0, 1);
      uint32_t c = 0;
      uint32_t nq[2] = {0, 0};
      uint32_t np[2] = {0, 0};  // p_full phases consumed per slot
      bool ok = true;
      auto issue_qk = [&](int s, int st) {
        const uint32_t qa = smem_u32(sQ + s * C::TILE_BYTES);
        const uint32_t ka = smem_u32(sK + st * C::TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          umma_ss(tb + s * 128, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024),
                  id_qk, kk > 0);
        }
        umma_commit(&sh.s_full[s]);
      };
      for (uint32_t k = 0; ok; ++k) {
        const int ring = k & 1;
        if (!(ok = mbar_wait(&sh.sched_full[ring], (k >> 1) & 1, ast, 10))) break;
        const int u = sh.sched_ring[ring];
        mbar_arrive(&sh.sched_empty[ring]);
        if (u >= p.n_units) break;
        const Unit w = decode_unit(p, u);
        for (int s = 0; s < 2 && ok; ++s) {
          if (!slot_active(w, s)) continue;
          ok = mbar_wait(&sh.q_full[s], nq[s] & 1, ast, 11);
          ++nq[s];
        }
        if (!ok) break;
        bool o_started[2] = {false, false};
        const int n = last_key_tile(w) + 1;
        // prologue: S for the diagonal tile
        {
          const int st = c % NS;
          if (!(ok = mbar_wait(&sh.k_full[st], (c / NS) & 1, ast, 12))) break;
          tc_fence_after();
          for (int s = 0; s < 2; ++s)
            if (slot_active(w, s)) issue_qk(s, st);
        }
        for (int t = 0; t < n && ok; ++t, ++c) {
          const int st = c % NS;
          bool v_ready = false, k_next_ready = false;
          for (int s = 0; s < 2 && ok; ++s) {
            if (!slot_active(w, s)) continue;
            if (!(ok = mbar_wait(&sh.p_full[s], np[s] & 1, ast, 13))) break;
            ++np[s];
            tc_fence_after();
            if (sh.dec[s]) {
              if (!v_ready && !(ok = v_ready = mbar_wait(&sh.v_full[st], (c / NS) & 1, ast, 14)))
                break;
              const uint32_t va = smem_u32(sV + st * C::TILE_BYTES);
#pragma unroll
              for (int kk = 0; kk < 8; ++kk)  // P of keys 16 kk .. (see the softmax's pass 2)
                umma_ts(tb + 256 + s * D, tb + s * 128 + (kk >> 2) * 64 + (kk & 3) * 8,
                        sdesc_sw128(va + kk * 2048, 16384, 1024), id_pv,
                        (o_started[s] || kk > 0) ? 1u : 0u);
              o_started[s] = true;
              umma_commit(&sh.o_done[s]);
            }
            if (t + 1 < n) {
              const uint32_t c1 = c + 1;
              if (!k_next_ready &&
                  !(ok = k_next_ready = mbar_wait(&sh.k_full[c1 % NS], (c1 / NS) & 1, ast, 15)))
                break;
              tc_fence_after();
              issue_qk(s, c1 % NS);
            }
          }
          if (!ok) break;
          // the stage is released only after its V load landed, even if no slot used it
          if (!v_ready && !(ok = mbar_wait(&sh.v_full[st], (c / NS) & 1, ast, 16))) break;
          umma_commit(&sh.kv_empty[st]);
        }
        if (!ok) break;
        for (int s = 0; s < 2; ++s)
          if (slot_active(w, s)) umma_commit(&sh.q_empty[s]);
      }
      // wait for every MMA this thread issued before TMEM is released
      umma_commit(&sh.final_bar);
      AbortState fin = ast;
      uint32_t zero = 0;
      fin.flag = &zero;
      fin.budget_ns = kTeardownBudgetNs;
      mbar_wait(&sh.final_bar, 0, fin, 17);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------------ softmax
    // warps 2..17: slot s = (warp - 2) / 8 and key-column half hf = ((warp - 2) / 4) % 2;
    // the warp reaches TMEM lanes 32 (warp % 4) .. + 31 (four consecutive warps cover the
    // 128 rows), so thread = query row r and each half handles 64 of the tile's 128 keys
    const int wsm = warp - 2;
    const int s = wsm >> 3;                 // slot
    const int hf = (wsm >> 2) & 1;          // key-column half
    const int wq = warp & 3;                // TMEM lane quarter
    const int r = wq * 32 + lane;           // row within the tile
    const int c0 = hf * 64;                 // this half's key columns [c0, c0 + 64)
    constexpr int DH = D / 2;               // this half's head-dim columns of O
    const uint32_t bar_slot = 1 + s;        // named barrier of the slot's 256 threads
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tb + s * 128 + lane_off;
    const uint32_t tO = tb + 256 + s * D + lane_off + hf * DH;
    const float NEG_INF = -INFINITY;
    uint32_t ns = 0, npv = 0;  // tiles tested / retained by this slot (also the stats)
    bool ok = true;
    for (uint32_t k = 0; ok; ++k) {
      const int ring = k & 1;
      // every exit of this loop is decided by a barrier reduction over the slot's 256
      // threads (a failed wait, or the abort flag seen by any of them), so that they
      // always leave together
      const bool got = mbar_wait(&sh.sched_full[ring], (k >> 1) & 1, ast, 20);
      if (named_bar_or(bar_slot, 256, !got || *ast.flag)) { ok = false; break; }
      const int u = sh.sched_ring[ring];
      mbar_arrive(&sh.sched_empty[ring]);
      if (u >= p.n_units) break;
      const Unit w = decode_unit(p, u);
      if (!slot_active(w, s)) continue;
      const int h = w.h0 + s;
      const int q = w.i * kTile + r;
      const bool valid = q < w.L;
      // L_q = position + 1 (the position is q in a full forward, off + q in a chunk)
      const float thr2 =
          kScreen ? (p.log2_tau - __log2f(static_cast<float>(w.off + q + 1))) : NEG_INF;
      // m2: running maximum (log2 units, the same in both halves); l: this half's share of
      // the running sum (the row's sum is the two halves' shares added)
      float m2 = NEG_INF, l = 0.f;
      const uint32_t npv_unit0 = npv;
      const int jl = last_key_tile(w);
      const int pos0 = w.off + w.i * kTile;  // position of the block's first row
      const int n = jl + 1;
      for (int t = 0; t < n; ++t) {
        const int j = jl - t;
        const bool got = mbar_wait_warp(&sh.s_full[s], ns & 1, ast, 21);
        ++ns;
        tc_fence_after();
        // pass 1: this half's row maximum of the raw scores (the scale is positive, so it
        // commutes with max); only tiles that reach past the block's first position and
        // rows past the end need masking: key c is legal for row r iff c <= lim
        const bool masked = (j * kTile + kTile - 1 > pos0) || !valid;
        const int lim = valid ? (pos0 + r - j * kTile) : -1;
        float rraw = NEG_INF;
        if (got) {
#pragma unroll
          for (int a = 0; a < 2; ++a) {  // 32 columns at a time (register budget)
            uint32_t v[32];
            tmem_ld32(tS + c0 + a * 32, v);
            tmem_wait_ld();
            if (masked) {
#pragma unroll
              for (int e = 0; e < 32; ++e) {
                const int col = c0 + a * 32 + e;
                rraw = fmaxf(rraw, col <= lim ? __uint_as_float(v[e]) : NEG_INF);
              }
            } else {
              // four independent three-input max chains
              float r0 = rraw, r1 = NEG_INF, r2 = NEG_INF, r3 = NEG_INF;
#pragma unroll
              for (int e = 0; e < 32; e += 8) {
                r0 = fmax3(r0, __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
                r1 = fmax3(r1, __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                r2 = fmax3(r2, __uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
                r3 = fmax3(r3, __uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
              }
              rraw = fmaxf(fmaxf(r0, r1), fmaxf(r2, r3));
            }
          }
        }
        // exchange with the other half: its row maximum of this tile and its share of the
        // running sum.  The barrier also orders every S load of the tile before the P
        // stores below, and the previous tile's reads of the exchange slots before these
        // writes (they come after that tile's vote / this barrier's predecessor).
        sh.xmax[s][hf][r] = rraw;
        sh.xsum[s][hf][r] = l;
        if (named_bar_or(bar_slot, 256, !got || *ast.flag)) { ok = false; break; }
        rraw = fmaxf(rraw, sh.xmax[s][hf ^ 1][r]);
        const float lrow = l + sh.xsum[s][hf ^ 1][r];
        const float rmax = rraw * p.scale_log2;
        bool keep = true;
        if (kScreen) {
          const float cut = m2 + __log2f(lrow) + thr2;
          const bool mine = (rmax != NEG_INF) && (lrow == 0.f || rmax >= cut);
          keep = named_bar_or(bar_slot, 256, mine);
          if (p.tile_margin && hf == 0) {
            // debug: the tile's margin max_q (rowmax - cut) in natural-log units (+inf for
            // a row's first retained tile, -inf for rows without a legal key)
            float x = (rmax == NEG_INF) ? NEG_INF : (lrow == 0.f ? INFINITY : rmax - cut);
            x = warp_max_f32(x);
            if (lane == 0)
              atomic_max_f32(p.tile_margin + ((static_cast<size_t>(w.b) * p.H + h) * p.T + w.i) *
                                                 p.Tk + j,
                             x * kLn2);
          }
        }
        if (p.tile_mask && r == 0 && hf == 0)
          p.tile_mask[((static_cast<size_t>(w.b) * p.H + h) * p.T + w.i) * p.Tk + j] = keep ? 1 : 0;
        if (!keep) {
          if (r == 0 && hf == 0) sh.dec[s] = 0;
          tc_fence_before();
          warp_arrive(&sh.p_full[s]);
          continue;
        }
        // lazy running-max update (identical in both halves)
        float m_new = m2;
        bool rescale = false;
        if (rmax > m2 + 8.0f) {
          m_new = rmax;
          rescale = (lrow > 0.f);
        }
        const float m_use = (m_new == NEG_INF) ? 0.f : m_new;
        const float alpha = rescale ? fast_exp2(m2 - m_new) : 1.f;
        if (__any_sync(0xffffffffu, rescale) &&
            // the previous PV of this slot must have landed before O is touched
            mbar_wait_warp(&sh.o_done[s], (npv - 1) & 1, ast, 22)) {
          tc_fence_after();
#pragma unroll
          for (int cc = 0; cc < DH / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + cc * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st32(tO + cc * 32, o);
          }
        }
        // pass 2: P = exp2(s * scale * log2(e) - m) over this half's 64 keys, 32 at a
        // time, packed into the first 32 columns of the half's own 64 (each store lands on
        // columns this thread has already read); the PV MMA reads keys 0..63 from columns
        // [0, 32) and keys 64..127 from columns [64, 96) of the slot's S region
        float ps0 = 0.f, ps1 = 0.f;  // two independent partial sums
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t v[32];
          if (got) {
            tmem_ld32(tS + c0 + cc * 32, v);
            tmem_wait_ld();
          }
          if (masked) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (c0 + cc * 32 + e > lim) v[e] = 0xff800000u;  // -inf: P = 0
          }
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(v[2 * e]), p.scale_log2, -m_use));
            const float p1 = fast_exp2(fmaf(__uint_as_float(v[2 * e + 1]), p.scale_log2, -m_use));
            if (e & 1) ps1 += p0 + p1; else ps0 += p0 + p1;
            pk[e] = pack_bf16(p0, p1);
          }
          tmem_st16(tS + c0 + cc * 16, pk);
        }
        tmem_wait_st();
        l = l * alpha + (ps0 + ps1);
        m2 = m_new;
        if (r == 0 && hf == 0) sh.dec[s] = 1;
        tc_fence_before();
        warp_arrive(&sh.p_full[s]);
        ++npv;
      }
      if (!ok) break;
      // epilogue: the row's sum from both halves (the exchange slots were last read before
      // the last tile's vote), then O = acc / l on this half's head-dim columns and
      // LSE = (m + log2 l) ln 2
      sh.xsum[s][hf][r] = l;
      named_bar_sync(bar_slot, 256);
      const float lrow = l + sh.xsum[s][hf ^ 1][r];
      bool o_ready = true;
      if (npv > npv_unit0) o_ready = mbar_wait_warp(&sh.o_done[s], (npv - 1) & 1, ast, 23);
      if (!o_ready) continue;  // aborting: the next barrier reduction exits (no barrier below)
      tc_fence_after();
      const float inv_l = (lrow > 0.f) ? 1.f / lrow : 0.f;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.O) +
                            ((static_cast<size_t>(w.b) * p.Lrows + w.qrow0 + q) * p.H + h) * D +
                            hf * DH;
#pragma unroll
      for (int cc = 0; cc < DH / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(tO + cc * 32, o);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int e8 = 0; e8 < 4; ++e8) {
            uint4 pk;
            pk.x = pack_bf16(__uint_as_float(o[e8 * 8 + 0]) * inv_l, __uint_as_float(o[e8 * 8 + 1]) * inv_l);
            pk.y = pack_bf16(__uint_as_float(o[e8 * 8 + 2]) * inv_l, __uint_as_float(o[e8 * 8 + 3]) * inv_l);
            pk.z = pack_bf16(__uint_as_float(o[e8 * 8 + 4]) * inv_l, __uint_as_float(o[e8 * 8 + 5]) * inv_l);
            pk.w = pack_bf16(__uint_as_float(o[e8 * 8 + 6]) * inv_l, __uint_as_float(o[e8 * 8 + 7]) * inv_l);
            *reinterpret_cast<uint4*>(orow + cc * 32 + e8 * 8) = pk;
          }
        }
      }
      if (valid && hf == 0)
        p.LSE[(static_cast<size_t>(w.b) * p.H + h) * p.Lrows + w.qrow0 + q] =
            (m2 + __log2f(lrow)) * kLn2;
      tc_fence_before();
    }
    if (r == 0 && hf == 0) stats_add(p.stats, ns, npv, 0);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tb, 512);
}

}  // namespace

// ---------------------------------------------------------------------------- launch

template <int D, bool kScreen>
static cudaError_t launch_fwd_impl(const CUtensorMap& tq, const CUtensorMap& tk,
                                   const CUtensorMap& tv, const FwdParams& p, int grid,
                                   cudaStream_t stream) {
  using C = FwdCfg<D>;
  auto kern = mala_fwd_kernel<D, kScreen>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<grid, C::THREADS, C::SMEM, stream>>>(tq, tk, tv, p);
  return cudaGetLastError();
}

cudaError_t launch_fwd_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                            const FwdParams& p, int d, bool screen, int grid,
                            cudaStream_t stream) {
  if (d == 128)
    return screen ? launch_fwd_impl<128, true>(tq, tk, tv, p, grid, stream)
                  : launch_fwd_impl<128, false>(tq, tk, tv, p, grid, stream);
  return screen ? launch_fwd_impl<64, true>(tq, tk, tv, p, grid, stream)
                : launch_fwd_impl<64, false>(tq, tk, tv, p, grid, stream);
}

}  // namespace mala
