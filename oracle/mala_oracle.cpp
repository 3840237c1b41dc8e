// MALA CPU oracle: plain fp64 restatement of MassAlloc Attention.
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
// cpu_baseline / reference leg of bench.py may load this library.  It shares no
// code, header, table or constant with the CUDA path and never calls it.
//
// Source: "MassAlloc Attention: Let Attention Allocate Its Own Compute"
//   §2.1  score discovery per legal causal tile, length-normalised tolerance tau/L_q
//   §2.2  Eq. (1)-(3) online forward test, Eq. (4) offline backward test
//   §2.4  split-KV decoding with per-split partial normalisers
//   App. A, Algorithm 1 (forward) and Algorithm 2 (backward); A.1 traversal order
//   App. B, Proposition 1 (the invariants the tests check)
//   §2.3  the same forward serves inference prefill: orc_mala_prefill takes a chunk of
//         queries at the end of a longer key sequence (causal offset Nk - Nq)
//
// Conventions (each one a reading of the page where it is silent or ambiguous):
//   * scores s = scale * <q, k>, natural exp / log (§2.1 absorbs the scale into Q)
//   * square tiles of `blk` rows/keys; tile (i, j) = query block i, key block j
//   * forward visits j = i, i-1, ..., 0 (diagonal first, A.1); only legal tiles
//   * retain iff max over rows of x_q >= 0 (skip needs strict '<' on every row, Eq. 3)
//   * a row whose running sum is zero has x_q = +inf (§2.2, "first legal tile")
//   * tau == 0 means threshold -inf: nothing is skipped (§2.3, tau -> 0 recovers FullAttn)
//   * GQA: query head h reads KV head h / (H / Hkv)
//   * layouts: Q, O, dO, dQ [B, L, H, d]; K, V, dK, dV [B, L, Hkv, d]; LSE [B, H, L]
//   * masks / margins are indexed [b, h, i, j] (T x T per head); -1 = tile not legal
//     or not evaluated, 0 = skipped, 1 = retained.  Margins are natural-log units.
//
// Inputs arrive as float (bf16 or fp32 values, widened exactly); all arithmetic
// is double.  Every function returns 0 on success, a negative code on bad args.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

const double kInf = std::numeric_limits<double>::infinity();

struct Dims {
  int B, H, Hkv, L, d, G, T;
  long long q_off(int b, int t, int h) const {  // [B, L, H, d]
    return (((long long)b * L + t) * H + h) * d;
  }
  long long kv_off(int b, int t, int g) const {  // [B, L, Hkv, d]
    return (((long long)b * L + t) * Hkv + g) * d;
  }
  long long lse_off(int b, int h, int t) const {  // [B, H, L]
    return ((long long)b * H + h) * L + t;
  }
  long long tile_off(int b, int h, int i, int j) const {  // [B, H, T, T]
    return (((long long)b * H + h) * T + i) * T + j;
  }
};

bool bad_dims(int B, int H, int Hkv, int L, int d, int blk) {
  return B <= 0 || H <= 0 || Hkv <= 0 || L <= 0 || d <= 0 || blk <= 0 || H % Hkv != 0;
}

Dims make_dims(int B, int H, int Hkv, int L, int d, int blk) {
  Dims D;
  D.B = B; D.H = H; D.Hkv = Hkv; D.L = L; D.d = d; D.G = H / Hkv;
  D.T = (L + blk - 1) / blk;
  return D;
}

double dot(const float* a, const float* b, int d) {
  double s = 0.0;
  for (int c = 0; c < d; ++c) s += (double)a[c] * (double)b[c];
  return s;
}

// log(tau / L_q), -inf when tau == 0 (no threshold).
double log_threshold(double tau, double Lq) {
  if (tau == 0.0) return -kInf;
  return std::log(tau) - std::log(Lq);
}

// ---------------------------------------------------------------------------
// Dense causal softmax attention, textbook two-pass form, one query row.
// Writes o[d] and returns z = log sum_k exp(s_k) over k <= q.
double dense_row(const Dims& D, const float* Q, const float* K, const float* V, double scale,
                 int b, int h, int q, double* o) {
  const int g = h / D.G;
  const float* qv = Q + D.q_off(b, q, h);
  std::vector<double> s(q + 1);
  double mx = -kInf;
  for (int k = 0; k <= q; ++k) {
    s[k] = scale * dot(qv, K + D.kv_off(b, k, g), D.d);
    if (s[k] > mx) mx = s[k];
  }
  double sum = 0.0;
  for (int k = 0; k <= q; ++k) sum += std::exp(s[k] - mx);
  const double z = mx + std::log(sum);
  for (int c = 0; c < D.d; ++c) o[c] = 0.0;
  for (int k = 0; k <= q; ++k) {
    const double p = std::exp(s[k] - z);
    const float* vv = V + D.kv_off(b, k, g);
    for (int c = 0; c < D.d; ++c) o[c] += p * (double)vv[c];
  }
  return z;
}

// ---------------------------------------------------------------------------
// MALA forward for one (b, h, query block i): Algorithm 1 in its online form.
void mala_fwd_block(const Dims& D, const float* Q, const float* K, const float* V, double scale,
                    double tau, int blk, int b, int h, int i, const signed char* force, double* O,
                    double* LSE, signed char* mask, double* margin) {
  const int g = h / D.G;
  const int q0 = i * blk;
  const int q1 = std::min(D.L, q0 + blk);
  const int nq = q1 - q0;
  std::vector<double> m(nq, -kInf), l(nq, 0.0), acc((size_t)nq * D.d, 0.0), theta(nq);
  for (int r = 0; r < nq; ++r) theta[r] = log_threshold(tau, (double)(q0 + r + 1));  // L_q = q + 1
  std::vector<double> S((size_t)nq * blk);
  std::vector<double> rowmax(nq);
  std::vector<char> has_key(nq);

  for (int j = i; j >= 0; --j) {  // diagonal first, then earlier key blocks
    const int k0 = j * blk;
    const int k1 = std::min(D.L, k0 + blk);
    // score discovery for the whole tile, causal mask at the boundary
    for (int r = 0; r < nq; ++r) {
      const int q = q0 + r;
      rowmax[r] = -kInf;
      has_key[r] = 0;
      const float* qv = Q + D.q_off(b, q, h);
      for (int k = k0; k < k1; ++k) {
        double s = -kInf;
        if (k <= q) {
          s = scale * dot(qv, K + D.kv_off(b, k, g), D.d);
          has_key[r] = 1;
          if (s > rowmax[r]) rowmax[r] = s;
        }
        S[(size_t)r * blk + (k - k0)] = s;
      }
    }
    // Eq. (3): x_q = rowmax - m - log(l) - log(tau / L_q); retain iff some row has x_q >= 0
    double X = -kInf;
    for (int r = 0; r < nq; ++r) {
      if (!has_key[r]) continue;  // rows without a legal key do not constrain the tile
      const double x = (l[r] == 0.0) ? kInf : rowmax[r] - m[r] - std::log(l[r]) - theta[r];
      if (x > X) X = x;
    }
    bool retain = (X >= 0.0);
    const long long to = D.tile_off(b, h, i, j);
    if (force && force[to] >= 0) retain = (force[to] != 0);
    if (mask) mask[to] = retain ? 1 : 0;
    if (margin) margin[to] = X;
    if (!retain) continue;  // a skipped tile leaves m, l, O unchanged
    // online-softmax update on the retained tile
    for (int r = 0; r < nq; ++r) {
      if (!has_key[r]) continue;
      const double mn = std::max(m[r], rowmax[r]);
      const double alpha = std::exp(m[r] - mn);  // exp(-inf) = 0 on the first retained tile
      double psum = 0.0;
      double* a = &acc[(size_t)r * D.d];
      for (int c = 0; c < D.d; ++c) a[c] *= alpha;
      for (int k = k0; k < k1; ++k) {
        const double s = S[(size_t)r * blk + (k - k0)];
        if (s == -kInf) continue;
        const double p = std::exp(s - mn);
        psum += p;
        const float* vv = V + D.kv_off(b, k, g);
        for (int c = 0; c < D.d; ++c) a[c] += p * (double)vv[c];
      }
      l[r] = alpha * l[r] + psum;
      m[r] = mn;
    }
  }
  // finalise: O = acc / l, LSE = m + log l
  for (int r = 0; r < nq; ++r) {
    const int q = q0 + r;
    double* o = O + D.q_off(b, q, h);
    for (int c = 0; c < D.d; ++c) o[c] = acc[(size_t)r * D.d + c] / l[r];
    LSE[D.lse_off(b, h, q)] = m[r] + std::log(l[r]);
  }
}

// ---------------------------------------------------------------------------
// MALA forward, second formulation (cross-check): keeps the explicit retained key
// set R_q of every row and recomputes log Z_q = log sum_{k in R_q} exp(s_qk) from
// scratch at every test (Eq. 1-2 without the m / l recurrence).
void mala_fwd_block_setsum(const Dims& D, const float* Q, const float* K, const float* V,
                           double scale, double tau, int blk, int b, int h, int i, double* O,
                           double* LSE, signed char* mask, double* margin) {
  const int g = h / D.G;
  const int q0 = i * blk;
  const int q1 = std::min(D.L, q0 + blk);
  const int nq = q1 - q0;
  // full score rows for the block (k <= q)
  std::vector<std::vector<double>> s(nq);
  std::vector<std::vector<char>> in_R(nq);
  for (int r = 0; r < nq; ++r) {
    const int q = q0 + r;
    s[r].resize(q + 1);
    in_R[r].assign(q + 1, 0);
    const float* qv = Q + D.q_off(b, q, h);
    for (int k = 0; k <= q; ++k) s[r][k] = scale * dot(qv, K + D.kv_off(b, k, g), D.d);
  }
  for (int j = i; j >= 0; --j) {
    const int k0 = j * blk;
    const int k1 = std::min(D.L, k0 + blk);
    double X = -kInf;
    for (int r = 0; r < nq; ++r) {
      const int q = q0 + r;
      if (k0 > q) continue;
      // largest contribution ratio of this tile for row q, in logs (Eq. 2)
      double top = -kInf;
      for (int k = k0; k < std::min(k1, q + 1); ++k) top = std::max(top, s[r][k]);
      // log Z over the retained set, two-pass logsumexp from scratch
      double zmax = -kInf;
      for (int k = 0; k <= q; ++k)
        if (in_R[r][k]) zmax = std::max(zmax, s[r][k]);
      double x;
      if (zmax == -kInf) {
        x = kInf;  // empty retained set: log-ratio +inf
      } else {
        double zs = 0.0;
        for (int k = 0; k <= q; ++k)
          if (in_R[r][k]) zs += std::exp(s[r][k] - zmax);
        const double logZ = zmax + std::log(zs);
        x = top - logZ - log_threshold(tau, (double)(q + 1));
      }
      X = std::max(X, x);
    }
    const bool retain = (X >= 0.0);
    const long long to = D.tile_off(b, h, i, j);
    if (mask) mask[to] = retain ? 1 : 0;
    if (margin) margin[to] = X;
    if (!retain) continue;
    for (int r = 0; r < nq; ++r) {
      const int q = q0 + r;
      for (int k = k0; k < std::min(k1, q + 1); ++k) in_R[r][k] = 1;
    }
  }
  for (int r = 0; r < nq; ++r) {
    const int q = q0 + r;
    double zmax = -kInf;
    for (int k = 0; k <= q; ++k)
      if (in_R[r][k]) zmax = std::max(zmax, s[r][k]);
    double zs = 0.0;
    for (int k = 0; k <= q; ++k)
      if (in_R[r][k]) zs += std::exp(s[r][k] - zmax);
    const double z = zmax + std::log(zs);
    LSE[D.lse_off(b, h, q)] = z;
    double* o = O + D.q_off(b, q, h);
    for (int c = 0; c < D.d; ++c) o[c] = 0.0;
    for (int k = 0; k <= q; ++k) {
      if (!in_R[r][k]) continue;
      const double p = std::exp(s[r][k] - z);
      const float* vv = V + D.kv_off(b, k, g);
      for (int c = 0; c < D.d; ++c) o[c] += p * (double)vv[c];
    }
  }
}

// ---------------------------------------------------------------------------
// MALA backward, Algorithm 2 with the offline test of Eq. (4).
// Tile decision shared by the key-major (dK, dV) and query-major (dQ) passes.
struct BwdCtx {
  Dims D;
  const float *Q, *K, *V, *dO;
  const double *O, *LSE;
  double scale, tau;
  int blk;
  std::vector<double> Drow;  // D_q = <O_q, dO_q>, [B, H, L]
};

// Evaluates Eq. (4) on tile (b, h, i, j); fills P and dS (blk x blk, row = query) when
// the tile is retained.  Returns the decision; *Y receives the tile margin.
bool bwd_tile(const BwdCtx& C, int b, int h, int i, int j, const signed char* force, double* Y,
              std::vector<double>& P, std::vector<double>& dS) {
  const Dims& D = C.D;
  const int g = h / D.G;
  const int blk = C.blk;
  const int q0 = i * blk, q1 = std::min(D.L, q0 + blk);
  const int k0 = j * blk, k1 = std::min(D.L, k0 + blk);
  P.assign((size_t)blk * blk, 0.0);
  dS.assign((size_t)blk * blk, 0.0);
  std::vector<double> S((size_t)blk * blk, -kInf);
  double Ymax = -kInf;
  for (int q = q0; q < q1; ++q) {
    const float* qv = C.Q + D.q_off(b, q, h);
    const double z = C.LSE[D.lse_off(b, h, q)];
    const double th = log_threshold(C.tau, (double)(q + 1));
    for (int k = k0; k < std::min(k1, q + 1); ++k) {
      const double s = C.scale * dot(qv, C.K + D.kv_off(b, k, g), D.d);
      S[(size_t)(q - q0) * blk + (k - k0)] = s;
      const double y = s - z - th;  // elementwise over legal entries
      if (y > Ymax) Ymax = y;
    }
  }
  bool retain = (Ymax >= 0.0);
  const long long to = D.tile_off(b, h, i, j);
  if (force && force[to] >= 0) retain = (force[to] != 0);
  *Y = Ymax;
  if (!retain) return false;
  for (int q = q0; q < q1; ++q) {
    const double z = C.LSE[D.lse_off(b, h, q)];
    const double Dq = C.Drow[D.lse_off(b, h, q)];
    const float* dov = C.dO + D.q_off(b, q, h);
    for (int k = k0; k < std::min(k1, q + 1); ++k) {
      const size_t e = (size_t)(q - q0) * blk + (k - k0);
      const double p = std::exp(S[e] - z);
      const double dp = dot(dov, C.V + D.kv_off(b, k, g), D.d);
      P[e] = p;
      dS[e] = p * (dp - Dq);
    }
  }
  return true;
}

// dK, dV rows of key block j of KV head g: sum over the group's heads and i >= j.
void bwd_kv_block(const BwdCtx& C, int b, int g, int j, const signed char* force, double* dK,
                  double* dV, signed char* mask, double* margin) {
  const Dims& D = C.D;
  const int blk = C.blk;
  const int k0 = j * blk, k1 = std::min(D.L, k0 + blk);
  for (int k = k0; k < k1; ++k) {
    double* dk = dK + D.kv_off(b, k, g);
    double* dv = dV + D.kv_off(b, k, g);
    for (int c = 0; c < D.d; ++c) dk[c] = dv[c] = 0.0;
  }
  std::vector<double> P, dS;
  for (int h = g * D.G; h < (g + 1) * D.G; ++h) {
    for (int i = j; i < D.T; ++i) {  // query blocks ascending from the diagonal
      double Y;
      const bool keep = bwd_tile(C, b, h, i, j, force, &Y, P, dS);
      const long long to = D.tile_off(b, h, i, j);
      if (mask) mask[to] = keep ? 1 : 0;
      if (margin) margin[to] = Y;
      if (!keep) continue;
      const int q0 = i * blk, q1 = std::min(D.L, q0 + blk);
      for (int q = q0; q < q1; ++q) {
        const float* qv = C.Q + D.q_off(b, q, h);
        const float* dov = C.dO + D.q_off(b, q, h);
        for (int k = k0; k < std::min(k1, q + 1); ++k) {
          const size_t e = (size_t)(q - q0) * blk + (k - k0);
          double* dk = dK + D.kv_off(b, k, g);
          double* dv = dV + D.kv_off(b, k, g);
          for (int c = 0; c < D.d; ++c) {
            dv[c] += P[e] * (double)dov[c];
            dk[c] += C.scale * dS[e] * (double)qv[c];
          }
        }
      }
    }
  }
}

// dQ rows of query block i of head h: sum over key blocks j <= i.
void bwd_q_block(const BwdCtx& C, int b, int h, int i, const signed char* force, double* dQ) {
  const Dims& D = C.D;
  const int g = h / D.G;
  const int blk = C.blk;
  const int q0 = i * blk, q1 = std::min(D.L, q0 + blk);
  for (int q = q0; q < q1; ++q) {
    double* dq = dQ + D.q_off(b, q, h);
    for (int c = 0; c < D.d; ++c) dq[c] = 0.0;
  }
  std::vector<double> P, dS;
  for (int j = 0; j <= i; ++j) {
    double Y;
    if (!bwd_tile(C, b, h, i, j, force, &Y, P, dS)) continue;
    const int k0 = j * blk, k1 = std::min(D.L, k0 + blk);
    for (int q = q0; q < q1; ++q) {
      double* dq = dQ + D.q_off(b, q, h);
      for (int k = k0; k < std::min(k1, q + 1); ++k) {
        const size_t e = (size_t)(q - q0) * blk + (k - k0);
        const float* kv = C.K + D.kv_off(b, k, g);
        for (int c = 0; c < D.d; ++c) dq[c] += C.scale * dS[e] * (double)kv[c];
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Chunked prefill: the forward of Algorithm 1 for a chunk of Nq queries that are the
// last Nq positions of a sequence of Nk >= Nq keys ("the same forward operator serves
// ... inference prefill", §2.3).  Query row q (0-based in the chunk) sits at absolute
// position p = off + q, off = Nk - Nq; it attends to keys k <= p, and L_q = p + 1.
// Query block i holds chunk rows [i*blk, (i+1)*blk); it visits the key blocks that hold
// a legal key of one of its rows, from the last one (the block of its last row's
// position) down to 0.
struct PDims {
  int B, H, Hkv, Nq, Nk, off, d, G, Tq, Tk;
  long long q_off(int b, int q, int h) const { return (((long long)b * Nq + q) * H + h) * d; }
  long long kv_off(int b, int k, int g) const { return (((long long)b * Nk + k) * Hkv + g) * d; }
  long long lse_off(int b, int h, int q) const { return ((long long)b * H + h) * Nq + q; }
  long long tile_off(int b, int h, int i, int j) const {
    return (((long long)b * H + h) * Tq + i) * Tk + j;
  }
};

void prefill_block(const PDims& D, const float* Q, const float* K, const float* V, double scale,
                   double tau, int blk, int b, int h, int i, const signed char* force, double* O,
                   double* LSE, signed char* mask, double* margin) {
  const int g = h / D.G;
  const int q0 = i * blk;
  const int q1 = std::min(D.Nq, q0 + blk);
  const int nq = q1 - q0;
  std::vector<double> m(nq, -kInf), l(nq, 0.0), acc((size_t)nq * D.d, 0.0), theta(nq);
  for (int r = 0; r < nq; ++r) theta[r] = log_threshold(tau, (double)(D.off + q0 + r + 1));
  std::vector<double> S((size_t)nq * blk), rowmax(nq);
  std::vector<char> has_key(nq);
  const int j_last = (D.off + q1 - 1) / blk;
  for (int j = j_last; j >= 0; --j) {
    const int k0 = j * blk;
    const int k1 = std::min(D.Nk, k0 + blk);
    for (int r = 0; r < nq; ++r) {
      const int pos = D.off + q0 + r;
      rowmax[r] = -kInf;
      has_key[r] = 0;
      const float* qv = Q + D.q_off(b, q0 + r, h);
      for (int k = k0; k < k1; ++k) {
        double sc = -kInf;
        if (k <= pos) {
          sc = scale * dot(qv, K + D.kv_off(b, k, g), D.d);
          has_key[r] = 1;
          if (sc > rowmax[r]) rowmax[r] = sc;
        }
        S[(size_t)r * blk + (k - k0)] = sc;
      }
    }
    double X = -kInf;  // Eq. (3) over the rows with a legal key in this tile
    for (int r = 0; r < nq; ++r) {
      if (!has_key[r]) continue;
      const double x = (l[r] == 0.0) ? kInf : rowmax[r] - m[r] - std::log(l[r]) - theta[r];
      if (x > X) X = x;
    }
    bool retain = (X >= 0.0);
    const long long to = D.tile_off(b, h, i, j);
    if (force && force[to] >= 0) retain = (force[to] != 0);
    if (mask) mask[to] = retain ? 1 : 0;
    if (margin) margin[to] = X;
    if (!retain) continue;
    for (int r = 0; r < nq; ++r) {
      if (!has_key[r]) continue;
      const double mn = std::max(m[r], rowmax[r]);
      const double alpha = std::exp(m[r] - mn);
      double psum = 0.0;
      double* a = &acc[(size_t)r * D.d];
      for (int c = 0; c < D.d; ++c) a[c] *= alpha;
      for (int k = k0; k < k1; ++k) {
        const double sc = S[(size_t)r * blk + (k - k0)];
        if (sc == -kInf) continue;
        const double pr = std::exp(sc - mn);
        psum += pr;
        const float* vv = V + D.kv_off(b, k, g);
        for (int c = 0; c < D.d; ++c) a[c] += pr * (double)vv[c];
      }
      l[r] = alpha * l[r] + psum;
      m[r] = mn;
    }
  }
  for (int r = 0; r < nq; ++r) {
    double* o = O + D.q_off(b, q0 + r, h);
    for (int c = 0; c < D.d; ++c) o[c] = acc[(size_t)r * D.d + c] / l[r];
    LSE[D.lse_off(b, h, q0 + r)] = m[r] + std::log(l[r]);
  }
}

}  // namespace

extern "C" {

int orc_version(void) { return 1; }

// Threads the parallel loops below use (1 without OpenMP): the core count that the timed
// CPU baseline reports.
int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// Dense causal attention (FullAttn), rows of the listed (b, h, i) blocks of `blk`
// rows (all rows when units == NULL).  O [B,L,H,d], LSE [B,H,L].
int orc_dense_fwd(const float* Q, const float* K, const float* V, int B, int H, int Hkv, int L,
                  int d, double scale, int blk, const int* units, int n_units, double* O,
                  double* LSE) {
  if (bad_dims(B, H, Hkv, L, d, blk)) return -1;
  const Dims D = make_dims(B, H, Hkv, L, d, blk);
  const long long n = units ? n_units : (long long)B * H * D.T;
#pragma omp parallel for schedule(dynamic, 1)
  for (long long u = 0; u < n; ++u) {
    int b, h, i;
    if (units) {
      b = units[3 * u]; h = units[3 * u + 1]; i = units[3 * u + 2];
    } else {
      b = (int)(u / ((long long)H * D.T)); h = (int)((u / D.T) % H); i = (int)(u % D.T);
    }
    for (int q = i * blk; q < std::min(L, (i + 1) * blk); ++q)
      LSE[D.lse_off(b, h, q)] = dense_row(D, Q, K, V, scale, b, h, q, O + D.q_off(b, q, h));
  }
  return 0;
}

// Dense causal attention backward (exact gradient of FullAttn) for all rows.
// dO given; dQ [B,L,H,d], dK/dV [B,L,Hkv,d] (summed over each KV head's query heads).
int orc_dense_bwd(const float* Q, const float* K, const float* V, const float* dO, int B, int H,
                  int Hkv, int L, int d, double scale, double* dQ, double* dK, double* dV) {
  if (bad_dims(B, H, Hkv, L, d, 1)) return -1;
  const Dims D = make_dims(B, H, Hkv, L, d, 1);
  const size_t nq = (size_t)B * L * H * d, nk = (size_t)B * L * Hkv * d;
  std::memset(dQ, 0, nq * sizeof(double));
  std::memset(dK, 0, nk * sizeof(double));
  std::memset(dV, 0, nk * sizeof(double));
  std::vector<double> o(d);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h) {
      const int g = h / D.G;
      for (int q = 0; q < L; ++q) {
        const double z = dense_row(D, Q, K, V, scale, b, h, q, o.data());
        const float* qv = Q + D.q_off(b, q, h);
        const float* dov = dO + D.q_off(b, q, h);
        double Dq = 0.0;
        for (int c = 0; c < d; ++c) Dq += o[c] * (double)dov[c];
        double* dq = dQ + D.q_off(b, q, h);
        for (int k = 0; k <= q; ++k) {
          const float* kv = K + D.kv_off(b, k, g);
          const double p = std::exp(scale * dot(qv, kv, d) - z);
          const double dp = dot(dov, V + D.kv_off(b, k, g), d);
          const double ds = p * (dp - Dq);
          double* dk = dK + D.kv_off(b, k, g);
          double* dv = dV + D.kv_off(b, k, g);
          for (int c = 0; c < d; ++c) {
            dv[c] += p * (double)dov[c];
            dk[c] += scale * ds * (double)qv[c];
            dq[c] += scale * ds * (double)kv[c];
          }
        }
      }
    }
  return 0;
}

// MALA forward (Algorithm 1, online form).  units: (b, h, i) triplets or NULL for all
// blocks.  force: [B,H,T,T] decisions to follow instead of the test (-1 entries fall
// back to the test), or NULL.  mask / margin: [B,H,T,T] outputs or NULL.
int orc_mala_fwd(const float* Q, const float* K, const float* V, int B, int H, int Hkv, int L,
                 int d, double scale, double tau, int blk, const int* units, int n_units,
                 const signed char* force, double* O, double* LSE, signed char* mask,
                 double* margin) {
  if (bad_dims(B, H, Hkv, L, d, blk) || !(tau >= 0.0)) return -1;
  const Dims D = make_dims(B, H, Hkv, L, d, blk);
  const long long n = units ? n_units : (long long)B * H * D.T;
#pragma omp parallel for schedule(dynamic, 1)
  for (long long u = 0; u < n; ++u) {
    int b, h, i;
    if (units) {
      b = units[3 * u]; h = units[3 * u + 1]; i = units[3 * u + 2];
    } else {
      b = (int)(u / ((long long)H * D.T)); h = (int)((u / D.T) % H); i = (int)(u % D.T);
    }
    mala_fwd_block(D, Q, K, V, scale, tau, blk, b, h, i, force, O, LSE, mask, margin);
  }
  return 0;
}

// Chunked prefill forward (see prefill_block).  Q, O [B, Nq, H, d]; K, V [B, Nk, Hkv, d];
// LSE [B, H, Nq]; mask / margin [B, H, Tq, Tk].  units: (b, h, i) or NULL for all.
int orc_mala_prefill(const float* Q, const float* K, const float* V, int B, int H, int Hkv,
                     int Nq, int Nk, int d, double scale, double tau, int blk, const int* units,
                     int n_units, const signed char* force, double* O, double* LSE,
                     signed char* mask, double* margin) {
  if (bad_dims(B, H, Hkv, Nq, d, blk) || Nk < Nq || !(tau >= 0.0)) return -1;
  PDims D;
  D.B = B; D.H = H; D.Hkv = Hkv; D.Nq = Nq; D.Nk = Nk; D.off = Nk - Nq; D.d = d;
  D.G = H / Hkv; D.Tq = (Nq + blk - 1) / blk; D.Tk = (Nk + blk - 1) / blk;
  const long long n = units ? n_units : (long long)B * H * D.Tq;
#pragma omp parallel for schedule(dynamic, 1)
  for (long long u = 0; u < n; ++u) {
    int b, h, i;
    if (units) {
      b = units[3 * u]; h = units[3 * u + 1]; i = units[3 * u + 2];
    } else {
      b = (int)(u / ((long long)H * D.Tq)); h = (int)((u / D.Tq) % H); i = (int)(u % D.Tq);
    }
    prefill_block(D, Q, K, V, scale, tau, blk, b, h, i, force, O, LSE, mask, margin);
  }
  return 0;
}

// MALA forward, explicit retained-set formulation (independent cross-check).
int orc_mala_fwd_setsum(const float* Q, const float* K, const float* V, int B, int H, int Hkv,
                        int L, int d, double scale, double tau, int blk, double* O, double* LSE,
                        signed char* mask, double* margin) {
  if (bad_dims(B, H, Hkv, L, d, blk) || !(tau >= 0.0)) return -1;
  const Dims D = make_dims(B, H, Hkv, L, d, blk);
  const long long n = (long long)B * H * D.T;
#pragma omp parallel for schedule(dynamic, 1)
  for (long long u = 0; u < n; ++u) {
    const int b = (int)(u / ((long long)H * D.T)), h = (int)((u / D.T) % H), i = (int)(u % D.T);
    mala_fwd_block_setsum(D, Q, K, V, scale, tau, blk, b, h, i, O, LSE, mask, margin);
  }
  return 0;
}

// MALA backward (Algorithm 2).  O and LSE are the forward's outputs (the oracle's own,
// or another implementation's to condition on them).  kv_units: (b, g, j) key blocks
// whose dK / dV rows are computed (NULL = all); q_units: (b, h, i) query blocks whose
// dQ rows are computed (NULL = all; n_q == 0 with a non-NULL pointer = none).
// mask / margin are written by the key-block pass only.
int orc_mala_bwd(const float* Q, const float* K, const float* V, const double* O,
                 const double* LSE, const float* dO, int B, int H, int Hkv, int L, int d,
                 double scale, double tau, int blk, const int* kv_units, int n_kv,
                 const int* q_units, int n_q, const signed char* force, double* dQ, double* dK,
                 double* dV, signed char* mask, double* margin) {
  if (bad_dims(B, H, Hkv, L, d, blk) || !(tau >= 0.0)) return -1;
  BwdCtx C;
  C.D = make_dims(B, H, Hkv, L, d, blk);
  C.Q = Q; C.K = K; C.V = V; C.dO = dO; C.O = O; C.LSE = LSE;
  C.scale = scale; C.tau = tau; C.blk = blk;
  // D_q = rowsum(O o dO) from the forward output (Algorithm 2, softmax-backward term)
  C.Drow.assign((size_t)B * H * L, 0.0);
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int q = 0; q < L; ++q) {
        double s = 0.0;
        const double* o = O + C.D.q_off(b, q, h);
        const float* dov = dO + C.D.q_off(b, q, h);
        for (int c = 0; c < d; ++c) s += o[c] * (double)dov[c];
        C.Drow[C.D.lse_off(b, h, q)] = s;
      }
  const Dims& D = C.D;
  const long long nkv = kv_units ? n_kv : (long long)B * Hkv * D.T;
#pragma omp parallel for schedule(dynamic, 1)
  for (long long u = 0; u < nkv; ++u) {
    int b, g, j;
    if (kv_units) {
      b = kv_units[3 * u]; g = kv_units[3 * u + 1]; j = kv_units[3 * u + 2];
    } else {
      b = (int)(u / ((long long)Hkv * D.T)); g = (int)((u / D.T) % Hkv); j = (int)(u % D.T);
    }
    bwd_kv_block(C, b, g, j, force, dK, dV, mask, margin);
  }
  const long long nqu = q_units ? n_q : (long long)B * H * D.T;
#pragma omp parallel for schedule(dynamic, 1)
  for (long long u = 0; u < nqu; ++u) {
    int b, h, i;
    if (q_units) {
      b = q_units[3 * u]; h = q_units[3 * u + 1]; i = q_units[3 * u + 2];
    } else {
      b = (int)(u / ((long long)H * D.T)); h = (int)((u / D.T) % H); i = (int)(u % D.T);
    }
    bwd_q_block(C, b, h, i, force, dQ);
  }
  return 0;
}

// MALA split-KV decode (§2.4): one query row per (b, h) sees all Nk cached keys,
// L_0 = Nk.  Key tiles of `blk`; split s owns tiles [s*T/S, (s+1)*T/S) (integer
// division) and visits them newest first with its own m, l.  Splits are merged by
// the log-sum-exp reduction.  q [B,H,d]; K, V [B,Nk,Hkv,d]; O [B,H,d]; LSE [B,H];
// mask / margin [B,H,T]; part_o [B,H,S,d] / part_z [B,H,S] per-split results (or NULL).
int orc_mala_decode(const float* q, const float* K, const float* V, int B, int H, int Hkv,
                    int Nk, int d, double scale, double tau, int blk, int num_splits,
                    const int* units, int n_units, const signed char* force, double* O,
                    double* LSE, signed char* mask, double* margin, double* part_o,
                    double* part_z) {
  if (bad_dims(B, H, Hkv, Nk, d, blk) || !(tau >= 0.0)) return -1;
  const int G = H / Hkv;
  const int T = (Nk + blk - 1) / blk;
  const int S = num_splits;
  if (S < 1 || S > T) return -2;
  const double theta = log_threshold(tau, (double)Nk);
  const long long n = units ? n_units : (long long)B * H;
#pragma omp parallel for schedule(dynamic, 1)
  for (long long u = 0; u < n; ++u) {
    int b, h;
    if (units) {
      b = units[2 * u]; h = units[2 * u + 1];
    } else {
      b = (int)(u / H); h = (int)(u % H);
    }
    const int g = h / G;
    const float* qv = q + ((long long)b * H + h) * d;
    std::vector<double> zs(S), os((size_t)S * d);
    std::vector<double> s(blk), acc(d);
    for (int sp = 0; sp < S; ++sp) {
      const int t_lo = (int)((long long)sp * T / S), t_hi = (int)((long long)(sp + 1) * T / S);
      double m = -kInf, l = 0.0;
      for (int c = 0; c < d; ++c) acc[c] = 0.0;
      for (int t = t_hi - 1; t >= t_lo; --t) {  // newest tile of the split first
        const int k0 = t * blk, k1 = std::min(Nk, k0 + blk);
        double r = -kInf;
        for (int k = k0; k < k1; ++k) {
          s[k - k0] = scale * dot(qv, K + (((long long)b * Nk + k) * Hkv + g) * d, d);
          r = std::max(r, s[k - k0]);
        }
        const double x = (l == 0.0) ? kInf : r - m - std::log(l) - theta;
        bool retain = (x >= 0.0);
        const long long to = ((long long)b * H + h) * T + t;
        if (force && force[to] >= 0) retain = (force[to] != 0);
        if (mask) mask[to] = retain ? 1 : 0;
        if (margin) margin[to] = x;
        if (!retain) continue;
        const double mn = std::max(m, r);
        const double alpha = std::exp(m - mn);
        double psum = 0.0;
        for (int c = 0; c < d; ++c) acc[c] *= alpha;
        for (int k = k0; k < k1; ++k) {
          const double p = std::exp(s[k - k0] - mn);
          psum += p;
          const float* vv = V + (((long long)b * Nk + k) * Hkv + g) * d;
          for (int c = 0; c < d; ++c) acc[c] += p * (double)vv[c];
        }
        l = alpha * l + psum;
        m = mn;
      }
      zs[sp] = m + std::log(l);
      for (int c = 0; c < d; ++c) os[(size_t)sp * d + c] = acc[c] / l;
    }
    // normaliser-aware merge: z = log sum_s exp(z_s), o = sum_s exp(z_s - z) o_s
    double zmax = -kInf;
    for (int sp = 0; sp < S; ++sp) zmax = std::max(zmax, zs[sp]);
    double tot = 0.0;
    for (int sp = 0; sp < S; ++sp) tot += std::exp(zs[sp] - zmax);
    const double z = zmax + std::log(tot);
    LSE[(long long)b * H + h] = z;
    double* o = O + ((long long)b * H + h) * d;
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (int sp = 0; sp < S; ++sp) {
      const double w = std::exp(zs[sp] - z);
      for (int c = 0; c < d; ++c) o[c] += w * os[(size_t)sp * d + c];
      if (part_z) part_z[((long long)b * H + h) * S + sp] = zs[sp];
      if (part_o)
        for (int c = 0; c < d; ++c) part_o[(((long long)b * H + h) * S + sp) * d + c] = os[(size_t)sp * d + c];
    }
  }
  return 0;
}

}  // extern "C"
