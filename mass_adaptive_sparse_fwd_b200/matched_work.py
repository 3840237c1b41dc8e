"""Matched-work allocation study on synthetic states.

"MassAlloc Attention: Let Attention Allocate Its Own Compute", §3 ("Normalized-Mass
Allocation at Matched Work", Table 1) and App. C.2.  Every policy keeps the same total
number of post-score key tiles as MALA realized; the controls rank the candidate key
tiles of each decision (input, head, 128-row query block) by their finalized dense
("reference") probability mass and keep the highest-mass ones.  They differ only in how
many tiles each decision receives:

  per_instance       exactly the count MALA realized for that decision;
  static_head_pos    the count averaged over inputs, per (head, query block);
  position_only      the count averaged over inputs and heads, per query block.

Averages are turned into integers without looking at the data: the budget of a cell
(the sum of MALA's counts over the instances the average spans) is spread as evenly as
possible over those instances in a fixed order, so totals match MALA's exactly.

Metrics per decision (App. C.2): omitted mass = mean over the block's rows of
1 - exp(LSE_retained - LSE_dense), i.e. the dense probability of the omitted keys, and
the relative output L2 error ||O_retained - O_dense|| / ||O_dense|| over the block, where
O_retained is softmax attention renormalised over the retained tiles.  Every policy is
evaluated this way in fp64, so the comparison isolates the allocation (MALA's bf16 output
rounding is not part of it).  Means are pooled over decisions and reported in percent.

The dense reference here is plain fp64 softmax attention (torch library ops, on the CPU
for the tests and on the GPU for the 8K study, where it is not the timed path); MALA's
decisions come from the GPU kernel's tile mask (``run_study``) or from any [X,H,T,T]
mask (``evaluate``).
"""

from __future__ import annotations

import json

import numpy as np

TILE = 128


def dense_reference(Q, K, V, scale, h, g, b=0, tile=TILE, device="cpu"):
    """fp64 dense causal attention of one head (torch, on `device`): returns P [L, L]
    (probabilities), O [L, d] and the per-(row, key tile) mass [L, T]."""
    import torch

    q = torch.as_tensor(Q[b, :, h], dtype=torch.float64, device=device)
    k = torch.as_tensor(K[b, :, g], dtype=torch.float64, device=device)
    v = torch.as_tensor(V[b, :, g], dtype=torch.float64, device=device)
    L = q.shape[0]
    S = (q @ k.T) * scale
    S.masked_fill_(torch.ones(L, L, dtype=torch.bool, device=device).triu_(1), float("-inf"))
    P = torch.softmax(S, dim=1)
    del S
    T = -(-L // tile)
    mass = torch.nn.functional.pad(P, (0, T * tile - L)).view(L, T, tile).sum(dim=2)
    return P, P @ v, mass, v


def _spread(total, n):
    """`total` split over n slots as evenly as possible (fixed order)."""
    base, extra = divmod(int(total), n)
    return np.array([base + (1 if i < extra else 0) for i in range(n)], dtype=np.int64)


def allocations(counts):
    """counts [X, H, T] (MALA's retained tiles per decision) -> dict of policy -> counts."""
    X, H, T = counts.shape
    shp = np.zeros_like(counts)
    pos = np.zeros_like(counts)
    for i in range(T):
        for h in range(H):
            shp[:, h, i] = _spread(counts[:, h, i].sum(), X)
        flat = _spread(counts[:, :, i].sum(), X * H)
        pos[:, :, i] = flat.reshape(X, H)
    return {"mala": counts, "per_instance": counts.copy(), "static_head_pos": shp,
            "position_only": pos}


def block_metrics(P, O_dense, V, keep_tiles, i, tile=TILE):
    """Omitted mass (mean over rows) and relative output L2 error of query block i when
    the key tiles in `keep_tiles` are retained (torch fp64 tensors)."""
    import torch

    L = P.shape[0]
    r0, r1 = i * tile, min(L, (i + 1) * tile)
    cols = torch.zeros(L, dtype=torch.float64, device=P.device)
    for j in keep_tiles:
        cols[j * tile:min(L, (j + 1) * tile)] = 1.0
    Pb = P[r0:r1] * cols[None, :]
    kept = Pb.sum(dim=1)
    omitted = float((1.0 - kept).mean())
    Ob = (Pb @ V) / kept[:, None]
    Od = O_dense[r0:r1]
    rel = float(torch.linalg.norm(Ob - Od) / max(float(torch.linalg.norm(Od)), 1e-300))
    return omitted, rel


def evaluate(Q, K, V, scale, mala_mask, tile=TILE, device="cpu"):
    """Q [X,L,H,d], K/V [X,L,Hkv,d] (X inputs), mala_mask [X,H,T,T] (1 = retained) ->
    per-policy mean omitted mass and relative L2 error (percent), plus slot totals."""
    X, L, H, _ = Q.shape
    G = H // K.shape[2]
    T = -(-L // tile)
    legal = np.tril(np.ones((T, T), dtype=bool))
    counts = np.where(legal[None, None], mala_mask == 1, False).sum(axis=3).astype(np.int64)
    alloc = allocations(counts)
    acc = {k: {"omitted": [], "rel_l2": []} for k in alloc}
    for x in range(X):
        for h in range(H):
            P, Od, mass, Vx = dense_reference(Q, K, V, scale, h, h // G, b=x, tile=tile,
                                              device=device)
            mass = mass.cpu().numpy()
            for i in range(T):
                r0, r1 = i * tile, min(L, (i + 1) * tile)
                region = mass[r0:r1, :i + 1].sum(axis=0)  # block mass of each legal tile
                order = np.argsort(-region, kind="stable")
                for name, a in alloc.items():
                    if name == "mala":
                        keep = np.nonzero(mala_mask[x, h, i, :i + 1] == 1)[0]
                    else:
                        keep = order[:int(a[x, h, i])]
                    om, rel = block_metrics(P, Od, Vx, keep, i, tile)
                    acc[name]["omitted"].append(om)
                    acc[name]["rel_l2"].append(rel)
    legal_tiles = int(X * H * legal.sum())
    out = {"decisions": X * H * T, "legal_tiles": legal_tiles,
           "slots_per_query": float(counts.sum()) * tile * tile / (X * H * L)}
    for name in alloc:
        out[name] = {"tiles": int(alloc[name].sum()),
                     "omitted_mass_pct": 100.0 * float(np.mean(acc[name]["omitted"])),
                     "rel_l2_pct": 100.0 * float(np.mean(acc[name]["rel_l2"]))}
    return out


def run_study(workload="prevvar8k", seeds=(8, 18, 28, 38), tau=1.0, L=None, device="cuda",
              on_decisions=None):
    """MALA's decisions from the GPU forward (tile mask) on X seeded instances of a
    workload (optionally at another length L), then ``evaluate``.  ``on_decisions``, if
    given, is called as on_decisions(w, inp, mask, margin) for every instance with the
    exact mask the study consumes and the forward's exported test margins (the
    library's debug hook is on for those calls), so a caller can audit the decisions."""
    import torch

    from . import mala, synth

    base = synth.WORKLOADS[workload]
    Qs, Ks, Vs, masks = [], [], [], []
    for sd in seeds:
        w = synth.Workload(base.name, base.B, base.H, base.H_kv, base.L, base.d, base.dtype,
                           base.structure, sd)
        inp = synth.make_training(w, L=L)
        q, k, v = (torch.from_numpy(inp[n]).to(device).to(torch.bfloat16)
                   for n in ("Q", "K", "V"))
        T = mala.n_tiles(inp["Q"].shape[1])
        m = torch.zeros((w.B, w.H, T, T), dtype=torch.uint8, device=device)
        if on_decisions is None:
            mala.mala_fwd(q, k, v, w.scale, tau, tile_mask=m)
        else:
            margin = torch.empty(w.B * w.H * T * T, dtype=torch.float32, device=device)
            with mala.debug_margins(margin):
                mala.mala_fwd(q, k, v, w.scale, tau, tile_mask=m)
        torch.cuda.synchronize()
        if on_decisions is not None:
            on_decisions(w, inp, m.cpu().numpy(), margin.view(w.B, w.H, T, T).cpu().numpy())
        Qs.append(inp["Q"][:1]); Ks.append(inp["K"][:1]); Vs.append(inp["V"][:1])
        masks.append(m.cpu().numpy()[:1])
    res = evaluate(np.concatenate(Qs), np.concatenate(Ks), np.concatenate(Vs), base.scale,
                   np.concatenate(masks), device=device)
    res["workload"] = (f"{workload}{'' if L is None else f' at L={L}'} x {len(seeds)} seeds "
                       f"{list(seeds)}, tau = {tau}")
    return res


if __name__ == "__main__":
    import argparse

    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", default="prevvar8k")
    ap.add_argument("--seeds", default="8,18,28,38")
    ap.add_argument("--tau", type=float, default=1.0)
    ap.add_argument("--length", type=int, default=None)
    a = ap.parse_args()
    print(json.dumps(run_study(a.workload, tuple(int(s) for s in a.seeds.split(",")), a.tau,
                               a.length)))
