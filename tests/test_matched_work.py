"""The matched-work allocation study (MassAlloc Attention §3 Table 1, App. C.2), on the CPU:
its dense reference and metrics are pinned against the oracle's MALA forward and torch's
dense attention, and its allocations against their defining properties."""

import numpy as np
import pytest

from mass_adaptive_sparse_fwd_b200 import matched_work as MW
from tests.test_oracle import _rand, _sdpa


def _study_inputs(seed, X=2, L=96, H=4, Hkv=2, d=16):
    Qs, Ks, Vs = [], [], []
    for x in range(X):
        Q, K, V, _ = _rand(1, L, H, Hkv, d, seed=seed + x, peak=5.0)
        Qs.append(Q); Ks.append(K); Vs.append(V)
    return np.concatenate(Qs), np.concatenate(Ks), np.concatenate(Vs)


def test_mala_metrics_match_the_oracle(orc):
    """With the oracle's own MALA decisions, the study's omitted mass equals
    1 - exp(LSE_mala - LSE_dense) from the oracle and torch, and its output error equals
    the oracle's MALA output against torch's dense output."""
    Q, K, V = _study_inputs(80)
    scale, blk = 0.25, 16
    masks, om_ref, rel_ref = [], [], []
    for x in range(Q.shape[0]):
        O_m, LSE_m, mask, _ = orc.mala_fwd(Q[x:x + 1], K[x:x + 1], V[x:x + 1], scale, 1.0, blk=blk)
        O_d, LSE_d = _sdpa(Q[x:x + 1], K[x:x + 1], V[x:x + 1], scale)
        masks.append(mask)
        eps = 1.0 - np.exp(LSE_m - LSE_d)  # [1, H, L]
        for h in range(Q.shape[2]):
            for i in range(mask.shape[-1]):
                rows = slice(i * blk, (i + 1) * blk)
                om_ref.append(eps[0, h, rows].mean())
                a, b = O_m[0, rows, h], O_d[0, rows, h]
                rel_ref.append(np.linalg.norm(a - b) / np.linalg.norm(b))
    res = MW.evaluate(Q, K, V, scale, np.concatenate(masks), tile=blk)
    assert (np.concatenate(masks) == 0).any()
    np.testing.assert_allclose(res["mala"]["omitted_mass_pct"], 100 * np.mean(om_ref), rtol=1e-9,
                               atol=1e-12)
    np.testing.assert_allclose(res["mala"]["rel_l2_pct"], 100 * np.mean(rel_ref), rtol=1e-9,
                               atol=1e-12)


def test_controls_match_work_and_the_oracle_control_is_optimal(orc):
    Q, K, V = _study_inputs(90, X=3)
    scale, blk = 0.25, 16
    masks = np.concatenate([orc.mala_fwd(Q[x:x + 1], K[x:x + 1], V[x:x + 1], scale, 1.0,
                                         blk=blk)[2] for x in range(3)])
    res = MW.evaluate(Q, K, V, scale, masks, tile=blk)
    tiles = {k: res[k]["tiles"] for k in ("mala", "per_instance", "static_head_pos",
                                          "position_only")}
    assert len(set(tiles.values())) == 1  # exactly matched total work
    # for the same per-block budget, the top-mass tiles omit no more mass than MALA's
    assert res["per_instance"]["omitted_mass_pct"] <= res["mala"]["omitted_mass_pct"] + 1e-12


def test_full_budget_omits_nothing():
    Q, K, V = _study_inputs(95, X=1)
    T = 96 // 16
    full = np.broadcast_to(np.tril(np.ones((T, T), np.int8)), (1, 4, T, T)).copy()
    res = MW.evaluate(Q, K, V, 0.25, full, tile=16)
    for k in ("mala", "per_instance", "static_head_pos", "position_only"):
        assert abs(res[k]["omitted_mass_pct"]) < 1e-10 and res[k]["rel_l2_pct"] < 1e-9


def test_allocations_are_integer_exact_and_data_independent():
    rng = np.random.default_rng(3)
    counts = rng.integers(1, 5, size=(3, 4, 6))
    counts = np.minimum(counts, np.arange(1, 7)[None, None, :])
    a = MW.allocations(counts)
    for k, v in a.items():
        assert v.sum() == counts.sum() and v.dtype.kind == "i"
    # the static allocation of a (head, block) cell depends only on the cell's total
    perm = counts[[2, 0, 1]]
    b = MW.allocations(perm)
    np.testing.assert_array_equal(a["static_head_pos"], b["static_head_pos"])
    np.testing.assert_array_equal(a["position_only"], b["position_only"])
    # and stays within the legal tiles of each block
    assert (a["static_head_pos"] <= np.arange(1, 7)).all()
