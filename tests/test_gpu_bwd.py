"""GPU parity of the MALA backward (C ABI -> sm_100a kernels) against the fp64 oracle.

The oracle runs in conditioned mode: it takes the GPU forward's O and LSE and follows
the GPU's backward tile decisions (each of which is checked against the oracle's own
margin first), so the gradients are compared on the same retained support."""

import numpy as np
import pytest
import torch

from mass_adaptive_sparse_fwd_b200 import synth
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mala():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from mass_adaptive_sparse_fwd_b200 import mala as m

    return m


def run_fwd_bwd(mala, inp, w, tau, flags=0):
    Q, K, V, dO = (P.to_dev(inp[k], w.dtype) for k in ("Q", "K", "V", "dO"))
    B, L, H, d = Q.shape
    Hkv = K.shape[2]
    T = mala.n_tiles(L)
    fmask = torch.full((B, H, T, T), 255, dtype=torch.uint8, device="cuda")
    bmask = torch.full((B, H, T, T), 255, dtype=torch.uint8, device="cuda")
    fmargin = P.margin_buffer(B * H * T * T)
    bmargin = P.margin_buffer(B * H * T * T)
    wsf = mala.alloc_workspace(mala.fwd_workspace_bytes(B, H, Hkv, L, d), "cuda")
    wsb = mala.alloc_workspace(mala.bwd_workspace_bytes(B, H, Hkv, L, d), "cuda")
    with mala.debug_margins(fmargin):
        O, LSE = mala.mala_fwd(Q, K, V, w.scale, tau, flags=flags, workspace=wsf, tile_mask=fmask)
    with mala.debug_margins(bmargin):
        dQ, dK, dV = mala.mala_bwd(Q, K, V, O, LSE, dO, w.scale, tau, flags=flags, workspace=wsb,
                                   tile_mask=bmask)
    torch.cuda.synchronize()
    assert mala.read_device_error(wsf) == 0
    assert mala.read_device_error(wsb) == 0
    # the backward call's work counters agree with its tile decisions
    legal = P.fwd_legal(B, H, T)
    bm = bmask.cpu().numpy()
    st = mala.get_stats(wsb)
    assert st["legal_tiles"] == legal.sum() and st["retained_tiles"] == (bm[legal] == 1).sum()
    cpu = lambda t: t.float().cpu().numpy()
    return (cpu(O), cpu(LSE), fmask.cpu().numpy(), cpu(dQ), cpu(dK), cpu(dV), bm,
            fmargin.view(B, H, T, T).cpu().numpy(), bmargin.view(B, H, T, T).cpu().numpy())


def check_bwd(orc, mala, w, inp, tau, kv_units=None, q_units=None, flags=0, max_flips=0):
    O, LSE, fmask, dQ, dK, dV, bmask, fmg, bmg = run_fwd_bwd(mala, inp, w, tau, flags)
    B, L, H, d = inp["Q"].shape
    Hkv = inp["K"].shape[2]
    T = (L + 127) // 128
    legal_all = P.fwd_legal(B, H, T)
    assert (bmask[~legal_all] == 255).all() and np.isin(bmask[legal_all], (0, 1)).all()
    force = np.where(legal_all, bmask.astype(np.int16), -1).astype(np.int8)
    oQ, oK, oV, _, omargin = orc.mala_bwd(inp["Q"], inp["K"], inp["V"], O.astype(np.float64),
                                          LSE.astype(np.float64), inp["dO"], w.scale, tau,
                                          kv_units=kv_units, q_units=q_units, force=force)
    label = (f"bwd {w.name}:{w.structure} B{B} H{H}/{Hkv} L{L} d{d} {w.dtype} tau={tau:g}"
             + (" always-test" if flags else ""))
    screen = tau > 0 or flags
    row = {"flips": 0}
    if screen:
        # decisions on the tiles the oracle evaluated (conditioned on the GPU's LSE)
        sel = legal_all & ~np.isnan(omargin)
        row = P.compare_decisions(label, "fp32" if w.dtype == "fp32" else "bwd", bmask, bmg,
                                  omargin, sel, max_flips)
        # nesting (§2.2): the backward margin of a tile never exceeds its forward margin,
        # because the final LSE bounds every running log-normaliser from above; checked on
        # the GPU's own margins over every legal tile, to rounding
        both = legal_all & np.isfinite(fmg) & np.isfinite(bmg)
        excess = (bmg - fmg)[both]
        assert excess.size == 0 or excess.max() <= 2 * P.MARGIN_ERR["bwd"], excess.max()
    viol = legal_all & (bmask == 1) & (fmask == 0)
    assert viol.sum() <= row["flips"], f"{viol.sum()} tiles retained by backward but not forward"
    rows_q = np.isfinite(oQ[..., 0])
    rows_k = np.isfinite(oK[..., 0])
    for name, g, o, rows in (("dQ", dQ, oQ, rows_q), ("dK", dK, oK, rows_k),
                             ("dV", dV, oV, rows_k)):
        if rows.any():
            err = P.rel_fro(g[rows], o[rows])
            assert err < P.GRAD_REL_FRO, f"{name}: relative Frobenius error {err}"
    if tau == 0:
        assert (bmask[legal_all] == 1).all()
    return {"tiles": int(legal_all.sum()), "flips": row["flips"],
            "bwd_retained": float(bmask[legal_all].mean()),
            "fwd_retained": float(fmask[legal_all].mean())}


@pytest.mark.parametrize("tau", [0.0, 1.0])
@pytest.mark.parametrize("shape", [
    dict(B=1, H=4, Hkv=2, L=256, d=128, structure="peaked"),
    dict(B=2, H=6, Hkv=2, L=300, d=64, structure="normal"),
    dict(B=1, H=2, Hkv=2, L=384, d=128, structure="peaked"),
    # few units: the query heads of a KV head are split over 4 CTAs, which add their dK /
    # dV shares in fp32 (ragged length, d = 64)
    dict(B=2, H=8, Hkv=2, L=333, d=64, structure="peaked"),
    # one KV head of 8 query heads at 1K: every query head gets its own CTA (P = 8)
    dict(B=1, H=8, Hkv=1, L=1024, d=128, structure="peaked"),
])
def test_bwd_small(orc, mala, shape, tau):
    w, inp = synth.small_training(**shape)
    check_bwd(orc, mala, w, inp, tau)


def test_bwd_always_test_flag_at_tau0(orc, mala):
    w, inp = synth.small_training(B=1, H=4, Hkv=1, L=512, d=128, structure="peaked")
    st = check_bwd(orc, mala, w, inp, 0.0, flags=1)
    assert st["bwd_retained"] == 1.0


def test_bwd_peaked1k_full(orc, mala):
    w = synth.WORKLOADS["peaked1k"]
    st = check_bwd(orc, mala, w, synth.make_training(w), 1.0)
    assert st["bwd_retained"] <= st["fwd_retained"]


def _sample(B, Hx, T, n, seed):
    rng = np.random.default_rng(seed)
    u = {(B - 1, Hx - 1, T - 1), (0, 0, 0), (0, Hx // 2, T // 2)}
    while len(u) < n:
        u.add((int(rng.integers(B)), int(rng.integers(Hx)), int(rng.integers(T))))
    return sorted(u)


@pytest.mark.parametrize("tau", [1.0, 0.0, 1e-4, 1e-3])
def test_bwd_mixed8k_sampled(orc, mala, tau):
    w = synth.WORKLOADS["mixed8k"]
    T = w.L // 128
    check_bwd(orc, mala, w, synth.make_training(w), tau,
              kv_units=_sample(w.B, w.H_kv, T, 3, seed=7), q_units=_sample(w.B, w.H, T, 3, seed=8))


@pytest.mark.slow
def test_bwd_sinkband32k_sampled(orc, mala):
    w = synth.WORKLOADS["sinkband32k"]
    T = w.L // 128
    check_bwd(orc, mala, w, synth.make_training(w), 1.0,
              kv_units=[(0, 7, T - 1), (0, 3, T // 2)], q_units=[(0, 31, T - 1), (0, 0, 5)])


@pytest.mark.parametrize("tau", [0.0, 1.0])
def test_bwd_tiny256_fp32(orc, mala, tau):
    w = synth.WORKLOADS["tiny256"]
    check_bwd(orc, mala, w, synth.make_training(w), tau)


def test_bwd_fp32_ragged_gqa(orc, mala):
    w, inp = synth.small_training(B=2, H=4, Hkv=2, L=200, d=32, dtype="fp32", structure="peaked")
    check_bwd(orc, mala, w, inp, 1.0)


@pytest.mark.slow
def test_bwd_sinkband128k_sampled(orc, mala):
    w = synth.WORKLOADS["sinkband128k"]
    T = w.L // 128
    check_bwd(orc, mala, w, synth.make_training(w), 1.0,
              kv_units=[(0, 0, T - 2)], q_units=[(0, 6, T - 1), (0, 1, 3)])


def test_bwd_prev_token_skips(orc, mala):
    w, inp = synth.small_training(B=1, H=4, Hkv=1, L=2048, d=128, structure="prev_token", seed=3)
    st = check_bwd(orc, mala, w, inp, 1.0)
    assert st["bwd_retained"] < 0.3


@pytest.mark.slow
@pytest.mark.parametrize("tau", [1.0, 0.0])
def test_bwd_prevtok32k_sampled(orc, mala, tau):
    """Concentrated states at 32K: the skip regime at tau = 1 and the dense path on the same
    extreme scores (one dominant key per row) at tau = 0."""
    w = synth.WORKLOADS["prevtok32k"]
    T = w.L // 128
    st = check_bwd(orc, mala, w, synth.make_training(w), tau,
                   kv_units=[(0, 5, T - 3), (0, 0, 7)], q_units=[(0, 31, T - 1), (0, 2, 40)])
    if tau > 0:
        assert st["bwd_retained"] < 0.05
