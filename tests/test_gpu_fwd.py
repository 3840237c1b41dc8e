"""GPU parity of the MALA forward (C ABI -> sm_100a kernels) against the fp64 oracle."""

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


def run_fwd(mala, inp, w, tau, flags=0, debug=True):
    Q, K, V = (P.to_dev(inp[k], w.dtype) for k in ("Q", "K", "V"))
    B, L, H, d = Q.shape
    T = mala.n_tiles(L)
    mask = torch.full((B, H, T, T), 255, dtype=torch.uint8, device="cuda")
    margin = P.margin_buffer(B * H * T * T)
    ws = mala.alloc_workspace(mala.fwd_workspace_bytes(B, H, K.shape[2], L, d), "cuda")
    if debug:
        with mala.debug_margins(margin):
            O, LSE = mala.mala_fwd(Q, K, V, w.scale, tau, flags=flags, workspace=ws,
                                   tile_mask=mask)
    else:
        O, LSE = mala.mala_fwd(Q, K, V, w.scale, tau, flags=flags, workspace=ws, tile_mask=mask)
    torch.cuda.synchronize()
    assert mala.read_device_error(ws) == 0
    mask = mask.cpu().numpy()
    # the call's work counters agree with its tile decisions
    legal = P.fwd_legal(B, H, T)
    st = mala.get_stats(ws)
    assert st["legal_tiles"] == legal.sum() and st["retained_tiles"] == (mask[legal] == 1).sum()
    return (O.float().cpu().numpy(), LSE.cpu().numpy(), mask,
            margin.view(B, H, T, T).cpu().numpy())


def label_of(kind, w, inp, tau, flags=0):
    B, L, H, d = inp["Q"].shape
    return (f"{kind} {w.name}:{w.structure} B{B} H{H}/{inp['K'].shape[2]} L{L} d{d} "
            f"{w.dtype} tau={tau:g}"
            + (" always-test" if flags else ""))


def check_fwd(orc, mala, w, inp, tau, units=None, flags=0, max_flips=0):
    O, LSE, mask, gmargin = run_fwd(mala, inp, w, tau, flags)
    B, L, H, d = inp["Q"].shape
    T = (L + 127) // 128
    legal_all = P.fwd_legal(B, H, T)
    # untouched entries only above the diagonal; decisions are 0/1 on legal tiles
    assert (mask[~legal_all] == 255).all()
    assert np.isin(mask[legal_all], (0, 1)).all()
    force = np.where(legal_all, mask.astype(np.int16), -1).astype(np.int8)
    oO, oLSE, omask, omargin = orc.mala_fwd(inp["Q"], inp["K"], inp["V"], w.scale, tau,
                                            units=units, force=force)
    legal = P.fwd_legal(B, H, T, units)
    label = label_of("fwd", w, inp, tau, flags)
    row = {"flips": 0}
    if tau > 0 or flags:
        row = P.compare_decisions(label, "fp32" if w.dtype == "fp32" else "fwd", mask, gmargin,
                                  omargin, legal, max_flips)
    rows = np.isfinite(oLSE)  # [B,H,L] rows the oracle computed
    rows_o = np.transpose(rows, (0, 2, 1))  # [B,L,H]
    P.check_output(O, oO, rows_o, label)
    assert np.abs(LSE - oLSE)[rows].max() < P.LSE_ABS
    if tau == 0:
        assert (mask[legal_all] == 1).all()
    return {"tiles": int(legal.sum()), "flips": row["flips"],
            "retained": float(mask[legal_all].mean()), "margin": gmargin}


@pytest.mark.parametrize("tau", [0.0, 1.0])
@pytest.mark.parametrize("shape", [
    dict(B=1, H=4, Hkv=2, L=256, d=128, structure="peaked"),   # 2 tiles, GQA pairs
    dict(B=2, H=6, Hkv=2, L=300, d=64, structure="normal"),    # ragged tail, odd group
    dict(B=1, H=2, Hkv=2, L=384, d=128, structure="peaked"),   # G = 1: one slot idle
])
def test_fwd_small(orc, mala, shape, tau):
    w, inp = synth.small_training(**shape)
    check_fwd(orc, mala, w, inp, tau)


def test_fwd_always_test_flag_at_tau0(orc, mala):
    w, inp = synth.small_training(B=1, H=4, Hkv=1, L=512, d=128, structure="peaked")
    st = check_fwd(orc, mala, w, inp, 0.0, flags=1)
    assert st["retained"] == 1.0


def test_fwd_peaked1k_full(orc, mala):
    w = synth.WORKLOADS["peaked1k"]
    inp = synth.make_training(w)
    # at L = 1024 the 4 random prefix keys of 128 rows land in every earlier tile, so
    # the oracle (and the kernel) retain all tiles here; decisions still must agree
    check_fwd(orc, mala, w, inp, 1.0)


def _units(B, H, T, n, seed):
    rng = np.random.default_rng(seed)
    u = {(B - 1, H - 1, T - 1), (0, 0, 0), (0, H // 2, T // 2)}
    while len(u) < n:
        u.add((int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(T))))
    return sorted(u)


@pytest.mark.parametrize("tau", [1.0, 0.0, 1e-4, 1e-3])
def test_fwd_mixed8k_sampled(orc, mala, tau):
    w = synth.WORKLOADS["mixed8k"]
    inp = synth.make_training(w)
    T = w.L // 128
    check_fwd(orc, mala, w, inp, tau, units=_units(w.B, w.H, T, 6, seed=int(tau * 1e4) + 1))


@pytest.mark.slow
def test_fwd_sinkband32k_sampled(orc, mala):
    w = synth.WORKLOADS["sinkband32k"]
    inp = synth.make_training(w)
    T = w.L // 128
    check_fwd(orc, mala, w, inp, 1.0, units=_units(w.B, w.H, T, 4, seed=5))


@pytest.mark.parametrize("tau", [0.0, 1.0])
def test_fwd_tiny256_fp32(orc, mala, tau):
    w = synth.WORKLOADS["tiny256"]
    check_fwd(orc, mala, w, synth.make_training(w), tau)


def test_fwd_fp32_ragged_gqa(orc, mala):
    w, inp = synth.small_training(B=2, H=4, Hkv=2, L=200, d=32, dtype="fp32", structure="peaked")
    check_fwd(orc, mala, w, inp, 1.0)


@pytest.mark.slow
def test_fwd_sinkband128k_sampled(orc, mala):
    w = synth.WORKLOADS["sinkband128k"]
    inp = synth.make_training(w)
    T = w.L // 128
    check_fwd(orc, mala, w, inp, 1.0, units=[(0, 7, T - 1), (0, 0, T // 3), (0, 3, 2)])


def test_fwd_prev_token_skips(orc, mala):
    """Concentrated heads: most off-diagonal tiles are skipped; decisions and O agree."""
    w, inp = synth.small_training(B=1, H=4, Hkv=1, L=2048, d=128, structure="prev_token", seed=3)
    st = check_fwd(orc, mala, w, inp, 1.0)
    assert st["retained"] < 0.3


@pytest.mark.slow
def test_fwd_prevtok32k_sampled(orc, mala):
    w = synth.WORKLOADS["prevtok32k"]
    inp = synth.make_training(w)
    T = w.L // 128
    st = check_fwd(orc, mala, w, inp, 1.0, units=_units(w.B, w.H, T, 6, seed=9))
    assert st["retained"] < 0.05


def test_fwd_debug_hook_changes_nothing(orc, mala):
    """The margin export does not alter the forward: same decisions, bitwise equal O and
    LSE with the hook on and off."""
    w, inp = synth.small_training(B=1, H=4, Hkv=1, L=2048, d=128, structure="prev_token", seed=4)
    a = run_fwd(mala, inp, w, 1.0, debug=True)
    b = run_fwd(mala, inp, w, 1.0, debug=False)
    assert np.array_equal(a[2], b[2])
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
