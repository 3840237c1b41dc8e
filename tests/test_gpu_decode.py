"""GPU parity of MALA split-KV decode (C ABI -> sm_100a kernel) against the fp64 oracle."""

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


def check_decode(orc, mala, inp, scale, tau, S, dtype="bf16", units=None, flags=0, max_flips=0,
                 name="decode"):
    q, K, V = (P.to_dev(inp[k], dtype) for k in ("q", "K", "V"))
    B, H, d = q.shape
    Nk, Hkv = K.shape[1], K.shape[2]
    T = mala.n_tiles(Nk)
    mask = torch.full((B, H, T), 255, dtype=torch.uint8, device="cuda")
    margin = P.margin_buffer(B * H * T)
    ws = mala.alloc_workspace(mala.decode_workspace_bytes(B, H, Hkv, Nk, d, 0, S), "cuda")
    with mala.debug_margins(margin):
        O, LSE = mala.mala_decode(q, K, V, scale, tau, num_splits=S, flags=flags, workspace=ws,
                                  tile_mask=mask)
    torch.cuda.synchronize()
    assert mala.read_device_error(ws) == 0
    O, LSE, mask = O.float().cpu().numpy(), LSE.cpu().numpy(), mask.cpu().numpy()
    gmargin = margin.view(B, H, T).cpu().numpy()
    assert np.isin(mask, (0, 1)).all()
    # the call's work counters: tested and retained (b, h, tile) pairs, V tiles fetched
    # (per KV group on the tensor-core path, per head on the fp32 path)
    st = mala.get_stats(ws)
    assert st["legal_tiles"] == mask.size and st["retained_tiles"] == mask.sum()
    v_tiles = mask.sum() if dtype == "fp32" else \
        mask.reshape(B, Hkv, H // Hkv, T).max(axis=2).sum()
    assert st["v_tiles_loaded"] == v_tiles
    oO, oLSE, _, omargin, _, _ = orc.mala_decode(inp["q"], inp["K"], inp["V"], scale, tau, S,
                                                  units=units, force=mask.astype(np.int8))
    sel = np.isfinite(oLSE)
    label = (f"{name} B{B} H{H}/{Hkv} Nk{Nk} d{d} {dtype} S{S} tau={tau:g}"
             + (" always-test" if flags else ""))
    if tau > 0 or flags:
        tiles = np.broadcast_to(sel[:, :, None], mask.shape)
        P.compare_decisions(label, "fp32" if dtype == "fp32" else "decode", mask, gmargin,
                            omargin, tiles, max_flips)
    P.check_output(O[sel], oO[sel], np.ones(O[sel].shape, bool), label)
    assert np.abs(LSE - oLSE)[sel].max() < P.LSE_ABS
    if tau == 0:
        assert (mask == 1).all()
    return mask


def _planted(B, H, Hkv, Nk, d, seed):
    w = synth.Workload("adhoc_decode", B, H, Hkv, Nk, d, "bf16", "planted", seed, decode=True)
    return w, synth.make_decode(w)


@pytest.mark.parametrize("tau", [0.0, 1.0])
@pytest.mark.parametrize("S", [1, 3])
@pytest.mark.parametrize("shape", [(2, 8, 2, 1000, 128), (1, 4, 1, 2048, 64), (3, 6, 2, 300, 128)])
def test_decode_small(orc, mala, shape, S, tau):
    w, inp = _planted(*shape, seed=21)
    mask = check_decode(orc, mala, inp, w.scale, tau, S)
    if tau > 0 and shape[3] >= 1000:
        assert (mask == 0).any()


@pytest.mark.parametrize("tau", [0.0, 1.0])
@pytest.mark.parametrize("S", [37, 0])
def test_decode_batch1_many_splits(orc, mala, S, tau):
    """One KV head at batch 1 (a rank of 8-way head sharding): many splits, so the merge
    runs its eight-deep unrolled loop several times plus a remainder (37 splits), and the
    automatic count of the split rule's merge term (22 at 8K)."""
    w, inp = _planted(1, 8, 1, 8192, 128, seed=23)
    if S == 0:
        S = mala.decode_num_splits(1, 8, 1, 8192)
        assert S == 22
    check_decode(orc, mala, inp, w.scale, tau, S, name="decode_b1")


def test_decode_always_test_flag(orc, mala):
    w, inp = _planted(2, 8, 2, 1024, 128, seed=22)
    check_decode(orc, mala, inp, w.scale, 0.0, 2, flags=1)


def test_decode128k_full(orc, mala):
    w = synth.WORKLOADS["decode128k"]
    inp = synth.make_decode(w)
    S = mala.decode_num_splits(w.B, w.H, w.H_kv, w.L)
    mask = check_decode(orc, mala, inp, w.scale, 1.0, S, name="decode128k")
    # splits that hold a planted key skip the tiles after it; splits without one test
    # against a small diffuse normaliser and keep most tiles (the oracle agrees)
    assert (mask == 0).any()


@pytest.mark.parametrize("tau", [0.0, 1.0])
def test_decode_fp32(orc, mala, tau):
    w = synth.Workload("fp32_decode", 2, 4, 2, 700, 64, "fp32", "planted", 23, decode=True)
    inp = synth.make_decode(w)
    check_decode(orc, mala, inp, w.scale, tau, 2, dtype="fp32")


@pytest.mark.parametrize("S", [2, 5])
def test_decode_heavy_small(orc, mala, S):
    """Heavy hitters in every split: most tiles and most V loads are skipped."""
    w = synth.Workload("adhoc_heavy", 2, 8, 2, 8192, 128, "bf16", "heavy", 24, decode=True)
    inp = synth.make_decode(w)
    mask = check_decode(orc, mala, inp, w.scale, 1.0, S, name="heavy")
    group = mask.reshape(w.B, w.H_kv, w.H // w.H_kv, -1).max(axis=2)
    assert group.mean() < 0.5


def test_heavy128k_full(orc, mala):
    w = synth.WORKLOADS["heavy128k"]
    inp = synth.make_decode(w)
    S = mala.decode_num_splits(w.B, w.H, w.H_kv, w.L)
    mask = check_decode(orc, mala, inp, w.scale, 1.0, S, name="heavy128k")
    group = mask.reshape(w.B, w.H_kv, w.H // w.H_kv, -1).max(axis=2)
    assert group.mean() < 0.35


@pytest.mark.parametrize("tau", [0.0, 1.0])
@pytest.mark.parametrize("shape", [(2, 16, 2, 3000, 128), (1, 24, 4, 1000, 64), (1, 5, 1, 700, 128)])
def test_decode_large_groups(orc, mala, shape, tau):
    """Groups of 5..8 query heads per KV head (e.g. 64 query / 8 KV heads)."""
    w, inp = _planted(*shape, seed=31)
    mask = check_decode(orc, mala, inp, w.scale, tau, 3)
    if tau > 0 and shape[3] >= 1000:
        assert (mask == 0).any()


def test_decode_heavy_group8(orc, mala):
    w = synth.Workload("adhoc_heavy8", 1, 16, 2, 8192, 128, "bf16", "heavy", 25, decode=True)
    inp = synth.make_decode(w)
    mask = check_decode(orc, mala, inp, w.scale, 1.0, 4)
    group = mask.reshape(w.B, w.H_kv, w.H // w.H_kv, -1).max(axis=2)
    assert group.mean() < 0.5
