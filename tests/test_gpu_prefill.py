"""GPU parity of the chunked-prefill forward (C ABI -> sm_100a kernels) against the fp64
oracle: a chunk of N_q queries at the end of a sequence of N_k keys (causal offset
N_k - N_q, "the same forward serves inference prefill", MassAlloc Attention §2.3)."""

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


def chunk(B, H, Hkv, Nq, Nk, d, structure, seed, dtype="bf16"):
    """A sequence of Nk positions from the seeded generator; the chunk is its last Nq
    query rows."""
    w, inp = synth.small_training(B=B, H=H, Hkv=Hkv, L=Nk, d=d, dtype=dtype,
                                  structure=structure, seed=seed)
    return w, np.ascontiguousarray(inp["Q"][:, Nk - Nq:]), inp["K"], inp["V"], inp["Q"]


def prefill_legal(B, H, Nq, Nk, units=None):
    Tq, Tk = -(-Nq // 128), -(-Nk // 128)
    off = Nk - Nq
    last = np.array([(off + min(Nq, (i + 1) * 128) - 1) // 128 for i in range(Tq)])
    legal = np.arange(Tk)[None, :] <= last[:, None]
    out = np.broadcast_to(legal, (B, H, Tq, Tk)).copy()
    if units is not None:
        sel = np.zeros_like(out)
        for b, h, i in units:
            sel[b, h, i] = out[b, h, i]
        out = sel
    return out


def run_prefill(mala, Qc, K, V, w, tau, flags=0):
    Q, Kd, Vd = (P.to_dev(x, w.dtype) for x in (Qc, K, V))
    B, Nq, H, d = Q.shape
    Nk, Hkv = Kd.shape[1], Kd.shape[2]
    Tq, Tk = mala.n_tiles(Nq), mala.n_tiles(Nk)
    mask = torch.full((B, H, Tq, Tk), 255, dtype=torch.uint8, device="cuda")
    margin = P.margin_buffer(B * H * Tq * Tk)
    ws = mala.alloc_workspace(mala.fwd_workspace_bytes(B, H, Hkv, Nq, d), "cuda")
    with mala.debug_margins(margin):
        O, LSE = mala.mala_fwd_prefill(Q, Kd, Vd, w.scale, tau, flags=flags, workspace=ws,
                                       tile_mask=mask)
    torch.cuda.synchronize()
    assert mala.read_device_error(ws) == 0
    mask = mask.cpu().numpy()
    legal = prefill_legal(B, H, Nq, Nk)
    assert (mask[~legal] == 255).all() and np.isin(mask[legal], (0, 1)).all()
    st = mala.get_stats(ws)
    assert st["legal_tiles"] == legal.sum() and st["retained_tiles"] == (mask[legal] == 1).sum()
    return (O.float().cpu().numpy(), LSE.cpu().numpy(), mask,
            margin.view(B, H, Tq, Tk).cpu().numpy())


def check_prefill(orc, mala, w, Qc, K, V, tau, units=None, flags=0, max_flips=0):
    O, LSE, mask, gmargin = run_prefill(mala, Qc, K, V, w, tau, flags)
    B, Nq, H, d = Qc.shape
    Nk = K.shape[1]
    legal_all = prefill_legal(B, H, Nq, Nk)
    force = np.where(legal_all, mask.astype(np.int16), -1).astype(np.int8)
    oO, oLSE, _, omargin = orc.mala_prefill(Qc, K, V, w.scale, tau, units=units, force=force)
    legal = prefill_legal(B, H, Nq, Nk, units)
    label = (f"prefill {w.structure} B{B} H{H}/{K.shape[2]} Nq{Nq} Nk{Nk} d{d} {w.dtype} "
             f"tau={tau:g}" + (" always-test" if flags else ""))
    row = {"flips": 0}
    if tau > 0 or flags:
        row = P.compare_decisions(label, "fp32" if w.dtype == "fp32" else "fwd", mask, gmargin,
                                  omargin, legal, max_flips)
    rows = np.isfinite(oLSE)
    P.check_output(O, oO, np.transpose(rows, (0, 2, 1)), label)
    assert np.abs(LSE - oLSE)[rows].max() < P.LSE_ABS
    if tau == 0:
        assert (mask[legal_all] == 1).all()
    return {"tiles": int(legal.sum()), "flips": row["flips"],
            "retained": float(mask[legal_all].mean())}


@pytest.mark.parametrize("tau", [0.0, 1.0])
@pytest.mark.parametrize("shape", [
    dict(B=1, H=4, Hkv=2, Nq=256, Nk=640, d=128, structure="peaked"),     # aligned offset
    dict(B=2, H=4, Hkv=1, Nq=300, Nk=777, d=128, structure="peaked"),     # unaligned, ragged
    dict(B=1, H=6, Hkv=2, Nq=129, Nk=1000, d=64, structure="peaked"),     # odd group, d=64
    dict(B=1, H=2, Hkv=2, Nq=1, Nk=513, d=128, structure="normal"),       # one query
    dict(B=1, H=4, Hkv=1, Nq=200, Nk=200, d=128, structure="prev_token"),  # N_q == N_k
])
def test_prefill_small(orc, mala, shape, tau):
    w, Qc, K, V, _ = chunk(shape["B"], shape["H"], shape["Hkv"], shape["Nq"], shape["Nk"],
                           shape["d"], shape["structure"], seed=61)
    check_prefill(orc, mala, w, Qc, K, V, tau)


def test_prefill_skips_on_concentrated_states(orc, mala):
    w, Qc, K, V, _ = chunk(1, 4, 1, 1000, 3000, 128, "prev_token", seed=62)
    st = check_prefill(orc, mala, w, Qc, K, V, 1.0)
    assert st["retained"] < 0.2


def test_prefill_aligned_chunk_equals_forward_tail_bitwise(mala):
    """With a 128-aligned offset the chunk's query blocks are the full forward's last
    blocks: same tiles, same order, same arithmetic -> identical bits."""
    w, Qc, K, V, Qf = chunk(1, 8, 2, 512, 1536, 128, "sink_band", seed=63)
    Oc, Lc, Mc, _ = run_prefill(mala, Qc, K, V, w, 1.0)
    Qd, Kd, Vd = (P.to_dev(x, "bf16") for x in (Qf, K, V))
    T = mala.n_tiles(1536)
    Mf = torch.full((1, 8, T, T), 255, dtype=torch.uint8, device="cuda")
    Of, Lf = mala.mala_fwd(Qd, Kd, Vd, w.scale, 1.0, tile_mask=Mf)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(Oc, Of.float().cpu().numpy()[:, 1024:])
    np.testing.assert_array_equal(Lc, Lf.cpu().numpy()[:, :, 1024:])
    np.testing.assert_array_equal(Mc, Mf.cpu().numpy()[:, :, 8:])


def test_prefill_always_test_flag_at_tau0(orc, mala):
    w, Qc, K, V, _ = chunk(1, 4, 2, 300, 700, 128, "peaked", seed=64)
    check_prefill(orc, mala, w, Qc, K, V, 0.0, flags=1)


@pytest.mark.parametrize("tau", [0.0, 1.0])
def test_prefill_fp32(orc, mala, tau):
    w, Qc, K, V, _ = chunk(1, 2, 1, 150, 333, 64, "normal", seed=65, dtype="fp32")
    check_prefill(orc, mala, w, Qc, K, V, tau)


@pytest.mark.slow
def test_prefill_4k_chunk_of_32k_sampled(orc, mala):
    """A 4K-token chunk at the end of the 32K sink + band sequence, sampled blocks."""
    w0 = synth.WORKLOADS["sinkband32k"]
    inp = synth.make_training(w0)
    Nq, Nk = 4096, w0.L
    Qc = np.ascontiguousarray(inp["Q"][:, Nk - Nq:])
    units = [(0, 0, 31), (0, 17, 0), (0, 31, 15)]
    check_prefill(orc, mala, w0, Qc, inp["K"], inp["V"], 1.0, units=units)


# ---------------------------------------------------------------------------- packed batches


def _packed(seqs, H, Hkv, d, structure="peaked"):
    """seqs: list of (N_q, N_k).  Returns per-sequence (Qc, K, V) and the packed arrays."""
    parts = []
    for s, (nq, nk) in enumerate(seqs):
        if nk == 0:
            parts.append((np.zeros((1, 0, H, d), np.float32), np.zeros((1, 0, Hkv, d), np.float32),
                          np.zeros((1, 0, Hkv, d), np.float32), None))
            continue
        w, Qc, K, V, _ = chunk(1, H, Hkv, nq, nk, d, structure, seed=70 + s)
        parts.append((Qc, K, V, w))
    cu_q = np.concatenate([[0], np.cumsum([p[0].shape[1] for p in parts])]).astype(int)
    cu_k = np.concatenate([[0], np.cumsum([p[1].shape[1] for p in parts])]).astype(int)
    Qp = np.concatenate([p[0][0] for p in parts], axis=0)
    Kp = np.concatenate([p[1][0] for p in parts], axis=0)
    Vp = np.concatenate([p[2][0] for p in parts], axis=0)
    return parts, cu_q, cu_k, Qp, Kp, Vp


@pytest.mark.parametrize("tau", [0.0, 1.0])
def test_varlen_equals_per_sequence_prefill_bitwise(mala, tau):
    H, Hkv, d = 4, 2, 128
    seqs = [(300, 777), (128, 128), (1, 513), (0, 50), (517, 517), (64, 1000)]
    parts, cu_q, cu_k, Qp, Kp, Vp = _packed(seqs, H, Hkv, d)
    scale = 1.0 / np.sqrt(d)
    Q, K, V = (P.to_dev(x, "bf16") for x in (Qp, Kp, Vp))
    ws = mala.alloc_workspace(mala.varlen_workspace_bytes(cu_q, H, Hkv, d), "cuda")
    O, LSE = mala.mala_fwd_varlen(Q, K, V, cu_q, cu_k, scale, tau, workspace=ws)
    torch.cuda.synchronize()
    assert mala.read_device_error(ws) == 0
    st = mala.get_stats(ws)
    O, LSE = O.float().cpu().numpy(), LSE.cpu().numpy()
    legal = retained = 0
    for s, (Qc, Ks, Vs, w) in enumerate(parts):
        if Qc.shape[1] == 0:
            continue
        Qd, Kd, Vd = (P.to_dev(x, "bf16") for x in (Qc, Ks, Vs))
        wss = mala.alloc_workspace(mala.fwd_workspace_bytes(1, H, Hkv, Qc.shape[1], d), "cuda")
        Os, Ls = mala.mala_fwd_prefill(Qd, Kd, Vd, scale, tau, workspace=wss)
        torch.cuda.synchronize()
        sst = mala.get_stats(wss)
        legal += sst["legal_tiles"]
        retained += sst["retained_tiles"]
        rows = slice(cu_q[s], cu_q[s + 1])
        np.testing.assert_array_equal(O[rows], Os.float().cpu().numpy()[0])
        np.testing.assert_array_equal(LSE[:, rows], Ls.cpu().numpy()[0])
    assert st["legal_tiles"] == legal and st["retained_tiles"] == retained


def test_varlen_parity_with_oracle(orc, mala):
    H, Hkv, d = 2, 1, 64
    seqs = [(200, 450), (90, 90), (333, 333)]
    parts, cu_q, cu_k, Qp, Kp, Vp = _packed(seqs, H, Hkv, d)
    scale = 1.0 / np.sqrt(d)
    Q, K, V = (P.to_dev(x, "bf16") for x in (Qp, Kp, Vp))
    O, LSE = mala.mala_fwd_varlen(Q, K, V, cu_q, cu_k, scale, 1.0)
    torch.cuda.synchronize()
    O, LSE = O.float().cpu().numpy(), LSE.cpu().numpy()
    for s, (Qc, Ks, Vs, w) in enumerate(parts):
        # the GPU's decisions for this sequence (from its own prefill call) are replayed
        _, _, mask, _ = run_prefill(mala, Qc, Ks, Vs, w, 1.0)
        legal = prefill_legal(1, H, Qc.shape[1], Ks.shape[1])
        force = np.where(legal, mask.astype(np.int16), -1).astype(np.int8)
        oO, oLSE, _, _ = orc.mala_prefill(Qc, Ks, Vs, scale, 1.0, force=force)
        rows = slice(cu_q[s], cu_q[s + 1])
        P.check_output(O[rows][None], oO, np.ones(oO.shape[:-1], bool))
        assert np.abs(LSE[:, rows] - oLSE[0]).max() < P.LSE_ABS
