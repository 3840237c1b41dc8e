"""Pins for the fp64 CPU oracle (no GPU).

Each check ties the oracle to something other than itself: hand-derived worked
examples (tests/golden), torch's scaled_dot_product_attention / autograd in fp64
(FullAttn is a library routine), central finite differences, brute-force numpy
re-evaluation of the tile tests from raw scores, and the invariants the attention page
states (tau = 0 recovers FullAttn §2.3; first legal tile retained §2.2; Proposition 1
of App. B; backward support nested in forward support §2.2).
"""

import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from mass_adaptive_sparse_fwd_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")


def _expr(s):
    s = s.strip()
    if s.startswith("ln "):
        return math.log(float(s[3:]))
    if "/" in s:
        a, b = s.split("/")
        return float(a) / float(b)
    return float(s)


def _rand(B, L, H, Hkv, d, seed, peak=0.0):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((B, L, H, d)).astype(np.float32)
    K = rng.standard_normal((B, L, Hkv, d)).astype(np.float32)
    V = rng.standard_normal((B, L, Hkv, d)).astype(np.float32)
    dO = rng.choice([-1.0, 1.0], size=(B, L, H, d)).astype(np.float32)
    if peak:
        # concentrate each row on one key (usually its own position, sometimes a random
        # earlier one) so that many tiles fall below the threshold and some do not
        G = H // Hkv
        for h in range(H):
            for t in range(L):
                p = t if rng.random() < 0.9 else int(rng.integers(0, t + 1))
                Q[:, t, h] += peak * K[:, p, h // G]
    return Q, K, V, dO


def _torch_bhld(x):
    return torch.from_numpy(np.ascontiguousarray(x.transpose(0, 2, 1, 3))).double()


def _expand_kv(x, G):
    return x.repeat_interleave(G, dim=1)


def _sdpa(Q, K, V, scale, mask=None):
    """FullAttn (or masked softmax attention) via torch in fp64.  mask [B,H,L,L] bool."""
    B, L, H, d = Q.shape
    G = H // K.shape[2]
    q, k, v = _torch_bhld(Q), _expand_kv(_torch_bhld(K), G), _expand_kv(_torch_bhld(V), G)
    causal = torch.ones(L, L, dtype=torch.bool).tril()
    m = causal if mask is None else (torch.from_numpy(mask) & causal)
    out = F.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale)
    s = (q @ k.transpose(-1, -2)) * scale
    lse = torch.logsumexp(s.masked_fill(~m, float("-inf")), dim=-1)
    return out.permute(0, 2, 1, 3).numpy(), lse.numpy()


def _scores(Q, K, scale):
    """Raw scores [B,H,L,L] (numpy, fp64) with -inf above the diagonal."""
    B, L, H, d = Q.shape
    G = H // K.shape[2]
    Kx = np.repeat(K.astype(np.float64), G, axis=2)
    s = np.einsum("bqhd,bkhd->bhqk", Q.astype(np.float64), Kx) * scale
    s[..., np.triu_indices(L, 1)[0], np.triu_indices(L, 1)[1]] = -np.inf
    return s


def _expand_tiles(mask, L, blk):
    """[B,H,T,T] tile mask -> [B,H,L,L] bool key mask (retained tiles only)."""
    m = np.repeat(np.repeat(mask == 1, blk, axis=2), blk, axis=3)
    return m[:, :, :L, :L]


# ----------------------------------------------------------------------------- golden


def test_golden_hand_fwd_bwd(orc):
    ex = json.load(open(GOLDEN))["fwd_bwd_tau1"]
    Q = np.array(ex["Q"], np.float32).reshape(1, 4, 1, 1)
    K = np.array([_expr(e) for e in ex["K_exprs"]], np.float32).reshape(1, 4, 1, 1)
    V = np.array(ex["V"], np.float32).reshape(1, 4, 1, 1)
    O, LSE, mask, _ = orc.mala_fwd(Q, K, V, 1.0, ex["tau"], blk=1)
    np.testing.assert_array_equal(mask[0, 0], np.array(ex["fwd_mask"]))
    np.testing.assert_allclose(O.ravel(), [_expr(e) for e in ex["O_exprs"]], rtol=1e-6)
    np.testing.assert_allclose(LSE.ravel(), [_expr(e) for e in ex["LSE_exprs"]], atol=1e-6)
    dO = np.ones_like(Q)
    _, _, _, bmask, _ = orc.mala_bwd(Q, K, V, O, LSE, dO, 1.0, ex["tau"], blk=1)
    np.testing.assert_array_equal(bmask[0, 0], np.array(ex["bwd_mask"]))


def test_golden_fwd_tie_retains(orc):
    ex = json.load(open(GOLDEN))["fwd_tie_tau2"]
    Q = np.array(ex["Q"], np.float32).reshape(1, 2, 1, 1)
    K = np.array([_expr(e) for e in ex["K_exprs"]], np.float32).reshape(1, 2, 1, 1)
    V = np.array(ex["V"], np.float32).reshape(1, 2, 1, 1)
    O, LSE, mask, margin = orc.mala_fwd(Q, K, V, 1.0, ex["tau"], blk=1)
    np.testing.assert_array_equal(mask[0, 0], np.array(ex["fwd_mask"]))
    assert margin[0, 0, 1, 0] == 0.0
    np.testing.assert_allclose(O.ravel(), [_expr(e) for e in ex["O_exprs"]], rtol=1e-12)
    np.testing.assert_allclose(LSE.ravel(), [_expr(e) for e in ex["LSE_exprs"]], atol=1e-12)


def test_golden_decode_split(orc):
    ex = json.load(open(GOLDEN))["decode_split"]
    q = np.array(ex["q"], np.float32).reshape(1, 1, 1)
    K = np.array([_expr(e) for e in ex["K_exprs"]], np.float32).reshape(1, 4, 1, 1)
    V = np.array(ex["V"], np.float32).reshape(1, 4, 1, 1)
    for S, key in ((1, "S1"), (2, "S2")):
        O, LSE, mask, _, _, _ = orc.mala_decode(q, K, V, 1.0, ex["tau"], S, blk=1)
        np.testing.assert_array_equal(mask.ravel(), ex[key + "_mask"])
        np.testing.assert_allclose(O.ravel(), [_expr(ex[key + "_O_expr"])], rtol=1e-6)
        np.testing.assert_allclose(LSE.ravel(), [_expr(ex[key + "_LSE_expr"])], atol=1e-6)


# ----------------------------------------------------------------------------- dense


@pytest.mark.parametrize("L,H,Hkv,d", [(70, 4, 2, 16), (33, 2, 2, 8)])
def test_dense_fwd_matches_torch(orc, L, H, Hkv, d):
    Q, K, V, _ = _rand(2, L, H, Hkv, d, seed=L)
    scale = 1 / math.sqrt(d)
    O, LSE = orc.dense_fwd(Q, K, V, scale, blk=16)
    O_t, LSE_t = _sdpa(Q, K, V, scale)
    np.testing.assert_allclose(O, O_t, atol=1e-12)
    np.testing.assert_allclose(LSE, LSE_t, atol=1e-12)


def test_dense_bwd_matches_autograd(orc):
    Q, K, V, dO = _rand(1, 37, 4, 2, 8, seed=3)
    scale = 0.3
    dQ, dK, dV = orc.dense_bwd(Q, K, V, dO, scale)
    q, k, v = (_torch_bhld(x).requires_grad_() for x in (Q, K, V))
    out = F.scaled_dot_product_attention(q, _expand_kv(k, 2), _expand_kv(v, 2), is_causal=True,
                                         scale=scale)
    (out * _torch_bhld(dO)).sum().backward()
    np.testing.assert_allclose(dQ, q.grad.permute(0, 2, 1, 3).numpy(), atol=1e-11)
    np.testing.assert_allclose(dK, k.grad.permute(0, 2, 1, 3).numpy(), atol=1e-11)
    np.testing.assert_allclose(dV, v.grad.permute(0, 2, 1, 3).numpy(), atol=1e-11)


def test_dense_bwd_finite_difference(orc):
    """Central differences of sum(O * dO) through the oracle's own dense forward.

    The oracle takes float32 inputs, so perturbations use h = 2**-10 on values that
    are multiples of 2**-6 (exact in float32) and the loss is evaluated in fp64."""
    rng = np.random.default_rng(5)
    B, L, H, Hkv, d = 1, 9, 2, 1, 4
    Q, K, V = (np.round(rng.standard_normal(s) * 64) / 64 for s in
               ((B, L, H, d), (B, L, Hkv, d), (B, L, Hkv, d)))
    Q, K, V = (x.astype(np.float32) for x in (Q, K, V))
    dO = rng.choice([-1.0, 1.0], size=(B, L, H, d)).astype(np.float32)
    scale = 0.5
    dQ, dK, dV = orc.dense_bwd(Q, K, V, dO, scale)

    def loss(Q_, K_, V_):
        O, _ = orc.dense_fwd(Q_, K_, V_, scale, blk=4)
        return float((O * dO).sum())

    h = 2.0 ** -10
    for name, X, G in (("Q", Q, dQ), ("K", K, dK), ("V", V, dV)):
        for idx in [(0, 0, 0, 0), (0, 4, 0, 2), (0, L - 1, X.shape[2] - 1, d - 1)]:
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += h
            Xm[idx] -= h
            args_p = {"Q": Q, "K": K, "V": V}
            args_m = dict(args_p)
            args_p[name], args_m[name] = Xp, Xm
            fd = (loss(**{k + "_": v for k, v in args_p.items()}) -
                  loss(**{k + "_": v for k, v in args_m.items()})) / (2 * h)
            assert abs(fd - G[idx]) < 2e-5 * max(1.0, abs(G[idx])), (name, idx, fd, G[idx])


# ----------------------------------------------------------------------------- MALA fwd


@pytest.mark.parametrize("L,blk", [(96, 16), (70, 16), (45, 8)])
def test_mala_tau0_is_dense(orc, L, blk):
    Q, K, V, _ = _rand(2, L, 4, 2, 16, seed=L + blk, peak=3.0)
    scale = 0.25
    O, LSE, mask, _ = orc.mala_fwd(Q, K, V, scale, 0.0, blk=blk)
    T = mask.shape[-1]
    legal = np.tril(np.ones((T, T), dtype=bool))
    assert (mask[:, :, legal] == 1).all() and (mask[:, :, ~legal] == -1).all()
    O_t, LSE_t = _sdpa(Q, K, V, scale)
    np.testing.assert_allclose(O, O_t, atol=1e-12)
    np.testing.assert_allclose(LSE, LSE_t, atol=1e-12)


@pytest.mark.parametrize("tau", [0.1, 1.0, 10.0])
def test_mala_online_equals_explicit_set_form(orc, tau):
    Q, K, V, _ = _rand(1, 100, 4, 2, 16, seed=7, peak=6.0)
    a = orc.mala_fwd(Q, K, V, 0.5, tau, blk=8)
    b = orc.mala_fwd_setsum(Q, K, V, 0.5, tau, blk=8)
    np.testing.assert_array_equal(a[2], b[2])
    fin = np.isfinite(a[3]) & np.isfinite(b[3])
    np.testing.assert_allclose(a[3][fin], b[3][fin], atol=1e-10)
    np.testing.assert_allclose(a[0], b[0], atol=1e-12)
    np.testing.assert_allclose(a[1], b[1], atol=1e-12)
    # both forms must make non-trivial decisions on this input
    assert (a[2] == 0).any() and (a[2] == 1).sum() > a[2].shape[-1]


def test_mala_diagonal_always_retained(orc):
    Q, K, V, _ = _rand(2, 128, 4, 2, 16, seed=9, peak=4.0)
    _, _, mask, margin = orc.mala_fwd(Q, K, V, 0.25, 1.0, blk=16)
    T = mask.shape[-1]
    for i in range(T):
        assert (mask[:, :, i, i] == 1).all()
        assert np.isinf(margin[:, :, i, i]).all()


def _check_eq7(Q, K, scale, tau, blk, mask):
    """Brute force of Eq. (3)/(7) from raw scores and the recorded decisions: a skipped
    tile has exp(s_qk) / Z_t < tau / L_q for every legal key; a retained one has a row
    with exp(max s) / Z_t >= tau / L_q (or Z_t = 0)."""
    s = _scores(Q, K, scale)
    B, H, L, _ = s.shape
    T = mask.shape[-1]
    n_checked = 0
    for b in range(B):
        for h in range(H):
            for i in range(T):
                rows = np.arange(i * blk, min(L, (i + 1) * blk))
                Z = np.zeros(len(rows))
                for j in range(i, -1, -1):
                    cols = np.arange(j * blk, min(L, (j + 1) * blk))
                    st = s[b, h][np.ix_(rows, cols)]
                    legal = np.isfinite(st)
                    top = np.where(legal, st, -np.inf).max(axis=1)
                    has = legal.any(axis=1)
                    with np.errstate(divide="ignore"):
                        ratio = np.where(Z > 0, np.exp(top) / np.where(Z > 0, Z, 1), np.inf)
                    thr = tau / (rows + 1)
                    retain = bool((has & (ratio >= thr)).any())
                    assert retain == (mask[b, h, i, j] == 1), (b, h, i, j)
                    n_checked += 1
                    if retain:
                        Z += np.where(legal, np.exp(np.where(legal, st, 0.0)), 0.0).sum(axis=1)
    return n_checked


@pytest.mark.parametrize("tau", [0.5, 1.0, 4.0])
def test_mala_fwd_decisions_brute_force(orc, tau):
    Q, K, V, _ = _rand(1, 80, 2, 1, 16, seed=int(tau * 10), peak=6.0)
    _, _, mask, _ = orc.mala_fwd(Q, K, V, 0.25, tau, blk=8)
    assert _check_eq7(Q, K, 0.25, tau, 8, mask) > 0
    assert (mask == 0).any()


@pytest.mark.parametrize("tau", [0.1, 1.0, 10.0])
def test_mala_prop1_omitted_mass_bound(orc, tau):
    Q, K, V, _ = _rand(2, 160, 4, 2, 16, seed=11, peak=6.0)
    scale = 0.25
    _, LSE, mask, _ = orc.mala_fwd(Q, K, V, scale, tau, blk=16)
    _, LSE_d = _sdpa(Q, K, V, scale)
    eps = 1.0 - np.exp(LSE - LSE_d)  # App. C.2 omitted-mass definition
    assert (eps >= -1e-12).all()
    assert eps.max() <= tau / (1 + tau) + 1e-12
    assert (mask == 0).any()


@pytest.mark.parametrize("tau", [0.3, 1.0])
def test_mala_output_is_softmax_over_retained_tiles(orc, tau):
    Q, K, V, _ = _rand(2, 75, 4, 2, 16, seed=13, peak=3.0)
    scale, blk = 0.25, 16
    O, LSE, mask, _ = orc.mala_fwd(Q, K, V, scale, tau, blk=blk)
    O_t, LSE_t = _sdpa(Q, K, V, scale, mask=_expand_tiles(mask, 75, blk))
    np.testing.assert_allclose(O, O_t, atol=1e-12)
    np.testing.assert_allclose(LSE, LSE_t, atol=1e-12)


def test_mala_huge_tau_is_block_diagonal(orc):
    Q, K, V, _ = _rand(1, 64, 2, 2, 8, seed=17)
    scale, blk = 0.3, 16
    O, LSE, mask, _ = orc.mala_fwd(Q, K, V, scale, 1e30, blk=blk)
    T = mask.shape[-1]
    assert (mask[:, :, np.eye(T, dtype=bool)] == 1).all()
    assert (mask[:, :, np.tril(np.ones((T, T), bool), -1)] == 0).all()
    blockdiag = np.kron(np.eye(T, dtype=bool), np.ones((blk, blk), bool))[None, None]
    O_t, LSE_t = _sdpa(Q, K, V, scale, mask=np.broadcast_to(blockdiag, (1, 2, 64, 64)).copy())
    np.testing.assert_allclose(O, O_t, atol=1e-12)
    np.testing.assert_allclose(LSE, LSE_t, atol=1e-12)


def test_mala_fwd_units_match_full(orc):
    Q, K, V, _ = _rand(2, 100, 4, 2, 16, seed=19, peak=3.0)
    full = orc.mala_fwd(Q, K, V, 0.25, 1.0, blk=16)
    units = [(1, 3, 6), (0, 0, 0), (0, 2, 4)]
    part = orc.mala_fwd(Q, K, V, 0.25, 1.0, blk=16, units=units)
    for b, h, i in units:
        rows = slice(i * 16, min(100, i * 16 + 16))
        np.testing.assert_array_equal(part[0][b, rows, h], full[0][b, rows, h])
        np.testing.assert_array_equal(part[2][b, h, i], full[2][b, h, i])


def test_mala_forced_decisions_are_followed(orc):
    Q, K, V, _ = _rand(1, 64, 2, 1, 8, seed=23, peak=3.0)
    _, _, mask, _ = orc.mala_fwd(Q, K, V, 0.3, 1.0, blk=8)
    force = mask.copy()
    # flip one off-diagonal decision and check it is followed
    i, j = 7, 2
    force[0, 0, i, j] = 1 - mask[0, 0, i, j]
    _, _, m2, _ = orc.mala_fwd(Q, K, V, 0.3, 1.0, blk=8, force=force)
    assert m2[0, 0, i, j] == force[0, 0, i, j]
    np.testing.assert_array_equal(m2, force)


# ----------------------------------------------------------------------------- MALA bwd


def test_mala_bwd_tau0_is_dense_gradient(orc):
    Q, K, V, dO = _rand(1, 50, 4, 2, 8, seed=29, peak=2.0)
    scale = 0.35
    O, LSE, _, _ = orc.mala_fwd(Q, K, V, scale, 0.0, blk=16)
    dQ, dK, dV, bmask, _ = orc.mala_bwd(Q, K, V, O, LSE, dO, scale, 0.0, blk=16)
    T = bmask.shape[-1]
    assert (bmask[:, :, np.tril(np.ones((T, T), bool))] == 1).all()
    rQ, rK, rV = orc.dense_bwd(Q, K, V, dO, scale)
    np.testing.assert_allclose(dQ, rQ, atol=1e-11)
    np.testing.assert_allclose(dK, rK, atol=1e-11)
    np.testing.assert_allclose(dV, rV, atol=1e-11)


@pytest.mark.parametrize("tau", [0.2, 1.0, 5.0])
def test_mala_bwd_support_nested_in_fwd(orc, tau):
    Q, K, V, dO = _rand(2, 144, 4, 2, 16, seed=31, peak=3.0)
    O, LSE, fmask, _ = orc.mala_fwd(Q, K, V, 0.25, tau, blk=16)
    _, _, _, bmask, _ = orc.mala_bwd(Q, K, V, O, LSE, dO, 0.25, tau, blk=16)
    legal = fmask >= 0
    assert ((bmask[legal] == 1) <= (fmask[legal] == 1)).all()
    assert (bmask[legal] == 0).sum() >= (fmask[legal] == 0).sum()


def test_mala_bwd_decisions_brute_force(orc):
    """Eq. (4) re-evaluated with numpy on the full score matrix."""
    Q, K, V, dO = _rand(2, 90, 4, 2, 16, seed=37, peak=4.0)
    scale, tau, blk = 0.4, 1.0, 16
    O, LSE, _, _ = orc.mala_fwd(Q, K, V, scale, tau, blk=blk)
    _, _, _, bmask, _ = orc.mala_bwd(Q, K, V, O, LSE, dO, scale, tau, blk=blk)
    s = _scores(Q, K, scale)
    L = s.shape[-1]
    th = np.log(tau) - np.log(np.arange(1, L + 1))
    y = s - LSE[..., None] - th[None, None, :, None]
    T = bmask.shape[-1]
    for i in range(T):
        for j in range(i + 1):
            blkmax = y[:, :, i * blk:(i + 1) * blk, j * blk:(j + 1) * blk].max(axis=(2, 3))
            np.testing.assert_array_equal(bmask[:, :, i, j], (blkmax >= 0).astype(np.int8))
    assert (bmask == 0).any() and (bmask == 1).any()


def test_mala_bwd_frozen_support_is_autograd_of_masked_softmax(orc):
    """With backward decisions forced to the forward support R, MALA backward is the
    exact gradient of softmax attention renormalised over R (a smooth function)."""
    Q, K, V, dO = _rand(1, 60, 4, 2, 16, seed=41, peak=4.0)
    scale, blk, tau = 0.4, 16, 1.0
    O, LSE, fmask, _ = orc.mala_fwd(Q, K, V, scale, tau, blk=blk)
    assert (fmask == 0).any()
    dQ, dK, dV, _, _ = orc.mala_bwd(Q, K, V, O, LSE, dO, scale, tau, blk=blk, force=fmask)
    m = torch.from_numpy(_expand_tiles(fmask, 60, blk)) & torch.ones(60, 60, dtype=torch.bool).tril()
    q, k, v = (_torch_bhld(x).requires_grad_() for x in (Q, K, V))
    out = F.scaled_dot_product_attention(q, _expand_kv(k, 2), _expand_kv(v, 2), attn_mask=m,
                                         scale=scale)
    (out * _torch_bhld(dO)).sum().backward()
    np.testing.assert_allclose(dQ, q.grad.permute(0, 2, 1, 3).numpy(), atol=1e-11)
    np.testing.assert_allclose(dK, k.grad.permute(0, 2, 1, 3).numpy(), atol=1e-11)
    np.testing.assert_allclose(dV, v.grad.permute(0, 2, 1, 3).numpy(), atol=1e-11)


def test_mala_bwd_frozen_support_finite_difference(orc):
    """Same frozen-support gradient checked by central differences of the oracle's own
    forward with its decisions forced (no library involved)."""
    rng = np.random.default_rng(43)
    B, L, H, Hkv, d, blk = 1, 24, 2, 1, 4, 4
    Q, K, V = (np.round(rng.standard_normal(s) * 64) / 64 for s in
               ((B, L, H, d), (B, L, Hkv, d), (B, L, Hkv, d)))
    Q[:, :, :] += 2.0 * K[:, rng.integers(0, L, size=L), :1]  # peaked rows
    Q, K, V = (np.round(x * 64).astype(np.float32) / 64 for x in (Q, K, V))
    dO = rng.choice([-1.0, 1.0], size=(B, L, H, d)).astype(np.float32)
    scale, tau = 0.5, 1.0
    O, LSE, fmask, _ = orc.mala_fwd(Q, K, V, scale, tau, blk=blk)
    dQ, dK, dV, _, _ = orc.mala_bwd(Q, K, V, O, LSE, dO, scale, tau, blk=blk, force=fmask)

    def loss(Q_, K_, V_):
        O_, _, _, _ = orc.mala_fwd(Q_, K_, V_, scale, tau, blk=blk, force=fmask)
        return float((O_ * dO).sum())

    h = 2.0 ** -10
    for name, X, G in (("Q", Q, dQ), ("K", K, dK), ("V", V, dV)):
        for idx in [(0, 1, 0, 0), (0, 13, 0, 3), (0, L - 1, X.shape[2] - 1, 1)]:
            args = {"Q_": Q, "K_": K, "V_": V}
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += h
            Xm[idx] -= h
            ap, am = dict(args), dict(args)
            ap[name + "_"], am[name + "_"] = Xp, Xm
            fd = (loss(**ap) - loss(**am)) / (2 * h)
            assert abs(fd - G[idx]) < 2e-5 * max(1.0, abs(G[idx])), (name, idx, fd, G[idx])


def test_mala_bwd_huge_tau_skips_everything(orc):
    Q, K, V, dO = _rand(1, 48, 2, 1, 8, seed=47)
    O, LSE, _, _ = orc.mala_fwd(Q, K, V, 0.3, 1e30, blk=16)
    dQ, dK, dV, bmask, _ = orc.mala_bwd(Q, K, V, O, LSE, dO, 0.3, 1e30, blk=16)
    assert (bmask[bmask >= 0] == 0).all()
    assert not dQ.any() and not dK.any() and not dV.any()


def test_mala_bwd_units_match_full(orc):
    Q, K, V, dO = _rand(2, 96, 4, 2, 16, seed=53, peak=3.0)
    O, LSE, _, _ = orc.mala_fwd(Q, K, V, 0.25, 1.0, blk=16)
    full = orc.mala_bwd(Q, K, V, O, LSE, dO, 0.25, 1.0, blk=16)
    kvu = [(1, 1, 2), (0, 0, 5)]
    qu = [(0, 3, 5), (1, 0, 1)]
    part = orc.mala_bwd(Q, K, V, O, LSE, dO, 0.25, 1.0, blk=16, kv_units=kvu, q_units=qu)
    for b, g, j in kvu:
        r = slice(j * 16, j * 16 + 16)
        np.testing.assert_array_equal(part[1][b, r, g], full[1][b, r, g])
        np.testing.assert_array_equal(part[2][b, r, g], full[2][b, r, g])
    for b, h, i in qu:
        r = slice(i * 16, i * 16 + 16)
        np.testing.assert_array_equal(part[0][b, r, h], full[0][b, r, h])


# ----------------------------------------------------------------------------- decode


def _decode_ref(q, K, V, scale, keymask=None):
    B, H, d = q.shape
    G = H // K.shape[2]
    qq = torch.from_numpy(q).double()[:, :, None, :]
    kk = _expand_kv(_torch_bhld(K), G)
    vv = _expand_kv(_torch_bhld(V), G)
    m = None if keymask is None else torch.from_numpy(keymask)[:, :, None, :]
    out = F.scaled_dot_product_attention(qq, kk, vv, attn_mask=m, scale=scale)[:, :, 0]
    s = (qq @ kk.transpose(-1, -2))[:, :, 0] * scale
    if m is not None:
        s = s.masked_fill(~m[:, :, 0], float("-inf"))
    return out.numpy(), torch.logsumexp(s, dim=-1).numpy()


@pytest.mark.parametrize("S", [1, 2, 5])
def test_decode_tau0_is_dense_last_row(orc, S):
    rng = np.random.default_rng(59)
    q = rng.standard_normal((2, 4, 16)).astype(np.float32)
    K = rng.standard_normal((2, 150, 2, 16)).astype(np.float32)
    V = rng.standard_normal((2, 150, 2, 16)).astype(np.float32)
    O, LSE, mask, _, _, _ = orc.mala_decode(q, K, V, 0.25, 0.0, S, blk=16)
    assert (mask == 1).all()
    O_t, LSE_t = _decode_ref(q, K, V, 0.25)
    np.testing.assert_allclose(O, O_t, atol=1e-12)
    np.testing.assert_allclose(LSE, LSE_t, atol=1e-12)


def _planted_decode(seed, B=2, H=4, Hkv=2, Nk=300, d=16):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, d)).astype(np.float32)
    K = rng.standard_normal((B, Nk, Hkv, d)).astype(np.float32)
    V = rng.standard_normal((B, Nk, Hkv, d)).astype(np.float32)
    G = H // Hkv
    for b in range(B):
        for g in range(Hkv):
            for r, p in enumerate(rng.choice(Nk, 6, replace=False)):
                h = g * G + r % G
                K[b, p, g] = 2.5 * q[b, h] / np.linalg.norm(q[b, h]) * math.sqrt(d)
    return q, K, V


@pytest.mark.parametrize("S,tau", [(1, 1.0), (3, 1.0), (4, 0.2)])
def test_decode_is_softmax_over_union_and_eq7(orc, S, tau):
    q, K, V = _planted_decode(61)
    scale, blk = 0.25, 16
    O, LSE, mask, _, part_o, part_z = orc.mala_decode(q, K, V, scale, tau, S, blk=blk)
    Nk = K.shape[1]
    T = mask.shape[-1]
    keymask = np.repeat(mask == 1, blk, axis=-1)[..., :Nk]
    O_t, LSE_t = _decode_ref(q, K, V, scale, keymask)
    np.testing.assert_allclose(O, O_t, atol=1e-12)
    np.testing.assert_allclose(LSE, LSE_t, atol=1e-12)
    assert (mask == 0).any()
    # Eq. (7) against each split's partial normaliser, brute force from raw scores
    G = q.shape[1] // K.shape[2]
    Kx = np.repeat(K.astype(np.float64), G, axis=2)
    s = np.einsum("bhd,bkhd->bhk", q.astype(np.float64), Kx) * scale
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            for lo, hi in orc.decode_split_bounds(T, S):
                Z = 0.0
                for t in range(hi - 1, lo - 1, -1):
                    st = s[b, h, t * blk:min(Nk, (t + 1) * blk)]
                    retain = Z == 0.0 or np.exp(st.max()) / Z >= tau / Nk
                    assert retain == (mask[b, h, t] == 1)
                    if t == hi - 1:
                        assert retain  # first tile of every split
                    if retain:
                        Z += np.exp(st).sum()
    # merge of the per-split partials is the log-sum-exp reduction
    z = np.logaddexp.reduce(part_z, axis=-1)
    np.testing.assert_allclose(z, LSE, atol=1e-12)


def test_decode_huge_tau_keeps_first_tile_of_each_split(orc):
    q, K, V = _planted_decode(67)
    _, _, mask, _, _, _ = orc.mala_decode(q, K, V, 0.25, 1e30, 3, blk=16)
    T = mask.shape[-1]
    first = np.zeros(T, np.int8)
    for lo, hi in orc.decode_split_bounds(T, 3):
        first[hi - 1] = 1
    assert (mask == first).all()


# ----------------------------------------------------------------------------- generator


def test_synth_is_deterministic_and_bf16_exact():
    w = synth.WORKLOADS["peaked1k"]
    a = synth.make_training(w, L=256)
    b = synth.make_training(w, L=256)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    for k in ("Q", "K", "V"):
        np.testing.assert_array_equal(synth.round_bf16(a[k]), a[k])
    assert set(np.unique(a["dO"])) == {-1.0, 1.0}
    t = torch.from_numpy(a["Q"]).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(t, a["Q"])  # torch's bf16 conversion agrees


def test_synth_round_bf16_ties_to_even():
    x = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.5, 3.0e38], np.float32)
    r = synth.round_bf16(x)
    np.testing.assert_array_equal(r[:3], [1.0, 1.0 + 2 ** -6, -1.5])
    np.testing.assert_array_equal(r, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


# ---------------------------------------------------------------------------- chunked prefill
# A chunk of Nq queries at the end of a sequence of Nk keys (§2.3: the forward serves
# inference prefill); row q sits at position Nk - Nq + q.


def _allowed_offset(B, H, Nq, Nk):
    off = Nk - Nq
    a = np.arange(Nk)[None, :] <= (off + np.arange(Nq))[:, None]
    return np.broadcast_to(a, (B, H, Nq, Nk)).copy()


def _sdpa_offset(Q, K, V, scale, allowed):
    """Softmax attention over an explicit key mask [B,H,Nq,Nk] via torch in fp64."""
    G = Q.shape[2] // K.shape[2]
    q, k, v = _torch_bhld(Q), _expand_kv(_torch_bhld(K), G), _expand_kv(_torch_bhld(V), G)
    m = torch.from_numpy(allowed)
    out = F.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale)
    s = (q @ k.transpose(-1, -2)) * scale
    lse = torch.logsumexp(s.masked_fill(~m, float("-inf")), dim=-1)
    return out.permute(0, 2, 1, 3).numpy(), lse.numpy()


def _rand_chunk(B, Nq, Nk, H, Hkv, d, seed, peak=0.0):
    Q, K, V, _ = _rand(B, Nk, H, Hkv, d, seed, peak=peak)
    return np.ascontiguousarray(Q[:, Nk - Nq:]), K, V, Q


def test_prefill_full_length_equals_forward(orc):
    Q, K, V, _ = _rand(2, 70, 4, 2, 16, seed=41, peak=4.0)
    a = orc.mala_prefill(Q, K, V, 0.25, 1.0, blk=16)
    b = orc.mala_fwd(Q, K, V, 0.25, 1.0, blk=16)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_prefill_aligned_offset_equals_tail_of_forward(orc):
    # off = 48 = 3 blocks of 16: the chunk's query blocks are the forward's blocks 3..5
    Qc, K, V, Qf = _rand_chunk(1, 48, 96, 2, 1, 16, seed=42, peak=5.0)
    O, LSE, mask, margin = orc.mala_prefill(Qc, K, V, 0.25, 1.0, blk=16)
    Of, LSEf, maskf, marginf = orc.mala_fwd(Qf, K, V, 0.25, 1.0, blk=16)
    np.testing.assert_array_equal(O, Of[:, 48:])
    np.testing.assert_array_equal(LSE, LSEf[:, :, 48:])
    np.testing.assert_array_equal(mask, maskf[:, :, 3:])
    np.testing.assert_array_equal(margin, marginf[:, :, 3:])
    assert (mask == 0).any()


@pytest.mark.parametrize("Nq,Nk", [(37, 101), (16, 16), (1, 50), (64, 77)])
def test_prefill_tau0_is_dense_with_offset(orc, Nq, Nk):
    Qc, K, V, _ = _rand_chunk(2, Nq, Nk, 4, 2, 16, seed=43 + Nq)
    O, LSE, mask, _ = orc.mala_prefill(Qc, K, V, 0.3, 0.0, blk=16)
    O_t, LSE_t = _sdpa_offset(Qc, K, V, 0.3, _allowed_offset(2, 4, Nq, Nk))
    np.testing.assert_allclose(O, O_t, atol=1e-12)
    np.testing.assert_allclose(LSE, LSE_t, atol=1e-12)
    assert (mask[mask >= 0] == 1).all()


def _check_eq3_offset(Q, K, scale, tau, blk, mask):
    """Brute force of Eq. (3) with the causal offset: every decision re-derived from raw
    scores and the recorded decisions of the tiles visited before it."""
    B, Nq, H, _ = Q.shape
    Nk = K.shape[1]
    off = Nk - Nq
    G = H // K.shape[2]
    s = np.einsum("bqhd,bkhd->bhqk", Q.astype(np.float64),
                  np.repeat(K.astype(np.float64), G, axis=2)) * scale
    s[~_allowed_offset(B, H, Nq, Nk)] = -np.inf
    Tq = mask.shape[2]
    n = 0
    for b in range(B):
        for h in range(H):
            for i in range(Tq):
                rows = np.arange(i * blk, min(Nq, (i + 1) * blk))
                pos = off + rows
                Z = np.zeros(len(rows))
                for j in range(pos[-1] // blk, -1, -1):
                    cols = np.arange(j * blk, min(Nk, (j + 1) * blk))
                    st = s[b, h][np.ix_(rows, cols)]
                    legal = np.isfinite(st)
                    top = np.where(legal, st, -np.inf).max(axis=1)
                    has = legal.any(axis=1)
                    with np.errstate(divide="ignore", over="ignore"):
                        ratio = np.where(Z > 0, np.exp(top) / np.where(Z > 0, Z, 1), np.inf)
                    retain = bool((has & (ratio >= tau / (pos + 1))).any())
                    assert retain == (mask[b, h, i, j] == 1), (b, h, i, j)
                    n += 1
                    if retain:
                        Z += np.where(legal, np.exp(np.where(legal, st, 0.0)), 0.0).sum(axis=1)
                assert (mask[b, h, i, pos[-1] // blk + 1:] == -1).all()  # not legal
    return n


@pytest.mark.parametrize("tau", [0.5, 1.0, 4.0])
def test_prefill_decisions_brute_force(orc, tau):
    Qc, K, V, _ = _rand_chunk(1, 45, 117, 2, 1, 16, seed=44, peak=6.0)
    _, _, mask, _ = orc.mala_prefill(Qc, K, V, 0.25, tau, blk=8)
    assert _check_eq3_offset(Qc, K, 0.25, tau, 8, mask) > 0
    assert (mask == 0).any()


def test_prefill_output_is_softmax_over_retained_tiles(orc):
    Qc, K, V, _ = _rand_chunk(2, 40, 93, 4, 2, 16, seed=45, peak=3.0)
    O, LSE, mask, _ = orc.mala_prefill(Qc, K, V, 0.25, 1.0, blk=16)
    keep = np.kron(np.where(mask == 1, 1, 0), np.ones((16, 16), int))[:, :, :40, :93] > 0
    allowed = _allowed_offset(2, 4, 40, 93) & keep
    O_t, LSE_t = _sdpa_offset(Qc, K, V, 0.25, allowed)
    np.testing.assert_allclose(O, O_t, atol=1e-12)
    np.testing.assert_allclose(LSE, LSE_t, atol=1e-12)


def test_prefill_huge_tau_keeps_the_blocks_own_key_tiles(orc):
    # off = 53 is not a multiple of 16: a query block spans two key tiles, and each of
    # them is some row's first legal tile (l = 0), so both are retained; older tiles go
    Nq, Nk, blk = 40, 93, 16
    Qc, K, V, _ = _rand_chunk(1, Nq, Nk, 2, 2, 8, seed=46)
    O, LSE, mask, _ = orc.mala_prefill(Qc, K, V, 0.3, 1e30, blk=blk)
    off = Nk - Nq
    first_tile = ((off + (np.arange(Nq) // blk) * blk) // blk)  # tile of the block's first row
    allowed = _allowed_offset(1, 2, Nq, Nk) & (np.arange(Nk)[None, :] >= first_tile[:, None] * blk)
    O_t, LSE_t = _sdpa_offset(Qc, K, V, 0.3, allowed)
    np.testing.assert_allclose(O, O_t, atol=1e-12)
    np.testing.assert_allclose(LSE, LSE_t, atol=1e-12)
    for i in range(mask.shape[2]):
        jf = (off + i * blk) // blk
        jl = (off + min(Nq, (i + 1) * blk) - 1) // blk
        assert (mask[:, :, i, jf:jl + 1] == 1).all() and (mask[:, :, i, :jf] == 0).all()


def test_prefill_units_match_full(orc):
    Qc, K, V, _ = _rand_chunk(2, 50, 130, 4, 2, 16, seed=47, peak=4.0)
    full = orc.mala_prefill(Qc, K, V, 0.25, 1.0, blk=16)
    units = [(1, 3, 3), (0, 0, 0), (1, 2, 1)]
    part = orc.mala_prefill(Qc, K, V, 0.25, 1.0, blk=16, units=units)
    for b, h, i in units:
        rows = slice(i * 16, min(50, (i + 1) * 16))
        np.testing.assert_array_equal(part[0][b, rows, h], full[0][b, rows, h])
        np.testing.assert_array_equal(part[2][b, h, i], full[2][b, h, i])


@pytest.mark.parametrize("name", ["sinkband32k", "prevtok32k", "prevvar8k", "mixed8k"])
def test_synth_training_structures_deterministic_and_bf16(name):
    w = synth.WORKLOADS[name]
    a = synth.make_training(w, L=384)
    b = synth.make_training(w, L=384)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    for k in ("Q", "K", "V"):
        np.testing.assert_array_equal(synth.round_bf16(a[k]), a[k])
        assert np.isfinite(a[k]).all()


@pytest.mark.parametrize("name", ["decode128k", "heavy128k"])
def test_synth_decode_structures_deterministic_and_bf16(name):
    w = synth.WORKLOADS[name]
    a = synth.make_decode(w, Nk=2048, B=1)
    b = synth.make_decode(w, Nk=2048, B=1)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
        np.testing.assert_array_equal(synth.round_bf16(a[k]), a[k])


def test_heavy_hitters_dominate_their_split(orc):
    """The heavy128k recipe's claim: every 8th key tile holds a key that every head of the
    group scores more than log(N_k / tau) = log(131072) ~ 11.8 above every other key, so a
    split's tiles after its first heavy hitter fall below tau / N_k."""
    w = synth.WORKLOADS["heavy128k"]
    d = synth.make_decode(w, Nk=4096, B=1)
    G = w.H // w.H_kv
    q = d["q"][0].astype(np.float64)
    K = d["K"][0].astype(np.float64)
    for h in range(w.H):
        s = K[:, h // G] @ q[h] * w.scale
        heavy = s[7 * 128 + 64::8 * 128]
        rest = np.delete(s, np.arange(7 * 128 + 64, 4096, 8 * 128))
        assert heavy.min() > rest.max() + math.log(131072)
