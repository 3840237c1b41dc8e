"""The allocation-free decode entry point against the regular one (GPU).

mala_decode_noalloc is meant for callers that may not allocate device memory on their
hot path; it runs the same decode kernel on scratch that lives in a fixed array inside
the library.  This file is collected last so that a run stopping at the first failure
has already run every other test."""

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


# (name, B, H, H_kv, N_k, d, dtype, splits): one head slot per decision lane (groups of
# up to 4), two slots (groups of 5..8) at d = 64, and the fp32 path
SHAPES = [
    ("group4_d128", 2, 8, 2, 3000, 128, "bf16", 3),
    ("group8_d64", 1, 16, 2, 2500, 64, "bf16", 4),
    ("fp32_d64", 2, 4, 2, 700, 64, "fp32", 2),
]


def _inputs(name, B, H, Hkv, Nk, d, dtype, seed=31):
    w = synth.Workload(f"noalloc_{name}", B, H, Hkv, Nk, d, dtype, "planted", seed, decode=True)
    dec = synth.make_decode(w)
    return w, dec, tuple(P.to_dev(dec[k], dtype) for k in ("q", "K", "V"))


def _regular(mala, q, K, V, scale, S):
    B, H, d = q.shape
    Nk, Hkv = K.shape[1], K.shape[2]
    mask = torch.full((B, H, mala.n_tiles(Nk)), 255, dtype=torch.uint8, device="cuda")
    dt = 0 if q.dtype == torch.bfloat16 else 1
    ws = mala.alloc_workspace(mala.decode_workspace_bytes(B, H, Hkv, Nk, d, dt, S), "cuda")
    O, L = mala.mala_decode(q, K, V, scale, 1.0, num_splits=S, workspace=ws, tile_mask=mask)
    torch.cuda.synchronize()
    assert mala.read_device_error(ws) == 0
    return O.float().cpu().numpy(), L.cpu().numpy(), mask.cpu().numpy()


def _noalloc(mala, q, K, V, scale, S):
    B, H, _ = q.shape
    mask = torch.full((B, H, mala.n_tiles(K.shape[1])), 255, dtype=torch.uint8, device="cuda")
    O, L = mala.mala_decode_noalloc(q, K, V, scale, 1.0, num_splits=S, tile_mask=mask)
    torch.cuda.synchronize()
    return O.float().cpu().numpy(), L.cpu().numpy(), mask.cpu().numpy()


@pytest.mark.parametrize("shape", SHAPES, ids=[s[0] for s in SHAPES])
def test_noalloc_decode_matches_regular_decode_twice(mala, orc, shape):
    name, B, H, Hkv, Nk, d, dtype, S = shape
    w, dec, (q, K, V) = _inputs(*shape[:7])
    O_ref, L_ref, M_ref = _regular(mala, q, K, V, w.scale, S)
    for _ in range(2):  # the second call sees the first call's leftovers in the array
        O, L, M = _noalloc(mala, q, K, V, w.scale, S)
        np.testing.assert_array_equal(M, M_ref)  # same decisions
        P.check_output(O, O_ref, np.ones(O.shape, bool))
        assert np.abs(L - L_ref).max() < P.LSE_ABS
    # and against the fp64 oracle on the same decisions
    oO, oL, _, _, _, _ = orc.mala_decode(dec["q"], dec["K"], dec["V"], w.scale, 1.0, S,
                                         force=M.astype(np.int8))
    P.check_output(O, oO, np.ones(O.shape, bool))
    assert np.abs(L - oL).max() < P.LSE_ABS


def test_noalloc_leftovers_of_a_larger_call(mala):
    """A larger call (more heads, more splits) leaves partials and tickets in the shared
    array; a smaller call right after it must not see them."""
    wb, _, (qb, Kb, Vb) = _inputs("large", 4, 32, 8, 4096, 128, "bf16", seed=41)
    ws, _, (qs, Ks, Vs) = _inputs("small", 1, 8, 2, 1100, 128, "bf16", seed=42)
    O_ref, L_ref, M_ref = _regular(mala, qs, Ks, Vs, ws.scale, 2)
    for _ in range(2):
        _noalloc(mala, qb, Kb, Vb, wb.scale, 16)
        O, L, M = _noalloc(mala, qs, Ks, Vs, ws.scale, 2)
        np.testing.assert_array_equal(M, M_ref)
        P.check_output(O, O_ref, np.ones(O.shape, bool))
        assert np.abs(L - L_ref).max() < P.LSE_ABS
