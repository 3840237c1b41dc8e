"""The allocation-free decode entry point against the regular one (GPU).

mala_decode_noalloc is meant for callers that may not allocate device memory on their
hot path; it runs the same decode kernel on scratch that lives in a fixed array inside
the library.  This file is collected last so that a run stopping at the first failure
has already run every other test."""

import ctypes

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


def test_noalloc_decode_matches_regular_decode_twice(mala):
    w = synth.Workload("noalloc_decode", 2, 8, 2, 3000, 128, "bf16", "planted", 31, decode=True)
    dec = synth.make_decode(w)
    q, K, V = (P.to_dev(dec[k], "bf16") for k in ("q", "K", "V"))
    S = 3
    ws = mala.alloc_workspace(mala.decode_workspace_bytes(2, 8, 2, 3000, 128, 0, S), "cuda")
    O_ref, L_ref = mala.mala_decode(q, K, V, w.scale, 1.0, num_splits=S, workspace=ws)
    torch.cuda.synchronize()
    assert mala.read_device_error(ws) == 0
    O_ref, L_ref = O_ref.float().cpu().numpy(), L_ref.cpu().numpy()
    for _ in range(2):  # the second call sees the first call's leftovers in the array
        O, L = mala.mala_decode_noalloc(q, K, V, w.scale, 1.0, num_splits=S)
        torch.cuda.synchronize()
        O, L = O.float().cpu().numpy(), L.cpu().numpy()
        P.check_output(O, O_ref, np.ones(O.shape, bool))
        assert np.abs(L - L_ref).max() < P.LSE_ABS


def test_noalloc_decode_rejects_oversized_problems(mala):
    lib = mala.lib()
    p = ctypes.c_void_p(1 << 20)
    # 64 x 64 heads x 1024 splits of (128 + 1) floats is far beyond the fixed scratch
    st = lib.mala_decode_noalloc(p, p, p, p, p, 64, 64, 8, 131072, 128, 0, 0.1, 1.0, 1024, 0,
                                 None, None)
    assert st == 5  # MALA_ERR_WORKSPACE
