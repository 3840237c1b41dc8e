"""Failure handling of the kernels' bounded waits, tested without a GPU fault: a wait
that nothing satisfies runs out, records MALA_ERR_TIMEOUT in the workspace error word,
returns, and the context keeps working (a normal forward afterwards is correct)."""

import time

import numpy as np
import pytest
import torch

from mass_adaptive_sparse_fwd_b200 import synth
from tests import parity as P

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_reports_timeout(orc):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from mass_adaptive_sparse_fwd_b200 import mala

    ws = mala.alloc_workspace(4096, "cuda")
    budget = 20_000_000  # 20 ms
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    mala.selftest_wait_timeout(ws, budget)
    err = mala.read_device_error(ws)  # synchronises
    elapsed = time.perf_counter() - t0
    assert err & 0xFF == 4  # MALA_ERR_TIMEOUT
    assert (err >> 8) == 0xF00 + 1  # which wait gave up
    assert elapsed >= budget * 1e-9 * 0.9
    assert mala.read_device_error(ws) == 0  # cleared by the read above

    # the context is still usable: a forward right after it matches the oracle
    w, inp = synth.small_training(B=1, H=2, Hkv=1, L=256, d=64, structure="peaked", seed=5)
    Q, K, V = (P.to_dev(inp[k], "bf16") for k in ("Q", "K", "V"))
    wsf = mala.alloc_workspace(mala.fwd_workspace_bytes(1, 2, 1, 256, 64), "cuda")
    O, LSE = mala.mala_fwd(Q, K, V, w.scale, 0.0, workspace=wsf)
    torch.cuda.synchronize()
    assert mala.read_device_error(wsf) == 0
    oO, oLSE = orc.dense_fwd(inp["Q"], inp["K"], inp["V"], w.scale)
    P.check_output(O.float().cpu().numpy(), oO, np.ones(oO.shape[:-1], bool))
