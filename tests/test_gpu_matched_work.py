"""The matched-work study (MassAlloc Attention §3 Table 1, App. C.2) with MALA's
decisions taken from the sm_100a forward's tile mask."""

import pytest
import torch

from mass_adaptive_sparse_fwd_b200 import matched_work as MW

pytestmark = pytest.mark.gpu


def test_study_on_gpu_decisions():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    res = MW.run_study("prevvar8k", seeds=(1, 3), tau=1.0, L=2048)
    names = ("mala", "per_instance", "static_head_pos", "position_only")
    assert len({res[k]["tiles"] for k in names}) == 1  # exactly matched total work
    assert res["mala"]["tiles"] < res["legal_tiles"]    # something was skipped
    assert res["per_instance"]["omitted_mass_pct"] <= res["mala"]["omitted_mass_pct"] + 1e-12
