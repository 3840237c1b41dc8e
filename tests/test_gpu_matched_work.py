"""The matched-work study (MassAlloc Attention §3 Table 1, App. C.2) with MALA's
decisions taken from the sm_100a forward's tile mask; the decisions the study consumes
are checked against the fp64 oracle first."""

import numpy as np
import pytest
import torch

from mass_adaptive_sparse_fwd_b200 import matched_work as MW
from tests import parity as P

pytestmark = pytest.mark.gpu


def test_study_on_gpu_decisions(orc):
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    seen = []

    def audit(w, inp, mask, margin):
        # the study's MALA decisions agree with the oracle's (GPU decisions replayed)
        B, L, H, _ = inp["Q"].shape
        T = mask.shape[-1]
        legal = P.fwd_legal(B, H, T)
        force = np.where(legal, mask.astype(np.int16), -1).astype(np.int8)
        oO, _, _, omargin = orc.mala_fwd(inp["Q"], inp["K"], inp["V"], w.scale, 1.0, force=force)
        P.compare_decisions(f"fwd {w.name}:{w.structure} seed {w.seed} L{L} (study)", "fwd",
                            mask, margin, omargin, legal)
        seen.append(float(mask[legal].mean()))

    res = MW.run_study("prevvar8k", seeds=(1, 3), tau=1.0, L=2048, on_decisions=audit)
    assert len(seen) == 2 and all(s < 1.0 for s in seen)
    names = ("mala", "per_instance", "static_head_pos", "position_only")
    assert len({res[k]["tiles"] for k in names}) == 1  # exactly matched total work
    assert res["mala"]["tiles"] < res["legal_tiles"]    # something was skipped
    assert res["per_instance"]["omitted_mass_pct"] <= res["mala"]["omitted_mass_pct"] + 1e-12
