"""Shared helpers of the GPU-vs-oracle parity tests.

Tolerances:
  * O: max-abs 1e-2 and mean-abs 1e-3 against the fp64 oracle (bf16 output).  The
    max-abs bound is applied to |O - O_ref| / max(1, |O_ref|): bf16 storage alone has a
    half-ulp of 2^-8 |O|, which exceeds 1e-2 once |O| > 2.56 (peaked rows copy a
    single V row, whose entries reach 4-5 for N(0, 1) values).  The raw max-abs and the
    number of elements above 1e-2 are recorded next to the scaled figure.
  * LSE: abs 2e-3 (fp32 accumulation with hardware exp2 / log2).
  * dQ, dK, dV: relative Frobenius error 2e-2.
  * Tile decisions.  The kernels export the margin of every test they run (the
    library's debug hook): the quantity whose sign is the decision, in natural-log
    units.  Each test compares it tile by tile with the fp64 oracle's margin for the
    same tile (the oracle replays the GPU's decisions, so both evaluate the same
    retained support) and asserts that
      - the exported margins reproduce the GPU's decisions exactly (margin >= 0 iff
        retained), and both sides agree on which tiles have an infinite margin (a row's
        first retained tile);
      - |margin_gpu - margin_oracle| <= MARGIN_ERR on every tile (a bound set from the
        measured error, a few times the largest seen over all configurations);
      - consequently a decision may differ from the oracle's only where the oracle's
        margin is within MARGIN_ERR of the threshold; the number of such flips is
        recorded and asserted per test.
    A 1e-6 band around the threshold would lie below the fp32 rounding of the quantities
    compared here (scores of magnitude 10-50, log-normalisers of magnitude 10-30,
    thresholds log(tau / L_q) near -10), so the bound is set from the measured error.
"""

from __future__ import annotations

import numpy as np
import torch

TILE = 128
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_ABS = 2e-3
GRAD_REL_FRO = 2e-2
# Largest allowed |margin_gpu - margin_oracle| (natural-log units), per kernel family:
# about 4x the largest error measured on a B200 over every parity case (forward and
# prefill 6.9e-6, backward 5.6e-6, decode 1.19e-5, fp32 path 7.7e-6).
MARGIN_ERR = {"fwd": 3e-5, "bwd": 2.5e-5, "decode": 5e-5, "fp32": 3e-5}

# One row per decision comparison and per output check, printed at the end of the run.
REPORT: list[dict] = []


def to_dev(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x)).to(device)
    return t.to(torch.bfloat16) if dtype == "bf16" else t.float()


def margin_buffer(n: int, device="cuda") -> torch.Tensor:
    return torch.empty(n, dtype=torch.float32, device=device)


def compare_decisions(label, family, gpu_mask, gpu_margin, orc_margin, sel, max_flips=0):
    """Decision parity on the tiles ``sel`` (legal tiles the oracle evaluated).

    ``gpu_margin`` / ``orc_margin`` are natural-log margins in the layout of the masks.
    Returns the report row (also appended to REPORT)."""
    bound = MARGIN_ERR[family]
    g = gpu_mask[sel].astype(np.int64)
    gm = np.asarray(gpu_margin, np.float64)[sel]
    om = np.asarray(orc_margin, np.float64)[sel]
    assert not np.isnan(gm).any(), f"{label}: a tested tile has no GPU margin"
    assert not np.isnan(om).any(), f"{label}: a selected tile has no oracle margin"
    # the exported margins are the kernel's own decisions
    assert np.array_equal(g == 1, gm >= 0), f"{label}: GPU margins disagree with GPU mask"
    # first-tile (+inf) structure agrees
    assert np.array_equal(np.isposinf(gm), np.isposinf(om)), f"{label}: infinite margins differ"
    assert not np.isneginf(gm).any() and not np.isneginf(om).any()
    fin = np.isfinite(gm)
    err = np.abs(gm[fin] - om[fin])
    flips = g != (om >= 0).astype(np.int64)
    row = {
        "label": label,
        "tiles": int(sel.sum()),
        "finite": int(fin.sum()),
        "retained": float(g.mean()) if g.size else 0.0,
        "flips": int(flips.sum()),
        "max_err": float(err.max()) if err.size else 0.0,
        "p999_err": float(np.quantile(err, 0.999)) if err.size else 0.0,
        "worst_flip": float(np.abs(om[flips]).max()) if flips.any() else 0.0,
        "min_abs_margin": float(np.abs(om[fin]).min()) if fin.any() else float("inf"),
        "bound": bound,
    }
    REPORT.append(row)
    assert row["max_err"] <= bound, (
        f"{label}: margin error {row['max_err']:.3g} above the bound {bound:.3g}")
    assert row["flips"] <= max_flips, f"{label}: {row['flips']} decisions flipped ({row})"
    return row


def check_output(O, O_ref, rows, label=None):
    diff = np.abs(O - O_ref)[rows]
    scaled = diff / np.maximum(1.0, np.abs(O_ref[rows]))
    out = {"label": label, "o_scaled_max": float(scaled.max()), "o_raw_max": float(diff.max()),
           "o_mean": float(diff.mean()), "o_over_1e-2": int((diff > O_MAX_ABS).sum()),
           "o_elems": int(diff.size)}
    if label is not None:
        REPORT.append(out)
    assert scaled.max() < O_MAX_ABS, (scaled.max(), diff.max())
    assert diff.mean() < O_MEAN_ABS, diff.mean()
    return float(diff.max()), float(diff.mean())


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def fwd_legal(B, H, T, units=None):
    legal = np.zeros((B, H, T, T), dtype=bool)
    if units is None:
        legal[:] = np.tril(np.ones((T, T), dtype=bool))
    else:
        for b, h, i in units:
            legal[b, h, i, : i + 1] = True
    return legal


def format_report(rows) -> str:
    lines = []
    dec = [r for r in rows if "flips" in r]
    out = [r for r in rows if "o_raw_max" in r]
    if dec:
        lines.append("decision parity (margins in natural-log units; GPU vs fp64 oracle)")
        lines.append(f"{'test':72s} {'tiles':>8s} {'kept':>6s} {'flips':>5s} {'max|dm|':>9s} "
                     f"{'p99.9|dm|':>9s} {'worst flip':>10s} {'min|m|':>9s}")
        for r in dec:
            lines.append(f"{r['label'][:72]:72s} {r['tiles']:8d} {r['retained']:6.3f} "
                         f"{r['flips']:5d} {r['max_err']:9.2e} {r['p999_err']:9.2e} "
                         f"{r['worst_flip']:10.2e} {r['min_abs_margin']:9.2e}")
    if out:
        lines.append("outputs (O vs oracle): scaled max |dO|/max(1,|O|), raw max, mean, "
                     "elements over 1e-2")
        for r in out:
            lines.append(f"{r['label'][:72]:72s} {r['o_scaled_max']:9.2e} {r['o_raw_max']:9.2e} "
                         f"{r['o_mean']:9.2e} {r['o_over_1e-2']:6d}/{r['o_elems']}")
    return "\n".join(lines)
