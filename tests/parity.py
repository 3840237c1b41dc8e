"""Shared helpers of the GPU-vs-oracle parity tests.

Tolerances (derived in the design doc):
  * O: max-abs 1e-2 and mean-abs 1e-3 against the fp64 oracle (bf16 output).  The
    max-abs bound is applied to |O - O_ref| / max(1, |O_ref|): bf16 storage alone has a
    half-ulp of 2^-8 |O|, which exceeds 1e-2 once |O| > 2.56 (peaked rows copy a
    single V row, whose entries reach 4-5 for N(0, 1) values).
  * LSE: abs 2e-3 (fp32 accumulation with hardware exp2 / log2).
  * dQ, dK, dV: relative Frobenius error 2e-2.
  * Tile decisions: bit-exact, except where the oracle's margin lies within the
    decision band of the tile: 1e-6 + 1e-5 (fp32 running-sum error) + the fp32 score
    error bound d * 2^-22 * scale * max|Q_q| * max|K_k| (Cauchy-Schwarz bound of the
    accumulated dot-product rounding).  Near-threshold flips are counted and reported.
"""

from __future__ import annotations

import numpy as np
import torch

TILE = 128
O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_ABS = 2e-3
GRAD_REL_FRO = 2e-2


def to_dev(x: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x)).to(device)
    return t.to(torch.bfloat16) if dtype == "bf16" else t.float()


def tile_bands(Q, K, scale, G):
    """Per-tile decision band [B, H, T, T] for the forward / backward tests."""
    B, L, H, d = Q.shape
    T = (L + TILE - 1) // TILE
    qn = np.linalg.norm(Q.astype(np.float64), axis=-1)  # [B, L, H]
    kn = np.linalg.norm(K.astype(np.float64), axis=-1)  # [B, L, Hkv]
    pad = T * TILE - L
    qn = np.pad(qn, ((0, 0), (0, pad), (0, 0))).reshape(B, T, TILE, H).max(axis=2)  # [B,T,H]
    kn = np.pad(kn, ((0, 0), (0, pad), (0, 0))).reshape(B, T, TILE, -1).max(axis=2)
    kn = np.repeat(kn, G, axis=2)  # per query head
    score_err = d * 2.0 ** -22 * scale * qn.transpose(0, 2, 1)[:, :, :, None] * \
        kn.transpose(0, 2, 1)[:, :, None, :]
    return 1e-6 + 1e-5 + score_err


def compare_masks(gpu_mask, oracle_margin, band, legal):
    """Returns (n_tiles, n_mismatch_in_band, n_bad, worst_bad_margin)."""
    g = gpu_mask[legal].astype(np.int64)
    m = oracle_margin[legal]
    b = np.broadcast_to(band, gpu_mask.shape)[legal]
    orc_keep = (m >= 0).astype(np.int64)
    mism = g != orc_keep
    near = mism & (np.abs(m) < b)
    bad = mism & ~near
    worst = float(np.abs(m[bad]).max()) if bad.any() else 0.0
    return int(legal.sum()), int(near.sum()), int(bad.sum()), worst


def check_output(O, O_ref, rows):
    diff = np.abs(O - O_ref)[rows]
    scaled = diff / np.maximum(1.0, np.abs(O_ref[rows]))
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
