"""Seeded synthetic inputs for the MALA workloads.

This module holds no attention arithmetic: it only draws tensors.  Both the CUDA path
(tests, bench) and the CPU oracle consume exactly these values.  Every draw comes from
numpy's Philox counter-based generator keyed by (config seed, tensor id, chunk), so a
tensor is reproducible on any machine with the same numpy.

All tensors are returned as float32 numpy arrays whose values are already rounded to
the compute dtype (round-to-nearest-even to bf16 for bf16 workloads), so converting
them to bf16 on the device is exact and the oracle widens the same values to fp64.

Workloads (the attention page's own experiments run on real model states, which are not
available; these synthetic distributions stand in for them):

* ``tiny256``     B=1, H=2, H_kv=2, L=256, d=64, fp32; Q, K, V ~ N(0, 1)
* ``peaked1k``    B=2, H=8, H_kv=2, L=1024, d=128, bf16; K ~ N(0, 1); query row t is
                  3.0 x the mean of 4 keys drawn uniformly (with replacement) from its
                  causal prefix [0, t] of its own KV head, plus N(0, 1) noise
* ``mixed8k``     B=1, H=16, H_kv=4, L=8192, d=128, bf16; heads 0-7 peaked as above,
                  heads 8-15 diffuse (Q ~ N(0, 1))
* ``sinkband32k`` B=1, H=32, H_kv=8, L=32768, d=128, bf16; K ~ N(0, 1) with key 0
                  scaled by 4 (attention sink); q_t = 0.5 u_t + sqrt(0.75) n_t with
                  u_t = (1/sqrt(w)) sum_{s=t-w}^{t-1} K_s, w = min(64, t), u_0 = 0
* ``decode128k``  B=4, H=32, H_kv=8, N_k=131072, d=128, bf16; K, V, q ~ N(0, 1); per
                  (b, KV head) 16 distinct random positions get a planted key
                  3.0 * sqrt(d) * q_h / |q_h| + N(0, 1), h cycling over the group's heads
* ``heavy128k``   decode128k's shape, K, V, q ~ N(0, 1), with one heavy hitter per
                  (b, KV head) at key 64 of every 8th tile (tiles 7, 15, ...):
                  28 * sum_h q_h / |q_h| + 0.1 N(0, 1) over the group's heads
* ``sinkband128k`` B=1, H=8, H_kv=1, L=131072, d=128, bf16; sink + band states as
                  ``sinkband32k`` (one rank of an 8-way head-sharded 64/8-head model)
* ``prevvar8k``   B=1, H=16, H_kv=4, L=8192, d=128, bf16; "previous-token" heads whose
                  strength (8 + 12 u_h) and noise (0.3 + 0.7 v_h) vary per head and seed
                  (the matched-work study's input)
* ``prevtok32k``  B=1, H=32, H_kv=8, L=32768, d=128, bf16; concentrated "previous-token"
                  heads: q_t = 18 sqrt(d) K_{t-1} / |K_{t-1}|^2 + 0.3 N(0, 1), so the
                  previous token's scaled score is ~18 and the rest of the row is a flat
                  tail of 1e-5 .. 2e-3 of the mass (most off-diagonal tiles skippable)

V ~ N(0, 1) everywhere; dO is a Rademacher (+-1) probe.
"""

from __future__ import annotations

import concurrent.futures as cf
import math
import os
from dataclasses import dataclass, field

import numpy as np

# tensor ids used in the Philox key
_Q, _K, _V, _DO, _POS, _NOISE, _PLANT = 1, 2, 3, 4, 5, 6, 7


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    H_kv: int
    L: int
    d: int
    dtype: str  # "bf16" or "fp32"
    structure: str  # normal | peaked | half_peaked | sink_band | planted
    seed: int
    decode: bool = False
    taus: tuple = field(default=(1.0,))

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


WORKLOADS = {
    "tiny256": Workload("tiny256", 1, 2, 2, 256, 64, "fp32", "normal", 0, taus=(0.0, 1.0)),
    "peaked1k": Workload("peaked1k", 2, 8, 2, 1024, 128, "bf16", "peaked", 1),
    "mixed8k": Workload("mixed8k", 1, 16, 4, 8192, 128, "bf16", "half_peaked", 2,
                        taus=(1.0, 0.0, 1e-4, 1e-3)),
    "sinkband32k": Workload("sinkband32k", 1, 32, 8, 32768, 128, "bf16", "sink_band", 3),
    "decode128k": Workload("decode128k", 4, 32, 8, 131072, 128, "bf16", "planted", 4,
                           decode=True),
    # decode with a heavy hitter every 8th key tile: every split holds dominant keys, so
    # the tiles between them (and their V) are skipped
    "heavy128k": Workload("heavy128k", 4, 32, 8, 131072, 128, "bf16", "heavy", 7,
                          decode=True),
    # 128K-token training on one GPU: the per-rank shape of a 64-query-head / 8-KV-head
    # model under 8-way head sharding, with the sink + band states of sinkband32k
    "sinkband128k": Workload("sinkband128k", 1, 8, 1, 131072, 128, "bf16", "sink_band", 5),
    # concentrated heads: each query copies the previous token's key (a "previous-token"
    # head), so most off-diagonal tiles fall below tau / L_q and are skipped
    "prevtok32k": Workload("prevtok32k", 1, 32, 8, 32768, 128, "bf16", "prev_token", 6),
    # previous-token heads of varying concentration at 8K: the matched-work study input
    "prevvar8k": Workload("prevvar8k", 1, 16, 4, 8192, 128, "bf16", "prev_token_var", 8),
}


def _rng(seed: int, tensor: int, chunk: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[seed, tensor * 1_000_003 + chunk]))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def _round(x: np.ndarray, dtype: str) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    return round_bf16(x) if dtype == "bf16" else x


_CHUNK = 1 << 22  # elements per generator chunk (each chunk has its own Philox key)


def _chunked(shape, fill):
    """Fills a float32 array of ``shape`` chunk by chunk (rows of the flattened leading
    dimensions), in parallel threads; chunk c is always drawn from key c, so the result
    does not depend on the thread count."""
    shape = tuple(int(x) for x in shape)
    out = np.empty(shape, dtype=np.float32)
    flat = out.reshape(-1, shape[-1]) if len(shape) > 1 else out.reshape(1, -1)
    rows = flat.shape[0]
    rows_per = max(1, _CHUNK // max(1, flat.shape[1]))
    starts = list(range(0, rows, rows_per))

    def work(c):
        r0 = starts[c]
        r1 = min(rows, r0 + rows_per)
        flat[r0:r1] = fill(c, (r1 - r0, flat.shape[1]))

    if len(starts) == 1:
        work(0)
    else:
        with cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(work, range(len(starts))))
    return out


def normal(seed: int, tensor: int, shape, dtype: str) -> np.ndarray:
    """N(0, 1) draws of ``shape``, rounded to ``dtype``."""
    def fill(c, sh):
        x = _rng(seed, tensor, c).standard_normal(sh, dtype=np.float32)
        return round_bf16(x) if dtype == "bf16" else x
    return _chunked(shape, fill)


def rademacher(seed: int, tensor: int, shape) -> np.ndarray:
    def fill(c, sh):
        bits = _rng(seed, tensor, c).integers(0, 2, size=sh, dtype=np.int8)
        return bits.astype(np.float32) * 2.0 - 1.0
    return _chunked(shape, fill)


def _peaked_queries(K: np.ndarray, heads, H: int, seed: int, dtype: str,
                    noise: np.ndarray) -> np.ndarray:
    """q_t = 3.0 * mean of 4 keys drawn from [0, t] of the head's KV head + noise."""
    B, L, Hkv, d = K.shape
    G = H // Hkv
    rng = _rng(seed, _POS)
    out = {}
    t = np.arange(L)
    for h in heads:
        g = h // G
        u = rng.random((B, L, 4))
        pos = np.minimum((u * (t[None, :, None] + 1)).astype(np.int64), t[None, :, None])
        keys = K[np.arange(B)[:, None, None], pos, g]  # [B, L, 4, d]
        out[h] = 3.0 * keys.astype(np.float64).mean(axis=2) + noise[:, :, h].astype(np.float64)
    return out


def make_training(w: Workload, L: int | None = None) -> dict:
    """Q, K, V, dO for a training-shape workload (optionally with a different L)."""
    assert not w.decode
    L = w.L if L is None else L
    B, H, Hkv, d = w.B, w.H, w.H_kv, w.d
    K = normal(w.seed, _K, (B, L, Hkv, d), w.dtype)
    V = normal(w.seed, _V, (B, L, Hkv, d), w.dtype)
    dO = rademacher(w.seed, _DO, (B, L, H, d))
    if w.structure == "normal":
        Q = normal(w.seed, _Q, (B, L, H, d), w.dtype)
    elif w.structure in ("peaked", "half_peaked"):
        noise = normal(w.seed, _NOISE, (B, L, H, d), "fp32")
        heads = range(H) if w.structure == "peaked" else range(H // 2)
        Q = noise.copy()  # diffuse heads: Q ~ N(0, 1)
        for h, q in _peaked_queries(K, heads, H, w.seed, w.dtype, noise).items():
            Q[:, :, h] = q
        Q = _round(Q, w.dtype)
    elif w.structure == "sink_band":
        K = K.copy()
        K[:, 0] = _round(K[:, 0] * 4.0, w.dtype)
        n = normal(w.seed, _NOISE, (B, L, H, d), "fp32")
        cs = np.zeros((B, L + 1, Hkv, d), dtype=np.float64)
        np.cumsum(K, axis=1, dtype=np.float64, out=cs[:, 1:])
        t = np.arange(L)
        wlen = np.minimum(64, t)
        win = cs[:, t] - cs[:, t - wlen]  # sum of K_{t-w} .. K_{t-1}
        u = win / np.sqrt(np.maximum(wlen, 1))[None, :, None, None]
        G = H // Hkv
        Q = np.empty((B, L, H, d), dtype=np.float32)
        for h in range(H):
            Q[:, :, h] = 0.5 * u[:, :, h // G] + math.sqrt(0.75) * n[:, :, h]
        Q = _round(Q, w.dtype)
    elif w.structure == "prev_token_var":
        # previous-token heads of varying concentration: head h uses strength
        # s0_h = 8 + 12 u_h and noise b_h = 0.3 + 0.7 v_h (u, v uniform, drawn from the
        # seed), otherwise as "prev_token"; weak heads keep a heavier, less flat tail
        rng = _rng(w.seed, _PLANT)
        s0 = 8.0 + 12.0 * rng.random(H)
        bn = 0.3 + 0.7 * rng.random(H)
        n = normal(w.seed, _NOISE, (B, L, H, d), "fp32")
        G = H // Hkv
        kp = K[:, :-1].astype(np.float64)
        kp = kp * (math.sqrt(d) / np.maximum((kp * kp).sum(-1, keepdims=True), 1e-6))
        Q = np.empty((B, L, H, d), dtype=np.float32)
        for h in range(H):
            Q[:, :, h] = bn[h] * n[:, :, h]
            Q[:, 1:, h] += (s0[h] * kp[:, :, h // G]).astype(np.float32)
        Q = _round(Q, w.dtype)
    elif w.structure == "prev_token":
        # q_t = s0 sqrt(d) K_{t-1} / |K_{t-1}|^2 + b n_t: the scaled score of the previous
        # token is s0 (up to the noise) for every row, the other scores spread with a
        # standard deviation near s0 / |K| + b, so each head puts all but a small, flat tail
        # of its mass on the previous token (q_0 = b n_0)
        s0, b = 18.0, 0.3
        n = normal(w.seed, _NOISE, (B, L, H, d), "fp32")
        G = H // Hkv
        kp = K[:, :-1].astype(np.float64)
        kp = kp * (s0 * math.sqrt(d) / np.maximum((kp * kp).sum(-1, keepdims=True), 1e-6))
        Q = b * n
        for h in range(H):
            Q[:, 1:, h] += kp[:, :, h // G].astype(np.float32)
        Q = _round(Q, w.dtype)
    else:
        raise ValueError(w.structure)
    return {"Q": Q, "K": K, "V": V, "dO": dO}


def make_decode(w: Workload, Nk: int | None = None, B: int | None = None) -> dict:
    """q [B,H,d] and the KV cache K, V [B,Nk,Hkv,d] for a decode workload."""
    assert w.decode
    Nk = w.L if Nk is None else Nk
    B = w.B if B is None else B
    H, Hkv, d = w.H, w.H_kv, w.d
    G = H // Hkv
    q = normal(w.seed, _Q, (B, H, d), w.dtype)
    K = normal(w.seed, _K, (B, Nk, Hkv, d), w.dtype)
    V = normal(w.seed, _V, (B, Nk, Hkv, d), w.dtype)
    rng = _rng(w.seed, _PLANT)
    if w.structure == "planted":
        n_plant = min(16, Nk)
        for b in range(B):
            for g in range(Hkv):
                pos = rng.choice(Nk, size=n_plant, replace=False)
                for r, p in enumerate(pos):
                    h = g * G + (r % G)
                    qh = q[b, h].astype(np.float64)
                    key = 3.0 * math.sqrt(d) * qh / np.linalg.norm(qh) + rng.standard_normal(d)
                    K[b, p, g] = _round(key.astype(np.float32), w.dtype)
    elif w.structure == "heavy":
        # one heavy hitter shared by the group in every 8th key tile (key 64 of tiles
        # 7, 15, 23, ...): k = 28 u + 0.1 N(0, 1), u = the sum of the group's unit query
        # directions, so each head scores it near 28 (17..33 over heads: |q_h| ~ sqrt(d),
        # nearly orthogonal query directions) against ~N(0, 1) for the other keys
        for b in range(B):
            for g in range(Hkv):
                qg = q[b, g * G:(g + 1) * G].astype(np.float64)
                u = (qg / np.linalg.norm(qg, axis=-1, keepdims=True)).sum(axis=0)
                for p in range(7 * 128 + 64, Nk, 8 * 128):
                    key = 28.0 * u + 0.1 * rng.standard_normal(d)
                    K[b, p, g] = _round(key.astype(np.float32), w.dtype)
    else:
        raise ValueError(w.structure)
    return {"q": q, "K": K, "V": V}


def small_training(B=1, H=2, Hkv=1, L=192, d=64, dtype="bf16", structure="normal", seed=11):
    """A small ad-hoc training workload (parity tests: ragged tails, GQA, d=64)."""
    w = Workload(f"adhoc{L}", B, H, Hkv, L, d, dtype, structure, seed)
    return w, make_training(w)
