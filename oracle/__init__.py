"""ctypes front end of the MALA fp64 CPU oracle (``mala_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py``.  The product path never imports it.

The C++ file restates MassAlloc Attention ("MassAlloc Attention: Let Attention
Allocate Its Own Compute", §2.1-§2.4, App. A Algorithms 1-2, App. B) in plain fp64
loops.  Inputs are float32 numpy arrays holding the exact values the GPU sees
(bf16-rounded for bf16 runs); outputs are float64.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading
import time

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mala_oracle.cpp")
_LIB = os.path.join(_HERE, "libmala_oracle.so")
_lock = threading.Lock()
_lib = None

# Wall-clock and process CPU seconds of the last oracle call, measured around the C call
# alone (the Python-side array set-up is excluded); the bench's CPU baseline uses them.
LAST_CALL = {"wall": 0.0, "cpu": 0.0}


class _Timed:
    def __enter__(self):
        self.w, self.c = time.perf_counter(), time.process_time()

    def __exit__(self, *exc):
        LAST_CALL["wall"] = time.perf_counter() - self.w
        LAST_CALL["cpu"] = time.process_time() - self.c
        return False

_f32p = np.ctypeslib.ndpointer(dtype=np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libmala_oracle.so`` (g++ -O2 -fopenmp)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c++17",
                               "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            vp = ctypes.c_void_p
            ci, cd = ctypes.c_int, ctypes.c_double
            lib.orc_dense_fwd.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, cd, ci, vp, ci, vp, vp]
            lib.orc_dense_bwd.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, cd, vp, vp, vp]
            lib.orc_mala_fwd.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, cd, cd, ci, vp, ci, vp,
                                         vp, vp, vp, vp]
            lib.orc_mala_fwd_setsum.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, cd, cd, ci, vp, vp,
                                                vp, vp]
            lib.orc_mala_bwd.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, cd, cd, ci,
                                         vp, ci, vp, ci, vp, vp, vp, vp, vp, vp]
            lib.orc_mala_decode.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, cd, cd, ci, ci, vp,
                                            ci, vp, vp, vp, vp, vp, vp, vp]
            lib.orc_mala_prefill.argtypes = [vp, vp, vp, ci, ci, ci, ci, ci, ci, cd, cd, ci, vp,
                                             ci, vp, vp, vp, vp, vp]
            lib.orc_num_threads.restype = ctypes.c_int
            for name in ("orc_dense_fwd", "orc_dense_bwd", "orc_mala_fwd", "orc_mala_fwd_setsum",
                         "orc_mala_bwd", "orc_mala_decode", "orc_mala_prefill"):
                getattr(lib, name).restype = ctypes.c_int
            _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def _f32(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a


def _units(u, width):
    if u is None:
        return None, 0
    u = np.ascontiguousarray(np.asarray(u, dtype=np.int32).reshape(-1, width))
    return u, u.shape[0]


def _check(rc, name):
    if rc != 0:
        raise ValueError(f"{name}: invalid arguments (code {rc})")


def n_tiles(L: int, blk: int) -> int:
    return (L + blk - 1) // blk


def dense_fwd(Q, K, V, scale, blk=128, units=None):
    """FullAttn forward.  Returns (O [B,L,H,d] f64, LSE [B,H,L] f64); rows outside
    ``units`` ((b, h, i) blocks of ``blk`` rows) are left as NaN."""
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    B, L, H, d = Q.shape
    Hkv = K.shape[2]
    O = np.full(Q.shape, np.nan)
    LSE = np.full((B, H, L), np.nan)
    u, n = _units(units, 3)
    rc = _load().orc_dense_fwd(_p(Q), _p(K), _p(V), B, H, Hkv, L, d, float(scale), blk, _p(u), n,
                               _p(O), _p(LSE))
    _check(rc, "dense_fwd")
    return O, LSE


def dense_bwd(Q, K, V, dO, scale):
    """Exact FullAttn gradients (dQ, dK, dV) in f64."""
    Q, K, V, dO = _f32(Q), _f32(K), _f32(V), _f32(dO)
    B, L, H, d = Q.shape
    Hkv = K.shape[2]
    dQ = np.zeros(Q.shape)
    dK = np.zeros(K.shape)
    dV = np.zeros(V.shape)
    rc = _load().orc_dense_bwd(_p(Q), _p(K), _p(V), _p(dO), B, H, Hkv, L, d, float(scale),
                               _p(dQ), _p(dK), _p(dV))
    _check(rc, "dense_bwd")
    return dQ, dK, dV


def mala_fwd(Q, K, V, scale, tau, blk=128, units=None, force=None):
    """MALA forward (online form).  Returns (O, LSE, mask, margin); mask / margin are
    [B,H,T,T] with -1 / NaN where a tile is illegal or not evaluated."""
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    B, L, H, d = Q.shape
    Hkv = K.shape[2]
    T = n_tiles(L, blk)
    O = np.full(Q.shape, np.nan)
    LSE = np.full((B, H, L), np.nan)
    mask = np.full((B, H, T, T), -1, dtype=np.int8)
    margin = np.full((B, H, T, T), np.nan)
    u, n = _units(units, 3)
    if force is not None:
        force = np.ascontiguousarray(force, dtype=np.int8)
        assert force.shape == (B, H, T, T)
    with _Timed():
        rc = _load().orc_mala_fwd(_p(Q), _p(K), _p(V), B, H, Hkv, L, d, float(scale), float(tau), blk,
                                  _p(u), n, _p(force), _p(O), _p(LSE), _p(mask), _p(margin))
    _check(rc, "mala_fwd")
    return O, LSE, mask, margin


def mala_prefill(Q, K, V, scale, tau, blk=128, units=None, force=None):
    """Chunked-prefill forward: Q [B,Nq,H,d] are the last Nq positions of a sequence whose
    keys K, V [B,Nk,Hkv,d] (Nk >= Nq) include them; row q sits at position Nk - Nq + q.
    Returns (O, LSE, mask, margin) with mask / margin [B,H,Tq,Tk]."""
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    B, Nq, H, d = Q.shape
    Nk, Hkv = K.shape[1], K.shape[2]
    Tq, Tk = n_tiles(Nq, blk), n_tiles(Nk, blk)
    O = np.full(Q.shape, np.nan)
    LSE = np.full((B, H, Nq), np.nan)
    mask = np.full((B, H, Tq, Tk), -1, dtype=np.int8)
    margin = np.full((B, H, Tq, Tk), np.nan)
    u, n = _units(units, 3)
    if force is not None:
        force = np.ascontiguousarray(force, dtype=np.int8)
        assert force.shape == (B, H, Tq, Tk)
    with _Timed():
        rc = _load().orc_mala_prefill(_p(Q), _p(K), _p(V), B, H, Hkv, Nq, Nk, d, float(scale),
                                      float(tau), blk, _p(u), n, _p(force), _p(O), _p(LSE), _p(mask),
                                      _p(margin))
    _check(rc, "mala_prefill")
    return O, LSE, mask, margin


def mala_fwd_setsum(Q, K, V, scale, tau, blk=128):
    """MALA forward, explicit retained-set formulation (cross-check of ``mala_fwd``)."""
    Q, K, V = _f32(Q), _f32(K), _f32(V)
    B, L, H, d = Q.shape
    Hkv = K.shape[2]
    T = n_tiles(L, blk)
    O = np.full(Q.shape, np.nan)
    LSE = np.full((B, H, L), np.nan)
    mask = np.full((B, H, T, T), -1, dtype=np.int8)
    margin = np.full((B, H, T, T), np.nan)
    rc = _load().orc_mala_fwd_setsum(_p(Q), _p(K), _p(V), B, H, Hkv, L, d, float(scale),
                                     float(tau), blk, _p(O), _p(LSE), _p(mask), _p(margin))
    _check(rc, "mala_fwd_setsum")
    return O, LSE, mask, margin


def mala_bwd(Q, K, V, O, LSE, dO, scale, tau, blk=128, kv_units=None, q_units=None, force=None):
    """MALA backward.  ``O`` / ``LSE`` are the forward's outputs (any source).  Returns
    (dQ, dK, dV, mask, margin); rows outside the requested units are NaN."""
    Q, K, V, dO = _f32(Q), _f32(K), _f32(V), _f32(dO)
    O = np.ascontiguousarray(O, dtype=np.float64)
    LSE = np.ascontiguousarray(LSE, dtype=np.float64)
    B, L, H, d = Q.shape
    Hkv = K.shape[2]
    T = n_tiles(L, blk)
    dQ = np.full(Q.shape, np.nan)
    dK = np.full(K.shape, np.nan)
    dV = np.full(V.shape, np.nan)
    mask = np.full((B, H, T, T), -1, dtype=np.int8)
    margin = np.full((B, H, T, T), np.nan)
    ku, nk = _units(kv_units, 3)
    qu, nq = _units(q_units, 3)
    if force is not None:
        force = np.ascontiguousarray(force, dtype=np.int8)
        assert force.shape == (B, H, T, T)
    with _Timed():
        rc = _load().orc_mala_bwd(_p(Q), _p(K), _p(V), _p(O), _p(LSE), _p(dO), B, H, Hkv, L, d,
                                  float(scale), float(tau), blk, _p(ku), nk, _p(qu), nq, _p(force),
                                  _p(dQ), _p(dK), _p(dV), _p(mask), _p(margin))
    _check(rc, "mala_bwd")
    return dQ, dK, dV, mask, margin


def decode_split_bounds(n_tiles_total: int, num_splits: int):
    """Tile ranges [lo, hi) of each split: split s owns [s*T//S, (s+1)*T//S)."""
    T, S = n_tiles_total, num_splits
    return [((s * T) // S, ((s + 1) * T) // S) for s in range(S)]


def mala_decode(q, K, V, scale, tau, num_splits, blk=128, units=None, force=None):
    """MALA split-KV decode.  q [B,H,d]; K, V [B,Nk,Hkv,d].  Returns
    (O [B,H,d], LSE [B,H], mask [B,H,T], margin [B,H,T], part_o [B,H,S,d], part_z [B,H,S])."""
    q, K, V = _f32(q), _f32(K), _f32(V)
    B, H, d = q.shape
    Nk, Hkv = K.shape[1], K.shape[2]
    T = n_tiles(Nk, blk)
    S = int(num_splits)
    O = np.full((B, H, d), np.nan)
    LSE = np.full((B, H), np.nan)
    mask = np.full((B, H, T), -1, dtype=np.int8)
    margin = np.full((B, H, T), np.nan)
    part_o = np.full((B, H, S, d), np.nan)
    part_z = np.full((B, H, S), np.nan)
    u, n = _units(units, 2)
    if force is not None:
        force = np.ascontiguousarray(force, dtype=np.int8)
        assert force.shape == (B, H, T)
    with _Timed():
        rc = _load().orc_mala_decode(_p(q), _p(K), _p(V), B, H, Hkv, Nk, d, float(scale), float(tau),
                                     blk, S, _p(u), n, _p(force), _p(O), _p(LSE), _p(mask),
                                     _p(margin), _p(part_o), _p(part_z))
    _check(rc, "mala_decode")
    return O, LSE, mask, margin, part_o, part_z


def num_threads() -> int:
    """Threads the oracle's parallel loops use (OpenMP), i.e. the cores it occupies."""
    return int(_load().orc_num_threads())
