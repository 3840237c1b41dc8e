"""Thin ctypes binding of the MALA C ABI (``include/mala.h``).

Argument marshalling only: every step of forward, backward and decode runs in the
CUDA kernels of ``libmala_b200.so``.  PyTorch supplies device memory and the current
stream.  There is no fallback: if the library is missing the import of this module
fails loudly.
"""

from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

_LIB_PATH = _build.LIB

MALA_OK = 0
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape or dtype", 3: "CUDA error",
          4: "device wait timed out", 5: "workspace too small"}
MALA_BF16, MALA_FP32 = 0, 1
MALA_FLAG_ALWAYS_TEST = 1
TILE = 128

EXPORTED = ("mala_fwd", "mala_fwd_prefill", "mala_fwd_varlen", "mala_bwd", "mala_decode",
            "mala_decode_noalloc", "mala_get_stats", "mala_fwd_varlen_workspace_bytes",
            "mala_selftest_wait_timeout",
            "mala_fwd_workspace_bytes",
            "mala_bwd_workspace_bytes", "mala_decode_workspace_bytes", "mala_decode_num_splits",
            "mala_read_device_error", "mala_set_wait_budget_ns", "mala_set_debug",
            "mala_status_string", "mala_version")


class MalaStats(ctypes.Structure):
    _fields_ = [("legal_tiles", ctypes.c_uint64), ("retained_tiles", ctypes.c_uint64),
                ("v_tiles_loaded", ctypes.c_uint64)]


class MalaDebug(ctypes.Structure):
    _fields_ = [("tile_margin", ctypes.c_void_p), ("tile_margin_count", ctypes.c_size_t)]


class MalaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {STATUS.get(status, status)} (status {status})")
        self.status = status


def load_library(path: str = _LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"MALA CUDA library not built: {path} (run python -m "
                          "mass_adaptive_sparse_fwd_b200.build)")
    lib = ctypes.CDLL(path)
    vp, ci, cf, cu, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_uint,
                          ctypes.c_size_t)
    lib.mala_fwd.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, cf, cu, vp, sz, vp, vp]
    lib.mala_fwd_prefill.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, ci, cf, cf, cu,
                                     vp, sz, vp, vp]
    ip = ctypes.POINTER(ctypes.c_int)
    lib.mala_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, ip, ip, ci, ci, ci, ci, ci, cf, cf, cu,
                                    vp, sz, vp]
    lib.mala_fwd_varlen_workspace_bytes.argtypes = [ip, ci, ci, ci, ci, ci]
    lib.mala_fwd_varlen_workspace_bytes.restype = sz
    lib.mala_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, cf,
                             cu, vp, sz, vp, vp]
    lib.mala_decode.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, cf, ci, cu, vp, sz,
                                vp, vp]
    lib.mala_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cf, cf, ci, cu,
                                        vp, vp]
    lib.mala_decode_noalloc.restype = ci
    for f in ("mala_fwd", "mala_fwd_prefill", "mala_fwd_varlen", "mala_bwd", "mala_decode",
              "mala_read_device_error",
              "mala_set_wait_budget_ns"):
        getattr(lib, f).restype = ci
    lib.mala_fwd_workspace_bytes.argtypes = [ci] * 6
    lib.mala_bwd_workspace_bytes.argtypes = [ci] * 6
    lib.mala_decode_workspace_bytes.argtypes = [ci] * 7
    for f in ("mala_fwd_workspace_bytes", "mala_bwd_workspace_bytes",
              "mala_decode_workspace_bytes"):
        getattr(lib, f).restype = sz
    lib.mala_decode_num_splits.argtypes = [ci] * 4
    lib.mala_decode_num_splits.restype = ci
    lib.mala_read_device_error.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_uint32), ci]
    lib.mala_set_wait_budget_ns.argtypes = [ctypes.c_uint64]
    lib.mala_selftest_wait_timeout.argtypes = [vp, ctypes.c_uint64, vp]
    lib.mala_selftest_wait_timeout.restype = ci
    lib.mala_get_stats.argtypes = [vp, vp, ctypes.POINTER(MalaStats)]
    lib.mala_get_stats.restype = ci
    lib.mala_set_debug.argtypes = [ctypes.POINTER(MalaDebug)]
    lib.mala_set_debug.restype = ci
    lib.mala_status_string.argtypes = [ci]
    lib.mala_status_string.restype = ctypes.c_char_p
    lib.mala_version.restype = ci
    return lib


_lib = load_library()


def lib() -> ctypes.CDLL:
    return _lib


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MALA_BF16
    if t.dtype == torch.float32:
        return MALA_FP32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(fn: str, status: int):
    if status != MALA_OK:
        raise MalaError(fn, status)


# The C ABI receives bare pointers and sizes, so a tensor whose shape, dtype or layout
# disagrees with the sizes passed next to it would send the kernels past its allocation.
# Every entry point below checks its tensors against the layouts of include/mala.h first
# (shape, dtype, contiguity, one device), and only then requires that device to be CUDA.


def _need(fn, name, t, shape, dtype, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{fn}: {name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{fn}: {name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{fn}: {name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{fn}: {name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{fn}: {name} is on {t.device}, the call's tensors on {device}")


def _need_buffer(fn, name, t, min_numel, dtype, device):
    """An optional flat buffer (tile mask): at least min_numel elements of dtype."""
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or t.dtype != dtype:
        raise TypeError(f"{fn}: {name} must be a {dtype} tensor")
    if t.numel() < min_numel:
        raise ValueError(f"{fn}: {name} holds {t.numel()} elements, needs {min_numel}")
    if not t.is_contiguous() or t.device != device:
        raise ValueError(f"{fn}: {name} must be contiguous and on {device}")


def _workspace_bytes(fn, workspace, device) -> int:
    if workspace is None:
        return 0
    if not isinstance(workspace, torch.Tensor) or not workspace.is_contiguous() or \
            workspace.device != device:
        raise ValueError(f"{fn}: workspace must be a contiguous tensor on {device}")
    return workspace.numel() * workspace.element_size()


def _need_cuda(fn, device):
    if device.type != "cuda":
        raise ValueError(f"{fn}: tensors must be on a CUDA device, got {device}")


def _qkv_dtype(fn, Q) -> torch.dtype:
    if not isinstance(Q, torch.Tensor):
        raise TypeError(f"{fn}: Q must be a torch.Tensor")
    _dtype_code(Q)  # bf16 or fp32
    return Q.dtype


def n_tiles(n: int) -> int:
    return (n + TILE - 1) // TILE


def fwd_workspace_bytes(B, H, H_kv, L, d, dtype=MALA_BF16) -> int:
    return _lib.mala_fwd_workspace_bytes(B, H, H_kv, L, d, dtype)


def bwd_workspace_bytes(B, H, H_kv, L, d, dtype=MALA_BF16) -> int:
    return _lib.mala_bwd_workspace_bytes(B, H, H_kv, L, d, dtype)


def decode_workspace_bytes(B, H, H_kv, Nk, d, dtype=MALA_BF16, num_splits=0) -> int:
    return _lib.mala_decode_workspace_bytes(B, H, H_kv, Nk, d, dtype, num_splits)


def decode_num_splits(B, H, H_kv, Nk) -> int:
    return _lib.mala_decode_num_splits(B, H, H_kv, Nk)


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    """A zeroed workspace buffer (uint8) suitable for any MALA call of that size."""
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)


def mala_fwd(Q, K, V, scale, tau, O=None, LSE=None, flags=0, workspace=None, tile_mask=None,
             stream=None):
    """MALA forward through the C ABI.  Q [B,L,H,d], K/V [B,L,H_kv,d] (bf16 or fp32,
    contiguous, on the GPU).  Returns (O, LSE)."""
    fn, dt = "mala_fwd", _qkv_dtype("mala_fwd", Q)
    B, L, H, d = Q.shape
    H_kv = K.shape[2] if isinstance(K, torch.Tensor) and K.dim() == 4 else -1
    dev = Q.device
    _need(fn, "Q", Q, (B, L, H, d), dt, dev)
    _need(fn, "K", K, (B, L, H_kv, d), dt, dev)
    _need(fn, "V", V, (B, L, H_kv, d), dt, dev)
    if O is None:
        O = torch.empty_like(Q)
    if LSE is None:
        LSE = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    _need(fn, "O", O, (B, L, H, d), dt, dev)
    _need(fn, "LSE", LSE, (B, H, L), torch.float32, dev)
    _need_buffer(fn, "tile_mask", tile_mask, B * H * n_tiles(L) ** 2, torch.uint8, dev)
    ws_bytes = _workspace_bytes(fn, workspace, dev)
    _need_cuda(fn, dev)
    st = _lib.mala_fwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, H, H_kv, L, d,
                       _dtype_code(Q), float(scale), float(tau), flags, _ptr(workspace), ws_bytes,
                       _ptr(tile_mask), _stream(stream))
    _check("mala_fwd", st)
    return O, LSE


def mala_fwd_prefill(Q, K, V, scale, tau, O=None, LSE=None, flags=0, workspace=None,
                     tile_mask=None, stream=None):
    """Forward of a prefill chunk through the C ABI: Q [B,N_q,H,d] are the last N_q
    positions of the sequence whose keys K/V [B,N_k,H_kv,d] (N_k >= N_q) include them.
    Returns (O [B,N_q,H,d], LSE [B,H,N_q])."""
    fn, dt = "mala_fwd_prefill", _qkv_dtype("mala_fwd_prefill", Q)
    B, Nq, H, d = Q.shape
    Nk, H_kv = (K.shape[1], K.shape[2]) if isinstance(K, torch.Tensor) and K.dim() == 4 \
        else (-1, -1)
    dev = Q.device
    _need(fn, "K", K, (B, Nk, H_kv, d), dt, dev)
    _need(fn, "V", V, (B, Nk, H_kv, d), dt, dev)
    _need(fn, "Q", Q, (B, Nq, H, d), dt, dev)
    if O is None:
        O = torch.empty_like(Q)
    if LSE is None:
        LSE = torch.empty((B, H, Nq), dtype=torch.float32, device=dev)
    _need(fn, "O", O, (B, Nq, H, d), dt, dev)
    _need(fn, "LSE", LSE, (B, H, Nq), torch.float32, dev)
    _need_buffer(fn, "tile_mask", tile_mask, B * H * n_tiles(Nq) * n_tiles(Nk), torch.uint8,
                 dev)
    ws_bytes = _workspace_bytes(fn, workspace, dev)
    _need_cuda(fn, dev)
    st = _lib.mala_fwd_prefill(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), B, H, H_kv, Nq, Nk,
                               d, _dtype_code(Q), float(scale), float(tau), flags,
                               _ptr(workspace), ws_bytes, _ptr(tile_mask), _stream(stream))
    _check("mala_fwd_prefill", st)
    return O, LSE


def _int_array(xs):
    xs = [int(x) for x in xs]
    return (ctypes.c_int * len(xs))(*xs)


def varlen_workspace_bytes(cu_seqlens_q, H, H_kv, d, dtype=MALA_BF16) -> int:
    return _lib.mala_fwd_varlen_workspace_bytes(_int_array(cu_seqlens_q), len(cu_seqlens_q) - 1,
                                                H, H_kv, d, dtype)


def mala_fwd_varlen(Q, K, V, cu_seqlens_q, cu_seqlens_k, scale, tau, O=None, LSE=None, flags=0,
                    workspace=None, stream=None):
    """Forward of a packed batch through the C ABI: Q [total_q,H,d], K/V [total_k,H_kv,d];
    cu_seqlens_* are host sequences of n+1 offsets.  Returns (O [total_q,H,d],
    LSE [H,total_q])."""
    fn, dt = "mala_fwd_varlen", _qkv_dtype("mala_fwd_varlen", Q)
    total_q, H, d = Q.shape
    H_kv = K.shape[1] if isinstance(K, torch.Tensor) and K.dim() == 3 else -1
    n = len(cu_seqlens_q) - 1
    if n < 1 or len(cu_seqlens_k) != n + 1:
        raise ValueError(f"{fn}: cu_seqlens_q / cu_seqlens_k need the same n + 1 >= 2 offsets")
    total_k = int(cu_seqlens_k[-1])
    if int(cu_seqlens_q[-1]) != total_q:
        raise ValueError(f"{fn}: cu_seqlens_q ends at {int(cu_seqlens_q[-1])}, Q has "
                         f"{total_q} rows")
    dev = Q.device
    _need(fn, "Q", Q, (total_q, H, d), dt, dev)
    _need(fn, "K", K, (total_k, H_kv, d), dt, dev)
    _need(fn, "V", V, (total_k, H_kv, d), dt, dev)
    if O is None:
        O = torch.empty_like(Q)
    if LSE is None:
        LSE = torch.empty((H, total_q), dtype=torch.float32, device=dev)
    _need(fn, "O", O, (total_q, H, d), dt, dev)
    _need(fn, "LSE", LSE, (H, total_q), torch.float32, dev)
    if workspace is None:
        _need_cuda(fn, dev)
        workspace = alloc_workspace(varlen_workspace_bytes(cu_seqlens_q, H, H_kv, d), dev)
    ws_bytes = _workspace_bytes(fn, workspace, dev)
    _need_cuda(fn, dev)
    st = _lib.mala_fwd_varlen(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE),
                              _int_array(cu_seqlens_q), _int_array(cu_seqlens_k), n, H, H_kv, d,
                              _dtype_code(Q), float(scale), float(tau), flags, _ptr(workspace),
                              ws_bytes, _stream(stream))
    _check("mala_fwd_varlen", st)
    return O, LSE


def mala_bwd(Q, K, V, O, LSE, dO, scale, tau, dQ=None, dK=None, dV=None, flags=0,
             workspace=None, tile_mask=None, stream=None):
    """MALA backward through the C ABI.  Returns (dQ, dK, dV)."""
    fn, dt = "mala_bwd", _qkv_dtype("mala_bwd", Q)
    B, L, H, d = Q.shape
    H_kv = K.shape[2] if isinstance(K, torch.Tensor) and K.dim() == 4 else -1
    dev = Q.device
    _need(fn, "Q", Q, (B, L, H, d), dt, dev)
    _need(fn, "K", K, (B, L, H_kv, d), dt, dev)
    _need(fn, "V", V, (B, L, H_kv, d), dt, dev)
    _need(fn, "O", O, (B, L, H, d), dt, dev)
    _need(fn, "LSE", LSE, (B, H, L), torch.float32, dev)
    _need(fn, "dO", dO, (B, L, H, d), dt, dev)
    dQ = torch.empty_like(Q) if dQ is None else dQ
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(V) if dV is None else dV
    _need(fn, "dQ", dQ, (B, L, H, d), dt, dev)
    _need(fn, "dK", dK, (B, L, H_kv, d), dt, dev)
    _need(fn, "dV", dV, (B, L, H_kv, d), dt, dev)
    _need_buffer(fn, "tile_mask", tile_mask, B * H * n_tiles(L) ** 2, torch.uint8, dev)
    ws_bytes = _workspace_bytes(fn, workspace, dev)
    _need_cuda(fn, dev)
    st = _lib.mala_bwd(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(LSE), _ptr(dO), _ptr(dQ), _ptr(dK),
                       _ptr(dV), B, H, H_kv, L, d, _dtype_code(Q), float(scale), float(tau), flags,
                       _ptr(workspace), ws_bytes, _ptr(tile_mask), _stream(stream))
    _check("mala_bwd", st)
    return dQ, dK, dV


def _decode_checks(fn, q, Kc, Vc, O, LSE, tile_mask):
    dt = _qkv_dtype(fn, q)
    B, H, d = q.shape
    Nk, H_kv = (Kc.shape[1], Kc.shape[2]) if isinstance(Kc, torch.Tensor) and Kc.dim() == 4 \
        else (-1, -1)
    dev = q.device
    _need(fn, "q", q, (B, H, d), dt, dev)
    _need(fn, "Kc", Kc, (B, Nk, H_kv, d), dt, dev)
    _need(fn, "Vc", Vc, (B, Nk, H_kv, d), dt, dev)
    if O is not None:
        _need(fn, "O", O, (B, H, d), dt, dev)
    if LSE is not None:
        _need(fn, "LSE", LSE, (B, H), torch.float32, dev)
    _need_buffer(fn, "tile_mask", tile_mask, B * H * n_tiles(Nk), torch.uint8, dev)
    return B, H, d, Nk, H_kv


def mala_decode(q, Kc, Vc, scale, tau, num_splits=0, O=None, LSE=None, flags=0, workspace=None,
                tile_mask=None, stream=None):
    """MALA split-KV decode through the C ABI.  q [B,H,d]; Kc/Vc [B,N_k,H_kv,d].
    Returns (O [B,H,d], LSE [B,H])."""
    fn = "mala_decode"
    B, H, d, Nk, H_kv = _decode_checks(fn, q, Kc, Vc, O, LSE, tile_mask)
    O = torch.empty_like(q) if O is None else O
    LSE = torch.empty((B, H), dtype=torch.float32, device=q.device) if LSE is None else LSE
    ws_bytes = _workspace_bytes(fn, workspace, q.device)
    _need_cuda(fn, q.device)
    st = _lib.mala_decode(_ptr(q), _ptr(Kc), _ptr(Vc), _ptr(O), _ptr(LSE), B, H, H_kv, Nk, d,
                          _dtype_code(q), float(scale), float(tau), int(num_splits), flags,
                          _ptr(workspace), ws_bytes, _ptr(tile_mask), _stream(stream))
    _check("mala_decode", st)
    return O, LSE


def mala_decode_noalloc(q, Kc, Vc, scale, tau, num_splits=0, O=None, LSE=None, flags=0,
                        tile_mask=None, stream=None):
    """Split-KV decode that allocates nothing on the device: its scratch is a fixed
    array inside the library (for callers that may not allocate device memory on their
    hot path).  Calls on one device share that array, so they must not overlap on the
    GPU.  Returns (O [B,H,d], LSE [B,H])."""
    fn = "mala_decode_noalloc"
    B, H, d, Nk, H_kv = _decode_checks(fn, q, Kc, Vc, O, LSE, tile_mask)
    O = torch.empty_like(q) if O is None else O
    LSE = torch.empty((B, H), dtype=torch.float32, device=q.device) if LSE is None else LSE
    _need_cuda(fn, q.device)
    st = _lib.mala_decode_noalloc(_ptr(q), _ptr(Kc), _ptr(Vc), _ptr(O), _ptr(LSE), B, H, H_kv,
                                  Nk, d, _dtype_code(q), float(scale), float(tau),
                                  int(num_splits), flags, _ptr(tile_mask), _stream(stream))
    _check("mala_decode_noalloc", st)
    return O, LSE


def read_device_error(workspace: torch.Tensor, clear: bool = True, stream=None) -> int:
    out = ctypes.c_uint32(0)
    _check("mala_read_device_error",
           _lib.mala_read_device_error(_ptr(workspace), _stream(stream), ctypes.byref(out),
                                       int(clear)))
    return out.value


def get_stats(workspace: torch.Tensor, stream=None) -> dict:
    """Work counters of the last call that ran on `workspace` (synchronises the stream):
    legal tiles tested, retained tiles and, for decode, V tiles loaded."""
    out = MalaStats()
    _check("mala_get_stats", _lib.mala_get_stats(_ptr(workspace), _stream(stream),
                                                 ctypes.byref(out)))
    return {"legal_tiles": out.legal_tiles, "retained_tiles": out.retained_tiles,
            "v_tiles_loaded": out.v_tiles_loaded}


def selftest_wait_timeout(workspace: torch.Tensor, budget_ns: int, stream=None):
    """Runs the bounded-wait self-test kernel (a wait that nothing satisfies)."""
    _check("mala_selftest_wait_timeout",
           _lib.mala_selftest_wait_timeout(_ptr(workspace), int(budget_ns), _stream(stream)))


def set_wait_budget_ns(ns: int):
    _check("mala_set_wait_budget_ns", _lib.mala_set_wait_budget_ns(int(ns)))


def set_debug(tile_margin=None):
    """Registers (or, with None, clears) a float32 CUDA buffer that receives the margin of
    every retention test of this thread's later forward, prefill, backward and decode
    calls, in the layout of their tile masks (see ``mala_set_debug`` in the header)."""
    if tile_margin is None:
        _check("mala_set_debug", _lib.mala_set_debug(None))
        return
    if not isinstance(tile_margin, torch.Tensor) or tile_margin.dtype != torch.float32 or \
            not tile_margin.is_contiguous():
        raise TypeError("set_debug: tile_margin must be a contiguous float32 tensor")
    _need_cuda("set_debug", tile_margin.device)
    dbg = MalaDebug(tile_margin.data_ptr(), tile_margin.numel())
    _check("mala_set_debug", _lib.mala_set_debug(ctypes.byref(dbg)))


class debug_margins:
    """Context manager: ``with debug_margins(buf): mala_fwd(...)`` fills ``buf`` with the
    call's tile margins and turns the hook off on exit."""

    def __init__(self, tile_margin):
        self.buf = tile_margin

    def __enter__(self):
        set_debug(self.buf)
        return self.buf

    def __exit__(self, *exc):
        set_debug(None)
        return False
