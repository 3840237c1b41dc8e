"""Host-side checks that need no GPU: the C ABI exports, argument validation (which
returns before any CUDA call), workspace-size queries, the bench's accounting helpers and
its multi-rank plumbing (world size 2 over gloo)."""

import ctypes
import os
import re
import subprocess
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            names += re.findall(r"^\s*(?:[\w\*]+\s+)+\**(mala_\w+)\s*\(", src, re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from mass_adaptive_sparse_fwd_b200 import build

    build.build_library()
    from mass_adaptive_sparse_fwd_b200 import mala

    return mala


def test_header_declares_the_three_operators():
    names = _declared_functions()
    for n in ("mala_fwd", "mala_bwd", "mala_decode"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    so = ctypes.CDLL(lib._LIB_PATH)
    for n in _declared_functions():
        assert hasattr(so, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", lib._LIB_PATH], capture_output=True,
                         text=True).stdout
    for n in _declared_functions():
        assert re.search(rf"\bT {n}\b", out), n


def test_version_and_status_strings(lib):
    L = lib.lib()
    assert L.mala_version() == 203
    assert L.mala_status_string(0) == b"ok"
    assert L.mala_status_string(4) == b"device wait timed out"


def test_invalid_arguments_are_rejected_before_any_launch(lib):
    L = lib.lib()
    p = ctypes.c_void_p(16 * 1024)  # never dereferenced: validation fails first
    vp = lambda: p
    # H not a multiple of H_kv
    assert L.mala_fwd(vp(), vp(), vp(), vp(), vp(), 1, 6, 4, 128, 128, 0, 0.1, 1.0, 0, None, 0,
                      None, None) == 1
    # negative tau, non-finite scale, zero length
    assert L.mala_fwd(vp(), vp(), vp(), vp(), vp(), 1, 4, 2, 128, 128, 0, 0.1, -1.0, 0, None, 0,
                      None, None) == 1
    assert L.mala_fwd(vp(), vp(), vp(), vp(), vp(), 1, 4, 2, 128, 128, 0, float("nan"), 1.0, 0,
                      None, 0, None, None) == 1
    assert L.mala_fwd(vp(), vp(), vp(), vp(), vp(), 1, 4, 2, 0, 128, 0, 0.1, 1.0, 0, None, 0,
                      None, None) == 1
    # null pointers and misaligned pointers
    assert L.mala_fwd(None, vp(), vp(), vp(), vp(), 1, 4, 2, 128, 128, 0, 0.1, 1.0, 0, None, 0,
                      None, None) == 1
    assert L.mala_fwd(ctypes.c_void_p(16 * 1024 + 2), vp(), vp(), vp(), vp(), 1, 4, 2, 128, 128,
                      0, 0.1, 1.0, 0, None, 0, None, None) == 1
    # unsupported head dim for the bf16 tensor-core path
    assert L.mala_fwd(vp(), vp(), vp(), vp(), vp(), 1, 4, 2, 128, 96, 0, 0.1, 1.0, 0, None, 0,
                      None, None) == 2
    # decode: split count out of range
    assert L.mala_decode(vp(), vp(), vp(), vp(), vp(), 1, 4, 2, 256, 128, 0, 0.1, 1.0, 3, 0,
                         None, 0, None, None) == 1
    # backward: bad dtype code
    assert L.mala_bwd(vp(), vp(), vp(), vp(), vp(), vp(), vp(), vp(), vp(), 1, 4, 2, 128, 128, 7,
                      0.1, 1.0, 0, None, 0, None, None) == 1
    # decode: a group of more than 8 query heads per KV head on the bf16 path
    assert L.mala_decode(vp(), vp(), vp(), vp(), vp(), 1, 18, 2, 256, 128, 0, 0.1, 1.0, 1, 0,
                         vp(), 1 << 20, None, None) == 2
    # prefill: more queries than keys
    assert L.mala_fwd_prefill(vp(), vp(), vp(), vp(), vp(), 1, 4, 2, 300, 200, 128, 0, 0.1, 1.0,
                              0, None, 0, None, None) == 1
    # statistics need a workspace and an output
    assert L.mala_get_stats(None, None, None) == 1
    # packed batches: offsets must start at 0 and every sequence needs N_k >= N_q
    ia = lambda xs: (ctypes.c_int * len(xs))(*xs)
    args = (1, 4, 2, 128, 0, 0.1, 1.0, 0, vp(), 1 << 20, None)
    assert L.mala_fwd_varlen(vp(), vp(), vp(), vp(), vp(), ia([5, 10]), ia([0, 10]), *args) == 1
    assert L.mala_fwd_varlen(vp(), vp(), vp(), vp(), vp(), ia([0, 10]), ia([0, 5]), *args) == 1
    assert L.mala_fwd_varlen_workspace_bytes(ia([0, 300, 300, 557]), 3, 4, 2, 128, 0) == \
        256 + (3 + 0 + 3) * 32
    # a batch with no query rows is done after the host checks (no CUDA call)
    assert L.mala_fwd_varlen(vp(), vp(), vp(), vp(), vp(), ia([0, 0, 0]), ia([0, 5, 7]), 2,
                             *args[1:]) == 0
    # workspace too small (checked before any CUDA call)
    assert L.mala_fwd(vp(), vp(), vp(), vp(), vp(), 1, 4, 2, 128, 128, 0, 0.1, 1.0, 0, vp(), 8,
                      None, None) == 5


def test_workspace_sizes_and_split_rule(lib):
    B, H, Hkv, L, d = 1, 32, 8, 32768, 128
    assert lib.fwd_workspace_bytes(B, H, Hkv, L, d) == 256
    assert lib.bwd_workspace_bytes(B, H, Hkv, L, d) >= 256 + B * L * H * d * 4 + B * H * L * 4
    S = lib.decode_num_splits(4, 32, 8, 131072)
    assert 1 <= S <= 1024
    assert lib.decode_num_splits(4, 32, 8, 131072) == S  # deterministic
    assert lib.decode_workspace_bytes(4, 32, 8, 131072, 128, 0, S) >= 256 + 4 * 32 * S * 129 * 4
    assert lib.decode_num_splits(1, 4, 1, 100) == 1
    assert lib.decode_workspace_bytes(1, 4, 2, 256, 128, 0, 5) == 0  # 5 splits > 2 tiles


def _round256(n):
    return (n + 255) // 256 * 256


def test_bwd_workspace_head_parts(lib):
    """The backward splits a unit's query heads into parts when a problem has few units
    (few KV heads, short sequences); the parts add dK / dV into two fp32 accumulators that
    the workspace then holds.  Many units (the 32K 32/8-head shape, the 128K 8/1-head
    shape): no split, no accumulators."""
    def base(B, H, Hkv, L, d):
        return 256 + _round256(B * L * H * d * 4) + _round256(B * H * L * 4)

    def kv(B, Hkv, L, d):
        return 2 * _round256(B * L * Hkv * d * 4)

    for shape in [(1, 32, 8, 32768, 128), (1, 8, 1, 131072, 128), (2, 6, 2, 300, 64),
                  (1, 2, 2, 384, 128)]:  # enough units, or G odd / G = 1: one part
        assert lib.bwd_workspace_bytes(*shape) == base(*shape)
    for B, H, Hkv, L, d in [(1, 8, 1, 32768, 128), (1, 8, 1, 1024, 128), (1, 16, 4, 8192, 128),
                            (2, 8, 2, 1024, 128), (1, 4, 1, 2048, 64)]:
        assert lib.bwd_workspace_bytes(B, H, Hkv, L, d) == base(B, H, Hkv, L, d) + kv(B, Hkv, L, d)


@pytest.mark.parametrize("shape,expect", [
    ((4, 32, 8, 131072), 9),    # 288 units: two full waves of 228 tiles per CTA
    ((4, 32, 8, 32768), 4),     # one wave of 128 CTAs
    ((1, 32, 8, 131072), 18),   # one wave of 144 CTAs
    ((8, 32, 8, 32768), 2),
    ((1, 8, 1, 524288), 147),
    ((64, 32, 8, 131072), 1),   # 512 (b, g) pairs: one split each
    ((1, 4, 1, 300), 3),        # one tile per split
    # one KV head at batch 1 (a rank of 8-way head sharding): the merge term moves the
    # count to the measured optimum (about 3 sqrt(T) splits)
    ((1, 8, 1, 8192), 22),
    ((1, 8, 1, 32768), 43),
    ((1, 8, 1, 131072), 94),
])
def test_split_rule_values(lib, shape, expect):
    """The split rule: at most two waves of 148 persistent CTAs, minimising
    waves x (tiles per split + 10) + splits / 9, fewer splits on ties."""
    assert lib.decode_num_splits(*shape) == expect


def test_auto_splits_fit_the_noalloc_scratch(lib):
    """With num_splits = 0 a bf16 decode (groups of up to 8) of a batch with
    B * H_kv <= 296 needs at most 296 units, so its scratch fits the in-library array of
    mala_decode_noalloc (4 MiB)."""
    for B in (1, 2, 3, 4, 8, 16, 37, 64):
        for Hkv in (1, 2, 4, 8):
            if B * Hkv > 296:
                continue
            for Nk in (1, 127, 129, 1000, 8192, 65536, 131072, 1 << 20):
                for d in (64, 128):
                    S = lib.decode_num_splits(B, 8 * Hkv, Hkv, Nk)
                    assert 1 <= S and B * Hkv * S <= 296
                    assert S <= -(-Nk // 128)
                    ws = lib.decode_workspace_bytes(B, 8 * Hkv, Hkv, Nk, d, 0, 0)
                    assert 0 < ws <= 4 << 20


def test_bench_reference_split_count(lib):
    import bench
    w = bench.synth.WORKLOADS[bench.DECODE]
    assert lib.decode_num_splits(w.B, w.H, w.H_kv, w.L) == bench.DECODE_SPLITS


def test_bench_accounting():
    sys.path.insert(0, ROOT)
    import bench
    from mass_adaptive_sparse_fwd_b200 import synth

    w = synth.WORKLOADS["sinkband32k"]
    full = bench.fwd_bwd_flops(w, 1.0, 1.0)
    # tile-granular dense counts exceed the exact causal counts only by the diagonal halves
    assert 1.0 < full["fwd_exec"] / full["fwd_dense_eq"] < 1.01
    assert 1.0 < full["bwd_exec"] / full["bwd_dense_eq"] < 1.01
    none = bench.fwd_bwd_flops(w, 0.0, 0.0)
    assert none["fwd_exec"] == pytest.approx(full["fwd_exec"] / 2)
    assert none["bwd_exec"] == pytest.approx(full["bwd_exec"] / 5)
    wd = synth.WORKLOADS["decode128k"]
    kbytes = wd.B * wd.H_kv * wd.L * wd.d * 2
    assert bench.decode_bytes(wd, 0, 1) > kbytes
    assert bench.decode_bytes(wd, 10, 1) - bench.decode_bytes(wd, 0, 1) == 10 * 128 * 128 * 2


_DIST_CHILD = r"""
import os, sys
sys.path.insert(0, {root!r})
import bench
d = bench.Dist().init("gloo")
r = d.rank
w = bench.rank_workload(bench.synth.WORKLOADS["sinkband32k"], r)
v = d.max(10.0 + r)
d.barrier()
print(f"rank={{r}} seed={{w.seed}} max={{v}}", flush=True)
d.close()
"""


def test_bench_two_ranks_gloo(tmp_path):
    script = tmp_path / "child.py"
    script.write_text(_DIST_CHILD.format(root=ROOT))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", "29533", str(script)]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=180)
    assert out.returncode == 0, out.stderr[-2000:]
    found = sorted(re.findall(r"rank=\d seed=\d+ max=[\d.]+", out.stdout))
    assert found == ["rank=0 seed=3 max=11.0", "rank=1 seed=1003 max=11.0"], out.stdout


_SHARD_CHILD = r"""
import os, sys
sys.path.insert(0, {root!r})
import numpy as np
import bench
import oracle
d = bench.Dist().init("gloo")
r, n = d.rank, d.world
w, inp = bench.synth.small_training(B=1, H=8, Hkv=4, L=384, d=32, structure="peaked", seed=5)
ws, part = bench.shard_training(w, inp, r, n)
O, LSE, mask, _ = oracle.mala_fwd(part["Q"], part["K"], part["V"], w.scale, 1.0)
dQ, dK, dV, bmask, _ = oracle.mala_bwd(part["Q"], part["K"], part["V"], O, LSE, part["dO"],
                                       w.scale, 1.0)
wd = bench.synth.Workload("shard_decode", 2, 8, 4, 1000, 32, "bf16", "planted", 6, decode=True)
dec = bench.synth.make_decode(wd)
wds, dpart = bench.shard_decode(wd, dec, r, n)
Od, Ld, dmask, _, _, _ = oracle.mala_decode(dpart["q"], dpart["K"], dpart["V"], wd.scale, 1.0, 3)
np.savez({out!r} + f"/rank{{r}}.npz", O=O, LSE=LSE, mask=mask, dQ=dQ, dK=dK, dV=dV,
         bmask=bmask, Od=Od, Ld=Ld, dmask=dmask, H=ws.H, Hkv=ws.H_kv)
v = d.max(10.0 + r)
d.barrier()
print(f"rank={{r}} heads={{ws.H}}/{{ws.H_kv}} max={{v}}", flush=True)
d.close()
"""


def test_head_sharding_partition():
    sys.path.insert(0, ROOT)
    import bench

    for world in (1, 2, 4, 8):
        got = [bench.head_shard(32, 8, r, world) for r in range(world)]
        # contiguous, disjoint, covering; query heads follow their KV heads (G = 4)
        assert got[0][0] == 0 and got[-1][1] == 8 and got[-1][3] == 32
        for (g0, g1, h0, h1), nxt in zip(got, got[1:] + [None]):
            assert g1 - g0 == 8 // world and (h0, h1) == (4 * g0, 4 * g1)
            if nxt:
                assert nxt[0] == g1 and nxt[2] == h1
    with pytest.raises(ValueError):
        bench.head_shard(32, 8, 0, 3)


def test_head_sharded_ranks_reproduce_the_unsharded_problem_gloo(tmp_path):
    """Two gloo ranks each run the oracle on their head shard of one problem; the shards,
    put back together along the head axis, equal the unsharded results exactly (every head
    is independent, so sharding changes nothing), and the timing reduction is a max."""
    import oracle
    from mass_adaptive_sparse_fwd_b200 import synth

    script = tmp_path / "child.py"
    script.write_text(_SHARD_CHILD.format(root=ROOT, out=str(tmp_path)))
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", "29541", str(script)]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    found = sorted(re.findall(r"rank=\d heads=\d+/\d+ max=[\d.]+", out.stdout))
    assert found == ["rank=0 heads=4/2 max=11.0", "rank=1 heads=4/2 max=11.0"], out.stdout
    parts = [np.load(tmp_path / f"rank{r}.npz") for r in range(2)]
    w, inp = synth.small_training(B=1, H=8, Hkv=4, L=384, d=32, structure="peaked", seed=5)
    O, LSE, mask, _ = oracle.mala_fwd(inp["Q"], inp["K"], inp["V"], w.scale, 1.0)
    dQ, dK, dV, bmask, _ = oracle.mala_bwd(inp["Q"], inp["K"], inp["V"], O, LSE, inp["dO"],
                                           w.scale, 1.0)
    cat = lambda k, ax: np.concatenate([p[k] for p in parts], axis=ax)
    np.testing.assert_array_equal(cat("O", 2), O)
    np.testing.assert_array_equal(cat("LSE", 1), LSE)
    np.testing.assert_array_equal(cat("mask", 1), mask)
    np.testing.assert_array_equal(cat("bmask", 1), bmask)
    for k, ref in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        np.testing.assert_array_equal(cat(k, 2), ref)
    wd = synth.Workload("shard_decode", 2, 8, 4, 1000, 32, "bf16", "planted", 6, decode=True)
    dec = synth.make_decode(wd)
    Od, Ld, dmask, _, _, _ = oracle.mala_decode(dec["q"], dec["K"], dec["V"], wd.scale, 1.0, 3)
    np.testing.assert_array_equal(cat("Od", 1), Od)
    np.testing.assert_array_equal(cat("Ld", 1), Ld)
    np.testing.assert_array_equal(cat("dmask", 1), dmask)


def test_noalloc_decode_rejects_oversized_problems(lib):
    """The size check of the allocation-free decode comes before any CUDA call: run on a
    machine without a GPU only, with placeholder addresses that are never dereferenced."""
    if torch.cuda.is_available():
        pytest.skip("host-only check (placeholder addresses)")
    L = lib.lib()
    # 64 x 64 heads x 1024 splits of (128 + 1) floats is far beyond the fixed scratch
    need = L.mala_decode_workspace_bytes(64, 64, 8, 131072, 128, 0, 1024)
    assert need > 4 << 20
    p = ctypes.c_void_p(1 << 20)
    st = L.mala_decode_noalloc(p, p, p, p, p, 64, 64, 8, 131072, 128, 0, 0.1, 1.0, 1024, 0,
                               None, None)
    assert st == 5  # MALA_ERR_WORKSPACE


def test_debug_margin_buffer_too_small_is_rejected_before_any_launch(lib):
    """mala_set_debug: a call that needs more margin entries than registered returns
    MALA_ERR_INVALID_ARG before any CUDA call (host only, placeholder addresses)."""
    if torch.cuda.is_available():
        pytest.skip("host-only check (placeholder addresses)")
    L = lib.lib()
    p = ctypes.c_void_p(16 * 1024)
    dbg = lib.MalaDebug(16 * 1024, 3)  # 3 entries; a 2-block forward needs 1*2*2*2 = 8
    assert L.mala_set_debug(ctypes.byref(dbg)) == 0
    try:
        assert L.mala_fwd(p, p, p, p, p, 1, 2, 1, 256, 128, 0, 0.1, 1.0, 0, None, 0, None,
                          None) == 1
        assert L.mala_bwd(p, p, p, p, p, p, p, p, p, 1, 2, 1, 256, 128, 0, 0.1, 1.0, 0, None, 0,
                          None, None) == 1
        assert L.mala_decode(p, p, p, p, p, 1, 2, 1, 1000, 128, 0, 0.1, 1.0, 1, 0, None, 0,
                             None, None) == 1  # [1, 2, 8] = 16 entries
    finally:
        assert L.mala_set_debug(None) == 0
    bad = lib.MalaDebug(16 * 1024 + 2, 8)  # misaligned buffer
    assert L.mala_set_debug(ctypes.byref(bad)) == 1
