#!/usr/bin/env python3
"""Benchmark of the MALA hot path on B200: training forward + backward at 32K and split-KV
decode at 128K, through the library's C ABI.

One step = mala_fwd + mala_bwd on the 32K training workload (B=1, H=32, H_kv=8,
L=32768, d=128, bf16, sink + local-band synthetic states, tau = 1) followed by one
mala_decode on the 128K decode workload (B=4, H=32, H_kv=8, N_k=131072, d=128, planted
keys, tau = 1).  The same steps are also timed at tau = 0 (the library's dense path).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mala|reference]
Multi-GPU: launched by torch.distributed.run, one rank per GPU; every rank runs its own
independent problem (different seeds) with no collective on the data path (weak
scaling); timing is the max over ranks.  Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

# the CPU oracle's OpenMP threads must not spin while idle: its baseline is measured in
# process CPU time (set before any OpenMP runtime is loaded)
os.environ.setdefault("OMP_WAIT_POLICY", "PASSIVE")

import numpy as np  # noqa: E402
import torch  # noqa: E402

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from mass_adaptive_sparse_fwd_b200 import synth  # noqa: E402

METRIC = "MALA fwd+bwd ms and TFLOPS at 32K, decode µs at 128K; % of bf16 tensor peak"
TRAIN = "sinkband32k"  # --train sinkband128k times the 128K one-GPU training shape instead
SKIP_TRAIN = "prevtok32k"  # concentrated states for the skip-regime block
SKIP_DECODE = "heavy128k"  # KV cache with a heavy hitter in every 8th key tile
DECODE = "decode128k"
# the split count mala_decode_num_splits gives the decode workload (a host test checks it);
# the reference arm, which does not load the library, runs its oracle decode with it
DECODE_SPLITS = 9
TAU = 1.0
KERNELS_PER_STEP = 5  # fwd 1, bwd 3 (D preprocess, main, dQ convert), decode 1


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                "bf16_tflops_sustained": pk["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def ncu_figures():
    """Counters of the main kernels at the bench workload from a committed ncu capture
    (profiles/ncu_bench_kernels.json), used only while every kernel source they were taken
    on is unchanged; None otherwise."""
    import hashlib

    prof = os.path.join(ROOT, "profiles", "ncu_bench_kernels.json")
    if not os.path.exists(prof):
        return None
    with open(prof) as f:
        fig = json.load(f)
    for name, sha in fig.get("sources_sha256_16", {}).items():
        with open(os.path.join(ROOT, "mass_adaptive_sparse_fwd_b200", "csrc", name), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] != sha:
                return None
    return fig


# ----------------------------------------------------------------------------- dist


class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend: str):
        if self.world > 1:
            import datetime

            import torch.distributed as dist

            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist
        return self

    def barrier(self):
        if self.pg is not None:
            if self.pg.get_backend() == "nccl":
                self.pg.barrier(device_ids=[self.local_rank])
            else:
                self.pg.barrier()

    def max(self, x: float, device="cpu") -> float:
        if self.pg is None:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def rank_workload(w: synth.Workload, rank: int) -> synth.Workload:
    """Each rank gets an independent problem of the same shape (weak scaling)."""
    return dataclasses.replace(w, seed=w.seed + 1000 * rank)


def head_shard(H: int, Hkv: int, rank: int, world: int):
    """Tensor-parallel head sharding of one problem (the page's TP setup, §3 "Operator
    Latency and Memory"): rank r owns KV heads [r Hkv / N, (r + 1) Hkv / N) and the G
    query heads that read each of them.  Returns (g0, g1, h0, h1)."""
    if world < 1 or Hkv % world != 0:
        raise ValueError(f"{Hkv} KV heads do not split evenly over {world} ranks")
    G = H // Hkv
    g0, g1 = rank * Hkv // world, (rank + 1) * Hkv // world
    return g0, g1, g0 * G, g1 * G


def shard_training(w: synth.Workload, inp: dict, rank: int, world: int):
    """The rank's slice of a training problem: Q, dO on its query heads, K, V on its KV
    heads (each a contiguous copy in the same [B, L, heads, d] layout)."""
    g0, g1, h0, h1 = head_shard(w.H, w.H_kv, rank, world)
    part = {k: np.ascontiguousarray(inp[k][:, :, h0:h1]) for k in ("Q", "dO")}
    part.update({k: np.ascontiguousarray(inp[k][:, :, g0:g1]) for k in ("K", "V")})
    return dataclasses.replace(w, H=h1 - h0, H_kv=g1 - g0), part


def shard_decode(w: synth.Workload, inp: dict, rank: int, world: int):
    """The rank's slice of a decode problem: q [B, heads, d], cache [B, N_k, KV heads, d]."""
    g0, g1, h0, h1 = head_shard(w.H, w.H_kv, rank, world)
    part = {"q": np.ascontiguousarray(inp["q"][:, h0:h1])}
    part.update({k: np.ascontiguousarray(inp[k][:, :, g0:g1]) for k in ("K", "V")})
    return dataclasses.replace(w, H=h1 - h0, H_kv=g1 - g0), part


# ----------------------------------------------------------------------------- work accounting


def fwd_bwd_flops(w: synth.Workload, fwd_retained: float, bwd_retained: float):
    """Executed and dense-equivalent FLOPs of one forward + backward (tile granular).
    Forward: QK^T on every legal tile + PV on retained tiles; backward: QK^T recompute on
    every legal tile + dP, dV, dK, dQ on retained tiles (Eq. (13)/(16) accounting)."""
    T = math.ceil(w.L / 128)
    legal = T * (T + 1) // 2 * w.B * w.H
    per = 2.0 * w.d * 128 * 128
    fwd_exec = per * legal * (1.0 + fwd_retained)
    bwd_exec = per * legal * (1.0 + 4.0 * bwd_retained)
    pairs = w.L * (w.L + 1) / 2 * w.B * w.H
    return {"fwd_exec": fwd_exec, "bwd_exec": bwd_exec, "fwd_dense_eq": 4.0 * w.d * pairs,
            "bwd_dense_eq": 10.0 * w.d * pairs, "legal_tiles": legal}


def decode_bytes(w: synth.Workload, vtiles_loaded: int, S: int) -> float:
    """Algorithmic HBM bytes of one decode call: all K, the V tiles some head of the
    group retained, q / O and the split partials."""
    kbytes = w.B * w.H_kv * w.L * w.d * 2
    vbytes = vtiles_loaded * 128 * w.d * 2
    qo = 2 * w.B * w.H * w.d * 2
    part = 2 * w.B * w.H * S * (w.d + 1) * 4
    return kbytes + vbytes + qo + part


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    sm.append(float(parts[0]))
                    smax.append(float(parts[1]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[4:8]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- CPU oracle


def _spread(lo: int, hi: int, n: int):
    """n block indices spread uniformly over [lo, hi], both ends included."""
    if n <= 1:
        return [hi]
    return [lo + round(k * (hi - lo) / (n - 1)) for k in range(n)]


def oracle_plan(wt: synth.Workload, n: int):
    """The sampled units of one oracle step, n per leg (one per oracle thread, so every
    thread is busy in every leg): forward and dQ query blocks spread over the whole block
    range (the last included), dK/dV key blocks spread over the last quarter (the heavier
    key blocks hold up to 4x the tiles and the per-tile cost does not depend on the
    block), heads cycled."""
    T = -(-wt.L // 128)
    fwd = [(0, (7 * k) % wt.H, i) for k, i in enumerate(_spread(0, T - 1, n))]
    dq = [(0, (11 * k + 3) % wt.H, i) for k, i in enumerate(_spread(0, T - 1, n))]
    kv = [(0, k % wt.H_kv, j) for k, j in enumerate(_spread(3 * T // 4, T - 1, n))]
    return fwd, kv, dq


def oracle_sample(wt: synth.Workload, wd: synth.Workload, train, dec, S: int):
    """Times the fp64 CPU oracle on a bounded sample of one step and extrapolates to the
    full step.  Every leg runs one sampled unit per oracle thread.  The estimate per leg is
    process CPU seconds per tile (measured around the oracle's C call alone, fixed per-call
    work subtracted) x the step's tiles / threads: the wall time of the full step, in
    which thousands of units keep every thread busy.  The backward legs are conditioned
    on a stand-in forward output (O = 0, LSE_q = log(q + 1)), the same in both arms; the
    decode leg runs every (b, h) row of the decode workload as it is (no extrapolation).
    Returns a dict with the extrapolated ms per step and the measured pieces."""
    import oracle

    oracle.build()
    n = oracle.num_threads()
    T = -(-wt.L // 128)
    G = wt.H // wt.H_kv
    legal = T * (T + 1) // 2 * wt.B * wt.H
    fwd_u, kv_u, q_u = oracle_plan(wt, n)
    none = np.zeros((0, 3), np.int32)
    t0 = time.perf_counter()
    oracle.mala_fwd(train["Q"], train["K"], train["V"], wt.scale, TAU, units=fwd_u)
    c_fwd = oracle.LAST_CALL["cpu"]
    LSEc = np.broadcast_to(np.log(np.arange(1, wt.L + 1, dtype=np.float64)),
                           (wt.B, wt.H, wt.L))
    Oc = np.zeros(train["Q"].shape)
    args = (train["Q"], train["K"], train["V"], Oc, LSEc, train["dO"], wt.scale, TAU)
    oracle.mala_bwd(*args, kv_units=none, q_units=none)  # fixed per-call work (D rows)
    w_fix, c_fix = oracle.LAST_CALL["wall"], oracle.LAST_CALL["cpu"]
    _, _, _, kmask, _ = oracle.mala_bwd(*args, kv_units=kv_u, q_units=none)
    c_kv = oracle.LAST_CALL["cpu"] - c_fix
    oracle.mala_bwd(*args, kv_units=none, q_units=q_u)
    c_q = oracle.LAST_CALL["cpu"] - c_fix
    oracle.mala_decode(dec["q"], dec["K"], dec["V"], wd.scale, TAU, S)
    w_dec = oracle.LAST_CALL["wall"]
    spent = time.perf_counter() - t0
    fwd_tiles = sum(i + 1 for _, _, i in fwd_u)
    kv_tiles = sum(G * (T - j) for _, _, j in kv_u)
    q_tiles = sum(i + 1 for _, _, i in q_u)
    fwd_ms = 1e3 * c_fwd / fwd_tiles * legal / n
    bwd_ms = 1e3 * (w_fix + c_kv / kv_tiles * legal / n + c_q / q_tiles * legal / n)
    dec_ms = 1e3 * w_dec
    desc = (f"fp64 oracle, {n} threads; one step = forward on {len(fwd_u)} query blocks "
            f"({fwd_tiles} tiles), dK/dV on {len(kv_u)} key blocks ({kv_tiles} tiles), dQ on "
            f"{len(q_u)} query blocks ({q_tiles} tiles) of {wt.name} (backward conditioned on "
            f"O = 0, LSE_q = log(q + 1)), and all {wd.B * wd.H} rows of {DECODE} (S = {S}); "
            f"extrapolated by process CPU seconds per tile x {legal} tiles / {n} threads")
    return {"ms": fwd_ms + bwd_ms + dec_ms, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
            "decode_ms": dec_ms, "threads": n, "spent_s": spent, "sample": desc,
            "bwd_sample_retained": float((kmask[kmask >= 0] == 1).mean())}


def run_reference(args, dist: Dist):
    """Reference arm: the CPU oracle as it stands, each step the bounded sample of
    ``oracle_sample`` (the plan the GPU arm's cpu_baseline uses)."""
    if dist.rank != 0:
        return
    wt, wd = synth.WORKLOADS[TRAIN], synth.WORKLOADS[DECODE]
    train = synth.make_training(wt)
    dec = synth.make_decode(wd)
    S = DECODE_SPLITS
    vals, last = [], None
    for s in range(args.warmup + args.steps):
        last = oracle_sample(wt, wd, train, dec, S)
        if s >= args.warmup:
            vals.append(last["ms"])
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "ms",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": value, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{TRAIN} fwd+bwd + {DECODE} decode", "tau": TAU},
            "cpu_baseline": {"value": value, "unit": "ms", "cores": last["threads"],
                             "kind": "oracle", "sample": last["sample"],
                             "legs_ms": {k: last[k] for k in ("fwd_ms", "bwd_ms", "decode_ms")},
                             "step_spread": [min(vals), max(vals)]},
            "e2e": {"value": value, "unit": "ms", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm


def run_mala(args, dist: Dist):
    from mass_adaptive_sparse_fwd_b200 import mala

    dev = torch.device("cuda", dist.local_rank)
    torch.cuda.set_device(dev)
    peaks = _peaks()
    if args.shard == "heads":
        # one problem, its KV heads (with their query heads) split across the ranks
        base_t, base_d = synth.WORKLOADS[args.train], synth.WORKLOADS[DECODE]
        wt, train = shard_training(base_t, synth.make_training(base_t), dist.rank, dist.world)
        wd, dec = shard_decode(base_d, synth.make_decode(base_d), dist.rank, dist.world)
    else:
        wt = rank_workload(synth.WORKLOADS[args.train], dist.rank)
        wd = rank_workload(synth.WORKLOADS[DECODE], dist.rank)
        train = synth.make_training(wt)
        dec = synth.make_decode(wd)
    bf = lambda x: torch.from_numpy(x).to(dev).to(torch.bfloat16)
    Q, K, V, dO = (bf(train[k]) for k in ("Q", "K", "V", "dO"))
    q, Kc, Vc = (bf(dec[k]) for k in ("q", "K", "V"))
    B, L, H, d = Q.shape
    Hkv = K.shape[2]
    S = mala.decode_num_splits(wd.B, wd.H, wd.H_kv, wd.L)
    O = torch.empty_like(Q)
    LSE = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    Od = torch.empty_like(q)
    LSEd = torch.empty((wd.B, wd.H), dtype=torch.float32, device=dev)
    wsf = mala.alloc_workspace(mala.fwd_workspace_bytes(B, H, Hkv, L, d), dev)
    wsb = mala.alloc_workspace(mala.bwd_workspace_bytes(B, H, Hkv, L, d), dev)
    wsd = mala.alloc_workspace(mala.decode_workspace_bytes(wd.B, wd.H, wd.H_kv, wd.L, d, 0, S),
                               dev)
    stream = torch.cuda.current_stream(dev)

    def step(tau, ev=None):
        if ev is not None:
            ev[0].record(stream)
        mala.mala_fwd(Q, K, V, wt.scale, tau, O=O, LSE=LSE, workspace=wsf)
        if ev is not None:
            ev[1].record(stream)
        mala.mala_bwd(Q, K, V, O, LSE, dO, wt.scale, tau, dQ=dQ, dK=dK, dV=dV, workspace=wsb)
        if ev is not None:
            ev[2].record(stream)
        mala.mala_decode(q, Kc, Vc, wd.scale, tau, num_splits=S, O=Od, LSE=LSEd, workspace=wsd)
        if ev is not None:
            ev[3].record(stream)

    def timed(tau, clocks=None):
        for _ in range(args.warmup):
            step(tau)
        torch.cuda.synchronize(dev)
        dist.barrier()
        torch.cuda.synchronize(dev)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        if clocks:
            clocks.start()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for k in range(args.steps):
            step(tau, evs[k])
        end.record(stream)
        torch.cuda.synchronize(dev)
        dist.barrier()
        torch.cuda.synchronize(dev)
        clk = clocks.stop() if clocks else None
        total = start.elapsed_time(end) / args.steps
        fwd = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
        bwd = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
        dcd = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
        for ws in (wsf, wsb, wsd):
            err = mala.read_device_error(ws)
            if err:
                raise RuntimeError(f"device error word 0x{err:x}")
        med = {"fwd_bwd_ms": statistics.median(e[0].elapsed_time(e[2]) for e in evs),
               "decode_us": 1e3 * statistics.median(e[2].elapsed_time(e[3]) for e in evs)}
        return {"step_ms": total, "fwd_ms": fwd, "bwd_ms": bwd, "decode_ms": dcd, "clocks": clk,
                "median": med}

    clocks = ClockSampler(torch.cuda.current_device()) if dist.rank == 0 else None
    res = timed(TAU, clocks)
    res0 = timed(0.0)
    # max over ranks of every figure (device timing)
    for r in (res, res0):
        for k in ("step_ms", "fwd_ms", "bwd_ms", "decode_ms"):
            r[k] = dist.max(r[k], device=dev)

    # retained work (one masked call of each operator, outside the timed region)
    T = mala.n_tiles(L)
    fmask = torch.zeros((B, H, T, T), dtype=torch.uint8, device=dev)
    bmask = torch.zeros((B, H, T, T), dtype=torch.uint8, device=dev)
    dmask = torch.zeros((wd.B, wd.H, mala.n_tiles(wd.L)), dtype=torch.uint8, device=dev)
    mala.mala_fwd(Q, K, V, wt.scale, TAU, O=O, LSE=LSE, workspace=wsf, tile_mask=fmask)
    mala.mala_bwd(Q, K, V, O, LSE, dO, wt.scale, TAU, dQ=dQ, dK=dK, dV=dV, workspace=wsb,
                  tile_mask=bmask)
    mala.mala_decode(q, Kc, Vc, wd.scale, TAU, num_splits=S, O=Od, LSE=LSEd, workspace=wsd,
                     tile_mask=dmask)
    torch.cuda.synchronize(dev)
    legal = torch.ones(T, T, dtype=torch.bool, device=dev).tril()
    fret = float(fmask[:, :, legal].float().mean())
    bret = float(bmask[:, :, legal].float().mean())
    G = wd.H // wd.H_kv
    group_keep = dmask.view(wd.B, wd.H_kv, G, -1).amax(dim=2)
    vtiles = int(group_keep.sum())
    dret = float(dmask.float().mean())
    # slots per query (M1): retained tiles contribute 128 key slots to each of their rows
    fl = fwd_bwd_flops(wt, fret, bret)
    dense_fl = fwd_bwd_flops(wt, 1.0, 1.0)
    step_fb = res["fwd_ms"] + res["bwd_ms"]
    dense_fb = res0["fwd_ms"] + res0["bwd_ms"]
    exec_tf = (fl["fwd_exec"] + fl["bwd_exec"]) / (step_fb * 1e-3) / 1e12
    deq_tf = (fl["fwd_dense_eq"] + fl["bwd_dense_eq"]) / (step_fb * 1e-3) / 1e12
    dense_exec_tf = (dense_fl["fwd_exec"] + dense_fl["bwd_exec"]) / (dense_fb * 1e-3) / 1e12
    dbytes = decode_bytes(wd, vtiles, S)
    dbytes0 = decode_bytes(wd, wd.B * wd.H_kv * mala.n_tiles(wd.L), S)
    dec_gbs = dbytes / (res["decode_ms"] * 1e-3) / 1e9
    dec_gbs0 = dbytes0 / (res0["decode_ms"] * 1e-3) / 1e9

    # roofline of the dominant kernel: the backward call (timed span includes its small
    # D-preprocess and dQ-convert kernels; the main kernel dominates the share).  Each call
    # is timed on its own (tens of ms at the boost clock), so the burst GEMM peak is the
    # denominator; the fraction of the sustained peak is given beside it.
    peak = peaks["bf16_tflops"]
    peak_sus = peaks["bf16_tflops_sustained"]
    bwd_tf = fl["bwd_exec"] / (res["bwd_ms"] * 1e-3) / 1e12
    ncu = ncu_figures()
    traffic = None
    if ncu and "mala_bwd_kernel<128,1>" in ncu["kernels"]:
        traffic = ncu["kernels"]["mala_bwd_kernel<128,1>"].get("dram_bytes")

    # end to end through the C ABI with host buffers (pinned), copies in the timed region.
    # Steps are pipelined over two sets of device buffers: while step k computes on its
    # stream, the inputs of step k + 1 are copied in on a second stream and the outputs of
    # step k - 1 copied out on a third (events order every reuse of a buffer), so the copy
    # engines overlap the kernels; every step's copies lie inside the timed region.
    e2e = None
    if not args.no_e2e:
        host_in = {k: torch.from_numpy(train[k]).to(torch.bfloat16).pin_memory()
                   for k in ("Q", "K", "V", "dO")}
        host_in["q"] = torch.from_numpy(dec["q"]).to(torch.bfloat16).pin_memory()
        out_like = {"O": O, "LSE": LSE, "dQ": dQ, "dK": dK, "dV": dV, "Od": Od, "LSEd": LSEd}
        host_out = [{n: torch.empty(t.shape, dtype=t.dtype).pin_memory()
                     for n, t in out_like.items()} for _ in range(2)]
        bufs = [{"Q": Q, "K": K, "V": V, "dO": dO, "q": q, **out_like}]
        bufs.append({n: torch.empty_like(t) for n, t in bufs[0].items()})
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        in_ready = [ev(), ev()]   # inputs of set b copied in
        in_free = [ev(), ev()]    # the step on set b has finished with its inputs
        computed = [ev(), ev()]   # outputs of set b written
        out_free = [ev(), ev()]   # outputs of set b copied out
        for e in in_free + out_free:
            e.record(stream)

        def run_on(bf_):
            mala.mala_fwd(bf_["Q"], bf_["K"], bf_["V"], wt.scale, TAU, O=bf_["O"], LSE=bf_["LSE"],
                          workspace=wsf)
            mala.mala_bwd(bf_["Q"], bf_["K"], bf_["V"], bf_["O"], bf_["LSE"], bf_["dO"], wt.scale,
                          TAU, dQ=bf_["dQ"], dK=bf_["dK"], dV=bf_["dV"], workspace=wsb)
            mala.mala_decode(bf_["q"], Kc, Vc, wd.scale, TAU, num_splits=S, O=bf_["Od"],
                             LSE=bf_["LSEd"], workspace=wsd)

        def e2e_steps(n):
            for k in range(n):
                b = k & 1
                with torch.cuda.stream(s_in):
                    s_in.wait_event(in_free[b])
                    for name, t in host_in.items():
                        bufs[b][name].copy_(t, non_blocking=True)
                    in_ready[b].record(s_in)
                stream.wait_event(in_ready[b])
                stream.wait_event(out_free[b])
                run_on(bufs[b])
                in_free[b].record(stream)
                computed[b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(computed[b])
                    for name in out_like:
                        host_out[b][name].copy_(bufs[b][name], non_blocking=True)
                    out_free[b].record(s_out)
            for b in range(2):  # the last copies out are part of the run
                stream.wait_event(out_free[b])

        e2e_steps(args.warmup)
        torch.cuda.synchronize(dev)
        dist.barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        s_in.wait_event(s0)
        e2e_steps(args.steps)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        dist.barrier()
        e2e_ms = dist.max(s0.elapsed_time(s1) / args.steps, device=dev)
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
        e2e = {"value": e2e_ms, "unit": "ms", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h,
               "note": "fwd+bwd+decode step incl. host->device inputs (Q,K,V,dO,q; the KV "
                       "cache is resident) and device->host outputs, from pinned host memory; "
                       "steps pipelined over two device buffer sets (the copies of neighbouring "
                       "steps overlap the kernels on their own streams)"}
        del bufs

    # skip regime: the same fwd + bwd on concentrated "previous-token" states, where most
    # tiles fall below tau / L_q; shows the step time following the retained work
    skip = None
    if not args.no_skip_regime:
        wl = rank_workload(synth.WORKLOADS[SKIP_TRAIN], dist.rank)
        loc = synth.make_training(wl)
        sQ, sK, sV, sdO = (bf(loc[k]) for k in ("Q", "K", "V", "dO"))
        del loc
        sO = torch.empty_like(sQ)
        sLSE = torch.empty((wl.B, wl.H, wl.L), dtype=torch.float32, device=dev)
        sdQ, sdK, sdV = torch.empty_like(sQ), torch.empty_like(sK), torch.empty_like(sV)
        swf = mala.alloc_workspace(mala.fwd_workspace_bytes(wl.B, wl.H, wl.H_kv, wl.L, wl.d), dev)
        swb = mala.alloc_workspace(mala.bwd_workspace_bytes(wl.B, wl.H, wl.H_kv, wl.L, wl.d), dev)

        def sfwd(tau, mask=None):
            mala.mala_fwd(sQ, sK, sV, wl.scale, tau, O=sO, LSE=sLSE, workspace=swf, tile_mask=mask)

        def sbwd(tau, mask=None):
            mala.mala_bwd(sQ, sK, sV, sO, sLSE, sdO, wl.scale, tau, dQ=sdQ, dK=sdK, dV=sdV,
                          workspace=swb, tile_mask=mask)

        def fb(tau):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            for _ in range(args.warmup):
                sfwd(tau)
                sbwd(tau)
            torch.cuda.synchronize(dev)
            dist.barrier()
            torch.cuda.synchronize(dev)
            ev[0].record(stream)
            for _ in range(args.steps):
                sfwd(tau)
            ev[1].record(stream)
            for _ in range(args.steps):
                sbwd(tau)
            ev[2].record(stream)
            torch.cuda.synchronize(dev)
            dist.barrier()
            for ws in (swf, swb):
                err = mala.read_device_error(ws)
                if err:
                    raise RuntimeError(f"device error word 0x{err:x}")
            return (dist.max(ev[0].elapsed_time(ev[1]) / args.steps, device=dev),
                    dist.max(ev[1].elapsed_time(ev[2]) / args.steps, device=dev))

        sf1, sb1 = fb(TAU)
        sf0, sb0 = fb(0.0)
        sT = mala.n_tiles(wl.L)
        sfm = torch.zeros((wl.B, wl.H, sT, sT), dtype=torch.uint8, device=dev)
        sbm = torch.zeros_like(sfm)
        sfwd(TAU, sfm)
        sbwd(TAU, sbm)
        torch.cuda.synchronize(dev)
        slegal = torch.ones(sT, sT, dtype=torch.bool, device=dev).tril()
        sfr = float(sfm[:, :, slegal].float().mean())
        sbr = float(sbm[:, :, slegal].float().mean())
        sfl = fwd_bwd_flops(wl, sfr, sbr)
        sfl0 = fwd_bwd_flops(wl, 1.0, 1.0)
        skip = {"workload": f"{SKIP_TRAIN} (B={wl.B},H={wl.H},H_kv={wl.H_kv},L={wl.L},d={wl.d}; "
                            "q_t = 18 sqrt(d) K_(t-1) / |K_(t-1)|^2 + 0.3 noise)",
                "retained": {"fwd_tiles": sfr, "bwd_tiles": sbr},
                "tau1": {"fwd_ms": sf1, "bwd_ms": sb1, "fwd_bwd_ms": sf1 + sb1,
                         "executed_tflops": (sfl["fwd_exec"] + sfl["bwd_exec"]) /
                                            ((sf1 + sb1) * 1e-3) / 1e12},
                "tau0": {"fwd_ms": sf0, "bwd_ms": sb0, "fwd_bwd_ms": sf0 + sb0},
                "speedup_vs_tau0": {"fwd": sf0 / sf1, "bwd": sb0 / sb1,
                                    "fwd_bwd": (sf0 + sb0) / (sf1 + sb1)},
                "work_ratio": {"fwd": sfl["fwd_exec"] / sfl0["fwd_exec"],
                               "bwd": sfl["bwd_exec"] / sfl0["bwd_exec"]}}
        del sQ, sK, sV, sdO, sO, sLSE, sdQ, sdK, sdV, swf, swb

        # decode on a cache whose every split holds dominant keys: the tiles between
        # them, and their V loads, are skipped
        wh = rank_workload(synth.WORKLOADS[SKIP_DECODE], dist.rank)
        loc = synth.make_decode(wh)
        hq, hK, hV = (bf(loc[k]) for k in ("q", "K", "V"))
        del loc
        hO = torch.empty_like(hq)
        hL = torch.empty((wh.B, wh.H), dtype=torch.float32, device=dev)
        hS = mala.decode_num_splits(wh.B, wh.H, wh.H_kv, wh.L)
        hws = mala.alloc_workspace(
            mala.decode_workspace_bytes(wh.B, wh.H, wh.H_kv, wh.L, wh.d, 0, hS), dev)

        def hdec(tau, mask=None):
            mala.mala_decode(hq, hK, hV, wh.scale, tau, num_splits=hS, O=hO, LSE=hL,
                             workspace=hws, tile_mask=mask)

        def dtime(tau):
            for _ in range(args.warmup):
                hdec(tau)
            torch.cuda.synchronize(dev)
            dist.barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                hdec(tau)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            dist.barrier()
            err = mala.read_device_error(hws)
            if err:
                raise RuntimeError(f"device error word 0x{err:x}")
            return dist.max(e0.elapsed_time(e1) / args.steps * 1e3, device=dev)

        hd1 = dtime(TAU)
        hd0 = dtime(0.0)
        hT = mala.n_tiles(wh.L)
        hmask = torch.zeros((wh.B, wh.H, hT), dtype=torch.uint8, device=dev)
        hdec(TAU, hmask)
        torch.cuda.synchronize(dev)
        hG = wh.H // wh.H_kv
        hv = int(hmask.view(wh.B, wh.H_kv, hG, -1).amax(dim=2).sum())
        hb1 = decode_bytes(wh, hv, hS)
        hb0 = decode_bytes(wh, wh.B * wh.H_kv * hT, hS)
        skip["decode"] = {
            "workload": f"{SKIP_DECODE} (B={wh.B},H={wh.H},H_kv={wh.H_kv},N_k={wh.L},d={wh.d}; "
                        "a heavy hitter shared by each KV group in every 8th key tile)",
            "splits": hS,
            "retained": {"tiles": float(hmask.float().mean()),
                         "v_tiles": hv / (wh.B * wh.H_kv * hT)},
            "tau1_us": hd1, "tau0_us": hd0, "speedup_vs_tau0": hd0 / hd1,
            "bytes_ratio": hb1 / hb0,
            "tau1_gbs": hb1 / (hd1 * 1e-6) / 1e9, "tau0_gbs": hb0 / (hd0 * 1e-6) / 1e9}
        del hq, hK, hV, hO, hL, hws

    # chunked prefill: the last 4096 queries of the 32K sink + band sequence against all
    # 32768 keys (causal offset 28672), tau = 1 and tau = 0
    prefill = None
    if not args.no_skip_regime:
        wp = rank_workload(synth.WORKLOADS[TRAIN], dist.rank)
        loc = synth.make_training(wp)
        Nq, Nk = 4096, wp.L
        pQ = bf(np.ascontiguousarray(loc["Q"][:, Nk - Nq:]))
        pK, pV = bf(loc["K"]), bf(loc["V"])
        vQ = bf(np.ascontiguousarray(loc["Q"][0]))  # the whole sequence, for the packed batch
        del loc
        pO = torch.empty_like(pQ)
        pL = torch.empty((wp.B, wp.H, Nq), dtype=torch.float32, device=dev)
        pws = mala.alloc_workspace(mala.fwd_workspace_bytes(wp.B, wp.H, wp.H_kv, Nq, wp.d), dev)

        def ptime(tau):
            for _ in range(args.warmup):
                mala.mala_fwd_prefill(pQ, pK, pV, wp.scale, tau, O=pO, LSE=pL, workspace=pws)
            torch.cuda.synchronize(dev)
            dist.barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                mala.mala_fwd_prefill(pQ, pK, pV, wp.scale, tau, O=pO, LSE=pL, workspace=pws)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            dist.barrier()
            st = mala.get_stats(pws)  # the last timed call's tile counts
            return dist.max(e0.elapsed_time(e1) / args.steps, device=dev), st

        pt1, pst = ptime(TAU)
        pt0, _ = ptime(0.0)

        # packed batch: the same 32K sequence cut into 10 documents of 1K..8K tokens,
        # attention within each document
        lens = [8192, 6144, 4096, 4096, 3072, 2048, 2048, 1024, 1024, 1024]
        cu = [0]
        for n_ in lens:
            cu.append(cu[-1] + n_)
        vK, vV = pK[0], pV[0]  # [total, H_kv, d] views of the same keys and values
        vO = torch.empty_like(vQ)
        vL = torch.empty((wp.H, cu[-1]), dtype=torch.float32, device=dev)
        vws = mala.alloc_workspace(mala.varlen_workspace_bytes(cu, wp.H, wp.H_kv, wp.d), dev)

        def vtime(tau):
            for _ in range(args.warmup):
                mala.mala_fwd_varlen(vQ, vK, vV, cu, cu, wp.scale, tau, O=vO, LSE=vL,
                                     workspace=vws)
            torch.cuda.synchronize(dev)
            dist.barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                mala.mala_fwd_varlen(vQ, vK, vV, cu, cu, wp.scale, tau, O=vO, LSE=vL,
                                     workspace=vws)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            dist.barrier()
            return dist.max(e0.elapsed_time(e1) / args.steps, device=dev), mala.get_stats(vws)

        vt1, vst = vtime(TAU)
        vt0, _ = vtime(0.0)
        vfl1 = 2.0 * wp.d * 128 * 128 * (vst["legal_tiles"] + vst["retained_tiles"])
        vfl0 = 2.0 * wp.d * 128 * 128 * 2 * vst["legal_tiles"]
        varlen = {"workload": f"{TRAIN} cut into {len(lens)} documents {lens} "
                              "(packed, attention within each)",
                  "legal_tiles": vst["legal_tiles"],
                  "retained": vst["retained_tiles"] / max(vst["legal_tiles"], 1),
                  "tau1_ms": vt1, "tau0_ms": vt0,
                  "tau1_executed_tflops": vfl1 / (vt1 * 1e-3) / 1e12,
                  "tau0_tflops": vfl0 / (vt0 * 1e-3) / 1e12}
        del vQ, vK, vV, vO, vL, vws
        per_tile = 2.0 * wp.d * 128 * 128
        fl1 = per_tile * (pst["legal_tiles"] + pst["retained_tiles"])
        fl0 = per_tile * 2 * pst["legal_tiles"]
        prefill = {"workload": f"last {Nq} queries of {TRAIN} against its {Nk} keys "
                               f"(B={wp.B},H={wp.H},H_kv={wp.H_kv},d={wp.d}; offset {Nk - Nq})",
                   "legal_tiles": pst["legal_tiles"],
                   "retained": pst["retained_tiles"] / max(pst["legal_tiles"], 1),
                   "tau1_ms": pt1, "tau0_ms": pt0, "speedup_vs_tau0": pt0 / pt1,
                   "tau1_executed_tflops": fl1 / (pt1 * 1e-3) / 1e12,
                   "tau0_tflops": fl0 / (pt0 * 1e-3) / 1e12, "varlen": varlen}
        del pQ, pK, pV, pO, pL, pws

    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        o = oracle_sample(wt, wd, train, dec, S)
        cpu = {"value": o["ms"], "unit": "ms", "cores": o["threads"], "kind": "oracle",
               "sample": o["sample"] + f" ({o['spent_s']:.1f} s wall for the sample)",
               "legs_ms": {k: o[k] for k in ("fwd_ms", "bwd_ms", "decode_ms")}}

    if dist.rank == 0:
        clk = res["clocks"] or {}
        line = {
            "metric": METRIC, "value": step_fb, "unit": "ms", "n_gpus": dist.world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": res["step_ms"], "higher_is_better": False,
            "scaling": "strong" if args.shard == "heads" else "weak",
            "median": res["median"],  # per-step medians on rank 0 (value and the rest: means)
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded generator; states stand in for real model states)",
            "config": {"workload": f"{args.train} fwd+bwd (B={wt.B},H={wt.H},H_kv={wt.H_kv},"
                                   f"L={wt.L},d={wt.d}) + {DECODE} decode "
                                   f"(B={wd.B},H={wd.H},H_kv={wd.H_kv},N_k={wd.L},d={wd.d})",
                       "tau": TAU, "decode_splits": S,
                       "l2": "inputs larger than L2 (Q 268 MB, dO 268 MB, KV cache 2.1 GB)",
                       "parallelism": (f"tp{dist.world}: one problem, {wt.H_kv} KV heads and "
                                       f"{wt.H} query heads per GPU (head sharding, no "
                                       "collective on the data path)"
                                       if args.shard == "heads" else
                                       f"weak: {dist.world} independent problem(s), one per GPU")},
            "fwd_ms": res["fwd_ms"], "bwd_ms": res["bwd_ms"], "decode_us": res["decode_ms"] * 1e3,
            "tflops": {"executed": exec_tf, "dense_equivalent": deq_tf},
            "pct_bf16_peak": {"executed": exec_tf / peak, "bwd_kernel": bwd_tf / peak,
                              "peak_tflops": peak, "peak": peaks["source"] + " burst",
                              "executed_of_sustained": exec_tf / peak_sus,
                              "sustained_tflops": peak_sus},
            # tensor-pipe utilisation of the kernels at this workload, from an ncu capture
            # of the same kernel sources (None once a kernel has changed since)
            "ncu_tensor_pipe_pct": (None if not ncu else
                                    {k: v.get("tensor_pipe_pct") for k, v in
                                     ncu["kernels"].items()}),
            "retained": {"fwd_tiles": fret, "bwd_tiles": bret, "decode_tiles": dret,
                         "decode_v_tiles": vtiles / (wd.B * wd.H_kv * mala.n_tiles(wd.L)),
                         "fwd_slots_per_query": fret * (L + 128) / 2.0},
            # exponentials evaluated (one per score of a retained tile; Eq. (13)/(16) counts)
            "exp_count": {"fwd": 128 * 128 * round(fret * fl["legal_tiles"]),
                          "bwd": 128 * 128 * round(bret * fl["legal_tiles"]),
                          "dense": 128 * 128 * fl["legal_tiles"]},
            "decode_gbs": dec_gbs,
            "dense_tau0": {"fwd_ms": res0["fwd_ms"], "bwd_ms": res0["bwd_ms"],
                           "fwd_bwd_ms": dense_fb, "decode_us": res0["decode_ms"] * 1e3,
                           "tflops": dense_exec_tf, "pct_bf16_peak": dense_exec_tf / peak,
                           "pct_bf16_sustained": dense_exec_tf / peak_sus,
                           "decode_gbs": dec_gbs0},
            "speedup_vs_tau0": {"fwd_bwd": dense_fb / step_fb,
                                "decode": res0["decode_ms"] / res["decode_ms"]},
            "roofline": {"bound": "tensor", "kernel": "mala_bwd (main kernel + 2 small kernels)",
                         "achieved": bwd_tf, "peak": peak, "unit": "TFLOP/s",
                         "frac": bwd_tf / peak, "traffic": traffic,
                         "frac_of_sustained": bwd_tf / peak_sus,
                         "peak_source": peaks["source"] + " bf16 burst (per-call kernel time)"},
            "decode_roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": peaks["hbm_gbs"],
                                "unit": "GB/s", "frac": dec_gbs / peaks["hbm_gbs"]},
            "clocks": {"sm_mhz": clk.get("sm_mhz"), "sm_max_mhz": clk.get("sm_max_mhz"),
                       "reasons": clk.get("reasons", [])},
            "gpu_launches": KERNELS_PER_STEP * args.steps,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "skip_regime": skip,
            "prefill": prefill,
        }
        print(json.dumps(line), flush=True)


def profile_case(case: str):
    """Two rounds (warm-up, then the one to capture) of the three main kernels on
    mid-size inputs for an ncu capture: a few GB on the device, inputs larger than L2.
    case "headline": sink + band states, B=1, H=32, H_kv=8, L=8192 and the planted
    decode cache at N_k=32768; case "skip": previous-token states at L=8192 and the
    heavy-hitter cache at N_k=32768.  tau = 1."""
    from mass_adaptive_sparse_fwd_b200 import mala

    if case == "bench32k":
        # the bench's training workload itself: one warm-up round, then forward and
        # backward at tau = 1 and at tau = 0 once each (the launches an ncu capture of the
        # bench-shape counters selects: 4 main-kernel launches per round)
        wt = synth.WORKLOADS[TRAIN]
        tr = synth.make_training(wt)
        bf = lambda x: torch.from_numpy(x).cuda().to(torch.bfloat16)
        Q, K, V, dO = (bf(tr[k]) for k in ("Q", "K", "V", "dO"))
        for _ in range(2):
            for tau in (TAU, 0.0):
                O, LSE = mala.mala_fwd(Q, K, V, wt.scale, tau)
                dQ, dK, dV = mala.mala_bwd(Q, K, V, O, LSE, dO, wt.scale, tau)
            torch.cuda.synchronize()
        print(json.dumps({"profile_case": case, "O": float(O.float().abs().mean()),
                          "dQ": float(dQ.float().abs().mean())}), flush=True)
        return
    train, dec = (("sinkband32k", "decode128k") if case == "headline"
                  else ("prevtok32k", "heavy128k"))
    wt, wd = synth.WORKLOADS[train], synth.WORKLOADS[dec]
    tr = synth.make_training(wt, L=8192)
    dc = synth.make_decode(wd, Nk=32768)
    bf = lambda x: torch.from_numpy(x).cuda().to(torch.bfloat16)
    Q, K, V, dO = (bf(tr[k]) for k in ("Q", "K", "V", "dO"))
    q, Kc, Vc = (bf(dc[k]) for k in ("q", "K", "V"))
    for _ in range(2):
        O, LSE = mala.mala_fwd(Q, K, V, wt.scale, TAU)
        dQ, dK, dV = mala.mala_bwd(Q, K, V, O, LSE, dO, wt.scale, TAU)
        Od, _ = mala.mala_decode(q, Kc, Vc, wd.scale, TAU)
        torch.cuda.synchronize()
    print(json.dumps({"profile_case": case, "O": float(O.float().abs().mean()),
                      "dQ": float(dQ.float().abs().mean()),
                      "O_decode": float(Od.float().abs().mean())}), flush=True)


SWEEP_LENGTHS = (1024, 2048, 4096, 8192, 16384, 32768, 65536, 131072)


def run_sweep(args):
    """Operator latency and peak memory across sequence lengths (the page's operator
    benchmark, App. C.5 "Operator Latency and Memory Setup": batch 1, lengths 1K-128K,
    25 warm-up and 100 timed iterations, peak per-rank allocation).  The shape is one
    rank's share of a 64-query-head / 8-KV-head model under 8-way head sharding (H=8,
    H_kv=1, d=128; the sharded ranks run independent problems of this shape), on the
    sink + band states.  Each length is timed at tau = 1 and at tau = 0 (the same
    library's dense path); memory is the peak device allocation over the operator path
    (inputs, outputs, workspaces and the forward and backward calls).  Decode is timed on
    the same rank shape at batch 1: the last position's query heads against the L-token
    K/V cache, with its own peak allocation (cache, query, outputs, workspace)."""
    from mass_adaptive_sparse_fwd_b200 import mala

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    base = synth.WORKLOADS["sinkband128k"]
    lengths = [int(x) for x in args.sweep.split(",")] if args.sweep != "all" else SWEEP_LENGTHS
    stream = torch.cuda.current_stream(dev)
    rows = []
    for L in lengths:
        w = dataclasses.replace(base, name=f"sinkband_L{L}", L=L)
        tr = synth.make_training(w)
        for tau in (TAU, 0.0):
            torch.cuda.synchronize(dev)
            torch.cuda.empty_cache()
            torch.cuda.reset_peak_memory_stats(dev)
            base_bytes = torch.cuda.memory_allocated(dev)
            Q, K, V, dO = (torch.from_numpy(tr[k]).to(dev).to(torch.bfloat16)
                           for k in ("Q", "K", "V", "dO"))
            B, _, H, d = Q.shape
            Hkv = K.shape[2]
            in_bytes = sum(t.numel() * t.element_size() for t in (Q, K, V, dO))
            wsf = mala.alloc_workspace(mala.fwd_workspace_bytes(B, H, Hkv, L, d), dev)
            wsb = mala.alloc_workspace(mala.bwd_workspace_bytes(B, H, Hkv, L, d), dev)
            ws_bytes = wsf.numel() + wsb.numel()
            torch.cuda.synchronize(dev)
            # the conversion temporaries of the inputs are freed: start the peak here
            torch.cuda.reset_peak_memory_stats(dev)
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)]
                   for _ in range(args.sweep_iters)]
            for it in range(args.sweep_warmup + args.sweep_iters):
                ev = evs[it - args.sweep_warmup] if it >= args.sweep_warmup else None
                if ev:
                    ev[0].record(stream)
                O, LSE = mala.mala_fwd(Q, K, V, w.scale, tau, workspace=wsf)
                if ev:
                    ev[1].record(stream)
                dQ, dK, dV = mala.mala_bwd(Q, K, V, O, LSE, dO, w.scale, tau, workspace=wsb)
                if ev:
                    ev[2].record(stream)
                del O, LSE, dQ, dK, dV
            torch.cuda.synchronize(dev)
            for ws in (wsf, wsb):
                err = mala.read_device_error(ws)
                if err:
                    raise RuntimeError(f"device error word 0x{err:x}")
            peak = torch.cuda.max_memory_allocated(dev) - base_bytes
            # decode: one query per head (the last position) against the whole K/V cache;
            # its peak = the cache (already resident) plus what the decode path allocates
            torch.cuda.synchronize(dev)
            torch.cuda.reset_peak_memory_stats(dev)
            dec_start = torch.cuda.memory_allocated(dev)
            q = Q[:, L - 1].contiguous()
            S = mala.decode_num_splits(B, H, Hkv, L)
            wsd = mala.alloc_workspace(mala.decode_workspace_bytes(B, H, Hkv, L, d, 0, S), dev)
            dev_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)]
                      for _ in range(args.sweep_iters)]
            for it in range(args.sweep_warmup + args.sweep_iters):
                ev = dev_ev[it - args.sweep_warmup] if it >= args.sweep_warmup else None
                if ev:
                    ev[0].record(stream)
                Od, Ld = mala.mala_decode(q, K, V, w.scale, tau, num_splits=S, workspace=wsd)
                if ev:
                    ev[1].record(stream)
                del Od, Ld
            torch.cuda.synchronize(dev)
            if mala.read_device_error(wsd):
                raise RuntimeError("decode device error")
            sd = mala.get_stats(wsd)
            dec_us = [1e3 * e[0].elapsed_time(e[1]) for e in dev_ev]
            dec_peak = (torch.cuda.max_memory_allocated(dev) - dec_start +
                        (K.numel() + V.numel()) * 2)
            del wsd, q
            sf, sb = mala.get_stats(wsf), mala.get_stats(wsb)
            fr = sf["retained_tiles"] / max(sf["legal_tiles"], 1)
            br = sb["retained_tiles"] / max(sb["legal_tiles"], 1)
            fl = fwd_bwd_flops(w, fr, br)
            fwd = [e[0].elapsed_time(e[1]) for e in evs]
            bwd = [e[1].elapsed_time(e[2]) for e in evs]
            tot = [a + b for a, b in zip(fwd, bwd)]
            rows.append({
                "L": L, "tau": tau,
                "fwd_ms": statistics.mean(fwd), "bwd_ms": statistics.mean(bwd),
                "fwd_bwd_ms": statistics.mean(tot), "fwd_bwd_median_ms": statistics.median(tot),
                "executed_tflops": (fl["fwd_exec"] + fl["bwd_exec"]) / statistics.mean(tot) / 1e9,
                "dense_eq_tflops": (fl["fwd_dense_eq"] + fl["bwd_dense_eq"]) /
                                   statistics.mean(tot) / 1e9,
                "retained": {"fwd_tiles": fr, "bwd_tiles": br},
                "peak_mem_mb": peak / 2**20,
                "inputs_mb": in_bytes / 2**20,
                "workspace_mb": ws_bytes / 2**20,
                "operator_mem_mb": (peak - in_bytes) / 2**20,
                "decode": {"us": statistics.mean(dec_us), "median_us": statistics.median(dec_us),
                           "splits": S,
                           "v_tiles_retained": sd["v_tiles_loaded"] / max(sd["legal_tiles"] / H * Hkv, 1),
                           "peak_mem_mb": dec_peak / 2**20},
            })
            del Q, K, V, dO, wsf, wsb
    print(json.dumps({
        "sweep": "operator latency and memory (fwd+bwd)",
        "workload": "sink + band states, B=1, H=8, H_kv=1, d=128 (one rank of 8-way head "
                    "sharding of a 64/8-head model), bf16",
        "protocol": f"{args.sweep_warmup} warm-up + {args.sweep_iters} timed iterations per "
                    "(L, tau), CUDA events on the launching stream, L2 not flushed; peak = "
                    "max allocated over the operator path above the allocation before it",
        "rows": rows}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("mala", "reference"), default="mala")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-skip-regime", action="store_true")
    ap.add_argument("--shard", choices=("replicas", "heads"), default="replicas",
                    help="N>1: independent problems per GPU (weak scaling, default) or one "
                         "problem head-sharded across the GPUs (strong scaling)")
    ap.add_argument("--train", default=TRAIN, choices=("sinkband32k", "sinkband128k"),
                    help="training workload of the step (default: the 32K headline shape)")
    ap.add_argument("--profile-case", choices=("headline", "skip", "bench32k"),
                    help="run the kernels once on a mid-size case for an ncu capture and exit")
    ap.add_argument("--sweep", metavar="all|L1,L2,...",
                    help="operator latency and peak memory across sequence lengths (one GPU; "
                         "prints one JSON line and exits)")
    ap.add_argument("--sweep-warmup", type=int, default=25)
    ap.add_argument("--sweep-iters", type=int, default=100)
    args = ap.parse_args()
    if args.profile_case:
        profile_case(args.profile_case)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    dist = Dist()
    if args.impl == "reference":
        run_reference(args, dist)  # rank 0 only; no process group needed
        return
    dist.init("nccl")
    try:
        run_mala(args, dist)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
