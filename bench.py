#!/usr/bin/env python3
"""Decode-step throughput of the SSA (gist token) hot path on B200.

One step = one fused ``ssa_decode`` call over a batch of B sequences (all
query heads of one layer): gist scoring, top-k chunk selection, hybrid
attention over the unfolded context and the combination of split partials.
The default workload is the 128K-context one (B=4, 32/8 heads, d=64, bf16,
lengths uniform in [64K, 128K], C=128, g=8, top-32).

Prints ONE JSON line (rank 0):
  value        decode queries/s over all GPUs, inputs resident in HBM; steps
               are CUDA-graph replays of the fused kernel, timed with CUDA
               events on the launching stream, max over ranks; 4 input sets
               rotate so every step starts with the previous steps' >= 3x83 MB
               of other data in L2 (L2 is 126 MB)
  e2e          the same metric through the public call per step, with the
               query and lengths copied host->device (pinned) and the output
               and selection copied back inside the timed region
  roofline     HBM roofline of the fused kernel: algorithmic bytes per launch
               (gist K + unselected gist V + selected raw K/V + tail + q, out,
               selection, lengths) / average launch time, vs the measured
               copy bandwidth in MEASURED_PEAKS.json
  cpu_baseline the fp64 CPU oracle on the host, on a bounded sample

``--impl reference`` times the fp64 CPU oracle (the reference arm) instead.
Multi-GPU: one process per GPU (torchrun); each rank decodes its own batch
(weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gist_token_chunk_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "decode queries/s and achieved HBM GB/s (% of B200 peak) at 32K–512K context"
UNIT = "queries/s"
DEFAULT_CONFIG = "llama1b_128k_var"
NSETS = 4
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0  # B200 HBM3e as specified (DGX figure), for the spec-based fraction


def log(*a):
    print(*a, file=sys.stderr, flush=True)


VARIANTS = {"none": None, "selected_only": (1, 0), "head_union": (0, 1),
            "selected_union": (1, 1)}

# ------------------------------------------------------------ bytes model ---

def algorithmic_bytes(w, seq_lens) -> int:
    """Bytes one decode step must move, each read once: per (sequence, KV
    head) the gist keys of all complete chunks, the gist values of the
    unselected ones, the raw K/V of the selected chunks and of the tail
    (two-level: meta keys, unselected meta values, candidate gist keys,
    unselected candidate gist values, selected raw K/V, tail), plus q, the
    output, the selection and the lengths."""
    e = 2 if w.dtype == "bf16" else 4
    tot = 0
    for n in seq_lens:
        n = int(n)
        M = n // w.C
        T = n - M * w.C
        if not w.two_level:
            k = min(w.topk, M)
            rows = M * w.g + (M - k) * w.g + 2 * k * w.C + 2 * T
        else:
            S = M // w.J
            R = M - S * w.J
            ks = min(w.topk_super, S)
            Mc = ks * w.J + R
            kc = min(w.topk, Mc)
            rows = (S * w.gm + (S - ks) * w.gm + Mc * w.g + (Mc - kc) * w.g + 2 * kc * w.C
                    + 2 * T)
        tot += w.Hkv * rows * w.d * e
    sel_k = w.topk + (w.topk_super if w.two_level else 0)
    tot += w.B * w.Hq * w.d * e + w.B * w.Hq * w.d * 4 + w.B * w.Hkv * sel_k * 4 + w.B * 4
    return tot


# ------------------------------------------------------------ host cost ---

def cuda_runtime():
    """The CUDA runtime that torch loaded, through ctypes (copies and events
    for the end-to-end leg, at a microsecond per call)."""
    import ctypes

    names = ["libcudart.so.12", "libcudart.so"]
    try:
        import nvidia.cuda_runtime as ncr

        names.insert(0, os.path.join(list(ncr.__path__)[0], "lib", "libcudart.so.12"))
    except Exception:
        pass
    lib = None
    for n in names:
        try:
            lib = ctypes.CDLL(n)
            break
        except OSError:
            continue
    if lib is None:
        raise SystemExit("CUDA runtime library not found")
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.cudaMemcpyAsync.argtypes = [vp, vp, sz, ctypes.c_int, vp]
    lib.cudaEventRecord.argtypes = [vp, vp]
    lib.cudaStreamWaitEvent.argtypes = [vp, vp, ctypes.c_uint]
    lib.cudaEventCreateWithFlags.argtypes = [ctypes.POINTER(vp), ctypes.c_uint]
    for f in ("cudaMemcpyAsync", "cudaEventRecord", "cudaStreamWaitEvent",
              "cudaEventCreateWithFlags"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


def host_call_cost(ssa, w, x, out, sel, sup, ws, stream, calls: int = 200) -> dict:
    """Host microseconds one decode call costs: through the Python binding,
    and through the C ABI alone (ctypes with the arguments prepared once).
    Each call enqueues a real step; the stream is drained before and after."""
    import ctypes

    torch.cuda.synchronize()
    sp = stream.cuda_stream
    sh = ssa.shape_of(x["q"], x["k_raw"])
    if w.two_level:
        def bind():
            ssa.ssa_decode_h2(x["q"], x["k_raw"], x["v_raw"], x["k_gist"], x["v_gist"],
                              x["k_meta"], x["v_meta"], x["seq_lens"], w.C, w.g, w.J, w.gm,
                              w.topk_super, w.topk, out=out, sel_super=sup, sel_idx=sel, ws=ws,
                              stream=stream)
        cargs = (ctypes.byref(sh), x["q"].data_ptr(), x["k_raw"].data_ptr(), x["v_raw"].data_ptr(),
                 x["k_gist"].data_ptr(), x["v_gist"].data_ptr(), x["k_meta"].data_ptr(),
                 x["v_meta"].data_ptr(), x["seq_lens"].data_ptr(), w.C, w.g, w.J, w.gm,
                 w.topk_super, w.topk, out.data_ptr(), sup.data_ptr(), sel.data_ptr(),
                 ws.data_ptr(), ws.numel(), sp)
        cfn = ssa.lib.ssa_decode_h2
    else:
        def bind():
            ssa.ssa_decode(x["q"], x["k_raw"], x["v_raw"], x["k_gist"], x["v_gist"],
                           x["seq_lens"], w.C, w.g, w.topk, out=out, sel_idx=sel, ws=ws,
                           stream=stream)
        cargs = (ctypes.byref(sh), x["q"].data_ptr(), x["k_raw"].data_ptr(), x["v_raw"].data_ptr(),
                 x["k_gist"].data_ptr(), x["v_gist"].data_ptr(), x["seq_lens"].data_ptr(), w.C,
                 w.g, w.topk, out.data_ptr(), sel.data_ptr(), ws.data_ptr(), ws.numel(), sp)
        cfn = ssa.lib.ssa_decode
    if cfn(*cargs) != 0:
        raise SystemExit("host cost: the C ABI call failed: " + ssa.lib.ssa_last_error().decode())
    res = {}
    for name, fn in (("binding", bind), ("c_abi", lambda: cfn(*cargs))):
        fn()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(calls):
            fn()
        res[name] = 1e6 * (time.perf_counter() - t0) / calls
        torch.cuda.synchronize()
    return res


def variant_bytes(w, seq_lens, sel, context: int) -> int:
    """Bytes one variant step must move, each read once: per (sequence, KV
    head) the gist keys of all complete chunks, the gist values of the
    unselected chunks (context 0) or of the selected ones (context 1), the
    raw K/V of the selected chunks (k_u = the selection's size) and the tail;
    plus q, out, selection and lengths."""
    e = 2 if w.dtype == "bf16" else 4
    tot = 0
    for b, n in enumerate(seq_lens):
        n = int(n)
        M = n // w.C
        T = n - M * w.C
        for j in range(w.Hkv):
            ku = int((sel[b, j] >= 0).sum())
            gv = (M - ku) * w.g if context == 0 else ku * w.g
            tot += (M * w.g + gv + 2 * ku * w.C + 2 * T) * w.d * e
    tot += w.B * w.Hq * w.d * e + w.B * w.Hq * w.d * 4 + sel.size * 4 + w.B * 4
    return tot


def hier_bytes(w, seq_lens, sels, J: int, g_sum, topks) -> int:
    """Bytes of a t-level step, each read once: per (sequence, KV head) and
    level, the summary keys of every candidate (scored) and the summary
    values of the unkept ones; the raw K/V of the kept chunks; the tail."""
    e = 2 if w.dtype == "bf16" else 4
    t = len(topks)
    gl = [w.g] + list(g_sum)
    tot = 0
    for b, n in enumerate(seq_lens):
        n = int(n)
        U = [n // w.C]
        for _ in range(1, t):
            U.append(U[-1] // J)
        T = n - U[0] * w.C
        for j in range(w.Hkv):
            kept_above = 0
            rows = 2 * T
            for l in range(t - 1, -1, -1):
                nc = U[l] if l == t - 1 else kept_above * J + (U[l] - U[l + 1] * J)
                kept = int((sels[l][b, j] >= 0).sum())
                rows += nc * gl[l] + (nc - kept) * gl[l]
                if l == 0:
                    rows += 2 * kept * w.C
                kept_above = kept
            tot += rows * w.d * e
    tot += w.B * w.Hq * w.d * e + w.B * w.Hq * w.d * 4 + sum(s.size for s in sels) * 4 + w.B * 4
    return tot


# --------------------------------------------------------- multi-rank ---

def rank_seed(seed: int, s: int, rank: int) -> int:
    """Seed of input set `s` on rank `rank`: every rank decodes its own batch
    of independent sequences (weak scaling, no exchange between ranks)."""
    return seed + 7919 * s + 100003 * rank


def max_over_ranks(x: float, pg, device) -> float:
    """The maximum of `x` over all ranks (the slowest rank's time)."""
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- peaks ---

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# The files the decode kernels and their launches are compiled from (the
# prefill is a translation unit of its own and changes none of them).
DECODE_SOURCES = ("ssa_api.cpp", "ssa_device.cuh", "ssa_fused.cuh", "ssa_generic.cuh",
                  "ssa_internal.h", "ssa_kernels.cu", "ssa_pipe.cuh")


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gist_token_chunk_b200", "csrc")
    for f in sorted(DECODE_SOURCES):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(config: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(config)
    except Exception:
        return None
    if not rec or rec.get("source_hash") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------- clocks ---

class ClockSampler:
    """Samples SM clock and throttle reasons with NVML during a region."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.ok = False
        self.samples = []
        self.reasons = 0
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            # NVML numbers GPUs without CUDA_VISIBLE_DEVICES: find ours by
            # UUID (a string -- pynvml passes its argument as a C pointer)
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover
            log("clock sampling unavailable:", e)

    def _sample(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
        self.reasons |= int(r) & ~0x1

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            self._stop.wait(0.005)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()
            try:
                self._sample()
            except Exception:
                pass

    def summary(self):
        if not self.ok or not self.samples:
            return None
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": float(self.max_mhz),
                "reasons": [n for bit, n in self.REASONS.items() if self.reasons & bit],
                "samples": len(self.samples)}


# ------------------------------------------------------------- cpu oracle ---

def oracle_time(inp, w, min_seconds: float, max_reps: int = 1000, variant=None, hier=None):
    """Time the fp64 oracle on whole decode steps of `inp` (host tensors),
    under the same reading (variant) or levels (hier) as the GPU arm."""
    from oracle import ssa_oracle

    orc = ssa_oracle.default()
    args = [inp["q"], inp["k_raw"], inp["v_raw"], inp["k_gist"], inp["v_gist"]]
    if w.two_level:
        args += [inp["k_meta"], inp["v_meta"]]
    import numpy as _np

    args = [_np.ascontiguousarray(a.float().numpy()) for a in args]
    lens = inp["seq_lens"].numpy()
    if hier:
        ks = [_np.ascontiguousarray(x.float().numpy()) for x in inp["k_sum"]]
        vs = [_np.ascontiguousarray(x.float().numpy()) for x in inp["v_sum"]]

    def one():
        if hier:
            orc.decode_hier(*args, ks, vs, lens, C=w.C, g=w.g, J=hier[0], topks=hier[2])
        elif variant:
            orc.decode(*args, lens, C=w.C, g=w.g, topk=w.topk, context=variant[0],
                       select=variant[1])
        elif w.two_level:
            orc.decode_h2(*args, lens, C=w.C, g=w.g, J=w.J, gm=w.gm, topk_super=w.topk_super,
                          topk_chunk=w.topk)
        else:
            orc.decode(*args, lens, C=w.C, g=w.g, topk=w.topk)

    reps, t0 = 0, time.perf_counter()
    while True:
        one()
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            return reps, el


def oracle_cores(pairs: int) -> int:
    n = os.environ.get("OMP_NUM_THREADS")
    avail = int(n) if n else (len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity")
                              else os.cpu_count())
    return max(1, min(avail, pairs))


def run_config(w, world: int, nsets: int) -> dict:
    """The `config` of both arms' JSON lines (identical, so the two lines
    describe the same workload and measurement)."""
    return dict(config_of(w), global_batch=w.B * world,
                l2=f"inputs larger than L2: {nsets} input sets rotate, each step follows "
                   f"{nsets - 1} steps over other sets",
                timing="GPU arm: CUDA-graph replays of the decode step, CUDA events on the "
                       "launching stream, max over ranks; reference arm: wall clock around "
                       "whole-batch oracle calls",
                parallelism=f"dp{world} (independent sequences per GPU, no collective)")


def config_of(w) -> dict:
    cfg = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "n_max": w.n_max,
           "C": w.C, "g": w.g, "topk": w.topk}
    if w.seq_range:
        cfg["seq_lens"] = f"uniform[{w.seq_range[0]},{w.seq_range[1]}]"
    else:
        cfg["seq_lens"] = list(w.seq_lens)
    if w.two_level:
        cfg.update({"J": w.J, "gm": w.gm, "topk_super": w.topk_super})
    return cfg


# -------------------------------------------------------- reference arm ---

def run_reference(args):
    """The reference arm: the fp64 CPU oracle, as it stands, on the host
    cores.  A step is one oracle call over a sample of the batch's sequences
    (all their KV heads; OpenMP over the (sequence, KV head) pairs on every
    core): the whole batch unless (steps + warmup) whole-batch calls would
    exceed the time budget, then the fewest leading sequences (at least one)
    that fit it."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    w = WORKLOADS[args.config]
    inp = make_inputs(w, seed=args.seed, device="cpu")
    from oracle import ssa_oracle

    orc = ssa_oracle.default()
    host = {k: np.ascontiguousarray(v.float().numpy()) for k, v in inp.items()
            if k not in ("seq_lens", "planted_idx")}
    lens = inp["seq_lens"].numpy()

    def call(nseq):
        sl = {k: v[:nseq] for k, v in host.items()}
        if w.two_level:
            orc.decode_h2(sl["q"], sl["k_raw"], sl["v_raw"], sl["k_gist"], sl["v_gist"],
                          sl["k_meta"], sl["v_meta"], lens[:nseq], C=w.C, g=w.g, J=w.J,
                          gm=w.gm, topk_super=w.topk_super, topk_chunk=w.topk)
        else:
            orc.decode(sl["q"], sl["k_raw"], sl["v_raw"], sl["k_gist"], sl["v_gist"],
                       lens[:nseq], C=w.C, g=w.g, topk=w.topk)

    t0 = time.perf_counter()
    call(w.B)  # one whole-batch call sizes the sample
    t_batch = time.perf_counter() - t0
    calls = args.steps + args.warmup
    nseq = w.B
    if calls * t_batch > args.ref_budget:
        nseq = max(1, int(w.B * args.ref_budget / (calls * t_batch)))
    for _ in range(args.warmup):
        call(nseq)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        call(nseq)
    el = time.perf_counter() - t0
    value = args.steps * nseq / el
    cores = oracle_cores(nseq * w.Hkv)
    if nseq == w.B:
        sample = f"each step = one oracle call over the whole batch ({w.B} sequences, all KV heads)"
    else:
        sample = (f"each step = one oracle call over the first {nseq} of the batch's {w.B} "
                  "sequences (all KV heads)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": run_config(w, world, args.sets),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------- prefill ---

# Prefill of one attention layer under the gist mask (Llama-3.2-1B heads).
PREFILL = {"workload": "prefill_llama1b_32k", "B": 1, "Hq": 32, "Hkv": 8, "d": 64,
           "n": 32768, "C": 128, "g": 8}


def prefill_visible_pairs(n: int, C: int, g: int) -> int:
    """(query, key) pairs the gist mask keeps for one sequence and head: raw
    row i of chunk m sees m g gists and i - m C + 1 raw tokens; gist (m, t)
    sees m g + t + 1 gists and the C raw tokens of its chunk."""
    M = n // C
    pairs = 0
    for m in range(M + 1):
        rows = min(C, n - m * C)
        if rows <= 0:
            break
        pairs += rows * m * g + rows * (rows + 1) // 2
    pairs += sum(M_ * g * g + g * (g + 1) // 2 + g * C for M_ in range(M))
    return pairs


def run_prefill(args):
    """Times ssa_prefill (one layer, plan built once outside the timed
    region) with CUDA events per step, L2 flushed between steps; prints one
    JSON line.  The dense causal SDPA over the same interleaved length is
    timed beside it for context."""
    from gist_token_chunk_b200 import ssa

    P = PREFILL
    B, Hq, Hkv, d, n, C, g = (P[k] for k in ("B", "Hq", "Hkv", "d", "n", "C", "g"))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    gen = torch.Generator(device=dev).manual_seed(args.seed)
    M = n // C
    f = lambda *sh: torch.randn(*sh, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    x = [f(B, Hq, n, d), f(B, Hq, M, g, d), f(B, Hkv, n, d), f(B, Hkv, M, g, d), f(B, Hkv, n, d),
         f(B, Hkv, M, g, d)]
    t0 = time.perf_counter()
    tiles, entries = ssa.ssa_prefill_plan([n] * B, n, C, g)
    plan_ms = (time.perf_counter() - t0) * 1e3
    tiles_d, entries_d = tiles.to(dev), entries.to(dev)
    o_raw = torch.empty((B, Hq, n, d), dtype=torch.float32, device=dev)
    o_gist = torch.empty((B, Hq, M, g, d), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        ssa.ssa_prefill(*x, C, g, tiles_d, entries_d, o_raw, o_gist, stream=stream)

    def timed(fn, steps):
        total = 0.0
        for _ in range(steps):
            flush.fill_(1)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            total += e0.elapsed_time(e1)
        return total / steps

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert ssa.ssa_prefill_get_status() == 0
    clocks = ClockSampler(0)
    with clocks:
        ms = timed(step, args.steps)
    T = B * (n + M * g)
    pairs = B * Hq * prefill_visible_pairs(n, C, g)
    flops = 4.0 * d * pairs                      # q.k and p.v per kept pair
    blocks = int(entries.numel()) * Hq           # (tile, block) pairs run per head
    exec_flops = blocks * SSA_BLOCK * SSA_BLOCK * (2.0 * d + 4.0 * d)  # p.v as a bf16 pair
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            peak, peak_kind = float(json.load(fh)["bf16_tflops"]), "measured"
    except Exception:
        peak, peak_kind = 1590.0, "fallback"
    achieved = flops / (ms * 1e-3) / 1e12

    # dense causal attention over the same interleaved length (context only),
    # on the fused SDPA kernels only: the unfused one would hold the whole
    # score matrix (tens of GB at this length)
    dense_ms = None
    try:
        from torch.nn.attention import SDPBackend, sdpa_kernel

        qd = torch.randn(B, Hq, n + M * g, d, device=dev, dtype=torch.bfloat16)
        kd = torch.randn(B, Hq, n + M * g, d, device=dev, dtype=torch.bfloat16)
        vd = torch.randn(B, Hq, n + M * g, d, device=dev, dtype=torch.bfloat16)
        fused = [SDPBackend.FLASH_ATTENTION, SDPBackend.CUDNN_ATTENTION,
                 SDPBackend.EFFICIENT_ATTENTION]

        def sdpa():
            with sdpa_kernel(fused):
                torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, is_causal=True)

        for _ in range(3):
            sdpa()
        dense_ms = timed(sdpa, max(3, min(args.steps, 20)))
        del qd, kd, vd
    except Exception as e:  # no fused SDPA kernel for these sizes
        log("dense SDPA not timed:", e)

    line = {
        "metric": "prefill tokens/s of one attention layer under the gist mask",
        "value": T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": P["workload"], "B": B, "Hq": Hq, "Hkv": Hkv, "d": d, "n": n,
                   "C": C, "g": g, "l2": "flushed between steps (256 MB write)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "peak_kind": f"bf16 dense, burst, {peak_kind}",
                     "flops": "4 d per kept (query, key) pair per head",
                     "executed_tflops": exec_flops / (ms * 1e-3) / 1e12},
        "plan": {"tiles": int(tiles.shape[0]), "entries": int(entries.numel()),
                 "host_ms": plan_ms, "kept_pairs_per_head": pairs // (B * Hq),
                 "block_pairs_per_head": int(entries.numel()) * SSA_BLOCK * SSA_BLOCK},
        "dense_causal_sdpa_ms": dense_ms,
        "clocks": clocks.summary(),
        "gpu_launches": args.steps,
    }
    print(json.dumps(line), flush=True)


SSA_BLOCK = 64


# ------------------------------------------------------------- GPU arm ---

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", default=DEFAULT_CONFIG, choices=sorted(WORKLOADS))
    ap.add_argument("--seed", type=int, default=1003)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-budget", type=float, default=150.0,
                    help="reference arm: seconds its warm-up and timed calls may take")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=1000,
                    help="steps of the end-to-end measurement (0: skip it)")
    ap.add_argument("--sets", type=int, default=NSETS,
                    help="rotating input sets (fewer only for profiling runs)")
    ap.add_argument("--variant", default="none", choices=sorted(VARIANTS),
                    help="another context / selection reading (ssa_decode_variant)")
    ap.add_argument("--levels", default="",
                    help="coarse-to-fine over t levels (ssa_decode_hier): 'J:g2,..,gt:k1,..,kt'")
    ap.add_argument("--prefill", action="store_true",
                    help="time the block-sparse prefill of one layer instead (1 GPU)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.prefill:
        return run_prefill(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    from gist_token_chunk_b200 import ssa

    w = WORKLOADS[args.config]
    # each rank decodes its own batch (independent sequences)
    NS = max(1, args.sets)
    sets = [make_inputs(w, seed=rank_seed(args.seed, s, rank), device=dev)
            for s in range(NS)]
    for s in sets:
        s.pop("planted_idx", None)
    shape = ssa.shape_of(sets[0]["q"], sets[0]["k_raw"])
    variant = VARIANTS[args.variant]
    hier = None
    if args.levels:
        if w.two_level or variant:
            ap.error("--levels takes a single-level workload and no --variant")
        J_s, g_s, k_s = args.levels.split(":")
        hier = (int(J_s), [int(x) for x in g_s.split(",") if x], [int(x) for x in k_s.split(",")])
        if len(hier[1]) != len(hier[2]) - 1:
            ap.error("--levels: t-1 summary sizes and t top-k's")
    if variant and w.two_level:
        ap.error("--variant takes a single-level workload")
    if hier:
        nbytes = ssa.ssa_workspace_size_hier(shape, w.C, w.g, hier[0], hier[1], hier[2])
    elif variant:
        nbytes = ssa.ssa_workspace_size_variant(shape, w.C, w.g, w.topk, *variant)
    elif w.two_level:
        nbytes = ssa.ssa_workspace_size_h2(shape, w.C, w.g, w.J, w.gm, w.topk_super, w.topk)
    else:
        nbytes = ssa.ssa_workspace_size(shape, w.C, w.g, w.topk)
    ws = ssa.workspace(nbytes, device=dev)
    cap = w.topk * (w.G if variant and variant[1] else 1)
    outs = [torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=dev) for _ in range(NS)]
    sels = [torch.empty(w.B, w.Hkv, max(cap, 1), dtype=torch.int32, device=dev)
            for _ in range(NS)]
    sups = [torch.empty(w.B, w.Hkv, max(w.topk_super, 1), dtype=torch.int32, device=dev)
            for _ in range(NS)]
    if hier:
        from gist_token_chunk_b200.inputs import make_level_summaries

        for s_i, x in enumerate(sets):
            x["k_sum"], x["v_sum"] = make_level_summaries(
                w, hier[0], hier[1], seed=rank_seed(args.seed, s_i, rank) + 17, device=dev)
        hsels = [[torch.empty(w.B, w.Hkv, max(k, 1), dtype=torch.int32, device=dev)
                  for k in hier[2]] for _ in range(NS)]

    def decode_call(x, s, out, sel, stream):
        """One decode step of set s's inputs x through the public call."""
        if hier:
            ssa.ssa_decode_hier(x["q"], x["k_raw"], x["v_raw"], x["k_gist"], x["v_gist"],
                                x["seq_lens"], w.C, w.g, hier[0], x["k_sum"], x["v_sum"],
                                hier[2], out=out, sels=hsels[s], ws=ws, stream=stream)
        elif variant:
            ssa.ssa_decode_variant(x["q"], x["k_raw"], x["v_raw"], x["k_gist"], x["v_gist"],
                                   x["seq_lens"], w.C, w.g, w.topk, variant[0], variant[1],
                                   out=out, sel_idx=sel, ws=ws, stream=stream)
        elif w.two_level:
            ssa.ssa_decode_h2(x["q"], x["k_raw"], x["v_raw"], x["k_gist"], x["v_gist"],
                              x["k_meta"], x["v_meta"], x["seq_lens"], w.C, w.g, w.J, w.gm,
                              w.topk_super, w.topk, out=out, sel_super=sups[s], sel_idx=sel,
                              ws=ws, stream=stream)
        else:
            ssa.ssa_decode(x["q"], x["k_raw"], x["v_raw"], x["k_gist"], x["v_gist"],
                           x["seq_lens"], w.C, w.g, w.topk, out=out, sel_idx=sel, ws=ws,
                           stream=stream)

    def step(i, stream=None):
        s = i % NS
        decode_call(sets[s], s, outs[s], sels[s], stream)

    if hier:
        kernel_name = "ssa::gen hier_score, hier_topk (per level) and hier_attend kernels"
        launches_per_step = 2 * len(hier[2]) + 1
    elif variant and (ssa.ssa_decode_path(shape, w.C, w.g, w.topk) == ssa.SSA_PATH_PIPELINE
                      and w.G * w.topk <= 1024):
        # the variants run on the pipeline wherever ssa_decode does
        kernel_name = ("ssa::pipe::score_kernel + ssa::pipe::attend_kernel<true>" if variant[1]
                       else "ssa::pipe::score_kernel + ssa::pipe::attend_kernel<false>")
        launches_per_step = 2
    elif variant:
        kernel_name = ("ssa::gen head_score, head_topk, union and attend kernels" if variant[1]
                       else "ssa::gen score, top-k and attend kernels")
        launches_per_step = 4 if variant[1] else 3
    elif w.two_level:
        path, kernel_name, launches_per_step = None, "ssa::fused::fused_kernel<64>", 1
    else:
        path = ssa.ssa_decode_path(shape, w.C, w.g, w.topk)
        kernel_name, launches_per_step = {
            ssa.SSA_PATH_PIPELINE: ("ssa::pipe::score_kernel + ssa::pipe::attend_kernel<false>", 2),
            ssa.SSA_PATH_FUSED: (f"ssa::fused::fused_kernel<{w.d}>", 1),
        }.get(path, ("ssa::gen score, top-k and attend kernels", 3))

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for i in range(NS):
            step(i)  # eager first use (workspace control region, attributes)
    stream.synchronize()
    # graphs: a chunk of REP*NS steps and single steps for the remainder
    REP = 8
    g_chunk = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_chunk, stream=stream):
        for i in range(REP * NS):
            step(i, stream=stream)
    g_one = []
    for s in range(NS):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(s, stream=stream)
        g_one.append(g)
    assert ssa.ssa_get_device_status(stream) == 0

    def run_steps(k):
        done = 0
        while k - done >= REP * NS:
            g_chunk.replay()
            done += REP * NS
        while done < k:
            g_one[done % NS].replay()
            done += 1

    with torch.cuda.stream(stream):
        run_steps(args.warmup)
    stream.synchronize()
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    with sampler:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            run_steps(args.steps)
            ev1.record(stream)
        ev1.synchronize()
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(ev0.elapsed_time(ev1), pg, dev)
    status = ssa.ssa_get_device_status(stream)
    if status != 0:
        raise SystemExit(f"device status {status} after the timed region")

    queries = args.steps * w.B * world
    value = queries / (ms / 1e3)
    ms_step = ms / args.steps
    # bytes model, averaged over the rotating sets
    if hier:
        bytes_per_launch = statistics.mean(
            hier_bytes(w, sets[s]["seq_lens"].cpu().tolist(), [x.cpu().numpy() for x in hsels[s]],
                       *hier) for s in range(NS))
    elif variant:
        bytes_per_launch = statistics.mean(
            variant_bytes(w, sets[s]["seq_lens"].cpu().tolist(), sels[s].cpu().numpy(), variant[0])
            for s in range(NS))
    else:
        bytes_per_launch = statistics.mean(
            algorithmic_bytes(w, s["seq_lens"].cpu().tolist()) for s in sets)
    per_launch_s = (ms / 1e3) / args.steps
    achieved = bytes_per_launch / per_launch_s / 1e9
    peak, peak_src = hbm_peak()

    # ---- end to end through the public call, host buffers
    ek = max(NS, min(args.steps, args.e2e_steps)) if args.e2e_steps > 0 else 0
    # one pinned staging buffer per direction and set: the query and the
    # lengths go up in one copy, the output and the selection come back in one
    def packed(tensors, device):
        sizes = [(t.numel() * t.element_size() + 15) // 16 * 16 for t in tensors]
        buf = torch.empty(sum(sizes), dtype=torch.uint8, device=device)
        if device == "cpu":
            buf = buf.pin_memory()
        views, off = [], 0
        for t, n in zip(tensors, sizes):
            nb = t.numel() * t.element_size()
            views.append(buf[off:off + nb].view(t.dtype).view(t.shape))
            off += n
        return buf, views

    up_host, up_dev, down_host, down_dev = [], [], [], []
    for s in range(NS):
        hb, (qh, lh) = packed([sets[s]["q"], sets[s]["seq_lens"]], "cpu")
        qh.copy_(sets[s]["q"].cpu())
        lh.copy_(sets[s]["seq_lens"].cpu())
        up_host.append(hb)
        up_dev.append(packed([sets[s]["q"], sets[s]["seq_lens"]], dev))
        down_dev.append(packed([outs[s], sels[s]], dev))
        down_host.append(packed([outs[s], sels[s]], "cpu")[0])

    # Copies run on their own streams so that step i+1's upload and step i's
    # download overlap the decode kernels; events keep each set's buffers
    # ordered: upload -> decode -> download -> the set's next upload/decode.
    # The copies and the event operations go straight to the CUDA runtime
    # (ctypes), a microsecond each, so that the host issues a step faster
    # than the device runs it; the decode itself is the public call.
    cr = cuda_runtime()
    up_stream = torch.cuda.Stream(device=dev)
    down_stream = torch.cuda.Stream(device=dev)
    sh_main, sh_up, sh_down = stream.cuda_stream, up_stream.cuda_stream, down_stream.cuda_stream

    def new_event():
        ev = ctypes.c_void_p()
        if cr.cudaEventCreateWithFlags(ctypes.byref(ev), 2) != 0:  # cudaEventDisableTiming
            raise SystemExit("cudaEventCreateWithFlags failed")
        return ev

    up_done = [new_event() for _ in range(NS)]
    dec_done = [new_event() for _ in range(NS)]
    down_done = [new_event() for _ in range(NS)]
    for s_i in range(NS):
        cr.cudaEventRecord(dec_done[s_i], sh_main)
        cr.cudaEventRecord(down_done[s_i], sh_main)
    e2e_x, e2e_bufs = [], []
    for s_i in range(NS):
        dbuf, (q_dev, len_dev) = up_dev[s_i]
        obuf, (o_dev, s_dev) = down_dev[s_i]
        e2e_x.append(dict(sets[s_i], q=q_dev, seq_lens=len_dev))
        e2e_bufs.append((dbuf.data_ptr(), up_host[s_i].data_ptr(), dbuf.numel(), o_dev, s_dev,
                         down_host[s_i].data_ptr(), obuf.data_ptr(), obuf.numel()))

    def e2e_step(i):
        s_i = i % NS
        dptr, hptr, nup, o_dev, s_dev, hout, optr, ndown = e2e_bufs[s_i]
        cr.cudaStreamWaitEvent(sh_up, dec_done[s_i], 0)      # the set's last decode read q
        cr.cudaMemcpyAsync(dptr, hptr, nup, 1, sh_up)        # host to device
        cr.cudaEventRecord(up_done[s_i], sh_up)
        cr.cudaStreamWaitEvent(sh_main, up_done[s_i], 0)
        cr.cudaStreamWaitEvent(sh_main, down_done[s_i], 0)   # its last output was read back
        decode_call(e2e_x[s_i], s_i, o_dev, s_dev, stream)
        cr.cudaEventRecord(dec_done[s_i], sh_main)
        cr.cudaStreamWaitEvent(sh_down, dec_done[s_i], 0)
        cr.cudaMemcpyAsync(hout, optr, ndown, 2, sh_down)    # device to host
        cr.cudaEventRecord(down_done[s_i], sh_down)

    e2e_value = None
    if ek > 0:
        with torch.cuda.stream(stream):
            for i in range(NS):
                e2e_step(i)
        torch.cuda.synchronize(dev)
        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            up_stream.wait_event(ev0)
            h0 = time.perf_counter()
            for i in range(ek):
                e2e_step(i)
            host_issue_s = time.perf_counter() - h0
            for s_i in range(NS):
                cr.cudaStreamWaitEvent(sh_main, down_done[s_i], 0)
            ev1.record(stream)
        ev1.synchronize()
        e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), pg, dev)
        e2e_value = ek * w.B * world / (e2e_ms / 1e3)
        host_cost = (None if hier or variant else
                     host_call_cost(ssa, w, sets[0], outs[0], sels[0], sups[0], ws, stream))
    h2d = sets[0]["q"].numel() * sets[0]["q"].element_size() + sets[0]["seq_lens"].numel() * 4
    d2h = outs[0].numel() * 4 + sels[0].numel() * 4

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": dict(run_config(w, world, NS),
                       **({"reading": args.variant} if variant else {}),
                       **({"levels": args.levels} if hier else {})),
        "hbm_gbs": achieved, "hbm_frac_of_peak": achieved / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": f"{peak_src} copy bandwidth",
                     "spec_peak": SPEC_HBM_GBS, "frac_of_spec": achieved / SPEC_HBM_GBS,
                     "algorithmic_bytes_per_launch": int(bytes_per_launch),
                     "traffic": profiled_traffic(args.config),
                     "kernel": kernel_name,
                     "per": "decode step (every kernel of the step; their launches overlap)"},
        "gpu_launches": args.steps * launches_per_step,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": ek,
                "host_issue_us_per_step": (1e6 * host_issue_s / ek) if ek > 0 else None,
                "host_us_per_call": host_cost if ek > 0 else None,
                "path": "the step's call per step (Python binding -> C ABI); query and lengths "
                        "up in one pinned copy, output and selection back in one, each on its "
                        "own stream so copies overlap the neighbouring steps' kernels"},
    }
    clk = sampler.summary()
    if clk is not None:
        line["clocks"] = clk

    # ---- CPU baseline: the oracle on the host (rank 0, N = 1 only)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        host = {k: ([x.cpu() for x in v] if isinstance(v, list) else v.cpu())
                for k, v in sets[0].items()}
        reps, el = oracle_time(host, w, args.cpu_seconds, variant=variant, hier=hier)
        line["cpu_baseline"] = {
            "value": reps * w.B / el, "unit": UNIT, "cores": oracle_cores(w.B * w.Hkv),
            "kind": "oracle",
            "sample": f"{reps} whole decode step(s) (B={w.B} sequences) of input set 0, "
                      f"{el:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg:
        del g_chunk, g_one
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
