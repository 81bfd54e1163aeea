#!/usr/bin/env python
"""Benchmark of the MTFM hybrid masked-attention hot path on B200.

One step = one pass of the whole hot path over one jagged batch of the
production-shape workload "hybrid pair": 32 users, L_H ~ U[256,1024],
L_R ~ U[32,256] (sorted timestamps), L_T ~ U[16,128]; Hq 8 / Hkv 2, head_dim 64:
    pack (metadata + work lists) -> Full-layer attention -> Full gate (GLN)
    -> Target-layer attention -> Target gate.
Inputs are resident in HBM, rotated over several copies so that no step reads
data left in L2 by the previous one.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mtfm|reference]

Prints one JSON line (rank 0).  ``value`` = unmasked attention TFLOP/s of the
whole step (4 * head_dim * Hq FLOPs per visible query/key pair, both layers),
summed over ranks and divided by the slowest rank's time.  Multi-GPU runs are
replicas: each rank packs and runs its own batch of users (no collective on the
data path), so scaling is weak.

``--impl reference`` times the fp64 CPU oracle on the host cores instead (the
only other place this script runs oracle code, besides the cpu_baseline leg).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import mtfm_synth as syn  # noqa: E402

METRIC = "masked-attn TFLOP/s (unmasked) & user-samples/s per layer; % BF16/HBM roofline"
WORKLOAD = ("hybrid pair: 32 users jagged, L_H~U[256,1024], L_R~U[32,256] sorted ts, "
            "L_T~U[16,128] over 3 scenarios; Hq 8 / Hkv 2, head_dim 64; pack + Full fwd + Target fwd "
            "(attention + GLN gate)")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = ["hybrid_masked_attention_b200/csrc/attn_tc.cu",
                  "hybrid_masked_attention_b200/csrc/sm100.cuh",
                  "hybrid_masked_attention_b200/csrc/mma_util.cuh",
                  "hybrid_masked_attention_b200/csrc/mtfm_internal.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_full_fwd_pair.md")


# ----------------------------------------------------------------------------- accounting

def visible_pairs(b: syn.JaggedBatch, target: bool) -> int:
    """Number of visible (query, key) pairs: H rows see L_H keys, R row a sees L_H + a + 1,
    a T row sees L_H + #{R : ts < exposure} keys plus its sibling block (itself, or the
    4 sub-tokens of its target in V2)."""
    ro = np.concatenate([[0], np.cumsum(b.L_R)])
    to = np.concatenate([[0], np.cumsum(b.L_T)])
    total = 0
    for u in range(b.B):
        LH, LR, LT = int(b.L_H[u]), int(b.L_R[u]), int(b.L_T[u])
        ts = b.r_ts[ro[u]:ro[u + 1]]
        ex = b.t_exp[to[u]:to[u + 1]]
        k = np.searchsorted(ts, ex, side="left") if LT else np.zeros(0)
        t_pairs = int(LT * LH + k.sum() + LT * b.v2_subtokens)
        if target:
            total += t_pairs
        else:
            total += LH * LH + LR * LH + LR * (LR + 1) // 2 + t_pairs
    return total


def attn_flops(b, heads, target) -> float:
    return 4.0 * heads.dh * heads.hq * visible_pairs(b, target)


def target_attn_bytes(b, heads) -> float:
    """Algorithmic bytes of Target attention: K, V of every row (bf16), Q_T (bf16), A_T (fp32)."""
    return b.total_tokens * 2 * heads.dkv * 2 + b.total_t * heads.dq * (2 + 4)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per launch of the Full attention kernel from the committed ncu summary,
    or None when the kernel source changed since the capture."""
    try:
        text = open(TRAFFIC_FILE).read()
    except OSError:
        return None
    sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", text)
    val = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    if not sha or not val or sha.group(1) != kernel_source_sha():
        return None
    return float(val.group(1))


# ----------------------------------------------------------------------------- ranks

def rank_batch_seed(rank: int) -> int:
    """Seed of rank `rank`'s batch: every rank packs and runs users of its own (weak scaling,
    no data-path collective)."""
    return 1001 + 7919 * rank


def reduce_over_ranks(ms: float, work, device):
    """(max over ranks of `ms`, per-entry sum over ranks of `work`); the identity on one rank.
    Every rank must call it, in the same order (two all-reduces on the process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms), [float(x) for x in work]
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    w = torch.tensor([float(x) for x in work], dtype=torch.float64, device=device)
    dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return float(t[0]), [float(x) for x in w]


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled while the timed region runs.

    A thread polls NVML every `interval_ms`; it is created (and NVML initialised) before the timed
    region, and `begin()` / `stop()` bracket the samples that count.  Without NVML it falls back to
    an `nvidia-smi --query-gpu ... -lms` subprocess."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits (nvml.h)
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device, interval_ms: int = 20):
        import threading
        self.samples, self.t_begin, self.proc, self.nvml = [], None, None, None
        self.interval = interval_ms / 1000.0
        self.stop_flag = threading.Event()
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            try:
                uuid = str(torch.cuda.get_device_properties(device).uuid)
                h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                h = pynvml.nvmlDeviceGetHandleByIndex(int(getattr(device, "index", device) or 0))
            self.nvml, self.handle = pynvml, h
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()
        except Exception:
            self.nvml = None
            self._start_smi(int(getattr(device, "index", device) or 0), max(50, interval_ms))

    def _poll(self):
        nv, h = self.nvml, self.handle
        while not self.stop_flag.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                mask = int(nv.nvmlDeviceGetCurrentClocksEventReasons(h))
                self.samples.append((time.monotonic(), mhz, mask))
            except Exception:
                pass
            self.stop_flag.wait(self.interval)

    def _start_smi(self, index, interval_ms):
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms={interval_ms}", f"-i={index}"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def begin(self):
        self.t_begin = time.monotonic()

    def stop(self):
        if self.nvml is not None:
            t_end = time.monotonic()
            self.stop_flag.set()
            self.thread.join(timeout=2)
            t0 = self.t_begin if self.t_begin is not None else 0.0
            win = [s for s in self.samples if t0 <= s[0] <= t_end] or self.samples[-1:]
            if not win:
                return None
            reasons = sorted(n for n, bit in self.REASON_BITS.items() if any(m & bit for _, _, m in win))
            return {"sm_mhz": statistics.median(m for _, m, _ in win), "sm_max_mhz": self.max_mhz,
                    "reasons": reasons, "samples": len(win), "source": "nvml"}
        if self.proc is None:
            return None
        time.sleep(0.06)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [l.strip().split(",") for l in self.out.read().splitlines() if l.strip()]
        os.unlink(self.out.name)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi"}


# ----------------------------------------------------------------------------- GPU arm

def run_mtfm(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import hybrid_masked_attention_b200 as M

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    heads = syn.PAIR_HEADS
    b = syn.pair_batch(args.users, seed=rank_batch_seed(rank))
    cfg = M.Config(b.B, b.total_tokens, b.total_r, b.total_t, heads.hq, heads.hkv, heads.dh)
    to_dev = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dtype=dt)).to(dev)
    bf = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    lens = (to_dev(b.L_H, np.int32), to_dev(b.L_R, np.int32), to_dev(b.L_T, np.int32),
            to_dev(b.r_ts, np.int64), to_dev(b.t_exp, np.int64))
    sets = []
    for r in range(args.sets):
        fi = syn.layer_inputs(b, heads, target=False, seed=11 + r)
        ti = syn.layer_inputs(b, heads, target=True, seed=111 + r)
        sets.append(dict(q=bf(fi.q), k=bf(fi.k), v=bf(fi.v), u=bf(fi.u),
                         g=to_dev(fi.gamma, np.float32), bt=to_dev(fi.beta, np.float32),
                         tq=bf(ti.q), tk=bf(ti.k), tv=bf(ti.v), tu=bf(ti.u),
                         tg=to_dev(ti.gamma, np.float32), tbt=to_dev(ti.beta, np.float32)))
    meta = M.alloc_meta(cfg, dev)
    f32 = dict(dtype=torch.float32, device=dev)
    A_f = torch.empty(b.total_tokens, heads.dq, **f32)
    Y_f = torch.empty(b.total_tokens, heads.dq, **f32)
    S_f = torch.empty(b.total_tokens, 2, **f32)
    A_t = torch.empty(b.total_t, heads.dq, **f32)
    Y_t = torch.empty(b.total_t, heads.dq, **f32)
    S_t = torch.empty(b.total_t, 2, **f32)
    # graphs cannot be captured on the legacy default stream: every launch goes to `stream`
    stream = torch.cuda.Stream(dev)
    launches_per_step = 7   # pack (2 kernels), Full attention, Full gate, Target clear, Target attention, Target gate

    def step(i, record=None, around_full=None, around_tgt=None, around_pack=None):
        s = sets[i % len(sets)]
        e = record
        if e: e[0].record(stream)
        if around_pack: around_pack[0].record(stream)
        M.pack(cfg, *lens, meta, stream)
        if around_pack: around_pack[1].record(stream)
        if e: e[1].record(stream)
        if around_full: around_full[0].record(stream)
        M.attn_full(cfg, meta, s["q"], s["k"], s["v"], A_f, stream)
        if around_full: around_full[1].record(stream)
        if e: e[2].record(stream)
        M.gate_fwd(cfg, meta, False, A_f, s["u"], s["g"], s["bt"], Y_f, S_f, stream)
        if e: e[3].record(stream)
        if around_tgt: around_tgt[0].record(stream)
        M.attn_target(cfg, meta, s["tq"], s["tk"], s["tv"], A_t, stream)
        if around_tgt: around_tgt[1].record(stream)
        if e: e[4].record(stream)
        M.gate_fwd(cfg, meta, True, A_t, s["tu"], s["tg"], s["tbt"], Y_t, S_t, stream)
        if e: e[5].record(stream)

    with torch.cuda.stream(stream):
        # correctness gate before timing: the metadata must be valid
        step(0)
        M.pack_check(meta, stream)
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize(dev)
    # The timed steps replay CUDA graphs of the step's launches (the 7 kernels: 2 pack, Full
    # attention, gate, the Target layer's conditional accumulator clear, attention, gate): one graph runs a step on each resident input set in turn;
    # its instrumented twin adds two event-record nodes around every Full attention launch
    # and is replayed last, so the kernel's duration is measured inside the timed region
    # without paying for event nodes in every step.  K = nset * reps + rem steps: the last
    # of the reps replays the twin, the rem steps replay one-step graphs.
    nset = len(sets)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        return g

    mk = lambda: [(torch.cuda.Event(enable_timing=True, external=True),
                   torch.cuda.Event(enable_timing=True, external=True)) for _ in range(nset)]
    full_ev, tgt_ev, pack_ev = mk(), mk(), mk()
    g_all = capture(lambda: [step(r) for r in range(nset)])
    g_ev = capture(lambda: [step(r, around_full=full_ev[r], around_tgt=tgt_ev[r], around_pack=pack_ev[r])
                            for r in range(nset)])
    singles = [capture(lambda r=r: step(r)) for r in range(nset)]
    singles_ev = [capture(lambda r=r: step(r, around_full=full_ev[r], around_tgt=tgt_ev[r], around_pack=pack_ev[r]))
                  for r in range(nset)]
    reps, rem = divmod(args.steps, nset)
    with torch.cuda.stream(stream):
        for _ in range(max(1, 3 // nset + 1)):
            g_all.replay()
    torch.cuda.synchronize(dev)
    M.pack_check(meta, stream)
    sampler = ClockSampler(dev) if rank == 0 else None
    # The K-step region is timed `repeats` times (each bracketed by a barrier and a
    # synchronize on both sides); the value is the median region, the spread is reported.
    region_ms, full_runs, tgt_runs, pack_runs = [], [], [], []
    if sampler:
        sampler.begin()
    for _ in range(max(1, args.repeats)):
        if world > 1:
            dist.barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            t0.record(stream)
            for i in range(reps):
                (g_ev if i == reps - 1 else g_all).replay()
            for r in range(rem):
                (singles_ev[r] if reps == 0 else singles[r]).replay()
            t1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        region_ms.append(t0.elapsed_time(t1))
        n_timed = nset if reps > 0 else rem
        full_runs += [a.elapsed_time(z) for a, z in full_ev[:n_timed]]
        tgt_runs += [a.elapsed_time(z) for a, z in tgt_ev[:n_timed]]
        pack_runs += [a.elapsed_time(z) for a, z in pack_ev[:n_timed]]
    clocks = sampler.stop() if sampler else None
    ms_total = statistics.median(region_ms)
    full_ms = statistics.median(full_runs)
    tgt_ms = statistics.median(tgt_runs)
    pack_ms = statistics.median(pack_runs)
    M.pack_check(meta, stream)

    # Per-part times from a separate eager pass with an event between launches (the events
    # themselves add a few microseconds per step, so the parts sum to more than a graph step).
    n_parts = max(1, min(args.steps, 500))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(n_parts)]
    with torch.cuda.stream(stream):
        for i in range(n_parts):
            step(i, ev[i])
    torch.cuda.synchronize(dev)

    def avg(a, z):
        return sum(ev[i][a].elapsed_time(ev[i][z]) for i in range(n_parts)) / n_parts

    ms_parts = {"pack": avg(0, 1), "full_attn": avg(1, 2), "full_gate": avg(2, 3),
                "target_attn": avg(3, 4), "target_gate": avg(4, 5)}
    del g_all, g_ev, singles, singles_ev
    fl_full = attn_flops(b, heads, False)
    fl_tgt = attn_flops(b, heads, True)
    flops_step = fl_full + fl_tgt

    # aggregate over ranks: time = max, work = sum
    ms_max, (flops_all, users_all) = reduce_over_ranks(ms_total, [flops_step, float(b.B)], dev)
    ms_per_step = ms_max / args.steps
    value = flops_all / (ms_per_step * 1e-3) / 1e12

    # end-to-end through the public API with host buffers
    e2e = run_e2e(args, M, cfg, b, heads, dev, stream, world)

    result = None
    if rank == 0:
        peaks, src = load_peaks()
        peak_tf = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
        full_tf = fl_full / (full_ms * 1e-3) / 1e12
        tgt_gbs = target_attn_bytes(b, heads) / (tgt_ms * 1e-3) / 1e9
        traffic = recorded_traffic()
        result = {
            "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "repeats": len(region_ms),
            "ms_per_step_spread": {"min": round(min(region_ms) / args.steps, 5),
                                   "max": round(max(region_ms) / args.steps, 5)},
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded; stands in for the pages' proprietary logs)",
            "config": {"workload": WORKLOAD, "users_per_gpu": b.B, "total_tokens": b.total_tokens,
                       "total_t": b.total_t, "flops_per_step_per_gpu": flops_step,
                       "l2": f"inputs rotated over {args.sets} resident copies "
                             f"({args.sets * 89} MB of inputs > 126 MB L2)",
                       "launch": "steps replay CUDA graphs of their launches (one graph: one step per input set)",
                       "parallelism": f"replicas x{world} (users sharded, no collective)"},
            "users_per_s": round(users_all * args.steps / (ms_max * 1e-3), 1),
            "per_layer": {
                "full": {"ms": round(ms_parts["full_attn"] + ms_parts["full_gate"], 5),
                         "attn_tflops": round(full_tf, 2),
                         "users_per_s": round(b.B / ((ms_parts["full_attn"] + ms_parts["full_gate"]) * 1e-3), 1)},
                "target": {"ms": round(ms_parts["target_attn"] + ms_parts["target_gate"], 5),
                           "attn_ms_in_graph": round(tgt_ms, 5),
                           "attn_tflops": round(fl_tgt / (tgt_ms * 1e-3) / 1e12, 2),
                           "attn_gbs": round(tgt_gbs, 1), "attn_hbm_frac": round(tgt_gbs / hbm, 4),
                           "attn_timing": "event-record nodes around the Target attention call (conditional "
                                          "accumulator clear + kernel) inside the timed region",
                           "users_per_s": round(b.B / ((ms_parts["target_attn"] + ms_parts["target_gate"]) * 1e-3), 1)},
                "pack_ms_in_graph": round(pack_ms, 5),
                "ms_parts": {k: round(v, 5) for k, v in ms_parts.items()},
                "ms_parts_note": "eager pass with an event between launches (not the graph-replayed step)",
            },
            "roofline": {"kernel": "Full-layer attention (attn_fwd_tc_kernel, tcgen05)", "bound": "tensor",
                         "achieved": round(full_tf, 2), "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": round(full_tf / peak_tf, 4), "traffic": traffic,
                         "peak_source": f"{src} bf16 dense (burst)",
                         "flops_per_launch": fl_full, "launch_ms": round(full_ms, 5),
                         "launch_ms_source": f"median of event-record nodes around the Full attention launches "
                                             f"of the last steps of each of the {len(region_ms)} timed regions"},
            "e2e": e2e,
            "clocks": clocks,
            "gpu_launches": launches_per_step * args.steps * len(region_ms),
        }
    return result, b, heads


def run_e2e(args, M, cfg, b, heads, dev, stream, world):
    """Same metric through the public layer calls, with inputs in pinned host memory and the
    host<->device copies of each step's inputs and outputs inside the timed region.

    The steps are pipelined the way a data loader would feed the GPU: two sets of device
    buffers, the inputs of step i+1 copied in (copy-in stream) while step i computes
    (the bench stream) and step i-1's outputs are copied out (copy-out stream).  The timed
    region runs from the first copy-in to the last copy-out, on the device clock."""
    import torch
    import torch.distributed as dist
    fi = syn.layer_inputs(b, heads, target=False, seed=11)
    ti = syn.layer_inputs(b, heads, target=True, seed=111)
    pin = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dtype=dt)).pin_memory()
    pbf = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()
    host = [pin(b.L_H, np.int32), pin(b.L_R, np.int32), pin(b.L_T, np.int32), pin(b.r_ts, np.int64),
            pin(b.t_exp, np.int64), pbf(fi.q), pbf(fi.k), pbf(fi.v), pbf(fi.u),
            pin(fi.gamma, np.float32), pin(fi.beta, np.float32), pbf(ti.q), pbf(ti.k), pbf(ti.v),
            pbf(ti.u), pin(ti.gamma, np.float32), pin(ti.beta, np.float32)]
    f32 = dict(dtype=torch.float32, device=dev)
    sets = []
    for _ in range(2):
        sets.append(dict(
            inp=[torch.empty_like(h, device=dev) for h in host], meta=M.alloc_meta(cfg, dev),
            f=(torch.empty(b.total_tokens, heads.dq, **f32), torch.empty(b.total_tokens, heads.dq, **f32),
               torch.empty(b.total_tokens, 2, **f32)),
            t=(torch.empty(b.total_t, heads.dq, **f32), torch.empty(b.total_t, heads.dq, **f32),
               torch.empty(b.total_t, 2, **f32)),
            out_f=torch.empty(b.total_tokens, heads.dq, dtype=torch.float32).pin_memory(),
            out_t=torch.empty(b.total_t, heads.dq, dtype=torch.float32).pin_memory(),
            ev_in=torch.cuda.Event(), ev_comp=torch.cuda.Event(), ev_out=torch.cuda.Event()))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    h2d = sum(h.numel() * h.element_size() for h in host)
    d2h = (b.total_tokens + b.total_t) * heads.dq * 4

    def step(i):
        z = sets[i & 1]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(z["ev_comp"])  # step i-2's compute no longer reads this set
            for h, d in zip(host, z["inp"]):
                d.copy_(h, non_blocking=True)
            z["ev_in"].record(s_in)
        stream.wait_event(z["ev_in"])
        if i >= 2:
            stream.wait_event(z["ev_out"])    # step i-2's outputs have been copied out
        lh, lr, lt, rts, tex, q, k, v, u, g, bt, tq, tk, tv, tu, tg, tbt = z["inp"]
        M.pack(cfg, lh, lr, lt, rts, tex, z["meta"], stream)
        M.attn_full_fwd(cfg, z["meta"], q, k, v, u, g, bt, *z["f"], stream)
        M.attn_target_fwd(cfg, z["meta"], tq, tk, tv, tu, tg, tbt, *z["t"], stream)
        z["ev_comp"].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(z["ev_comp"])
            z["out_f"].copy_(z["f"][0], non_blocking=True)
            z["out_t"].copy_(z["t"][0], non_blocking=True)
            z["ev_out"].record(s_out)

    steps = max(3, min(args.steps, args.e2e_steps))
    for i in range(3):
        step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(steps):
        step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(stream)
    t1.record(s_out)
    torch.cuda.synchronize(dev)
    ms = t0.elapsed_time(t1)
    fl = attn_flops(b, heads, False) + attn_flops(b, heads, True)
    ms, (fl,) = reduce_over_ranks(ms, [fl], dev)
    return {"value": round(fl / (ms / steps * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "ms_per_step": round(ms / steps, 4),
            "pipelining": "two buffer sets; copy-in, compute and copy-out on three streams"}


# ----------------------------------------------------------------------------- CPU oracle

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def oracle_time(b, heads, users, seeds=(11, 111)):
    """Time the fp64 oracle's Full + Target forward on the given users; returns (seconds, flops)."""
    from oracle import mtfm_oracle as O  # the CPU-baseline leg is allowed to run the oracle
    fi = syn.layer_inputs(b, heads, target=False, seed=seeds[0])
    ti = syn.layer_inputs(b, heads, target=True, seed=seeds[1])
    t = time.perf_counter()
    O.full_fwd(b, heads, fi, users=set(users))
    O.target_fwd(b, heads, ti, users=set(users))
    dt = time.perf_counter() - t
    sub = syn.JaggedBatch(b.L_H[users], b.L_R[users], b.L_T[users],
                          np.concatenate([b.r_ts[int(np.sum(b.L_R[:u])):int(np.sum(b.L_R[:u + 1]))] for u in users]),
                          np.concatenate([b.t_exp[int(np.sum(b.L_T[:u])):int(np.sum(b.L_T[:u + 1]))] for u in users]),
                          b.scenario, b.v2_subtokens)
    return dt, attn_flops(sub, heads, False) + attn_flops(sub, heads, True)


def cpu_baseline(b, heads, budget_s=20.0):
    """The oracle as it stands on the host cores, on a bounded sample of the same workload."""
    users, spent, fl = [], 0.0, 0.0
    order = list(range(b.B))
    for u in order:
        dt, f = oracle_time(b, heads, [u])
        users.append(u)
        spent += dt
        fl += f
        if spent >= budget_s:
            break
    return {"value": round(fl / spent / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"fp64 numpy oracle, Full + Target forward of {len(users)} of {b.B} users "
                      f"of the same batch ({spent:.1f} s of CPU work)"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    heads = syn.PAIR_HEADS
    b = syn.pair_batch(args.users, seed=1001)
    # each step: the oracle on one user of the batch (users in turn); bounded so the run ends in minutes
    per_user = oracle_time(b, heads, [0])[0]
    budget = 150.0
    steps = max(1, min(args.steps, int(budget / max(per_user, 1e-3)) - args.warmup))
    warm = min(args.warmup, 3)
    for i in range(warm):
        oracle_time(b, heads, [i % b.B])
    spent, fl = 0.0, 0.0
    for i in range(steps):
        dt, f = oracle_time(b, heads, [i % b.B])
        spent += dt
        fl += f
    value = fl / spent / 1e12
    cores = blas_threads()
    sample = (f"fp64 numpy oracle; each step = Full + Target forward of one user of the "
              f"{b.B}-user batch (users in turn); {steps} steps timed")
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
            "steps": steps, "steps_requested": args.steps, "warmup": warm,
            "ms_per_step": round(spent / steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "users_per_gpu": b.B},
            "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- other workloads

class GraphStep:
    """One step's launches captured as two CUDA graphs: plain, and an instrumented twin with
    event-record nodes around the named launches.  ``timed`` replays K steps (the last one the
    twin, so every kernel duration is read inside the timed region without paying for event
    nodes in every step), ``repeats`` times, each region bracketed by a synchronize."""

    def __init__(self, dev, fn, labels):
        import torch
        self.torch, self.dev = torch, dev
        self.stream = torch.cuda.Stream(dev)
        self.ev = {l: (torch.cuda.Event(enable_timing=True, external=True),
                       torch.cuda.Event(enable_timing=True, external=True)) for l in labels}
        mark = lambda l, i: self.ev[l][i].record(self.stream)
        with torch.cuda.stream(self.stream):
            fn(None)                       # eager once (lazy module loads, workspaces)
        torch.cuda.synchronize(dev)
        self.g = self._capture(lambda: fn(None))
        self.gi = self._capture(lambda: fn(mark))

    def _capture(self, f):
        g = self.torch.cuda.CUDAGraph()
        with self.torch.cuda.graph(g, stream=self.stream):
            f()
        return g

    def timed(self, steps, warmup, repeats, sampler=None):
        torch = self.torch
        with torch.cuda.stream(self.stream):
            for _ in range(max(3, warmup)):
                self.g.replay()
        torch.cuda.synchronize(self.dev)
        if sampler:
            sampler.begin()
        per_step = []
        for _ in range(repeats):
            a = torch.cuda.Event(enable_timing=True)
            z = torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize(self.dev)
            with torch.cuda.stream(self.stream):
                a.record(self.stream)
                for i in range(steps):
                    (self.gi if i == steps - 1 else self.g).replay()
                z.record(self.stream)
            torch.cuda.synchronize(self.dev)
            per_step.append(a.elapsed_time(z) / steps)
        clocks = sampler.stop() if sampler else None
        kernels = {l: a.elapsed_time(z) for l, (a, z) in self.ev.items()}
        return per_step, kernels, clocks


def _spread(per_step):
    return {"median": round(statistics.median(per_step), 5), "min": round(min(per_step), 5),
            "max": round(max(per_step), 5), "repeats": len(per_step)}


def _dev_inputs(dev, seed):
    import torch
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    return lambda std, *shape: (std * torch.randn(*shape, generator=gen, device=dev)).to(torch.bfloat16)


def _packed(M, b, heads, dev):
    import torch
    from hybrid_masked_attention_b200.session import HybridAttention
    cfg = M.Config(b.B, b.total_tokens, b.total_r, b.total_t, heads.hq, heads.hkv, heads.dh, b.v2_subtokens)
    s = HybridAttention(cfg, dev)
    it = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dtype=dt)).to(dev)
    lens = (it(b.L_H, np.int32), it(b.L_R, np.int32), it(b.L_T, np.int32), it(b.r_ts, np.int64),
            it(b.t_exp, np.int64))
    s.pack(*lens, check=True)
    return cfg, s, lens


def sweep_entry(dev, N, v2, steps, warmup, repeats, heads=syn.PAIR_HEADS, total_tokens=1 << 21):
    """Sequence-length sweep point: 2^21 tokens (or total_tokens, for smaller profiling runs) of
    users of N tokens each (H:R:T ~ 70:15:15; V2: targets of 4 sub-tokens).  A step is the pair step's path at this shape: pack, Full attention
    + gate, Target attention + gate.  Activations are seeded device-side N(0, 1) bf16 (GBs, far
    larger than L2)."""
    import torch
    import hybrid_masked_attention_b200 as M
    b = syn.sweep_batch(N, v2=v2, total_tokens=total_tokens, seed=1003)
    cfg, s, lens = _packed(M, b, heads, dev)
    rnd = _dev_inputs(dev, 1003)
    Nt, T, D, Dkv = b.total_tokens, b.total_t, heads.dq, heads.dkv
    gam, bet = torch.ones(3, D, device=dev), torch.zeros(3, D, device=dev)
    F = dict(q=rnd(1, Nt, D), k=rnd(1, Nt, Dkv), v=rnd(1, Nt, Dkv), u=rnd(1, Nt, D))
    Tg = dict(q=rnd(1, T, D), k=rnd(1, Nt, Dkv), v=rnd(1, Nt, Dkv), u=rnd(1, T, D))
    out_f, out_t = s._fwd_out(Nt, True), s._fwd_out(T, True)

    def step(mark):
        s.pack(*lens)
        if mark: mark("full_attn", 0)
        M.attn_full(cfg, s.meta, F["q"], F["k"], F["v"], out_f[1])
        if mark: mark("full_attn", 1)
        M.gate_fwd(cfg, s.meta, False, out_f[1], F["u"], gam, bet, out_f[0], out_f[2])
        if mark: mark("target_attn", 0)
        M.attn_target(cfg, s.meta, Tg["q"], Tg["k"], Tg["v"], out_t[1])
        if mark: mark("target_attn", 1)
        M.gate_fwd(cfg, s.meta, True, out_t[1], Tg["u"], gam, bet, out_t[0], out_t[2])

    gs = GraphStep(dev, step, ["full_attn", "target_attn"])
    per_step, kern, clocks = gs.timed(steps, warmup, repeats, ClockSampler(dev))
    M.pack_check(s.meta)
    peaks, src = load_peaks()
    peak_s = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    ff, ft = attn_flops(b, heads, False), attn_flops(b, heads, True)
    ms = statistics.median(per_step)
    tf = lambda fl, t: fl / (t * 1e-3) / 1e12
    tgt_gbs = target_attn_bytes(b, heads) / (kern["target_attn"] * 1e-3) / 1e9
    tgt_ai = ft / target_attn_bytes(b, heads)
    ridge = peak_s * 1e12 / (hbm * 1e9)
    return {
        "workload": f"sweep N={N}{' V2' if v2 else ''}: {b.B} users x {N} tokens "
                    f"(L_H {int(b.L_H[0])}, L_R {int(b.L_R[0])}, L_T {int(b.L_T[0])}); Hq {heads.hq} / "
                    f"Hkv {heads.hkv}, head_dim {heads.dh}",
        "value": round(tf(ff + ft, ms), 3), "unit": "TFLOP/s", "ms_per_step": round(ms, 5),
        "step_ms": _spread(per_step), "steps": steps, "users_per_s": round(b.B / (ms * 1e-3), 1),
        "total_tokens": Nt, "total_t": T,
        "kernels_in_graph_ms": {k: round(v, 5) for k, v in kern.items()},
        "roofline": {"kernel": "Full-layer attention (attn_fwd_tc_kernel)", "bound": "tensor",
                     "achieved": round(tf(ff, kern["full_attn"]), 2), "peak": peak_s, "unit": "TFLOP/s",
                     "frac": round(tf(ff, kern["full_attn"]) / peak_s, 4),
                     "peak_source": f"{src} bf16 dense (sustained: the step runs for milliseconds)"},
        "target_roofline": {"kernel": "Target-layer attention call (conditional accumulator clear + attn_fwd_tgt_kernel)",
                            "bound": "hbm" if tgt_ai < ridge else "tensor",
                            "achieved_gbs": round(tgt_gbs, 1), "frac_hbm": round(tgt_gbs / hbm, 4),
                            "achieved_tflops": round(tf(ft, kern["target_attn"]), 2),
                            "frac_tensor": round(tf(ft, kern["target_attn"]) / peak_s, 4),
                            "flop_per_byte": round(tgt_ai, 1), "ridge_flop_per_byte": round(ridge, 1)},
        "clocks": clocks, "l2": "inputs of GBs, far larger than the 126 MB L2",
    }


def train_entry(dev, users, steps, warmup, repeats, heads=syn.PAIR_HEADS):
    """Training step at the production-shape distributions: pack, forward and backward (dQ, dK,
    dV, dU, dgamma, dbeta) of one Full and one Target layer; dY ~ N(0, 1) bf16."""
    import torch
    import hybrid_masked_attention_b200 as M
    b = syn.pair_batch(users, seed=1005)
    cfg, s, lens = _packed(M, b, heads, dev)
    rnd = _dev_inputs(dev, 1005)
    Nt, T, D, Dkv = b.total_tokens, b.total_t, heads.dq, heads.dkv
    gam, bet = torch.ones(3, D, device=dev), torch.zeros(3, D, device=dev)
    F = dict(q=rnd(1, Nt, D), k=rnd(1, Nt, Dkv), v=rnd(1, Nt, Dkv), u=rnd(1, Nt, D), dy=rnd(1, Nt, D))
    Tg = dict(q=rnd(1, T, D), k=rnd(1, Nt, Dkv), v=rnd(1, Nt, Dkv), u=rnd(1, T, D), dy=rnd(1, T, D))
    out_f, out_t = s._fwd_out(Nt, True), s._fwd_out(T, True)
    s.workspace(False), s.workspace(True)
    gf = s.full_bwd(F["q"], F["k"], F["v"], F["u"], gam, bet, out_f[1], out_f[2], F["dy"])
    gt = s.target_bwd(Tg["q"], Tg["k"], Tg["v"], Tg["u"], gam, bet, out_t[1], out_t[2], Tg["dy"])
    order = ("dq", "dk", "dv", "du", "dgamma", "dbeta")

    def step(mark):
        s.pack(*lens)
        if mark: mark("full_fwd", 0)
        s.full_fwd(F["q"], F["k"], F["v"], F["u"], gam, bet, out=out_f)
        if mark: mark("full_fwd", 1)
        s.target_fwd(Tg["q"], Tg["k"], Tg["v"], Tg["u"], gam, bet, out=out_t)
        if mark: mark("full_bwd", 0)
        M.attn_full_bwd(cfg, s.meta, F["q"], F["k"], F["v"], F["u"], gam, bet, out_f[1], out_f[2], F["dy"],
                        *[gf[k] for k in order], s.workspace(False))
        if mark: mark("full_bwd", 1)
        if mark: mark("target_bwd", 0)
        M.attn_target_bwd(cfg, s.meta, Tg["q"], Tg["k"], Tg["v"], Tg["u"], gam, bet, out_t[1], out_t[2],
                          Tg["dy"], *[gt[k] for k in order], s.workspace(True))
        if mark: mark("target_bwd", 1)

    gs = GraphStep(dev, step, ["full_fwd", "full_bwd", "target_bwd"])
    per_step, kern, clocks = gs.timed(steps, warmup, repeats, ClockSampler(dev))
    M.pack_check(s.meta)
    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    ff, ft = attn_flops(b, heads, False), attn_flops(b, heads, True)
    ms = statistics.median(per_step)
    tf = lambda fl, t: fl / (t * 1e-3) / 1e12
    return {
        "workload": f"training step: {b.B} users, production-shape lengths; fwd + bwd of one Full and one "
                    f"Target layer; Hq {heads.hq} / Hkv {heads.hkv}, head_dim {heads.dh}",
        "value": round(tf(3.5 * (ff + ft), ms), 3), "unit": "TFLOP/s",
        "flop_convention": "forward unmasked FLOPs x 3.5 (backward counted as 2.5x forward)",
        "ms_per_step": round(ms, 5), "step_ms": _spread(per_step), "steps": steps,
        "users_per_s": round(b.B / (ms * 1e-3), 1), "total_tokens": Nt, "total_t": T,
        "kernels_in_graph_ms": {k: round(v, 5) for k, v in kern.items()},
        "roofline": {"kernel": "Full-layer backward call (gate backward + "
                               f"{'attn_bwd_tc_kernel' if heads.dh == 64 else 'attn_bwd_mma_kernel'})", "bound": "tensor",
                     "achieved": round(tf(2.5 * ff, kern["full_bwd"]), 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(tf(2.5 * ff, kern["full_bwd"]) / peak, 4),
                     "peak_source": f"{src} bf16 dense (burst)"},
        "clocks": clocks, "l2": f"step working set {(Nt * (4 * D + 2 * Dkv) * 2 + Nt * D * 12) / 1e6:.0f} MB > 126 MB L2",
    }


def stack_entry(dev, users, steps, warmup, repeats, heads=syn.PAIR_HEADS, d=512):
    """The 16-layer backbone stack (4 x (Full, Target, Target, Target)) forward: seeded
    device-side weights N(0, 0.02), output projections N(0, 0.02 / sqrt(16)), X ~ N(0, 1);
    the whole mtfm_stack_fwd call replayed as one CUDA graph per step."""
    import torch
    import hybrid_masked_attention_b200 as M
    b = syn.pair_batch(users, seed=1002)
    cfg, s, lens = _packed(M, b, heads, dev)
    rnd = _dev_inputs(dev, 1002)
    Nt, T, D, Dkv = b.total_tokens, b.total_t, heads.dq, heads.dkv
    kinds = syn.STACK_KINDS
    layers = []
    for k in kinds:
        w_in = rnd(0.02, 2 * D + 2 * Dkv, d) if k == "F" else rnd(0.02, 2 * D, d)
        w_kv = rnd(0.02, 2 * Dkv, d) if k == "T" else None
        layers.append(M.LayerWeights(k, torch.ones(d, device=dev), w_in, w_kv, rnd(0.02 / np.sqrt(len(kinds)), d, D),
                                     torch.ones(3, D, device=dev), torch.zeros(3, D, device=dev)))
    x = rnd(1.0, Nt, d).float()
    ws = torch.empty(M.stack_workspace_bytes(cfg, d), dtype=torch.uint8, device=dev)

    def step(mark):
        s.pack(*lens)
        if mark: mark("stack", 0)
        M.stack_fwd(cfg, s.meta, d, layers, x, ws)
        if mark: mark("stack", 1)

    gs = GraphStep(dev, step, ["stack"])
    per_step, kern, clocks = gs.timed(steps, warmup, repeats, ClockSampler(dev))
    M.pack_check(s.meta)
    assert torch.isfinite(x).all().item()
    peaks, src = load_peaks()
    peak_s = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    ff, ft = attn_flops(b, heads, False), attn_flops(b, heads, True)
    g_full = 2.0 * Nt * d * (2 * D + 2 * Dkv) + 2.0 * Nt * D * d
    g_tgt = 2.0 * T * d * 2 * D + 2.0 * Nt * d * 2 * Dkv + 2.0 * T * D * d
    n_f = sum(k == "F" for k in kinds)
    n_t = len(kinds) - n_f
    fl = n_f * (ff + g_full) + n_t * (ft + g_tgt)
    ms = statistics.median(per_step)
    tf = lambda f, t: f / (t * 1e-3) / 1e12
    return {
        "workload": f"16-layer backbone stack, 4 x (Full, Target, Target, Target): {b.B} users, production-shape "
                    f"lengths, d_model {d}, Hq {heads.hq} / Hkv {heads.hkv}, head_dim {heads.dh}",
        "value": round(tf(fl, ms), 3), "unit": "TFLOP/s",
        "flop_convention": "unmasked attention FLOPs + projection GEMM FLOPs",
        "ms_per_step": round(ms, 5), "step_ms": _spread(per_step), "steps": steps,
        "users_per_s": round(b.B / (ms * 1e-3), 1), "per_layer_users_per_s": round(b.B * len(kinds) / (ms * 1e-3), 1),
        "total_tokens": Nt, "total_t": T, "attn_flops": n_f * ff + n_t * ft, "gemm_flops": n_f * g_full + n_t * g_tgt,
        "kernels_in_graph_ms": {k: round(v, 5) for k, v in kern.items()},
        "roofline": {"kernel": "whole stack call (RMSNorm, tcgen05 GEMMs, attention, gates)", "bound": "tensor",
                     "achieved": round(tf(fl, kern["stack"]), 2), "peak": peak_s, "unit": "TFLOP/s",
                     "frac": round(tf(fl, kern["stack"]) / peak_s, 4),
                     "peak_source": f"{src} bf16 dense (sustained)"},
        "clocks": clocks, "l2": "per-layer working set (X fp32 + scratch) larger than the 126 MB L2",
    }


def v2_layer_entry(dev, users, seqlen, steps, warmup, repeats, heads=syn.PAIR_HEADS, d=512, dff=1024):
    """One V2 Target Scale-Up layer (per-sub-token [U Q] projections and SwiGLU FFNs, mixing of
    each target's 4 sub-tokens; Meituan tech blog §3.3.2) on users of seqlen tokens with V2
    targets (H:R:T ~ 70:15:15); seeded device-side weights, X ~ N(0, 1)."""
    import torch
    import hybrid_masked_attention_b200 as M
    b = syn.sweep_batch(seqlen, v2=True, B=users, seed=1016)
    cfg, s, lens = _packed(M, b, heads, dev)
    rnd = _dev_inputs(dev, 1016)
    Nt, T, D, Dkv = b.total_tokens, b.total_t, heads.dq, heads.dkv
    ones, zeros = lambda *sh: torch.ones(*sh, device=dev), lambda *sh: torch.zeros(*sh, device=dev)
    w = M.V2LayerWeights(ones(d), [rnd(0.02, 2 * D, d) for _ in range(4)], rnd(0.02, 2 * Dkv, d), rnd(0.02, d, D),
                         ones(3, D), zeros(3, D), ones(d), [rnd(0.02, dff, d) for _ in range(4)],
                         [rnd(0.02, dff, d) for _ in range(4)], [rnd(0.02, d, dff) for _ in range(4)])
    x = rnd(1.0, Nt, d).float()
    ws = torch.empty(M.v2_workspace_bytes(cfg, d, dff), dtype=torch.uint8, device=dev)

    def step(mark):
        s.pack(*lens)
        if mark: mark("v2_layer", 0)
        M.v2_target_layer_fwd(cfg, s.meta, d, dff, w, x, ws)
        if mark: mark("v2_layer", 1)

    gs = GraphStep(dev, step, ["v2_layer"])
    per_step, kern, clocks = gs.timed(steps, warmup, repeats, ClockSampler(dev))
    M.pack_check(s.meta)
    peaks, src = load_peaks()
    peak_s = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    ft = attn_flops(b, heads, True)
    gemm = 2.0 * Nt * d * 2 * Dkv + 2.0 * T * d * 2 * D + 2.0 * T * D * d + 2.0 * T * d * 2 * dff + 2.0 * T * dff * d
    ms = statistics.median(per_step)
    tf = lambda f, t: f / (t * 1e-3) / 1e12
    return {
        "workload": f"V2 Target Scale-Up layer: {b.B} users x {seqlen} tokens, {T // 4} targets of 4 sub-tokens; "
                    f"d_model {d}, d_ff {dff}, Hq {heads.hq} / Hkv {heads.hkv}, head_dim {heads.dh}",
        "value": round(tf(ft + gemm, ms), 3), "unit": "TFLOP/s",
        "flop_convention": "unmasked attention FLOPs + projection / FFN GEMM FLOPs",
        "ms_per_step": round(ms, 5), "step_ms": _spread(per_step), "steps": steps,
        "users_per_s": round(b.B / (ms * 1e-3), 1), "targets_per_s": round(T / 4 / (ms * 1e-3), 1),
        "total_tokens": Nt, "total_t": T, "attn_flops": ft, "gemm_flops": gemm,
        "kernels_in_graph_ms": {k: round(v, 5) for k, v in kern.items()},
        "roofline": {"kernel": "whole V2 layer call (RMSNorm, tcgen05 GEMMs, Target attention, gate, mixing)",
                     "bound": "tensor", "achieved": round(tf(ft + gemm, kern["v2_layer"]), 2), "peak": peak_s,
                     "unit": "TFLOP/s", "frac": round(tf(ft + gemm, kern["v2_layer"]) / peak_s, 4),
                     "peak_source": f"{src} bf16 dense (sustained)"},
        "clocks": clocks,
    }


PER_CONFIG = (
    ("sweep_n8192", lambda dev, a: sweep_entry(dev, 8192, False, max(2, a.config_steps // 4), a.warmup, 3)),
    ("sweep_n512", lambda dev, a: sweep_entry(dev, 512, False, a.config_steps, a.warmup, 3)),
    ("sweep_n1024", lambda dev, a: sweep_entry(dev, 1024, False, a.config_steps, a.warmup, 3)),
    ("sweep_n2048", lambda dev, a: sweep_entry(dev, 2048, False, max(2, a.config_steps // 2), a.warmup, 3)),
    ("sweep_n4096", lambda dev, a: sweep_entry(dev, 4096, False, max(2, a.config_steps // 4), a.warmup, 3)),
    ("sweep_v2_n2048", lambda dev, a: sweep_entry(dev, 2048, True, max(2, a.config_steps // 2), a.warmup, 3)),
    ("stack_b64", lambda dev, a: stack_entry(dev, 64, a.config_steps, a.warmup, 5)),
    ("train_b96", lambda dev, a: train_entry(dev, 96, a.config_steps, a.warmup, 5)),
    ("train_b160", lambda dev, a: train_entry(dev, 160, a.config_steps, a.warmup, 5)),
    ("v2_layer_n2048", lambda dev, a: v2_layer_entry(dev, 64, 2048, a.config_steps, a.warmup, 5)),
    ("stack_b64_d768_dh256", lambda dev, a: stack_entry(dev, 64, a.config_steps, a.warmup, 5,
                                                        heads=syn.Heads(3, 1, 256), d=768)),
    ("train_b96_dh256", lambda dev, a: train_entry(dev, 96, a.config_steps, a.warmup, 5,
                                                   heads=syn.Heads(3, 1, 256))),
)


def run_workload(args):
    """--workload sweep|train|stack: one JSON line for that configuration alone."""
    import torch
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    heads = syn.Heads(*(int(x) for x in args.heads.split(",")))
    steps = max(1, args.steps)
    if args.workload == "sweep":
        e = sweep_entry(dev, args.seqlen, args.v2, steps, args.warmup, args.repeats, heads, args.tokens)
    elif args.workload == "train":
        e = train_entry(dev, args.users or 96, steps, args.warmup, args.repeats, heads)
    elif args.workload == "v2layer":
        e = v2_layer_entry(dev, args.users or 64, args.seqlen, steps, args.warmup, args.repeats, heads, args.dmodel)
    else:
        e = stack_entry(dev, args.users or 64, steps, args.warmup, args.repeats, heads, args.dmodel)
    out = {"metric": METRIC, "value": e.pop("value"), "unit": e.pop("unit"), "n_gpus": 1, "steps": steps,
           "warmup": max(3, args.warmup), "ms_per_step": e.pop("ms_per_step"), "higher_is_better": True,
           "dtype": "bf16", "data": "synthetic", "config": {"workload": e.pop("workload")}, **e}
    print(json.dumps(out), flush=True)


def run_infer(args):
    """Request-level Target attention over a cached key/value prefix: --users requests (default
    128), each a user whose 2000-token prefix (H 1800, R 200, sorted timestamps) has its
    keys/values in the cache, scored against 200 candidates with their own exposures.  A step
    is pack + the cached-prefix Target layer forward (attention + gate), replayed as a CUDA
    graph; the same layer on the concatenated [prefix; candidates] layout is timed beside it.
    The prefix cache (128 users: 131 MB) plus the candidates' tensors exceed the 126 MB L2."""
    import torch
    import hybrid_masked_attention_b200 as M
    dev = torch.device("cuda", 0)
    heads = syn.PAIR_HEADS
    B = args.users if args.users is not None else 128
    LH, LR, LT = 1800, 200, 200
    b = syn.fixed_batch([LH] * B, [LR] * B, [LT] * B, seed=1006)
    cfg = M.Config(b.B, b.total_tokens, b.total_r, b.total_t, heads.hq, heads.hkv, heads.dh)
    inp = syn.layer_inputs(b, heads, target=True, seed=1006)
    it = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a, dtype=dt)).to(dev)
    bf = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    lens = (it(b.L_H, np.int32), it(b.L_R, np.int32), it(b.L_T, np.int32), it(b.r_ts, np.int64),
            it(b.t_exp, np.int64))
    rows = np.arange(b.total_tokens).reshape(B, LH + LR + LT)
    pre_rows, cand_rows = rows[:, :LH + LR].reshape(-1), rows[:, LH + LR:].reshape(-1)
    q, u, k, v = bf(inp.q), bf(inp.u), bf(inp.k), bf(inp.v)
    kp, vp, kc, vc = bf(inp.k[pre_rows]), bf(inp.v[pre_rows]), bf(inp.k[cand_rows]), bf(inp.v[cand_rows])
    g, bt = it(inp.gamma, np.float32), it(inp.beta, np.float32)
    meta = M.alloc_meta(cfg, dev)
    f32 = dict(dtype=torch.float32, device=dev)
    T, D = b.total_t, heads.dq
    y, a, st = torch.empty(T, D, **f32), torch.empty(T, D, **f32), torch.empty(T, 2, **f32)
    side = torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def cached(s):
        M.pack(cfg, *lens, meta, s)
        M.attn_target_cached_fwd(cfg, meta, q, kp, vp, kc, vc, u, g, bt, y, a, st, s)

    def concat(s):
        M.pack(cfg, *lens, meta, s)
        M.attn_target_fwd(cfg, meta, q, k, v, u, g, bt, y, a, st, s)

    def timed_graph(fn, steps):
        with torch.cuda.stream(side):
            for _ in range(max(3, args.warmup)):
                fn(side)
        torch.cuda.synchronize()
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=side):
            fn(side)
        with torch.cuda.stream(side):
            for _ in range(3):
                gr.replay()
            torch.cuda.synchronize()
            e0, e1 = ev(), ev()
            e0.record(side)
            for _ in range(steps):
                gr.replay()
            e1.record(side)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    steps = max(1, args.steps)
    clocks = ClockSampler(dev)
    clocks.begin()
    ms = timed_graph(cached, steps)
    clk = clocks.stop()
    ms_concat = timed_graph(concat, steps)
    M.pack_check(meta, side)
    fl = attn_flops(b, heads, True)
    peaks, src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    # bytes a step must move: the prefix K/V, the candidates' Q, K, V, U, and Y (fp32)
    moved = (kp.numel() + vp.numel() + kc.numel() + vc.numel() + q.numel() + u.numel()) * 2 + T * D * 4
    out = {"metric": METRIC, "value": round(fl / (ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
           "n_gpus": 1, "steps": steps, "warmup": max(3, args.warmup), "ms_per_step": round(ms, 5),
           "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": f"inference: {B} requests, cached {LH + LR}-token prefix (H {LH}, R {LR}), "
                                  f"{LT} candidates each; pack + cached-prefix Target layer forward",
                      "requests": B, "candidates": T, "flops_per_step": fl,
                      "l2": f"prefix cache + candidate tensors {moved / 1e6:.0f} MB > 126 MB L2",
                      "launch": "one CUDA graph per step"},
           "candidates_per_s": round(T / (ms * 1e-3), 1),
           "gbs": round(moved / (ms * 1e-3) / 1e9, 1), "frac_hbm": round(moved / (ms * 1e-3) / 1e9 / hbm, 4),
           "concatenated_layout_ms": round(ms_concat, 5),
           "clocks": clk}
    print(json.dumps(out), flush=True)


# ----------------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["mtfm", "reference"], default="mtfm")
    ap.add_argument("--users", type=int, default=None,
                    help="users (default 32; 64 for --workload stack, 128 requests for infer)")
    ap.add_argument("--sets", type=int, default=4, help="resident input copies rotated across steps")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["pair", "sweep", "train", "stack", "infer", "v2layer"], default="pair",
                    help="pair: the headline step; sweep/train/stack/infer: timings of the other configs")
    ap.add_argument("--seqlen", type=int, default=2048, help="sweep: tokens per user")
    ap.add_argument("--tokens", type=int, default=1 << 21,
                    help="sweep: total tokens (default 2^21; smaller for profiler captures)")
    ap.add_argument("--v2", action="store_true", help="sweep: V2 targets (4 sub-tokens each)")
    ap.add_argument("--dmodel", type=int, default=512, help="stack: d_model")
    ap.add_argument("--heads", default="8,2,64",
                    help="stack/sweep/train: Hq,Hkv,head_dim (e.g. 3,1,256 with --dmodel 768)")
    ap.add_argument("--repeats", type=int, default=10,
                    help="the K-step timed region is run this many times; value is the median region")
    ap.add_argument("--config-steps", type=int, default=8,
                    help="steps per timed region of each per_config entry")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the other configurations' entries of the JSON line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)

    if args.workload == "infer":
        run_infer(args)
        return
    if args.workload != "pair":
        run_workload(args)
        return
    if args.users is None:
        args.users = 32
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res, b, heads = run_mtfm(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_per_config:
                # the other configurations, each on this GPU (one process, no collective)
                dev = torch.device("cuda", local_rank)
                res["per_config"] = {}
                for name, fn in PER_CONFIG:
                    res["per_config"][name] = fn(dev, args)
                    torch.cuda.empty_cache()
            if world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(b, heads)
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
