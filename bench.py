"""Benchmark: k-MIP attention query-heads/s, forward and forward+backward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload gmm_n100000] [--k 15] [--no-configs] [--no-baselines]
                    [--no-k-sweep] [--no-e2e] [--no-cpu-baseline]

One step is the whole hot path over one batch: the forward (work list,
fused score + top-k + softmax + V gather) and the backward (recompute,
dQ, dK/dV scatter) of one graph of N = 100,000 nodes, 4 heads of 32, k = 15,
keys from a 64-component Gaussian mixture.  The value is N * H / step time,
summed over ranks.  With N > 1 GPUs (torchrun) every rank runs its own
independent batch (a different seed) -- there is no data-path collective;
the only collectives are the barriers and the max-over-ranks of the time.

Timing: W untimed warm-up steps, then K steps, each phase bracketed by CUDA
events on the launching stream; between steps, outside the events, a 256 MiB
buffer is written to flush the L2 (126 MB) and a ~5 ms device-side spin holds
the stream until the step's launches are queued (a host stall then delays
the spin, not the timed kernels).  A barrier and a device synchronise
bracket the whole timed loop.  Besides the headline step the line
carries: per-step times and SM clocks, the backward's and the gather stage's
GB/s, the deterministic backward, the k sweep, the other four workloads
(`configs`), torch's full attention and dense top-k on the same inputs with
the Figure 8 diagnostics (`baselines`), the end-to-end run from pinned host
buffers (`e2e`) and the fp64 oracle on the host cores (`cpu_baseline`).
One JSON line is printed by rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from graph_transformer_sparse_kmip_b200 import binding  # noqa: E402
from graph_transformer_sparse_kmip_b200 import workloads as wl  # noqa: E402

METRIC = "k-MIP attn query-heads/s fwd & fwd+bwd at N=1e5; % of B200 bf16 tensor peak"
UNIT = "query-heads/s"
FWD_KERNEL_SOURCE = os.path.join(ROOT, "graph_transformer_sparse_kmip_b200", "csrc")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_inputs(w, rank: int):
    """This rank's batch: the workload's inputs drawn with a rank-specific
    seed, so ranks work on independent batches (weak scaling)."""
    return wl.make_inputs(w, with_grad_out=True, seed=w.seed + 7919 * rank)


def max_over_ranks(vals, ws: int, device):
    """Element-wise maximum of per-rank timings (the slowest rank sets the
    job's time); the identity for one rank."""
    vals = [float(v) for v in vals]
    if ws == 1:
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_throughput(units_per_rank: int, ws: int, ms_per_step: float) -> float:
    """Whole-job units per second: every rank's units over the slowest
    rank's time per step."""
    return units_per_rank * ws / (ms_per_step * 1e-3)


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def _score_flops(offsets: torch.Tensor, H: int, d: int) -> float:
    n = torch.diff(offsets.long()).double()
    return float(2.0 * d * H * (n * n).sum())


def _kernel_hash(names) -> str:
    h = hashlib.sha256()
    for n in names:
        h.update(open(os.path.join(FWD_KERNEL_SOURCE, n), "rb").read())
    return h.hexdigest()[:16]


def _traffic(kernel_key: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (else null)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p)).get(kernel_key)
    except Exception:
        return None
    if not d or d.get("source_sha") != _kernel_hash(d.get("sources", [])):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle sampling.  The sampler starts before the
    warm-up (its start-up costs host time and driver calls) and the summary
    keeps the samples whose timestamps fall inside the timed window
    (mark_start / mark_end)."""

    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: torch.device):
        self.idx = str(device.index or 0)
        try:  # nvidia-smi numbers GPUs physically; the UUID is unambiguous
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            if uuid:
                self.idx = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            pass
        self.proc = None
        self.window = None
        self.lines = []

    def mark_start(self):
        self.window = [datetime.datetime.now(), None]

    def mark_end(self):
        if self.window:
            self.window[1] = datetime.datetime.now()

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def _rows(self):
        rows = []
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f")
                rows.append((ts, float(f[2]), float(f[3]), f[6:10]))
            except ValueError:
                continue
        return rows

    def summary(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        rows = self._rows()
        window = "timed region"
        if self.window and self.window[1]:
            # a sample describes the 50 ms before it: keep those that end
            # inside the window, and the first one after it
            a, b = self.window
            inside = [r for r in rows if a <= r[0] <= b]
            after = [r for r in rows if r[0] > b][:1]
            sel = inside + after
            if not sel:
                sel, window = rows, "whole run (no sample in the timed region)"
        else:
            sel, window = rows, "whole run"
        if not sel:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        reasons = set()
        for r in sel:
            for nm, v in zip(names, r[3]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(r[1] for r in sel), "sm_max_mhz": sel[-1][2],
                "reasons": sorted(reasons), "samples": len(sel), "window": window}


def _flush(buf):
    buf.add_(1)  # read + write 256 MiB: evicts the 126 MB L2


GATE_CYCLES = 10_000_000  # about 5 ms at 1.97 GHz


def _flush_and_gate(buf):
    """Between timed steps, outside the events: flush the L2, then hold the
    stream in a short device-side spin, so that the step's start event and
    launches are all queued before the device reaches them.  A host stall
    (another process on the host's cores, the sampler's start-up) then
    delays the spin, not the timed kernels: the events measure device work
    alone."""
    _flush(buf)
    torch.cuda._sleep(GATE_CYCLES)


class SmClock:
    """Instantaneous SM clock through NVML (None when NVML is unavailable)."""

    def __init__(self, device: torch.device):
        self.h = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nv = pynvml
        except Exception:
            self.h = None

    def read(self):
        if self.h is None:
            return None
        try:
            return int(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        except Exception:
            return None


def _bwd_bytes_per_unit(d: int, k: int, elem: int) -> int:
    """Algorithmic bytes of the backward per (query, head): dO, Q rows
    (elem * d each), lse (4), idx (4k), the k kept K and V rows
    (2 k elem d), dQ (4d) and the fp32 dK/dV reductions (2 k 4 d, read and
    written by the reduction unit: counted once each)."""
    return 2 * elem * d + 4 + 4 * k + 2 * k * elem * d + 4 * d + 2 * k * 4 * d


def _gather_bytes_per_unit(d: int, k: int, elem: int) -> int:
    """Algorithmic bytes of the softmax + V gather per (query, head): the k
    kept V rows, idx and out written, lse written."""
    return k * (elem * d + 4) + elem * d + 4


class Case:
    """One workload's device inputs and output buffers."""

    def __init__(self, w, k, dev, rank=0, nodes=None):
        self.w, self.k = w, k
        self.inp = rank_inputs(w, rank) if nodes is None else None
        inp = self.inp
        N, H, d = inp["Q"].shape
        self.N, self.H, self.d = N, H, d
        self.bwd = "bwd" in w.phases
        self.g = {n: t.to(dev) for n, t in inp.items()}
        self.out = torch.empty_like(self.g["Q"])
        self.idx = torch.empty((N, H, k), dtype=torch.int32, device=dev)
        self.lse = torch.empty((N, H), dtype=torch.float32, device=dev)
        if self.bwd:
            self.dQ = torch.empty((N, H, d), dtype=torch.float32, device=dev)
            self.dK = torch.empty_like(self.dQ)
            self.dV = torch.empty_like(self.dQ)
        self.flops = _score_flops(inp["offsets"], H, d)
        self.scores = int(round(self.flops / (2 * d)))  # H * sum_g n_g^2 (query, key) pairs
        self.elem = self.g["Q"].element_size()

    def fwd(self, stream, k=None, idx=None):
        k = k or self.k
        idx = self.idx if idx is None else idx
        g = self.g
        rc = binding.kmip_attn_fwd(g["Q"], g["K"], g["V"], g["offsets"], self.N, self.H, self.d,
                                   k, self.w.scale, self.out, idx, self.lse, stream)
        if rc:
            raise binding.KmipError(rc, "kmip_attn_fwd")

    def bwd_call(self, stream, k=None, idx=None):
        k = k or self.k
        idx = self.idx if idx is None else idx
        g = self.g
        rc = binding.kmip_attn_bwd(g["dO"], g["Q"], g["K"], g["V"], idx, self.lse, self.dQ,
                                   self.dK, self.dV, stream, self.N, self.H, self.d, k,
                                   self.w.scale)
        if rc:
            raise binding.KmipError(rc, "kmip_attn_bwd")


def time_case(case, stream, steps, warmup, flush, clock=None, k=None, idx=None):
    """Per-step device times (ms) of the forward and the backward, each
    bracketed by CUDA events on the launching stream (torch's current
    stream), the L2 flushed and the stream gated between steps outside the
    events; the SM clock read after every step."""
    fwd_ms, bwd_ms, mhz = [], [], []
    for it in range(warmup + steps):
        e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        _flush_and_gate(flush)
        e0.record(stream)
        case.fwd(stream, k, idx)
        e1.record(stream)
        if case.bwd:
            case.bwd_call(stream, k, idx)
        e2.record(stream)
        torch.cuda.synchronize()
        if it >= warmup:
            fwd_ms.append(e0.elapsed_time(e1))
            bwd_ms.append(e1.elapsed_time(e2))
            mhz.append(clock.read() if clock else None)
    return fwd_ms, bwd_ms, mhz


def _filter_roofline(scores: int, ms: float, sms: int, mhz) -> dict:
    """The forward's second bound: its top-k filter reduces every score once
    on the ALU pipe (a group's maximum of 16 scores is 15 two-input maxima,
    or 8 three-input ones at half rate).  That pipe reduces 16 values per
    clock per SM sub-partition, 64 per SM: 148 x 64 x clock scores/s."""
    mhz = float(mhz or 1965.0)
    peak = sms * 64 * mhz * 1e6
    got = scores / (ms * 1e-3)
    return {"bound": "alu", "scores": scores, "scores_per_s": got, "peak_scores_per_s": peak,
            "frac": got / peak, "peak_from": f"{sms} SMs x 64 ALU lanes x {mhz:.0f} MHz"}


def _fp32_fma_peak_tflops(sms: int, mhz: float) -> float:
    """fp32 FMA peak of the fp32-input forward: 128 FMA lanes per SM per
    clock, 2 flops each."""
    return sms * 128 * 2 * mhz * 1e6 / 1e12


def config_summary(case, fwd_ms, bwd_ms, peaks, sms, max_mhz):
    N, H = case.N, case.H
    f = statistics.mean(fwd_ms)
    b = statistics.mean(bwd_ms)
    path = binding.kmip_fwd_path(case.d, case.k, binding.dtype_code(case.g["Q"].dtype))
    if path == 1:
        peak, bound = float(peaks["bf16_tflops"]), "tensor (bf16, burst peak)"
    else:
        peak, bound = _fp32_fma_peak_tflops(sms, max_mhz or 1965.0), "fp32 fma (derived peak)"
    ach = case.flops / (f * 1e-3) / 1e12
    r = {"N": N, "H": H, "d": case.d, "k": case.k, "graphs": int(case.g["offsets"].numel() - 1),
         "dtype": case.w.dtype, "steps": len(fwd_ms),
         "fwd": {"ms": f, "ms_min": min(fwd_ms), "ms_max": max(fwd_ms),
                 "query_heads_per_s": N * H / (f * 1e-3),
                 "score_tflops": ach, "peak_tflops": peak, "frac": ach / peak, "bound": bound,
                 "path": {1: "tcgen05 tensor cores", 0: "fp32 FMA"}.get(path, "?")}}
    if case.bwd:
        byts = N * H * _bwd_bytes_per_unit(case.d, case.k, case.elem)
        r["bwd"] = {"ms": b, "algorithmic_bytes": byts, "gbs": byts / (b * 1e-3) / 1e9,
                    "frac_hbm": byts / (b * 1e-3) / 1e9 / float(peaks["hbm_gbs"])}
        r["fwd_bwd_query_heads_per_s"] = N * H / ((f + b) * 1e-3)
    return r


def run_ours(args, ws, rank, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    binding.load()
    w = wl.WORKLOADS[args.workload]
    k = args.k or w.k
    case = Case(w, k, dev, rank)
    N, H, d = case.N, case.H, case.d
    inp, g = case.inp, case.g
    scale = w.scale
    stream = torch.cuda.current_stream()
    flush = torch.zeros(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    clock = SmClock(dev)

    clk = ClockSampler(dev).__enter__()
    for _ in range(args.warmup):
        case.fwd(stream)
        case.bwd_call(stream)
        _flush(flush)
    torch.cuda.synchronize()
    binding.check_status()

    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clk.mark_start()
    fwd_ms, bwd_ms, mhz = time_case(case, stream, args.steps, 0, flush, clock)
    torch.cuda.synchronize()
    if ws > 1:
        torch.distributed.barrier()
    clk.mark_end()
    time.sleep(0.15)  # one more sample after the window
    clk.__exit__(None, None, None)
    binding.check_status()
    tot_ms = [a + b for a, b in zip(fwd_ms, bwd_ms)]
    t_fwd, t_bwd, t_tot = max_over_ranks([sum(fwd_ms), sum(bwd_ms), sum(tot_ms)], ws, dev)
    ms_step = t_tot / args.steps
    ms_fwd = t_fwd / args.steps
    ms_bwd = t_bwd / args.steps
    value = job_throughput(N * H, ws, ms_step)
    fwd_value = job_throughput(N * H, ws, ms_fwd)
    idx_ref = case.idx.cpu()

    peaks, peak_kind = _peaks()
    flops = case.flops
    achieved = flops / (ms_fwd * 1e-3) / 1e12
    peak = float(peaks["bf16_tflops"])
    bwd_bytes = N * H * _bwd_bytes_per_unit(d, k, case.elem)
    clocks = clk.summary()

    # the softmax + V gather stage by itself (kmip_attn_gather over the
    # forward's sets): what the fused forward's last stage moves, plus the
    # K rows it needs to recompute the kept scores
    gat_ms = []
    o_g, l_g = torch.empty_like(case.out), torch.empty_like(case.lse)
    for it in range(3 + max(3, args.steps // 2)):
        _flush_and_gate(flush)
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        rc = binding.kmip_attn_gather(g["Q"], g["K"], g["V"], case.idx, N, H, d, k, scale, o_g,
                                      l_g, stream)
        b_.record(stream)
        if rc:
            raise binding.KmipError(rc, "kmip_attn_gather")
        torch.cuda.synchronize()
        if it >= 3:
            gat_ms.append(a_.elapsed_time(b_))
    gat_ms_mean = statistics.mean(gat_ms)
    # the deterministic backward (sorted gather, no atomics) on the same step
    det_ms = []
    for it in range(3 + max(3, args.steps // 2)):
        _flush_and_gate(flush)
        a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a_.record(stream)
        rc = binding.kmip_attn_bwd_deterministic(g["dO"], g["Q"], g["K"], g["V"], case.idx,
                                                 case.lse, case.dQ, case.dK, case.dV, stream,
                                                 N, H, d, k, scale)
        b_.record(stream)
        if rc:
            raise binding.KmipError(rc, "kmip_attn_bwd_deterministic")
        torch.cuda.synchronize()
        if it >= 3:
            det_ms.append(a_.elapsed_time(b_))
    binding.check_status()
    gat_bytes = N * H * (_gather_bytes_per_unit(d, k, case.elem) + k * case.elem * d + case.elem * d)
    del o_g, l_g

    # k sweep: forward and backward at the workload's other k values
    sweep = {}
    if args.k_sweep and w.k_sweep:
        nsw = max(3, args.steps // 4)
        for ks in w.k_sweep:
            if ks == k:
                sweep[str(ks)] = {"ms_fwd": ms_fwd, "ms_bwd": ms_bwd,
                                  "frac": achieved / peak}
                continue
            idx_s = torch.empty((N, H, ks), dtype=torch.int32, device=dev)
            f_ms, b_ms, _ = time_case(case, stream, nsw, 3, flush, None, ks, idx_s)
            fm = statistics.mean(f_ms)
            sweep[str(ks)] = {"ms_fwd": fm, "ms_bwd": statistics.mean(b_ms),
                              "frac": flops / (fm * 1e-3) / 1e12 / peak}
        binding.check_status()

    # the other workloads: forward (and backward where the workload has one)
    configs = {}
    if args.configs and rank == 0:
        for name, wo in wl.WORKLOADS.items():
            if name == w.name:
                continue
            c2 = Case(wo, wo.k, dev)
            f_ms, b_ms, _ = time_case(c2, stream, max(3, args.steps // 4), 3, flush)
            configs[name] = config_summary(c2, f_ms, b_ms, peaks, sms, clocks.get("sm_max_mhz"))
            del c2
        binding.check_status()

    # end to end through the public API: pinned host inputs in, host results out.
    # Steps are pipelined the way a serving loop runs them: two slots of device
    # buffers and three streams, so step s+1's host-to-device copy and step
    # s-1's device-to-host copy overlap step s's kernels; every step still
    # copies its own inputs in and its own results out.
    e2e = None
    if args.e2e:
        hostin = {n: inp[n].pin_memory() for n in ("Q", "K", "V", "dO")}
        off_h = inp["offsets"].pin_memory()
        names = {"out": case.out, "idx": case.idx, "lse": case.lse, "dQ": case.dQ,
                 "dK": case.dK, "dV": case.dV}
        hostout = [{n: torch.empty(t.shape, dtype=t.dtype).pin_memory() for n, t in names.items()}
                   for _ in range(2)]
        dIn = [{n: torch.empty_like(g[n]) for n in ("Q", "K", "V", "dO")} for _ in range(2)]
        dOff = [torch.empty_like(g["offsets"]) for _ in range(2)]
        dOut = [{n: torch.empty_like(t) for n, t in names.items()} for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in hostin.values()) + off_h.numel() * 4
        d2h = sum(t.numel() * t.element_size() for t in hostout[0].values())
        s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of a slot landed
        ev_run = [torch.cuda.Event() for _ in range(2)]    # kernels of a slot done
        ev_out = [torch.cuda.Event() for _ in range(2)]    # results of a slot copied out
        for e in ev_run + ev_out:
            e.record(s_run)

        def e2e_step(i):
            j = i % 2
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_run[j])          # slot j's inputs no longer read
                for n in dIn[j]:
                    dIn[j][n].copy_(hostin[n], non_blocking=True)
                dOff[j].copy_(off_h, non_blocking=True)
                ev_in[j].record(s_in)
            s_run.wait_event(ev_in[j])
            s_run.wait_event(ev_out[j])             # slot j's results copied out
            o = dOut[j]
            rc = binding.kmip_attn_fwd(dIn[j]["Q"], dIn[j]["K"], dIn[j]["V"], dOff[j], N, H, d,
                                       k, scale, o["out"], o["idx"], o["lse"], s_run)
            if rc:
                raise binding.KmipError(rc, "kmip_attn_fwd")
            rc = binding.kmip_attn_bwd(dIn[j]["dO"], dIn[j]["Q"], dIn[j]["K"], dIn[j]["V"],
                                       o["idx"], o["lse"], o["dQ"], o["dK"], o["dV"], s_run,
                                       N, H, d, k, scale)
            if rc:
                raise binding.KmipError(rc, "kmip_attn_bwd")
            ev_run[j].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_run[j])
                for n, t in o.items():
                    hostout[j][n].copy_(t, non_blocking=True)
                ev_out[j].record(s_out)

        for i in range(args.warmup):
            e2e_step(i)
        torch.cuda.synchronize()
        if ws > 1:
            torch.distributed.barrier()
        e_a, e_b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_a.record(s_in)
        s_run.wait_event(e_a)
        s_out.wait_event(e_a)
        for i in range(args.steps):
            e2e_step(i)
        s_out.wait_event(ev_run[(args.steps - 1) % 2])
        e_b.record(s_out)
        torch.cuda.synchronize()
        t_e2e = max_over_ranks([e_a.elapsed_time(e_b)], ws, dev)[0]
        binding.check_status()
        last = hostout[(args.steps - 1) % 2]
        if not torch.equal(last["idx"], idx_ref):
            raise RuntimeError("end-to-end results differ from the device-resident run")
        e2e = {"value": job_throughput(N * H, ws, t_e2e / args.steps), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": t_e2e / args.steps, "streams": "copy-in, kernels, copy-out"}

    cpu = None
    if rank == 0 and ws == 1 and args.cpu_baseline:
        cpu = cpu_baseline(inp, k, scale, budget_s=args.cpu_seconds)

    baselines = None
    if rank == 0 and args.baselines:
        baselines = comparison_baselines(case, stream, flush)

    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "N": N, "H": H, "d": d, "k": k,
                   "graphs": int(inp["offsets"].numel() - 1), "keys": w.values,
                   "step": "fwd+bwd", "parallelism": f"independent batch per GPU x{ws}",
                   "l2": "flushed between steps (256 MiB write, then a 5 ms device-side gate; both outside the timed events)"},
        "fwd": {"value": fwd_value, "unit": UNIT, "ms_per_step": ms_fwd},
        "roofline": {"bound": "tensor", "kernel": "forward (score + top-k + softmax + gather)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": _traffic("fwd"),
                     "peak_source": f"{peak_kind} bf16_tflops (burst)",
                     "algorithmic_flops_per_launch": flops,
                     "path": {1: "tcgen05 tensor cores", 0: "fp32 FMA"}.get(
                         binding.kmip_fwd_path(d, k, binding.dtype_code(g["Q"].dtype)), "?")},
        "phases": {
            "fwd": {"ms": ms_fwd, "score_tflops": achieved, "frac_bf16_peak": achieved / peak,
                    "gather_bytes_per_launch": N * H * _gather_bytes_per_unit(d, k, case.elem),
                    "topk_filter": _filter_roofline(case.scores, ms_fwd, sms,
                                                    clocks.get("sm_max_mhz"))},
            "gather_stage": {"kernel": "kmip_attn_gather (softmax + V gather over the forward's sets)",
                             "ms": gat_ms_mean, "algorithmic_bytes": gat_bytes,
                             "gbs": gat_bytes / (gat_ms_mean * 1e-3) / 1e9,
                             "frac_hbm": gat_bytes / (gat_ms_mean * 1e-3) / 1e9 / float(peaks["hbm_gbs"])},
            "bwd_deterministic": {"ms": statistics.mean(det_ms),
                                  "kernels": "coefficients + stable radix sort + in-order gather"},
            "bwd": {"ms": ms_bwd, "algorithmic_bytes": bwd_bytes,
                    "gbs": bwd_bytes / (ms_bwd * 1e-3) / 1e9,
                    "frac_hbm": bwd_bytes / (ms_bwd * 1e-3) / 1e9 / float(peaks["hbm_gbs"]),
                    "hbm_peak_gbs": float(peaks["hbm_gbs"]), "peak_source": peak_kind},
        },
        "per_step": {"ms_fwd": [round(x, 4) for x in fwd_ms],
                     "ms_bwd": [round(x, 4) for x in bwd_ms],
                     "sm_mhz_after_step": mhz},
        "gpu_launches": 3 * args.steps,
    }
    if sweep:
        res["k_sweep"] = sweep
    if configs:
        res["configs"] = configs
    if e2e:
        res["e2e"] = e2e
    if cpu:
        res["cpu_baseline"] = cpu
    if baselines:
        res["baselines"] = baselines
    res["clocks"] = clocks
    return res


def comparison_baselines(case, stream, flush, reps=3):
    """The two alternatives the k-MIP pages compare against (Figure 2,
    Tables 10-12), measured on the same inputs with torch's own kernels:
      full attention   softmax over every key of the graph (torch SDPA,
                       flash backend), forward and forward + backward;
      dense top-k      the non-symbolic k-MIP: the score matrix written to
                       HBM by a matmul, torch.topk over it, softmax over the
                       kept scores and a gather of V; done in blocks of query
                       rows so that the score block stays within a fixed
                       memory budget (the whole [H, N, N] fp32 matrix is
                       reported as what the unblocked form would need).
    Library kernels, reported next to the fused kernel for context; they
    are not part of the library's path.  Single-graph workloads only."""
    import torch.nn.functional as F
    g, N, H, d, k = case.g, case.N, case.H, case.d, case.k
    if case.g["offsets"].numel() != 2:
        return None
    scale = case.w.scale
    res = {}
    q = g["Q"].permute(1, 0, 2).unsqueeze(0)   # [1, H, N, d] views, last dim contiguous
    kk = g["K"].permute(1, 0, 2).unsqueeze(0)
    v = g["V"].permute(1, 0, 2).unsqueeze(0)

    def timed(fn):
        ts = []
        for it in range(reps + 1):
            _flush_and_gate(flush)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            if it:
                ts.append(a.elapsed_time(b))
        return statistics.mean(ts)

    try:
        with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.FLASH_ATTENTION):
            ms_f = timed(lambda: F.scaled_dot_product_attention(q, kk, v, scale=scale))
            qg, kg, vg = (x.detach().clone().requires_grad_(True) for x in (q, kk, v))
            do = g["dO"].permute(1, 0, 2).unsqueeze(0)

            def fb():
                o = F.scaled_dot_product_attention(qg, kg, vg, scale=scale)
                o.backward(do)
            ms_fb = timed(fb)
        res["full_attention_sdpa"] = {"ms_fwd": ms_f, "ms_fwd_bwd": ms_fb,
                                      "query_heads_per_s_fwd": N * H / (ms_f * 1e-3),
                                      "query_heads_per_s_fwd_bwd": N * H / (ms_fb * 1e-3)}
        del qg, kg, vg
    except Exception as e:  # noqa: BLE001
        res["full_attention_sdpa"] = {"unavailable": str(e).splitlines()[0][:200]}

    # Figure 8's two diagnostics: the share of the full softmax weight the k
    # kept keys carry, exp(lse - lse_all) with lse_all from the library's
    # all-key pass, and the L2 distance between k-MIP and full attention.
    try:
        out, idx, lse, lse_all = binding.attn_fwd_diag(g["Q"], g["K"], g["V"], k, scale,
                                                       g["offsets"], stream)
        with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.FLASH_ATTENTION):
            full = F.scaled_dot_product_attention(q, kk, v, scale=scale)[0].permute(1, 0, 2)
        share = torch.exp(lse.double() - lse_all.double())
        dist = (out.double() - full.double()).norm(dim=-1)
        rel = dist / full.double().norm(dim=-1).clamp_min(1e-30)
        res["figure8_diagnostics"] = {
            "topk_weight_share_mean": float(share.mean()), "topk_weight_share_min": float(share.min()),
            "l2_distance_mean": float(dist.mean()), "l2_distance_rel_mean": float(rel.mean()),
            "full_attention_from": "torch SDPA (flash)", "lse_all_from": "kmip_attn_fwd_diag"}
        ms_diag = timed(lambda: binding.attn_fwd_diag(g["Q"], g["K"], g["V"], k, scale,
                                                      g["offsets"], stream))
        res["figure8_diagnostics"]["ms_fwd_diag"] = ms_diag
        del out, idx, lse, lse_all, full
    except Exception as e:  # noqa: BLE001
        res["figure8_diagnostics"] = {"unavailable": str(e).splitlines()[0][:200]}

    block = max(1, min(N, (8 << 30) // (4 * H * N)))    # <= 8 GiB of fp32 scores per block
    Kh = g["K"].permute(1, 2, 0).float()               # [H, d, N]
    Vh = g["V"].permute(1, 0, 2).float()               # [H, N, d]

    def dense_topk():
        for i0 in range(0, N, block):
            Qb = g["Q"][i0:i0 + block].permute(1, 0, 2).float()   # [H, b, d]
            S = torch.bmm(Qb, Kh)                                  # [H, b, N] in HBM
            top, ti = torch.topk(S, k, dim=-1)
            p = torch.softmax(top * scale, dim=-1)
            Vg = torch.gather(Vh.unsqueeze(1).expand(H, Qb.shape[1], N, d), 2,
                              ti.unsqueeze(-1).expand(-1, -1, -1, d))
            torch.einsum("hbk,hbkd->hbd", p, Vg)
    try:
        torch.cuda.reset_peak_memory_stats(case.g["Q"].device)
        base = torch.cuda.memory_allocated(case.g["Q"].device)
        ms_d = timed(dense_topk)
        peak = torch.cuda.max_memory_allocated(case.g["Q"].device) - base
        res["dense_scores_topk"] = {"ms_fwd": ms_d, "query_heads_per_s_fwd": N * H / (ms_d * 1e-3),
                                    "query_block": block, "peak_extra_bytes": int(peak),
                                    "unblocked_score_bytes_fp32": 4 * H * N * N}
    except Exception as e:  # noqa: BLE001
        res["dense_scores_topk"] = {"unavailable": str(e).splitlines()[0][:200]}
    torch.cuda.empty_cache()
    return res


def cpu_baseline(inp, k, scale, budget_s=15.0, pairs_per_batch=None):
    """The fp64 oracle, as it stands, on a bounded sample of (query, head)
    pairs of the same workload: selection against all keys, softmax, V sum,
    then the backward over the sampled pairs' sets.  Returns fwd+bwd
    query-heads/s."""
    import numpy as np

    import oracle
    N, H = inp["Q"].shape[:2]
    threads = oracle.default_threads()
    Qd = oracle._f64(inp["Q"]); Kd = oracle._f64(inp["K"]); Vd = oracle._f64(inp["V"])
    dOd = oracle._f64(inp["dO"])
    per = pairs_per_batch or max(64, threads * 8)
    done, t_used, batch = 0, 0.0, 0
    while t_used < budget_s and done < N * H:
        pq, ph = wl.sample_pairs(N, H, per, seed=1000 + batch)
        t0 = time.perf_counter()
        r = oracle.fwd_pairs(Qd, Kd, Vd, inp["offsets"], k, scale, pq.numpy(), ph.numpy(),
                             nthreads=threads)
        full = np.full((N, H, k), -1, dtype=np.int32)
        full[pq.numpy(), ph.numpy()] = r["idx"]
        oracle.given_idx(Qd, Kd, Vd, full, inp["offsets"], scale, dO=dOd)
        t_used += time.perf_counter() - t0
        done += len(pq)
        batch += 1
    return {"value": done / t_used, "unit": UNIT, "cores": threads, "kind": "oracle",
            "pairs": done,
            "sample": f"{done} (query, head) pairs of the same workload in {batch} batches; "
                      f"fwd (all-key fp64 scores + full sort) and bwd; {t_used:.1f} s"}


def run_reference(args, ws, rank):
    """The oracle as the reference arm: each step is a bounded sample of
    (query, head) pairs of the same workload on the host cores.  value is
    the sampled pairs per second; ms_per_step is the real wall time of one
    sampled step (the full-step time it would take is reported apart)."""
    if rank != 0:
        return None
    w = wl.WORKLOADS[args.workload]
    k = args.k or w.k
    inp = wl.make_inputs(w, with_grad_out=True)
    N, H = inp["Q"].shape[:2]
    per_step_s = max(1.0, min(20.0, 120.0 / max(1, args.steps + args.warmup)))
    vals, samples, walls = [], [], []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        r = cpu_baseline(inp, k, w.scale, budget_s=per_step_s)
        wall = time.perf_counter() - t0
        if s >= args.warmup:
            vals.append(r["value"])
            samples.append(r)
            walls.append(wall)
    value = statistics.mean(vals)
    pairs = [r["pairs"] for r in samples]
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.mean(walls) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "N": N, "H": H, "d": w.d, "k": k,
                   "graphs": int(inp["offsets"].numel() - 1), "keys": w.values,
                   "step": "fwd+bwd", "parallelism": "host cores (oracle)",
                   "l2": "not applicable (host)"},
        "sample_pairs_per_step": statistics.mean(pairs),
        "full_step_ms_extrapolated": N * H / value * 1e3,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": samples[-1]["cores"],
                         "kind": "oracle",
                         "sample": f"{statistics.mean(pairs):.0f} (query, head) pairs per step on "
                                   f"average over {len(pairs)} steps (last step: "
                                   + samples[-1]["sample"] + ")"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_profile_calls(args):
    """A few forward calls of the workload and nothing else (with --profile-bwd:
    one forward, then that many backward calls): the command an ncu capture of
    one kernel runs (no timing loop, no baselines)."""
    import dataclasses
    w = wl.WORKLOADS[args.workload]
    if args.nodes:
        if w.sizes_range is not None:
            raise SystemExit("--nodes applies to single-graph workloads")
        w = dataclasses.replace(w, N=args.nodes)
    k = args.k or w.k
    dev = torch.device("cuda", 0)
    inp = wl.make_inputs(w, with_grad_out=args.profile_bwd)
    g = {n: t.to(dev) for n, t in inp.items()}
    if args.profile_bwd:
        out, idx, lse = binding.attn_fwd(g["Q"], g["K"], g["V"], k, w.scale, g["offsets"])
        for _ in range(args.profile_calls):
            binding.attn_bwd(g["dO"], g["Q"], g["K"], g["V"], idx, lse, w.scale)
    else:
        for _ in range(args.profile_calls):
            binding.attn_fwd(g["Q"], g["K"], g["V"], k, w.scale, g["offsets"])
    torch.cuda.synchronize()
    binding.check_status()
    print(json.dumps({"profile_calls": args.profile_calls, "workload": w.name, "N": w.N, "k": k,
                      "kernel": "bwd" if args.profile_bwd else "fwd"}))


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gmm_n100000", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--k", type=int, default=None)
    ap.add_argument("--no-k-sweep", dest="k_sweep", action="store_false")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip timing the other workloads")
    ap.add_argument("--no-baselines", dest="baselines", action="store_false",
                    help="skip the full-attention and dense top-k comparison kernels")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--nodes", type=int, default=None,
                    help="override N of a single-graph workload (profiling only)")
    ap.add_argument("--profile-calls", type=int, default=0,
                    help="run this many forward calls and exit (for ncu captures)")
    ap.add_argument("--profile-bwd", action="store_true",
                    help="with --profile-calls: one forward, then backward calls")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    ws, rank, local = _dist()
    if args.gpus != ws:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE is {ws}: launch N > 1 ranks with "
                 "torchrun (one process per GPU)")
    if args.profile_calls:
        run_profile_calls(args)
        return
    if args.impl == "reference":
        res = run_reference(args, ws, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if ws > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    try:
        res = run_ours(args, ws, rank, local)
    finally:
        if ws > 1:
            torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
