"""SSD forward benchmark (Mamba-2 SSD layer, forward pass) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload mamba2_2p7b] [--path auto|simt|tensor]

One step = one ssd_fwd over the whole workload (every kernel of the path).
Prints ONE JSON line on rank 0. For N > 1 (torchrun, one process per GPU)
every rank runs its own copy of the workload (independent problems: weak
scaling, no data-path collective); the step time is the max over ranks.

--impl reference times the fp64 CPU oracle (the slow, obviously-correct
recurrence) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import os
import signal
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import ssd_inputs  # noqa: E402

L2_FLUSH_BYTES = 512 << 20        # > 4x the 126 MB L2
METRIC = "SSD fwd tokens/s at 1 B200; % of BF16 tensor-core / HBM roofline"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0            # B200 HBM3e data-sheet bandwidth (8 TB/s), for context beside the measured peak
THROTTLE_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


# --------------------------------------------------------------- accounting

def algorithmic_bytes(inp: dict) -> int:
    """Compulsory I/O of one forward: x, y, dt, B, C (+ initial / final states)."""
    x, dt, B, C = inp["x"], inp["dt"], inp["B"], inp["C"]
    es = 2 if inp["io_dtype"] == "bf16" else 4
    n = (2 * x.size + dt.size + B.size + C.size) * es
    H, P, N = x.shape[2], x.shape[3], B.shape[3]
    nseq = inp["workload"].nseq
    if inp.get("initial_states") is not None:
        n += nseq * H * P * N * 4
    if inp.get("want_final_states"):
        n += nseq * H * P * N * 4
    return int(n)


def algorithmic_flops(inp: dict, block_len: int) -> int:
    """Useful (causal-halved) FLOPs of the chunked algorithm per forward:
    per token H * (4PN + Q*P) + G * Q * N, with Q the diagonal-block length the
    path actually evaluates (128 on the tensor-core path, chunk_len on the
    SIMT path)."""
    x, B = inp["x"], inp["B"]
    tokens = x.shape[0] * x.shape[1]
    H, P, G, N = x.shape[2], x.shape[3], B.shape[2], B.shape[3]
    Q = block_len
    return int(tokens * (H * (4 * P * N + Q * P) + G * Q * N))


def full_tile_flops(inp: dict, block_len: int) -> int:
    """The same with whole Q x Q diagonal tiles (no causal halving), the work a
    tiled evaluation issues: per token H * (4PN + 2QP) + 2GQN."""
    x, B = inp["x"], inp["B"]
    tokens = x.shape[0] * x.shape[1]
    H, P, G, N = x.shape[2], x.shape[3], B.shape[2], B.shape[3]
    Q = block_len
    return int(tokens * (H * (4 * P * N + 2 * Q * P) + 2 * G * Q * N))


def _code_only(text: str) -> str:
    """CUDA/C++ source without comments and with whitespace collapsed, so that
    editing a comment does not change the hash (the sources contain no comment
    markers inside string literals)."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


# the sources of the tensor-core forward kernels, whose DRAM traffic profiles/traffic.json records
TC_SOURCES = ("ssd_common.cuh", "ssd_tc.cu", "ssd_tc.cuh", "ssd_tc_prims.cuh")


def kernel_source_hash() -> str:
    """Hash of the tensor-core forward kernels' CUDA sources (code only): the
    committed ncu traffic figures apply while it matches."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mamba_ssd_layer_fwd_b200", "csrc")
    for fn in TC_SOURCES:
        h.update(fn.encode() + b"\0" + _code_only(open(os.path.join(csrc, fn)).read()).encode() + b"\0")
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def committed_traffic(workload: str, kernel: str):
    """dram read+write bytes per launch from the committed ncu summary, if it
    was taken on the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        e = d[workload]
        if e.get("kernel") == kernel and e.get("source_hash") == kernel_source_hash():
            return int(e["dram_bytes_per_launch"])
    except Exception:
        return None
    return None


# ------------------------------------------------------------------- clocks

class ClockSampler:
    def __init__(self, gpu_index: int):
        self.proc = None
        self.path = None
        self.gpu_index = gpu_index

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
            os.close(fd)
            q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.gpu_index)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.send_signal(signal.SIGTERM)
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 5:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), int(parts[4], 16)))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for _, _, bits in rows:
            for b, name in THROTTLE_BITS.items():
                if bits & b and name != "gpu_idle":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------ CPU baseline

def cpu_oracle_rate(inp: dict, budget_s: float = 10.0):
    """Time the fp64 oracle on the host cores on a bounded sample of
    (sequence, head) pairs; returns (tokens/s scaled to the full workload,
    cores, description)."""
    import oracle
    oracle.build()
    cores = oracle.max_threads()
    x = inp["x"]
    H = x.shape[2]
    bounds = ssd_inputs.seq_bounds(inp)
    order = [(s, h) for h in range(H) for s in range(len(bounds))]
    rng = np.random.default_rng(0)
    order = [order[i] for i in rng.permutation(len(order))]
    oracle.recurrence_pairs(inp, order[:1])             # warm (load, page in)
    done_tok = 0
    done_pairs = 0
    t_total = 0.0
    i = 0
    batch = cores
    while i < len(order) and t_total < budget_s:
        pairs = order[i:i + batch]
        t0 = time.perf_counter()
        oracle.recurrence_pairs(inp, pairs, nthreads=cores)
        dt = time.perf_counter() - t0
        t_total += dt
        done_tok += sum(bounds[s][1] for s, _ in pairs)
        done_pairs += len(pairs)
        i += len(pairs)
        if dt > 0 and t_total < budget_s:
            batch = max(cores, int(len(pairs) * min(4.0, (budget_s - t_total) / dt)))
    token_heads_per_s = done_tok / t_total
    desc = (f"{done_pairs} of {len(order)} (sequence, head) pairs ({done_tok} token-heads), "
            f"random order, full sequence length; tokens/s = token-heads/s / {H} heads")
    return token_heads_per_s / H, cores, desc, t_total


# ------------------------------------------------------------------ helpers

def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks of the default
    process group (identity without one). Every rank calls it at the same
    point, in warm-up, timing and error paths alike."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_throughput(tokens_per_rank: int, world: int, step_ms_max: float) -> float:
    """Weak scaling: every rank runs its own copy of the workload; the job's
    throughput is all ranks' tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (step_ms_max * 1e-3)


def make_workload(args):
    w = ssd_inputs.workload(args.workload)
    return ssd_inputs.make_inputs(w, seed=args.seed)


def config_of(inp, args, n_gpus):
    w = inp["workload"]
    return {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen, "num_seqs": w.num_seqs,
            "nheads": w.nheads, "headdim": w.headdim, "dstate": w.dstate, "ngroups": w.ngroups,
            "chunk_len": inp["chunk_len"], "io_dtype": w.io_dtype,
            "initial_states": bool(w.with_initial_states), "final_states": bool(w.with_final_states),
            "tokens_per_gpu": w.tokens, "parallelism": f"replicas x{n_gpus}" if n_gpus > 1 else "1 gpu",
            "l2": "flushed before every timed step (512 MiB write)", "path": args.path}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inp = make_workload(args)
    tokens = inp["x"].shape[0] * inp["x"].shape[1]
    per_step = []
    cores = 1
    desc = ""
    budget = max(1.0, min(args.ref_seconds, 150.0 / (args.warmup + args.steps)))
    for i in range(args.warmup + args.steps):
        rate, cores, desc, t = cpu_oracle_rate(inp, budget_s=budget)
        if i >= args.warmup:
            per_step.append(rate)
    value = float(statistics.median(per_step))
    line = {
        "impl": "reference", "metric": DECODE_METRIC if args.op == "decode" else METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * tokens / value, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": config_of(inp, args, 1),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": "each step: " + desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _device_inputs(inp, dev):
    """Pinned host copies and device copies of a workload's inputs."""
    import torch
    io = torch.bfloat16 if inp["io_dtype"] == "bf16" else torch.float32
    host = {k: torch.from_numpy(inp[k]).to(io).pin_memory() for k in ("x", "dt", "B", "C")}
    for k in ("A_log", "D", "initial_states"):
        host[k] = None if inp[k] is None else torch.from_numpy(inp[k]).pin_memory()
    host["cu_seqlens"] = None if inp["cu_seqlens"] is None else torch.from_numpy(inp["cu_seqlens"]).pin_memory()
    d = {k: (None if v is None else v.to(dev)) for k, v in host.items()}
    return host, d


def _stats(v):
    return {"mean": statistics.mean(v), "median": statistics.median(v), "min": min(v)}


class Forward:
    """One workload resident on the device, with its outputs, workspace and a
    step() that runs one ssd_fwd with events around the compute kernels."""

    def __init__(self, ssd, inp, dev, path, stream):
        import torch
        self.ssd, self.inp, self.path, self.stream = ssd, inp, path, stream
        self.host, self.d = _device_inputs(inp, dev)
        x = self.d["x"]
        nseq = inp["workload"].nseq
        H, P, N = x.shape[2], x.shape[3], self.d["B"].shape[3]
        self.y = torch.empty_like(x)
        self.fin = (torch.empty((nseq, H, P, N), dtype=torch.float32, device=dev)
                    if inp["want_final_states"] else None)
        self.params = ssd.params_for(x, self.d["B"], inp["chunk_len"], self.d["cu_seqlens"], True, path)
        self.ws = torch.empty(ssd.workspace_size(self.params), dtype=torch.uint8, device=dev)
        self.launches = ssd.launch_count(self.params)
        self.resolved = ssd.resolved_path(self.params)

    def step(self, events=None):
        d = self.d
        self.ssd.ssd_fwd(d["x"], d["dt"], d["A_log"], d["B"], d["C"], d["D"], chunk_len=self.inp["chunk_len"],
                         initial_states=d["initial_states"], cu_seqlens=d["cu_seqlens"], y=self.y,
                         final_states=self.fin, workspace=self.ws, stream=self.stream, path=self.path,
                         instrumentation=None if events is None else self.ssd.make_instrumentation(events))

    def status(self):
        return self.ssd.library().ssd_get_status(self.ws.data_ptr(), self.stream.cuda_stream or None)

    def timed(self, steps, warmup, flush, on_timed_start=None):
        """Warm-up, then `steps` timed steps (L2 flushed before each, unless
        `flush` is None: then what the last step left in L2 stays there);
        returns per-step lists of (step ms, compute ms, output-pass ms)."""
        import torch
        for _ in range(warmup):
            if flush is not None:
                flush.zero_()
            self.step()
        torch.cuda.synchronize()
        rc = self.status()
        if rc != 0:
            raise self.ssd.SsdError(rc, "warm-up device status")
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
        for row in ev:              # torch creates events lazily: record once so the handles exist
            for e in row:
                e.record(self.stream)
        torch.cuda.synchronize()
        if on_timed_start:
            on_timed_start()
        torch.cuda.synchronize()
        wall0 = time.perf_counter()
        for i in range(steps):
            if flush is not None:
                flush.zero_()
            ev[i][0].record(self.stream)
            self.step(events=(ev[i][1], ev[i][2], ev[i][3]))
            ev[i][4].record(self.stream)
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
        step_ms = [ev[i][0].elapsed_time(ev[i][4]) for i in range(steps)]
        comp_ms = [ev[i][1].elapsed_time(ev[i][3]) for i in range(steps)]
        main_ms = [ev[i][2].elapsed_time(ev[i][3]) for i in range(steps)]
        return step_ms, comp_ms, main_ms, wall

    def check(self, pairs_wanted=4, seed=1):
        """Output of the last call against the oracle on sampled (sequence,
        head) pairs: max|dy| / max|y_oracle| and the same for final states."""
        import torch
        import oracle
        torch.cuda.synchronize()
        inp = self.inp
        bounds = ssd_inputs.seq_bounds(inp)
        H, P = inp["x"].shape[2], inp["x"].shape[3]
        rng = np.random.default_rng(seed)
        cand = [(s, h) for s in range(len(bounds)) for h in range(H) if bounds[s][1] > 0]
        pick = [cand[i] for i in rng.choice(len(cand), size=min(pairs_wanted, len(cand)), replace=False)]
        ys, fs = oracle.recurrence_pairs(inp, pick)
        yg = self.y.float().cpu().numpy().reshape(-1, H, P)
        fg = None if self.fin is None else self.fin.cpu().numpy()
        ey = ef = 0.0
        for (s, h), yr, fr in zip(pick, ys, fs):
            t0, n = bounds[s]
            ey = max(ey, float(np.max(np.abs(yg[t0:t0 + n, h] - yr)) / max(np.max(np.abs(yr)), 1e-30)))
            if fg is not None:
                ef = max(ef, float(np.max(np.abs(fg[s, h] - fr)) / max(np.max(np.abs(fr)), 1e-30)))
        tol = 2e-2 if inp["io_dtype"] == "bf16" else 1e-4
        return {"pairs": [list(p) for p in pick], "max_rel_err_y": ey,
                "max_rel_err_final": ef if fg is not None else None, "tol": tol,
                "ok": bool(ey <= tol and ef <= tol)}

    def roofline(self, comp_ms, main_ms, workload_name):
        inp = self.inp
        alg_bytes = algorithmic_bytes(inp)
        peak, peak_kind = measured_peaks()
        # tensor path: the walk launches (ssd_tc_walk, and ssd_tc_fused for rows cut into segments)
        kernel = "ssd_tc_walk+fused" if self.resolved == "tensor" else "chunk_scan_kernel"
        cm = statistics.median(comp_ms)
        mm = statistics.median(main_ms)
        achieved = alg_bytes / (cm * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": committed_traffic(workload_name, kernel), "kernel": kernel,
                "kernel_ms": cm, "alg_bytes": alg_bytes,
                "timed": "every compute kernel of one forward (CUDA events on the call's stream, median)",
                "output_pass_ms": mm, "output_pass_frac": alg_bytes / (mm * 1e-3) / 1e9 / peak,
                "peak_source": f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                "spec_gbs": SPEC_HBM_GBS, "frac_of_spec": achieved / SPEC_HBM_GBS}


def warm_l2_stats(fw, steps):
    """The same forward timed without the L2 flush between steps, after the
    flushed measurement: inputs that fit in the 126 MB L2 (small_bf16's do)
    are then read from it.  Context only; a failure is reported in the line,
    never fatal to it."""
    try:
        s, c, m, _ = fw.timed(steps, 3, None)
    except Exception as e:  # noqa: BLE001 - reported in the JSON line
        return {"error": f"{type(e).__name__}: {e}"}
    return {"steps": steps, "step_ms": _stats(s), "compute_ms": _stats(c), "output_pass_ms": _stats(m)}


# bf16 workloads measured after the headline (one sub-object each in the JSON line)
SUB_WORKLOADS = ("small_bf16", "mamba2_2p7b", "long16k_gva", "varlen32k")


def run_ours(args):
    import torch
    import torch.distributed as dist
    import mamba_ssd_layer_fwd_b200 as ssd

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    inp = make_workload(args)
    stream = torch.cuda.current_stream()
    fw = Forward(ssd, inp, dev, args.path, stream)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    K = args.steps
    sampler = ClockSampler(torch.cuda.current_device() if world == 1 else local)

    def start_clocks():
        if rank == 0:
            sampler.start()
            time.sleep(0.3)
        if world > 1:
            dist.barrier()

    step_ms, comp_ms, main_ms, wall = fw.timed(K, args.warmup, flush, on_timed_start=start_clocks)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if rank == 0 else None
    ms, cms = max_over_ranks([statistics.mean(step_ms), statistics.median(comp_ms)], dev)
    check = fw.check() if rank == 0 else None

    # end to end: pinned host inputs -> device -> ssd_fwd -> result back to pinned host memory
    host, d, y, fin = fw.host, fw.d, fw.y, fw.fin
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    fin_host = torch.empty(fin.shape, dtype=fin.dtype).pin_memory() if fin is not None else None
    h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
    d2h = y_host.numel() * y_host.element_size() + (fin_host.numel() * 4 if fin_host is not None else 0)
    e2e_ms = []
    for i in range(args.warmup + min(K, 20)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.zero_()
        e0.record(stream)
        for k, v in host.items():
            if v is not None:
                d[k].copy_(v, non_blocking=True)
        fw.step()
        y_host.copy_(y, non_blocking=True)
        if fin_host is not None:
            fin_host.copy_(fin, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            e2e_ms.append(e0.elapsed_time(e1))
    e2e = max_over_ranks([statistics.mean(e2e_ms)], dev)[0]

    tokens = inp["x"].shape[0] * inp["x"].shape[1]
    value = whole_job_throughput(tokens, world, ms)
    block_len = 128 if fw.resolved == "tensor" else inp["chunk_len"]
    flops = algorithmic_flops(inp, block_len)
    roof = fw.roofline(comp_ms, main_ms, args.workload)
    roof["kernel_ms"] = cms
    roof["achieved"] = roof["alg_bytes"] / (cms * 1e-3) / 1e9
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["frac_of_spec"] = roof["achieved"] / SPEC_HBM_GBS
    warm = warm_l2_stats(fw, max(10, min(K, 50))) if world == 1 and not args.no_sub_workloads else None

    # the other workloads, one after another, after the headline's timed region (1 GPU only)
    subs = {}
    if args.workload in SUB_WORKLOADS and rank == 0:
        subs[args.workload] = {"steps": K, "step_ms": _stats(step_ms), "compute_ms": _stats(comp_ms),
                               "output_pass_ms": _stats(main_ms), "tokens_per_s": tokens / (statistics.median(step_ms) * 1e-3),
                               "frac": roof["frac"], "output_pass_frac": roof["output_pass_frac"],
                               "alg_bytes": roof["alg_bytes"], "traffic": roof["traffic"], "path": fw.resolved,
                               "launches": fw.launches, "check": check, "headline": True,
                               "frac_of_spec": roof["frac_of_spec"], "warm_l2": warm}
    if world == 1 and not args.no_sub_workloads:
        del fw
        torch.cuda.empty_cache()
        for name in SUB_WORKLOADS:
            if name == args.workload:
                continue
            sinp = ssd_inputs.make_inputs(ssd_inputs.workload(name), seed=args.seed)
            sfw = Forward(ssd, sinp, dev, "auto", stream)
            sk = max(10, min(K, 50))
            s_step, s_comp, s_main, _ = sfw.timed(sk, 3, flush)
            r = sfw.roofline(s_comp, s_main, name)
            s_check = sfw.check()
            s_warm = warm_l2_stats(sfw, sk)
            stoks = sinp["x"].shape[0] * sinp["x"].shape[1]
            subs[name] = {"steps": sk, "step_ms": _stats(s_step), "compute_ms": _stats(s_comp),
                          "output_pass_ms": _stats(s_main), "tokens_per_s": stoks / (statistics.median(s_step) * 1e-3),
                          "frac": r["frac"], "output_pass_frac": r["output_pass_frac"], "alg_bytes": r["alg_bytes"],
                          "traffic": r["traffic"], "path": sfw.resolved, "launches": sfw.launches,
                          "check": s_check, "frac_of_spec": r["frac_of_spec"], "warm_l2": s_warm}
            del sfw
            torch.cuda.empty_cache()

    backward = decode = None
    if world == 1 and not args.no_sub_workloads:
        backward = measure_backward(ssd, args, dev, flush)
        decode = measure_decode(ssd, args, dev, flush)

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            rate, cores, desc, _ = cpu_oracle_rate(inp, budget_s=args.ref_seconds)
            cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": inp["io_dtype"],
            "data": "synthetic (seeded generator, value distributions of the workload)",
            "config": config_of(inp, args, world),
            "step_ms": _stats(step_ms), "compute_ms": _stats(comp_ms), "output_pass_ms": _stats(main_ms),
            "roofline": roof,
            "tflops": flops / (ms * 1e-3) / 1e12, "flops_block_len": block_len,
            "tflops_full_tile": full_tile_flops(inp, block_len) / (ms * 1e-3) / 1e12,
            "check": check,
            "cpu_baseline": cpu,
            "e2e": {"value": whole_job_throughput(tokens, world, e2e), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": fw_launches(ssd, inp, args.path) * K,
            "clocks": clocks,
            "path": ssd.resolved_path(ssd.params_for(d["x"], d["B"], inp["chunk_len"], d["cu_seqlens"], True,
                                                     args.path)),
            "wall_s_timed_region": wall,
            "workloads": subs,
            "backward": backward,
            "decode": decode,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def backward_bytes(inp: dict) -> int:
    """Compulsory traffic of one backward: x, dt, B, C, dy read (io dtype),
    dx, ddt, dB, dC written (fp32), states read / gradients written."""
    x, dt, B = inp["x"], inp["dt"], inp["B"]
    es = 2 if inp["io_dtype"] == "bf16" else 4
    n = (2 * x.size + dt.size + 2 * B.size) * es + (x.size + dt.size + 2 * B.size) * 4
    H, P, N = x.shape[2], x.shape[3], B.shape[3]
    nseq = inp["workload"].nseq
    if inp.get("initial_states") is not None:
        n += 2 * nseq * H * P * N * 4
    return int(n)


def measure_backward(ssd, args, dev, flush, steps=10):
    """ssd_bwd on the headline workload after the timed forward region:
    median device time of `steps` calls (L2 flushed before each), the output
    checked against the gradient oracle on one sampled sequence."""
    import torch
    import oracle
    inp = make_workload(args)
    if inp["io_dtype"] != "bf16":
        return None
    host, d = _device_inputs(inp, dev)
    rng = np.random.default_rng(1)
    dy = ssd_inputs.round_to_bf16(rng.standard_normal(inp["x"].shape).astype(np.float32))
    dy_t = torch.from_numpy(dy).to(dev, torch.bfloat16)
    stream = torch.cuda.current_stream()

    def run():
        return ssd.ssd_bwd(d["x"], d["dt"], d["A_log"], d["B"], d["C"], d["D"], dy_t,
                           initial_states=d["initial_states"], cu_seqlens=d["cu_seqlens"], stream=stream)

    for _ in range(2):
        flush.zero_()
        g = run()
    torch.cuda.synchronize()
    ms = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g = run()
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    # check one sequence (all its heads) against the gradient oracle
    bounds = ssd_inputs.seq_bounds(inp)
    t0, n = bounds[0]
    one = dict(inp, x=inp["x"].reshape(-1, *inp["x"].shape[2:])[t0:t0 + n][None],
               dt=inp["dt"].reshape(-1, inp["dt"].shape[2])[t0:t0 + n][None],
               B=inp["B"].reshape(-1, *inp["B"].shape[2:])[t0:t0 + n][None],
               C=inp["C"].reshape(-1, *inp["C"].shape[2:])[t0:t0 + n][None],
               initial_states=None if inp["initial_states"] is None else inp["initial_states"][:1],
               cu_seqlens=None)
    want = oracle.recurrence_grad(one, dy.reshape(-1, *dy.shape[2:])[t0:t0 + n][None])
    errs = {}
    for k, kw in (("dx", "dx"), ("ddt", "ddt"), ("dB", "dB"), ("dC", "dC")):
        got = g[k].reshape(-1, *g[k].shape[2:])[t0:t0 + n].double().cpu().numpy()
        w = want[kw][0]
        errs[k] = float(np.abs(got - w).max() / max(np.abs(w).max(), 1e-30))
    tokens = inp["x"].shape[0] * inp["x"].shape[1]
    med = statistics.median(ms)
    nb = backward_bytes(inp)
    peak, _ = measured_peaks()
    return {"workload": inp["workload"].name, "ms": _stats(ms), "tokens_per_s": tokens / (med * 1e-3),
            "alg_bytes": nb, "frac_hbm": nb / (med * 1e-3) / 1e9 / peak, "path": "simt (CUDA cores, fp32)",
            "check": {"sequence": 0, "max_rel_err": errs, "tol": 1e-3,
                      "ok": bool(max(errs.values()) <= 1e-3)}}


def measure_decode(ssd, args, dev, flush, steps=50):
    """One ssd_decode_step over every row of decode_2p7b (64 rows of the 2.7B
    layer shape, state resident), L2 flushed before each timed step; the
    first step's y and state checked against the oracle's recurrence."""
    import torch
    import oracle
    inp = ssd_inputs.make_inputs(ssd_inputs.workload("decode_2p7b"), seed=args.seed)
    d = {k: torch.from_numpy(np.ascontiguousarray(inp[k][:, 0])).to(dev, torch.bfloat16) for k in ("x", "dt", "B", "C")}
    A_log = torch.from_numpy(inp["A_log"]).to(dev)
    D = torch.from_numpy(inp["D"]).to(dev)
    state0 = torch.from_numpy(inp["initial_states"]).to(dev)
    state = state0.clone()
    y = torch.empty_like(d["x"])
    stream = torch.cuda.current_stream()
    ssd.ssd_decode_step(d["x"], d["dt"], A_log, d["B"], d["C"], D, state, y=y, stream=stream)
    torch.cuda.synchronize()
    y_ref, fin_ref = oracle.recurrence(inp)
    ey = float(np.abs(y.double().cpu().numpy() - y_ref[:, 0]).max() / np.abs(y_ref).max())
    ef = float(np.abs(state.double().cpu().numpy() - fin_ref).max() / np.abs(fin_ref).max())
    ms = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        ssd.ssd_decode_step(d["x"], d["dt"], A_log, d["B"], d["C"], D, state, y=y, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    med = statistics.median(ms)
    nb = decode_bytes(inp)
    peak, _ = measured_peaks()
    rows = inp["x"].shape[0]
    return {"workload": "decode_2p7b", "ms": _stats(ms), "tokens_per_s": rows / (med * 1e-3), "alg_bytes": nb,
            "frac_hbm": nb / (med * 1e-3) / 1e9 / peak,
            "check": {"max_rel_err_y": ey, "max_rel_err_state": ef, "tol": 2e-2, "ok": bool(ey <= 2e-2 and ef <= 2e-2)}}


def fw_launches(ssd, inp, path):
    w = inp["workload"]
    p = ssd.make_params(batch=w.batch, seqlen=w.seqlen, nheads=w.nheads, headdim=w.headdim, dstate=w.dstate,
                        ngroups=w.ngroups, chunk_len=inp["chunk_len"], num_seqs=w.num_seqs, io_dtype=w.io_dtype,
                        path=path)
    return ssd.launch_count(p)


DECODE_METRIC = "SSD decode step tokens/s at 1 B200; % of HBM roofline"


def decode_bytes(inp: dict) -> int:
    """Compulsory traffic of one decoding step: the fp32 state read and
    written, plus x, y, dt, B, C of the new token."""
    x, B = inp["x"], inp["B"]
    b, H, P = x.shape[0], x.shape[2], x.shape[3]
    G, N = B.shape[2], B.shape[3]
    es = 2 if inp["io_dtype"] == "bf16" else 4
    return int(2 * b * H * P * N * 4 + (2 * b * H * P + b * H + 2 * b * G * N) * es)


def run_backward(args):
    """The backward sub-object alone (one GPU): `ssd_bwd` on the workload, with
    the same timing and check as in the forward's JSON line."""
    import torch
    import mamba_ssd_layer_fwd_b200 as ssd
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    b = measure_backward(ssd, args, dev, flush, steps=args.steps)
    print(json.dumps({"op": "backward", **(b or {"unavailable": "the workload is not bf16"})}))
    return 0


def run_decode(args):
    """One `ssd_decode_step` per step over every row of the decode workload
    (the state stays resident on the device, as in serving)."""
    import torch
    import torch.distributed as dist
    import mamba_ssd_layer_fwd_b200 as ssd

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    inp = ssd_inputs.make_inputs(ssd_inputs.workload(args.workload), seed=args.seed)
    if inp["x"].shape[1] != 1:
        raise SystemExit("--op decode needs a one-token workload (decode_2p7b)")
    io = torch.bfloat16 if inp["io_dtype"] == "bf16" else torch.float32
    host = {k: torch.from_numpy(np.ascontiguousarray(inp[k][:, 0])).to(io).pin_memory()
            for k in ("x", "dt", "B", "C")}
    d = {k: v.to(dev) for k, v in host.items()}
    A_log = torch.from_numpy(inp["A_log"]).to(dev)
    D = torch.from_numpy(inp["D"]).to(dev)
    state = torch.from_numpy(inp["initial_states"]).to(dev)
    y = torch.empty_like(d["x"])
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        ssd.ssd_decode_step(d["x"], d["dt"], A_log, d["B"], d["C"], D, state, y=y, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for row in ev:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device() if world == 1 else local)
    if rank == 0:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    wall0 = time.perf_counter()
    for i in range(K):
        flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    wall = time.perf_counter() - wall0
    clocks = sampler.stop() if rank == 0 else None
    ms = max_over_ranks([statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(K))], dev)[0]

    # end to end: the new token's inputs from pinned host memory, y back to the host
    y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = y_host.numel() * y_host.element_size()
    e2e_ms = []
    for i in range(args.warmup + K):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.zero_()
        e0.record(stream)
        for k, v in host.items():
            d[k].copy_(v, non_blocking=True)
        step()
        y_host.copy_(y, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= args.warmup:
            e2e_ms.append(e0.elapsed_time(e1))
    e2e = max_over_ranks([statistics.mean(e2e_ms)], dev)[0]

    rows = inp["x"].shape[0]
    value = whole_job_throughput(rows, world, ms)
    nbytes = decode_bytes(inp)
    peak, peak_kind = measured_peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            rate, cores, desc, _ = cpu_oracle_rate(inp, budget_s=args.ref_seconds)
            cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}
        w = inp["workload"]
        line = {
            "metric": DECODE_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": inp["io_dtype"],
            "data": "synthetic (seeded generator, value distributions of the workload)",
            "config": {"workload": w.name, "rows": rows, "nheads": w.nheads, "headdim": w.headdim,
                       "dstate": w.dstate, "ngroups": w.ngroups, "io_dtype": w.io_dtype,
                       "state": "fp32, resident, updated in place",
                       "parallelism": f"replicas x{world}" if world > 1 else "1 gpu",
                       "l2": "flushed before every timed step (512 MiB write)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None, "kernel": "ssd_decode_kernel",
                         "kernel_ms": ms, "alg_bytes": nbytes,
                         "peak_source": f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"},
            "cpu_baseline": cpu,
            "e2e": {"value": whole_job_throughput(rows, world, e2e), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": K,
            "clocks": clocks,
            "wall_s_timed_region": wall,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mamba2_2p7b", choices=sorted(ssd_inputs.WORKLOADS))
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tensor"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--ref-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub-workloads", action="store_true",
                    help="skip the per-workload measurements that follow the headline")
    ap.add_argument("--op", choices=["fwd", "decode", "backward"], default="fwd",
                    help="fwd: the chunked forward (default); decode: one recurrent step per row; "
                         "backward: ssd_bwd alone on the workload (its sub-object, printed as one JSON line)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)      # at least 3 untimed warm-up steps
    if args.op == "decode" and args.workload == "mamba2_2p7b":
        args.workload = "decode_2p7b"
    if args.impl == "reference":
        return run_reference(args)
    if args.op == "decode":
        return run_decode(args)
    if args.op == "backward":
        return run_backward(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
