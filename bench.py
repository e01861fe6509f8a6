#!/usr/bin/env python
"""Benchmark of the streaming lightning-indexer top-k on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload v4flash]

One step = one si_indexer_topk call over the whole workload (score every
causally visible (query, key) pair with 64 indexer heads, keep the top-512
per query).  Default workload: the V4-Flash shape, B=1, S=65,536, m=4
(T=16,384), H_I=64, D=128, k=512, planted-boost Gaussian inputs, seed 3.
Inputs are synthetic and resident in HBM before timing; q (1 GiB) exceeds the
126 MB L2 and L2 is also flushed before every timed step.

Under torchrun (N>1) each rank runs its own independent sequence of the same
shape (weak scaling, no collective on the data path); the timing is the max
over ranks.  `--impl reference` times the CPU oracle instead, on rank 0 only,
on a bounded sample of query rows per step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "visible q·k pairs/s (TFLOP/s, % bf16 TC peak) at S=65,536; peak HBM GB"
FLOP_PER_PAIR = None  # 2 * H_I * D, set per workload


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def measure_fp8_peak(dev) -> float | None:
    """Dense e4m3 matmul throughput of this GPU (torch._scaled_mm, 8192^3,
    bf16 output, best of 10 after 3 warm-ups, CUDA events): the denominator
    of the e4m3 roofline.  None when the probe is unavailable."""
    import torch
    try:
        n = 8192
        a = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), device=dev).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev, dtype=torch.float32)
        best = None
        for i in range(13):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize(dev)
            if i >= 3:
                t = e0.elapsed_time(e1)
                best = t if best is None else min(best, t)
        del a, b
        return 2.0 * n ** 3 / (best * 1e-3) / 1e12
    except Exception:  # noqa: BLE001 -- an unavailable probe falls back to the nominal ratio
        return None


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in ("si_stream.cu", "si_topk.cuh", "si_ptx.cuh"):
        h.update(open(os.path.join(ROOT, "streaming_top_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per launch of the streaming kernel from the committed ncu
    summary, if it was taken on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "stream_topk_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("kernel_source_hash") != kernel_source_hash():
        return None
    return d.get("per_launch_dram_bytes", {}).get(workload)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons)}


def config_dict(wl, n_gpus: int, shard: str = "seq", bounds=None) -> dict:
    c = {"workload": f"{wl.name}: B={wl.B}, S={wl.S}, m={wl.m} (T={wl.T}), H_I={wl.H}, D={wl.D}, "
                     f"k={wl.k}, {wl.kind} inputs, seed {wl.seed}",
         "B_per_gpu": wl.B, "S": wl.S, "T": wl.T, "H_I": wl.H, "D": wl.D, "m": wl.m, "k": wl.k,
         "visible_pairs_per_gpu": wl.visible_pairs(), "parallelism": f"independent sequences x{n_gpus}",
         "l2": "q (1 GiB) > L2, and L2 flushed before each timed step"}
    if shard == "rows":
        c["parallelism"] = f"row shards x{n_gpus} of the same sequences (equal visible pairs, keys replicated)"
        c["row_bounds"] = bounds
        c["visible_pairs_total"] = wl.visible_pairs()
        c["visible_pairs_per_gpu"] = wl.visible_pairs() / n_gpus
    return c


def shard_pairs(wl, r0: int, r1: int) -> int:
    """Visible pairs of query rows r0 .. r1-1 over the B sequences."""
    return wl.B * (synth.visible_pairs(r1, wl.T, wl.m) - synth.visible_pairs(r0, wl.T, wl.m))


# ------------------------------------------------------------------ CPU oracle
def rank_seed(wl, rank: int) -> int:
    """Each rank runs its own independent sequences of the same shape."""
    return wl.seed + 1000 * rank


def max_over_ranks(x: float, device) -> float:
    """The slowest rank's figure (all ranks must call this, in the same order)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, pairs_per_rank: int, ms_step: float) -> float:
    """Whole-job throughput: every rank's pairs over the slowest rank's time."""
    return world * pairs_per_rank / (ms_step * 1e-3)


TWO_STAGE = {"block": 8, "n_keep": 2048}  # the V4.1-Flash indexer's candidate stage: 2048 blocks of 8
TWO_STAGE_CHUNK = 65536


def two_stage_pairs(wl) -> tuple[int, int]:
    """(coarse pairs, fine pairs) the two-stage path scores: per row, the
    complete visible blocks, and the kept blocks' keys plus the incomplete
    block's visible keys."""
    t = np.arange(wl.S, dtype=np.int64)
    n = np.minimum(wl.T, (t + 1) // wl.m)
    nbv = n // TWO_STAGE["block"]
    fine = np.minimum(nbv, TWO_STAGE["n_keep"]) * TWO_STAGE["block"] + (n - nbv * TWO_STAGE["block"])
    return wl.B * int(nbv.sum()), wl.B * int(fine.sum())


def oracle_sample(wl, inp, rows, two_stage: bool = False) -> tuple[float, int]:
    import oracle
    t0 = time.perf_counter()
    if two_stage:
        oracle.topk_two_stage(inp["q"], inp["kc"], inp["w"], wl.m, wl.k, G=TWO_STAGE["block"],
                              n_keep=TWO_STAGE["n_keep"], rows=rows)
        dt = time.perf_counter() - t0
        return dt, int(sum(min(wl.T, (int(r) % wl.S + 1) // wl.m) for r in rows))
    oracle.topk(inp["q"], inp["kc"], inp["w"], wl.m, wl.k, rows=rows, q_scale=inp.get("q_scale"),
                kc_scale=inp.get("kc_scale"), kc_mx_scale=inp.get("kc_mx_scale"))
    dt = time.perf_counter() - t0
    pairs = int(sum(min(wl.T, (int(r) % wl.S + 1) // wl.m) for r in rows))
    return dt, pairs


def oracle_all_cores(wl, inp, two_stage: bool, seconds: float) -> dict:
    """The same oracle, unchanged, on every host core: one thread per core,
    each running the C oracle (which releases the GIL) on its own 16-row
    groups of uniformly sampled rows, for about `seconds` of wall time."""
    import threading
    cores = os.cpu_count() or 1
    rows = synth.sample_rows(16 * 64 * cores, wl.m * 4, wl.S, seed=wl.seed + 98)
    np.random.default_rng(wl.seed).shuffle(rows)
    lock = threading.Lock()
    state = {"next": 0, "pairs": 0, "rows": 0}
    t_end = time.perf_counter() + seconds

    def worker():
        while time.perf_counter() < t_end:
            with lock:
                i = state["next"]
                state["next"] += 16
            if i >= len(rows):
                return
            _, pr = oracle_sample(wl, inp, np.sort(rows[i:i + 16]), two_stage)
            with lock:
                state["pairs"] += pr
                state["rows"] += 16

    t0 = time.perf_counter()
    threads = [threading.Thread(target=worker) for _ in range(cores)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    dt = time.perf_counter() - t0
    return {"value": state["pairs"] / dt, "unit": "pairs/s", "cores": cores, "kind": "oracle",
            "sample": f"{state['rows']} uniformly sampled query rows of the {wl.name} workload ({state['pairs']} "
                      f"visible pairs, {dt:.1f} s wall), the C oracle unchanged on {cores} threads, one per "
                      "host core, fp64, full sort"}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    inp = synth.make_inputs(wl, fmt=args.fmt)
    per_step = args.ref_rows
    allrows = synth.sample_rows(per_step * (args.steps + args.warmup), wl.m * 4, wl.S, seed=wl.seed + 77)
    rng = np.random.default_rng(wl.seed)
    rng.shuffle(allrows)
    times, pairs = [], []
    for i in range(args.warmup + args.steps):
        rows = np.sort(allrows[i * per_step:(i + 1) * per_step])
        dt, pr = oracle_sample(wl, inp, rows, args.method == "two-stage")
        if i >= args.warmup:
            times.append(dt)
            pairs.append(pr)
    tot_t, tot_p = sum(times), sum(pairs)
    value = tot_p / tot_t
    ref_bounds = None
    if args.shard == "rows":
        import streaming_top_b200 as si  # the row partition only (host arithmetic)
        ref_bounds = si.row_shards(wl.S, wl.T, wl.m, args.gpus)
    line = {
        "metric": METRIC, "value": value, "unit": "pairs/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True,
        "scaling": "strong" if args.shard == "rows" else "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(wl, args.gpus, args.shard, ref_bounds), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "pairs/s", "cores": 1, "kind": "oracle",
                         "sample": f"{per_step} sampled query rows per step of the {wl.name} workload "
                                   f"({tot_p // args.steps} visible pairs per step on average), "
                                   "single-threaded C oracle, fp64, full sort"},
        "e2e": {"value": value, "unit": "pairs/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------- million-token record
def million_record(args, dev, sampler_index: int) -> dict:
    """The million-token workload (B=1, S=1,048,576, T=262,144, k=512, planted
    inputs, seed 4) beside the headline: one streaming call per format (bf16,
    e4m3 with per-row scales) with all inputs resident, W=1 + K=2 timed calls,
    and the bf16 call once more end to end through si_indexer_topk_host (host
    buffers, query chunks streamed through the device).  Peak HBM is the
    path's own device memory: inputs, outputs and library scratch."""
    import torch

    import streaming_top_b200 as si
    wl = synth.WORKLOADS["million"]
    B, S, T, H, D, k = wl.B, wl.S, wl.T, wl.H, wl.D, wl.k
    P = wl.visible_pairs()
    flop = P * 2 * H * D
    peaks = load_peaks()
    fp8_peak = measure_fp8_peak(dev)
    out = {"workload": f"million: B={B}, S={S}, m={wl.m} (T={T}), H_I={H}, D={D}, k={k}, planted inputs, "
                       f"seed {wl.seed}", "visible_pairs": P, "calls": "1 warm-up + 2 timed per format"}
    stream = torch.cuda.current_stream(dev)
    chunk = 16384
    # bf16 q in page-locked host memory (also the host-buffer call's input)
    hq = torch.empty((B, S, H, D), dtype=torch.int16).pin_memory()
    hqn = hq.numpy().view(np.uint16)
    for t0 in range(0, S, chunk):
        synth.q_rows(wl, 0, t0, min(chunk, S - t0), "bf16", out=hqn[0, t0:t0 + chunk])
    for fmt in ("bf16", "e4m3"):
        rest = synth.make_inputs(wl, fmt=fmt, skip_q=True)
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
        base_mem = torch.cuda.memory_allocated(dev)
        torch.cuda.reset_peak_memory_stats(dev)
        if fmt == "bf16":
            q = hq.to(dev, non_blocking=True).view(torch.bfloat16)
            kc = torch.from_numpy(rest["kc"].view(np.int16)).view(torch.bfloat16).to(dev)
            qs = ks = None
        else:
            q = torch.empty((B, S, H, D), dtype=torch.uint8, device=dev)
            qs = torch.empty((B, S, H), dtype=torch.float32, device=dev)
            buf = torch.empty((chunk, H, D), dtype=torch.uint8).pin_memory()
            sbuf = torch.empty((chunk, H), dtype=torch.float32).pin_memory()
            for t0 in range(0, S, chunk):
                n = min(chunk, S - t0)
                torch.cuda.synchronize(dev)
                synth.q_rows(wl, 0, t0, n, "e4m3", out=buf.numpy()[:n], scale_out=sbuf.numpy()[:n])
                q[0, t0:t0 + n].copy_(buf[:n], non_blocking=True)
                qs[0, t0:t0 + n].copy_(sbuf[:n], non_blocking=True)
            kc = torch.from_numpy(rest["kc"]).to(dev)
            ks = torch.from_numpy(rest["kc_scale"]).to(dev)
        w = torch.from_numpy(rest["w"]).to(dev)
        oi = torch.empty((B, S, k), dtype=torch.int32, device=dev)
        osc = torch.empty((B, S, k), dtype=torch.float32, device=dev)
        torch.cuda.synchronize(dev)
        path_bytes = sum(t.numel() * t.element_size() for t in (q, qs, kc, ks, w, oi, osc) if t is not None)

        def call(mid=None):
            si.indexer_topk(q, kc, w, wl.m, k, q_scale=qs, kc_scale=ks, out_idx=oi, out_score=osc, unsorted=True,
                            stream=stream)
            if mid is not None:
                mid.record(stream)
            si.sort_topk_rows(oi, osc, stream=stream)

        call()
        sampler = ClockSampler(sampler_index)
        sampler.start()
        time.sleep(0.3)
        evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(2)]
        for e0, em, e1 in evs:
            e0.record(stream)
            call(em)
            e1.record(stream)
        torch.cuda.synchronize(dev)
        clocks = sampler.stop()
        if si.device_status(stream) != si.SI_OK:
            raise RuntimeError(f"device error in the million-token {fmt} calls")
        ms = sum(a.elapsed_time(b) for a, _, b in evs) / len(evs)
        ms_k = sum(a.elapsed_time(b) for a, b, _ in evs) / len(evs)
        if fmt == "e4m3" and fp8_peak:
            peak_tc, peak_src = fp8_peak, "measured in this run: torch._scaled_mm e4m3 8192^3, burst"
        else:
            peak_tc = peaks["bf16_tflops"] * (2.0 if fmt == "e4m3" else 1.0)
            peak_src = (f"{peaks['source']} bf16 dense matmul, burst" +
                        (" x2 (nominal fp8 / bf16 dense ratio)" if fmt == "e4m3" else ""))
        rec = {"ms_per_call": ms, "kernel_ms": ms_k, "pairs_per_s": P / (ms * 1e-3),
               "tflops": flop / (ms * 1e-3) / 1e12,
               "frac_peak": flop / (ms * 1e-3) / 1e12 / peak_tc,
               "kernel_frac_peak": flop / (ms_k * 1e-3) / 1e12 / peak_tc,
               "peak": peak_tc, "peak_source": peak_src,
               "peak_hbm_gb": (torch.cuda.max_memory_allocated(dev) - base_mem) / 1e9,
               "hbm_breakdown_gb": {"q": (q.numel() * q.element_size() + (qs.numel() * 4 if qs is not None else 0))
                                    / 1e9, "kc": kc.numel() * kc.element_size() / 1e9, "w": w.numel() * 4 / 1e9,
                                    "out_idx + out_score": 2 * oi.numel() * 4 / 1e9, "library_workspace": 0.0},
               "path_bytes_gb": path_bytes / 1e9, "clocks": clocks}
        out[fmt] = rec
        del q, qs, kc, ks, w, oi, osc
        torch.cuda.empty_cache()
    # the same bf16 workload end to end from host buffers: only the keys and
    # two chunks of query rows are ever on the device
    rest = synth.make_inputs(wl, fmt="bf16", skip_q=True)
    hk = torch.from_numpy(rest["kc"].view(np.int16)).view(torch.bfloat16).pin_memory()
    hw = torch.from_numpy(rest["w"]).pin_memory()
    hqb = hq.view(torch.bfloat16)
    h_idx = torch.empty((B, S, k), dtype=torch.int32).pin_memory()
    h_sc = torch.empty((B, S, k), dtype=torch.float32).pin_memory()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    si.indexer_topk_host(hqb, hk, hw, wl.m, k, out_idx=h_idx, out_score=h_sc, stream=stream, device=dev)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    dev_bytes = si.indexer_topk_host_workspace_size(B, S, T, H, D, k)
    out["bf16_host_streamed"] = {
        "api": "si_indexer_topk_host (C ABI): host q, kc, w in, host results out; 4096-row query chunks through "
               "two device slots, copies overlapped with the scoring",
        "ms_per_call": e0.elapsed_time(e1), "pairs_per_s": P / (e0.elapsed_time(e1) * 1e-3),
        "peak_hbm_gb": dev_bytes / 1e9,
        "h2d_bytes": hq.numel() * 2 + hk.numel() * 2 + hw.numel() * 4, "d2h_bytes": 2 * B * S * k * 4,
        "calls": "1 (after the device-resident calls)"}
    out["pages_context"] = ("StreamIndex (abstract) reports 6.21 GB peak at S=1,048,576 on one H200 for the indexer "
                            "step, without saying how q is held; here the resident path holds q (16 GiB bf16), all "
                            "outputs (4 GiB) and no scratch, the host-streamed path only the keys and two query "
                            "chunks")
    del hq, hqn, hk, hw, h_idx, h_sc
    return out


# ------------------------------------------------------------------ CUDA path
def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    import streaming_top_b200 as si

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    fp8 = args.fmt == "e4m3"
    mx = args.fmt == "mxfp4"  # bf16 queries, MXFP4 keys (decoded to bf16 inside the call)
    rows_mode = args.shard == "rows"
    two = args.method == "two-stage"
    if rows_mode:
        # every rank holds the same sequences' keys and weights and only its
        # own query rows (equal visible pairs per rank)
        bounds = si.row_shards(wl.S, wl.T, wl.m, world)
        r0, r1 = bounds[rank], bounds[rank + 1]
        if r1 <= r0:
            raise RuntimeError(f"rank {rank} has an empty row shard: {bounds}")
        inp = synth.make_inputs(wl, fmt=args.fmt, seed=wl.seed, skip_q=True)
        inp["w"] = np.ascontiguousarray(inp["w"][:, r0:r1])
        qr = [synth.q_rows(wl, b, r0, r1 - r0, args.fmt, wl.seed) for b in range(wl.B)]
        if fp8:
            inp["q"] = np.stack([a for a, _ in qr])
            inp["q_scale"] = np.stack([sc for _, sc in qr])
        else:
            inp["q"] = np.stack(qr)
        rows_here = r1 - r0
    else:
        bounds, r0, rows_here = None, None, wl.S
        inp = synth.make_inputs(wl, fmt=args.fmt, seed=rank_seed(wl, rank))

    def host_tensor(name):
        a = inp[name]
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16 else torch.from_numpy(a)

    q, kc, w = (host_tensor(n).to(dev) for n in ("q", "kc", "w"))
    qs = torch.from_numpy(inp["q_scale"]).to(dev) if fp8 else None
    ks = torch.from_numpy(inp["kc_scale"]).to(dev) if fp8 else None
    kms = torch.from_numpy(inp["kc_mx_scale"]).to(dev) if mx else None
    out_idx = torch.empty((wl.B, rows_here, wl.k), dtype=torch.int32, device=dev)
    out_score = torch.empty((wl.B, rows_here, wl.k), dtype=torch.float32, device=dev)
    # library scratch, allocated here so that torch's peak counts it
    if two:
        ws_bytes = si.two_stage_workspace_size(wl.B, wl.S, wl.T, query_chunk=TWO_STAGE_CHUNK, **TWO_STAGE)
    elif mx:
        ws_bytes = si.workspace_size(wl.B, rows_here, wl.T, wl.H, wl.D, wl.m, wl.k, mxfp4=True)
    else:
        ws_bytes = 0
    workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev) if ws_bytes else None
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)  # > 126 MB L2
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)
    torch.cuda.reset_peak_memory_stats(dev)

    # one step = what si_indexer_topk does, as its two launches: the
    # streaming kernel (rows left unsorted), then the row sort; an event
    # between them times the streaming kernel alone for the roofline
    def step(mid=None):
        if two:
            # one si_indexer_topk_two_stage call (pool, coarse, fine, select, row sort)
            si.indexer_topk_two_stage(q, kc, w, wl.m, wl.k, query_chunk=TWO_STAGE_CHUNK, out_idx=out_idx,
                                      out_score=out_score, stream=stream, workspace=workspace, **TWO_STAGE)
            if mid is not None:
                mid.record(stream)
            return
        if rows_mode:
            si.indexer_topk_rows(q, kc, w, wl.m, wl.k, r0, q_scale=qs, kc_scale=ks, out_idx=out_idx,
                                 out_score=out_score, unsorted=True, stream=stream, kc_mx_scale=kms,
                                 workspace=workspace)
        else:
            si.indexer_topk(q, kc, w, wl.m, wl.k, q_scale=qs, kc_scale=ks, out_idx=out_idx,
                            out_score=out_score, unsorted=True, stream=stream, kc_mx_scale=kms, workspace=workspace)
        if mid is not None:
            mid.record(stream)
        si.sort_topk_rows(out_idx, out_score, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    if si.device_status(stream) != si.SI_OK:
        raise RuntimeError("device error during warm-up")

    evs = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
    sampler = ClockSampler(local if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local]))
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    wall0 = time.perf_counter()
    for e0, em, e1 in evs:
        flush.zero_()
        e0.record(stream)
        step(em)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - wall0
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    st = si.device_status(stream)
    if st != si.SI_OK:
        raise RuntimeError(f"device error during the timed steps: {st}")
    ms = [e0.elapsed_time(e1) for e0, _, e1 in evs]
    ms_step = sum(ms) / len(ms)
    ms_kernel = sum(e0.elapsed_time(em) for e0, em, _ in evs) / len(evs)
    ms_sort = sum(em.elapsed_time(e1) for _, em, e1 in evs) / len(evs)
    peak_mem = torch.cuda.max_memory_allocated(dev)
    if world > 1:
        ms_step = max_over_ranks(ms_step, dev)
        ms_kernel = max_over_ranks(ms_kernel, dev)
        ms_sort = max_over_ranks(ms_sort, dev)

    # end to end through the C ABI's host-buffer entry point (si_indexer_topk_host):
    # page-locked host inputs in, host results out, the copies of the query
    # chunks overlapped with the scoring inside the call
    hq, hk, hw = (host_tensor(n).pin_memory() for n in ("q", "kc", "w"))
    hqs = torch.from_numpy(inp["q_scale"]).pin_memory() if fp8 else None
    hks = torch.from_numpy(inp["kc_scale"]).pin_memory() if fp8 else None
    hkms = torch.from_numpy(inp["kc_mx_scale"]).pin_memory() if mx else None
    h_idx = torch.empty((wl.B, rows_here, wl.k), dtype=torch.int32).pin_memory()
    h_score = torch.empty((wl.B, rows_here, wl.k), dtype=torch.float32).pin_memory()
    bufs = {}

    def e2e_step():
        if two:
            si.indexer_topk_two_stage_host(hq, hk, hw, wl.m, wl.k, device=dev, bufs=bufs,
                                           query_chunk=TWO_STAGE_CHUNK, **TWO_STAGE)
        else:
            si.indexer_topk_host(hq, hk, hw, wl.m, wl.k, q_scale=hqs, kc_scale=hks, kc_mx_scale=hkms,
                                 row0=r0 or 0, out_idx=h_idx, out_score=h_score, stream=stream, device=dev)

    for _ in range(max(1, args.warmup)):
        e2e_step()
    e2e_dev = torch.cuda.memory_allocated(dev)
    e2e_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    for e0, e1 in e2e_ev:
        e0.record(stream)
        e2e_step()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev) / args.steps
    if world > 1:
        e2e_ms = max_over_ranks(e2e_ms, dev)
    def nbytes(*ts):
        return sum(t.numel() * t.element_size() for t in ts if t is not None)

    h2d = nbytes(hq, hk, hw, hqs, hks, hkms)
    d2h = out_idx.numel() * 4 + out_score.numel() * 4
    # device memory of the host-buffer call: the keys and two chunks of rows
    e2e_device_bytes = (si.two_stage_workspace_size(wl.B, rows_here, wl.T, **TWO_STAGE,
                                                    query_chunk=TWO_STAGE_CHUNK) + nbytes(q, kc, w, out_idx, out_score)
                        if two else si.indexer_topk_host_workspace_size(
                            wl.B, rows_here, wl.T, wl.H, wl.D, wl.k,
                            dtype=si.SI_DTYPE_FP8_E4M3 if fp8 else (si.SI_DTYPE_MXFP4_KEYS if mx else si.SI_DTYPE_BF16)))
    del bufs, e2e_dev

    million = None
    if world == 1 and wl.name == "v4flash" and args.fmt == "bf16" and not two and not args.no_million:
        million = million_record(args, dev, sampler.idx)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    flop_pair = 2 * wl.H * wl.D
    peaks = load_peaks()
    if rows_mode:
        # one job (the whole sequences) over the slowest rank's time; the
        # per-GPU figures take the average rank's share of the pairs
        value = wl.visible_pairs() / (ms_step * 1e-3)
        e2e_value = wl.visible_pairs() / (e2e_ms * 1e-3)
        P = wl.visible_pairs() / world
    else:
        P = wl.visible_pairs()
        value = job_value(world, P, ms_step)
        e2e_value = job_value(world, P, e2e_ms)
    tflops = P * flop_pair / (ms_step * 1e-3) / 1e12
    kernel_tflops = P * flop_pair / (ms_kernel * 1e-3) / 1e12
    if two:
        # the pairs the two stages actually score (pooled keys, then candidates)
        cp, fpairs = two_stage_pairs(wl)
        kernel_tflops = (cp + fpairs) * flop_pair / (ms_kernel * 1e-3) / 1e12
    alg_bytes = nbytes(q, kc, w, out_idx, out_score, qs, ks, kms)
    # the committed DRAM capture is of the whole-sequence bf16 launch
    traffic = None if fp8 or mx or two or (rows_mode and world > 1) else ncu_traffic(wl.name)
    # a contraction is measured against the peak of its own type: fp8 takes a
    # dense e4m3 matmul measured in this run (else the measured bf16 peak times
    # the nominal fp8 / bf16 ratio, 4.5 / 2.25)
    fp8_peak = measure_fp8_peak(dev) if fp8 else None
    if fp8 and fp8_peak:
        peak_tc, peak_src = fp8_peak, "measured in this run: torch._scaled_mm e4m3 8192^3, burst"
    else:
        peak_tc = peaks["bf16_tflops"] * (2.0 if fp8 else 1.0)
        peak_src = (f"{peaks['source']} bf16 dense matmul, burst" +
                    (", x2 (nominal fp8 / bf16 dense ratio)" if fp8 else ""))
    cpu = None
    if world == 1 and args.cpu_seconds > 0:
        rows = synth.sample_rows(4096, wl.m * 4, wl.S, seed=wl.seed + 99)
        rng = np.random.default_rng(wl.seed)
        rng.shuffle(rows)
        done, t_tot, p_tot = 0, 0.0, 0
        while t_tot < args.cpu_seconds and done < len(rows):
            chunk = np.sort(rows[done:done + 16])
            dt, pr = oracle_sample(wl, inp, chunk, two)
            t_tot += dt
            p_tot += pr
            done += len(chunk)
        cpu = {"value": p_tot / t_tot, "unit": "pairs/s", "cores": 1, "kind": "oracle",
               "sample": f"{done} uniformly sampled query rows of the {wl.name} workload ({p_tot} visible "
                         f"pairs, {t_tot:.1f} s), single-threaded C oracle, fp64, full sort"}
        cpu["all_cores"] = oracle_all_cores(wl, inp, two, seconds=min(args.cpu_seconds, 10.0))
    line = {
        "metric": METRIC, "value": value, "unit": "pairs/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if rows_mode else "weak",
        "vs_baseline": None, "dtype": "bf16" if mx else args.fmt, "data": "synthetic",
        "config": dict(config_dict(wl, world, args.shard, bounds),
                       **({"keys": "MXFP4 (E2M1 codes, E8M0 scale per 32 values), decoded to bf16 "
                                   "inside the call"} if mx else {}),
                       **({"method": f"two-stage: the best {TWO_STAGE['n_keep']} blocks of {TWO_STAGE['block']} "
                                     f"keys by their pooled key, then the top-{wl.k} of their keys; value counts "
                                     "the workload's visible pairs, the roofline the pairs the two stages score "
                                     f"({two_stage_pairs(wl)[0]} pooled + {two_stage_pairs(wl)[1]} candidate)",
                           "query_chunk": TWO_STAGE_CHUNK} if two else {})),
        "tflops": tflops,
        "frac_bf16_peak": tflops / peaks["bf16_tflops"],
        "frac_bf16_peak_sustained": tflops / peaks["bf16_tflops_sustained"] if peaks["bf16_tflops_sustained"] else None,
        "hbm_gbs": alg_bytes / (ms_step * 1e-3) / 1e9,
        "frac_hbm": alg_bytes / (ms_step * 1e-3) / 1e9 / peaks["hbm_gbs"],
        # the path's own device memory: inputs, outputs and library scratch
        # (torch's peak less the bench's L2-flush buffer, which is no part of it)
        "peak_hbm_gb": (peak_mem - flush.numel()) / 1e9,
        "hbm_breakdown_gb": {"q": nbytes(q, qs) / 1e9, "kc": nbytes(kc, ks, kms) / 1e9, "w": nbytes(w) / 1e9,
                             "out_idx": nbytes(out_idx) / 1e9, "out_score": nbytes(out_score) / 1e9,
                             "library_workspace": ws_bytes / 1e9,
                             "bench_l2_flush_buffer (not counted)": flush.numel() / 1e9},
        "kernel_ms": ({"indexer_topk_two_stage call": ms_kernel} if two else
                      {"stream_topk_kernel": ms_kernel, "row_sort_kernel": ms_sort}),
        "roofline": {"bound": "tensor",
                     "kernel": ("two-stage call (pool, coarse stream_topk_kernel, fine_score_kernel, select, "
                                "row sort)" if two else "stream_topk_kernel"),
                     "achieved": kernel_tflops,
                     "peak": peak_tc, "unit": "TFLOP/s",
                     "frac": kernel_tflops / peak_tc,
                     "peak_source": peak_src,
                     "traffic": traffic, "algorithmic_bytes": alg_bytes},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "pairs/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "api": ("indexer_topk_two_stage on device copies (Python)" if two else
                        "si_indexer_topk_host (C ABI, host buffers; query chunks of 4096 rows through two "
                        "device slots, copies overlapped with the scoring)"),
                "device_gb": e2e_device_bytes / 1e9},
        "gpu_launches": ((2 + 3 * wl.B * -(-wl.S // TWO_STAGE_CHUNK)) if two else 2) * args.steps,
        "clocks": clocks,
        "wall_s_timed": wall,
    }
    if million is not None:
        line["million"] = million
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------ sparse attention
ATTN_H, ATTN_DK, ATTN_DV = 64, 576, 512


def run_attention(args, wl):
    """One step = one si_sparse_attention call over the workload's queries:
    every query's 64 heads attend over the 512 latents its indexer top-k
    selected (the indexer runs once, untimed, on the workload's own planted
    inputs).  Latents [T, 576] and attention queries [S, 64, 576] are N(0, 1)
    bf16; out [S, 64, 512] bf16 and lse [S, 64] fp32."""
    import torch

    import streaming_top_b200 as si
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = synth.make_inputs(wl)
    qi = torch.from_numpy(inp["q"].view(np.int16)).view(torch.bfloat16).to(dev)
    kc = torch.from_numpy(inp["kc"].view(np.int16)).view(torch.bfloat16).to(dev)
    idx, _ = si.indexer_topk(qi, kc, torch.from_numpy(inp["w"]).to(dev), wl.m, wl.k)
    del qi, kc
    q, kv = synth.attention_inputs(wl.B, wl.S, wl.T, seed=wl.seed + 500)
    qd = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).to(dev)
    kvd = torch.from_numpy(kv.view(np.int16)).view(torch.bfloat16).to(dev)
    del q, kv
    out = torch.empty((wl.B, wl.S, ATTN_H, ATTN_DV), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((wl.B, wl.S, ATTN_H), dtype=torch.float32, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush.zero_()
        si.sparse_attention(qd, kvd, idx, out=out, lse=lse, stream=stream)
    if si.device_status(stream) != si.SI_OK:
        raise RuntimeError("device error during warm-up")
    sampler = ClockSampler(0 if "CUDA_VISIBLE_DEVICES" not in os.environ else
                           int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[0]))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        si.sparse_attention(qd, kvd, idx, out=out, lse=lse, stream=stream)
        e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if si.device_status(stream) != si.SI_OK:
        raise RuntimeError("device error during the timed steps")
    ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
    nq = wl.B * wl.S
    sel = int((idx >= 0).sum())
    flop = 2 * ATTN_H * sel * (ATTN_DK + ATTN_DV)   # selected entries only
    alg_bytes = sum(t.numel() * t.element_size() for t in (qd, out, lse, idx)) + kvd.numel() * 2
    gathered = sel * (ATTN_DK + ATTN_DV) * 2
    peaks = load_peaks()
    line = {
        "metric": "sparse attention over the indexer's selected latents: queries/s (TFLOP/s, % bf16 TC peak)",
        "value": nq / (ms * 1e-3), "unit": "queries/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"sparse attention at the {wl.name} shape: B={wl.B}, S={wl.S} queries x 64 heads, "
                               f"T={wl.T} latents of 576 (values: the first 512), the indexer's top-{wl.k} "
                               f"of the planted inputs (seed {wl.seed}) as the selection",
                   "selected_entries": sel,
                   "l2": f"q ({qd.numel() * 2 / 1e9:.1f} GB) > L2, and L2 flushed before each timed step"},
        "tflops": flop / (ms * 1e-3) / 1e12,
        "roofline": {"bound": "tensor", "kernel": "sparse_attn_kernel", "achieved": flop / (ms * 1e-3) / 1e12,
                     "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": flop / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                     "peak_source": f"{peaks['source']} bf16 dense matmul, burst", "traffic": None,
                     "algorithmic_bytes": alg_bytes, "gathered_latent_bytes_from_l2": gathered},
        "hbm_gbs": alg_bytes / (ms * 1e-3) / 1e9,
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    print(json.dumps(line))
    return 0


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="v4flash", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--fmt", default="bf16", choices=["bf16", "e4m3", "mxfp4"],
                    help="input format: bf16 (default), fp8 e4m3 with per-row scales, or mxfp4 keys "
                         "(E2M1 + E8M0 per 32 values) with bf16 queries")
    ap.add_argument("--ref-rows", type=int, default=32)
    ap.add_argument("--no-million", action="store_true",
                    help="leave out the million-token record the default run adds beside the headline")
    ap.add_argument("--method", default="one-stage", choices=["one-stage", "two-stage", "sparse-attention"],
                    help="one-stage (the streaming top-k over all visible keys) or the two-stage indexer "
                         "(2048 blocks of 8 kept by their pooled key, then the top-k of their keys)")
    ap.add_argument("--shard", default="seq", choices=["seq", "rows"],
                    help="N>1: independent sequences per GPU (seq, weak scaling) or the same sequences' "
                         "query rows split over the GPUs at equal visible pairs (rows, strong scaling)")
    args = ap.parse_args()
    if args.method == "two-stage" and (args.fmt != "bf16" or args.shard == "rows"):
        raise SystemExit("--method two-stage runs bf16 inputs over whole sequences")
    wl = synth.WORKLOADS[args.workload]
    if args.method == "sparse-attention":
        if args.impl == "reference" or args.gpus != 1:
            raise SystemExit("--method sparse-attention times the CUDA kernel on one GPU")
        return run_attention(args, wl)
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
