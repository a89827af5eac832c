#!/usr/bin/env python
"""Benchmark of the selective mixed-precision (NVFP4 + FP16) attention forward on B200.

Metric: attention-forward effective TFLOPS (4 B Hq N^2 d, halved when causal) of one whole step
-- NVFP4 quantisation of Q, K, V, block selection, attention -- on the 32K causal LLM-prefill
workload (B=1, 32 query / 8 KV heads, d=128, 128x64 blocks, k = 5 % of the valid pairs), plus
the attention kernel's fraction of the blended NVFP4/FP16 tensor-core roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With --workload decode131k (or another decode workload) it times one decode step instead: the new
query rows against a 131K-key cache held in FP16 and NVFP4 (selection + attention), reported as
the step's algorithmic cache bytes per second against the measured HBM bandwidth.

One process per GPU (torchrun for N > 1); each rank runs its own copy of the workload (weak
scaling, no collective on the data path); timing is CUDA events on the launching stream, max over
ranks.  Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "attn fwd effective TFLOPS & % of NVFP4/FP16 tensor roofline, N=32K causal k=5%"
DECODE_METRIC = "decode step: algorithmic KV-cache GB/s (NVFP4 + selected FP16 blocks) & % of HBM roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_traffic.json")
ATTN_SRC = os.path.join(ROOT, "precision_attention_block_b200", "csrc", "attn.cu")
NVFP4_PER_FP16 = 4.0  # nominal dense NVFP4 : FP16 tensor throughput on B200 (9 : 2.25 PFLOP/s)
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill32k", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--budget-bp", type=int, default=None, help="override the FP16 budget (basis points)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-units", type=int, default=8)
    ap.add_argument("--quality-units", type=int, default=8, help="query blocks sampled for the quality context "
                    "(0: skip it)")
    ap.add_argument("--sparse", action="store_true",
                    help="the compute-matched sparse variant: only the selected pairs, in FP16")
    return ap.parse_args()


def max_over_ranks(values, device, dist):
    """Element-wise maximum of per-rank timings over all ranks (the slowest rank sets the job
    time); the values themselves when there is a single process."""
    import torch
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def elementwise_bound(n_elem, d, block_k, mufu_lanes, fma_lanes, sm_count, sm_mhz, poly_fma_ops=8):
    """Lower bound on the attention kernel's time from the elementwise work of reading R1 alone,
    at the measured pipe rates (lanes per SM clock).  Per score element: one exponential, and on
    the FMA pipe the exponent argument (1), the unquantised sum (1) and the merge of the key
    block's PV product into the output (d / block_k: d output columns per row per block of
    block_k keys).  An exponential runs on the MUFU unit or as a polynomial on the FMA pipe
    (poly_fma_ops operations); the bound takes the split that balances the two pipes.  Ignores
    instruction issue, the E2M1/E4M3 conversions and the group maxima (other pipes), so the real
    floor is higher."""
    e = float(n_elem)
    f = e * (2.0 + d / block_k)
    rm = mufu_lanes * sm_count
    rf = fma_lanes * sm_count
    x = (e * rf - f * rm) / (rf + poly_fma_ops * rm)
    x = min(max(x, 0.0), e)
    cycles = max((e - x) / rm, (f + poly_fma_ops * x) / rf)
    return {"ms": cycles / (sm_mhz * 1e6) * 1e3, "exps_per_elem": 1.0, "fma_ops_per_elem": 2.0 + d / block_k,
            "poly_share": x / e if e else 0.0, "elements": e, "mufu_lanes_per_clk_sm": mufu_lanes,
            "fma_lanes_per_clk_sm": fma_lanes, "sm_mhz": sm_mhz, "poly_fma_ops": poly_fma_ops}


def reference_rows(q, k, v, w, units, tau):
    """float64 softmax attention (every pair exact, FP16 inputs widened) for the rows of the
    listed (b, h, i) units: the quality context's full-precision reference.  [rows, d]."""
    g = w.Hq // w.Hkv
    out = []
    for (b, h, i) in units:
        rows = np.arange(i * w.block_q, (i + 1) * w.block_q)
        kend = (i + 1) * w.block_q if w.causal else w.N
        qq = q[b, h, rows].astype(np.float64)
        kk = k[b, h // g, :kend].astype(np.float64)
        vv = v[b, h // g, :kend].astype(np.float64)
        s = tau * (qq @ kk.T)
        if w.causal:
            s = np.where(np.arange(kend)[None, :] > rows[:, None], -np.inf, s)
        s = s - s.max(1, keepdims=True)
        p = np.exp(s)
        out.append((p @ vv) / p.sum(1, keepdims=True))
    return np.concatenate(out)


def gap_recovery(err_fp4, err_k):
    """Share of the uniform-NVFP4 error removed by the FP16 budget: (err_FP4 - err_k) / err_FP4."""
    return (err_fp4 - err_k) / err_fp4 if err_fp4 > 0 else 0.0


def quality_block(pab, torch, w, q, k, v, gq, gk, gv, n_units):
    """rel-L2 of the library's output against float64 softmax attention on a stratified sample of
    query blocks, for uniform NVFP4 (k = 0), the workload's budget and every pair in FP16, and the
    synthetic gap recovery.  Context only (the pages' quality figures come from model benchmarks)."""
    units = workloads.sample_units(w, n_units)
    tau = float(np.float32(1.0) / np.sqrt(np.float32(w.d)))
    ref = reference_rows(q, k, v, w, units, tau)
    rel = {}
    for bp in (0, w.topk_bp, 10000):
        wb = w.with_budget(bp)
        cfg = pab.Config.from_workload(wb)
        out, _ = pab.attn_fwd_auto(gq, gk, gv, cfg)
        o = out.cpu().numpy().astype(np.float64)
        rows = np.concatenate([o[b, h, i * w.block_q:(i + 1) * w.block_q] for (b, h, i) in units])
        rel[bp] = float(np.linalg.norm(rows - ref) / np.linalg.norm(ref))
    return {"reference": "float64 softmax attention of the FP16 inputs",
            "sample": f"{len(units)} stratified (b, head, query block) units",
            "rel_l2": {"k=0 (uniform NVFP4)": rel[0], f"k={w.topk_bp / 100:g}%": rel[w.topk_bp],
                       "k=all (FP16)": rel[10000]},
            "gap_recovery": gap_recovery(rel[0], rel[w.topk_bp])}


def effective_flops(w) -> float:
    f = 4.0 * w.B * w.Hq * w.N * w.N * w.d
    return f / 2 if w.causal else f


def unit_effective_flops(w, i) -> float:
    """Effective FLOPs of one (b, h, query block i) unit under the same convention."""
    if not w.causal:
        return 4.0 * w.block_q * w.N * w.d
    keys = sum(min(w.N, r + 1) for r in range(i * w.block_q, (i + 1) * w.block_q))
    return 4.0 * keys * w.d


def valid_pairs_per_head(w) -> int:
    if not w.causal:
        return w.n_qb * w.n_kb
    return sum(((i + 1) * w.block_q - 1) // w.block_k + 1 for i in range(w.n_qb))


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), \
            float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, 1400.0, 6650.0, "fallback"


def attn_src_hash() -> str:
    """Hash of the attention kernel's sources (the kernel file and the inline-PTX header it
    includes): stored DRAM counters count only for the kernel they were taken on."""
    h = hashlib.sha256()
    for path in (ATTN_SRC, os.path.join(os.path.dirname(ATTN_SRC), "sm100.cuh")):
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic(workload: str):
    """DRAM bytes per attention launch from a committed ncu capture, if the kernel source is
    unchanged since it was taken; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        e = t.get(workload)
        if e and e.get("attn_src_sha256_16") == attn_src_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed region runs."""

    NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
             0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
             0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self.h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nvml = pynvml
            props = torch.cuda.get_device_properties(device_index)
            uuid = str(getattr(props, "uuid", ""))
            if uuid:
                u = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
                try:
                    self.h = pynvml.nvmlDeviceGetHandleByUUID(u)
                except Exception:
                    self.h = None
            if self.h is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                idx = int(vis.split(",")[device_index]) if vis and vis.split(",")[0].isdigit() else device_index
                self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.h = None

    def _run(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                try:
                    r = n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except Exception:
                    r = n.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.reasons |= int(r) & ~0x1
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.h is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": [v for k, v in self.NAMES.items() if self.reasons & k], "samples": len(self.samples)}


def cpu_baseline(w, q, k, v, n_units: int):
    """The oracle, as it stands, on the host cores: full NVFP4 quantisation and selection of the
    workload, then attention on a stratified sample of (b, h, query block) units; the value is the
    sample's effective FLOPs over its time plus the sample's share of quantise + select."""
    import oracle
    threads = os.cpu_count() or 1
    t0 = time.perf_counter()
    q4, k4, v4 = oracle.quantize_all(q, k, v)
    scores = oracle.block_scores(q, k, w)
    sel, _, _ = oracle.select(scores, w)
    t_prep = time.perf_counter() - t0
    units = workloads.sample_units(w, n_units, seed_offset=3)
    t0 = time.perf_counter()
    oracle.attn(q, k, v, q4, k4, v4, sel, w, units=units, threads=threads)
    t_attn = time.perf_counter() - t0
    f_sample = sum(unit_effective_flops(w, i) for (_, _, i) in units)
    share = f_sample / effective_flops(w)
    t = t_attn + t_prep * share
    return {"value": f_sample / t / 1e12, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
            "sample": f"{len(units)} stratified (b, head, 128-row query block) units of {w.name}; attention "
                      f"{t_attn:.1f} s on {threads} threads + their {share:.2e} share of the full "
                      f"quantise/select ({t_prep:.1f} s)"}


def run_reference(args, rank):
    """--impl reference: the oracle on the host cores, one bounded sample per step."""
    if rank != 0:
        return
    import oracle
    w = workloads.WORKLOADS[args.workload]
    if args.budget_bp is not None:
        w = w.with_budget(args.budget_bp)
    q, k, v = workloads.make_qkv(w)
    threads = os.cpu_count() or 1
    if w.is_decode:
        run_reference_decode(args, w, q, k, v, threads)
        return
    t0 = time.perf_counter()
    q4, k4, v4 = oracle.quantize_all(q, k, v)
    scores = oracle.block_scores(q, k, w)
    sel, _, _ = oracle.select(scores, w)
    t_prep = time.perf_counter() - t0
    per_step = max(1, min(threads, 8))
    pool = workloads.sample_units(w, per_step * 8, seed_offset=5)
    flops, secs = 0.0, 0.0
    for s in range(args.warmup + args.steps):
        units = [pool[(s * per_step + u) % len(pool)] for u in range(per_step)]
        t0 = time.perf_counter()
        oracle.attn(q, k, v, q4, k4, v4, sel, w, units=units, threads=threads)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            f = sum(unit_effective_flops(w, i) for (_, _, i) in units)
            flops += f
            secs += dt + t_prep * f / effective_flops(w)
    value = flops / secs / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                       "causal": w.causal, "block_q": w.block_q, "block_k": w.block_k, "topk_bp": w.topk_bp},
            "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                             "sample": f"{per_step} (b, head, query block) units per step, cycled from a "
                                       f"stratified sample, plus their share of the full quantise/select"},
            "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_reference_decode(args, w, q, k, v, threads):
    """--impl reference on a decode workload: whole oracle decode steps (the cache's NVFP4 copies
    built once beforehand), the same bytes-per-second metric as the GPU line."""
    import oracle
    k4, v4 = oracle.quantize_nvfp4(k, 0), oracle.quantize_nvfp4(v, 1)
    r = oracle.decode_forward(w, q, k, v, k4=k4, v4=v4, threads=threads)
    alg_bytes, _, _ = decode_bytes(w, r["sel"][:, :, 0, :].astype(bool))
    steps = max(1, min(args.steps, 10))
    secs = 0.0
    for s in range(min(args.warmup, 1) + steps):
        t0 = time.perf_counter()
        oracle.decode_forward(w, q, k, v, k4=k4, v4=v4, threads=threads)
        if s >= min(args.warmup, 1):
            secs += time.perf_counter() - t0
    value = alg_bytes * steps / secs / 1e9
    line = {"impl": "reference", "metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": min(args.warmup, 1), "ms_per_step": 1e3 * secs / steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.n_query, "Nk": w.N,
                       "d": w.d, "causal": w.causal, "block_k": w.block_k, "topk_bp": w.topk_bp},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": f"{steps} whole decode steps (quantise the query rows, score, select, "
                                       f"attend); cache NVFP4 copies built once beforehand"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    import torch
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        if args.impl == "ours":
            torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl" if args.impl == "ours" else "gloo",
                                timeout=datetime.timedelta(seconds=300))
    if args.impl == "reference":
        run_reference(args, rank)
        if dist:
            dist.destroy_process_group()
        return

    import precision_attention_block_b200 as pab
    from precision_attention_block_b200 import build
    if rank == 0 or world == 1:
        build.build()
    if dist:
        dist.barrier()
    pab.load()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)

    w = workloads.WORKLOADS[args.workload]
    if args.budget_bp is not None:
        w = w.with_budget(args.budget_bp)
    if w.is_decode:
        main_decode(args, w, pab, torch, device, world, rank, local_rank, dist)
        return
    cfg = pab.Config.from_workload(w)
    q, k, v = workloads.make_qkv(w)
    gq, gk, gv = (torch.from_numpy(x).to(device) for x in (q, k, v))
    q4 = pab.NVFP4Tensor.empty(w.B * w.Hq, w.N, w.d, 0, device)
    k4 = pab.NVFP4Tensor.empty(w.B * w.Hkv, w.N, w.d, 0, device)
    v4 = pab.NVFP4Tensor.empty(w.B * w.Hkv, w.N, w.d, 1, device)
    ws = pab.Workspace.for_config(cfg, device)
    sel = pab.block_select(gq, gk, cfg, ws=ws)
    out = torch.empty_like(gq)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def step(evs=None):
        if not args.sparse:
            pab.quantize_nvfp4(gq, 0, out=q4, ws=ws)
            pab.quantize_nvfp4(gk, 0, out=k4, ws=ws)
            pab.quantize_nvfp4(gv, 1, out=v4, ws=ws)
        if evs:
            evs[0].record(stream)
        pab.block_select(gq, gk, cfg, ws=ws, out=sel)
        if evs:
            evs[1].record(stream)
        if args.sparse:
            pab.attn_fwd_sparse(gq, gk, gv, sel, cfg, out=out, lse=lse, ws=ws)
        else:
            pab.attn_fwd(gq, gk, gv, q4, k4, v4, sel, cfg, out=out, lse=lse, ws=ws)
        if evs:
            evs[2].record(stream)

    rates = pab.pipe_rates(device) if not args.sparse else None
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    launches_per_step = (0 if args.sparse else 3 * 2) + 5 + 1  # amax + encode per tensor; selection; attention
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    ev_start = torch.cuda.Event(enable_timing=True)
    ev_end = torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local_rank)
    with sampler:
        ev_start.record(stream)
        prev = ev_start
        step_starts = []
        for s in range(args.steps):
            step_starts.append(prev)
            step(evs[s])
            prev = evs[s][2]
        ev_end.record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    total_ms = ev_start.elapsed_time(ev_end)
    attn_ms = [evs[s][1].elapsed_time(evs[s][2]) for s in range(args.steps)]
    sel_ms = [evs[s][0].elapsed_time(evs[s][1]) for s in range(args.steps)]
    quant_ms = [step_starts[s].elapsed_time(evs[s][0]) for s in range(args.steps)]
    total_ms, attn_mean_ms = max_over_ranks([total_ms, statistics.mean(attn_ms)], device, dist)

    # status word: any device-side timeout invalidates the run
    status = pab.device_status(ws)

    # roofline of the attention kernel: algorithmic FLOPs of the valid block pairs by precision
    counts = sel.counts.sum().item()
    mode_fp16_all = cfg.topk_abs < 0 and cfg.topk_bp == 10000
    mode_fp4_all = cfg.topk_abs == 0 or (cfg.topk_abs < 0 and cfg.topk_bp == 0)
    valid_total = valid_pairs_per_head(w) * w.B * w.Hq
    k_total = valid_total if mode_fp16_all else (0 if mode_fp4_all else counts)
    per_pair = 4.0 * w.block_q * w.block_k * w.d
    F16, F4 = k_total * per_pair, (valid_total - k_total) * per_pair
    if args.sparse:  # only the selected pairs run
        F16, F4 = counts * per_pair, 0.0
    bf16_burst, bf16_sustained, hbm_gbs, peak_src = peaks()
    p16, p4 = bf16_burst * 1e12, bf16_burst * NVFP4_PER_FP16 * 1e12
    t_roof = F16 / p16 + F4 / p4
    achieved = (F16 + F4) / (attn_mean_ms * 1e-3) / 1e12
    peak_blend = (F16 + F4) / t_roof / 1e12
    traffic = stored_traffic(w.name) if args.budget_bp is None and not args.sparse else None

    eff = effective_flops(w)
    qkv_mb = (q.nbytes + k.nbytes + v.nbytes) / 1e6
    value = world * eff * args.steps / (total_ms * 1e-3) / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4+fp16 (fp32 accumulate)",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d,
                       "causal": w.causal, "block_q": w.block_q, "block_k": w.block_k, "topk_bp": w.topk_bp,
                       "parallelism": f"replica x{world} (each rank its own batch)",
                       "l2": (f"inputs larger than L2 (Q, K, V {qkv_mb:.0f} MB FP16)" if qkv_mb > 126
                              else f"inputs smaller than L2 ({qkv_mb:.0f} MB); no flush")},
            "breakdown_ms": {"quantize": statistics.mean(quant_ms), "select": statistics.mean(sel_ms),
                             "attention": attn_mean_ms},
            "variant": "sparse (selected pairs only, FP16; effective FLOPs of the dense problem)" if args.sparse
                       else "mixed NVFP4/FP16",
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_blend, "unit": "TFLOP/s",
                         "frac": achieved / peak_blend, "traffic": traffic,
                         "peak_note": f"blend of {peak_src} bf16 burst {bf16_burst:.1f} TF/s (FP16) and "
                                      f"x{NVFP4_PER_FP16:.0f} for NVFP4; F16={F16:.3e} F4={F4:.3e}"},
            "gpu_launches": launches_per_step * args.steps,
            "device_status": status}

    line["clocks"] = sampler.summary()
    if rates is not None:
        sm_mhz = line["clocks"].get("sm_mhz") or 1965.0
        eb = elementwise_bound((F16 + F4) / (4.0 * w.d), w.d, w.block_k, rates["mufu_ex2"], rates["fma"],
                               torch.cuda.get_device_properties(device).multi_processor_count, sm_mhz)
        eb["attention_ms"] = attn_mean_ms
        eb["frac"] = eb["ms"] / attn_mean_ms
        eb["tensor_roofline_ms"] = t_roof * 1e3
        eb["max_tensor_frac"] = min(1.0, t_roof * 1e3 / eb["ms"])
        line["roofline"]["elementwise"] = eb
    if rank == 0 and not args.sparse and args.quality_units > 0:
        line["quality"] = quality_block(pab, torch, w, q, k, v, gq, gk, gv, args.quality_units)
    if not args.no_e2e and not args.sparse:
        line["e2e"] = e2e_measure(pab, torch, w, cfg, q, k, v, device, args, world, dist)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.sparse:
        line["cpu_baseline"] = cpu_baseline(w, q, k, v, args.cpu_units)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


def decode_bytes(w, mask_bits):
    """Algorithmic HBM bytes of one decode step for a selection: per (batch, KV head, key block)
    the NVFP4 K and V (codes and E4M3 scales) when some query head of the group computes the block
    in NVFP4, the FP16 K and V when some head selected it, plus the key-block means the selection
    reads.  mask_bits: bool [B, Hq, nKb]."""
    G = w.Hq // w.Hkv
    g = mask_bits.reshape(w.B, w.Hkv, G, -1)
    blocks16 = int(g.any(2).sum())
    blocks4 = int((~g).any(2).sum())
    per4 = 2 * w.block_k * w.d * (1 / 2 + 1 / 16)
    per16 = 2 * w.block_k * w.d * 2
    kbar = w.B * w.Hkv * (w.N // w.block_k) * w.d * 8
    return blocks4 * per4 + blocks16 * per16 + kbar, blocks4, blocks16


def main_decode(args, w, pab, torch, device, world, rank, local_rank, dist):
    """One decode step per iteration: quantise the query rows, select key blocks, attend.  The
    cache (FP16, NVFP4 copies, key block means) is built once and stays resident.  Steps are
    replayed from a CUDA graph of one step (the launches of a step take less GPU time than the
    host needs to issue them one by one)."""
    cfg = pab.DecodeConfig.from_workload(w)
    q, k, v = workloads.make_qkv(w)
    gq, gk, gv = (torch.from_numpy(x).to(device) for x in (q, k, v))
    cache = pab.KVCache.build(gk, gv, w.block_k)
    ws = cfg.workspace(device)
    out = torch.empty_like(gq)
    lse = torch.empty((w.B, w.Hq, w.n_query), dtype=torch.float32, device=device)
    sel = pab.decode_select(gq, cache, cfg, ws=ws)
    torch.cuda.synchronize()
    mask = sel.mask.cpu().numpy().view(np.uint32)
    bits = ((mask[..., :, None] >> np.arange(32, dtype=np.uint32)) & 1).reshape(w.B, w.Hq, -1)[..., :cfg.n_kb]
    alg_bytes, blocks4, blocks16 = decode_bytes(w, bits.astype(bool))
    cache_mb = (gk.numel() + gv.numel()) * 2 / 1e6

    side = torch.cuda.Stream(device)
    side.wait_stream(torch.cuda.current_stream())

    def graph_of(fn):
        with torch.cuda.stream(side):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            fn()
        return g

    step_graph = graph_of(lambda: pab.decode_fwd(gq, cache, cfg, out=out, lse=lse, ws=ws))
    attn_graph = graph_of(lambda: pab.decode_attn(gq, cache, sel, cfg, out=out, lse=lse, ws=ws))
    cfg16 = pab.DecodeConfig.from_workload(w.with_budget(10000))
    ws16 = cfg16.workspace(device)
    fp16_graph = graph_of(lambda: pab.decode_attn(gq, cache, None, cfg16, out=out, lse=lse, ws=ws16))
    sparse_graph = graph_of(lambda: pab.decode_attn_sparse(gq, cache, sel, cfg, out=out, lse=lse, ws=ws))

    def timed(g, steps, warmup):
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            g.replay()
        b.record()
        torch.cuda.synchronize()
        return max_over_ranks([a.elapsed_time(b)], device, dist)[0] / steps

    sampler = ClockSampler(local_rank)
    with sampler:
        step_ms = timed(step_graph, args.steps, args.warmup)
    attn_ms = timed(attn_graph, args.steps, args.warmup)
    fp16_ms = timed(fp16_graph, max(3, args.steps // 4), 2)
    sparse_ms = timed(sparse_graph, max(3, args.steps // 4), 2)
    status = pab.device_status(ws)
    _, _, hbm_gbs, peak_src = peaks()
    attn_bytes = alg_bytes - w.B * w.Hkv * (w.N // w.block_k) * w.d * 8
    achieved = attn_bytes / (attn_ms * 1e-3) / 1e9
    value = world * alg_bytes / (step_ms * 1e-3) / 1e9
    line = {"metric": DECODE_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4+fp16 (fp32 accumulate)", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.n_query, "Nk": w.N,
                       "d": w.d, "causal": w.causal, "block_k": w.block_k, "topk_bp": w.topk_bp,
                       "parallelism": f"replica x{world} (each rank its own batch)",
                       "l2": f"cache larger than L2 (K, V {cache_mb:.0f} MB FP16 + NVFP4 copies)"
                             if cache_mb > 126 else f"cache {cache_mb:.0f} MB: L2 not flushed"},
            "breakdown_us": {"step": 1e3 * step_ms, "attention": 1e3 * attn_ms,
                             "select_and_quantize": 1e3 * (step_ms - attn_ms),
                             "all_fp16_attention_same_kernel": 1e3 * fp16_ms,
                             "sparse_attention_selected_blocks_only": 1e3 * sparse_ms},
            "blocks": {"nvfp4": blocks4, "fp16": blocks16, "of": w.B * w.Hkv * (w.N // w.block_k)},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_gbs, "unit": "GB/s",
                         "frac": achieved / hbm_gbs, "traffic": None,
                         "peak_note": f"{peak_src} HBM copy bandwidth; achieved = the attention kernels' "
                                      f"algorithmic bytes ({attn_bytes / 1e6:.1f} MB) / their time"},
            "gpu_launches": 6 * args.steps,  # amax, encode (query rows), scores, top-k, attention, combine
            "device_status": status}
    if not args.no_e2e:
        hq = torch.from_numpy(q).pin_memory()
        ho = torch.empty(out.shape, dtype=torch.float16).pin_memory()
        hl = torch.empty(lse.shape, dtype=torch.float32).pin_memory()

        def e2e_step():
            gq.copy_(hq, non_blocking=True)
            pab.decode_fwd(gq, cache, cfg, out=out, lse=lse, ws=ws)
            ho.copy_(out, non_blocking=True)
            hl.copy_(lse, non_blocking=True)

        e2e_ms = timed(graph_of(e2e_step), args.steps, args.warmup)
        line["e2e"] = {"value": world * alg_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                       "h2d_bytes_per_step": int(hq.numel() * 2),
                       "d2h_bytes_per_step": int(ho.numel() * 2 + hl.numel() * 4), "ms_per_step": e2e_ms,
                       "note": "query rows copied in and the output copied out every step; the cache stays "
                               "resident, as in a decode loop"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        threads = os.cpu_count() or 1
        k4o, v4o = oracle.quantize_nvfp4(k, 0), oracle.quantize_nvfp4(v, 1)
        t0 = time.perf_counter()
        oracle.decode_forward(w, q, k, v, k4=k4o, v4=v4o, threads=threads)
        t = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": alg_bytes / t / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
                                "sample": f"one whole decode step of {w.name} ({t:.2f} s on {threads} threads); "
                                          "cache NVFP4 copies built beforehand, outside the timing"}
    line["clocks"] = sampler.summary()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.destroy_process_group()


def e2e_measure(pab, torch, w, cfg, q, k, v, device, args, world, dist):
    """The same metric through thrift_attn_fwd_auto with host buffers: every step copies Q, K, V
    from pinned host memory, runs quantise + select + attend, and copies O and lse back.  As a
    serving loop would, the steps are pipelined over two buffer sets and three streams: the
    host-to-device copy of step i + 1 and the device-to-host copy of step i - 1 run on the copy
    engines while step i computes.  The timed region spans all copies of all timed steps."""
    hq, hk, hv = (torch.from_numpy(x).pin_memory() for x in (q, k, v))
    sets = []
    for _ in range(2):
        gq, gk, gv = (torch.empty(x.shape, dtype=torch.float16, device=device) for x in (q, k, v))
        out = torch.empty_like(gq)
        lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=device)
        ho = torch.empty(out.shape, dtype=torch.float16).pin_memory()
        hl = torch.empty(lse.shape, dtype=torch.float32).pin_memory()
        sets.append((gq, gk, gv, out, lse, ho, hl))
    ws = pab.Workspace.for_config(cfg, device, auto=True)
    s_c = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = {name: [torch.cuda.Event(), torch.cuda.Event()] for name in ("in_ready", "in_free", "out_ready", "out_free")}

    def step(i):
        gq, gk, gv, out, lse, ho, hl = sets[i % 2]
        b = i % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev["in_free"][b])      # step i - 2 has finished reading this set
            gq.copy_(hq, non_blocking=True)
            gk.copy_(hk, non_blocking=True)
            gv.copy_(hv, non_blocking=True)
            ev["in_ready"][b].record(s_in)
        s_c.wait_event(ev["in_ready"][b])
        s_c.wait_event(ev["out_free"][b])          # step i - 2's output has left this set
        pab.attn_fwd_auto(gq, gk, gv, cfg, out=out, lse=lse, ws=ws)
        ev["in_free"][b].record(s_c)
        ev["out_ready"][b].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev["out_ready"][b])
            ho.copy_(out, non_blocking=True)
            hl.copy_(lse, non_blocking=True)
            ev["out_free"][b].record(s_out)

    def join():
        s_c.wait_stream(s_in)
        s_c.wait_stream(s_out)

    steps = max(3, min(args.steps, 20))
    for i in range(max(3, args.warmup)):
        step(i)
    join()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_c)
    s_in.wait_stream(s_c)
    s_out.wait_stream(s_c)
    for i in range(steps):
        step(i)
    join()
    b.record(s_c)
    torch.cuda.synchronize()
    ms = max_over_ranks([a.elapsed_time(b)], device, dist)
    value = world * effective_flops(w) * steps / (ms[0] * 1e-3) / 1e12
    return {"value": value, "unit": "TFLOPS", "steps": steps,
            "h2d_bytes_per_step": int(hq.numel() * 2 + hk.numel() * 2 + hv.numel() * 2),
            "d2h_bytes_per_step": int(sets[0][5].numel() * 2 + sets[0][6].numel() * 4),
            "ms_per_step": ms[0] / steps,
            "note": "steps pipelined over two buffer sets: host-to-device copies of the next step and "
                    "device-to-host copies of the previous step overlap the current step's kernels"}


if __name__ == "__main__":
    main()
