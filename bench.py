#!/usr/bin/env python
"""Benchmark of the RRAttention sparse prefill layer (estimate + select + sparse attention).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2] [--impl ours|reference]

One step = one full layer of the named workload (default: the Llama-3-8B-shaped layer at
L = 131072, 32/8 heads, d = 128, S = 16, B = 128, tau = 0.9) on seeded synthetic bf16 inputs.
Prints one JSON line.  ``value`` is effective TFLOP/s: dense-causal attention FLOPs
4*d*H*L(L+1)/2 per layer, times the layers all ranks processed, divided by the max-over-ranks
device time.  Under torchrun each rank runs its own layer (independent problems, weak
scaling, no data-path collective); with ``--shard heads`` the ranks split one layer by whole
KV groups instead (strong scaling, still no data-path collective).  ``--impl reference``
times the CPU oracle on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "ms/layer sparse prefill (estimate+select+attn) at 128K; effective TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def dense_causal_flops(w) -> float:
    return 4.0 * w.d * w.H * w.L * (w.L + 1) / 2.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def profile_record(name):
    """The committed counter record ``profiles/<name>.json`` of one kernel (written from an
    ncu capture), or None.  It carries the sha256 (first 16 hex digits) of every source the
    kernel is built from; the record is stale, and None is returned, when any differs now."""
    import hashlib

    path = os.path.join(ROOT, "profiles", name + ".json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    for src, digest in rec.get("sources", {}).items():
        full = os.path.join(ROOT, src)
        if not os.path.exists(full) or hashlib.sha256(open(full, "rb").read()).hexdigest()[:16] != digest:
            return None
    return rec


# committed DRAM counter record of the prefill kernel that serves each block size
PREFILL_RECORDS = {128: "prefill_pp_llama3-8b-layer-L32k"}


def prefill_traffic_per_launch(w):
    """DRAM bytes (read + write) per prefill launch from the committed capture, scaled by L
    from the captured layer to this one (Q, K, V and O all grow linearly with L at fixed heads
    and d).  None when the kernel changed since the capture, no capture covers this block
    size, or the layer shape differs."""
    name = PREFILL_RECORDS.get(w.B)
    rec = profile_record(name) if name else None
    if rec is None:
        return None
    if (w.H, w.Hkv, w.d, w.B) != tuple(rec["shape"][k] for k in ("H", "Hkv", "d", "B")):
        return None
    return (rec["dram_bytes_read"] + rec["dram_bytes_write"]) * w.L / rec["shape"]["L"]


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float across the process group (the value itself when the job
    has one rank).  Every rank must call it at the same point."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world: int, flops_per_rank: float, ms: float) -> float:
    """Whole-job throughput: every rank processed flops_per_rank in the (max-over-ranks) ms."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        loaded = [x for x in sm if x >= 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------- CPU oracle
def oracle_sample(w, t, head: int, n_rows: int, seed: int):
    """One bounded sample of the oracle on the layer: the estimate and selection of query head
    `head` (all of its query blocks) and n_rows random prefill rows of that head under its
    selection, extrapolated linearly to the layer's H heads (the prefill part scaled by the keys
    attended by all rows of the head over the keys attended by the sampled rows).
    Returns (layer_seconds, seconds_measured, (A, row_ptr, col_idx, diag) of the head)."""
    import oracle

    h = head
    g = h // (w.H // w.Hkv)
    t0 = time.perf_counter()
    A = oracle.estimate(t["Q"], t["K"], w.S, w.B, heads=(h, h + 1))[h:h + 1]
    t1 = time.perf_counter()
    rp, ci, dg = oracle.select(A, w.tau, True, diag=True)
    t2 = time.perf_counter()
    rng = np.random.default_rng(seed)
    qs = np.sort(rng.choice(w.L, n_rows, replace=False))
    rows = [(0, int(q)) for q in qs]
    oracle.prefill_rows(t["Q"][h:h + 1], t["K"][g:g + 1], t["V"][g:g + 1], w.B, rp, ci, rows)
    t3 = time.perf_counter()
    est, sel, pre = t1 - t0, t2 - t1, t3 - t2
    B = w.B
    n_off = np.zeros(w.Nb, np.int64)
    has_diag = np.zeros(w.Nb, bool)
    for I in range(w.Nb):
        sel_I = ci[rp[I]:rp[I + 1]]
        has_diag[I] = bool((sel_I == I).any())
        n_off[I] = len(sel_I) - int(has_diag[I])
    keys_all = float((n_off * B * B).sum() + has_diag.sum() * B * (B + 1) / 2)
    Iq = qs // B
    keys_sample = float((n_off[Iq] * B + has_diag[Iq] * (qs - Iq * B + 1)).sum())
    layer = w.H * (est + sel + pre * keys_all / max(keys_sample, 1.0))
    return layer, t3 - t0, (A[0], rp, ci, dg)


def sample_text(w, n_rows):
    return (f"per sample: the oracle's estimate and selection of one query head (all {w.Nb} query "
            f"blocks) and {n_rows} random prefill rows of that head, extrapolated linearly to {w.H} "
            f"heads and {w.L} rows (the prefill part scaled by attended keys); value from the "
            f"median sample")


# ---------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle

    w = workloads.get(args.workload)
    if args.L:
        w = w.with_(L=args.L)
    t = workloads.generate(w)
    layer, measured = [], []
    for i in range(args.warmup + args.steps):
        layer_s, meas_s, _ = oracle_sample(w, t, head=i % w.H, n_rows=args.ref_rows, seed=i)
        if i >= args.warmup:
            layer.append(layer_s)
            measured.append(meas_s)
    layer_ms = 1e3 * statistics.median(layer)
    val = dense_causal_flops(w) / (layer_ms * 1e-3) / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        # the time one step (one bounded sample) actually took; the layer time it stands for is
        # extrapolated from it
        "ms_per_step": 1e3 * statistics.median(measured),
        "ms_per_layer_extrapolated": layer_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w, world),
        "cpu_baseline": {"kind": "oracle", "value": val, "unit": "TFLOP/s",
                         "cores": oracle.threads(), "sample": sample_text(w, args.ref_rows)},
        "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w, world, shard="replicas"):
    if world == 1:
        par = "single"
    elif shard == "heads":
        par = f"heads{world} (KV groups split across ranks, no data-path collective)"
    else:
        par = f"replicas{world}"
    return {"workload": w.name, "H": w.H, "Hkv": w.Hkv, "L": w.L, "d": w.d, "S": w.S, "B": w.B,
            "tau": w.tau, "recipe": w.recipe,
            "global_batch": world if shard == "replicas" else 1, "seq_len": w.L,
            "parallelism": par,
            "l2": "inputs larger than L2 (Q+K+V %.2f GB > 126 MB); no flush" %
                  (2 * w.L * w.d * (w.H + 2 * w.Hkv) / 1e9)}


# ---------------------------------------------------------------------------- our arm
def selected_flops(rp, ci, H, Nb, B, d):
    rows = np.repeat(np.arange(H * Nb) % Nb, np.diff(rp))
    diag = int((ci == rows).sum())
    off = len(ci) - diag
    return 4.0 * d * (off * B * B + diag * B * (B + 1) / 2.0), diag, off


def run_ours(args):
    import torch

    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        import datetime

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    import long_context_prefill_estimate_b200 as rr

    rr.lib()  # fail loudly if the CUDA library is missing
    w = workloads.get(args.workload)
    if args.L:
        w = w.with_(L=args.L)
    if args.shard == "heads":
        # one layer split by whole KV groups: every rank holds the same layer and computes
        # its query heads [h0, h1) with their layer-wide round-robin offsets (strong scaling)
        full = workloads.generate(w, seed=0)
        h0, h1, g0, g1 = rr.head_shard(rank, world, w.H, w.Hkv)
        host = {"Q": full["Q"][h0:h1].contiguous(), "K": full["K"][g0:g1].contiguous(),
                "V": full["V"][g0:g1].contiguous()}
        wl = w.with_(H=h1 - h0, Hkv=g1 - g0)
    else:
        # one independent layer per rank (weak scaling)
        full = host = workloads.generate(w, seed=rank)
        h0, wl = 0, w
    d = {k: v.to(dev) for k, v in host.items()}
    Q, K, V = d["Q"], d["K"], d["V"]
    ws = rr.Workspace(wl.H, wl.Hkv, wl.L, wl.d, wl.S, wl.B, device=dev)
    O = torch.empty_like(Q)
    st = torch.cuda.current_stream(dev)

    def step(ev=None, tau=None):
        if ev:
            ev[0].record(st)
        rr.estimate(Q, K, w.S, w.B, out=ws.block_scores, workspace=ws.est, head_base=h0)
        if ev:
            ev[1].record(st)
        rr.select(ws.block_scores, w.tau if tau is None else tau, True, row_ptr=ws.row_ptr,
                  col_idx=ws.col_idx, nnz=ws.nnz, workspace=ws.sel)
        if ev:
            ev[2].record(st)
        rr.sparse_prefill(Q, K, V, ws.row_ptr, ws.col_idx, w.B, out=O)
        if ev:
            ev[3].record(st)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clk = ClockSampler(dev.index if dev.index is not None else 0)
    clk.start()
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(st)
    for i in range(args.steps):
        step(evs[i])
    t_end.record(st)
    torch.cuda.synchronize()
    barrier()
    clocks = clk.stop()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), dev)
    ms_step = total_ms / args.steps
    stage = {k: statistics.mean(e[a].elapsed_time(e[b]) for e in evs)
             for k, (a, b) in {"estimate_ms": (0, 1), "select_ms": (1, 2),
                               "prefill_ms": (2, 3)}.items()}
    rp = ws.row_ptr.cpu().numpy()
    nnz = int(rp[-1])
    ci = ws.col_idx[:nnz].cpu().numpy()
    A_sample = ws.block_scores[:min(args.cpu_samples, wl.H)].cpu().numpy() \
        if rank == 0 and not args.no_cpu_baseline else None
    sel_flops, n_diag, n_off = selected_flops(rp, ci, wl.H, wl.Nb, wl.B, wl.d)
    causal_blocks = wl.H * wl.Nb * (wl.Nb + 1) // 2
    dense = dense_causal_flops(w)
    # whole-job throughput: weak scaling processes one layer per rank, head sharding one
    # layer in all
    layers = world if args.shard == "replicas" else 1
    peaks, peak_kind = load_peaks()
    prefill_tflops = sel_flops / (stage["prefill_ms"] * 1e-3) / 1e12
    est_bytes = (2 * wl.Hkv * wl.L * wl.d           # K read
                 + 2 * wl.H * wl.Ns * wl.d          # sampled Q rows
                 + 4 * wl.Hkv * wl.Ns * wl.d * 2    # pooled keys written + read
                 + 4 * wl.H * wl.Nb * wl.Nb)        # block scores written
    sel_bytes = 4 * wl.H * wl.Nb * wl.Nb + 4 * (wl.H * wl.Nb + 1) + 4 * nnz
    # estimator's algorithmic work: one logit (2*d FLOP) and one exponential per causal
    # stride pair (i, j <= i) of every query head
    pairs = wl.H * wl.Ns * (wl.Ns + 1) / 2
    est_s = stage["estimate_ms"] * 1e-3
    line = {
        "metric": METRIC,
        "value": aggregate_tflops(layers, dense, ms_step),
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_step, "ms_per_layer": ms_step,
        "higher_is_better": True, "scaling": "weak" if args.shard == "replicas" else "strong",
        "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded generator, no datasets or weights)",
        "config": config_dict(w, world, args.shard),
        "stages": {**stage,
                   "estimate_gbs": est_bytes / (stage["estimate_ms"] * 1e-3) / 1e9,
                   "select_gbs": sel_bytes / (stage["select_ms"] * 1e-3) / 1e9,
                   "estimate_tflops": 2 * wl.d * pairs / est_s / 1e12,
                   "estimate_gexp_per_s": pairs / est_s / 1e9,
                   "prefill_tflops_selected": prefill_tflops},
        "density": nnz / causal_blocks,
        "selected_blocks": nnz, "diag_blocks": n_diag,
        "roofline": {"kernel": "sparse prefill", "bound": "tensor", "achieved": prefill_tflops,
                     "peak": peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                     "unit": "TFLOP/s",
                     "frac": prefill_tflops / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                     "frac_of_burst": prefill_tflops / peaks["bf16_tflops"],
                     "peak_source": f"{peak_kind} bf16 (sustained)",
                     "flops_per_launch": sel_flops,
                     "traffic": prefill_traffic_per_launch(wl),
                     "traffic_unit": "bytes/launch (ncu dram read+write at L=32768, scaled by L)"},
        # per step: key pooling, estimate, select (warp-per-row kernel, plus the sorting kernel
        # when rows exceed 1024 blocks), count scan, CSR emit, prefill
        "gpu_launches": (6 + (1 if wl.Nb > 1024 else 0)) * args.steps,
        "clocks": clocks,
    }
    # estimator against its two candidate bounds: the bf16 tensor peak (its logits) and the
    # SFU (16 exp2 per clock per SM x 148 SMs at the measured SM clock)
    st_ = line["stages"]
    st_["estimate_frac_tensor"] = st_["estimate_tflops"] / line["roofline"]["peak"]
    if clocks and clocks.get("sm_mhz"):
        st_["estimate_frac_sfu"] = st_["estimate_gexp_per_s"] / (16 * 148 * clocks["sm_mhz"] * 1e-3)
    # ---- extra measurements (outside the timed region)
    if rank == 0 and not args.quick:
        line["tau_sweep"] = tau_sweep(wl, step, st, ws, torch)
        line["dense_reference"] = dense_comparison(wl, Q, K, V, ws, rr, torch, st, ms_step)
        line["pattern_discovery"] = pattern_discovery(wl, Q, K, ws, rr, torch, st, stage)
    line["e2e"] = e2e(w, wl, host, h0, layers, rr, torch, dev, args)
    if rank == 0 and not args.no_cpu_baseline:
        import oracle
        from long_context_prefill_estimate_b200 import diagnostics

        heads = [i % wl.H for i in range(args.cpu_samples)]
        layer, measured, counts = [], 0.0, None
        gpu_rows = diagnostics.csr_rows(rp, ci)
        for i, h in enumerate(heads):
            layer_s, meas_s, (A_o, rp_o, ci_o, dg_o) = oracle_sample(wl, host, h, args.ref_rows, seed=i)
            layer.append(layer_s)
            measured += meas_s
            if i < wl.H:  # masks of each sampled head against the GPU's (boundary rule 1e-4)
                c, bad = diagnostics.classify_masks(gpu_rows[h * wl.Nb:(h + 1) * wl.Nb],
                                                    diagnostics.csr_rows(rp_o, ci_o), dg_o, A_o,
                                                    A_sample[h])
                c["unexplained"] = len(bad)
                counts = c if counts is None else {k: counts[k] + c[k] for k in c}
        layer_s = statistics.median(layer)
        line["cpu_baseline"] = {
            "value": dense / layer_s / 1e12 * (1 if args.shard == "replicas" else wl.H / w.H),
            "unit": "TFLOP/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": sample_text(wl, args.ref_rows) + f"; {len(heads)} samples, "
                      f"{measured:.1f} s measured",
        }
        line["mask_parity"] = {**counts, "heads": sorted(set(heads)),
                               "rule": "GPU vs oracle masks of the sampled heads, each side "
                                       "from its own scores; boundary = oracle cum within 1e-4 "
                                       "of tau*T (all heads: profiles/mask_parity_full_size.json)"}
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def tau_sweep(w, step, st, ws, torch):
    out = {}
    for tau in (0.8, 0.9, 0.95):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        step(tau=tau)
        torch.cuda.synchronize()
        step(ev, tau=tau)
        torch.cuda.synchronize()
        nnz = int(ws.row_ptr[-1].item())
        out[str(tau)] = {"density": nnz / (w.H * w.Nb * (w.Nb + 1) // 2),
                         "ms": ev[0].elapsed_time(ev[3]),
                         "prefill_ms": ev[2].elapsed_time(ev[3])}
    return out


def pattern_discovery(w, Q, K, ws, rr, torch, st, stage):
    """Pattern-discovery time (estimate + select) of the round-robin estimator (the timed
    stages) and of XAttention's antidiagonal estimator on the same layer (the comparison of the
    RRAttention page, Sec. 4.2 "Runtime Efficiency", Fig. 3(b)), with the density each keeps."""
    res = {"rr_ms": stage["estimate_ms"] + stage["select_ms"]}
    try:
        A = torch.empty_like(ws.block_scores)
        rp = torch.empty_like(ws.row_ptr)
        ci = torch.empty_like(ws.col_idx)
        nnz = torch.empty_like(ws.nnz)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        t_est, t_sel = [], []
        for i in range(4):
            ev[0].record(st)
            rr.xattn_estimate(Q, K, w.S, w.B, out=A)
            ev[1].record(st)
            rr.select(A, w.tau, True, row_ptr=rp, col_idx=ci, nnz=nnz, workspace=ws.sel)
            ev[2].record(st)
            torch.cuda.synchronize()
            if i:
                t_est.append(ev[0].elapsed_time(ev[1]))
                t_sel.append(ev[1].elapsed_time(ev[2]))
        res["xattention_estimate_ms"] = statistics.median(t_est)
        res["xattention_ms"] = statistics.median(t_est) + statistics.median(t_sel)
        res["rr_time_saved"] = 1.0 - res["rr_ms"] / res["xattention_ms"]
        res["xattention_density"] = int(nnz.item()) / (w.H * w.Nb * (w.Nb + 1) // 2)
    except Exception as exc:  # sizes the comparison kernel does not cover
        res["xattention_error"] = str(exc)[:200]
    return res


def dense_comparison(w, Q, K, V, ws, rr, torch, st, ms_sparse):
    """Dense causal attention on the same GPU: our kernel with every causal block, and torch
    SDPA (flash/cuDNN library kernel) as context."""
    res = {}
    Nb = w.Nb
    counts = np.tile(np.arange(1, Nb + 1), w.H)
    rp = torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)).to(Q.device)
    ci = torch.from_numpy(np.concatenate([np.arange(I + 1) for _ in range(w.H) for I in range(Nb)]
                                         ).astype(np.int32)).to(Q.device)
    O = torch.empty_like(Q)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    rr.sparse_prefill(Q, K, V, rp, ci, w.B, out=O)
    e0.record(st)
    rr.sparse_prefill(Q, K, V, rp, ci, w.B, out=O)
    e1.record(st)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    res["ours_tau1_ms"] = ms
    res["ours_tau1_tflops"] = dense_causal_flops(w) / (ms * 1e-3) / 1e12
    res["speedup_vs_ours_dense"] = ms / ms_sparse
    try:
        G = w.H // w.Hkv
        q = Q.unsqueeze(0)
        k = K.unsqueeze(0)
        v = V.unsqueeze(0)
        torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)
        e0.record(st)
        torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)
        e1.record(st)
        torch.cuda.synchronize()
        ms2 = e0.elapsed_time(e1)
        res["sdpa_ms"] = ms2
        res["sdpa_tflops"] = dense_causal_flops(w) / (ms2 * 1e-3) / 1e12
        res["speedup_vs_sdpa"] = ms2 / ms_sparse
        del G
    except Exception as exc:  # library kernel unavailable for this shape
        res["sdpa_error"] = str(exc)[:200]
    return res


def e2e(w, wl, host, h0, layers, rr, torch, dev, args):
    """The rank's part of the job through the public API from pinned host buffers: H2D of
    Q/K/V, the three stages, D2H of O, every step inside the timed region (the API overlaps
    the copies of one slice of KV groups with the compute of another)."""
    pinned = {k: v.pin_memory() for k, v in host.items()}
    out = torch.empty(pinned["Q"].shape, dtype=torch.bfloat16, pin_memory=True)
    st = torch.cuda.current_stream(dev)
    run = lambda: rr.prefill(pinned["Q"], pinned["K"], pinned["V"], w.S, w.B, w.tau, out=out,
                             head_base=h0)
    for _ in range(max(1, args.warmup)):
        run()
    n = max(1, args.steps)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(n):
        run()
    e1.record(st)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / n, dev)
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    return {"value": aggregate_tflops(layers, dense_causal_flops(w), ms), "unit": "TFLOP/s",
            "ms_per_step": ms, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": out.numel() * out.element_size(), "steps": n,
            "pipeline": f"{len(rr.host_slices(wl.H, wl.Hkv, rr.default_chunks(wl.Hkv)))} slices "
                        f"(whole KV groups; the first and last query heads alone); copy-in, "
                        f"compute and copy-out on three streams"}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=2, help="index into workloads.WORKLOADS")
    ap.add_argument("--L", type=int, default=0, help="override the sequence length")
    ap.add_argument("--quick", action="store_true", help="skip the tau sweep and dense comparison")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-samples", type=int, default=12,
                    help="oracle samples (one query head each) of the CPU baseline")
    ap.add_argument("--ref-rows", type=int, default=1024,
                    help="prefill rows per oracle sample (CPU baseline and reference arm)")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="replicas: one independent layer per GPU (weak scaling); heads: one "
                         "layer split across the GPUs by whole KV groups (strong scaling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
