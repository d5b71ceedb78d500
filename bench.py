#!/usr/bin/env python
"""Benchmark: one step = the whole hot path on the 128K last-chunk workload.

Workload (one LLaMA-3.1-8B attention layer, last chunk of a 128K prompt):
32 query heads / 8 KV heads, head_dim 128, bf16, prefix 129024 + chunk 2048
tokens, block = page = 64 tokens, randomly permuted pages, vertical-slash
masks (sink, 8-block local window, 5% columns shared 70% within a group).

Step = ca_build_tables (Q-block + intra-group union, compaction) followed by
ca_chunk_attention (paged, in place) on device-resident inputs.  Four input
sets (distinct page buffers and masks) rotate between steps so that a step
never finds the previous step's selected pages in L2.

value = selected-block FLOPs per step / device time per step (TFLOP/s);
e2e   = the same metric through the public API with pinned host buffers:
        H2D of the mask, Q, the chunk's new K/V rows and the page table,
        KV append into the paged cache + build + attention, D2H of O and LSE,
        all inside the timed region, pipelined over three streams (copies of
        one step overlap the compute of the previous one).
Also reported: the density-100% path on the same shapes (attention speedup),
the batched table builder in GB/s (32 masks per launch, and 128 to show
saturation), roofline fractions
against the measured peaks, and the float64 oracle timed on host cores.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]
Under torchrun every rank runs its own replica of the workload (weak scaling,
no collective on the data path); rank 0 prints one JSON line.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "chunk attn ms & TFLOP/s (selected blocks) vs dense at 128K; table build GB/s"
WORKLOAD = ("ctx128k: Hq 32 / Hkv 8, d 128, bf16, prefix 129024 + chunk 2048, block 64, "
            "paged KV with random page permutation, vertical-slash masks (rho_col 0.05, "
            "corr 0.7, window 8)")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return d, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


def kernel_source_digest(path):
    """sha256 of a CUDA source (and the csrc headers it includes) with comments
    and blank lines removed, so that a comment edit does not count as a kernel
    change."""
    import hashlib
    import re
    d = os.path.dirname(path)
    text = "".join(open(os.path.join(d, f)).read()
                   for f in [os.path.basename(path), "attn_common.cuh", "ptx.cuh", "internal.h"]
                   if os.path.exists(os.path.join(d, f)))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    lines = [ln.rstrip() for ln in text.splitlines() if ln.strip()]
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()


def load_traffic():
    """DRAM bytes per attention launch from the committed ncu capture
    (profiles/chunk_attn_pair_kernel_ctx128k_traffic.json), or None when the
    kernel source has changed since that capture."""
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles",
                                          "chunk_attn_pair_kernel_ctx128k_traffic.json")))
        src = os.path.join(ROOT, "block_sparse_chunked_b200", "csrc", "attn_pair.cu")
        if kernel_source_digest(src) != rec["source_digest"]:
            return None
        return float(rec["dram_bytes_read"]) + float(rec["dram_bytes_write"])
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 20 ms during the timed
    region (the default 400 steps take ~0.2 s); the SM clock is the median of
    the samples under load (power draw in the upper half of the range seen, all
    samples if the range is flat)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        return self.summarize(self.lines)

    @staticmethod
    def summarize(lines):
        """The clock record from nvidia-smi CSV lines (the query above, no
        header or units): median SM clock of the samples under load, the max
        clock seen, and the throttle reasons active in any sample."""
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = sm
        if len(power) == len(sm) and max(power) - min(power) > 20.0:
            cut = (max(power) + min(power)) / 2
            loaded = [c for c, w in zip(sm, power) if w >= cut]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "samples": len(sm), "samples_under_load": len(loaded),
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons)}


def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of a list of floats over all ranks (the device times
    of a step are reported as the slowest rank's)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def make_sets(w, nsets, dev):
    """nsets input sets on the device: distinct page buffers (same values, distinct
    addresses) and masks drawn with seeds 0..nsets-1."""
    import torch

    import workloads
    x = workloads.make_qkv_pages(w, seed=0)
    base = {k: v.to(dev) for k, v in x.items()}
    sets = []
    for s in range(nsets):
        m = torch.from_numpy(workloads.mask_for(w, seed=s)).to(dev)
        d = {"Q": base["Q"].clone(), "K": base["K_pages"].clone(), "V": base["V_pages"].clone(),
             "pt": base["page_table"].clone(), "mask": m,
             "tables": torch.empty(w.Hkv, w.nKblk, dtype=torch.int32, device=dev),
             "counts": torch.empty(w.Hkv, dtype=torch.int32, device=dev),
             "O": torch.empty_like(base["Q"]),
             "LSE": torch.empty(w.Hq, w.chunk_len, dtype=torch.float32, device=dev)}
        sets.append(d)
    return x, sets


def run_sweep(bsc, dev, stream, n_chunks=32):
    """The full chunked-prefill sweep: 131072 tokens in 32 chunks of 4096 over one
    growing paged cache (random page permutation).  Per chunk the KV append is
    timed apart; the method's time is the table build + attention.  Chunk data
    come from a seeded device generator; each chunk runs once, in order."""
    import numpy as np
    import torch

    import workloads as wl
    last = wl.sweep_chunk(n_chunks - 1)
    nK_all, Hkv, B, d, Hq = last.nKblk, last.Hkv, last.block, last.head_dim, last.Hq
    rng = np.random.default_rng(0)
    pt = torch.from_numpy(rng.permutation(nK_all).astype(np.int32)).to(dev)
    K = torch.zeros(nK_all, Hkv, B, d, dtype=torch.bfloat16, device=dev)
    V = torch.zeros_like(K)
    g = torch.Generator(device=dev).manual_seed(0)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    method_ms, append_ms, sel, dense = [], [], 0.0, 0.0
    for c in range(n_chunks):
        w = wl.sweep_chunk(c)
        L = w.chunk_len
        kn, vn = (torch.randn(L, Hkv, d, generator=g, device=dev).bfloat16() for _ in range(2))
        q = torch.randn(L, Hq, d, generator=g, device=dev).bfloat16()
        mask = torch.from_numpy(wl.mask_for(w)).to(dev)
        tables = torch.empty(Hkv, w.nKblk, dtype=torch.int32, device=dev)
        counts = torch.empty(Hkv, dtype=torch.int32, device=dev)
        O = torch.empty_like(q)
        lse = torch.empty(Hq, L, dtype=torch.float32, device=dev)
        append_ms.append(timed_launch(stream, lambda: bsc.append_kv(kn, vn, K, V, pt, w.prefix_len,
                                                                      err_flag=err)))

        def method():
            bsc.build_tables(mask, Hkv, tables, counts)
            bsc.chunk_attention(q, K, V, pt, tables, counts, w.prefix_len, err_flag=err, out=O,
                                lse=lse)
        method_ms.append(timed_launch(stream, method))
        sel += bsc.selected_flops(tables.cpu().numpy(), counts.cpu().numpy(), Hq, w.nPblk,
                                  w.nQblk, B, d)
        dense += bsc.dense_flops(Hq, w.nPblk, w.nQblk, B, d)
    bsc.check(err)
    tot = sum(method_ms)
    return {"chunks": n_chunks, "tokens": n_chunks * last.chunk_len,
            "method_total_ms": tot, "append_total_ms": sum(append_ms),
            "selected_tflop": sel / 1e12, "dense_tflop": dense / 1e12,
            "tflops_selected": sel / (tot * 1e-3) / 1e12,
            "per_chunk_ms_first_last": [method_ms[0], method_ms[-1]]}


# The bench's two batches: 8 sequences of long unaligned chunks (many units),
# and 4 short chunks over long prefixes (9 query spans x 8 groups x 2 head
# pairs = 144 units, fewer than the SMs).
VARLEN_LONG = [(121037, 2048), (64005, 1500), (32868, 1024), (100063, 777), (8000, 512),
               (120001, 2000), (50030, 1900), (90011, 1100)]
VARLEN_SHORT = [(121037, 192), (64005, 128), (32868, 160), (100063, 64)]


def run_varlen(bsc, dev, stream, seqs=VARLEN_LONG, n_splits=1, reps=12,
               note="ca_chunk_attention_varlen, unaligned prefixes and chunk lengths, one launch"):
    """A batch of sequences with unaligned prefixes and chunk lengths over one
    shuffled page pool, through one ca_chunk_attention_varlen launch (tables
    built per sequence beforehand).  Seeded device data; 32/8 heads, d 128.
    Times lone launches (behind a sleep kernel) and, for the same work, eight
    launches back to back between one pair of events."""
    import numpy as np
    import torch

    import workloads as wl
    Hq, Hkv, d, B = 32, 8, 128, 64
    nKs = [-(-(P + L) // B) for P, L in seqs]
    num_pages = sum(nKs)
    g = torch.Generator(device=dev).manual_seed(0)
    K = torch.randn(num_pages, Hkv, B, d, generator=g, device=dev).bfloat16()
    V = torch.randn(num_pages, Hkv, B, d, generator=g, device=dev).bfloat16()
    rng = np.random.default_rng(0)
    pt = torch.from_numpy(rng.permutation(num_pages).astype(np.int32)).to(dev)
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum([L for _, L in seqs])]), dtype=torch.int32,
                        device=dev)
    cu_pages = torch.tensor(np.concatenate([[0], np.cumsum(nKs)]), dtype=torch.int32, device=dev)
    prefix = torch.tensor([P for P, _ in seqs], dtype=torch.int32, device=dev)
    total_q = int(cu_q[-1])
    Q = torch.randn(total_q, Hq, d, generator=g, device=dev).bfloat16()
    flat = torch.full((Hkv * num_pages,), -1, dtype=torch.int32, device=dev)
    counts = torch.zeros(len(seqs), Hkv, dtype=torch.int32, device=dev)
    flops = 0.0
    off = 0
    for s, (P, L) in enumerate(seqs):
        w = wl.Workload("vb", Hq, Hkv, d, "bf16", P, L, B, "vslash", rho=0.05, corr=0.7,
                        window=8, seed=s)
        t = flat[Hkv * off:Hkv * (off + nKs[s])].view(Hkv, nKs[s])
        bsc.build_tables(torch.from_numpy(wl.mask_for(w)).to(dev), Hkv, t, counts[s])
        flops += bsc.selected_flops_pl(t.cpu().numpy(), counts[s].cpu().numpy(), Hq, P, L, B, d)
        off += nKs[s]
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    O = torch.empty_like(Q)
    lse = torch.empty(Hq, total_q, dtype=torch.float32, device=dev)
    max_kv = max(P + L for P, L in seqs)
    n = bsc.lib.ca_workspace_size_varlen(0, Hq, Hkv, d, B, len(seqs), total_q, max_kv, num_pages,
                                         n_splits)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    call = lambda: bsc.chunk_attention_varlen(  # noqa: E731
        Q, K, V, cu_q, prefix, pt, cu_pages, flat, counts, max_kv, n_splits=n_splits,
        err_flag=err, out=O, lse=lse, workspace=ws)
    ts = []
    for r in range(reps):
        t_ = timed_launch(stream, call)
        if r >= 3:
            ts.append(t_)
    b2b = timed_launch(stream, lambda: [call() for _ in range(8)]) / 8
    bsc.check(err)
    ms = sum(ts) / len(ts)
    units = sum(-(-L // 64) for _, L in seqs) * Hkv * ((Hq // Hkv + 1) // 2)
    return {"sequences": len(seqs), "query_tokens": total_q, "kv_tokens": sum(P + L for P, L in seqs),
            "units": units, "n_splits": n_splits, "ms": ms, "selected_gflop": flops / 1e9,
            "tflops": flops / (ms * 1e-3) / 1e12, "back_to_back_ms": b2b,
            "back_to_back_tflops": flops / (b2b * 1e-3) / 1e12, "note": note}


def run_density_sweep(bsc, dev, stream, reps=5):
    """The 64K density / correlation sweep: prefix 63488 + chunk 2048, 32/8 heads,
    d 128, bf16, block 64 and 128.  rho is the vertical-slash generator's column
    density (sink block and 8-block (B 64) or 4-block (B 128) local window on
    top); rho = 1 is the all-ones mask, once per block size.  Per cell: the
    attention's device time (mean of `reps` launches after one warm-up), the
    selected FLOPs, the table density, and the speedup over the same block
    size's rho = 1 cell.  Page data are seeded device normals, one pool per
    block size (256 MiB of K and V, more than L2 holds)."""
    import numpy as np
    import torch

    import workloads as wl
    out = {"rho_meaning": "column density of the vertical-slash generator (sink and local "
                          "window added on top); rho = 1: all-ones mask",
           "cells": []}
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for block in (64, 128):
        w1 = wl.density_cell(1.0, 0.0, block=block)
        g = torch.Generator(device=dev).manual_seed(block)
        K = torch.randn(w1.num_pages, w1.Hkv, block, w1.head_dim, generator=g, device=dev).bfloat16()
        V = torch.randn(w1.num_pages, w1.Hkv, block, w1.head_dim, generator=g, device=dev).bfloat16()
        Q = torch.randn(w1.chunk_len, w1.Hq, w1.head_dim, generator=g, device=dev).bfloat16()
        pt = torch.from_numpy(np.random.default_rng(block).permutation(w1.num_pages)
                              .astype(np.int32)).to(dev)
        O = torch.empty_like(Q)
        lse = torch.empty(w1.Hq, w1.chunk_len, dtype=torch.float32, device=dev)
        n = bsc.workspace_size(torch.bfloat16, w1.Hq, w1.Hkv, w1.head_dim, block, w1.chunk_len,
                               w1.prefix_len, w1.num_pages)
        ws = torch.empty(max(n, 1), dtype=torch.uint8, device=dev)
        cells = [(1.0, 0.0)] + [(r, c) for r in (0.5, 0.2, 0.1, 0.05) for c in (0.0, 0.5, 1.0)]
        base_ms = None
        for rho, corr in cells:
            w = wl.density_cell(rho, corr, block=block)
            tables, counts = bsc.build_tables(torch.from_numpy(wl.mask_for(w)).to(dev), w.Hkv)
            run = lambda: bsc.chunk_attention(Q, K, V, pt, tables, counts, w.prefix_len,
                                              err_flag=err, out=O, lse=lse, workspace=ws)
            run()
            ms = statistics.mean(timed_launch(stream, run) for _ in range(reps))
            flops = bsc.selected_flops(tables.cpu().numpy(), counts.cpu().numpy(), w.Hq, w.nPblk,
                                       w.nQblk, block, w.head_dim)
            if base_ms is None:
                base_ms = ms
            out["cells"].append({"block": block, "rho": rho, "corr": corr, "ms": ms,
                                 "tflops": flops / (ms * 1e-3) / 1e12,
                                 "table_density": float(counts.float().mean().item() / w.nKblk),
                                 "selected_gflop": flops / 1e9,
                                 "speedup_vs_rho1": base_ms / ms})
        bsc.check(err)
        del K, V
    return out


def timed_launch(stream, fn):
    """Device time (ms) of the launches fn() makes.  A sleep kernel keeps the
    GPU busy while the host enqueues them, so the host-side call overhead of a
    lone launch does not land between the two events."""
    import torch

    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(200_000)  # ~0.1 ms at the B200's clocks
    a.record(stream)
    fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def run_step(bsc, w, s, ws, err):
    bsc.build_tables(s["mask"], w.Hkv, s["tables"], s["counts"])
    bsc.chunk_attention(s["Q"], s["K"], s["V"], s["pt"], s["tables"], s["counts"],
                        w.prefix_len, err_flag=err, out=s["O"], lse=s["LSE"], workspace=ws)


def cpu_oracle_sample(w, x, mask, budget_s=12.0, stride=None):
    """Time the float64 oracle (tables in full + attention on a row sample) on host cores."""
    import numpy as np

    import oracle
    t0 = time.perf_counter()
    t, c = oracle.oracle_tables(mask, w.Hkv)
    t_tab = time.perf_counter() - t0
    G = w.G
    live = {}
    for g in range(w.Hkv):
        row = t[g, :c[g]]
        live[g] = np.searchsorted(row, w.nPblk + np.arange(w.nQblk), side="right")
    # calibrate: a first small sample, then grow the stride-sample to fill the budget
    Qd = x["Q"].double().numpy()
    stride = stride or 4
    rows = [(h, i) for i in range(0, w.chunk_len, stride) for h in range(w.Hq)]
    t0 = time.perf_counter()
    oracle.oracle_rows(Qd, x["K_pages"], x["V_pages"], x["page_table"].numpy(), t, c,
                       w.prefix_len, rows)
    dt = time.perf_counter() - t0
    flops = sum(4.0 * w.head_dim * w.block * live[h // G][i // w.block] for h, i in rows)
    # total selected FLOPs of the chunk, from the oracle's own tables (this leg
    # must not load the CUDA library)
    tot_flops = sum(4.0 * w.head_dim * w.block * w.block * int(live[h // G].sum())
                    for h in range(w.Hq))
    try:
        from threadpoolctl import threadpool_info
        blas = max([d.get("num_threads", 1) for d in threadpool_info()] or [1])
    except Exception:
        blas = 1
    return {
        "value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": int(blas),
        "host_cpus": len(os.sched_getaffinity(0)), "kind": "oracle",
        "sample": (f"float64 oracle: tables for the full mask ({t_tab:.2f} s) + attention for "
                   f"{len(rows)} of {w.Hq * w.chunk_len} query rows (all heads, every "
                   f"{stride}th token), {flops / 1e9:.1f} of {tot_flops / 1e9:.1f} selected GFLOP, "
                   f"{dt:.2f} s"),
        "seconds": dt + t_tab,
    }


def reference_arm(args, rank):
    """The oracle as the reference implementation, timed on the host cores."""
    import workloads
    if rank != 0:
        return
    w = workloads.get_config("ctx128k")
    x = workloads.make_qkv_pages(w, seed=0)
    mask = workloads.mask_for(w, seed=0)
    for _ in range(args.warmup):
        cpu_oracle_sample(w, x, mask, stride=256)
    # every 64th token per step up to 150 steps, then a sparser sample per step
    # (the stride doubles), so that K steps stay around a minute of host time
    stride = 64
    while stride < w.chunk_len and args.steps > 150 * (stride // 64):
        stride *= 2
    res = [cpu_oracle_sample(w, x, mask, stride=stride) for _ in range(args.steps)]
    v = statistics.mean(r["value"] for r in res)
    secs = statistics.mean(r["seconds"] for r in res)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "reference": "float64 CPU oracle (no published code)"},
        "cpu_baseline": {k: res[-1][k] for k in ("kind", "cores", "sample", "unit")} | {"value": v},
        "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sets", type=int, default=4)
    ap.add_argument("--builder-only", type=int, default=0, metavar="NB",
                    help="only run the batched table builder on NB 128K masks per launch "
                         "(the case used for the builder's ncu capture) and exit")
    ap.add_argument("--skip-extras", action="store_true",
                    help="time the step only (no dense path, batched builder, e2e): the small "
                         "case used for ncu captures")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        reference_arm(args, rank)
        return

    import numpy as np
    import torch

    import __graft_entry__
    __graft_entry__.build()
    import block_sparse_chunked_b200 as bsc
    import workloads

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    peaks, peak_src = load_peaks()
    w = workloads.get_config("ctx128k")
    if args.builder_only:
        nb = args.builder_only
        base = workloads.mask_for(w, seed=0)
        rng = np.random.default_rng(1)
        # distinct masks: each one a random column rotation of the seeded mask
        masks = torch.from_numpy(np.stack([np.roll(base, int(r), axis=2)
                                           for r in rng.integers(0, w.nKblk, nb)])).to(dev)
        tb = torch.empty(nb, w.Hkv, w.nKblk, dtype=torch.int32, device=dev)
        cb = torch.empty(nb, w.Hkv, dtype=torch.int32, device=dev)
        ts = []
        stream = torch.cuda.current_stream()
        for i in range(args.warmup + args.steps):
            t_ = timed_launch(stream, lambda: bsc.build_tables_batched(masks, w.Hkv, tb, cb))
            if i >= args.warmup:
                ts.append(t_)
        nbytes = bsc.builder_bytes(nb, w.Hq, w.Hkv, w.nQblk, w.nKblk)
        print(json.dumps({"builder_masks": nb, "bytes": nbytes, "us": statistics.mean(ts) * 1e3,
                          "GB/s": nbytes / (statistics.mean(ts) * 1e-3) / 1e9}), flush=True)
        return
    x, sets = make_sets(w, args.sets, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    ws_n = bsc.workspace_size(torch.bfloat16, w.Hq, w.Hkv, w.head_dim, w.block, w.chunk_len,
                              w.prefix_len, w.num_pages)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev)
    launches_per_step = 2 + (1 if ws_n > 0 else 0)
    stream = torch.cuda.current_stream()

    # ---- warm-up
    for i in range(args.warmup):
        run_step(bsc, w, sets[i % len(sets)], ws, err)
    torch.cuda.synchronize()
    bsc.check(err)

    # ---- timed region: K steps, per-step events around the builder and the attention
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    for i in range(args.steps):
        s = sets[i % len(sets)]
        ev[i][0].record(stream)
        bsc.build_tables(s["mask"], w.Hkv, s["tables"], s["counts"])
        ev[i][1].record(stream)
        bsc.chunk_attention(s["Q"], s["K"], s["V"], s["pt"], s["tables"], s["counts"],
                            w.prefix_len, err_flag=err, out=s["O"], lse=s["LSE"], workspace=ws)
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    clk = clocks.stop()
    bsc.check(err)
    step_ms = [ev[i][0].elapsed_time(ev[i][2]) for i in range(args.steps)]
    build_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]
    attn_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(args.steps)]
    set_flops = [bsc.selected_flops(s["tables"].cpu().numpy(), s["counts"].cpu().numpy(),
                                    w.Hq, w.nPblk, w.nQblk, w.block, w.head_dim) for s in sets]
    flops = [set_flops[i % len(sets)] for i in range(args.steps)]
    mean_step = statistics.mean(step_ms)
    mean_attn = statistics.mean(attn_ms)
    mean_flops = statistics.mean(flops)
    mean_step, mean_attn = max_over_ranks([mean_step, mean_attn], pg, dev)
    value = world * mean_flops / (mean_step * 1e-3) / 1e12
    attn_tflops = mean_flops / (mean_attn * 1e-3) / 1e12

    if args.skip_extras:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": world * mean_flops / (mean_step * 1e-3) / 1e12,
                              "unit": "TFLOP/s", "ms_per_step": mean_step, "attention_ms": mean_attn,
                              "note": "step only (--skip-extras)"}), flush=True)
        if pg:
            pg.destroy_process_group()
        return

    # ---- density-100% path on the same shapes (all blocks selected)
    dense_t = torch.arange(w.nKblk, dtype=torch.int32, device=dev).repeat(w.Hkv, 1).contiguous()
    dense_c = torch.full((w.Hkv,), w.nKblk, dtype=torch.int32, device=dev)
    dense_ms = []
    for i in range(2 + 4):
        s = sets[i % len(sets)]
        t_ = timed_launch(stream, lambda: bsc.chunk_attention(
            s["Q"], s["K"], s["V"], s["pt"], dense_t, dense_c, w.prefix_len, err_flag=err,
            out=s["O"], lse=s["LSE"], workspace=ws))
        if i >= 2:
            dense_ms.append(t_)
    bsc.check(err)
    dense_flops = bsc.dense_flops(w.Hq, w.nPblk, w.nQblk, w.block, w.head_dim)
    dense_ms_mean = statistics.mean(dense_ms)

    # ---- batched table builder: 32 masks per launch (one per layer), 4 rotating batches
    nb = 32
    import workloads as wl
    mb = [torch.from_numpy(np.stack([wl.mask_for(w, seed=100 + 32 * r + k) for k in range(nb)]))
          .to(dev) for r in range(4)]
    tb = torch.empty(nb, w.Hkv, w.nKblk, dtype=torch.int32, device=dev)
    cb = torch.empty(nb, w.Hkv, dtype=torch.int32, device=dev)
    for r in range(4):
        bsc.build_tables_batched(mb[r], w.Hkv, tb, cb)
    bt = []
    for r in range(12):
        bt.append(timed_launch(stream, lambda: bsc.build_tables_batched(mb[r % 4], w.Hkv, tb, cb)))
    bbytes = bsc.builder_bytes(nb, w.Hq, w.Hkv, w.nQblk, w.nKblk)
    build_gbs = bbytes / (statistics.mean(bt) * 1e-3) / 1e9
    # the same 12 launches back to back between one pair of events (each set
    # was last read three launches, 207 MB, earlier), and the floor a lone
    # launch pays under this event method: an empty kernel timed the same way
    a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(200_000)
    a_.record(stream)
    for r in range(12):
        bsc.build_tables_batched(mb[r % 4], w.Hkv, tb, cb)
    b_.record(stream)
    torch.cuda.synchronize()
    b2b_us = a_.elapsed_time(b_) * 1e3 / 12
    floor_us = statistics.mean(timed_launch(stream, lambda: torch.cuda._sleep(0))
                               for _ in range(8)) * 1e3
    # saturation: the four batches as one launch of 128 masks (277 MB, more than L2 holds)
    mb_all = torch.cat(mb)
    tb_all = torch.empty(4 * nb, w.Hkv, w.nKblk, dtype=torch.int32, device=dev)
    cb_all = torch.empty(4 * nb, w.Hkv, dtype=torch.int32, device=dev)
    bsc.build_tables_batched(mb_all, w.Hkv, tb_all, cb_all)
    bt_all = [timed_launch(stream, lambda: bsc.build_tables_batched(mb_all, w.Hkv, tb_all, cb_all))
              for _ in range(8)]
    sat_gbs = (bsc.builder_bytes(4 * nb, w.Hq, w.Hkv, w.nQblk, w.nKblk)
               / (statistics.mean(bt_all) * 1e-3) / 1e9)
    build_sat = {"masks_per_launch": 4 * nb, "us": statistics.mean(bt_all) * 1e3, "GB/s": sat_gbs,
                 "frac_of_measured_hbm": sat_gbs / peaks.get("hbm_gbs", FALLBACK["hbm_gbs"])}
    del mb_all, tb_all, cb_all
    # the same union from bit-packed masks (one bit per block), 32 and 128 masks per launch
    bits_res = {}
    for nbb in (32, 128):
        nrot = 4 if nbb == 32 else 2
        bb = [torch.from_numpy(wl.pack_mask_bits(np.stack([wl.mask_for(w, seed=300 + nbb * r + k)
                                                           for k in range(nbb)])).view(np.int32))
              .to(dev) for r in range(nrot)]
        tbb = torch.empty(nbb, w.Hkv, w.nKblk, dtype=torch.int32, device=dev)
        cbb = torch.empty(nbb, w.Hkv, dtype=torch.int32, device=dev)
        for r in range(nrot):
            bsc.build_tables_bits(bb[r], w.Hkv, w.nKblk, tbb, cbb)
        tt = []
        for r in range(12):
            tt.append(timed_launch(stream, lambda: bsc.build_tables_bits(bb[r % nrot], w.Hkv,
                                                                        w.nKblk, tbb, cbb)))
        nbytes = bsc.builder_bytes(nbb, w.Hq, w.Hkv, w.nQblk, w.nKblk, bits=True)
        gbs = nbytes / (statistics.mean(tt) * 1e-3) / 1e9
        bits_res[str(nbb)] = {"us": statistics.mean(tt) * 1e3, "GB/s": gbs,
                              "frac_of_measured_hbm": gbs / peaks.get("hbm_gbs", FALLBACK["hbm_gbs"]),
                              "mask_bytes_per_mask": w.Hq * w.nQblk * 4 * ((w.nKblk + 31) // 32)}
        del bb
    single_bytes = bsc.builder_bytes(1, w.Hq, w.Hkv, w.nQblk, w.nKblk)

    # ---- the builder fused into the attention prologue (bit-packed masks, one launch)
    for s_ in sets:
        s_["bits"] = torch.from_numpy(wl.pack_mask_bits(s_["mask"].cpu().numpy()).view(np.int32)).to(dev)
    ws_m = bsc.lib.ca_workspace_size_masked(0, w.Hq, w.Hkv, w.head_dim, w.block, w.chunk_len,
                                             w.prefix_len, w.num_pages, 0)
    ws_mt = torch.empty(max(ws_m, 1), dtype=torch.uint8, device=dev)
    fused_ms = []
    for i in range(args.warmup + 24):
        s_ = sets[i % len(sets)]
        t_ = timed_launch(stream, lambda: bsc.chunk_attention_masked(
            s_["Q"], s_["K"], s_["V"], s_["pt"], s_["bits"], w.prefix_len, err_flag=err,
            out=s_["O"], lse=s_["LSE"], workspace=ws_mt))
        if i >= args.warmup:
            fused_ms.append(t_)
    bsc.check(err)
    fused_res = {"ms": statistics.mean(fused_ms),
                 "tflops": mean_flops / (statistics.mean(fused_ms) * 1e-3) / 1e12,
                 "note": "ca_chunk_attention_masked: tables built in each CTA from bit-packed "
                         "masks, one launch; compare ms_per_step (builder + attention)"}

    # ---- E4M3 paged cache (one byte per K/V element, one scale per page and head)
    K8, sK8 = wl.quantize_pages_e4m3(x["K_pages"])
    V8, sV8 = wl.quantize_pages_e4m3(x["V_pages"])
    K8, sK8, V8, sV8 = K8.to(dev), sK8.to(dev), V8.to(dev), sV8.to(dev)
    ws_f8 = torch.empty(bsc.lib.ca_workspace_size_fp8(w.Hq, w.Hkv, w.head_dim, w.block,
                                                      w.chunk_len, w.prefix_len, w.num_pages, 0),
                        dtype=torch.uint8, device=dev)
    fp8_ms = []
    for i in range(args.warmup + 24):
        s_ = sets[i % len(sets)]
        t_ = timed_launch(stream, lambda: bsc.chunk_attention_fp8(
            s_["Q"], K8, V8, sK8, sV8, s_["pt"], s_["tables"], s_["counts"], w.prefix_len,
            err_flag=err, out=s_["O"], lse=s_["LSE"], workspace=ws_f8))
        if i >= args.warmup:
            fp8_ms.append(t_)
    bsc.check(err)
    fp8_res = {"ms": statistics.mean(fp8_ms),
               "tflops": mean_flops / (statistics.mean(fp8_ms) * 1e-3) / 1e12,
               "kv_cache_bytes": 2 * K8.numel(), "bf16_kv_cache_bytes": 4 * K8.numel(),
               "role": "memory-capacity option: half the KV cache bytes, not a speed-up",
               "vs_bf16_time": statistics.mean(fp8_ms) / mean_attn,
               "why_slower": "the MMAs need f16 operands (an 8-bit MMA would need Q and P in "
                             "8 bits, ~2^-4 score error); two warps widen each stage's E4M3 "
                             "bytes to f16 in shared memory, which doubles the kernel's "
                             "instructions and runs on the two-tile kernel",
               "note": "ca_chunk_attention_fp8 incl. the Q cast and scale gather; one page "
                       "buffer (not rotated)"}
    del K8, V8

    # ---- a batch of sequences with unaligned lengths (one varlen launch)
    varlen_res = run_varlen(bsc, dev, stream)
    varlen_short = {
        "auto": run_varlen(bsc, dev, stream, VARLEN_SHORT, n_splits=0,
                           note="ca_chunk_attention_varlen, 4 short chunks over long prefixes, "
                                "automatic plan"),
        "one_cta_per_unit": run_varlen(bsc, dev, stream, VARLEN_SHORT, n_splits=1,
                                       note="the same batch, n_splits = 1"),
    }

    # ---- the full chunked-prefill sweep (32 x 4096 tokens), one pass
    sweep_res = run_sweep(bsc, dev, stream)

    # ---- the 64K density / correlation sweep (26 cells)
    density_res = run_density_sweep(bsc, dev, stream)

    # ---- end to end through the public API with pinned host buffers
    chunk_blocks = list(range(w.nPblk, w.nKblk))
    # masks travel bit-packed (one bit per block, 8x fewer bytes than uint8)
    h_bits = torch.from_numpy(wl.pack_mask_bits(wl.mask_for(w, seed=0)).view(np.int32)).pin_memory()
    h_q = x["Q"].pin_memory()
    h_pt = x["page_table"].pin_memory()
    pt_np = x["page_table"].numpy()
    chunk_pages = torch.from_numpy(pt_np[chunk_blocks]).long()

    def chunk_rows(pages):  # the chunk's own keys (values) as [L, Hkv, d] rows
        return (pages[chunk_pages].permute(0, 2, 1, 3)
                .reshape(w.chunk_len, w.Hkv, w.head_dim).contiguous().pin_memory())

    h_kn, h_vn = chunk_rows(x["K_pages"]), chunk_rows(x["V_pages"])
    d_kn2 = [torch.empty_like(h_kn, device=dev) for _ in range(2)]
    d_vn2 = [torch.empty_like(h_vn, device=dev) for _ in range(2)]
    d_kn, d_vn = d_kn2[0], d_vn2[0]
    h_o2 = [torch.empty(w.chunk_len, w.Hq, w.head_dim, dtype=torch.bfloat16).pin_memory()
            for _ in range(2)]
    h_l2 = [torch.empty(w.Hq, w.chunk_len, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = (h_bits.numel() * 4 + h_q.numel() * 2 + h_pt.numel() * 4 + h_kn.numel() * 2 * 2)
    d2h = h_o2[0].numel() * 2 + h_l2[0].numel() * 4
    # Serving-style pipeline: step i's host->device copies (stream 1) overlap
    # step i-1's append + build + attention (stream 2) and step i-2's
    # device->host read (stream 3); every step's copies are in the timed span.
    s_h2d, s_comp, s_d2h = (torch.cuda.Stream(device=dev) for _ in range(3))

    def e2e_steps(n):
        comp, outd = [], []
        for i in range(n):
            s_ = sets[i % len(sets)]
            kb = i % 2
            with torch.cuda.stream(s_h2d):
                if i >= len(sets):
                    s_h2d.wait_event(outd[i - len(sets)])  # the set's previous step is read out
                if i >= 2:
                    s_h2d.wait_event(comp[i - 2])          # its chunk-row buffer is free
                s_["bits"].copy_(h_bits, non_blocking=True)
                s_["Q"].copy_(h_q, non_blocking=True)
                s_["pt"].copy_(h_pt, non_blocking=True)
                d_kn2[kb].copy_(h_kn, non_blocking=True)
                d_vn2[kb].copy_(h_vn, non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_h2d)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in)
                bsc.append_kv(d_kn2[kb], d_vn2[kb], s_["K"], s_["V"], s_["pt"], w.prefix_len,
                              err_flag=err)
                bsc.build_tables_bits(s_["bits"].unsqueeze(0), w.Hkv, w.nKblk, s_["tables"],
                                      s_["counts"])
                bsc.chunk_attention(s_["Q"], s_["K"], s_["V"], s_["pt"], s_["tables"],
                                    s_["counts"], w.prefix_len, err_flag=err, out=s_["O"],
                                    lse=s_["LSE"], workspace=ws)
                ev_c = torch.cuda.Event()
                ev_c.record(s_comp)
                comp.append(ev_c)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_c)
                h_o2[kb].copy_(s_["O"], non_blocking=True)
                h_l2[kb].copy_(s_["LSE"], non_blocking=True)
                ev_o = torch.cuda.Event()
                ev_o.record(s_d2h)
                outd.append(ev_o)

    e2e_steps(args.warmup)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_h2d)
    e2e_steps(args.steps)
    b.record(s_d2h)
    torch.cuda.synchronize()
    bsc.check(err)
    e2e_ms = [a.elapsed_time(b) / args.steps]
    # ---- the KV append kernel alone (chunk rows already resident)
    ta = []
    for r in range(12):
        s = sets[r % len(sets)]
        t_ = timed_launch(stream, lambda: bsc.append_kv(d_kn, d_vn, s["K"], s["V"], s["pt"],
                                                        w.prefix_len, err_flag=err))
        if r >= 4:
            ta.append(t_)
    bsc.check(err)
    append_bytes = 2 * 2 * d_kn.numel() * d_kn.element_size()   # K and V, read once + written once
    append_res = {"us": statistics.mean(ta) * 1e3,
                  "GB/s": append_bytes / (statistics.mean(ta) * 1e-3) / 1e9,
                  "bytes_per_launch": append_bytes}
    e2e_flops = bsc.selected_flops(sets[0]["tables"].cpu().numpy(),
                                   sets[0]["counts"].cpu().numpy(), w.Hq, w.nPblk, w.nQblk,
                                   w.block, w.head_dim)
    e2e_mean = max_over_ranks([statistics.mean(e2e_ms)], pg, dev)[0]
    e2e_value = world * e2e_flops / (e2e_mean * 1e-3) / 1e12

    if rank == 0:
        peak = peaks.get("bf16_tflops", FALLBACK["bf16_tflops"])
        peak_sus = peaks.get("bf16_tflops_sustained", FALLBACK["bf16_tflops_sustained"])
        hbm = peaks.get("hbm_gbs", FALLBACK["hbm_gbs"])
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) Q/K/V, vertical-slash masks)",
            "config": {"workload": WORKLOAD, "parallelism": f"replicas x{world}",
                       "l2": f"{len(sets)} rotating input sets (distinct page buffers and masks)",
                       "selected_gflop_per_step": mean_flops / 1e9,
                       "table_density": float(np.mean([
                           s["counts"].float().mean().item() / w.nKblk for s in sets]))},
            "attention_ms": mean_attn, "attention_tflops": attn_tflops,
            "table_build_us": statistics.mean(build_ms) * 1e3,
            "table_build_single_gbs": single_bytes / (statistics.mean(build_ms) * 1e-3) / 1e9,
            "dense_ms": dense_ms_mean, "dense_tflops": dense_flops / (dense_ms_mean * 1e-3) / 1e12,
            "speedup_vs_dense": dense_ms_mean / mean_attn,
            "table_build_bits": bits_res,
            "sweep_131k": sweep_res,
            "density_sweep_64k": density_res,
            "fused_step": fused_res,
            "fp8_kv": fp8_res,
            "varlen_batch": varlen_res,
            "varlen_short_batch": varlen_short | {
                "vs_single_sequence": varlen_short["auto"]["tflops"] / attn_tflops,
                "vs_single_sequence_back_to_back":
                    varlen_short["auto"]["back_to_back_tflops"] / attn_tflops},
            "kv_append": append_res,
            "table_build_batched": {"masks_per_launch": nb, "us": statistics.mean(bt) * 1e3,
                                    "GB/s": build_gbs, "frac_of_measured_hbm": build_gbs / hbm,
                                    "frac_of_8TBs_nominal": build_gbs / 8000.0,
                                    "back_to_back_us": b2b_us,
                                    "back_to_back_frac_of_measured_hbm":
                                        bbytes / (b2b_us * 1e-6) / 1e9 / hbm,
                                    "empty_launch_floor_us": floor_us,
                                    "saturation": build_sat},
            "roofline": {"bound": "tensor", "kernel": "chunk_attn_pair_kernel",
                         "achieved": attn_tflops, "peak": peak, "unit": "TFLOP/s",
                         "frac": attn_tflops / peak, "peak_source": f"{peak_src} bf16 burst",
                         "frac_of_sustained": attn_tflops / peak_sus,
                         "per_launch": "selected FLOPs of one 2048-token chunk (32 heads)",
                         "traffic": load_traffic(),
                         "traffic_unit": "bytes per launch (ncu, cold L2)"},
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h), "ms_per_step": e2e_mean,
                    "pipeline": "H2D of step i, compute of step i-1, D2H of step i-2 on "
                                "three streams; K steps timed as one span",
                    "inputs": "bit-packed masks, Q, the chunk's K/V rows and the page table "
                              "in; O and LSE out; append + bit-packed table build + attention"},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk,
        }
        if world == 1 and not args.no_cpu_baseline:
            cb_ = cpu_oracle_sample(w, x, wl.mask_for(w, seed=0))
            cb_.pop("seconds", None)
            line["cpu_baseline"] = cb_
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
