"""Benchmark of the InfLLM v2 block-sparse attention path on B200.

A step is one whole prefill of a 128K-token sequence (compress keys -> select blocks ->
sparse attention) on seeded synthetic inputs already resident in HBM.  The line also
reports one decode step (select -> sparse attention over a filled cache) of 32 ragged
sequences of 64K-128K tokens, the same prefill end to end through host buffers, the
per-kernel rooflines and the CPU oracle timed on a bounded sample.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torch.distributed.run) every rank runs its own independent
sequence: weak scaling, no collective on the data path.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from trainable_block_sparse_compress_b200 import build as lib_build  # noqa: E402
from trainable_block_sparse_compress_b200 import dist  # noqa: E402
from trainable_block_sparse_compress_b200 import ops  # noqa: E402
from trainable_block_sparse_compress_b200.synthetic import WORKLOADS, as_u16, make_inputs  # noqa: E402

METRIC = "128K prefill tokens/s + decode µs/step on 1 B200; % of TC/HBM roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


# ------------------------------------------------------------------ helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# CUDA sources each kernel is built from (its own header, the headers it includes, and the
# host file that sets its launch shape)
KERNEL_SOURCES = {
    "compress_kernel": ["compress.cuh", "common.cuh", "infllmv2.cu"],
    "select_prefill_tc_kernel": ["select_prefill_tc.cuh", "select_prefill.cuh", "topk.cuh", "tcgen05.cuh",
                                 "common.cuh", "infllmv2.cu"],
    "select_prefill_kernel": ["select_prefill.cuh", "topk.cuh", "common.cuh", "infllmv2.cu"],
    "attn_tc_kernel": ["attn_tc.cuh", "attn.cuh", "tcgen05.cuh", "common.cuh", "infllmv2.cu"],
    "attn_kernel": ["attn.cuh", "common.cuh", "infllmv2.cu"],
    "select_decode_kernel": ["select_decode.cuh", "select_prefill.cuh", "topk.cuh", "common.cuh", "infllmv2.cu"],
    "attn_decode_cluster_kernel": ["attn_dec.cuh", "attn.cuh", "common.cuh", "infllmv2.cu"],
    "decode_step_kernel": ["decode_step.cuh", "select_decode.cuh", "attn_dec.cuh", "select_prefill.cuh", "topk.cuh",
                           "attn.cuh", "common.cuh", "infllmv2.cu"],
    "bwd_dkdv_tc_kernel": ["attn_bwd_tc.cuh", "attn_bwd.cuh", "attn.cuh", "tcgen05.cuh", "common.cuh", "infllmv2.cu"],
}


def source_sha(kernel: str) -> str:
    """Hash of the CUDA sources `kernel` is built from: a DRAM-traffic figure counts only
    when it was taken on exactly these sources."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "trainable_block_sparse_compress_b200", "csrc")
    for name in sorted(KERNEL_SOURCES[kernel]):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def dram_traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch from the committed ncu summary, if it was
    taken on the kernel's current sources and the same workload (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path) or kernel not in KERNEL_SOURCES:
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get("kernels", {}).get(kernel, {})
    if e.get("source_sha") != source_sha(kernel) or e.get("workload") != workload:
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.dev)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        loaded = [s for s in sm if s > 0.5 * (mx or max(sm))] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def prefill_flops(p: ops.Params, L: int):
    """Algorithmic FLOPs of one prefill: (selection, attention on selected blocks)."""
    t = np.arange(L, dtype=np.int64)
    nk_vis = np.where(t >= 31, (t - 31) // 16 + 1, 0)
    sel = 2 * 2 * p.head_dim * p.num_q_heads * p.batch * int(nk_vis.sum())  # 2 passes x 2 flop/MAC
    cur = t // 64
    nsel = np.minimum(p.topk, cur + 1)
    keys = 64 * (nsel - 1) + (t - 64 * cur + 1)
    attn = 4 * p.head_dim * p.num_q_heads * p.batch * int(keys.sum())  # QK^T and PV
    gather = 2 * 2 * p.head_dim * 64 * p.num_kv_heads * p.batch * int(nsel.sum())  # K+V bytes
    return sel, attn, gather


def decode_bytes(p: ops.Params, lens: np.ndarray):
    """Algorithmic bytes of one decode step: (selection: Kc + Q, attention: K/V keys + Q + O)."""
    lens = lens.astype(np.int64)
    nk = np.where(lens >= 32, (lens - 32) // 16 + 1, 0)
    qbytes = p.batch * p.num_q_heads * p.head_dim * 2
    sel = int(nk.sum()) * p.num_kv_heads * p.head_dim * 2 + qbytes
    cur = (lens - 1) // 64
    nsel = np.minimum(p.topk, cur + 1)
    keys = 64 * (nsel - 1) + (lens - 1 - 64 * cur + 1)
    attn = int(keys.sum()) * p.num_kv_heads * p.head_dim * 2 * 2 + 2 * qbytes
    return sel, attn


# ----------------------------------------------------------------- our path

def run_ours(args, rank, world, device):
    pk, peak_src = peaks()
    wl = WORKLOADS[args.workload]
    p = ops.Params.from_workload(wl)
    L = wl.seq_len
    x = make_inputs(wl, seed=dist.rank_seed(args.seed, rank))
    q, k, v = x.q.to(device), x.k.to(device), x.v.to(device)
    nk = ops.num_kernels(p, L)
    kc = torch.empty((p.batch, p.num_kv_heads, nk, p.head_dim), dtype=torch.bfloat16, device=device)
    idx = torch.empty((p.batch, p.num_kv_heads, L, p.topk), dtype=torch.int32, device=device)
    o = torch.empty_like(q)
    lse = torch.empty((p.batch, p.num_q_heads, L), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def step():
        ops.compress_keys(p, k, out=kc)
        ops.select_blocks_prefill(p, q, kc, out=idx)
        ops.sparse_attn_prefill(p, q, k, v, idx, out=o, lse=lse)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # per-kernel device times (events on the launching stream), separate pass
    names = ["compress", "select", "attn"]
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for s in range(args.steps):
        ev[s][0].record(stream)
        ops.compress_keys(p, k, out=kc)
        ev[s][1].record(stream)
        ops.select_blocks_prefill(p, q, kc, out=idx)
        ev[s][2].record(stream)
        ops.sparse_attn_prefill(p, q, k, v, idx, out=o, lse=lse)
        ev[s][3].record(stream)
    torch.cuda.synchronize()
    kern_ms = {n: statistics.mean(ev[s][i].elapsed_time(ev[s][i + 1]) for s in range(args.steps))
               for i, n in enumerate(names)}

    # the timed region: exactly K steps, barrier + synchronize on both sides
    dist.barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
    dist.barrier(world)
    ms = dist.max_over_ranks(t0.elapsed_time(t1), world, device)
    ms_per_step = ms / args.steps
    tokens_per_step = p.batch * L
    value = dist.weak_scaling_rate(world, tokens_per_step, args.steps, ms / 1e3)

    sel_flops, attn_flops, gather_bytes = prefill_flops(p, L)
    comp_bytes = p.batch * p.num_kv_heads * (L + nk) * p.head_dim * 2
    # per-kernel event timings: the burst peak is the denominator (cuBLAS timed alone);
    # the sustained figure (a seconds-long loop under the power cap) is given beside it
    tc_peak = pk["bf16_tflops"]
    kern = {
        "compress": {"ms": kern_ms["compress"], "bound": "hbm", "algorithmic_bytes": comp_bytes,
                     "achieved": comp_bytes / kern_ms["compress"] / 1e6, "unit": "GB/s", "peak": pk["hbm_gbs"]},
        "select": {"ms": kern_ms["select"], "bound": "tensor", "algorithmic_flops": sel_flops,
                   "achieved": sel_flops / kern_ms["select"] / 1e9, "unit": "TFLOP/s", "peak": tc_peak},
        "attn": {"ms": kern_ms["attn"], "bound": "tensor", "algorithmic_flops": attn_flops,
                 "achieved": attn_flops / kern_ms["attn"] / 1e9, "unit": "TFLOP/s", "peak": tc_peak,
                 "gather_bytes": gather_bytes, "gather_GBps": gather_bytes / kern_ms["attn"] / 1e6},
    }
    for kv in kern.values():
        kv["frac"] = kv["achieved"] / kv["peak"]
        if kv["bound"] == "tensor":
            kv["frac_of_sustained"] = kv["achieved"] / pk["bf16_tflops_sustained"]
    top = max(kern, key=lambda n: kern[n]["ms"])
    tc = p.num_q_heads // p.num_kv_heads == 16  # the tensor-core (tcgen05) prefill kernels serve G = 16
    names = {"compress": "compress_kernel",
             "select": "select_prefill_tc_kernel" if tc else "select_prefill_kernel",
             "attn": "attn_tc_kernel" if tc else "attn_kernel"}
    for n, kv in kern.items():
        kv["kernel"] = names[n]
        kv["traffic"] = dram_traffic(names[n], args.workload)
    kname = names[top]
    roof = {"kernel": kname, "bound": kern[top]["bound"], "achieved": kern[top]["achieved"],
            "peak": kern[top]["peak"], "unit": kern[top]["unit"], "frac": kern[top]["frac"],
            "traffic": kern[top]["traffic"],
            "peak_source": f"{peak_src} ({'bf16_tflops, burst' if kern[top]['bound'] == 'tensor' else 'hbm_gbs'})"}

    result = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "batch": p.batch, "seq_len": L, "num_q_heads": p.num_q_heads,
                   "num_kv_heads": p.num_kv_heads, "head_dim": p.head_dim, "block": p.block_size,
                   "kernel": p.kernel_size, "stride": p.kernel_stride, "topk": p.topk, "n_init": p.n_init,
                   "n_local": p.n_local, "seed": args.seed, "parallelism": f"dp{world} (independent sequences)",
                   "l2": "inputs larger than L2: each step reads Q (1 GiB) and writes O (1 GiB)"},
        "roofline": roof,
        "kernels": kern,
        "gpu_launches": 3 * args.steps,
        "clocks": clk.summary(),
    }
    del kc, idx, o, lse

    if rank == 0 and not args.no_e2e:
        result["e2e"] = run_e2e(args, p, x, device)
    del q, k, v
    torch.cuda.empty_cache()
    if not args.no_decode:
        result["decode"] = run_decode(args, args.decode_workload, rank, world, device, pk, peak_src)
        if args.decode_workload_2:
            result["decode_2"] = run_decode(args, args.decode_workload_2, rank, world, device, pk, peak_src)
    if rank == 0 and not args.no_extras:
        try:
            result["extras"] = run_extras(args, device, pk, peak_src)
        except Exception as e:  # the extra timings never cost the main line
            result["extras"] = {"error": f"{type(e).__name__}: {e}"}
            torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(args, wl, x)
    return result


def run_e2e(args, p, x, device):
    """Same prefill through the public calls with host buffers: every step copies its
    pinned host Q, K, V in and its O back out, inside the timed region.  Steps are
    pipelined over two device buffer sets: step i+1's inputs travel on a copy stream and
    step i-1's output on another while step i computes, as a serving loop would run."""
    qh, kh, vh = x.q.pin_memory(), x.k.pin_memory(), x.v.pin_memory()
    L = x.q.shape[1]
    nb = 2
    qd = [torch.empty_like(qh, device=device) for _ in range(nb)]
    kd = [torch.empty_like(kh, device=device) for _ in range(nb)]
    vd = [torch.empty_like(vh, device=device) for _ in range(nb)]
    od = [torch.empty_like(qh, device=device) for _ in range(nb)]
    oh = [torch.empty_like(qh).pin_memory() for _ in range(nb)]
    kc = [torch.empty((p.batch, p.num_kv_heads, ops.num_kernels(p, L), p.head_dim), dtype=torch.bfloat16,
                      device=device) for _ in range(nb)]
    idx = [torch.empty((p.batch, p.num_kv_heads, L, p.topk), dtype=torch.int32, device=device) for _ in range(nb)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(device) for _ in range(3))
    done_cmp = [None] * nb  # compute of the last step that used buffer set b
    done_out = [None] * nb  # read-back of the last step that used buffer set b

    def step(i):
        b = i % nb
        with torch.cuda.stream(s_in):
            if done_cmp[b] is not None:
                s_in.wait_event(done_cmp[b])  # that step no longer reads these inputs
            qd[b].copy_(qh, non_blocking=True)
            kd[b].copy_(kh, non_blocking=True)
            vd[b].copy_(vh, non_blocking=True)
            e_in = torch.cuda.Event()
            e_in.record(s_in)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(e_in)
            if done_out[b] is not None:
                s_cmp.wait_event(done_out[b])  # its output was read back
            ops.compress_keys(p, kd[b], out=kc[b])
            ops.select_blocks_prefill(p, qd[b], kc[b], out=idx[b])
            ops.sparse_attn_prefill(p, qd[b], kd[b], vd[b], idx[b], out=od[b], want_lse=False)
            done_cmp[b] = torch.cuda.Event()
            done_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done_cmp[b])
            oh[b].copy_(od[b], non_blocking=True)
            done_out[b] = torch.cuda.Event()
            done_out[b].record(s_out)

    n = max(4, min(args.steps, 8))
    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    for i in range(n):
        step(i)
    t1.record(s_out)  # after the last read-back, which waits for everything before it
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / n
    h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
    d2h = oh[0].numel() * oh[0].element_size()
    return {"value": p.batch * L / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n,
            "overlap": "copies of neighbouring steps overlap the compute (two buffer sets, three streams)"}


def run_decode(args, workload, rank, world, device, pk, peak_src):
    """One decode step over filled caches, in one launch: the new token appended (its K/V
    rows and the semantic kernel it completes), block selection, attention.  L2 flushed
    before every step (outside the timed events).  Inputs: the same seed as the parity
    tests; the appended token is each sequence's last one (rewritten in place, so every
    step sees the same cache).  The step without the append and the two separate calls are
    timed too, for the split."""
    wl = WORKLOADS[workload]
    p = ops.Params.from_workload(wl)
    x = make_inputs(wl, seed=dist.rank_seed(args.seed, rank))
    Lmax = wl.seq_len
    q, k, v, lens = x.q.to(device), x.k.to(device), x.v.to(device), x.lens.to(device)
    kc = ops.compress_keys(p, k, lens=lens)  # cache maintenance, not timed
    idx = torch.empty((p.batch, p.num_kv_heads, 1, p.topk), dtype=torch.int32, device=device)
    o = torch.empty_like(q)
    lse = torch.empty((p.batch, p.num_q_heads), dtype=torch.float32, device=device)
    ws_s = torch.empty(ops.workspace_size(p, 2, Lmax), dtype=torch.uint8, device=device)
    ws_a = torch.empty(ops.workspace_size(p, 4, Lmax), dtype=torch.uint8, device=device)
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    last = (lens.long() - 1).clamp(min=0)
    bidx = torch.arange(p.batch, device=device)
    k_new = k[bidx, :, last].contiguous()
    v_new = v[bidx, :, last].contiguous()
    lens_prev = lens - 1  # cached tokens before the step
    lens_out = torch.empty_like(lens)

    def step():
        ops.decode_step(p, q, k, v, kc, lens_prev, k_new=k_new, v_new=v_new, lens_out=lens_out, block_idx=idx,
                        out=o, lse=lse)

    def step_no_append():
        ops.decode_step(p, q, k, v, kc, lens, block_idx=idx, out=o, lse=lse)

    for _ in range(max(3, args.warmup)):
        step()
        step_no_append()
    n = max(args.steps, 20)

    def flush_l2():
        flush.zero_()  # evict the caches' lines from L2 ...
        flush.view(torch.int32).sum()  # ... and leave it clean, so no write-back lands in the step

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    for s in range(n):
        flush_l2()
        ev[s][0].record(stream)
        step()
        ev[s][1].record(stream)
    torch.cuda.synchronize()
    step_us = [ev[s][0].elapsed_time(ev[s][1]) * 1e3 for s in range(n)]
    evn = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    for s in range(n):
        flush_l2()
        evn[s][0].record(stream)
        step_no_append()
        evn[s][1].record(stream)
    torch.cuda.synchronize()
    noapp_us = statistics.median(evn[s][0].elapsed_time(evn[s][1]) * 1e3 for s in range(n))
    # the two separate calls: the pair (the attention launch overlaps the end of the
    # selection), then each kernel alone (an event between them keeps the attention from
    # starting early)
    evp = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    evk = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
    for s in range(n):
        flush_l2()
        evp[s][0].record(stream)
        ops.select_blocks_decode(p, q, kc, lens, Lmax, out=idx, ws=ws_s)
        ops.sparse_attn_decode(p, q, k, v, lens, idx, out=o, lse=lse, ws=ws_a)
        evp[s][1].record(stream)
        flush_l2()
        evk[s][0].record(stream)
        ops.select_blocks_decode(p, q, kc, lens, Lmax, out=idx, ws=ws_s)
        evk[s][1].record(stream)
        ops.sparse_attn_decode(p, q, k, v, lens, idx, out=o, lse=lse, ws=ws_a)
        evk[s][2].record(stream)
    torch.cuda.synchronize()
    pair_us = [evp[s][0].elapsed_time(evp[s][1]) * 1e3 for s in range(n)]
    sel_us = [evk[s][0].elapsed_time(evk[s][1]) * 1e3 for s in range(n)]
    att_us = [evk[s][1].elapsed_time(evk[s][2]) * 1e3 for s in range(n)]
    us = statistics.median(step_us)
    us = dist.max_over_ranks(us, world, device)
    # the standalone append kernel (infllmv2_append_kv), for comparison: re-append each
    # sequence's last token, which rewrites the same rows and kernel and leaves lens as it was
    lens_w = torch.empty_like(lens)
    eva = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
    for s in range(n):
        lens_w.copy_(lens - 1)
        flush_l2()
        eva[s][0].record(stream)
        ops.append_kv(p, k_new, v_new, k, v, lens_w, kc)
        eva[s][1].record(stream)
    torch.cuda.synchronize()
    app_us = statistics.median(eva[s][0].elapsed_time(eva[s][1]) * 1e3 for s in range(n))
    app_bytes = p.batch * p.num_kv_heads * 2 * 2 * p.head_dim  # the new K and V rows read and written
    sel_b, att_b = decode_bytes(p, x.lens.numpy())
    assert torch.equal(lens_out, lens)
    step_b = sel_b + att_b + app_bytes  # Kc, the selected K/V blocks, the appended rows
    att_kernel = "attn_decode_cluster_kernel" if ws_a.numel() == 0 else "attn_kernel + attn_merge_kernel"
    hbm = pk["hbm_gbs"]
    sel_med, att_med = statistics.median(sel_us), statistics.median(att_us)
    tr_f = dram_traffic("decode_step_kernel", workload)
    tr_s = dram_traffic("select_decode_kernel", workload)
    tr_a = dram_traffic(att_kernel, workload)
    return {
        "workload": workload, "value": us, "unit": "us/step", "higher_is_better": False,
        "batch": p.batch, "mean_len": float(x.lens.float().mean()), "steps": n,
        "l2": "flushed before every step (write then read a 2x L2 buffer, outside the timed events)",
        "roofline": {"bound": "hbm", "achieved": step_b / us / 1e3, "peak": hbm, "unit": "GB/s",
                     "frac": step_b / us / 1e3 / hbm, "algorithmic_bytes": step_b,
                     "traffic": tr_f, "peak_source": f"{peak_src} (hbm_gbs)"},
        "kernels": {
            "step": {"kernel": "decode_step_kernel", "us": us, "algorithmic_bytes": step_b,
                     "achieved_GBps": step_b / us / 1e3, "traffic": tr_f},
        },
        "gpu_launches_per_step": 1,
        "step": "append of the new token + block selection + sparse attention (infllmv2_decode_step with k_new)",
        "step_without_append_us": noapp_us,
        "separate_calls": {
            "note": "infllmv2_select_blocks(DECODE) then infllmv2_sparse_attn_decode on the same inputs",
            "pair_us": statistics.median(pair_us),
            "select": {"kernel": "select_decode_kernel", "us": sel_med, "algorithmic_bytes": sel_b,
                       "achieved_GBps": sel_b / sel_med / 1e3, "traffic": tr_s},
            "attn": {"kernel": att_kernel, "us": att_med, "algorithmic_bytes": att_b,
                     "achieved_GBps": att_b / att_med / 1e3, "traffic": tr_a},
        },
        "append": {"kernel": "append_kv_kernel", "us": app_us, "bytes_per_step": app_bytes,
                   "note": "the standalone cache-maintenance call, timed apart; the step above appends itself"},
    }


# ------------------------------------------------- chunks, variants, backward

def _time_ms(fn, reps, stream):
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    fn()
    torch.cuda.synchronize()
    ev[0].record(stream)
    for _ in range(reps):
        fn()
    ev[1].record(stream)
    torch.cuda.synchronize()
    return ev[0].elapsed_time(ev[1]) / reps


def run_extras(args, device, pk, peak_src):
    """The other calls of the library, each timed with CUDA events on its own (rank 0):
    a prefill chunk against a 128K cache, the selection variants at 128K, and the
    backward pass at 32K.  Inputs are the seeded workloads of the parity tests."""
    stream = torch.cuda.current_stream()
    reps = max(3, min(args.steps, 10))
    tc_peak = pk["bf16_tflops"]
    out = {"peak_source": f"{peak_src} (bf16_tflops, burst)"}

    wl = WORKLOADS["prefill_128k"]
    p = ops.Params.from_workload(wl)
    L = wl.seq_len
    x = make_inputs(wl, seed=args.seed)
    q, k, v = x.q.to(device), x.k.to(device), x.v.to(device)
    del x
    kc = ops.compress_keys(p, k)

    # a chunk of the last m queries against the whole cache (positions L-m .. L-1)
    m = 8192
    qc = q[:, L - m:].contiguous()
    idx_c = torch.empty((p.batch, p.num_kv_heads, m, p.topk), dtype=torch.int32, device=device)
    o_c = torch.empty_like(qc)

    def chunk_step():
        ops.select_blocks_chunk(p, qc, kc, L, out=idx_c)
        ops.sparse_attn_chunk(p, qc, k, v, idx_c, out=o_c, want_lse=False)
    ms_chunk = _time_ms(chunk_step, reps, stream)
    ms_attn_c = _time_ms(lambda: ops.sparse_attn_chunk(p, qc, k, v, idx_c, out=o_c, want_lse=False), reps, stream)
    t = np.arange(L - m, L, dtype=np.int64)
    cur = t // 64
    keys = 64 * (np.minimum(p.topk, cur + 1) - 1) + (t - 64 * cur + 1)
    fl = 4 * p.head_dim * p.num_q_heads * int(keys.sum())
    out["chunk"] = {"workload": f"prefill_128k cache, chunk of the last {m} queries", "ms": ms_chunk,
                    "tokens_per_s": m / (ms_chunk / 1e3), "attn_ms": ms_attn_c,
                    "attn_tflops": fl / ms_attn_c / 1e9, "attn_frac": fl / ms_attn_c / 1e9 / tc_peak}
    del qc, idx_c, o_c

    # selection variants over the whole 128K prefill
    idx = torch.empty((p.batch, p.num_kv_heads, L, p.topk), dtype=torch.int32, device=device)
    sel_flops, _, _ = prefill_flops(p, L)
    var = {}
    for sm, pm in ((0, 0), (1, 0), (0, 1), (1, 1)):
        pv = dataclasses.replace(p, score_mode=sm, pool_mode=pm)
        ms_sel = _time_ms(lambda: ops.select_blocks_prefill(pv, q, kc, out=idx), reps, stream)
        flops = sel_flops if sm == 0 else sel_flops // 2  # logit-sum: one pass over the kernels
        var[f"score{sm}_pool{pm}"] = {"ms": ms_sel, "tflops": flops / ms_sel / 1e9,
                                      "frac": flops / ms_sel / 1e9 / tc_peak}
    out["select_variants_128k"] = var
    del q, k, v, kc, idx
    torch.cuda.empty_cache()

    # backward at 32K: the forward once, then the backward timed alone
    wl = WORKLOADS["prefill_32k"]
    p = ops.Params.from_workload(wl)
    L = wl.seq_len
    x = make_inputs(wl, seed=args.seed)
    q, k, v = x.q.to(device), x.k.to(device), x.v.to(device)
    g = torch.Generator().manual_seed(args.seed + 7)
    d_o = torch.randn(x.q.shape, generator=g).to(torch.bfloat16).to(device)
    del x
    o, lse, idx, kc = ops.prefill(p, q, k, v)
    ws = torch.empty(ops.workspace_size(p, 5, L), dtype=torch.uint8, device=device)
    ms_bwd = _time_ms(lambda: ops.sparse_attn_backward(p, q, k, v, o, lse, d_o, idx, ws=ws), reps, stream)
    _, attn_flops, _ = prefill_flops(p, L)
    bwd_flops = attn_flops * 5 // 2  # recompute S, dP, dV, dK, dQ: 5 products of the forward's 2
    out["backward_32k"] = {"workload": "prefill_32k (B=1, L=32768, 32/2 heads, top-96)", "ms": ms_bwd,
                           "tflops": bwd_flops / ms_bwd / 1e9, "frac": bwd_flops / ms_bwd / 1e9 / tc_peak,
                           "algorithmic_flops": bwd_flops,
                           "dkdv_kernel_traffic": dram_traffic("bwd_dkdv_tc_kernel", "prefill_32k backward"),
                           "note": "kernels run 7 products (S and dP are recomputed in both passes): "
                                   "dq on m16n8k16 MMAs, dK / dV on tcgen05 (TMEM accumulators)"}
    del q, k, v, d_o, o, lse, idx, kc, ws
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------- CPU oracle

def oracle_rows_time(wl, x, rows):
    import oracle
    op = oracle.Params(wl.batch, wl.num_q_heads, wl.num_kv_heads, wl.head_dim, wl.block_size, wl.kernel_size,
                       wl.kernel_stride, wl.topk, wl.n_init, wl.n_local)
    q, k, v = as_u16(x.q), as_u16(x.k), as_u16(x.v)
    t0 = time.perf_counter()
    kc = oracle.compress(op, k)
    idx = oracle.select(op, q, kc, rows=rows)
    oracle.attn(op, q, k, v, idx, rows=rows)
    return time.perf_counter() - t0


def sample_rows(L, n):
    # evenly strided over the sequence, so the mean cost per row matches the full prefill
    return np.unique(np.linspace(0, L - 1, n).astype(np.int64))


def cpu_baseline(args, wl, x, target_s=12.0):
    import oracle
    L = wl.seq_len
    rows = sample_rows(L, 64)
    dt = oracle_rows_time(wl, x, rows)
    n = int(min(L, max(64, len(rows) * target_s / max(dt, 1e-3))))
    rows = sample_rows(L, n)
    dt = oracle_rows_time(wl, x, rows)
    return {"value": wl.batch * len(rows) / dt, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle", "seconds": dt,
            "sample": f"{len(rows)} query rows evenly strided over the {L}-token prefill (all heads), "
                      f"plus key compression of the whole sequence; tokens/s = rows / time"}


def run_reference(args):
    """The CPU oracle as it stands, on bounded samples of the same workload."""
    import oracle
    oracle.build()
    wl = WORKLOADS[args.workload]
    x = make_inputs(wl, seed=args.seed)
    L = wl.seq_len
    rows = sample_rows(L, args.reference_rows)
    for _ in range(args.warmup):
        oracle_rows_time(wl, x, rows[:8])
    times = [oracle_rows_time(wl, x, rows) for _ in range(args.steps)]
    dt = sum(times)
    value = wl.batch * len(rows) * args.steps / dt
    cores = oracle.num_threads()
    sample = (f"{len(rows)} query rows evenly strided over the {L}-token prefill per step (all heads), "
              f"plus key compression of the whole sequence")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": args.workload, "batch": wl.batch, "seq_len": L, "num_q_heads": wl.num_q_heads,
                       "num_kv_heads": wl.num_kv_heads, "topk": wl.topk, "seed": args.seed},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def profile_run(name, device, backward=False):
    """The hot path of one workload, twice (a warm-up and one more run), for single-kernel
    profiler captures: prefill (compress, select, attend) or a decode step (compress the
    caches, then the fused step, then the separate selection and attention calls on the
    same inputs); with `backward` (prefill workloads), the forward once and then the
    backward twice, with the upstream gradient of the bench's backward line.  Prints
    nothing."""
    wl = WORKLOADS[name]
    p = ops.Params.from_workload(wl)
    x = make_inputs(wl, seed=0)
    q, k, v = x.q.to(device), x.k.to(device), x.v.to(device)
    if backward:
        assert wl.mode == "prefill", "the backward runs on prefill workloads"
        g = torch.Generator().manual_seed(7)
        d_o = torch.randn(x.q.shape, generator=g).to(torch.bfloat16).to(device)
        o, lse, idx, _ = ops.prefill(p, q, k, v)
        ws = torch.empty(ops.workspace_size(p, 5, wl.seq_len), dtype=torch.uint8, device=device)
        for _ in range(2):
            ops.sparse_attn_backward(p, q, k, v, o, lse, d_o, idx, ws=ws)
        torch.cuda.synchronize()
        assert ops.device_error(clear=True) == 0
        return
    for _ in range(2):
        if wl.mode == "prefill":
            ops.prefill(p, q, k, v)
        else:
            lens = x.lens.to(device)
            kc = ops.compress_keys(p, k, lens=lens)
            ops.decode(p, q, k, v, kc, lens, wl.seq_len)
            idx = ops.select_blocks_decode(p, q, kc, lens, wl.seq_len)
            ops.sparse_attn_decode(p, q, k, v, lens, idx)
    torch.cuda.synchronize()
    assert ops.device_error(clear=True) == 0


# ---------------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_128k")
    ap.add_argument("--decode-workload", default="decode_ragged_128k")
    ap.add_argument("--decode-workload-2", default="decode_32k", help="second decode line ('' for none)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the chunk / variant / backward timings")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--reference-rows", type=int, default=96)
    ap.add_argument("--profile-run", default=None, metavar="WORKLOAD",
                    help="run WORKLOAD's hot path twice and exit (for profiler captures)")
    ap.add_argument("--profile-backward", action="store_true",
                    help="with --profile-run: the forward once, then the backward twice")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.profile_run:
        lib_build.build()
        profile_run(args.profile_run, torch.device("cuda", 0), backward=args.profile_backward)
        return

    ri = dist.rank_info()
    rank, world, local = ri.rank, ri.world, ri.local

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    lib_build.build()
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=device)
    try:
        res = run_ours(args, rank, world, device)
        err = ops.device_error(clear=True)
        res["device_error"] = err
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
