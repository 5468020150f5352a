#!/usr/bin/env python
"""Benchmark of tree-verification attention (LongSpec hybrid tree attention) on B200.

One step = one full verification-attention call (partials kernel + combine kernel) over one
batch of synthetic input of the named workload, inputs resident in HBM. L2 is flushed
(a write of twice the L2 size) before every timed step, outside the timed events.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

N > 1 runs under torchrun: every rank runs an independent problem of the same workload
on its own GPU (replicas, weak scaling, no collective on the data path); the step time
is the max over ranks. Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
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

from tree_verification_attention_longspec_b200.inputs import make_inputs  # noqa: E402
from tree_verification_attention_longspec_b200.workloads import (  # noqa: E402
    HEADLINE, WORKLOADS, algorithmic_bytes, algorithmic_flops)

METRIC = "verify-attn µs/call and KV HBM GB/s (% roofline) at L=64k, T=64, bf16"
UNIT = "us/call"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DOMINANT_KERNEL_SRC = os.path.join(ROOT, "tree_verification_attention_longspec_b200", "csrc")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def workload_figures(inp, cross=False):
    w = inp.workload
    L = inp.prefix_lengths
    total_L = int(L.sum())
    if inp.cu_tree is not None:
        # trees of T_b nodes: 4*d flops per (query row, prefix or tree key) pair of each
        # sequence; bytes as below with N = sum T_b nodes
        Tb = np.diff(inp.cu_tree).astype(np.int64)
        N = int(Tb.sum())
        rows = N * w.num_q_heads
        kv_bytes = 4 * total_L * w.num_kv_heads * w.head_dim
        flops = int(sum(4 * int(t) * w.num_q_heads * w.head_dim * (int(l) + int(t)) for t, l in zip(Tb, L)))
        tree_bytes = 4 * N * w.num_kv_heads * w.head_dim
        step_bytes = kv_bytes + tree_bytes + 4 * rows * w.head_dim + 4 * rows
        return dict(total_L=total_L, step_bytes=step_bytes, step_flops=flops, partials_flops=flops,
                    partials_bytes=kv_bytes + tree_bytes + 2 * rows * w.head_dim, kv_bytes=kv_bytes, rows=rows)
    if cross:
        # prefix-only attention: 4*d flops per (query row, prefix key); bytes: the prefix
        # K/V, the queries, out and lse
        rows = w.batch * w.tree_size * w.num_q_heads
        kv_bytes = 4 * total_L * w.num_kv_heads * w.head_dim
        flops = 4 * w.head_dim * w.tree_size * w.num_q_heads * total_L
        step_bytes = kv_bytes + 4 * rows * w.head_dim + 4 * rows
        return dict(total_L=total_L, step_bytes=step_bytes, step_flops=flops, partials_flops=flops,
                    partials_bytes=kv_bytes + 2 * rows * w.head_dim, kv_bytes=kv_bytes, rows=rows)
    step_bytes = algorithmic_bytes(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.tree_size,
                                   total_L)
    step_flops = algorithmic_flops(w.num_q_heads, w.head_dim, w.tree_size, L)
    # the partials kernel (the dominant one) does every flop of the step: 4*d per (query
    # row, prefix or tree key) pair; its compulsory bytes are the prefix and tree K/V and
    # the queries
    rows = w.batch * w.tree_size * w.num_q_heads
    kv_bytes = 4 * total_L * w.num_kv_heads * w.head_dim
    partials_flops = step_flops
    partials_bytes = kv_bytes + 4 * w.batch * w.tree_size * w.num_kv_heads * w.head_dim + 2 * rows * w.head_dim
    return dict(total_L=total_L, step_bytes=step_bytes, step_flops=step_flops,
                partials_flops=partials_flops, partials_bytes=partials_bytes, kv_bytes=kv_bytes, rows=rows)


def config_of(inp, l2_note):
    w = inp.workload
    L = inp.prefix_lengths
    return {"workload": w.name, "batch": w.batch, "num_q_heads": w.num_q_heads,
            "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "tree_size": w.tree_size,
            "tree": w.tree, "prefix_len": int(L[0]) if len(set(L.tolist())) == 1 else "ragged",
            "total_prefix_len": int(L.sum()), "seed": inp.seed, "l2": l2_note,
            **({"tree_sizes": f"T_b ~ U{{{w.tree_size_range[0]}..{w.tree_size_range[1]}}}, sum {inp.num_nodes}"}
               if w.tree_size_range else {})}


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(values, device=None):
    """Element-wise maximum of `values` over all ranks (the step time of a multi-GPU run
    is that of its slowest rank); the values themselves when running alone."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU through NVML in a thread."""

    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4}

    def __init__(self, device_index, period_s=0.005):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report without clocks
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                util = nv.nvmlDeviceGetUtilizationRates(self.h).gpu
                self.samples.append((mhz, rs, util))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        # Every sample is taken inside the timed region, whose GPU queue never empties
        # (spin, L2 flush and measured kernels back to back). NVML's utilisation is a
        # trailing average that can still read 0 over so short a window: the samples it
        # marks busy are used when there are any, else all of them, and the line says which.
        busy = [s for s in self.samples if s[2] > 0]
        loaded = busy or self.samples
        reasons = set()
        for _, rs, _ in loaded:
            for name, bit in self.REASONS.items():
                if rs & bit:
                    reasons.add(name)
        med = statistics.median([s[0] for s in loaded]) if loaded else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons),
                "samples": len(self.samples), "samples_under_load": len(loaded),
                "load_basis": ("NVML utilisation above 0" if busy else
                               "all samples (each inside the timed region, GPU queue full)")}


# ----------------------------------------------------------------------------- traffic record
def code_lines(text):
    """The source's code: each line cut at a `//` comment outside a string literal,
    trailing blanks removed, empty lines dropped (a comment edit leaves it unchanged)."""
    out = []
    for line in text.splitlines():
        in_str, cut = False, len(line)
        for i, ch in enumerate(line):
            if ch == '"' and (i == 0 or line[i - 1] != "\\"):
                in_str = not in_str
            elif not in_str and line.startswith("//", i):
                cut = i
                break
        code = line[:cut].rstrip()
        if code:
            out.append(code)
    return "\n".join(out)


def kernel_source_hash():
    """Hash of the CUDA sources' code (comments excluded), which the recorded ncu traffic
    must match."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(DOMINANT_KERNEL_SRC)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(DOMINANT_KERNEL_SRC, name), encoding="utf-8") as f:
                h.update(name.encode() + code_lines(f.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name):
    """DRAM bytes per launch of the partials kernel from the committed ncu summary, when it
    was taken on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        r = rec.get(workload_name)
        if r and r.get("source_hash") == kernel_source_hash():
            return r.get("dram_bytes_per_launch")
    except Exception:
        pass
    return None


# ----------------------------------------------------------------------------- oracle timing
def oracle_rows(inp, rows, cores):
    """The fp64 oracle on the given output rows (node n, head h) -> n*H_q + h."""
    import oracle
    if inp.cu_tree is None:
        return oracle.verify_attn_oracle_inputs(inp, rows=rows, nthreads=cores)
    w = inp.workload
    off, cu, Hq = inp.cu_tree, inp.cu_seqlens, w.num_q_heads
    for b in range(w.batch):
        s, e = int(off[b]), int(off[b + 1])
        sel = rows[(rows >= s * Hq) & (rows < e * Hq)]
        if len(sel) == 0:
            continue
        l0, l1 = int(cu[b]), int(cu[b + 1])
        oracle.verify_attn_oracle(inp.q[s:e], inp.k_cache[l0:l1], inp.v_cache[l0:l1], inp.k_tree[s:e],
                                  inp.v_tree[s:e], inp.parent[s:e], np.array([0, l1 - l0], dtype=np.int32),
                                  num_q_heads=Hq, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                                  tree_size=e - s, scale=inp.scale, rows=sel - s * Hq, nthreads=cores)


def time_oracle(inp, target_s=12.0, max_rows=None):
    """Time the fp64 oracle on a bounded sample of rows with every host core; returns
    (us per full call, rows sampled, seconds, cores)."""
    w = inp.workload
    total = inp.num_nodes * w.num_q_heads
    cores = len(os.sched_getaffinity(0))
    rng = np.random.default_rng(123)
    probe = np.sort(rng.choice(total, size=min(total, max(cores, 8)), replace=False))
    t0 = time.perf_counter()
    oracle_rows(inp, probe, cores)
    t_probe = max(time.perf_counter() - t0, 1e-6)
    per_row = t_probe / len(probe)
    n = int(min(total, max(len(probe), target_s / per_row)))
    if max_rows:
        n = min(n, max_rows)
    rows = np.sort(rng.choice(total, size=n, replace=False))
    t0 = time.perf_counter()
    oracle_rows(inp, rows, cores)
    dt = time.perf_counter() - t0
    return dt / n * total * 1e6, n, dt, cores


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    inp = make_inputs(w, seed=0)
    total = inp.num_nodes * w.num_q_heads
    per_step_target = max(0.5, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    vals = []
    n_rows = cores = None
    for s in range(args.warmup + args.steps):
        us, n_rows, dt, cores = time_oracle(inp, target_s=per_step_target)
        if s >= args.warmup:
            vals.append(us)
    v = float(statistics.mean(vals))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": v / 1000.0,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(inp, "n/a (CPU)"),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{n_rows} of {total} query rows per step, scaled to one call"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------- other configs
CONFIG_WORKLOADS = ("tiny_L1k_T16_h4x1_d64", "llama8b_L16k_T64_h32x8_d128", "70b_L128k_T128_h64x8_d128_bfs",
                    "ragged_b8_L4k-32k_T64_h32x8_d128")


def roofline_of(fig, part_s, step_s, peaks):
    """Kernel and step roofline fractions of one workload against the measured peaks."""
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tc = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    t_bytes = fig["partials_bytes"] / (hbm * 1e9)
    t_flops = fig["partials_flops"] / (tc * 1e12)
    bound = "tensor" if t_flops >= t_bytes else "hbm"
    roof_step = max(fig["step_bytes"] / (hbm * 1e9), fig["step_flops"] / (tc * 1e12))
    return {"bound": bound, "kernel_frac": max(t_flops, t_bytes) / part_s, "step_frac": roof_step / step_s,
            "roofline_us": roof_step * 1e6}


def time_config(name, steps, warmup, spin_cycles, flush, dev, peaks):
    """One BASELINE config timed like the headline (L2 flushed and the step queued before
    each call): whole ls_verify_attn call and the partials kernel alone, µs per call."""
    import torch

    from tree_verification_attention_longspec_b200 import binding
    w = WORKLOADS[name]
    inp = make_inputs(w, seed=0)
    fig = workload_figures(inp)

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)

    d_in = dict(q=bf(inp.q), k_cache=bf(inp.k_cache), v_cache=bf(inp.v_cache), k_tree=bf(inp.k_tree),
                v_tree=bf(inp.v_tree),
                parent=torch.from_numpy(np.ascontiguousarray(inp.parent, dtype=np.int32)).to(dev),
                cu=torch.from_numpy(np.ascontiguousarray(inp.cu_seqlens, dtype=np.int32)).to(dev))
    op = binding.VerifyAttn(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.tree_size,
                            cu_seqlens_host=inp.cu_seqlens, device=dev)
    out = torch.empty_like(d_in["q"])
    lse = torch.empty(out.shape[0], w.num_q_heads, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    ptr = {k: v.data_ptr() for k, v in d_in.items()}
    dims, ws, wsb = op.dims, op.workspace.data_ptr(), op.ws_bytes

    def full_call():
        rc = binding.call_raw(ptr["q"], ptr["k_cache"], ptr["v_cache"], ptr["k_tree"], ptr["v_tree"],
                              ptr["parent"], ptr["cu"], out.data_ptr(), lse.data_ptr(), dims, ws, wsb, sp)
        if rc:
            raise binding.LSError(rc, "ls_verify_attn")

    def partials():
        rc = binding.call_partials_raw(ptr["q"], ptr["k_cache"], ptr["v_cache"], ptr["k_tree"], ptr["v_tree"],
                                       ptr["parent"], ptr["cu"], dims, ws, wsb, sp)
        if rc:
            raise binding.LSError(rc, "ls_verify_attn_partials")

    for _ in range(warmup):
        flush.zero_()
        full_call()
    torch.cuda.synchronize(dev)
    times = {}
    for label, fn in (("call", full_call), ("partials", partials)):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        for k in range(steps):
            flush.zero_()
            torch.cuda._sleep(spin_cycles)
            ev[k][0].record(stream)
            fn()
            ev[k][1].record(stream)
        torch.cuda.synchronize(dev)
        times[label] = float(statistics.mean(e[0].elapsed_time(e[1]) for e in ev))
    st = op.check()
    if st != 0:
        raise binding.LSError(st, f"device status ({name})")
    call_ms, part_ms = max_over_ranks([times["call"], times["partials"]], device=dev)
    r = roofline_of(fig, part_ms / 1000.0, call_ms / 1000.0, peaks)
    return {"us_per_call": call_ms * 1000.0, "partials_us": part_ms * 1000.0, "bound": r["bound"],
            "kernel_frac": r["kernel_frac"], "step_frac": r["step_frac"], "roofline_us": r["roofline_us"],
            "kv_hbm_gbs": fig["kv_bytes"] / (call_ms / 1000.0) / 1e9, "steps": steps, "plan": op.plan}


# ----------------------------------------------------------------------------- our arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    from tree_verification_attention_longspec_b200 import binding

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    binding.load_library()

    w = WORKLOADS[args.workload]
    if args.cross:
        # the draft's cross-attention: args.cross queries per sequence over the same cache
        w = dataclasses.replace(w, name=f"{w.name}_cross{args.cross}", tree_size=args.cross, tree="chain")
    inp = make_inputs(w, seed=rank)   # independent problem per rank
    fig = workload_figures(inp, cross=bool(args.cross))

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)

    def i32(a):
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)

    d_in = dict(q=bf(inp.q), k_cache=bf(inp.k_cache), v_cache=bf(inp.v_cache), k_tree=bf(inp.k_tree),
                v_tree=bf(inp.v_tree), parent=i32(inp.parent), cu=i32(inp.cu_seqlens))
    op = binding.VerifyAttn(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.tree_size,
                            cu_seqlens_host=inp.cu_seqlens, device=dev)
    out = torch.empty_like(d_in["q"])
    lse = torch.empty(out.shape[0], w.num_q_heads, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream
    ptr = {k: v.data_ptr() for k, v in d_in.items()}
    dims, ws, wsb = op.dims, op.workspace.data_ptr(), op.ws_bytes

    def partials():
        rc = binding.call_partials_raw(ptr["q"], ptr["k_cache"], ptr["v_cache"], ptr["k_tree"], ptr["v_tree"],
                                       ptr["parent"], ptr["cu"], dims, ws, wsb, sp)
        if rc:
            raise binding.LSError(rc, "ls_verify_attn_partials")

    def full_call():
        rc = binding.call_raw(ptr["q"], ptr["k_cache"], ptr["v_cache"], ptr["k_tree"], ptr["v_tree"],
                              ptr["parent"], ptr["cu"], out.data_ptr(), lse.data_ptr(), dims, ws, wsb, sp)
        if rc:
            raise binding.LSError(rc, "ls_verify_attn")

    def check_status():
        return binding.check(dims, ws_x.data_ptr(), sp) if args.cross else op.check()

    if args.cross:
        wsb_x = binding.cross_workspace_size(dims)
        ws_x = torch.empty(wsb_x, dtype=torch.uint8, device=dev)

        def full_call():  # noqa: F811
            rc = binding.call_cross_raw(ptr["q"], ptr["k_cache"], ptr["v_cache"], ptr["cu"], out.data_ptr(),
                                        lse.data_ptr(), dims, ws_x.data_ptr(), wsb_x, sp)
            if rc:
                raise binding.LSError(rc, "ls_cross_attn")

        partials = full_call  # noqa: F811  (timed as one call)
        args.no_e2e = True

    if args.paged:
        # the same keys in a paged cache: every sequence's pages in random physical order
        ps = args.paged
        cu = inp.cu_seqlens
        n_pages = [(int(x) + ps - 1) // ps for x in np.diff(cu)]
        total = max(1, sum(n_pages))
        perm = np.random.default_rng(1234).permutation(total)
        max_pages = max(1, max(n_pages))
        table = np.zeros((w.batch, max_pages), dtype=np.int32)
        src_rows = np.zeros(total * ps, dtype=np.int64)   # packed row of every paged row
        valid = np.zeros(total * ps, dtype=bool)
        nxt = 0
        for b in range(w.batch):
            for i in range(n_pages[b]):
                phys = int(perm[nxt])
                nxt += 1
                table[b, i] = phys
                k0, k1 = cu[b] + i * ps, min(cu[b] + (i + 1) * ps, cu[b + 1])
                src_rows[phys * ps: phys * ps + (k1 - k0)] = np.arange(k0, k1)
                valid[phys * ps: phys * ps + (k1 - k0)] = True
        kp = np.where(valid[:, None, None], inp.k_cache[src_rows], 0).astype(np.uint16)
        vp = np.where(valid[:, None, None], inp.v_cache[src_rows], 0).astype(np.uint16)
        d_pages = dict(k=bf(kp), v=bf(vp), table=torch.from_numpy(table).to(dev))
        pg = binding.PagedKV(ps, max_pages, total, d_pages["table"].data_ptr())

        def full_call():  # noqa: F811
            rc = binding.call_paged_raw(ptr["q"], d_pages["k"].data_ptr(), d_pages["v"].data_ptr(), pg,
                                        ptr["k_tree"], ptr["v_tree"], ptr["parent"], ptr["cu"], out.data_ptr(),
                                        lse.data_ptr(), dims, ws, wsb, sp)
            if rc:
                raise binding.LSError(rc, "ls_verify_attn_paged")

        partials = full_call  # noqa: F811  (the paged call has no separate partials stage)
        args.no_e2e = True

    if inp.cu_tree is not None or args.rope > 0 or args.window > 0:
        # per-sequence trees and/or in-kernel RoPE: the general entry, timed as one call
        # (tree kernel when rotating, partials, combine)
        if args.paged:
            raise SystemExit("--paged with per-sequence trees or --rope is not a bench mode")
        cu_tree_d = i32(inp.cu_tree) if inp.cu_tree is not None else None
        topt = binding.TreeOpts(cu_tree=cu_tree_d.data_ptr() if cu_tree_d is not None else None,
                                total_nodes=inp.num_nodes if cu_tree_d is not None else 0, window=args.window,
                                rope_theta=float(args.rope))
        wsb_t = binding.ex_workspace_size(dims, topt)
        ws_t = torch.empty(wsb_t, dtype=torch.uint8, device=dev)

        def full_call():  # noqa: F811
            rc = binding.call_ex_raw(ptr["q"], ptr["k_cache"], ptr["v_cache"], None, ptr["k_tree"], ptr["v_tree"],
                                     ptr["parent"], ptr["cu"], topt, out.data_ptr(), lse.data_ptr(), dims,
                                     ws_t.data_ptr(), wsb_t, sp)
            if rc:
                raise binding.LSError(rc, "ls_verify_attn_ex")

        def check_status():  # noqa: F811
            return binding.check(dims, ws_t.data_ptr(), sp)

        partials = full_call  # noqa: F811
        args.no_e2e = True

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)

    for _ in range(args.warmup):
        flush.zero_()
        full_call()
        flush.zero_()
        partials()
    torch.cuda.synchronize(dev)
    st = check_status()
    if st != 0:
        raise binding.LSError(st, "device status after warm-up")

    # The GPU spins for a while before each timed step so that the host has queued the
    # whole step by the time the first event fires: the events then bracket the kernels'
    # own execution, not host submission gaps (those are in the e2e figure).
    spin_cycles = int(args.spin_us * 2000)  # >= spin_us at any SM clock up to 2 GHz
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    evp = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with sampler:
        # timed steps: one ls_verify_attn call each (partials kernel + combine kernel,
        # the second launched as a programmatic dependent of the first)
        for k in range(K):
            flush.zero_()
            torch.cuda._sleep(spin_cycles)
            ev[k][0].record(stream)
            full_call()
            ev[k][1].record(stream)
        # the dominant kernel alone, under the same conditions, for its roofline figure
        for k in range(K):
            flush.zero_()
            torch.cuda._sleep(spin_cycles)
            evp[k][0].record(stream)
            partials()
            evp[k][1].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    step_ms = [e[0].elapsed_time(e[1]) for e in ev]
    partials_ms = [e[0].elapsed_time(e[1]) for e in evp]
    ms_per_step = float(statistics.mean(step_ms))
    partials_avg_ms = float(statistics.mean(partials_ms))
    ms_per_step, partials_avg_ms = max_over_ranks([ms_per_step, partials_avg_ms], device=dev)
    st = check_status()
    if st != 0:
        raise binding.LSError(st, "device status after timing")

    # the other BASELINE configs, timed the same way in the same run (fewer steps each)
    configs = None
    plain = not (args.cross or args.paged or args.rope > 0 or args.window > 0 or inp.cu_tree is not None)
    if plain and not args.no_configs and w.name == HEADLINE.name:
        peaks_c, _ = load_peaks()
        cfg_sampler = ClockSampler(local)
        with cfg_sampler:
            configs = {name: time_config(name, max(3, min(K, args.config_steps)), args.warmup, spin_cycles, flush,
                                         dev, peaks_c)
                       for name in CONFIG_WORKLOADS}
        configs["clocks"] = cfg_sampler.summary()
        configs["timing"] = ("each config: L2 flushed and the step queued before every call, CUDA events; "
                             "us_per_call = ls_verify_attn, partials_us = the partials kernel alone; "
                             "kernel_frac / step_frac against MEASURED_PEAKS.json (bf16 burst, HBM copy)")

    # e2e through the public call with host buffers: H2D of every input, the call, D2H of out+lse
    e2e = None
    if not args.no_e2e:
        h_in = {k: v.cpu().pin_memory() for k, v in d_in.items()}
        h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h_lse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        d2 = {k: torch.empty_like(v) for k, v in d_in.items()}
        h2d = sum(v.numel() * v.element_size() for v in h_in.values())
        d2h = h_out.numel() * h_out.element_size() + h_lse.numel() * h_lse.element_size()
        n_e2e = max(3, min(K, 20))
        times = []
        for k in range(2 + n_e2e):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush.zero_()
            e0.record(stream)
            for name in d2:
                d2[name].copy_(h_in[name], non_blocking=True)
            o2, l2_ = op(d2["q"], d2["k_cache"], d2["v_cache"], d2["k_tree"], d2["v_tree"], d2["parent"],
                         d2["cu"], out, lse)
            h_out.copy_(o2, non_blocking=True)
            h_lse.copy_(l2_, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if k >= 2:
                times.append(e0.elapsed_time(e1))
        e2e_ms = float(statistics.mean(times))
        e2e_ms = max_over_ranks([e2e_ms], device=dev)[0]
        e2e = {"value": e2e_ms * 1000.0 / world, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": n_e2e}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    whole_call = inp.cu_tree is not None or args.rope > 0 or args.window > 0
    peaks, peak_kind = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tc = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    part_s = partials_avg_ms / 1000.0
    t_bytes = fig["partials_bytes"] / (hbm * 1e9)
    t_flops = fig["partials_flops"] / (tc * 1e12)
    if t_flops >= t_bytes:
        roof = {"bound": "tensor", "achieved": fig["partials_flops"] / part_s / 1e12, "peak": tc,
                "unit": "TFLOP/s"}
    else:
        roof = {"bound": "hbm", "achieved": fig["partials_bytes"] / part_s / 1e9, "peak": hbm,
                "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = recorded_traffic(w.name)
    roof["kernel"] = "partials (ls_verify_attn_partials: prefix and tree blocks)"
    roof["peak_source"] = f"{peak_kind} (MEASURED_PEAKS.json burst)" if peak_kind == "measured" else "fallback"
    roof["kernel_us"] = partials_avg_ms * 1000.0
    step_s = ms_per_step / 1000.0
    roof_step_s = max(fig["step_bytes"] / (hbm * 1e9), fig["step_flops"] / (tc * 1e12))

    line = {"metric": METRIC, "value": ms_per_step * 1000.0 / world, "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16, random draft trees)",
            "config": dict(config_of(inp, "flushed before every step (write of 2x L2), outside the timed events; "
                                    "the step is fully queued before its first event"),
                           **({"kv_layout": f"paged: {args.paged} keys per page, pages in random order"}
                              if args.paged else {}),
                           **({"attention": f"prefix-only (ls_cross_attn), {args.cross} queries per sequence"}
                              if args.cross else {}),
                           **({"rope_theta": args.rope, "rope": "q and k_tree rotated in-kernel at L_b + depth"}
                              if args.rope > 0 else {}),
                           **({"window": args.window} if args.window > 0 else {})),
            "kv_hbm_gbs": fig["kv_bytes"] / step_s / 1e9,
            "roofline_step": {"roofline_us": roof_step_s * 1e6, "frac": roof_step_s / step_s,
                              "bytes": fig["step_bytes"], "flops": fig["step_flops"]},
            "roofline": roof, "gpu_launches": (3 if args.rope > 0 else 2) * K, "plan": op.plan,
            "kernel_timing": ("paged, cross-attention, per-sequence-tree or RoPE call: the roofline figure "
                              "times the whole call"
                              if (args.paged or args.cross or whole_call) else
                              "partials kernel timed in K further partials-only launches after the K "
                              "steps, same L2 flush and queueing"),
            "clocks": sampler.summary(), "e2e": e2e}
    if configs is not None:
        line["configs"] = configs
    if world == 1 and not args.no_cpu_baseline:
        us, n, dt, cores = time_oracle(inp, target_s=args.cpu_seconds)
        line["cpu_baseline"] = {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"{n} of {fig['rows']} query rows ({dt:.1f} s), scaled to one call"}
    print(json.dumps(line))
    return 0


def run_accept(args):
    """Greedy acceptance (ls_tree_accept_greedy) over the workload's trees with bf16
    logits of args.accept entries per node: one JSON line, HBM roofline of the logits read."""
    import torch

    from tree_verification_attention_longspec_b200 import binding
    from tree_verification_attention_longspec_b200.inputs import make_accept_inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    sizes = None
    if w.tree_size_range:
        sizes = np.random.default_rng(1).integers(w.tree_size_range[0], w.tree_size_range[1] + 1, size=w.batch)
    inp = make_accept_inputs(w.batch, w.tree_size, args.accept, "bf16", tree=w.tree, match_prob=0.8, seed=0,
                             tree_sizes=sizes)
    N, V = inp.logits.shape
    logits = torch.from_numpy(np.ascontiguousarray(inp.logits).view(np.int16)).to(dev)
    tok = torch.from_numpy(inp.tokens).to(dev)
    par = torch.from_numpy(inp.parent).to(dev)
    cu = torch.from_numpy(inp.cu_tree).to(dev) if inp.cu_tree is not None else None
    dims = binding.AcceptDims(inp.batch, inp.tree_size, V, binding.LS_DTYPE_BF16)
    wsb = binding.accept_workspace_size(dims, N)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    alen = torch.empty(inp.batch, dtype=torch.int32, device=dev)
    path = torch.empty(inp.batch, inp.tree_size, dtype=torch.int32, device=dev)
    nxt = torch.empty(inp.batch, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    sp = stream.cuda_stream

    def call():
        rc = binding.call_accept_raw(logits.data_ptr(), tok.data_ptr(), par.data_ptr(),
                                     cu.data_ptr() if cu is not None else None, N, alen.data_ptr(),
                                     path.data_ptr(), nxt.data_ptr(), dims, ws.data_ptr(), wsb, sp)
        if rc:
            raise binding.LSError(rc, "ls_tree_accept_greedy")

    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        flush.zero_()
        call()
    torch.cuda.synchronize(dev)
    got_len = alen.cpu().tolist()
    K = args.steps
    spin_cycles = int(args.spin_us * 2000)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    sampler = ClockSampler(0)
    with sampler:
        for k in range(K):
            flush.zero_()
            torch.cuda._sleep(spin_cycles)
            ev[k][0].record(stream)
            call()
            ev[k][1].record(stream)
        torch.cuda.synchronize(dev)
    ms = float(statistics.mean(e[0].elapsed_time(e[1]) for e in ev))
    peaks, peak_kind = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    nbytes = N * V * 2 + 3 * N * 4 + inp.batch * (inp.tree_size + 2) * 4
    ach = nbytes / (ms / 1000.0) / 1e9
    line = {"metric": "greedy tree acceptance µs/call (argmax over the logits + tree walk)", "value": ms * 1000.0,
            "unit": UNIT, "n_gpus": 1, "steps": K, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (N(0,1) logits with planted peaks; draft tokens copy the parent's peak w.p. 0.8)",
            "config": {"workload": f"{w.name}_accept_V{V}", "batch": inp.batch, "nodes": N, "vocab": V,
                       "l2": "flushed before every call, outside the timed events"},
            "roofline": {"bound": "hbm", "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
                         "traffic": None, "kernel": "ls_tree_accept_greedy (argmax + walk, whole call)",
                         "peak_source": peak_kind},
            "accept_len": got_len, "gpu_launches": 2 * K, "clocks": sampler.summary(), "e2e": None}
    print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=HEADLINE.name, choices=sorted(WORKLOADS))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cross", type=int, default=0,
                    help="time ls_cross_attn (prefix-only attention) with this many queries per sequence")
    ap.add_argument("--paged", type=int, default=0,
                    help="time ls_verify_attn_paged with pages of this many keys (no e2e figure)")
    ap.add_argument("--rope", type=float, default=0.0,
                    help="RoPE base: q and k_tree arrive unrotated and are rotated in-kernel")
    ap.add_argument("--window", type=int, default=0,
                    help="sliding-window attention over the last WINDOW positions (draft self-attention)")
    ap.add_argument("--accept", type=int, default=0,
                    help="time greedy tree acceptance with bf16 logits of this vocabulary size instead")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip timing the other BASELINE configs after the headline")
    ap.add_argument("--config-steps", type=int, default=30,
                    help="timed calls per other config (at most --steps)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--spin-us", type=float, default=150.0,
                    help="GPU spin before each timed step so the step is queued before it starts")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.accept:
        return run_accept(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
