#!/usr/bin/env python
"""Benchmark of the paged-KV decode layer-step on B200.

One step = pa_reshape_and_cache of the step's new token per sequence, then
pa_decode (partition kernel + partition-merge kernel) over every sequence's
whole context.  Default workload: the Llama-3-70B GQA decode layer (128
sequences, 64 q / 8 kv heads, head_dim 128, bf16, 16-token blocks, context
lengths lognormal with median 2048 clipped to [16, 8192], shuffled pool).

Prints ONE JSON line (rank 0).  `value` = decode algorithmic bytes (K and V
of every valid context token + q + out) per second, summed over ranks, with
inputs resident in HBM; the KV pool (~1.2 GB) is far larger than the 126 MB
L2, so no flush is needed between steps.  Multi-GPU runs are independent
replicas (weak scaling; decode needs no exchange between GPUs): under
torchrun each rank is one GPU; `--gpus N` without a launcher starts the N
processes itself.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

Other workloads: --workload mixed_step_fp8 (fp8-cache decode of 256 sequences
next to a 2 x 512-query chunked prefill, on two streams) and --workload
spec_verify_bf16 (the Llama-3-70B GQA cache with 5 new queries per sequence,
pa_decode_multi, as when draft tokens are verified); --workload alloc_host
(the host block allocator with prefix caching under a serving trace; no GPU);
--workload swap_bf16 (pa_swap_blocks moving 256 MB of blocks device <-> pinned
host per direction).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention HBM GB/s (% of B200 peak); seqs/s per layer-step"
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; replicas only)
# ---------------------------------------------------------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def dist_init(world: int, backend: str):
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=120))
    return dist


def reduce_over_ranks(x: float, op: str, world: int, device=None) -> float:
    """Max or sum of a scalar over all ranks (identity when world == 1)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX if op == "max" else dist.ReduceOp.SUM)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ---------------------------------------------------------------------------
# measured peaks and clocks
# ---------------------------------------------------------------------------

def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.rows = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", gpu_id], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 8:
                self.rows.append(parts)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.t.join(timeout=2)
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4)
                          if r[4 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows)}


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------

def describe(spec, ctx, num_blocks):
    from pagedattention_paged_kv_pa_b200 import workloads as W
    return (f"{spec.name}: {spec.num_seqs} seqs, {spec.n_q_heads} q / {spec.n_kv_heads} kv "
            f"heads, head_dim {spec.head_dim}, q {W.DTYPE_NAMES[spec.q_dtype]}, kv "
            f"{W.DTYPE_NAMES[spec.kv_dtype]}, block 16, ctx {spec.ctx_kind}{spec.ctx_args} "
            f"(sum {int(ctx.sum())} tokens), shuffled pool of {num_blocks} blocks")


def get_spec(name):
    from pagedattention_paged_kv_pa_b200 import workloads as W
    return {"llama3_70b_gqa_bf16": W.LLAMA3_70B_GQA_BF16, "llama2_7b_fp16": W.LLAMA2_7B_FP16,
            "llama3_70b_gqa_bf16_ctx8k": W.LLAMA3_70B_GQA_BF16_CTX8K,
            "mixed_step_fp8_decode": W.MIXED_DECODE_FP8, "tiny_fp32": W.TINY_FP32}[name]


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline leg and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(inp, budget_s: float, max_units=None, threads=None):
    """Time the oracle on a bounded prefix of the workload's sequences, on
    `threads` host threads (default: all cores).
    Returns (seconds, bytes, seqs, tokens, threads)."""
    import oracle as orc
    from pagedattention_paged_kv_pa_b200 import workloads as W
    spec = inp.spec
    q = inp.q.cpu()
    bt = inp.block_tables.cpu().numpy()
    cl = inp.context_lens.cpu().numpy()
    kp, vp = inp.k_pool, inp.v_pool
    threads = threads or os.cpu_count() or 1
    done_s, done_bytes, done_seqs, done_tok = 0.0, 0, 0, 0
    s = 0
    chunk = max(1, threads // max(1, spec.n_kv_heads) or 1)
    while s < spec.num_seqs and done_s < budget_s:
        idx = list(range(s, min(s + chunk, spec.num_seqs)))
        need = sorted({int(b) for i in idx for b in bt[i, :-(-int(cl[i]) // 16)]})
        remap = {b: j for j, b in enumerate(need)}
        bt2 = np.full((len(idx), bt.shape[1]), -1, np.int32)
        for r, i in enumerate(idx):
            n = -(-int(cl[i]) // 16)
            bt2[r, :n] = [remap[int(b)] for b in bt[i, :n]]
        import torch
        sel = torch.tensor(need, dtype=torch.long, device=kp.device)
        k_sub = kp[sel].cpu() if len(need) else kp[:1].cpu()
        v_sub = vp[sel].cpu() if len(need) else vp[:1].cpu()
        t0 = time.perf_counter()
        orc.paged_decode(q[idx], k_sub, v_sub, bt2, cl[idx], inp.scale, spec.q_dtype,
                         spec.kv_dtype, inp.k_scale, inp.v_scale, nthreads=threads)
        done_s += time.perf_counter() - t0
        done_bytes += W.decode_algorithmic_bytes(cl[idx], spec.n_q_heads, spec.n_kv_heads,
                                                 spec.head_dim, W.ELEM_BYTES[spec.q_dtype],
                                                 W.ELEM_BYTES[spec.kv_dtype])
        done_seqs += len(idx)
        done_tok += int(cl[idx].sum())
        s += len(idx)
    return done_s, done_bytes, done_seqs, done_tok, threads


def oracle_sample_multi(inp, qm, q_len: int, budget_s: float):
    """Time the oracle's causal chunk (query i of a sequence with context c at
    position c - q_len + i) on a bounded prefix of the sequences.
    Returns (seconds, bytes, seqs, context tokens, threads)."""
    import torch
    import oracle as orc
    from pagedattention_paged_kv_pa_b200 import workloads as W
    spec = inp.spec
    bt = inp.block_tables.cpu().numpy()
    cl = inp.context_lens.cpu().numpy()
    qc = qm.cpu()
    threads = os.cpu_count() or 1
    eb, qb = W.ELEM_BYTES[spec.kv_dtype], W.ELEM_BYTES[spec.q_dtype]
    done_s, done_bytes, done_seqs, done_tok = 0.0, 0, 0, 0
    s = 0
    chunk = max(1, threads // max(1, spec.n_kv_heads) or 1)
    while s < spec.num_seqs and done_s < budget_s:
        idx = [i for i in range(s, min(s + chunk, spec.num_seqs)) if cl[i] > 0]
        s = min(s + chunk, spec.num_seqs)
        if not idx:
            continue
        need = sorted({int(b) for i in idx for b in bt[i, :-(-int(cl[i]) // 16)]})
        remap = {b: j for j, b in enumerate(need)}
        bt2 = np.full((len(idx), bt.shape[1]), -1, np.int32)
        for r, i in enumerate(idx):
            nb = -(-int(cl[i]) // 16)
            bt2[r, :nb] = [remap[int(b)] for b in bt[i, :nb]]
        sel = torch.tensor(need, dtype=torch.long, device=inp.k_pool.device)
        k_sub, v_sub = inp.k_pool[sel].cpu(), inp.v_pool[sel].cpu()
        m = [int(min(q_len, cl[i])) for i in idx]
        qs = torch.cat([qc[i, q_len - k:] for i, k in zip(idx, m)])
        qsl = np.concatenate([[0], np.cumsum(m)]).astype(np.int32)
        t0 = time.perf_counter()
        orc.paged_prefill(qs, k_sub, v_sub, bt2, qsl, cl[idx].astype(np.int32), inp.scale,
                          spec.q_dtype, spec.kv_dtype, inp.k_scale, inp.v_scale,
                          nthreads=threads)
        done_s += time.perf_counter() - t0
        done_bytes += (int(cl[idx].sum()) * 2 * spec.n_kv_heads * spec.head_dim * eb
                       + len(idx) * q_len * spec.n_q_heads * spec.head_dim * 2 * qb)
        done_seqs += len(idx)
        done_tok += int(cl[idx].sum())
    return done_s, done_bytes, done_seqs, done_tok, threads


# ---------------------------------------------------------------------------
# end-to-end staging: one pinned host buffer per step, two device buffers
# ---------------------------------------------------------------------------

class Staging:
    """A step's host inputs packed into one pinned buffer (16-byte aligned
    segments) and moved by ONE host-to-device copy into one of two device
    buffers, whose segments the kernels read as typed views; outputs come back
    by one device-to-host copy each.  Copies run on their own streams, so step
    i+1's upload and step i's download overlap the kernels of step i."""

    def __init__(self, tensors, outs, dev):
        import torch
        self.dev = dev
        sizes = [t.numel() * t.element_size() for t in tensors]
        offs, o = [], 0
        for n in sizes:
            offs.append(o)
            o += (n + 15) // 16 * 16
        self.host = torch.empty(o, dtype=torch.uint8).pin_memory()
        for t, off, n in zip(tensors, offs, sizes):
            self.host[off:off + n].copy_(t.detach().cpu().contiguous().view(-1).view(torch.uint8))
        self.bufs = [torch.empty(o, dtype=torch.uint8, device=dev) for _ in range(2)]
        self.views = [[b[off:off + n].view(t.dtype).view(t.shape)
                       for t, off, n in zip(tensors, offs, sizes)] for b in self.bufs]
        self.outs = [[torch.empty_like(t) for t in outs] for _ in range(2)]
        self.outs_h = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
                       for _ in range(2)]
        self.h2d_bytes = o
        self.d2h_bytes = sum(t.numel() * t.element_size() for t in outs)
        self.up = torch.cuda.Stream(dev)
        self.down = torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()
        self.uploaded = [ev(), ev()]
        self.consumed = [ev(), ev()]   # kernels done with input buffer b
        self.downloaded = [ev(), ev()]  # output buffer b copied out
        self.used = [False, False]

    def run(self, steps, kernels):
        """`steps` pipelined steps; kernels(inputs, outputs) queues one step's
        work on the current stream.  Returns the device time in ms, from
        before the first upload to after the last download."""
        import torch
        comp = torch.cuda.current_stream(self.dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        self.up.wait_event(e0)
        self.down.wait_event(e0)
        self.used = [False, False]
        for i in range(steps):
            b = i & 1
            if self.used[b]:
                self.up.wait_event(self.consumed[b])
            with torch.cuda.stream(self.up):
                self.bufs[b].copy_(self.host, non_blocking=True)
                self.uploaded[b].record(self.up)
            comp.wait_event(self.uploaded[b])
            if self.used[b]:
                comp.wait_event(self.downloaded[b])
            kernels(self.views[b], self.outs[b])
            self.consumed[b].record(comp)
            self.down.wait_event(self.consumed[b])
            with torch.cuda.stream(self.down):
                for dst, src in zip(self.outs_h[b], self.outs[b]):
                    dst.copy_(src, non_blocking=True)
                self.downloaded[b].record(self.down)
            self.used[b] = True
        comp.wait_stream(self.down)
        comp.wait_stream(self.up)
        e1.record(comp)
        torch.cuda.synchronize(self.dev)
        return e0.elapsed_time(e1)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, local):
    import torch
    from pagedattention_paged_kv_pa_b200 import binding as B
    from pagedattention_paged_kv_pa_b200 import workloads as W

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist_init(world, "nccl")
    spec = get_spec(args.workload)
    inp = W.make_decode_inputs(spec, device=dev)
    ctx = inp.context_lens.cpu().numpy()
    n = spec.num_seqs
    # the step's new token (position ctx-1) of every sequence
    key, val = W.make_new_kv(n, spec.n_kv_heads, spec.head_dim,
                             spec.q_dtype if spec.kv_dtype == W.FP8_E4M3 else spec.kv_dtype,
                             dev, seed=spec.seed + 7)
    slots = torch.from_numpy(W.slots_from_positions(
        inp.block_tables.cpu().numpy(), np.arange(n), np.maximum(ctx - 1, 0))).to(dev)
    slots[torch.from_numpy(ctx == 0).to(dev)] = -1
    out = torch.empty_like(inp.q)
    mb = inp.block_tables.shape[1]
    ws = B.alloc_decode_workspace(inp.q, mb)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    kvdt = B.dtype_code(inp.k_pool)
    algo_bytes = W.decode_algorithmic_bytes(ctx, spec.n_q_heads, spec.n_kv_heads, spec.head_dim,
                                            W.ELEM_BYTES[spec.q_dtype], W.ELEM_BYTES[spec.kv_dtype])
    n_parts = -(-mb * 16 // (2048 if spec.kv_dtype == W.FP8_E4M3 else 1024))
    launches_per_step = 2 + (1 if n_parts > 1 else 0)

    def step(ev_a=None, ev_b=None):
        B.pa_reshape_and_cache(inp.k_pool, inp.v_pool, key, val, slots, inp.k_scale,
                               inp.v_scale, dev_err=err)
        if ev_a is not None:
            ev_a.record()
        B.pa_decode_partitions(out, inp.q, inp.k_pool, inp.v_pool, inp.block_tables,
                               inp.context_lens, inp.scale, inp.k_scale, inp.v_scale,
                               workspace=ws, dev_err=err)
        if ev_b is not None:
            ev_b.record()
        B.pa_decode_reduce(out, inp.context_lens, mb, kvdt, inp.v_scale, workspace=ws)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flags {int(err.item())}")

    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if hasattr(props, "uuid") else str(local))
    time.sleep(0.3)
    K = args.steps
    # the timed steps carry no events between their kernels (an event record
    # between two programmatically dependent launches costs their overlap)
    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    torch.cuda.synchronize()
    t_start.record()
    for i in range(K):
        step()
    t_stop.record()
    torch.cuda.synchronize()
    barrier(world, dev)
    clocks = sampler.stop()
    ms_total = t_start.elapsed_time(t_stop)
    # the partition kernel alone: events around it, in a second loop of steps
    KE = max(3, min(K, 200))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(KE)]
    for i in range(KE):
        step(*evs[i])
    torch.cuda.synchronize()
    kern_ms = [a.elapsed_time(b) for a, b in evs]
    ms_max = reduce_over_ranks(ms_total, "max", world, dev)
    total_bytes = reduce_over_ranks(algo_bytes * K, "sum", world, dev)
    value = total_bytes / (ms_max / 1e3) / 1e9

    # ---- end to end through the public API from pinned host buffers: per
    # step one upload of q, the new K/V, slots, block tables and context
    # lengths (packed), the step's kernels, one download of the output
    stg = Staging([inp.q, key, val, slots, inp.block_tables, inp.context_lens], [out], dev)

    def e2e_kernels(ins, outs):
        q_d, key_d, val_d, slots_d, bt_d, cl_d = ins
        B.pa_reshape_and_cache(inp.k_pool, inp.v_pool, key_d, val_d, slots_d, inp.k_scale,
                               inp.v_scale, dev_err=err)
        B.pa_decode(outs[0], q_d, inp.k_pool, inp.v_pool, bt_d, cl_d, inp.scale, inp.k_scale,
                    inp.v_scale, workspace=ws, dev_err=err)

    K2 = max(3, min(K, 200))
    stg.run(3, e2e_kernels)
    barrier(world, dev)
    e2e_ms = reduce_over_ranks(stg.run(K2, e2e_kernels), "max", world, dev)
    barrier(world, dev)
    e2e_value = reduce_over_ranks(algo_bytes * K2, "sum", world, dev) / (e2e_ms / 1e3) / 1e9
    h2d, d2h = stg.h2d_bytes, stg.d2h_bytes
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flags {int(err.item())}")
    # the last step's downloaded output is the resident-input decode's, bit for bit
    B.pa_decode(out, inp.q, inp.k_pool, inp.v_pool, inp.block_tables, inp.context_lens,
                inp.scale, inp.k_scale, inp.v_scale, workspace=ws, dev_err=err)
    if not torch.equal(stg.outs_h[(K2 - 1) & 1][0], out.cpu()):
        raise RuntimeError("end-to-end output differs from the resident-input decode")

    # ---- roofline of the dominant kernel (partition kernel), live events
    kern_avg_ms = sum(kern_ms) / len(kern_ms)
    kern_med_ms = statistics.median(kern_ms)
    peak, peak_src = hbm_peak()
    achieved = algo_bytes / (kern_avg_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4),
                "traffic": traffic_from_profile(args.workload),
                "kernel": "decode_mma_kernel (partition kernel)",
                "kernel_avg_us": round(kern_avg_ms * 1e3, 2),
                "kernel_median_us": round(kern_med_ms * 1e3, 2),
                "frac_at_median": round(algo_bytes / (kern_med_ms / 1e3) / 1e9 / peak, 4),
                "kernel_events": len(kern_ms),
                "kernel_timing": "events around the partition kernel in a separate loop of "
                                 "the same steps, after the timed loop",
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                if peak_src == "measured" else "fallback 6.65 TB/s"}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_max / K, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype":
            {W.F32: "f32", W.F16: "f16", W.BF16: "bf16"}[spec.q_dtype]
            + ("+fp8kv" if spec.kv_dtype == W.FP8_E4M3 else ""),
        "data": "synthetic (seeded N(0,1) values, seeded context lengths and block shuffle)",
        "config": {"workload": describe(spec, ctx, inp.num_blocks), "global_batch": n * world,
                   "seq_len": int(ctx.max()), "tokens_per_step": int(ctx.sum()),
                   "algorithmic_bytes_per_step": int(algo_bytes),
                   "step": "reshape_and_cache (1 new token/seq) + decode partitions + reduce",
                   "l2": "inputs larger than L2 (KV pool > 1 GB vs 126 MB L2); no flush",
                   "parallelism": f"replicas x{world}"},
        "pct_of_peak": round(100 * value / world / peak, 2),
        "seqs_per_s": round(n * world / (ms_max / K / 1e3), 1),
        "tokens_per_s": round(float(ctx.sum()) * world / (ms_max / K / 1e3), 1),
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": K2,
                "ms_per_step": round(e2e_ms / K2, 4),
                "pipeline": "per step one packed pinned upload (q, new K/V, slots, block "
                            "tables, context lengths) and one download of the output, on "
                            "two copy streams double-buffered against the kernels"},
        "roofline": roofline,
        "gpu_launches": launches_per_step * K,
        "clocks": clocks,
    }
    if rank == 0 and args.workload == "llama3_70b_gqa_bf16" and not args.no_configs:
        del stg
        line["configs"] = extra_configs(dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, b, ns, nt, th = oracle_sample(inp, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": round(b / secs / 1e9, 4), "unit": "GB/s", "cores": th,
                                "kind": "oracle",
                                "sample": f"first {ns} of {n} sequences ({nt} tokens) of the "
                                          f"same workload, {secs:.1f} s, fp64 C oracle"}
        # the same oracle on one host thread (a smaller sample)
        secs1, b1, ns1, nt1, _ = oracle_sample(inp, budget_s=min(3.0, args.cpu_budget),
                                               threads=1)
        line["cpu_baseline"]["single_thread"] = {
            "value": round(b1 / secs1 / 1e9, 4), "unit": "GB/s", "cores": 1,
            "sample": f"first {ns1} sequences ({nt1} tokens), {secs1:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def tensor_peak():
    """Measured dense bf16 burst TFLOP/s (f16 shares the nominal 2.25 PF)."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured bf16_tflops (burst)"
    except Exception:
        return 1590.0, "fallback 1.59 PF"


def extra_configs(dev, iters: int = 30):
    """The other workloads' dominant kernels, each timed alone with CUDA events
    on the launching stream (median of `iters` launches after 3 warm-ups) and
    set against its roofline: Llama-2-7B fp16 decode, shared-prefix sampling
    decode (L2 flushed before each call), the mixed step's fp8 decode and its
    chunked prefill (tensor cores), and draft-token verification."""
    import torch
    from pagedattention_paged_kv_pa_b200 import binding as B
    from pagedattention_paged_kv_pa_b200 import workloads as W
    peak, psrc = hbm_peak()
    tpeak, tsrc = tensor_peak()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    mk = lambda: torch.cuda.Event(enable_timing=True)

    def med_ms(fn, flush=False):
        for _ in range(3):
            fn()
        evs = [(mk(), mk()) for _ in range(iters)]
        for a, b in evs:
            if flush:
                _l2_flush(dev)
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize(dev)
        return statistics.median(a.elapsed_time(b) for a, b in evs)

    def hbm_entry(name, kernel, ms, nbytes, **kw):
        gbs = nbytes / (ms / 1e3) / 1e9
        e = {"workload": name, "kernel": kernel, "median_us": round(ms * 1e3, 2),
             "events": iters, "algorithmic_bytes": int(nbytes), "achieved": round(gbs, 1),
             "unit": "GB/s", "peak": peak, "frac": round(gbs / peak, 4), "bound": "hbm",
             "peak_source": psrc}
        e.update(kw)
        return e

    res = {}
    # Llama-2-7B fp16 decode layer and the mixed step's fp8 decode: partition kernel
    for key, spec in (("llama2_7b_fp16", W.LLAMA2_7B_FP16),
                      ("mixed_step_fp8_decode", W.MIXED_DECODE_FP8)):
        inp = W.make_decode_inputs(spec, device=dev)
        out = torch.empty_like(inp.q)
        ws = B.alloc_decode_workspace(inp.q, inp.block_tables.shape[1])
        ctx = inp.context_lens.cpu().numpy()
        nbytes = W.decode_algorithmic_bytes(ctx, spec.n_q_heads, spec.n_kv_heads, spec.head_dim,
                                            W.ELEM_BYTES[spec.q_dtype], W.ELEM_BYTES[spec.kv_dtype])
        ms = med_ms(lambda: B.pa_decode_partitions(
            out, inp.q, inp.k_pool, inp.v_pool, inp.block_tables, inp.context_lens, inp.scale,
            inp.k_scale, inp.v_scale, workspace=ws, dev_err=err))
        res[key] = hbm_entry(describe(spec, ctx, inp.num_blocks), "decode_mma_kernel", ms,
                             nbytes, traffic=traffic_from_profile(key if key != "mixed_step_fp8_decode"
                                                                  else "mixed_step_fp8_decode"))
        del inp, out, ws
    # shared-prefix sampling: one call (group + sequence partitions, merge)
    inp, _ = W.make_shared_prefix_inputs(dev)
    spec = inp.spec
    ctx = inp.context_lens.cpu().numpy()
    groups = B.prefix_groups(inp.block_tables, inp.context_lens, spec.n_q_heads,
                             spec.n_kv_heads, spec.kv_dtype)
    gdev = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in groups.items()}
    out = torch.empty_like(inp.q)
    ws = B.alloc_decode_workspace(inp.q, inp.block_tables.shape[1])
    logical = W.decode_algorithmic_bytes(ctx, spec.n_q_heads, spec.n_kv_heads, spec.head_dim, 2, 2)
    shared_tok = int(sum((len([m for m in row if m >= 0]) - 1) * nb * 16 for row, nb in
                         zip(groups["members"].tolist(), groups["shared_blocks"].tolist())))
    unique = logical - shared_tok * 2 * spec.n_kv_heads * spec.head_dim * 2
    ms = med_ms(lambda: B.pa_decode_shared_prefix(
        out, inp.q, inp.k_pool, inp.v_pool, inp.block_tables, inp.context_lens, inp.scale, gdev,
        workspace=ws, dev_err=err), flush=True)
    res["shared_prefix_bf16"] = hbm_entry(
        "shared-prefix sampling: 16 prompts x 4 samples, bf16, 32 q / 8 kv heads",
        "pa_decode_shared_prefix (one partition launch + merge), on unique bytes", ms, unique,
        logical_bytes=int(logical), logical_gbs=round(logical / (ms / 1e3) / 1e9, 1),
        l2="flushed (256 MB write) before every call")
    del inp, out, ws
    # draft-token verification: pa_decode_multi (partition kernel + merge)
    spec, q_len = W.SPEC_VERIFY_BF16, W.SPEC_VERIFY_Q_LEN
    inp = W.make_decode_inputs(spec, device=dev)
    qm = W.make_multi_queries(inp, q_len, seed=spec.seed + 1)
    out = torch.empty_like(qm)
    ctx = inp.context_lens.cpu().numpy()
    mb = inp.block_tables.shape[1]
    ws = torch.empty(max(B.pa_decode_workspace_size(spec.num_seqs, spec.n_q_heads * q_len,
                                                    spec.head_dim, mb), 16),
                     dtype=torch.uint8, device=dev)
    nbytes = (int(ctx.sum()) * 2 * spec.n_kv_heads * spec.head_dim * 2
              + spec.num_seqs * q_len * spec.n_q_heads * spec.head_dim * 4)
    ms = med_ms(lambda: B.pa_decode_multi(out, qm, inp.k_pool, inp.v_pool, inp.block_tables,
                                          inp.context_lens, inp.scale, workspace=ws,
                                          dev_err=err))
    res["spec_verify_bf16"] = hbm_entry(describe(spec, ctx, inp.num_blocks)
                                        + f"; {q_len} queries per sequence",
                                        "pa_decode_multi: mq_tc_kernel + mq_merge_kernel",
                                        ms, nbytes,
                                        traffic=traffic_from_profile("spec_verify_bf16", "mq"))
    del inp, qm, out, ws
    # the mixed step's chunked prefill: widening pass + tensor-core kernel
    pspec = W.MIXED_PREFILL_FP8
    pinp = W.make_prefill_inputs(pspec, device=dev)
    pout = torch.empty_like(pinp.q)
    pws = B.alloc_prefill_workspace(pinp.k_pool, pinp.block_tables)
    flops = prefill_causal_flops(pinp)
    ms = med_ms(lambda: B.pa_prefill_paged(
        pout, pinp.q, pinp.k_pool, pinp.v_pool, pinp.block_tables, pinp.query_start_loc,
        pinp.context_lens, pinp.scale, pspec.chunk_len, pinp.k_scale, pinp.v_scale,
        workspace=pws, dev_err=err))
    tf = flops / (ms / 1e3) / 1e12
    res["mixed_step_fp8_prefill"] = {
        "workload": "2 chunks x 512 queries over 4096-token paged histories, 32 q / 8 kv heads, "
                    "q bf16, fp8 KV, causal", "kernel": "prefill_widen_kernel + prefill_tc_kernel",
        "median_us": round(ms * 1e3, 2), "events": iters, "algorithmic_flop": int(flops),
        "achieved": round(tf, 1), "unit": "TFLOP/s", "peak": tpeak, "frac": round(tf / tpeak, 4),
        "bound": "tensor", "peak_source": tsrc,
        "traffic": traffic_from_profile("mixed_step_fp8_prefill", "prefill")}
    del pinp, pout, pws
    torch.cuda.synchronize(dev)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flags {int(err.item())}")
    torch.cuda.empty_cache()
    return res


def prefill_causal_flops(inp) -> int:
    """Algorithmic flops of causal chunked prefill: 2 products x 2 flop x d per
    (query row, q head, visible key)."""
    qsl = inp.query_start_loc.cpu().numpy()
    cl = inp.context_lens.cpu().numpy()
    keys = 0
    for c in range(len(cl)):
        L = int(qsl[c + 1] - qsl[c])
        H = int(cl[c]) - L
        keys += L * H + L * (L + 1) // 2
    s = inp.spec
    return 4 * s.head_dim * s.n_q_heads * keys


def run_mixed(args, rank, world, local):
    """Mixed continuous-batching step: slot writes of all new tokens, then the
    decode (256 sequences) on one stream and the chunked prefill (2 chunks of
    512 queries over 4096 tokens of history) on another, fp8 KV cache."""
    import torch
    from pagedattention_paged_kv_pa_b200 import binding as B
    from pagedattention_paged_kv_pa_b200 import workloads as W

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist_init(world, "nccl")
    dspec, pspec = W.MIXED_DECODE_FP8, W.MIXED_PREFILL_FP8
    dinp = W.make_decode_inputs(dspec, device=dev)
    pinp = W.make_prefill_inputs(pspec, device=dev)
    ctx = dinp.context_lens.cpu().numpy()
    n = dspec.num_seqs
    # new tokens: one per decode sequence, the whole chunk for each prefill
    dkey, dval = W.make_new_kv(n, dspec.n_kv_heads, dspec.head_dim, W.BF16, dev, seed=3005)
    dslots = torch.from_numpy(W.slots_from_positions(
        dinp.block_tables.cpu().numpy(), np.arange(n), ctx - 1)).to(dev)
    qsl = pinp.query_start_loc.cpu().numpy()
    pcl = pinp.context_lens.cpu().numpy()
    seq_ids = np.concatenate([np.full(int(qsl[c + 1] - qsl[c]), c) for c in range(len(pcl))])
    pos = np.concatenate([np.arange(int(pcl[c]) - int(qsl[c + 1] - qsl[c]), int(pcl[c]))
                          for c in range(len(pcl))])
    pslots = torch.from_numpy(W.slots_from_positions(pinp.block_tables.cpu().numpy(), seq_ids,
                                                     pos)).to(dev)
    pkey, pval = W.make_new_kv(len(pos), pspec.n_kv_heads, pspec.head_dim, W.BF16, dev,
                               seed=3006)
    dout = torch.empty_like(dinp.q)
    pout = torch.empty_like(pinp.q)
    mb = dinp.block_tables.shape[1]
    ws = B.alloc_decode_workspace(dinp.q, mb)
    pws = B.alloc_prefill_workspace(pinp.k_pool, pinp.block_tables)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    s_dec = torch.cuda.current_stream(dev)
    s_pre = torch.cuda.Stream(dev)
    dec_bytes = W.decode_algorithmic_bytes(ctx, dspec.n_q_heads, dspec.n_kv_heads,
                                           dspec.head_dim, 2, 1)
    flops = prefill_causal_flops(pinp)

    def decode_part(ev=None):
        B.pa_reshape_and_cache(dinp.k_pool, dinp.v_pool, dkey, dval, dslots, dinp.k_scale,
                               dinp.v_scale, dev_err=err, stream=s_dec)
        if ev is not None:
            ev[0].record(s_dec)
        B.pa_decode_partitions(dout, dinp.q, dinp.k_pool, dinp.v_pool, dinp.block_tables,
                               dinp.context_lens, dinp.scale, dinp.k_scale, dinp.v_scale,
                               workspace=ws, dev_err=err, stream=s_dec)
        if ev is not None:
            ev[1].record(s_dec)
        B.pa_decode_reduce(dout, dinp.context_lens, mb, B.PA_FP8_E4M3, dinp.v_scale,
                           workspace=ws, stream=s_dec)

    def prefill_part(ev=None):
        B.pa_reshape_and_cache(pinp.k_pool, pinp.v_pool, pkey, pval, pslots, pinp.k_scale,
                               pinp.v_scale, dev_err=err, stream=s_pre)
        if ev is not None:
            ev[0].record(s_pre)
        B.pa_prefill_paged(pout, pinp.q, pinp.k_pool, pinp.v_pool, pinp.block_tables,
                           pinp.query_start_loc, pinp.context_lens, pinp.scale,
                           pspec.chunk_len, pinp.k_scale, pinp.v_scale, workspace=pws,
                           dev_err=err, stream=s_pre)
        if ev is not None:
            ev[1].record(s_pre)

    def step(dev_ev=None, pre_ev=None):
        s_pre.wait_stream(s_dec)
        prefill_part(pre_ev)
        decode_part(dev_ev)
        s_dec.wait_stream(s_pre)

    mk = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flags {int(err.item())}")

    # each part alone (kernel rooflines), then the concurrent step
    def time_alone(fn, k):
        evs = [(mk(), mk()) for _ in range(k)]
        torch.cuda.synchronize()
        for i in range(k):
            fn(evs[i])
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs) / k

    K = args.steps
    dec_ms = time_alone(decode_part, min(K, 200))
    s_pre.wait_stream(s_dec)
    pre_ms = time_alone(prefill_part, min(K, 200))
    torch.cuda.synchronize()

    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if hasattr(props, "uuid") else str(local))
    time.sleep(0.3)
    t0, t1 = mk(), mk()
    barrier(world, dev)
    torch.cuda.synchronize()
    t0.record(s_dec)
    for _ in range(K):
        step()
    t1.record(s_dec)
    torch.cuda.synchronize()
    barrier(world, dev)
    clocks = sampler.stop()
    ms = reduce_over_ranks(t0.elapsed_time(t1), "max", world, dev)
    value = reduce_over_ranks(dec_bytes * K, "sum", world, dev) / (ms / 1e3) / 1e9
    peak, _ = hbm_peak()
    try:
        tflops_peak = float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"])
        tsrc = "measured bf16_tflops (burst; f16 and bf16 share the nominal 2.25 PF)"
    except Exception:
        tflops_peak, tsrc = 1590.0, "fallback 1.59 PF"
    pre_tflops = flops / (pre_ms / 1e3) / 1e12
    dec_gbs = dec_bytes / (dec_ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16+fp8kv",
        "data": "synthetic (seeded N(0,1) values, seeded lengths and block shuffle)",
        "config": {"workload": "mixed continuous-batching step: " + describe(dspec, ctx, dinp.num_blocks)
                   + f"; + prefill of 2 chunks x 512 queries over 4096-token paged histories, "
                     f"32 q / 8 kv heads, fp8 KV; slot writes of all {n + len(pos)} new tokens; "
                     "decode and prefill on two streams",
                   "global_batch": n * world, "seq_len": int(ctx.max()),
                   "l2": "inputs larger than L2 (decode KV 2.2 GB); no flush",
                   "parallelism": f"replicas x{world}"},
        "value_counts": "decode algorithmic bytes per concurrent step time",
        "decode_alone": {"us": round(dec_ms * 1e3, 2), "achieved_gbs": round(dec_gbs, 1),
                         "frac": round(dec_gbs / peak, 4),
                         "includes": "slot write + partition kernel"},
        "prefill_alone": {"us": round(pre_ms * 1e3, 2), "algorithmic_flop": int(flops),
                          "achieved_tflops": round(pre_tflops, 1),
                          "peak_tflops": tflops_peak, "frac": round(pre_tflops / tflops_peak, 4),
                          "peak_source": tsrc, "includes": "slot write + widening pass + prefill kernel"},
        "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(dec_gbs / peak, 4),
                     "traffic": traffic_from_profile("mixed_step_fp8_decode"),
                     "kernel": "decode_mma_kernel (fp8 cache)"},
        # per step: two slot writes, decode partition + merge, widening pass + prefill
        "gpu_launches": 6 * K,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


DECODE_SOURCES = ("decode.cu", "pa_internal.h", "pa_device.cuh")
PREFILL_SOURCES = ("prefill.cu", "pa_internal.h", "pa_device.cuh")
MQ_SOURCES = ("decode_multi_tc.cu", "mq_tc.h", "tc_ops.cuh", "pa_internal.h", "pa_device.cuh")
KERNEL_SOURCES = {"decode": DECODE_SOURCES, "prefill": PREFILL_SOURCES, "mq": MQ_SOURCES}


def source_hash(files=DECODE_SOURCES):
    """First 16 hex digits of the SHA-256 of a kernel's sources."""
    import hashlib
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "pagedattention_paged_kv_pa_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def decode_source_hash():
    return source_hash(DECODE_SOURCES)


def traffic_from_profile(workload, kernel="decode"):
    """DRAM bytes per launch of the decode partition kernel (kernel="decode",
    profiles/decode_traffic.txt), of the tensor-core prefill kernel
    (kernel="prefill", profiles/prefill_traffic.txt) or of the multi-query
    kernel (kernel="mq", profiles/mq_traffic.txt) from the committed ncu
    summaries, if they were taken on the current kernel sources; None
    otherwise."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.txt")
    files = KERNEL_SOURCES[kernel]
    try:
        rec = {}
        for line in open(path):
            if ":" in line and not line.startswith("#"):
                k, v = line.split(":", 1)
                rec[k.strip()] = v.strip()
        if rec.get(f"{kernel}_src_sha256_16") != source_hash(files):
            return None
        return int(rec[workload]) if workload in rec else None
    except Exception:
        return None


# ---------------------------------------------------------------------------
# reference arm: the fp64 CPU oracle, as it stands
# ---------------------------------------------------------------------------

def run_reference(args, rank, world, local):
    if rank != 0:
        return
    import torch
    from pagedattention_paged_kv_pa_b200 import workloads as W
    spec = get_spec(args.workload)
    inp = W.make_decode_inputs(spec, device="cpu")
    steps, warm = args.steps, args.warmup
    per_step = max(0.05, min(2.0, 150.0 / max(1, steps + warm)))
    for _ in range(warm):
        oracle_sample(inp, per_step)
    tot_s = tot_b = 0.0
    ns = nt = 0
    th = 1
    for _ in range(steps):
        s, b, a, t, th = oracle_sample(inp, per_step)
        tot_s += s
        tot_b += b
        ns, nt = a, t
    value = tot_b / tot_s / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": steps, "warmup": warm,
            "ms_per_step": round(1e3 * tot_s / steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": describe(spec, inp.context_lens.numpy(), inp.num_blocks)},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": th,
                             "kind": "oracle",
                             "sample": f"each step: first {ns} sequences ({nt} tokens), "
                                       f"about {per_step:.2f} s of fp64 C oracle work"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_spec_verify(args, rank, world, local):
    """Draft-token verification step on the Llama-3-70B GQA cache: the slot
    write of each sequence's q_len new tokens, then pa_decode_multi (query i
    of a sequence with context c attends to keys 0 .. c - q_len + i)."""
    import torch
    import oracle as orc
    from pagedattention_paged_kv_pa_b200 import binding as B
    from pagedattention_paged_kv_pa_b200 import workloads as W

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist_init(world, "nccl")
    spec, q_len = W.SPEC_VERIFY_BF16, W.SPEC_VERIFY_Q_LEN
    inp = W.make_decode_inputs(spec, device=dev)
    qm = W.make_multi_queries(inp, q_len, seed=spec.seed + 1)
    ctx = inp.context_lens.cpu().numpy()
    n = spec.num_seqs
    # the step's q_len new tokens of every sequence: positions c - q_len .. c - 1
    pos = ctx[:, None] - q_len + np.arange(q_len)[None, :]
    seq_ids = np.repeat(np.arange(n), q_len)
    key, val = W.make_new_kv(n * q_len, spec.n_kv_heads, spec.head_dim, spec.kv_dtype, dev,
                             seed=spec.seed + 7)
    slots_np = W.slots_from_positions(inp.block_tables.cpu().numpy(), seq_ids,
                                      np.maximum(pos.reshape(-1), 0))
    slots_np[pos.reshape(-1) < 0] = -1
    slots = torch.from_numpy(slots_np).to(dev)
    out = torch.empty_like(qm)
    mb = inp.block_tables.shape[1]
    ws = torch.empty(max(B.pa_decode_workspace_size(n, spec.n_q_heads * q_len, spec.head_dim,
                                                    mb), 16), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    eb = W.ELEM_BYTES[spec.kv_dtype]
    qo_bytes = n * q_len * spec.n_q_heads * spec.head_dim * 2 * W.ELEM_BYTES[spec.q_dtype]
    algo_bytes = int(ctx.sum()) * 2 * spec.n_kv_heads * spec.head_dim * eb + qo_bytes

    def step(ev_a=None, ev_b=None):
        B.pa_reshape_and_cache(inp.k_pool, inp.v_pool, key, val, slots, dev_err=err)
        if ev_a is not None:
            ev_a.record()
        B.pa_decode_multi(out, qm, inp.k_pool, inp.v_pool, inp.block_tables, inp.context_lens,
                          inp.scale, workspace=ws, dev_err=err)
        if ev_b is not None:
            ev_b.record()

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flags {int(err.item())}")
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if hasattr(props, "uuid") else str(local))
    time.sleep(0.3)
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    torch.cuda.synchronize()
    t0.record()
    for i in range(K):
        step(*evs[i])
    t1.record()
    torch.cuda.synchronize()
    barrier(world, dev)
    clocks = sampler.stop()
    ms_max = reduce_over_ranks(t0.elapsed_time(t1), "max", world, dev)
    value = reduce_over_ranks(algo_bytes * K, "sum", world, dev) / (ms_max / 1e3) / 1e9
    kern_ms = sum(a.elapsed_time(b) for a, b in evs) / K

    # ---- end to end through the public API: one packed upload, one download
    stg = Staging([qm, key, val, slots, inp.block_tables, inp.context_lens], [out], dev)

    def e2e_kernels(ins, outs):
        q_d, key_d, val_d, slots_d, bt_d, cl_d = ins
        B.pa_reshape_and_cache(inp.k_pool, inp.v_pool, key_d, val_d, slots_d, dev_err=err)
        B.pa_decode_multi(outs[0], q_d, inp.k_pool, inp.v_pool, bt_d, cl_d, inp.scale,
                          workspace=ws, dev_err=err)

    K2 = max(3, min(K, 200))
    stg.run(3, e2e_kernels)
    barrier(world, dev)
    e2e_ms = reduce_over_ranks(stg.run(K2, e2e_kernels), "max", world, dev)
    barrier(world, dev)
    h2d, d2h = stg.h2d_bytes, stg.d2h_bytes
    e2e_value = reduce_over_ranks(algo_bytes * K2, "sum", world, dev) / (e2e_ms / 1e3) / 1e9
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flags {int(err.item())}")

    peak, peak_src = hbm_peak()
    achieved = algo_bytes / (kern_ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_max / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) values, seeded context lengths and block shuffle)",
        "config": {"workload": describe(spec, ctx, inp.num_blocks)
                   + f"; {q_len} queries per sequence (draft-token verification)",
                   "global_batch": n * world, "q_len": q_len, "seq_len": int(ctx.max()),
                   "tokens_per_step": int(ctx.sum()), "algorithmic_bytes_per_step": algo_bytes,
                   "step": f"reshape_and_cache ({q_len} new tokens/seq) + pa_decode_multi",
                   "l2": "inputs larger than L2 (KV pool > 1 GB vs 126 MB L2); no flush",
                   "parallelism": f"replicas x{world}"},
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": K2,
                "ms_per_step": round(e2e_ms / K2, 4),
                "pipeline": "one packed pinned upload and one download per step on two copy "
                            "streams, double-buffered against the kernels"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": traffic_from_profile("spec_verify_bf16", "mq"),
                     "kernel": "pa_decode_multi: mq_tc_kernel (bf16 tensor cores, 64-row "
                               "tiles, persistent CTAs with equal shares of the key tiles) + "
                               "mq_merge_kernel (timed together)",
                     "kernel_avg_us": round(kern_ms * 1e3, 2),
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"},
        "gpu_launches": 3 * K,  # slot write + the multi-query kernel + its merge
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, b, ns, nt, th = oracle_sample_multi(inp, qm, q_len, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": round(b / secs / 1e9, 4), "unit": "GB/s", "cores": th,
                                "kind": "oracle",
                                "sample": f"first {ns} of {n} sequences ({nt} context tokens, "
                                          f"{q_len} queries each) of the same workload, "
                                          f"{secs:.1f} s, fp64 C oracle (causal chunk)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_shared_prefix(args, rank, world, local):
    """Decode over the shared-prefix sampling workload (16 prompts x 4 samples,
    each prompt's 2048+ token prefix in blocks its samples share), with
    pa_decode_shared_prefix (each group's shared blocks read once for the
    group) and, for comparison, plain pa_decode.  GB/s are reported on logical
    bytes (every sequence's whole context) and on unique bytes (each shared
    block once)."""
    import torch
    from pagedattention_paged_kv_pa_b200 import binding as B
    from pagedattention_paged_kv_pa_b200 import workloads as W
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist_init(world, "nccl")
    inp, _ = W.make_shared_prefix_inputs(dev)
    spec = inp.spec
    ctx = inp.context_lens.cpu().numpy()
    groups = B.prefix_groups(inp.block_tables, inp.context_lens, spec.n_q_heads,
                             spec.n_kv_heads, spec.kv_dtype)
    gdev = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in groups.items()}
    out = torch.empty_like(inp.q)
    mb = inp.block_tables.shape[1]
    ws = B.alloc_decode_workspace(inp.q, mb)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    logical = W.decode_algorithmic_bytes(ctx, spec.n_q_heads, spec.n_kv_heads, spec.head_dim, 2, 2)
    shared_tok = int(sum((len([m for m in row if m >= 0]) - 1) * nb * 16 for row, nb in
                         zip(groups["members"].tolist(), groups["shared_blocks"].tolist())))
    unique = logical - shared_tok * 2 * spec.n_kv_heads * spec.head_dim * 2

    def call(shared):
        if shared:
            B.pa_decode_shared_prefix(out, inp.q, inp.k_pool, inp.v_pool, inp.block_tables,
                                      inp.context_lens, inp.scale, gdev, workspace=ws,
                                      dev_err=err)
        else:
            B.pa_decode(out, inp.q, inp.k_pool, inp.v_pool, inp.block_tables, inp.context_lens,
                        inp.scale, workspace=ws, dev_err=err)

    def timed(shared, K):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
        for i in range(K):
            # the unique K/V (210 MB) is not far above the 126 MB L2: flush it
            # before each timed call
            _l2_flush(dev)
            evs[i][0].record()
            call(shared)
            evs[i][1].record()
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs) / K

    for shared in (True, False):
        for _ in range(max(args.warmup, 3)):
            call(shared)
    torch.cuda.synchronize()
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if hasattr(props, "uuid") else str(local))
    time.sleep(0.3)
    K = args.steps
    barrier(world, dev)
    ms = reduce_over_ranks(timed(True, K), "max", world, dev)
    ms_plain = reduce_over_ranks(timed(False, K), "max", world, dev)
    barrier(world, dev)
    clocks = sampler.stop()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flags {int(err.item())}")
    peak, _ = hbm_peak()
    line = {
        "metric": METRIC, "value": round(logical * world / (ms / 1e3) / 1e9, 1), "unit": "GB/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded)",
        "config": {"workload": f"shared-prefix sampling: 16 prompts x 4 samples, prompt 2048 + "
                               f"U{{1..15}}, 0-512 divergent tokens, 32 q / 8 kv heads, bf16 "
                               f"(sum {int(ctx.sum())} tokens, {inp.num_blocks} unique blocks, "
                               f"{len(groups['members'])} groups)",
                   "logical_bytes": int(logical), "unique_bytes": int(unique),
                   "l2": "flushed (256 MB write) before every timed call",
                   "parallelism": f"replicas x{world}"},
        "unique_gbs": round(unique / (ms / 1e3) / 1e9, 1),
        "roofline": {"bound": "hbm", "achieved": round(unique / (ms / 1e3) / 1e9, 1),
                     "peak": peak, "unit": "GB/s",
                     "frac": round(unique / (ms / 1e3) / 1e9 / peak, 4), "traffic": None,
                     "kernel": "pa_decode_shared_prefix (group + per-sequence partition "
                               "kernels + merge), on unique bytes"},
        "plain_decode": {"us": round(ms_plain * 1e3, 2),
                         "logical_gbs": round(logical / (ms_plain / 1e3) / 1e9, 1),
                         "unique_gbs": round(unique / (ms_plain / 1e3) / 1e9, 1)},
        "speedup_vs_plain_decode": round(ms_plain / ms, 3),
        "gpu_launches": 3 * K,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


_FLUSH = {}


def _l2_flush(dev):
    """Write 256 MB (twice the L2) so that no K/V stays cached between calls."""
    import torch
    buf = _FLUSH.get(dev)
    if buf is None:
        buf = _FLUSH[dev] = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    buf.fill_(1)


def run_swap(args, rank, world, local):
    """Swap preemption's data path: 4,096 blocks of the Llama-3-70B GQA layer
    (8 kv heads x 16 tokens x 128 dims, bf16, K and V: 256 MB) from the device
    pool to a pinned host pool and 4,096 back, per step, with pa_swap_blocks
    (one kernel per direction; the pair lists live in pinned host memory).
    The roofline denominator is a contiguous 256 MB pinned-host <-> device
    copy measured in the same run (the host link's copy-engine rate)."""
    import torch
    from pagedattention_paged_kv_pa_b200 import binding as B
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist_init(world, "nccl")
    n_kv, d, n_dev, n_host, n_move = 8, 128, 8192, 4096, 4096
    shape = (n_dev, n_kv, 16, d)
    kp = torch.randn(shape, dtype=torch.bfloat16, device=dev)
    vp = torch.randn(shape, dtype=torch.bfloat16, device=dev)
    hk = torch.empty((n_host,) + shape[1:], dtype=torch.bfloat16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    rng = np.random.default_rng(1008)
    out_pairs = torch.from_numpy(np.stack([rng.permutation(n_dev)[:n_move],
                                           np.arange(n_move)], 1).astype(np.int64)).pin_memory()
    in_pairs = torch.from_numpy(np.stack([np.arange(n_move), rng.permutation(n_dev)[:n_move]],
                                         1).astype(np.int64)).pin_memory()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    block_bytes = n_kv * 16 * d * 2
    moved = 2 * n_move * block_bytes  # K and V, one direction

    def step(evs=None):
        if evs:
            evs[0].record()
        B.pa_swap_blocks(hk, hv, kp, vp, out_pairs, dev_err=err)
        if evs:
            evs[1].record()
        B.pa_swap_blocks(kp, vp, hk, hv, in_pairs, dev_err=err)
        if evs:
            evs[2].record()

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flags {int(err.item())}")
    # the host link's contiguous copy rate, each direction
    flat_d = torch.empty(moved // 2, dtype=torch.bfloat16, device=dev)
    flat_h = torch.empty(moved // 2, dtype=torch.bfloat16).pin_memory()
    ref = {}
    for name, fn in (("d2h", lambda: flat_h.copy_(flat_d, non_blocking=True)),
                     ("h2d", lambda: flat_d.copy_(flat_h, non_blocking=True))):
        fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(5):
            fn()
        b.record()
        torch.cuda.synchronize()
        ref[name] = moved / (a.elapsed_time(b) / 5 / 1e3) / 1e9
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if hasattr(props, "uuid") else str(local))
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    barrier(world, dev)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for i in range(K):
        step(evs[i])
    t1.record()
    torch.cuda.synchronize()
    barrier(world, dev)
    clocks = sampler.stop()
    if int(err.item()) != 0:
        raise RuntimeError(f"device error flags {int(err.item())}")
    ms = reduce_over_ranks(t0.elapsed_time(t1), "max", world, dev)
    out_ms = sum(e[0].elapsed_time(e[1]) for e in evs) / K
    in_ms = sum(e[1].elapsed_time(e[2]) for e in evs) / K
    value = reduce_over_ranks(2 * moved * K, "sum", world, dev) / (ms / 1e3) / 1e9
    out_gbs, in_gbs = moved / (out_ms / 1e3) / 1e9, moved / (in_ms / 1e3) / 1e9
    line = {
        "metric": "KV block swap GB/s (device <-> pinned host, both directions)",
        "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"swap out {n_move} and in {n_move} random blocks of a "
                               f"{n_dev}-block device pool via a {n_host}-block pinned host "
                               f"pool; block = {n_kv} kv heads x 16 tokens x {d} dims bf16, "
                               f"K and V ({2 * block_bytes} B)",
                   "bytes_per_direction": moved, "parallelism": f"replicas x{world}"},
        "swap_out": {"us": round(out_ms * 1e3, 1), "gbs": round(out_gbs, 2),
                     "contiguous_copy_gbs": round(ref["d2h"], 2),
                     "frac": round(out_gbs / ref["d2h"], 4)},
        "swap_in": {"us": round(in_ms * 1e3, 1), "gbs": round(in_gbs, 2),
                    "contiguous_copy_gbs": round(ref["h2d"], 2),
                    "frac": round(in_gbs / ref["h2d"], 4)},
        "roofline": {"bound": "host_link", "achieved": round(min(out_gbs, in_gbs), 2),
                     "peak": round(min(ref["d2h"], ref["h2d"]), 2), "unit": "GB/s",
                     "frac": round(min(out_gbs / ref["d2h"], in_gbs / ref["h2d"]), 4),
                     "traffic": None, "kernel": "copy_blocks_kernel (pa_swap_blocks)",
                     "peak_source": "contiguous pinned-host <-> device copy, same run"},
        "gpu_launches": 2 * K,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_alloc_host(args, rank=0, world=1):
    """Host allocator under a synthetic serving trace (no GPU): requests drawn
    from 8 shared system prompts (256-1024 tokens) plus 16-256 private tokens
    are admitted with prefix caching on, decode 32 tokens one at a time, and
    finish; at most 64 run at once in a pool of 6,000 blocks, so cached blocks
    are evicted under pressure.  Reports allocator calls per second and the
    share of prompt tokens whose prefill the cache saved."""
    from pagedattention_paged_kv_pa_b200 import binding as B
    dist_init(world, "gloo")  # host-only replicas: the scalars go over gloo
    rng = np.random.default_rng(1007)
    prompts = [rng.integers(0, 1 << 30, size=int(rng.integers(256, 1025))).tolist()
               for _ in range(8)]
    n_req = max(200, args.steps)
    reqs = []
    for _ in range(n_req):
        p = prompts[int(rng.integers(0, 8))]
        reqs.append(p + rng.integers(0, 1 << 30, size=int(rng.integers(16, 257))).tolist())
    a = B.BlockAllocator(6000, 16)
    assert a.set_prefix_caching(True) == 0
    running, calls, prompt_toks, cached_toks, next_req = [], 0, 0, 0, 0
    t0 = time.perf_counter()
    while next_req < n_req or running:
        while next_req < n_req and len(running) < 64:
            st, _, nc = a.admit(next_req, reqs[next_req])
            calls += 1
            if st != 0:
                break
            prompt_toks += len(reqs[next_req])
            cached_toks += nc
            running.append([next_req, 32])
            next_req += 1
        for r in running:
            a.append_tokens(r[0], [int(rng.integers(0, 1 << 30))])
            calls += 1
            r[1] -= 1
        for r in [r for r in running if r[1] == 0]:
            a.free_seq(r[0])
            calls += 1
            running.remove(r)
    secs = time.perf_counter() - t0
    # replicas: every rank runs the trace; calls summed over the slowest rank's time
    secs_max = reduce_over_ranks(secs, "max", world)
    calls_all = reduce_over_ranks(calls, "sum", world)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": "host block allocator calls/s (prefix caching on)",
        "value": round(calls_all / secs_max), "unit": "calls/s", "n_gpus": 0, "ranks": world,
        "scaling": "weak", "steps": n_req, "warmup": 0,
        "higher_is_better": True, "data": "synthetic serving trace (seeded)",
        "config": {"workload": "8 shared prompts of 256-1024 tokens + 16-256 private tokens, "
                               "32 decode tokens per request, <= 64 running, 6000-block pool",
                   "requests": n_req},
        "prompt_tokens_saved": round(cached_toks / max(prompt_toks, 1), 4),
        "us_per_call": round(secs / calls * 1e6, 3), "cores": world,
        "note": "includes the Python binding's marshalling of every call"}), flush=True)


def spawn_replicas(n: int, argv) -> int:
    """`--gpus N` without a launcher: start N copies of this script, one per
    GPU (RANK = LOCAL_RANK = i, WORLD_SIZE = N, rendezvous on 127.0.0.1), as
    torchrun would; rank 0 prints the job's line.  Returns the worst exit
    code."""
    import socket
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    procs = []
    for r in range(n):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(n),
                   LOCAL_WORLD_SIZE=str(n), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, os.path.abspath(__file__)] + list(argv),
                                      env=env))
    return max(p.wait() for p in procs)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="llama3_70b_gqa_bf16")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads' kernel rooflines in the default line")
    args = ap.parse_args(argv)
    rank, world, local = dist_env()
    if "WORLD_SIZE" in os.environ:
        if args.gpus != world:
            sys.stderr.write(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}\n")
            return 2
    elif args.gpus > 1:
        return spawn_replicas(args.gpus, sys.argv[1:] if argv is None else argv)
    if args.impl == "reference":
        run_reference(args, rank, world, local)
    elif args.workload == "mixed_step_fp8":
        run_mixed(args, rank, world, local)
    elif args.workload == "spec_verify_bf16":
        run_spec_verify(args, rank, world, local)
    elif args.workload == "alloc_host":
        run_alloc_host(args, rank, world)
    elif args.workload == "swap_bf16":
        run_swap(args, rank, world, local)
    elif args.workload == "shared_prefix_bf16":
        run_shared_prefix(args, rank, world, local)
    else:
        run_ours(args, rank, world, local)
    return 0


if __name__ == "__main__":
    sys.exit(main())
