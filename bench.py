#!/usr/bin/env python3
"""Benchmark of block-sparse attention with hybrid top-k + top-p block masks on B200.

One step is one attention call through the whole path, on inputs resident in HBM:
    pool Q,K per block -> block scores + hybrid selection -> block-sparse attention
at the Wan2.1-14B-720p self-attention shape (B=1, H=40, N=75600, d=128, block 128) with k for
95 % block sparsity (k=30) and p=0.9, on seeded synthetic Q/K/V of the video-DiT structure
described in block_sparse_attention_blocks_b200/workloads.py.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {bsa,reference}]

Prints one JSON line (rank 0).  `value` is effective TFLOPS over the executed block pairs
(4*d*rows*cols per pair, valid tokens only) per whole call, summed over ranks; `ms_per_step` is
ms per call.  Multi-GPU: one process per GPU (torchrun), every rank runs its own independent
call (the (b, h) units of the path never exchange data), so the scaling is weak and there is no
collective on the data path; the step time is the max over ranks.

`--impl reference` times the fp64 CPU oracle (a deliberately slow, obviously correct program)
on the host cores on a bounded sample of the same workload and prints the same line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "ms/call and effective TFLOPS (% BF16 peak) of block-sparse attn at 95% sparsity"
WORKLOAD = "wan14b_720p"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 2**20


# ----------------------------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fwd_kernel_wan14b_720p_traffic.txt")
KERNEL_SOURCES = ("block_sparse_attention_blocks_b200/csrc/attn.cu",
                  "block_sparse_attention_blocks_b200/csrc/softmax.cuh",
                  "block_sparse_attention_blocks_b200/csrc/ptx.cuh")


def attention_traffic(workload: str, heads: int, pairs: int):
    """DRAM bytes (read + write) of one attention launch from the committed ncu capture, or None
    when the kernel sources changed since the capture or the workload is not the captured one."""
    import hashlib

    try:
        fields = {}
        with open(TRAFFIC_FILE) as f:
            for line in f:
                if line.startswith("#") or ":" not in line:
                    continue
                k, v = line.split(":", 1)
                fields[k.strip()] = v.strip()
        h = hashlib.sha256()
        for rel in KERNEL_SOURCES:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
    except OSError:
        return None
    if fields.get("source_sha256") != h.hexdigest():
        return None
    if not fields.get("workload", "").startswith(workload + " ") or f"({pairs} executed" not in \
            fields.get("workload", "") or heads != 40:
        return None
    return int(fields["dram_bytes_read"]) + int(fields["dram_bytes_write"])


def launches_per_step(bh: int) -> int:
    """Kernels of one step: pooling, block scores, row selection, attention."""
    return 4


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
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
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(smax)),
                "power_w_max": float(max(power)), "samples": len(sm), "reasons": sorted(reasons)}


def executed_flops(kv_cnt, mask, N, d, bs):
    """4*d*sum over executed (query block, key block) pairs of valid rows x valid columns."""
    import torch

    nb = kv_cnt.shape[-1]
    rows = torch.full((nb,), float(bs), dtype=torch.float64, device=kv_cnt.device)
    rows[-1] = float(N - (nb - 1) * bs)
    cols_sum = kv_cnt.to(torch.float64) * bs - mask[..., -1].to(torch.float64) * (bs - rows[-1])
    pairs = int(kv_cnt.sum().item())
    flops = float((4.0 * d * (cols_sum * rows).sum()).item())
    return flops, pairs


def max_over_ranks(x: float, device=None) -> float:
    """The largest value of x over all ranks (identity on one process)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_heads(n: int, rank: int, world: int):
    """The flat (batch, head) indices rank `rank` of `world` computes when the heads of one call
    are split across ranks: a contiguous slice, sizes differing by at most one."""
    lo = rank * n // world
    hi = (rank + 1) * n // world
    return list(range(lo, hi))


def sum_over_ranks(x: float, device=None) -> float:
    """The sum of x over all ranks (identity on one process)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def make_inputs(w, rank, world, split_heads=False):
    """Seeded inputs; rank 0 generates them once and shares them through /dev/shm.  With
    split_heads every rank generates only its own slice of the heads (shard_heads)."""
    from block_sparse_attention_blocks_b200 import workloads as W

    if world == 1:
        return W.make_qkv(w)
    if split_heads:
        return W.make_qkv(w, heads=shard_heads(w.B * w.H, rank, world))
    import torch.distributed as dist

    names = None
    if rank == 0:
        q, k, v = W.make_qkv(w)
        base = f"/dev/shm/bsa_bench_{w.name}_{os.getpid()}"
        for nm, x in zip("qkv", (q, k, v)):
            np.save(f"{base}_{nm}.npy", x)
        names = [base]
    obj = [names[0] if names else None]
    dist.broadcast_object_list(obj, src=0)
    base = obj[0]
    if rank != 0:
        q, k, v = (np.load(f"{base}_{nm}.npy", mmap_mode="r") for nm in "qkv")
        q, k, v = (np.ascontiguousarray(x) for x in (q, k, v))
    dist.barrier()
    if rank == 0:
        for nm in "qkv":
            try:
                os.remove(f"{base}_{nm}.npy")
            except OSError:
                pass
    return q, k, v


# ----------------------------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ----------------------------------------------------------------------------------------------
def oracle_sample(w, q, k, v, heads, qblocks_per_head, seed=0):
    """Time the oracle on a bounded sample: pool + select for `heads` heads in full, then masked
    attention for `qblocks_per_head` seeded query blocks of each.  Returns a dict with the time
    and the executed-pair FLOPs of the sampled attention."""
    import oracle

    BH, N, d, bs, nb = w.B * w.H, w.N, w.d, w.bs, w.nb
    qf, kf, vf = (x.reshape(BH, N, d) for x in (q, k, v))
    hs = list(heads)
    t0 = time.perf_counter()
    qp = oracle.pool_blocks(qf[hs], bs)
    kp = oracle.pool_blocks(kf[hs], bs)
    sel = oracle.select(qp, kp, w.topk, w.topp, w.scale)
    t_ps = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    picks = [(hi, int(i)) for hi in range(len(hs))
             for i in rng.choice(nb, size=min(qblocks_per_head, nb), replace=False)]
    mask = sel.mask.reshape(len(hs), nb, nb)
    t0 = time.perf_counter()
    oracle.masked_attention(qf[hs], kf[hs], vf[hs], mask, bs, w.scale, picks)
    t_att = time.perf_counter() - t0
    flops = 0.0
    last = N - (nb - 1) * bs
    for hi, i in picks:
        rows = bs if i < nb - 1 else last
        cols = mask[hi, i].sum() * bs - (bs - last) * mask[hi, i, nb - 1]
        flops += 4.0 * d * rows * cols
    pairs_sel = mask.sum()
    # executed-pair FLOPs of every query block of the sampled heads (valid rows and keys only)
    rows_of = np.full(nb, float(bs))
    rows_of[-1] = last
    cols = mask.sum(axis=2) * bs - (bs - last) * mask[:, :, nb - 1]
    flops_heads = float((4.0 * d * rows_of[None, :] * cols).sum())
    # the full call: pool+select of all heads scales with heads, attention with executed pairs
    return {"t_pool_select": t_ps, "t_attn": t_att, "attn_flops": flops, "heads": len(hs),
            "qblocks": len(picks), "pairs_heads": int(pairs_sel), "flops_heads": flops_heads,
            "threads": oracle.num_threads()}


def cpu_estimate(w, s, total_flops):
    """Extrapolate a sample to the full call: pool+select by heads, attention by FLOPs."""
    t_ps_full = s["t_pool_select"] * (w.B * w.H) / s["heads"]
    t_att_full = s["t_attn"] * total_flops / max(s["attn_flops"], 1.0)
    ms = (t_ps_full + t_att_full) * 1e3
    return ms, total_flops / (ms * 1e-3) / 1e12


ORACLE_CONFIGS = (("pr1_1k", None), ("wan1.3b_480p", 64), ("stress_mixed", 64))


def oracle_config_timing(name: str, qblocks):
    """The oracle on workload `name`: pooling and selection of every head in full, then masked
    attention of every query block (qblocks None) or of `qblocks` seeded query blocks spread over
    the heads, extrapolated to the whole call by executed-pair FLOPs.  Returns a dict."""
    import oracle
    from block_sparse_attention_blocks_b200 import workloads as W

    w = W.get(name)
    q, k, v = W.make_qkv(w)
    BH, N, d, bs, nb = w.B * w.H, w.N, w.d, w.bs, w.nb
    qf, kf, vf = (x.reshape(BH, N, d) for x in (q, k, v))
    t0 = time.perf_counter()
    sel = oracle.select(oracle.pool_blocks(qf, bs), oracle.pool_blocks(kf, bs), w.topk, w.topp,
                        w.scale)
    t_ps = time.perf_counter() - t0
    mask = sel.mask.reshape(BH, nb, nb)
    last = N - (nb - 1) * bs
    rows_of = np.full(nb, float(bs))
    rows_of[-1] = last
    cols = mask.sum(axis=2) * bs - (bs - last) * mask[:, :, nb - 1]
    flops_block = 4.0 * d * rows_of[None, :] * cols  # [BH, nb]
    if qblocks is None:
        picks = [(h, i) for h in range(BH) for i in range(nb)]
    else:
        rng = np.random.default_rng(0)
        picks = sorted({(int(rng.integers(BH)), int(rng.integers(nb))) for _ in range(qblocks)})
    t0 = time.perf_counter()
    oracle.masked_attention(qf, kf, vf, mask, bs, w.scale, picks)
    t_att = time.perf_counter() - t0
    f_sample = float(sum(flops_block[h, i] for h, i in picks))
    f_call = float(flops_block.sum())
    ms_call = (t_ps + t_att * f_call / max(f_sample, 1.0)) * 1e3
    return {"workload": name, "threads": oracle.num_threads(), "full": qblocks is None,
            "pool_select_s": t_ps, "attention_s": t_att, "attention_query_blocks": len(picks),
            "ms_per_call": ms_call, "tflops": f_call / (ms_call * 1e-3) / 1e12}


def oracle_config_timings():
    """oracle_config_timing on every host core and, in a child process, on one core."""
    out = []
    for name, qb in ORACLE_CONFIGS:
        rec = oracle_config_timing(name, qb)
        env = dict(os.environ, OMP_NUM_THREADS="1")
        code = ("import json, bench; print(json.dumps(bench.oracle_config_timing(%r, %r)))"
                % (name, qb))
        try:
            res = subprocess.run([sys.executable, "-c", code], cwd=ROOT, env=env,
                                 capture_output=True, text=True, timeout=600)
            one = json.loads(res.stdout.strip().splitlines()[-1])
            rec["one_core"] = {"ms_per_call": one["ms_per_call"], "threads": one["threads"]}
        except Exception as e:  # noqa: BLE001 - a missing one-core time is reported, not fatal
            rec["one_core"] = {"error": str(e)[:200]}
        out.append(rec)
    return out


def run_reference(args, w):
    """--impl reference: the oracle, as it stands, on the host cores."""
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    from block_sparse_attention_blocks_b200 import workloads as W

    q, k, v = W.make_qkv(w)
    # warm-up and timed steps; one step = pool + select of one head in full and masked attention
    # of two seeded query blocks of that head (a bounded sample of the call), extrapolated to the
    # whole call the way the GPU arm's cpu_baseline is: pool + select by heads, attention by the
    # executed-pair FLOPs (the call's FLOPs estimated from the sampled head's selection)
    BH = w.B * w.H

    def step(i):
        return oracle_sample(w, q, k, v, [i % BH], 2, seed=i)

    for i in range(args.warmup):
        step(i)
    samples = []
    t0 = time.perf_counter()
    for i in range(args.steps):
        samples.append(step(args.warmup + i))
    elapsed = time.perf_counter() - t0
    call_ms, call_flops = 0.0, 0.0
    for s in samples:
        flops_call = s["flops_heads"] * BH / s["heads"]
        ms, _ = cpu_estimate(w, s, flops_call)
        call_ms += ms
        call_flops += flops_call
    value = call_flops / (call_ms * 1e-3) / 1e12 if call_ms > 0 else 0.0
    threads = samples[0]["threads"] if samples else 0
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": call_ms / max(args.steps, 1), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, None),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": threads, "kind": "oracle",
                         "sample": "per step: fp64 pool + scores + hybrid selection of one head "
                                   "in full, then masked attention of two seeded query blocks of "
                                   "that head, extrapolated to the whole call (pool + select by "
                                   "heads, attention by executed-pair FLOPs); ms_per_step is the "
                                   "extrapolated call, the sampled work took "
                                   f"{elapsed * 1e3 / max(args.steps, 1):.0f} ms per step"},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(w, extra):
    tensor_mb = w.B * w.H * w.N * w.d * 2 / 1e6
    c = {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "block": w.bs,
         "topk": w.topk, "topp": w.topp,
         "latent_grid": list(w.grid),
         "l2": (f"inputs larger than L2: Q, K, V are {tensor_mb:.0f} MB each (L2 "
                f"{L2_BYTES / 2**20:.0f} MiB); pooling streams Q and K every step"
                if tensor_mb * 1e6 > L2_BYTES else
                f"inputs fit in L2 ({tensor_mb:.1f} MB per tensor): a parity-size case, not the "
                f"bench line")}
    if extra:
        c.update(extra)
    return c


# ----------------------------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------------------------
def run_gpu(args, w):
    import torch

    world, rank, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import block_sparse_attention_blocks_b200 as bsa

    split = args.split == "heads" and world > 1
    q_np, k_np, v_np = make_inputs(w, rank, world, split_heads=split)
    if split:
        # this rank's heads, as one batch of len(heads) heads (the units never exchange data)
        from dataclasses import replace

        w_full = w
        w = replace(w, B=1, H=q_np.shape[1])
    as_bf16 = lambda a: torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16)
    q, k, v = (as_bf16(a).to(dev) for a in (q_np, k_np, v_np))
    B, H, N, d, bs, nb = w.B, w.H, w.N, w.d, w.bs, w.nb
    qp = torch.empty(B, H, nb, d, device=dev, dtype=torch.float32)
    kp = torch.empty_like(qp)
    mask = torch.empty(B, H, nb, nb, device=dev, dtype=torch.uint8)
    kv_idx = torch.empty(B, H, nb, nb, device=dev, dtype=torch.int32)
    kv_cnt = torch.empty(B, H, nb, device=dev, dtype=torch.int32)
    o = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        # pooling and selection in one call, then attention
        if ev is not None:
            ev[0].record(stream)
        bsa.pool_select_topk_topp(q, k, bs, w.topk, w.topp, qp=qp, kp=kp, mask=mask,
                                  kv_idx=kv_idx, kv_cnt=kv_cnt)
        if ev is not None:
            ev[1].record(stream)
        bsa.block_sparse_attn_fwd(q, k, v, kv_idx, kv_cnt, bs, o=o)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    err = bsa.device_error()
    if err:
        raise RuntimeError(f"device error {err} during warm-up")
    flops, pairs = executed_flops(kv_cnt, mask, N, d, bs)
    density = pairs / float(B * H * nb * nb)
    # FLOPs of the whole job per step: every rank's own call (replicas), or the sum of the
    # ranks' slices of one call (head split)
    job_flops = sum_over_ranks(flops, dev) if split else world * flops

    # ---------------------------------------------------------------- timed region
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.3)  # let the sampler attach before the work starts
    start.record(stream)
    for i in range(args.steps):
        step(evs[i])
    end.record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    ms_total = start.elapsed_time(end)
    t_ps = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    t_att = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    ms_total = max_over_ranks(ms_total, dev)
    ms_step = ms_total / args.steps
    err = bsa.device_error()
    if err:
        raise RuntimeError(f"device error {err} in the timed region")

    # ---------------------------------------------------------------- end to end from the host
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (as_bf16(a).pin_memory() for a in (q_np, k_np, v_np))
        oh = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
        e2e_steps = max(1, min(args.steps, args.e2e_steps))

        def e2e_step():
            # the public call with host tensors: heads in chunks, copies overlapping kernels
            bsa.sparse_attention(qh, kh, vh, bs, w.topk, w.topp, out=oh)

        e2e_step()
        torch.cuda.synchronize(dev)
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        s2.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e2.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = max_over_ranks(s2.elapsed_time(e2) / e2e_steps, dev)
        nbytes = q.numel() * 2
        e2e = {"value": job_flops / (ms_e2e * 1e-3) / 1e12, "unit": "TFLOPS",
               "ms_per_step": ms_e2e, "steps": e2e_steps,
               "h2d_bytes_per_step": 3 * nbytes, "d2h_bytes_per_step": nbytes,
               "path": "bsa.sparse_attention on pinned host Q,K,V: 8 head chunks, each copied "
                       "in, pooled/selected/attended through the C ABI and copied out, copies "
                       "overlapping the other chunks' kernels; O into pinned host memory"}

    # ---------------------------------------------------------------- dense control (context)
    dense = None
    if not args.no_dense and rank == 0:
        od = torch.empty_like(q)
        bsa.dense_attn_fwd(q, k, v, o=od)
        torch.cuda.synchronize(dev)
        sd, ed = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sd.record(stream)
        for _ in range(args.dense_steps):
            bsa.dense_attn_fwd(q, k, v, o=od)
        ed.record(stream)
        torch.cuda.synchronize(dev)
        ms_d = sd.elapsed_time(ed) / args.dense_steps
        ld = float(N - (nb - 1) * bs)
        dense_flops = 4.0 * d * N * N * B * H
        dense = {"ms": ms_d, "tflops": dense_flops / (ms_d * 1e-3) / 1e12,
                 "sparse_call_speedup": ms_d / ms_step}
        del od

    # ---------------------------------------------------------------- static pattern (context)
    static = None
    if not args.no_static and rank == 0:
        # every head: a diagonal band of half-width 7 blocks plus the first 16 key blocks (a
        # vertical stripe), about the realized density of the hybrid selection at this shape
        pats = [(5, 7, 0, 16)] * H
        ms_, ix_, ct_ = bsa.static_mask(pats, B, nb, device=dev)
        bsa.block_sparse_attn_fwd(q, k, v, ix_, ct_, bs, o=o)
        torch.cuda.synchronize(dev)
        s0, s1, s2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        reps = 5
        s0.record(stream)
        for _ in range(reps):
            bsa.static_mask(pats, B, nb, device=dev, mask=ms_, kv_idx=ix_, kv_cnt=ct_)
        s1.record(stream)
        for _ in range(reps):
            bsa.block_sparse_attn_fwd(q, k, v, ix_, ct_, bs, o=o)
        s2.record(stream)
        torch.cuda.synchronize(dev)
        f_st, p_st = executed_flops(ct_, ms_, N, d, bs)
        ms_att = s1.elapsed_time(s2) / reps
        static = {"pattern": "per head: |i - j| <= 7 blocks, or j < 16 (band + vertical stripe)",
                  "density": p_st / float(B * H * nb * nb), "mask_ms": s0.elapsed_time(s1) / reps,
                  "attention_ms": ms_att, "attention_tflops": f_st / (ms_att * 1e-3) / 1e12}
        del ms_, ix_, ct_

    # ---------------------------------------------------------------- SQuad (context)
    squad = None
    wsz = int(w.grid[1] * w.grid[2])  # tokens of one latent frame
    if not args.no_squad and rank == 0 and N % wsz == 0:
        osq = torch.empty_like(q)
        bsa.squad_attn_fwd(q, k, v, wsz, o=osq)
        torch.cuda.synchronize(dev)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 3
        s0.record(stream)
        for _ in range(reps):
            bsa.squad_attn_fwd(q, k, v, wsz, o=osq)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        ms_sq = s0.elapsed_time(s1) / reps
        # each query meets the wsz keys of its window, then the N / wsz keys at its position
        f_sq = 4.0 * d * N * (wsz + N // wsz) * B * H
        squad = {"window_tokens": wsz, "windows": N // wsz, "ms": ms_sq,
                 "tflops": f_sq / (ms_sq * 1e-3) / 1e12,
                 "pattern": "local pass within each latent frame, global pass across frames at "
                            "each position (SQuad, w = tokens of one frame)"}
        del osq

    # ---------------------------------------------------------------- (k, p) sweep
    sweep = None
    if not args.no_sweep and rank == 0 and w.sweep:
        peaks_s, _ = load_peaks()
        peak_s = peaks_s.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        sweep = []
        for topk, topp in w.sweep:
            sm_, si_, sc_ = (torch.empty_like(t) for t in (mask, kv_idx, kv_cnt))
            bsa.pool_select_topk_topp(q, k, bs, topk, topp, qp=qp, kp=kp, mask=sm_, kv_idx=si_,
                                      kv_cnt=sc_)
            bsa.block_sparse_attn_fwd(q, k, v, si_, sc_, bs, o=o)
            torch.cuda.synchronize(dev)
            s0, s1, s2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            reps = 5
            s0.record(stream)
            for _ in range(reps):
                bsa.pool_select_topk_topp(q, k, bs, topk, topp, qp=qp, kp=kp, mask=sm_,
                                          kv_idx=si_, kv_cnt=sc_)
            s1.record(stream)
            for _ in range(reps):
                bsa.block_sparse_attn_fwd(q, k, v, si_, sc_, bs, o=o)
            s2.record(stream)
            torch.cuda.synchronize(dev)
            f_s, p_s = executed_flops(sc_, sm_, N, d, bs)
            ms_a = s1.elapsed_time(s2) / reps
            tf = f_s / (ms_a * 1e-3) / 1e12
            sweep.append({"topk": topk, "topp": topp, "density": p_s / float(B * H * nb * nb),
                          "pool_select_ms": s0.elapsed_time(s1) / reps, "attention_ms": ms_a,
                          "attention_tflops": tf, "frac_of_burst_peak": tf / peak_s})
            del sm_, si_, sc_
        err = bsa.device_error()
        if err:
            raise RuntimeError(f"device error {err} in the sweep")

    # ---------------------------------------------------------------- SVG2 (context)
    svg2 = None
    if not args.no_svg2 and rank == 0:
        Cq, Ck = args.svg2_clusters
        # first centroid cache: the tokens at evenly spaced positions of each head; every later
        # call starts from the previous call's centroids (the cache of SVG2 section C)
        cq = q[:, :, torch.linspace(0, N - 1, Cq, device=dev).long(), :].float().contiguous()
        ck = k[:, :, torch.linspace(0, N - 1, Ck, device=dev).long(), :].float().contiguous()
        osv = torch.empty_like(q)
        ws = torch.empty(int(bsa.lib.sa_svg2_workspace_bytes(B, H, N, d, Cq, Ck)),
                         dtype=torch.uint8, device=dev)
        _, sel = bsa.svg2_attn_fwd(q, k, v, cq, ck, args.svg2_iters, w.topp, o=osv, workspace=ws)
        torch.cuda.synchronize(dev)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        reps = 5
        ev[0].record(stream)
        for _ in range(reps):
            bsa.svg2_attn_fwd(q, k, v, cq, ck, args.svg2_iters, w.topp, o=osv, sel=sel,
                              workspace=ws)
        ev[1].record(stream)
        # the stages of one call, through their own entry points: the two k-means (from copies
        # of the cache), the centroid top-p, the attention over the selected clusters (cluster
        # tables, permuted copies and the variable-length attention kernel)
        cq2, ck2 = cq.clone(), ck.clone()
        for _ in range(reps):
            cq2.copy_(cq)
            ck2.copy_(ck)
            aq, _, _, qsz = bsa.kmeans(q, cq2, args.svg2_iters)
            ak, _, _, ksz = bsa.kmeans(k, ck2, args.svg2_iters)
        ev[2].record(stream)
        for _ in range(reps):
            sel2 = bsa.centroid_topp(cq2, ck2, ksz, w.topp)
        ev[3].record(stream)
        for _ in range(reps):
            bsa.cluster_attn_fwd(q, k, v, aq, ak, sel2, o=osv)
        ev[4].record(stream)
        torch.cuda.synchronize(dev)
        err = bsa.device_error()
        if err:
            raise RuntimeError(f"device error {err} in the SVG2 timing")
        qsz, ksz = qsz.double(), ksz.double()
        pairs_sv = float(torch.einsum("bha,bhaj,bhj->", qsz, sel2.double(), ksz))
        ms_sv = ev[0].elapsed_time(ev[1]) / reps
        ms_att_sv = ev[3].elapsed_time(ev[4]) / reps
        f_sv = 4.0 * d * pairs_sv
        # the nearest-centroid contraction of one k-means pass: 2 N C d per head
        km_flops = 2.0 * B * H * N * d * (Cq + Ck) * (args.svg2_iters + 1)
        ms_km = ev[1].elapsed_time(ev[2]) / reps
        svg2 = {"query_clusters": Cq, "key_clusters": Ck, "kmeans_iters": args.svg2_iters,
                "topp": w.topp, "ms": ms_sv, "density": pairs_sv / float(B * H * N * N),
                "tflops": f_sv / (ms_sv * 1e-3) / 1e12,
                "stages_ms": {"kmeans_q_and_k": ms_km,
                              "centroid_topp": ev[2].elapsed_time(ev[3]) / reps,
                              "cluster_attention": ms_att_sv},
                "kmeans_assign_tflops": km_flops / (ms_km * 1e-3) / 1e12,
                "cluster_attention_tflops": f_sv / (ms_att_sv * 1e-3) / 1e12,
                "pattern": "k-means of Q and K warm-started from the previous call's centroids, "
                           "centroid top-p, attention over the selected clusters (SVG2)"}
        del osv, ws, sel, sel2, cq2, ck2

    # ---------------------------------------------------------------- SparsePR (context)
    sparsepr = None
    if not args.no_sparsepr and rank == 0:
        m = min(args.sparsepr_probes, N)
        gen = torch.Generator(device="cpu").manual_seed(7)
        probes = torch.stack([torch.randperm(N, generator=gen)[:m].sort().values
                              for _ in range(B * H)]).to(torch.int32).reshape(B, H, m).to(dev)
        opr = torch.empty_like(q)
        wsp = torch.empty(int(bsa.lib.sa_sparsepr_workspace_bytes(B, H, N, d, m)),
                          dtype=torch.uint8, device=dev)
        bsa.sparsepr_attn_fwd(q, k, v, kv_idx, kv_cnt, probes, bs, o=opr, workspace=wsp)
        torch.cuda.synchronize(dev)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        s0.record(stream)
        for _ in range(reps):
            bsa.sparsepr_attn_fwd(q, k, v, kv_idx, kv_cnt, probes, bs, o=opr, workspace=wsp)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        err = bsa.device_error()
        if err:
            raise RuntimeError(f"device error {err} in the SparsePR timing")
        ms_pr = s0.elapsed_time(s1) / reps
        sparsepr = {"probes_per_head": m, "ms": ms_pr,
                    "correction_ms": ms_pr - t_att,
                    "pattern": "block-sparse attention at the workload's selection, the exact "
                               "outputs of m seeded probe rows per head, the per-head fp64 "
                               "least-squares fit of their residuals and the correction of every "
                               "row (SparsePR); correction_ms = ms - the sparse attention alone"}
        del opr, wsp, probes

    # ---------------------------------------------------------------- pool + select, L2 flushed
    ps_flushed = None
    if rank == 0:
        flush = torch.empty(512 * 2**20, dtype=torch.uint8, device=dev)
        tot = 0.0
        reps = 10
        for _ in range(reps):
            flush.zero_()
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            bsa.pool_select_topk_topp(q, k, bs, w.topk, w.topp, qp=qp, kp=kp, mask=mask,
                                      kv_idx=kv_idx, kv_cnt=kv_cnt)
            f1.record(stream)
            torch.cuda.synchronize(dev)
            tot += f0.elapsed_time(f1)
        ps_flushed = tot / reps
        del flush

    peaks, peak_src = load_peaks()
    # the attention kernel is timed alone in a short region: the burst GEMM figure is its peak
    peak_tc = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_tc_s = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    att_tflops = flops / (t_att * 1e-3) / 1e12
    ps_bytes = (2 * q.numel() * 2 + 2 * qp.numel() * 4            # pool: read Q,K, write Qp,Kp
                + 2 * qp.numel() * 4 + mask.numel()                 # select: read Qp,Kp, mask
                + 4 * (kv_cnt.numel() + pairs))                     # kv_cnt + kept ids
    ps_gbs = ps_bytes / (t_ps * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": job_flops / (ms_step * 1e-3) / 1e12,
        "unit": "TFLOPS",
        "n_gpus": world, "steps": args.steps, "warmup": max(args.warmup, 3),
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "strong" if split else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": config_dict(w_full if split else w, {
            **({"parallelism": f"heads split over {world} ranks ({H} heads on rank 0)"} if split
               else {"parallelism": f"{world} independent replicas" if world > 1 else "1 GPU"}),
            "realized_density": density, "executed_pairs": pairs,
                                  "effective_flops_per_call": flops}),
        "roofline": {"kernel": "attn_fwd_kernel<128,128,BlockWalk>", "bound": "tensor",
                     "achieved": att_tflops, "peak": peak_tc, "unit": "TFLOP/s",
                     "frac": att_tflops / peak_tc,
                     "traffic": attention_traffic(w.name, B * H, pairs),
                     "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one "
                                       "full-size launch (profiles/attn_fwd_kernel_wan14b_720p_"
                                       "traffic.txt); null when the kernel changed since",
                     "peak_source": f"bf16_tflops (burst cuBLAS GEMM) of {peak_src}",
                     "frac_of_sustained_peak": att_tflops / peak_tc_s,
                     "algorithmic": "4*d*rows*cols per executed (query block, key block) pair, "
                                    "valid tokens only; x pairs per launch"},
        "roofline_pool_select": {"bound": "hbm", "achieved": ps_gbs, "peak": peak_hbm,
                                 "unit": "GB/s", "frac": ps_gbs / peak_hbm,
                                 "bytes_per_call": ps_bytes,
                                 "timed": "sa_pool_select_topk_topp: pooling, block scores "
                                          "and row selection kernels",
                                 "peak_source": f"hbm_gbs of {peak_src}",
                                 "frac_l2_flushed": (ps_bytes / (ps_flushed * 1e-3) / 1e9 / peak_hbm
                                                     if ps_flushed else None)},
        "kernels_ms": {"pool_select": t_ps, "attention": t_att,
                       "pool_select_l2_flushed": ps_flushed},
        "gpu_launches": launches_per_step(B * H) * args.steps,
        "clocks": clk,
    }
    if e2e:
        line["e2e"] = e2e
    if dense:
        line["dense_control"] = dense
    if static:
        line["static_pattern"] = static
    if squad:
        line["squad"] = squad
    if svg2:
        line["svg2"] = svg2
    if sparsepr:
        line["sparsepr"] = sparsepr
    if sweep:
        line["sweep"] = sweep

    # ---------------------------------------------------------------- oracle on the host
    if rank == 0 and world == 1 and not args.no_cpu:
        s = oracle_sample(w, q_np, k_np, v_np, heads=range(min(4, B * H)), qblocks_per_head=4)
        ms_cpu, tf_cpu = cpu_estimate(w, s, flops)
        line["cpu_baseline"] = {
            "value": tf_cpu, "unit": "TFLOPS", "cores": s["threads"], "kind": "oracle",
            "ms_per_call_extrapolated": ms_cpu,
            "sample": f"fp64 pool + scores + selection of {s['heads']} heads in full "
                      f"({s['t_pool_select']:.2f} s) and masked attention of {s['qblocks']} seeded "
                      f"query blocks ({s['t_attn']:.2f} s); extrapolated to the call by heads and "
                      f"by executed-pair FLOPs"}
        if not args.no_oracle_configs:
            line["cpu_baseline"]["other_workloads"] = oracle_config_timings()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("bsa", "reference"), default="bsa")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--topk", type=int, default=None)
    ap.add_argument("--topp", type=float, default=None)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--dense-steps", type=int, default=3)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-static", action="store_true", help="skip the static-pattern timing")
    ap.add_argument("--no-squad", action="store_true", help="skip the SQuad timing")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the pool+select and attention timings at every (k, p) point of "
                         "the workload's sweep")
    ap.add_argument("--no-svg2", action="store_true",
                    help="skip the SVG2 path timing (k-means, centroid top-p, cluster attention)")
    ap.add_argument("--no-sparsepr", action="store_true",
                    help="skip the SparsePR timing (sparse attention + probe-fitted correction)")
    ap.add_argument("--sparsepr-probes", type=int, default=256,
                    help="probe query rows per head for the SparsePR timing")
    ap.add_argument("--no-oracle-configs", action="store_true",
                    help="skip the oracle timings on the other workloads")
    ap.add_argument("--svg2-clusters", type=lambda s: tuple(int(x) for x in s.split(",")),
                    default=(128, 256), help="query,key cluster counts for --svg2")
    ap.add_argument("--svg2-iters", type=int, default=2, help="k-means update steps for --svg2")
    ap.add_argument("--split", choices=("replicas", "heads"), default="replicas",
                    help="with several GPUs: every rank runs the whole call (replicas, weak "
                         "scaling) or the heads of one call are split across ranks (strong)")
    ap.add_argument("--heads", type=int, default=None,
                    help="run only the first H heads (small cases for profiling; not a bench line)")
    args = ap.parse_args()
    from block_sparse_attention_blocks_b200 import workloads as W

    w = W.get(args.workload)
    if args.topk is not None or args.topp is not None:
        w = w.with_selection(args.topk if args.topk is not None else w.topk,
                             args.topp if args.topp is not None else w.topp)
    if args.heads is not None:
        from dataclasses import replace

        w = replace(w, H=args.heads, sink_heads=tuple(h for h in w.sink_heads if h < args.heads))
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
