"""Benchmark of the MaskLLM mask sampler's hot path on B200.

One step = every block of every weight matrix of the workload gets one forward (noise, soft
index, soft mask, W.M, regulariser) and one backward + AdamW, as in one training step of
the method. Default loop ("fused"): the forward of step 0 runs once before timing; then per
step and per layer (in reverse order, as a backward pass visits them) one launch does step
t's backward + AdamW and, from the updated logits, step t+1's forward. "--loop separate"
times the unfused form: per step a forward launch per layer, then a backward + AdamW launch
per layer in reverse. Metric: blocks/s over whole steps (blocks = groups of M weights, each
with its C logits), whole job; plus each kernel's achieved HBM bandwidth against the
measured copy bandwidth.

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--loop fused|separate]
                  [--impl reference]
  python bench.py --mode masked_linear [--tokens T] [--steps K]
      (the sampler inside the frozen network's linear layers of a LLaMA-2-7B layer: fused
       mllm_masked_linear_* calls against the sampler calls + cuBLAS GEMMs)
  python bench.py --mode sparse_linear [--workload NAME] [--serve-nm 2:4|4:8] [--steps K --warmup W]
      (serving leg: the workload's matrices as packed hard masks, y = x W*^T per call for
       1, 8, 16, 32 and 64 tokens, against dense cuBLAS; one JSON line)

The training line also carries "extras": once-per-run calls timed over the whole stack
(mask statistics, mask difference, candidate code, prior from a given mask) and the
serving product on the stack's own learned masks.

Default workload: the full LLaMA-2-7B-shaped stack at 2:4 (32 layers x 7 matrices,
1,619,001,344 blocks; logits and AdamW moments resident in HBM, ~130 GB, plus the next
step's soft-masked weights of every layer, 13 GB). Under torchrun each rank runs its own
stack (weak scaling, disjoint global block ids); the only exchange is an all-reduce of the
step's regulariser sums.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "mask-sampling blocks/sec (fwd, fused bwd+Adam) and % of B200 HBM roofline"
UNIT = "blocks/s"
# algorithmic HBM bytes per block: fwd reads W + logits, writes X; bwd+Adam reads W, G,
# logits, m, v and writes logits, m, v; pack reads W + logits, writes values + metadata
# the fused kernel reads W, G, logits, m, v and writes logits, m, v and the next step's X
BYTES = {6: {"fwd": 40, "bwd": 160, "fused": 168, "pack": 36.5, "init": 80},
         70: {"fwd": 312, "bwd": 1712, "fused": 1728, "pack": 306, "init": 856}}
FALLBACK_HBM_GBS = 6650.0


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


FALLBACK_BF16_TFLOPS = 1590.0


def bf16_peak():
    """Dense bf16 tensor-core TFLOP/s (burst) and its kind."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


def tensor_stats(T, shapes_rows_cols, ms):
    """Prefill-sized products are bound by the tensor cores: the dense-equivalent rate
    2 T rows cols / time, against the 2:4 sparse peak, twice the dense bf16 peak (the
    nominal ratio of the sparse mode)."""
    flops = 2.0 * T * sum(r * c for r, c in shapes_rows_cols)
    peak, kind = bf16_peak()
    tf = flops / (ms / 1e3) / 1e12
    return {"tflops_dense_equiv": round(tf, 1), "tensor_peak_tflops": 2 * peak, "tensor_peak_kind": kind,
            "tensor_frac": round(tf / (2 * peak), 4)}


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.dev)], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        power = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        smax = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        # samples under load: power above the midpoint of the observed range
        if power and max(power) > min(power) + 50:
            thr = (max(power) + min(power)) / 2
            loaded = [s for s, p in zip(sm, power) if p >= thr]
        else:
            loaded = sm
        return {"sm_mhz": float(np.median(loaded or sm)), "sm_max_mhz": smax, "reasons": reasons,
                "samples": len(sm), "samples_under_load": len(loaded), "power_w_max": max(power) if power else None}


# ------------------------------------------------------------------------------ GPU arm

def gpu_arm(args, w):
    import torch
    import torch.distributed as dist
    import sparsity_mask_sampling_b200 as pkg

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pkg.lib()
    hbm_peak, peak_kind = peaks()
    fused = args.loop == "fused"

    from sparsity_mask_sampling_b200.stack import SamplerStack

    t0 = time.time()
    stack = SamplerStack(w, dev, rank, x_per_layer=fused)
    stack.prior_init(seed=0)
    torch.cuda.synchronize()
    log(f"[rank {rank}] stack ready: {stack.blocks:,} blocks, {torch.cuda.memory_allocated(dev)/1e9:.1f} GB, {time.time()-t0:.1f}s")

    # once-per-run rows: prior init (pack after the timed steps), timed on the device
    init_ms = time_once(lambda: stack.prior_init(seed=0))

    def reduce_all():
        if world > 1:
            dist.all_reduce(stack.reg, op=dist.ReduceOp.SUM)

    L = w.layers

    def step(t, ev=None, **kw):
        if fused:
            stack.step_fused(t, ev=ev, **kw)
        else:
            stack.step(t, ev=ev, **kw)

    # prologue (the first forward of a fused loop) and warm-up steps
    if fused:
        stack.forward_all(0)
    for t in range(args.warmup):
        step(t)
        reduce_all()
    torch.cuda.synchronize()

    # device-timed steps: every block gets one forward and one backward + AdamW per step
    if fused:
        evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(L)] for _ in range(args.steps)]
    else:
        evs = [{k: [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(L)]
                for k in ("fwd", "bwd")} for _ in range(args.steps)]
    sampler = ClockSampler(local) if rank == 0 else None
    if sampler:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for k in range(args.steps):
        step(args.warmup + k, ev=evs[k])
        reduce_all()
    end.record()
    torch.cuda.synchronize()
    elapsed_ms = start.elapsed_time(end)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    durs = {}
    if fused:
        durs["fused"] = [ev[l][0].elapsed_time(ev[l][1]) for ev in evs for l in range(L)]
    else:
        for name in ("fwd", "bwd"):
            durs[name] = [ev[name][l][0].elapsed_time(ev[name][l][1]) for ev in evs for l in range(L)]
    t_max = elapsed_ms
    if world > 1:
        tt = torch.tensor([elapsed_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        t_max = float(tt.item())
    ms_per_step = t_max / args.steps
    value = stack.blocks * world * args.steps / (t_max / 1e3)

    # the two unfused kernels, one pass over every layer each (reference timings)
    ref = standalone_timings(stack, L, 5000)

    # pack (once, after training), then the mask diagnostics, codec and transfer prior
    pack_ms = time_pack(stack)
    extras = time_extras(stack, hbm_peak)
    extras["sparse_linear"] = time_sparse_linear(stack, hbm_peak)

    # end-to-end: upstream gradients from pinned host memory, regulariser read back
    e2e = e2e_leg(args, stack, w, world, dist if world > 1 else None, dev, step, fused)

    blocks_per_layer = w.blocks_per_layer()
    fb = BYTES[w.C]
    stack_blocks = stack.blocks

    # the other workloads, each at its full shape: every call timed on its own
    if not args.no_configs:
        del stack
        torch.cuda.empty_cache()
        extras["configs"] = config_legs(args, dev, hbm_peak, cpu=(world == 1 and rank == 0 and not args.no_cpu_baseline))
        extras["masked_linear"] = masked_linear_leg(dev, hbm_peak, reps=args.config_reps)

    def kstats(ms_list, bpb, name):
        avg = float(np.mean(ms_list))
        gbs = blocks_per_layer * bpb / (avg / 1e3) / 1e9
        return {"kernel": name, "avg_launch_ms": round(avg, 4), "launches": len(ms_list),
                "blocks_per_launch": blocks_per_layer, "bytes_per_block": bpb,
                "achieved_gbs": round(gbs, 1), "frac": round(gbs / hbm_peak, 4)}

    kernels = {}
    if fused:
        kernels["bwd_adam_fwd"] = kstats(durs["fused"], fb["fused"],
                                         "bwd_adam_fwd_kernel: backward + AdamW of step t, forward of step t+1")
        dom = kernels["bwd_adam_fwd"]
        traffic = traffic_from_profile("bwd_adam_fwd", w)
    else:
        kernels["fwd"] = kstats(durs["fwd"], fb["fwd"], "fwd_kernel")
        kernels["bwd_adam"] = kstats(durs["bwd"], fb["bwd"], "bwd_adam_kernel")
        dom = kernels["bwd_adam"]
        traffic = traffic_from_profile("bwd", w)
    kernels["fwd_standalone"] = kstats(ref["fwd"], fb["fwd"], "fwd_kernel (first step of a loop)")
    kernels["bwd_adam_standalone"] = kstats(ref["bwd"], fb["bwd"], "bwd_adam_kernel (unfused)")
    kernels["pack_once"] = once_stats(pack_ms, stack_blocks, fb["pack"], hbm_peak)
    kernels["prior_init_once"] = once_stats(init_ms, stack_blocks, fb["init"], hbm_peak)
    roofline = {"bound": "hbm", "kernel": dom["kernel"], "achieved": dom["achieved_gbs"], "peak": hbm_peak,
                "unit": "GB/s", "frac": round(dom["achieved_gbs"] / hbm_peak, 4), "peak_kind": peak_kind,
                "bytes_per_block": dom["bytes_per_block"], "traffic": traffic}
    out = None
    if rank == 0:
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": config_of(w, world, args.loop),
            "roofline": roofline,
            "kernels": kernels,
            "extras": extras,
            "e2e": e2e,
            "gpu_launches": (1 if fused else 2) * L * args.steps * n_groups(w),
            "clocks": clocks,
        }
        if world == 1 and not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(w, target_s=args.cpu_seconds)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return out


def standalone_timings(stack, L, t):
    """Per-launch device time of the unfused forward and backward + AdamW, each run once
    over every layer (outside the timed steps)."""
    import torch

    hp = stack.hparams(t).to_c()
    out = {"fwd": [], "bwd": []}
    for name, fn in (("fwd", stack.forward), ("bwd", stack.backward)):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(L)]
        for l in range(L):
            evs[l][0].record()
            fn(l, hp)
            evs[l][1].record()
        torch.cuda.synchronize()
        out[name] = [a.elapsed_time(b) for a, b in evs]
    return out


def n_groups(w):
    return math.ceil(len(w.matrices) / 16)


def time_once(fn):
    import torch

    fn()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    fn()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e)


def time_pack(stack):
    import torch
    import sparsity_mask_sampling_b200 as pkg
    from sparsity_mask_sampling_b200 import buffers

    # packed outputs of one layer are reused across layers (the pack runs once; only its cost matters)
    w = stack.w
    outs = []
    for m in w.matrices:
        (vs, (ms, mdt)) = buffers.pack_shapes(m.rows, m.cols, w.nm)
        outs.append((torch.empty(vs, dtype=torch.bfloat16, device=stack.dev), torch.empty(ms, dtype=mdt, device=stack.dev),
                     torch.empty(m.rows * m.cols // w.nm[1], dtype=torch.uint8, device=stack.dev)))
    arrs = []
    for l in range(w.layers):
        for mb, (v, mt, ci) in zip(stack.bufs[l], outs):
            mb.pack_values, mb.pack_meta, mb.cand_idx = v, mt, ci
        arrs.append(pkg.MatrixArray(stack.bufs[l]))

    def go():
        for a in arrs:
            pkg.mllm_hard_pack(a, w.nm)
    return time_once(go)


def time_extras(stack, peak):
    """Once-per-run calls around training, timed over the whole stack on the device: mask
    statistics (Fig. 5b/6), mask difference between two hard masks (Fig. 5a/8), the
    candidate-index code, and a prior initialisation from a given mask (transfer)."""
    import torch
    import sparsity_mask_sampling_b200 as pkg

    w = stack.w
    L = w.layers
    dev = stack.dev
    B = stack.blocks
    out = {}
    stats = torch.zeros(4, dtype=torch.float64, device=dev)
    out["mask_stats_once"] = once_stats(
        time_once(lambda: [pkg.mllm_mask_stats(stack.view(l), w.nm, w.kappa[1], stats, stack.ws) for l in range(L)]),
        B, (16 if w.w_dtype == "f32" else 8) + 4 * w.C, peak)
    # the whole stack's hard masks as one array (each matrix's candidate indices a view at its
    # global block offset), so that the mask difference and the candidate code take one launch
    flat = torch.empty(B, dtype=torch.uint8, device=dev)
    base = stack.bufs[0][0].block_offset
    for mats in stack.bufs:
        for mb in mats:
            nb = mb.W.numel() // w.nm[1]
            mb.cand_idx = flat[mb.block_offset - base: mb.block_offset - base + nb]
        pkg.mllm_hard_pack(pkg.MatrixArray(mats), w.nm)
    idx = [mb.cand_idx for mb in stack.bufs[0]]
    other = torch.roll(flat, 1)
    cnt = torch.zeros(1, dtype=torch.int64, device=dev)
    out["mask_diff_once"] = once_stats(time_once(lambda: pkg.mllm_mask_diff(flat, other, cnt)), B, 2, peak)
    D = 12 if w.nm == (2, 4) else 5
    words = torch.empty((B + D - 1) // D, dtype=torch.int32, device=dev)
    out["encode_once"] = once_stats(time_once(lambda: pkg.mllm_encode_candidates(w.nm, flat, words)),
                                    B, 1 + 4.0 / D, peak)
    del other, words
    pri = [idx] * L
    arrs = [stack.view(l) for l in range(L)]
    out["prior_from_mask_once"] = once_stats(
        time_once(lambda: [pkg.mllm_prior_init_from_mask(arrs[l], w.nm, pri[l], w.alpha, w.init_std, 0) for l in range(L)]),
        B, 1 + 12 * w.C, peak)
    return out


def time_median(fn, reps=5):
    import torch

    fn()
    torch.cuda.synchronize()
    out = []
    for _ in range(reps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        fn()
        e.record()
        torch.cuda.synchronize()
        out.append(s.elapsed_time(e))
    return float(np.median(out))


def time_sparse_linear(stack, peak, token_counts=(1, 8, 16, 32, 64, 128, 512, 2048)):
    """Serving the learned sparse network (s.3.2, inference): y = x W*^T for every matrix of
    the stack from its own packed hard mask (one mllm_sparse_linear call for all of them: a
    launch per 16 matrices), as
    one decode step of T tokens through all linear layers, beside the same products with the
    dense bf16 weights through cuBLAS (torch.nn.functional.linear). Bytes are those of the
    compressed weights, metadata, activations and outputs; the packed stack (7.3 GB for
    LLaMA-2-7B at 2:4) is larger than L2, so every pass streams it from HBM."""
    import torch
    import torch.nn.functional as F
    import sparsity_mask_sampling_b200 as pkg
    from sparsity_mask_sampling_b200 import buffers

    w = stack.w
    if w.w_dtype != "bf16":
        return None
    dev = stack.dev
    L = w.layers
    packed = []
    for l in range(L):
        outs = []
        for mb, m in zip(stack.bufs[l], w.matrices):
            (vs, (ms, mdt)) = buffers.pack_shapes(m.rows, m.cols, w.nm)
            mb.pack_values = torch.empty(vs, dtype=torch.bfloat16, device=dev)
            mb.pack_meta = torch.empty(ms, dtype=mdt, device=dev)
            mb.cand_idx = None
            outs.append((mb.pack_values, mb.pack_meta))
        pkg.mllm_hard_pack(pkg.MatrixArray(stack.bufs[l]), w.nm)
        packed.append(outs)
    wbytes = sum(v.numel() * 2 + mt.numel() * mt.element_size() for outs in packed for v, mt in outs)
    dense_bytes = sum(mb.W.numel() * 2 for mats in stack.bufs for mb in mats)
    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    spl_ws = pkg.sparse_linear_workspace(dev)
    res = {"launches_per_pass": math.ceil(L * len(w.matrices) / 16), "compressed_weight_gb": round(wbytes / 1e9, 3)}
    for T in token_counts:
        xs = {c: torch.randn(T, c, device=dev, generator=gen).to(torch.bfloat16) for c in {m.cols for m in w.matrices}}
        ys = [torch.empty(T, m.rows, dtype=torch.float32, device=dev) for m in w.matrices]
        arr = pkg.SparseOperandArray([(v, mt, xs[m.cols], y) for l in range(L)
                                      for (v, mt), m, y in zip(packed[l], w.matrices, ys)])
        io = L * sum(T * m.cols * 2 + T * m.rows * 4 for m in w.matrices)
        ms = time_median(lambda: pkg.mllm_sparse_linear(arr, w.nm, T, spl_ws))
        ms_dense = time_median(lambda: [F.linear(xs[mb.W.shape[1]], mb.W) for mats in stack.bufs for mb in mats])
        gbs = (wbytes + io) / (ms / 1e3) / 1e9
        res[f"tokens_{T}"] = {
            "ms": round(ms, 4), "achieved_gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
            "dense_cublas_ms": round(ms_dense, 4),
            "dense_cublas_gbs": round((dense_bytes + io) / (ms_dense / 1e3) / 1e9, 1),
            "speedup_vs_dense": round(ms_dense / ms, 3)}
        if T > 64:
            res[f"tokens_{T}"].update(tensor_stats(T, [(m.rows, m.cols) for _ in range(L) for m in w.matrices], ms))
    for mats in stack.bufs:
        for mb in mats:
            mb.pack_values = mb.pack_meta = None
    del packed
    torch.cuda.empty_cache()
    return res


def once_stats(ms, blocks, bpb, peak):
    gbs = blocks * bpb / (ms / 1e3) / 1e9
    return {"ms": round(ms, 3), "blocks_per_s": blocks / (ms / 1e3), "achieved_gbs": round(gbs, 1),
            "frac": round(gbs / peak, 4)}


def e2e_leg(args, stack, w, world, dist, dev, step, fused):
    """Same steps through the public API with the step inputs on the host: each layer's
    upstream gradients are copied from pinned host memory (a copy stream, overlapped with
    the kernels), and the regulariser sums are read back to the host every step."""
    import torch

    L = w.layers
    host_g = []
    for p in range(2):
        host_g.append([g.cpu().pin_memory() for (_, g) in stack.pool[p]])
    h2d = sum(g.numel() * g.element_size() for (_, g) in stack.pool[0]) * L
    reg_host = torch.empty(L, dtype=torch.float64, pin_memory=True)
    d2h = reg_host.numel() * reg_host.element_size()
    main = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(dev)
    g_free = [torch.cuda.Event(), torch.cuda.Event()]
    for e in g_free:
        e.record(main)

    def copy_fn(l):
        p = l % 2
        with torch.cuda.stream(copy):
            copy.wait_event(g_free[p])
            for (_, g), hg in zip(stack.pool[p], host_g[p]):
                g.copy_(hg, non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(copy)
        main.wait_event(ready)

    steps = max(2, min(args.steps, 5))
    t0 = 2000
    if fused:
        stack.forward_all(t0 - 1)
    step(t0 - 1, g_free=g_free, copy_fn=copy_fn)
    reg_host.copy_(stack.reg, non_blocking=True)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for t in range(steps):
        step(t0 + t, g_free=g_free, copy_fn=copy_fn)
        if dist is not None:
            dist.all_reduce(stack.reg, op=dist.ReduceOp.SUM)
        reg_host.copy_(stack.reg, non_blocking=True)
        main.synchronize()
        _ = float(reg_host.sum())
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e)
    if dist is not None:
        tt = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt.item())
    return {"value": stack.blocks * world * steps / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": steps,
            "ms_per_step": ms / steps}


def config_of(w, world, loop="fused"):
    return {"workload": w.name, "loop": {"fused": "fused: per layer one launch of step t's backward + AdamW "
                                                  "with step t+1's forward (the first forward in the prologue)",
                                         "separate": "separate: per layer a forward launch, then a backward + "
                                                     "AdamW launch"}[loop], "nm": f"{w.nm[0]}:{w.nm[1]}", "layers": w.layers,
            "matrices_per_layer": len(w.matrices),
            "shapes_out_in": [[m.rows, m.cols] for m in w.matrices],
            "blocks_per_step_per_gpu": w.total_blocks(), "candidates": w.C,
            "weights": f"{w.w_dtype} ~N(0,{w.w_std}^2), {w.outlier_frac:.0%} outlier input channels x{w.outlier_scale:g}",
            "upstream_grad": f"{w.g_dtype} ~N(0,{w.g_std}^2)",
            "tau": list(w.tau), "kappa": list(w.kappa), "lr": w.lr, "lambda": w.lam,
            "launches": "one grouped launch per layer per kernel",
            "l2": "inputs larger than L2 (each launch streams >= 280 MB); no flush",
            "parallelism": f"dp{world} (independent shards)"}


def traffic_from_profile(kernel, w):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current
    source of the kernel (its sha256 is recorded there); otherwise None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    ent = d.get(f"{kernel}_{w.nm[0]}of{w.nm[1]}")
    if not ent or ent.get("source_sha256") != kernel_source_sha(w.nm):
        return None
    return ent["dram_bytes_per_block"] * w.blocks_per_layer()


def kernel_source_sha(nm=(2, 4)):
    """sha256 of the files that hold the sampler kernels' device code for a pattern (the
    shared device helpers and the pattern's kernel file)."""
    csrc = os.path.join(ROOT, "sparsity_mask_sampling_b200", "csrc")
    h = hashlib.sha256()
    for fn in ("device_common.cuh", "kernels_2of4.cuh" if nm == (2, 4) else "kernels_4of8.cuh"):
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# ------------------------------------------------------------------------------ other workloads

CONFIG_LEGS = ("tiny_2of4", "gpt3_843m_layer_2of4", "llama2_7b_layer_2of4", "general_4of8")


def config_legs(args, dev, peak, cpu=True):
    """Every workload other than the headline stack, at its full shape: the forward, the
    backward + AdamW, the fused step call (backward + AdamW of step t with the forward of
    step t+1) and the hard pack, each timed alone as the median of `reps` calls with CUDA
    events, L2 flushed (a 1 GB write) before every call. The tiny workload is reported as
    latency (us per call; no roofline claim at 2,048 blocks). Each workload carries the
    oracle's rates on the host cores for the same calls (all threads and 1 thread)."""
    from sparsity_mask_sampling_b200 import configs

    out = {}
    for name in CONFIG_LEGS:
        w = configs.WORKLOADS[name]
        out[name] = config_leg(w, dev, peak, reps=args.config_reps)
        if cpu:
            out[name]["cpu_baseline"] = cpu_kernel_rates(w, seconds=args.config_cpu_seconds)
    return out


def config_leg(w, dev, peak, reps=10):
    import torch
    import sparsity_mask_sampling_b200 as pkg
    from sparsity_mask_sampling_b200 import buffers
    from sparsity_mask_sampling_b200.stack import SamplerStack

    stack = SamplerStack(w, dev, x_per_layer=True)
    stack.prior_init(seed=0)
    for mats in stack.bufs:
        for mb, m in zip(mats, w.matrices):
            (vs, (ms, mdt)) = buffers.pack_shapes(m.rows, m.cols, w.nm)
            mb.pack_values = torch.empty(vs, dtype=mb.W.dtype, device=dev)
            mb.pack_meta = torch.empty(ms, dtype=mdt, device=dev)
            mb.cand_idx = torch.empty(m.rows * m.cols // w.nm[1], dtype=torch.uint8, device=dev)
    stack.rebuild_views()
    flush = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    L = w.layers
    t = 5  # a step inside the schedule
    hp, hpn = stack.hparams(t).to_c(), stack.hparams(t + 1).to_c()
    calls = {
        "fwd": lambda: [stack.forward(l, hp) for l in range(L)],
        "bwd_adam": lambda: [stack.backward(l, hp) for l in range(L)],
        "bwd_adam_fwd": lambda: [stack.backward_forward(l, hp, hpn) for l in range(L)],
        "pack": lambda: [pkg.mllm_hard_pack(stack.view(l), w.nm) for l in range(L)],
    }
    fb = BYTES[w.C]
    bpb = {"fwd": fb["fwd"], "bwd_adam": fb["bwd"], "bwd_adam_fwd": fb["fused"], "pack": fb["pack"]}
    if w.w_dtype == "f32":  # fp32 W, X and G: 8 more bytes per block for each of them
        bpb = {"fwd": 56, "bwd_adam": 176, "bwd_adam_fwd": 192, "pack": 50.5}
    blocks = stack.blocks
    res = {"blocks": blocks, "nm": f"{w.nm[0]}:{w.nm[1]}", "reps": reps,
           "timing": "median of the reps, each call alone on the device after a 1 GB L2 flush"}
    for k, fn in calls.items():
        fn()
        torch.cuda.synchronize()
        ms_list = []
        for _ in range(reps):
            flush.zero_()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            fn()
            e.record()
            torch.cuda.synchronize()
            ms_list.append(s.elapsed_time(e))
        ms = float(np.median(ms_list))
        gbs = blocks * bpb[k] / (ms / 1e3) / 1e9
        ent = {"ms": round(ms, 4), "blocks_per_s": blocks / (ms / 1e3), "bytes_per_block": bpb[k],
               "achieved_gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
        if blocks < 1e5:
            ent = {"us": round(ms * 1e3, 2), "blocks_per_s": blocks / (ms / 1e3), "bytes_per_block": bpb[k],
                   "note": "latency: launch-bound at this size, no roofline claim"}
        res[k] = ent
    del stack, flush
    torch.cuda.empty_cache()
    return res


def masked_linear_leg(dev, peak, tokens=256, reps=10, bwd_tokens=2048):
    """The sampler inside the frozen network's linear layers (s.3.2 "Frozen LLM Backbone"), on
    the LLaMA-2-7B layer's seven matrices at `tokens` tokens (seeded synthetic activations A
    and output gradients dY, bf16). Fused: mllm_masked_linear_fwd (Y = A X^T with X made in
    shared memory) and mllm_masked_linear_bwd_adam (G = dY^T A in tensor memory, then the
    logits' backward + AdamW from it). Unfused, on the same box: mllm_sample_fwd writes X, then
    cuBLAS Y = A X^T (torch F.linear); cuBLAS G = dY^T A (bf16 out), then mllm_sample_bwd_adam
    reads it. Each call timed alone (median of reps, CUDA events, L2 flushed before each)."""
    import torch
    import torch.nn.functional as F
    import sparsity_mask_sampling_b200 as pkg
    from sparsity_mask_sampling_b200 import configs, inputs

    w = configs.WORKLOADS["llama2_7b_layer_2of4"]
    mats, ios_f, ios_b, As, dYs = [], [], [], [], []
    off = 0
    for i, m in enumerate(w.matrices):
        W = inputs.weights(m.rows, m.cols, "bf16", 0.02, seed=100 + i, outlier_frac=0.01, device=dev)
        mb = pkg.alloc_matrix(W, (2, 4), off, fwd=True, bwd=True)
        mb.logits.copy_(inputs.logits(m.rows * m.cols // 4, 6, 0.02, seed=200 + i, device=dev))
        A = inputs.weights(tokens, m.cols, "bf16", 1.0, seed=300 + i, device=dev)
        dY = inputs.upstream_grad(tokens, m.rows, "bf16", 1e-3, seed=400 + i, device=dev)
        y = torch.empty(tokens, m.rows, dtype=torch.float32, device=dev)
        mats.append(mb)
        ios_f.append((A, y, None))
        ios_b.append((A, None, dY))
        As.append(A)
        dYs.append(dY)
        off += m.rows * m.cols // 4
    arr = pkg.MatrixArray(mats)
    fused_mats = [pkg.MatrixBuffers(W=mb.W, logits=mb.logits, adam_m=mb.adam_m, adam_v=mb.adam_v,
                                    block_offset=mb.block_offset) for mb in mats]
    farr = pkg.MatrixArray(fused_mats)
    mlws = pkg.masked_linear_workspace(dev)
    ws = torch.zeros(pkg.mllm_workspace_bytes(), dtype=torch.uint8, device=dev)
    reg = torch.zeros(1, dtype=torch.float64, device=dev)
    hp = pkg.Hparams(kappa=300.0, tau=1.0, lambda_=1e-5, lr=5e-4, adam_step=5, step=4, seed=0)
    flush = torch.empty(1 << 30, dtype=torch.uint8, device=dev)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        out = []
        for _ in range(reps):
            flush.zero_()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            fn()
            e.record()
            torch.cuda.synchronize()
            out.append(s.elapsed_time(e))
        return float(np.median(out))

    def unfused_fwd():
        pkg.mllm_sample_fwd(arr, (2, 4), hp, reg, ws)
        for mb, (A, y, _) in zip(mats, ios_f):
            y.copy_(F.linear(A, mb.X))

    def unfused_bwd():
        for mb, A, dY in zip(mats, As, dYs):
            torch.matmul(dY.t(), A, out=mb.G)
        pkg.mllm_sample_bwd_adam(arr, (2, 4), hp)

    t = {
        "fused_fwd_ms": timed(lambda: pkg.mllm_masked_linear_fwd(farr, ios_f, (2, 4), tokens, hp, mlws, reg)),
        "unfused_fwd_ms": timed(unfused_fwd),
        "fused_bwd_adam_ms": timed(lambda: pkg.mllm_masked_linear_bwd_adam(farr, ios_b, (2, 4), tokens, hp, mlws)),
        "unfused_bwd_adam_ms": timed(unfused_bwd),
    }
    blocks = w.blocks_per_layer()
    flops = 2.0 * tokens * blocks * 4  # one product per weight per token
    res = {"workload": w.name, "tokens": tokens, "blocks": blocks,
           "timing": "median of the reps, each call alone after a 1 GB L2 flush"}
    for k, v in t.items():
        res[k] = round(v, 4)
    res["fwd_speedup"] = round(t["unfused_fwd_ms"] / t["fused_fwd_ms"], 3)
    res["bwd_adam_speedup"] = round(t["unfused_bwd_adam_ms"] / t["fused_bwd_adam_ms"], 3)
    # The backward sums over the tokens (its MMA's K), so one call takes a whole sequence:
    # the same two backward plans at bwd_tokens tokens.
    if bwd_tokens and bwd_tokens != tokens:
        ios_l, As_l, dYs_l = [], [], []
        for i, m in enumerate(w.matrices):
            A = inputs.weights(bwd_tokens, m.cols, "bf16", 1.0, seed=500 + i, device=dev)
            dY = inputs.upstream_grad(bwd_tokens, m.rows, "bf16", 1e-3, seed=600 + i, device=dev)
            ios_l.append((A, None, dY))
            As_l.append(A)
            dYs_l.append(dY)

        def unfused_bwd_l():
            for mb, A, dY in zip(mats, As_l, dYs_l):
                torch.matmul(dY.t(), A, out=mb.G)
            pkg.mllm_sample_bwd_adam(arr, (2, 4), hp)

        fb = timed(lambda: pkg.mllm_masked_linear_bwd_adam(farr, ios_l, (2, 4), bwd_tokens, hp, mlws))
        ub = timed(unfused_bwd_l)
        res["bwd_tokens"] = bwd_tokens
        res["fused_bwd_adam_ms_at_bwd_tokens"] = round(fb, 4)
        res["unfused_bwd_adam_ms_at_bwd_tokens"] = round(ub, 4)
        res["bwd_adam_speedup_at_bwd_tokens"] = round(ub / fb, 3)
    # HBM bytes per block and step. Fused: forward reads W + logits (32), backward reads W and
    # logits/m/v and writes logits/m/v (152). Unfused as timed here: sampler forward 40 + the
    # GEMM's read of X 8, the GEMM's write of G 8 + sampler backward 160. (A loop built on the
    # sampler's own fused step, which reads W and the logits once per step, moves 168 + 16 =
    # 184, as the fused layer does; what the fused layer saves there is the X and G buffers.)
    res["hbm_bytes_per_block_per_step"] = {"fused": 32 + 152, "unfused_as_timed": 48 + 168,
                                           "unfused_with_fused_sampler_step": 168 + 16}
    res["bytes_saved_per_block_per_step"] = 48 + 168 - (32 + 152)
    res["buffers_not_held_gb_per_layer"] = round(blocks * 16 / 1e9, 3)  # X and G, bf16
    res["fused_fwd_tflops"] = round(flops / (t["fused_fwd_ms"] / 1e3) / 1e12, 1)
    res["fused_fwd_gbs"] = round(blocks * 32 / (t["fused_fwd_ms"] / 1e3) / 1e9, 1)
    res["fused_bwd_adam_gbs"] = round(blocks * 152 / (t["fused_bwd_adam_ms"] / 1e3) / 1e9, 1)
    del mats, fused_mats, arr, farr, flush
    torch.cuda.empty_cache()
    return res


def _rate(fn, samples, threads):
    start = time.perf_counter()
    with cf.ThreadPoolExecutor(threads) as ex:
        list(ex.map(fn, samples))
    return time.perf_counter() - start


def cpu_kernel_rates(w, seconds=1.0):
    """The oracle's forward, backward + AdamW and hard pack on the host cores (all threads,
    then 1 thread), each on a bounded random sample of the workload's blocks sized to take
    about `seconds`; blocks/s per call."""
    import oracle as orc

    orc.build()
    n, m = w.nm
    t = 5
    kappa, tau = w.kappa_at(t % w.steps), w.tau_at(t % w.steps)

    def fwd(s):
        gids, W, G, pi = s
        orc.sample_fwd(n, m, W, pi, gids, kappa, tau, 0, t)

    def bwd(s):
        gids, W, G, pi = s
        g, _ = orc.sample_bwd(n, m, W, G, pi, gids, kappa, tau, w.lam, 0, t)
        z = np.zeros_like(g)
        orc.adamw(pi, z, z, g, w.lr, 0.9, 0.999, 1e-8, w.weight_decay, t + 1)

    def pack(s):
        gids, W, G, pi = s
        raw = np.ascontiguousarray(W.astype(np.float32)).view(np.uint32).reshape(-1, 8 * m)
        orc.hard_pack(n, m, raw, pi)

    threads = os.cpu_count() or 1
    out = {"cores": threads, "kind": "oracle", "unit": "blocks/s"}
    for name, fn in (("fwd", fwd), ("bwd_adam", bwd), ("pack", pack)):
        probe = [make_sample(w, 2048, seed=31)]
        dt = max(_rate(fn, probe, 1), 1e-6)
        per_thread = int(min(max(2048 / dt * seconds, 2048), 4e6)) // 8 * 8
        samples = [make_sample(w, per_thread, seed=41 + i) for i in range(threads)]
        dt_n = _rate(fn, samples, threads)
        dt_1 = _rate(fn, samples[:1], 1)
        out[name] = {"value": per_thread * threads / dt_n, "value_1_core": per_thread / dt_1}
    out["sample"] = (f"per call and thread count, random blocks of {w.name} (same seeded distributions), "
                     f"sized for about {seconds:g} s per thread")
    return out


# ------------------------------------------------------------------------------ CPU (oracle)

def make_sample(w, n_blocks, seed=0):
    """A bounded sample of the workload's blocks: their global ids, weights, logits and
    upstream gradients (seeded, same distributions as the GPU workload)."""
    import torch
    from sparsity_mask_sampling_b200 import inputs

    rng = np.random.default_rng(seed)
    gids = rng.integers(0, w.total_blocks(), size=n_blocks, dtype=np.uint64)
    M = w.nm[1]
    W = inputs.weights(n_blocks, M, w.w_dtype, w.w_std, seed=seed).float().double().numpy()
    G = inputs.upstream_grad(n_blocks, M, w.g_dtype, w.g_std, seed=seed + 1).float().double().numpy()
    pi = inputs.logits(n_blocks, w.C, 0.02, seed=seed + 2).numpy()
    return gids, W, G, pi


def oracle_step(orc, w, sample, t):
    """The oracle on one sample for one step: forward, backward, AdamW."""
    gids, W, G, pi = sample
    kappa, tau = w.kappa_at(t % w.steps), w.tau_at(t % w.steps)
    n, m = w.nm
    orc.sample_fwd(n, m, W, pi, gids, kappa, tau, 0, t)
    g, _ = orc.sample_bwd(n, m, W, G, pi, gids, kappa, tau, w.lam, 0, t)
    z = np.zeros_like(g)
    orc.adamw(pi, z, z, g, w.lr, 0.9, 0.999, 1e-8, w.weight_decay, t + 1)


def cpu_run(w, n_blocks, threads, steps, t0=0):
    import oracle as orc

    orc.build()
    per = max(1, n_blocks // threads)
    samples = [make_sample(w, per, seed=17 + i) for i in range(threads)]
    start = time.perf_counter()
    with cf.ThreadPoolExecutor(threads) as ex:
        for t in range(steps):
            list(ex.map(lambda s: oracle_step(orc, w, s, t0 + t), samples))
    return time.perf_counter() - start, per * threads


def cpu_baseline(w, target_s=15.0):
    threads = os.cpu_count() or 1
    dt, n = cpu_run(w, 2000 * threads, threads, 1)
    rate = n / dt
    n_blocks = int(min(max(rate * target_s, 1000 * threads), 5e7))
    dt, n = cpu_run(w, n_blocks, threads, 1)
    # the same on one core, on a sample of ~2 s
    dt1, n1 = cpu_run(w, max(1000, int(rate / threads * 2.0)), 1, 1)
    return {"value": n / dt, "unit": UNIT, "cores": threads, "kind": "oracle",
            "value_1_core": n1 / dt1,
            "sample": f"{n:,} blocks drawn from {w.name} (random global ids; weights, logits and "
                      f"gradients from the same seeded distributions), one forward + backward + "
                      f"AdamW step, {dt:.1f} s on {threads} threads; value_1_core: {n1:,} blocks, "
                      f"{dt1:.1f} s on 1 thread"}


def reference_arm(args, w):
    """The oracle as it stands on the host cores: each step runs the oracle's forward,
    backward and AdamW on a bounded sample of the workload's blocks."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    threads = os.cpu_count() or 1
    dt, n = cpu_run(w, 2000 * threads, threads, 1)
    per_step = int(min(max(n / dt * args.ref_step_seconds, 1000 * threads), 5e7))
    cpu_run(w, per_step, threads, args.warmup)
    dt, n = cpu_run(w, per_step, threads, args.steps, t0=args.warmup)
    value = n * args.steps / dt
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, 1, args.loop), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{n:,} blocks per step drawn from {w.name}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def sparse_linear_arm(args, w):
    """--mode sparse_linear: serving the learned sparse network (s.3.2, inference). Every
    matrix of the workload as a packed hard-masked bf16 weight; one pass = y = x W*^T for all
    of them (one mllm_sparse_linear call, a launch per 16 matrices) for T = 1-64 tokens, timed per
    call with CUDA events (median of --steps calls after --warmup), beside the same products
    with dense bf16 weights through cuBLAS (torch.nn.functional.linear)."""
    import torch
    import torch.nn.functional as F
    import sparsity_mask_sampling_b200 as pkg

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    pkg.lib()
    hbm_peak, peak_kind = peaks()
    from sparsity_mask_sampling_b200 import inputs

    gen = torch.Generator(device=dev)
    gen.manual_seed(0)
    shapes = [(m.rows, m.cols) for _ in range(w.layers) for m in w.matrices]
    packed = [inputs.packed_hard_mask(r, c, w.nm, seed=1000 + i, device=dev) for i, (r, c) in enumerate(shapes)]
    dense = [torch.randn(r, c, device=dev, generator=gen).to(torch.bfloat16) for r, c in shapes]
    wbytes = sum(v.numel() * 2 + mt.numel() * mt.element_size() for v, mt in packed)
    dbytes = sum(d.numel() * 2 for d in dense)
    ws = pkg.sparse_linear_workspace(dev)

    def med(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        out = []
        for _ in range(args.steps):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            fn()
            e.record()
            torch.cuda.synchronize()
            out.append(s.elapsed_time(e))
        return float(np.median(out))

    res = {}
    for T in (1, 8, 16, 32, 64, 128, 512, 2048):
        xs = {c: torch.randn(T, c, device=dev, generator=gen).to(torch.bfloat16) for c in {c for _, c in shapes}}
        ys = [torch.empty(T, r, dtype=torch.float32, device=dev) for r, _ in shapes]
        arr = pkg.SparseOperandArray([(v, mt, xs[c], y) for (v, mt), (r, c), y in zip(packed, shapes, ys)])
        io = sum(T * c * 2 + T * r * 4 for r, c in shapes)
        ms = med(lambda: pkg.mllm_sparse_linear(arr, w.nm, T, ws))
        ms_d = med(lambda: [F.linear(xs[d.shape[1]], d) for d in dense])
        gbs = (wbytes + io) / (ms / 1e3) / 1e9
        res[f"tokens_{T}"] = {"ms": round(ms, 4), "achieved_gbs": round(gbs, 1), "frac": round(gbs / hbm_peak, 4),
                              "dense_cublas_ms": round(ms_d, 4),
                              "dense_cublas_gbs": round((dbytes + io) / (ms_d / 1e3) / 1e9, 1),
                              "speedup_vs_dense": round(ms_d / ms, 3)}
        if T > 64:
            res[f"tokens_{T}"].update(tensor_stats(T, shapes, ms))
    t8 = res["tokens_8"]
    return {"metric": "sparse_linear_bandwidth", "value": t8["achieved_gbs"], "unit": "GB/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t8["ms"], "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic (random packed masks and values)",
            "config": {"workload": w.name, "matrices": len(shapes), "nm": f"{w.nm[0]}:{w.nm[1]}",
                       "compressed_weight_gb": round(wbytes / 1e9, 3), "launches_per_call": math.ceil(len(shapes) / 16),
                       "tokens_timed": 8},
            "roofline": {"bound": "hbm", "achieved": t8["achieved_gbs"], "peak": hbm_peak, "unit": "GB/s",
                         "frac": t8["frac"], "peak_kind": peak_kind},
            "tokens": res}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--mode", default="train", choices=["train", "sparse_linear", "masked_linear"])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="llama2_7b_stack_2of4")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--loop", default="fused", choices=["fused", "separate"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-step-seconds", type=float, default=2.0)
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' per-call timings")
    ap.add_argument("--tokens", type=int, default=256, help="--mode masked_linear: tokens per call (1-256)")
    ap.add_argument("--config-reps", type=int, default=10)
    ap.add_argument("--config-cpu-seconds", type=float, default=1.0)
    ap.add_argument("--serve-nm", default=None, choices=["2:4", "4:8"],
                    help="--mode sparse_linear: pack the workload's matrices with this pattern instead of its own")
    args = ap.parse_args()
    if args.warmup < 3:
        log("warm-up raised to 3 steps")
        args.warmup = 3
    from sparsity_mask_sampling_b200 import configs

    w = configs.WORKLOADS[args.workload]
    if args.serve_nm is not None:
        if args.mode != "sparse_linear":
            ap.error("--serve-nm applies to --mode sparse_linear")
        import dataclasses
        nm = tuple(int(v) for v in args.serve_nm.split(":"))
        w = dataclasses.replace(w, nm=nm, name=f"{w.name} packed {args.serve_nm}")
    if args.mode == "sparse_linear":
        out = sparse_linear_arm(args, w)
    elif args.mode == "masked_linear":
        import torch

        dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
        torch.cuda.set_device(dev)
        r = masked_linear_leg(dev, peaks()[0], tokens=args.tokens, reps=args.steps)
        out = {"metric": "masked linear layer, fused vs sampler + cuBLAS (ms per call)", "mode": "masked_linear",
               "value": r["fused_fwd_ms"] + r["fused_bwd_adam_ms"], "unit": "ms", "higher_is_better": False,
               "n_gpus": 1, "steps": args.steps, "dtype": "bf16 operands, fp32 accumulation", "data": "synthetic",
               "config": {"workload": r["workload"], "tokens": r["tokens"]}, "result": r}
    elif args.impl == "reference":
        out = reference_arm(args, w)
    else:
        out = gpu_arm(args, w)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
