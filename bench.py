#!/usr/bin/env python3
"""Benchmark of the hybrid Top-k+Top-p block-sparse attention path on B200.

One step = the whole path over one synthetic attention layer: block mask
(pool Q/K, pooled softmax, hybrid selection, CSC), sparse forward (O, LSE) and
sparse backward (dQ, dK, dV), each through the C ABI of libspa2.so.

Default workload: a Wan2.1-1.3B-shaped self-attention layer, B=1 H=12 N=32760
(21x30x52 latent grid) d=128, bf16 Q/K/V from a seeded spatio-temporally
smoothed Gaussian field with 4 sink keys, dO ~ N(0, 1), b_q=128 b_kv=64, the
hybrid mask calibrated to 95% block sparsity (k = 2.5%, p bisected).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Prints one JSON line. `value` is the sparse (algorithmic) TFLOP/s of the whole
step over all GPUs: forward 4*d*sum(kept rows x cols), backward 2.5x that,
divided by the step time, which includes the mask. Under torchrun each rank
runs its own layer (weak scaling, no data-path collective); the step time is
the max over ranks. `--impl reference` times the float64 CPU oracle on a
bounded sample of the same workload instead.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-attn fwd/bwd TFLOPS & speedup vs dense at 95% sparsity (1×B200)"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOADS = {
    "wan2.1-1.3b-layer": dict(B=1, H=12, N=32760, d=128, gen="smoothed"),
    "wan2.1-14b-layer": dict(B=1, H=40, N=75600, d=128, gen="smoothed"),
    "pr1": dict(B=1, H=2, N=512, d=64, gen="gaussian"),
}


def code_text_digest(text):
    """sha256 of source text with its // comments and blank lines removed, so a
    comment-only edit keeps a profile's counters attached to the same code."""
    import hashlib
    lines = [ln.split("//", 1)[0].rstrip() for ln in text.splitlines()]
    return hashlib.sha256("\n".join(ln for ln in lines if ln).encode()).hexdigest()


def code_digest(path):
    with open(path, encoding="utf-8") as f:
        return code_text_digest(f.read())


KERNEL_SOURCES = {
    "pool_kernel": "mask.cu", "logits_kernel": "mask.cu", "select_kernel": "mask.cu", "csc_kernel": "mask.cu",
    "v_to_f16_kernel": "attn_fwd.cu", "fwd_kernel": "attn_fwd.cu",
    "bwd_pre_kernel": "attn_bwd.cu", "bwd_dkdv_kernel": "attn_bwd.cu", "bwd_dq_kernel": "attn_bwd.cu",
}


def profiled_traffic(kernel, workload):
    """DRAM bytes (read + write) per launch of `kernel` on this workload, from the
    ncu summary profiles/traffic_<kernel>.txt, or None when the summary is missing,
    covers another workload, or was taken on different code (the digest of the
    kernel's source file, comments and blank lines removed, must match)."""
    src_name = KERNEL_SOURCES.get(kernel)
    if src_name is None:
        return None
    path = os.path.join(ROOT, "profiles", f"traffic_{kernel}.txt")
    src = os.path.join(ROOT, "trainable_block_sparse_pooled_b200", "csrc", src_name)
    try:
        fields = dict(line.split(":", 1) for line in open(path, encoding="utf-8")
                      if ":" in line and not line.startswith("#"))
        digest = code_digest(src)
    except OSError:
        return None
    fields = {k.strip(): v.strip() for k, v in fields.items()}
    if fields.get("code_sha256") != digest or fields.get("workload") != workload:
        return None
    try:
        return int(fields["bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def clock_scaled_peak(pk, clk):
    """bf16 tensor peak for a kernel timed at this run's clocks: the burst peak
    (taken at the maximum SM clock) scaled by median / maximum SM clock of the
    samples taken during the timed region, never above the burst peak."""
    burst = pk["bf16_tflops"]
    med, top = clk.get("sm_mhz"), clk.get("sm_max_mhz") or pk.get("sm_max_mhz")
    if not med or not top:
        return burst, "burst (no clock samples)"
    ratio = min(1.0, med / top)
    if ratio >= 0.99:
        return burst, f"burst: SM clock median {med:.0f} of {top:.0f} MHz"
    return burst * ratio, f"burst x {ratio:.3f} (SM clock median {med:.0f} of {top:.0f} MHz)"


def kernel_work(name, B, H, N, d, Tm, Tn, kept, fwd_flops):
    """Algorithmic work of one launch of a library kernel on this layer:
    (bound, amount, unit) with unit 'flop' for tensor-core kernels (forward
    4 d per kept token pair; the dK/dV pass holds 4 of the backward's 5
    products, the dQ pass 1) and 'byte' for HBM-bound kernels (every input read
    once, every output written once)."""
    e = B * H * N * d
    if name == "fwd_kernel":
        return "tensor", fwd_flops, "flop"
    if name == "bwd_dkdv_kernel":
        return "tensor", 2.0 * fwd_flops, "flop"
    if name == "bwd_dq_kernel":
        return "tensor", 0.5 * fwd_flops, "flop"
    if name == "pool_kernel":     # Q and K read, Qbar and Kbar written
        return "hbm", 2.0 * e * 2 + 4.0 * B * H * (Tm + Tn) * d, "byte"
    if name == "logits_kernel":   # Qbar and Kbar read, pooled logits written
        return "hbm", 4.0 * B * H * (Tm + Tn) * d + 4.0 * B * H * Tm * Tn, "byte"
    if name == "select_kernel":   # pooled logits read, CSR and kept-bit words written
        return "hbm", 4.0 * B * H * Tm * Tn + 4.0 * (kept + B * H * Tm) + 4.0 * B * H * Tm * ((Tn + 31) // 32), "byte"
    if name == "csc_kernel":
        return "hbm", 4.0 * B * H * Tm * ((Tn + 31) // 32) + 4.0 * (kept + B * H * Tn), "byte"
    if name == "v_to_f16_kernel":
        return "hbm", 4.0 * e, "byte"
    if name == "bwd_pre_kernel":     # O, O_lo, dO, Q read; fp16 dO, Q and D written
        return "hbm", 12.0 * e + 4.0 * B * H * N, "byte"
    return None, 0.0, None


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU, launched by torchrun)
# ---------------------------------------------------------------------------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value: float, dist) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist):
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------
def make_inputs(wl, seed, device):
    from trainable_block_sparse_pooled_b200 import synth
    B, H, N, d = wl["B"], wl["H"], wl["N"], wl["d"]
    if wl["gen"] == "smoothed":
        q, k, v = synth.smoothed_field(B=B, H=H, N=N, d=d, seed=seed, device=device)
    else:
        q, k, v = synth.gaussian_with_sinks(B=B, H=H, N=N, d=d, seed=seed, device=device)
    dout = synth.normal_like(q.shape, seed=seed + 1000, device=device)
    return q.contiguous(), k.contiguous(), v.contiguous(), dout.contiguous()


def kept_flops(mask, N, d, bq=128, bkv=64):
    """Forward flops 4*d*sum over kept (i, j) of valid rows x valid cols, from the
    CSR form of the mask (torch, on the mask's device)."""
    import torch
    dev = mask.row_cnt.device
    Tm, Tn = mask.row_idx.shape[-2], mask.row_idx.shape[-1]
    rows = (torch.clamp(N - torch.arange(Tm, device=dev) * bq, max=bq)).double()
    cols = (torch.clamp(N - torch.arange(Tn, device=dev) * bkv, max=bkv)).double()
    valid = torch.arange(Tn, device=dev) < mask.row_cnt[..., None]
    idx = mask.row_idx.long().clamp(0, Tn - 1)
    colsum = (cols[idx] * valid).sum(-1)
    return float(4.0 * d * (colsum * rows).sum().item())


def cpu_oracle_sample(q, k, v, dout, kf, pf, budget_s, max_blocks=None):
    """Time the float64 oracle on a bounded sample: head 0's mask, then forward and
    backward of its q-blocks in order until `budget_s` seconds have passed."""
    import numpy as np
    import oracle
    f = lambda t: t[0:1, 0:1].float().cpu().numpy().astype(np.float64)  # noqa: E731
    Q, K, V, dO = f(q), f(k), f(v), f(dout)
    N, d = Q.shape[-2], Q.shape[-1]
    scale = 1.0 / math.sqrt(d)
    t0 = time.perf_counter()
    _, _, mask = oracle.block_mask(Q, K, 128, 64, kf, pf)
    done, flops = 0, 0.0
    Tm = mask.shape[-2]
    for i in range(Tm):
        oracle.masked_attn_fwd_rows(Q, K, V, mask, 128, 64, scale, 0, 0, [i])
        oracle.masked_attn_bwd_rows(Q, K, V, mask, dO, 128, 64, scale, 0, 0, [i])
        rows = min(N, (i + 1) * 128) - i * 128
        cols = sum(min(N, (j + 1) * 64) - j * 64 for j in np.flatnonzero(mask[0, 0, i]))
        flops += 14.0 * d * rows * cols   # forward 4d + backward 10d per kept element
        done += 1
        if time.perf_counter() - t0 > budget_s or (max_blocks and done >= max_blocks):
            break
    dt = time.perf_counter() - t0
    return flops, dt, done


# ---------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args, wl, name):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import numpy as np
    import torch

    import oracle
    from trainable_block_sparse_pooled_b200 import calibrate
    torch.set_num_threads(os.cpu_count() or 1)
    qa, ka, va, da = make_inputs(wl, seed=0, device="cpu")               # every head of the layer
    # calibrate p over all heads with the oracle's own mask, as the GPU arm does with its kernels
    Qb = oracle.pool_blocks(qa.float().numpy().astype(np.float64), 128)
    Kb = oracle.pool_blocks(ka.float().numpy().astype(np.float64), 64)
    pbar32 = oracle.pooled_attention(Qb, Kb, wl["d"]).astype(np.float32)
    kf, pf, _ = calibrate.calibrate_p(lambda a, c: int(oracle.select_blocks(pbar32, a, c).sum()), pbar32.size,
                                      args.target_sparsity)
    q, k, v, dout = (x[:, :1].contiguous() for x in (qa, ka, va, da))   # head 0 is the timed sample
    del qa, ka, va, da
    per_step_s = min(4.0, max(0.5, 120.0 / args.steps))   # the whole run stays near two minutes
    for _ in range(args.warmup):
        cpu_oracle_sample(q, k, v, dout, kf, pf, per_step_s / 4, max_blocks=2)
    fl, tt, blocks = 0.0, 0.0, 0
    for _ in range(args.steps):
        f_, t_, b_ = cpu_oracle_sample(q, k, v, dout, kf, pf, per_step_s)
        fl += f_
        tt += t_
        blocks += b_
    value = fl / tt / 1e12
    cores = os.cpu_count()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": name, **{x: wl[x] for x in ("B", "H", "N", "d")}, "bq": 128, "bkv": 64,
                   "k_frac": kf, "p_frac": pf},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"head 0: oracle mask, then forward+backward of its first q-blocks for about "
                                   f"{per_step_s:.0f} s per step ({blocks} q-blocks over {args.steps} steps)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def dense_pass(s, q, k, v, dout, o, lse, o_lo, dq, dk, dv, N, d, fwd_ms, bwd_ms, step_ms):
    """k = 100% through the same kernels: dense times, speedups, dense-equivalent rate."""
    import torch
    dmask = s.new_mask()
    s.block_mask(q, k, 1.0, 0.0, dmask)
    dense_flops = kept_flops(dmask, N, d)
    e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
    s.fwd(q, k, v, dmask, o=o, lse=lse, o_lo=o_lo)
    s.bwd(q, k, v, o, lse, dout, dmask, dq=dq, dk=dk, dv=dv, o_lo=o_lo)
    torch.cuda.synchronize()
    fwd_d = bwd_d = 0.0
    iters = 3
    for _ in range(iters):
        e0.record()
        s.fwd(q, k, v, dmask, o=o, lse=lse, o_lo=o_lo)
        e1.record()
        s.bwd(q, k, v, o, lse, dout, dmask, dq=dq, dk=dk, dv=dv, o_lo=o_lo)
        e2.record()
        torch.cuda.synchronize()
        fwd_d += e0.elapsed_time(e1) / iters
        bwd_d += e1.elapsed_time(e2) / iters
    s.check()
    B, H = q.shape[0], q.shape[1]
    return {"fwd_ms": fwd_d, "bwd_ms": bwd_d, "fwd_tflops": dense_flops / (fwd_d * 1e-3) / 1e12,
            "bwd_tflops": 2.5 * dense_flops / (bwd_d * 1e-3) / 1e12,
            "speedup_fwd": fwd_d / fwd_ms, "speedup_fwd_bwd": (fwd_d + bwd_d) / (fwd_ms + bwd_ms),
            "speedup_step_incl_mask": (fwd_d + bwd_d) / step_ms,
            "dense_equiv_tflops": 14.0 * d * B * H * N * N / (step_ms * 1e-3) / 1e12}


def run_gpu(args, wl, name):
    import torch
    ws, rank, local = dist_env()
    dist = None
    if ws > 1:
        import torch.distributed as dist_mod
        from datetime import timedelta
        torch.cuda.set_device(local)
        dist_mod.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
        dist = dist_mod
    else:
        torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from trainable_block_sparse_pooled_b200 import binding as b
    from trainable_block_sparse_pooled_b200 import calibrate

    B, H, N, d = wl["B"], wl["H"], wl["N"], wl["d"]
    q, k, v, dout = make_inputs(wl, seed=rank, device=dev)
    s = b.Spa2(B, H, N, d, device=dev)
    mask = s.new_mask()
    total_blocks = B * H * s.Tm * s.Tn

    def kept(kf, pf):
        s.block_mask(q, k, kf, pf, mask)
        return int(mask.row_cnt.sum().item())

    kf, pf, sparsity = calibrate.calibrate_p(kept, total_blocks, args.target_sparsity)
    s.block_mask(q, k, kf, pf, mask)
    s.check(b.OP_MASK)
    fwd_flops = kept_flops(mask, N, d)
    bwd_flops = 2.5 * fwd_flops
    step_flops = fwd_flops + bwd_flops

    o = torch.empty_like(q)
    o_lo = torch.empty_like(q)
    lse = torch.empty(B, H, N, dtype=torch.float32, device=dev)
    gt = torch.float32
    dq = torch.empty(q.shape, dtype=gt, device=dev)
    dk = torch.empty(q.shape, dtype=gt, device=dev)
    dv = torch.empty(q.shape, dtype=gt, device=dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record()
        s.block_mask(q, k, kf, pf, mask)
        if ev is not None:
            ev[1].record()
        s.fwd(q, k, v, mask, o=o, lse=lse, o_lo=o_lo)
        if ev is not None:
            ev[2].record()
        s.bwd(q, k, v, o, lse, dout, mask, dq=dq, dk=dk, dv=dv, o_lo=o_lo)
        if ev is not None:
            ev[3].record()

    for _ in range(args.warmup):
        step()
    s.check()

    # ---- timed region: K steps, events on the launching (current) stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    vis = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    phys = int(vis[local]) if local < len(vis) and vis[local].strip().isdigit() else local
    clocks = ClockSampler(phys)
    barrier(dist)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.15)
    torch.cuda.nvtx.range_push("spa2_timed")     # ncu --nvtx-include "spa2_timed/" selects this region
    t_start.record()
    for i in range(args.steps):
        step(evs[i])
    t_end.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    # The same K steps again with a CUDA event pair around every kernel launch
    # (spa2_timing_enable): per-kernel durations for `kernels` and `roofline`.
    # Kept out of the headline steps above because an event between two kernels
    # stops the second from starting early (programmatic dependent launch).
    b.spa2_timing_read()
    b.spa2_timing_enable(True)
    p_start, p_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p_start.record()
    for i in range(args.steps):
        step()
    p_end.record()
    torch.cuda.synchronize()
    b.spa2_timing_enable(False)
    per_kernel = b.spa2_timing_read()
    profiled_ms = p_start.elapsed_time(p_end) / args.steps
    clk = clocks.stop()
    barrier(dist)
    s.check()
    local_ms = t_start.elapsed_time(t_end) / args.steps
    ms = max_over_ranks(local_ms, dist)
    op_ms = [sum(e[j].elapsed_time(e[j + 1]) for e in evs) / args.steps for j in range(3)]
    mask_ms, fwd_ms, bwd_ms = op_ms

    # ---- dense pass through the same kernels (k = 100%)
    dense = None
    if not args.no_dense:
        dense = dense_pass(s, q, k, v, dout, o, lse, o_lo, dq, dk, dv, N, d, fwd_ms, bwd_ms, ms)
    # ---- end to end through the C ABI with host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hdo = (x.cpu().pin_memory() for x in (q, k, v, dout))
        ho = torch.empty(q.shape, dtype=q.dtype).pin_memory()
        hdq, hdk, hdv = (torch.empty(q.shape, dtype=gt).pin_memory() for _ in range(3))
        q_in, k_in, v_in, do_in = (torch.empty_like(x) for x in (q, k, v, dout))

        def e2e_step():
            q_in.copy_(hq, non_blocking=True)
            k_in.copy_(hk, non_blocking=True)
            v_in.copy_(hv, non_blocking=True)
            do_in.copy_(hdo, non_blocking=True)
            s.block_mask(q_in, k_in, kf, pf, mask)
            s.fwd(q_in, k_in, v_in, mask, o=o, lse=lse, o_lo=o_lo)
            s.bwd(q_in, k_in, v_in, o, lse, do_in, mask, dq=dq, dk=dk, dv=dv, o_lo=o_lo)
            ho.copy_(o, non_blocking=True)
            hdq.copy_(dq, non_blocking=True)
            hdk.copy_(dk, non_blocking=True)
            hdv.copy_(dv, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        e2e_steps = max(1, min(args.steps, 5))
        barrier(dist)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        for _ in range(e2e_steps):
            e2e_step()
        a1.record()
        torch.cuda.synchronize()
        barrier(dist)
        s.check()
        e2e_ms = max_over_ranks(a0.elapsed_time(a1) / e2e_steps, dist)
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hdo))
        d2h = sum(x.numel() * x.element_size() for x in (ho, hdq, hdk, hdv))
        e2e = {"value": step_flops * ws / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    # ---- CPU baseline (rank 0, N=1 only)
    cpu = None
    if ws == 1 and not args.no_cpu_baseline:
        import torch as _t
        _t.set_num_threads(os.cpu_count() or 1)
        fl, dt, blocks = cpu_oracle_sample(q, k, v, dout, kf, pf, args.cpu_budget)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": _t.get_num_threads(), "kind": "oracle",
               "sample": f"head 0 of the same layer: oracle mask, then float64 forward+backward of its first "
                         f"{blocks} q-blocks ({dt:.1f} s)"}

    pk, pk_kind = peaks()
    value = step_flops * ws / (ms * 1e-3) / 1e12
    bwd_tf = bwd_flops / (bwd_ms * 1e-3) / 1e12
    fwd_tf = fwd_flops / (fwd_ms * 1e-3) / 1e12
    kept = int(mask.row_cnt.sum().item())
    mask_bytes = 2.0 * B * H * N * d * 2 + 4.0 * (B * H * s.Tm + kept * 2 + B * H * s.Tn)
    mask_gbs = mask_bytes / (mask_ms * 1e-3) / 1e9
    tensor_peak, tensor_peak_kind = clock_scaled_peak(pk, clk)
    kernels = {}
    for kname, (n_launch, tot_ms) in per_kernel.items():
        bound, work, unit = kernel_work(kname, B, H, N, d, s.Tm, s.Tn, kept, fwd_flops)
        avg_ms = tot_ms / n_launch
        ent = {"launches": n_launch, "avg_us": avg_ms * 1e3, "share": tot_ms / (profiled_ms * args.steps)}
        if bound == "tensor":
            ent.update(bound="tensor", achieved=work / (avg_ms * 1e-3) / 1e12, unit="TFLOP/s")
            ent["frac"] = ent["achieved"] / tensor_peak
        elif bound == "hbm":
            ent.update(bound="hbm", achieved=work / (avg_ms * 1e-3) / 1e9, unit="GB/s")
            ent["frac"] = ent["achieved"] / pk["hbm_gbs"]
        kernels[kname] = ent
    dom = max(kernels, key=lambda k: kernels[k]["share"])
    dk = kernels[dom]
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": name, "B": B, "H": H, "N": N, "d": d, "bq": 128, "bkv": 64,
                   "k_frac": kf, "p_frac": pf, "block_sparsity": sparsity,
                   "inputs": ("seeded smoothed spatio-temporal Gaussian field, K = 0.5 Q + sqrt(0.75) noise, "
                              "4 sink keys, dO ~ N(0,1)") if wl["gen"] == "smoothed" else
                             "seeded N(0,1) with 2 sink keys, dO ~ N(0,1)",
                   "grad_dtype": "fp32", "l2": "inputs larger than L2 (Q, K, V, dO are 4 x %.0f MB)" %
                   (B * H * N * d * 2 / 1e6), "parallelism": f"independent layer per GPU x{ws}"},
        "roofline": {"bound": dk.get("bound"), "kernel": dom, "achieved": dk.get("achieved"),
                     "peak": tensor_peak if dk.get("bound") == "tensor" else pk["hbm_gbs"],
                     "unit": dk.get("unit"), "frac": dk.get("frac"),
                     "traffic": profiled_traffic(dom, name),
                     "avg_launch_us": dk["avg_us"], "share_of_step": dk["share"],
                     "peak_kind": (f"{pk_kind} bf16 {tensor_peak_kind}" if dk.get("bound") == "tensor"
                                   else f"{pk_kind} HBM copy bandwidth")},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": sum(v["launches"] for v in kernels.values()),
        "kernel_timing": {"steps": args.steps, "ms_per_step": profiled_ms,
                          "how": "the timed steps repeated with a CUDA event pair on the launch stream around each "
                                 "kernel; avg_us = summed event time / launches; share = of that pass's step time"},
        "clocks": clk,
        "kernels": kernels,
        "ops": {"mask_us": mask_ms * 1e3, "mask_GBps": mask_gbs, "mask_hbm_frac": mask_gbs / pk["hbm_gbs"],
                "fwd_ms": fwd_ms, "fwd_tflops": fwd_tf, "fwd_frac": fwd_tf / tensor_peak,
                "bwd_ms": bwd_ms, "bwd_tflops": bwd_tf, "bwd_frac": bwd_tf / tensor_peak,
                "fwd_flops": fwd_flops, "bwd_flops": bwd_flops,
                "note": "per-op times are CUDA events around each C-ABI call in the timed steps; fractions "
                        "use the clock-scaled burst peak of roofline.peak_kind"},
        "dense": dense,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_sweep(args):
    """Sparsity sweep on the 1.3B layer shape (B1 H12 d128, smoothed-field inputs):
    block sparsity 80 / 90 / 95 / 97% (k = (1 - target) / 2, p calibrated) and the
    k = 100% pass, at N in {8192, 32760, 65536}. One JSON line per point: mask,
    forward and backward times (CUDA events, median of --steps after --warmup),
    sparse and dense-equivalent TFLOP/s, and speedup over the k = 100% pass, each with
    the SM clocks sampled (nvidia-smi) while that N's points were timed."""
    import torch
    from trainable_block_sparse_pooled_b200 import binding as b
    from trainable_block_sparse_pooled_b200 import calibrate, synth
    torch.cuda.set_device(0)
    B, H, d = 1, 12, 128
    pk, _ = peaks()

    def med_ms(fn):
        for _ in range(args.warmup):
            fn()
        ts = []
        for _ in range(args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return sorted(ts)[len(ts) // 2]

    for N in (8192, 32760, 65536):
        q, k, v = synth.smoothed_field(B=B, H=H, N=N, d=d, seed=11, device="cuda")
        dout = synth.normal_like(q.shape, seed=12, device="cuda")
        s = b.Spa2(B, H, N, d)
        mask = s.new_mask()
        o, o_lo = torch.empty_like(q), torch.empty_like(q)
        lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
        dq, dk, dv = (torch.empty(q.shape, dtype=torch.float32, device="cuda") for _ in range(3))
        total = B * H * s.Tm * s.Tn
        dense_flops = 4.0 * B * H * N * N * d

        def kept(kf, pf):
            s.block_mask(q, k, kf, pf, mask)
            return mask.kept_blocks()

        points, dense_ms = [], None
        clocks = ClockSampler(0)
        clocks.start()
        time.sleep(0.15)
        for target in (None, 0.80, 0.90, 0.95, 0.97):
            if target is None:
                kf, pf = 1.0, 0.0
                sparsity = 1.0 - kept(kf, pf) / total
            else:
                kf, pf, sparsity = calibrate.calibrate_p(kept, total, target)
            s.block_mask(q, k, kf, pf, mask)
            flops = kept_flops(mask, N, d)
            mask_ms = med_ms(lambda: s.block_mask(q, k, kf, pf, mask))
            fwd_ms = med_ms(lambda: s.fwd(q, k, v, mask, o=o, lse=lse, o_lo=o_lo))
            bwd_ms = med_ms(lambda: s.bwd(q, k, v, o, lse, dout, mask, dq=dq, dk=dk, dv=dv, o_lo=o_lo))
            s.check()
            if target is None:
                dense_ms = (fwd_ms, bwd_ms)
            line = {"sweep": "sparsity", "N": N, "target_sparsity": target, "block_sparsity": sparsity,
                    "k_frac": kf, "p_frac": pf, "mask_us": mask_ms * 1e3, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
                    "fwd_tflops": flops / (fwd_ms * 1e-3) / 1e12, "bwd_tflops": 2.5 * flops / (bwd_ms * 1e-3) / 1e12,
                    "fwd_frac_burst": flops / (fwd_ms * 1e-3) / 1e12 / pk["bf16_tflops"],
                    "fwd_dense_equiv_tflops": dense_flops / (fwd_ms * 1e-3) / 1e12,
                    "speedup_fwd": dense_ms[0] / fwd_ms, "speedup_fwd_bwd": sum(dense_ms) / (fwd_ms + bwd_ms),
                    "steps": args.steps, "warmup": args.warmup}
            points.append(line)
        clk = clocks.stop()
        for line in points:
            line["clocks"] = clk
            print(json.dumps(line), flush=True)
        del q, k, v, dout, s, mask, o, o_lo, lse, dq, dk, dv
        torch.cuda.empty_cache()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["spa2", "reference"], default="spa2")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="wan2.1-1.3b-layer")
    ap.add_argument("--target-sparsity", type=float, default=0.95)
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true", help="skip the k = 100%% comparison pass")
    ap.add_argument("--sweep", action="store_true",
                    help="sparsity sweep (80/90/95/97%% and k = 100%%) at N = 8192, 32760, 65536: one JSON line per point")
    ap.add_argument("--heads", type=int, default=0,
                    help="override the workload's head count (a smaller case of the same layer, for profiling)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.sweep:
        return run_sweep(args)
    wl = dict(WORKLOADS[args.workload])
    name = args.workload
    if args.heads > 0:
        wl["H"] = args.heads
        name = f"{args.workload} ({args.heads} heads)"
    if args.impl == "reference":
        return run_reference(args, wl, name)
    return run_gpu(args, wl, name)


if __name__ == "__main__":
    sys.exit(main())
