#!/usr/bin/env python
"""SLA HSTU attention fwd+bwd throughput on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload hist16k]
    python bench.py --impl reference ...        # the CPU oracle as the reference arm

A step is one forward and one backward pass (work list, attention kernels,
dq conversion) over one synthetic jagged batch.  The metric is TFLOP/s counted
over unmasked (row, key) pairs: 4d FLOPs per pair per head forward, 10d
backward.  Inputs (q, k, v, dout: 4 x 403 MB for the 16K workload) exceed the
126 MB L2, so no flush is needed between steps.  N > 1 runs one process per
GPU (torchrun), each on its own batch of the same shape (weak scaling, no
collective on the data path); time is the max over ranks.

Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_hstu_attention_b200 import flops as F  # noqa: E402
from workloads import WORKLOADS, make_batch  # noqa: E402

METRIC = "SLA HSTU attn fwd+bwd TFLOP/s (unmasked pairs), % of B200 BF16 peak"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}
# sources a kernel's device code is compiled from (its .cu and the shared headers)
_HDRS = ("sparse_hstu_attention_b200/csrc/sm100.cuh", "sparse_hstu_attention_b200/csrc/sla_common.cuh")
# (head_dim 128 kernels: the workloads this bench times all have d = 128)
KERNEL_SOURCES = {"fwd": ("sparse_hstu_attention_b200/csrc/fwd_tc.cu",) + _HDRS,
                  "bwd": ("sparse_hstu_attention_b200/csrc/bwd_fused.cu",) + _HDRS}
KERNEL_NAMES = {"fwd": "fwd_tc_kernel",
                "bwd": "bwd_kvq_kernel (one pass, dQ via fp32 workspace) + dq_convert_kernel"}
# kernels of this library per call: forward = work list + attention; backward
# (d = 128) = work list + one-pass kernel + dq conversion (the workspace
# zeroing is a cudaMemsetAsync, not counted)
LAUNCHES_PER_STEP = {"fwd": 2, "bwd": 3}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def _sha1(paths):
    """SHA-1 over the concatenated contents of `paths` (None if one is missing)."""
    h = hashlib.sha1()
    for path in paths:
        p = os.path.join(ROOT, path)
        if not os.path.exists(p):
            return None
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _traffic(which, workload):
    """DRAM bytes per launch from a committed ncu capture, if the kernel source
    is unchanged since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{KERNEL_NAMES[which]}/{workload}")
    if not e or e.get("source_sha1") != _sha1(KERNEL_SOURCES[which]):
        return None
    return e.get("dram_bytes_per_launch")


def roofline(flops, alg_bytes, ms, peaks, peak_src, clk):
    """The dominant kernel against the roof its arithmetic intensity puts it
    under: the tensor roof (measured dense bf16 GEMM) when flops / bytes is at
    or above the ridge, else the HBM roof (measured copy bandwidth).

    The tensor denominator is the burst GEMM figure, measured at the maximum
    SM clock, the clock a kernel runs at in a short timed loop.  The
    sustained figure was measured seconds into a power-capped loop at a lower
    clock; the fraction of it is reported beside, with both clock medians,
    but never as `frac`."""
    tflops = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    s = ms * 1e-3
    ach_t = flops / s / 1e12
    ach_b = alg_bytes / s / 1e9
    ridge = tflops * 1e12 / (hbm * 1e9)
    ai = flops / alg_bytes
    tensor = ai >= ridge
    r = {"bound": "tensor" if tensor else "hbm",
         "achieved": ach_t if tensor else ach_b,
         "peak": tflops if tensor else hbm,
         "unit": "TFLOP/s" if tensor else "GB/s",
         "frac": (ach_t / tflops) if tensor else (ach_b / hbm),
         "peak_source": (f"bf16_tflops (burst) of {peak_src}" if tensor
                         else f"hbm_gbs of {peak_src}"),
         "arithmetic_intensity": ai, "ridge_flop_per_byte": ridge,
         "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": alg_bytes,
         "tensor_tflops": ach_t, "frac_of_tensor_peak": ach_t / tflops,
         "hbm_gbs": ach_b, "frac_of_hbm_peak": ach_b / hbm}
    sus = peaks.get("bf16_tflops_sustained")
    if sus:
        under = (peaks.get("clocks_under_load") or {}).get("sm_mhz_median")
        r["frac_of_sustained_tensor_peak"] = ach_t / float(sus)
        r["sustained_peak_sm_mhz"] = under
        r["run_sm_mhz"] = clk.get("sm_mhz")
    return r


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 50 ms while active."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.file = None

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.dev)], stdout=self.file,
                stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.file.seek(0)
        rows = [l.strip().split(", ") for l in self.file if l.strip()]
        os.unlink(self.file.name)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
                power.append(float(r[3]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        pmax = max(power) if power else 0
        loaded = [s for s, p in zip(sm, power) if p >= 0.5 * pmax] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": pmax}


def _setup_dist(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    return world, rank, local


def _sample_cost_flops(p, rows, d, H, row_pairs, key_pairs):
    """Metric-equivalent FLOPs of an oracle sample: forward on the sampled rows
    plus the backward split evenly between the sampled rows (dq) and the same
    tokens taken as keys (dk, dv)."""
    rp = float(row_pairs[rows].sum())
    kp = float(key_pairs[rows].sum())
    return H * d * (4.0 * rp + 10.0 * 0.5 * (rp + kp)), rp


def _oracle_sample(batch, n_tokens, seed, rab=None):
    import oracle
    p = oracle.Problem.from_batch(batch, **(rab or {}))
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(batch.T, size=min(n_tokens, batch.T), replace=False))
    t0 = time.perf_counter()
    p.fwd(batch.q, batch.k, batch.v, rows=rows)
    p.bwd_dq(batch.q, batch.k, batch.v, batch.dout, rows=rows)
    p.bwd_dkv(batch.q, batch.k, batch.v, batch.dout, keys=rows)
    return time.perf_counter() - t0, rows


def _pair_tables(batch):
    w = batch.workload
    return F.pairs_per_token(batch.lengths, batch.num_targets, w.contextual_len, w.K1, w.K2)


def cpu_baseline(batch, target_s=15.0, rab=None):
    """The oracle, as it stands, on a bounded random sample of the workload's
    tokens (rab: the oracle's relative-attention-bias arguments, or None)."""
    w = batch.workload
    rp, kp = _pair_tables(batch)
    # The oracle runs its loops on all host cores, so a small sample costs
    # more per token than a large one: grow the sample geometrically until a
    # run takes a second or more, then scale it to the target time.
    n, t = 64, 0.0
    while n < batch.T:
        t, _ = _oracle_sample(batch, n, seed=7, rab=rab)
        if t >= 1.0:
            break
        n = min(batch.T, n * 4)
    n = int(min(batch.T, max(64, n * target_s / max(t, 1e-3))))
    t, rows = _oracle_sample(batch, n, seed=8, rab=rab)
    fl, _ = _sample_cost_flops(None, rows, w.d, w.H, rp, kp)
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    cores = int(os.environ.get("OMP_NUM_THREADS", cores))
    return {"value": fl / t / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(rows)} random tokens of the {w.name} batch: forward and dq for them "
                      f"as rows, dk/dv for them as keys"
                      f"{' (with the relative attention bias)' if rab else ''}; fp64 C loops; "
                      f"{t:.1f} s",
            "seconds": t}


def run_reference(args):
    """The oracle timed on the host cores as the reference arm (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    if args.workload == "mot":
        print(json.dumps({"impl": "reference",
                          "unavailable": "the oracle arm times single workloads; "
                                         "run it on mot_long's shape via the default workloads"}))
        return
    w = WORKLOADS[args.workload]
    batch = make_batch(w)
    rp, kp = _pair_tables(batch)
    per_step_s = max(0.5, min(10.0, 150.0 / (args.steps + args.warmup)))
    t, _ = _oracle_sample(batch, 64, seed=1)
    n = int(min(batch.T, max(16, 64 * per_step_s / max(t, 1e-3))))
    total_t, total_fl = 0.0, 0.0
    for s in range(args.warmup + args.steps):
        t, rows = _oracle_sample(batch, n, seed=100 + s)
        if s >= args.warmup:
            fl, _ = _sample_cost_flops(None, rows, w.d, w.H, rp, kp)
            total_t += t
            total_fl += fl
    value = total_fl / total_t / 1e12
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    cores = int(os.environ.get("OMP_NUM_THREADS", cores))
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total_t / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(w, batch),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": f"{n} random tokens per step of the {w.name} batch"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def rank_batch(w, world, rank, strong=False):
    """This rank's batch.  N = 1: the workload's batch.  N > 1: a global batch
    split by whole sequences (sharding.partition_sequences: longest first on
    the closed-form pair count), no exchange on the data path.  strong: the
    global batch is the workload's one batch (total work fixed as N grows);
    else it is N batches of the recipe (one per rank's seed), so the work per
    GPU stays fixed (weak scaling) while the sequences still go to the ranks
    by the balancer, not one draw per rank."""
    from sparse_hstu_attention_b200 import sharding
    from workloads import draw_lengths
    if world == 1:
        return make_batch(w), None
    if strong:
        lengths = draw_lengths(w)
    else:
        lengths = np.concatenate([draw_lengths(w, seed=w.seed + 7919 * r) for r in range(world)])
    nts = np.minimum(np.full(len(lengths), w.num_targets), lengths)
    owned = sharding.partition_sequences(lengths, nts, world, w.contextual_len, w.K1, w.K2)
    mine = owned[rank]
    info = {"global_sequences": int(len(lengths)), "global_tokens": int(lengths.sum()),
            "rank0_sequences": [int(lengths[b]) for b in owned[0]],
            "balancer": "longest-first on closed-form unmasked pairs"}
    return make_batch(w, lengths=lengths[mine], num_targets=nts[mine],
                      seed=w.seed + 7919 * rank), info


def _config(w, batch):
    pairs = F.total_pairs(batch.lengths, batch.num_targets, w.contextual_len, w.K1, w.K2)
    in_bytes = 4 * batch.T * w.H * w.d * 2
    return {"workload": w.name, "B": int(len(batch.lengths)), "T": int(batch.T), "H": w.H,
            "d": w.d, "K1": w.K1, "K2": w.K2, "contextual_len": w.contextual_len,
            "num_targets": w.num_targets, "N": w.N, "alpha": w.alpha,
            "lengths": [int(x) for x in batch.lengths], "pairs_per_head": pairs,
            "l2": f"inputs {in_bytes / 1e6:.0f} MB > 126 MB L2; no flush"}


def stu_cpu_baseline(w, lengths, nts, dr, cfg_full, fp8=False, budget_s=10.0):
    """The STU oracle, as it stands (fp64 numpy around the C attention), on a
    bounded sample: layer 1 forward and backward, one sequence at a time from
    the shortest up, until about budget_s seconds of CPU work are done; FLOPs
    counted as the GPU line counts them."""
    from oracle import stu as S
    offs = np.concatenate([[0], np.cumsum(lengths)])
    dm = cfg_full.d_model
    wo = S.Weights.of(**{k: dr.layers[0][k].float().numpy() for k in
                         ("ln1_w", "ln1_b", "w1", "b1", "ln2_w", "ln2_b", "w2", "b2")})
    cfg = S.AttnCfg(cfg_full.H, cfg_full.d, cfg_full.contextual_len, cfg_full.K1, cfg_full.K2,
                    cfg_full.alpha, cfg_full.N, cfg_full.ln_eps)
    rng = np.random.default_rng(0)
    t, fl, toks, nseq = 0.0, 0.0, 0, 0
    for b in np.argsort(lengths, kind="stable"):
        s0, s1 = int(offs[b]), int(offs[b + 1])
        L = s1 - s0
        x = dr.x[s0:s1].float().numpy().astype(np.float64)
        g = rng.standard_normal((L, dm))
        t0 = time.perf_counter()
        _, cache = S.layer_fwd(x, wo, np.array([0, L]), nts[b:b + 1], cfg, fp8=fp8)
        S.layer_bwd(g, wo, cache)
        t += time.perf_counter() - t0
        pairs = F.total_pairs(np.array([L]), nts[b:b + 1], w.contextual_len, w.K1, w.K2)
        fl += 3 * 2 * dm * 5 * dm * L + F.fwd_flops(pairs, w.H, w.d) + \
            F.bwd_flops(pairs, w.H, w.d)
        toks, nseq = toks + L, nseq + 1
        if t >= budget_s:
            break
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    cores = int(os.environ.get("OMP_NUM_THREADS", cores))
    return {"value": fl / t / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"layer 1 forward and backward on the {nseq} shortest sequences "
                      f"({toks} tokens){', E4M3 forward projections' if fp8 else ''}; "
                      f"fp64; {t:.1f} s",
            "seconds": t}


def run_stu(args, world, rank, local):
    """The 6-layer STU stack workload (truncation after layer 3): one step is
    the stack's forward and backward, every parameter gradient included.
    --fp8: the forward projections in E4M3, the weights' E4M3 copies redone
    inside every step (as after each optimizer update)."""
    from sparse_hstu_attention_b200 import stu
    from workloads import (STU_LAYERS, STU_TAIL, STU_TRUNC_AFTER, draw_lengths, draw_stu,
                           offsets_from_lengths)
    dev = torch.device("cuda", local)
    w = WORKLOADS["stu"]
    lengths = draw_lengths(w)
    nts = np.minimum(np.full(len(lengths), w.num_targets), lengths)
    c, tail = w.contextual_len, STU_TAIL
    tl = stu.truncated_lengths(lengths, nts, c, tail)
    full = stu.StuConfig(w.H, w.d, c, w.K1, w.K2, w.alpha, w.N)
    cut = stu.StuConfig(w.H, w.d, c, w.K1, w.K2, w.alpha, float(c + tail + w.num_targets))
    offs = offsets_from_lengths(lengths)
    T, T_out, dm = int(offs[-1]), int(tl.sum()), full.d_model
    dr = draw_stu(T, T_out, dm, STU_LAYERS, seed=w.seed + 7919 * rank)
    ws = [stu.StuWeights.from_host(lw, dev) for lw in dr.layers]
    stack = stu.StuStack(ws, full, cut, STU_TRUNC_AFTER, tail, fp8=args.fp8, remat=args.remat)
    offs_d = torch.tensor(offs, dtype=torch.int32, device=dev)
    nts_d = torch.tensor(nts, dtype=torch.int32, device=dev)
    x, dout = dr.x.to(dev), dr.dout.to(dev)
    # FLOPs: per layer the two projections (2 T dm (4 dm + dm)) forward and
    # twice that backward (input and weight gradients); attention 4d / 10d
    # per unmasked pair per head
    p_full = F.total_pairs(lengths, nts, c, w.K1, w.K2)
    p_cut = F.total_pairs(tl, nts, c, w.K1, w.K2)
    n_full, n_cut = STU_TRUNC_AFTER, STU_LAYERS - STU_TRUNC_AFTER
    gemm = 3 * 2 * dm * 5 * dm * (n_full * T + n_cut * T_out)
    attn = (F.fwd_flops(p_full, w.H, w.d) + F.bwd_flops(p_full, w.H, w.d)) * n_full + \
           (F.fwd_flops(p_cut, w.H, w.d) + F.bwd_flops(p_cut, w.H, w.d)) * n_cut

    def step():
        if args.fp8:
            stack.requantize()
        out, ctx = stack.forward(x, offs_d, nts_d, lengths, nts)
        stack.backward(dout, ctx)

    # bytes each layer's forward keeps for its backward (beyond its input)
    _, ctx0 = stack.forward(x, offs_d, nts_d, lengths, nts)
    saved = [st.saved_bytes() for st in ctx0[0]]
    del ctx0
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        t0.record()
        for _ in range(K):
            step()
        t1.record()
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
    ms = t0.elapsed_time(t1) / K
    if world > 1:
        tt = torch.tensor([ms], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
        ms = float(tt.item())
    if rank == 0:
        peaks, src = _peaks()
        peak = float(peaks.get("bf16_tflops_sustained") or peaks.get("bf16_tflops"))
        value = world * (gemm + attn) / (ms * 1e-3) / 1e12
        print(json.dumps({
            "metric": "STU stack fwd+bwd TFLOP/s (projections + SLA attention over unmasked pairs)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16, forward projections e4m3" if args.fp8 else "bf16",
            "data": "synthetic (seeded N(0,1) inputs, Xavier-uniform weights)",
            "config": {"workload": "stu", "fp8_forward_projections": bool(args.fp8),
                       "remat": bool(args.remat), "layers": STU_LAYERS,
                       "trunc_after": STU_TRUNC_AFTER,
                       "tail": tail, "B": int(len(lengths)), "T": T, "T_truncated": T_out,
                       "d_model": dm, "H": w.H, "d": w.d, "K1": w.K1, "K2": w.K2,
                       "contextual_len": c, "num_targets": w.num_targets,
                       "N": [w.N, cut.N]},
            "flops_per_step": {"projections": gemm, "attention": attn},
            "saved_activation_bytes_per_layer": saved,
            "frac_of_sustained_peak": value / world / peak,
            "frac_of_burst_peak": value / world / float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])),
            "gpu_launches": K * (STU_LAYERS * (6 + 11 + (2 if args.fp8 else 0) +
                                              (3 if args.remat else 0)) + 3),
            "clocks": clocks.summary(),
            **({} if (world > 1 or args.no_cpu_baseline) else
               {"cpu_baseline": stu_cpu_baseline(w, lengths, nts, dr, full, args.fp8)})}),
            flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def run_mot(args, world, rank, local):
    """Mixture of Transducers: the SLA attention of three channels (each its own
    sequences, heads and SLA window) forward and backward, as one grouped
    launch per pass; the same work as three separate calls per pass is timed
    beside it."""
    import sparse_hstu_attention_b200 as sla
    from workloads import MOT_CHANNELS
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    chans, groups, fl = [], [], 0.0
    for name, w in MOT_CHANNELS.items():
        b = make_batch(w, seed=w.seed + 7919 * rank)
        pairs = F.total_pairs(b.lengths, b.num_targets, w.contextual_len, w.K1, w.K2)
        fl += F.fwd_flops(pairs, w.H, w.d) + F.bwd_flops(pairs, w.H, w.d)
        q, k, v, dout = (t.to(dev) for t in (b.q, b.k, b.v, b.dout))
        g = dict(q=q, k=k, v=v, dout=dout,
                 seq_offsets=torch.tensor(b.seq_offsets, dtype=torch.int32, device=dev),
                 num_targets=torch.tensor(b.num_targets, dtype=torch.int32, device=dev),
                 contextual_len=w.contextual_len, K1=w.K1, K2=w.K2, alpha=w.alpha, N=w.N,
                 max_seq_len=int(b.lengths.max()), out=torch.empty_like(q))
        groups.append(g)
        chans.append({"name": name, "B": int(len(b.lengths)), "T": b.T, "H": w.H, "d": w.d,
                      "K1": w.K1, "K2": w.K2, "contextual_len": w.contextual_len,
                      "num_targets": w.num_targets, "N": w.N, "unmasked_pairs_per_head": pairs})
    sizes = [(g["q"].shape[0], g["seq_offsets"].numel() - 1, g["q"].shape[1], 128)
             for g in groups]
    ws_f = torch.empty(sla.hstu_sla_grouped_workspace_bytes(0, sizes), dtype=torch.uint8,
                       device=dev)
    ws_b = torch.empty(sla.hstu_sla_grouped_workspace_bytes(1, sizes), dtype=torch.uint8,
                       device=dev)
    sep_ws = [(torch.empty(sla.hstu_sla_workspace_bytes(0, *sz), dtype=torch.uint8, device=dev),
               torch.empty(sla.hstu_sla_workspace_bytes(1, *sz), dtype=torch.uint8, device=dev))
              for sz in sizes]
    fwd_keys = ("contextual_len", "K1", "K2", "alpha", "N", "max_seq_len")

    def grouped_step():
        sla.hstu_sla_fwd_grouped(groups, workspace=ws_f)
        sla.hstu_sla_bwd_grouped(groups, workspace=ws_b)

    def separate_step():
        for g, (wf, wb) in zip(groups, sep_ws):
            kw = {k: g[k] for k in fwd_keys}
            sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["seq_offsets"], g["num_targets"],
                             out=g["out"], workspace=wf, **kw)
            sla.hstu_sla_bwd(g["dout"], g["q"], g["k"], g["v"], g["seq_offsets"],
                             g["num_targets"], workspace=wb, **kw)

    def timed(fn, K):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        e0.record(stream)
        for _ in range(K):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / K
        if world > 1:
            tt = torch.tensor([ms], device=dev, dtype=torch.float64)
            torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
            ms = float(tt.item())
        return ms

    K = args.steps
    with ClockSampler(local) as clocks:
        ms = timed(grouped_step, K)
    status = max(sla.hstu_sla_get_error(ws_f), sla.hstu_sla_get_error(ws_b))
    if status != 0:
        raise RuntimeError(f"device status {status}")
    ms_sep = timed(separate_step, K)
    if rank == 0:
        peaks, src = _peaks()
        peak = float(peaks.get("bf16_tflops_sustained") or peaks.get("bf16_tflops"))
        value = world * fl / (ms * 1e-3) / 1e12
        print(json.dumps({
            "metric": "MoT channels SLA attn fwd+bwd TFLOP/s (unmasked pairs), grouped launch",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16, jagged lengths per channel recipe)",
            "config": {"workload": "mot", "channels": chans,
                       "l2": "inputs > 126 MB L2; no flush"},
            "separate_calls_ms_per_step": ms_sep, "grouped_speedup": ms_sep / ms,
            "frac_of_sustained_peak": value / world / peak,
            "frac_of_burst_peak": value / world / float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])),
            # forward: 3 work lists + 1 kernel; backward: 3 work lists + 1 kernel
            # + 3 dq conversions (memsets not counted)
            "gpu_launches": K * (3 + 1 + 3 + 1 + 3),
            "clocks": clocks.summary()}), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="hist16k", choices=sorted(WORKLOADS) + ["mot"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-overlap", action="store_true",
                    help="run the backward's preparation inside the backward call instead of "
                         "beside the forward on a side stream")
    ap.add_argument("--strong", action="store_true",
                    help="N > 1: shard the workload's one batch across the GPUs (strong "
                         "scaling); by default N batches of the recipe are sharded (weak)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--rab", action="store_true",
                    help="attention workloads: with the relative attention bias (32 position and "
                         "32 time buckets per head, seeded tables and timestamps)")
    ap.add_argument("--fp8", action="store_true",
                    help="stu workload: E4M3 forward projections (weights requantized every step)")
    ap.add_argument("--remat", action="store_true",
                    help="stu workload: keep only the rematerialisation save set per layer "
                         "(u, attention output, norm statistics); the backward recomputes the rest")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        return run_reference(args)

    import sparse_hstu_attention_b200 as sla

    world, rank, local = _setup_dist(args)
    torch.cuda.set_device(local)
    if args.workload == "stu":
        return run_stu(args, world, rank, local)
    if args.workload == "mot":
        return run_mot(args, world, rank, local)
    dev = torch.device("cuda", local)
    w = WORKLOADS[args.workload]
    batch, shard_info = rank_batch(w, world, rank, strong=args.strong)
    T, H, d = batch.T, w.H, w.d
    pairs = F.total_pairs(batch.lengths, batch.num_targets, w.contextual_len, w.K1, w.K2)
    fl_f, fl_b = F.fwd_flops(pairs, H, d), (0.0 if w.fwd_only else F.bwd_flops(pairs, H, d))

    offs = torch.tensor(batch.seq_offsets, dtype=torch.int32, device=dev)
    nts = torch.tensor(batch.num_targets, dtype=torch.int32, device=dev)
    q, k, v = (t.to(dev) for t in (batch.q, batch.k, batch.v))
    dout = batch.dout.to(dev)
    out = torch.empty_like(q)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws_f = torch.empty(sla.hstu_sla_workspace_bytes(0, T, len(batch.lengths), H, d),
                       dtype=torch.uint8, device=dev)
    ws_b = torch.empty(sla.hstu_sla_workspace_bytes(1, T, len(batch.lengths), H, d),
                       dtype=torch.uint8, device=dev)
    kw = dict(contextual_len=w.contextual_len, K1=w.K1, K2=w.K2, alpha=w.alpha, N=w.N,
              max_seq_len=int(batch.lengths.max()))
    if args.rab:
        from workloads import draw_rab_tables, draw_timestamps
        rp, rt = draw_rab_tables(H, 32, 32, w.seed)
        kw.update(timestamps=torch.from_numpy(
            draw_timestamps(batch.lengths, batch.num_targets, w.seed)).to(dev),
            rab_pos=rp.to(dev), rab_time=rt.to(dev))
    stream = torch.cuda.current_stream()

    def new_events(n):
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
        for e in evs:
            e.record(stream)  # force creation of the underlying cudaEvent
        return evs

    K = args.steps
    fb, fe, bb, be = new_events(K), new_events(K), new_events(K), new_events(K)
    # The backward's preparation (its work list and the clear of its fp32 dQ
    # accumulator) reads only the batch geometry: it runs on a side stream
    # beside the forward, from the start of the step (the previous backward
    # is done with the workspace by then), and the backward waits for it.
    overlap = not w.fwd_only and not args.no_overlap
    prep_stream = torch.cuda.Stream(dev)
    ev_step, ev_prep = torch.cuda.Event(), torch.cuda.Event()
    kw_prep = {n: x for n, x in kw.items() if n not in ("timestamps", "rab_pos", "rab_time")}

    def step(i=None):
        evf = (fb[i], fe[i]) if i is not None else None
        evb = (bb[i], be[i]) if i is not None else None
        if overlap:
            ev_step.record(stream)
            prep_stream.wait_event(ev_step)
            sla.hstu_sla_bwd_prepare(q, offs, nts, workspace=ws_b, stream=prep_stream, **kw_prep)
            ev_prep.record(prep_stream)
        sla.hstu_sla_fwd(q, k, v, offs, nts, out=out, workspace=ws_f, events=evf, **kw)
        if not w.fwd_only:
            if overlap:
                stream.wait_event(ev_prep)
            sla.hstu_sla_bwd(dout, q, k, v, offs, nts, dq=dq, dk=dk, dv=dv, workspace=ws_b,
                             events=evb, prepared=overlap, **kw)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = max(sla.hstu_sla_get_error(ws_f), 0 if w.fwd_only else sla.hstu_sla_get_error(ws_b))
    if status != 0:
        raise RuntimeError(f"device status {status}")

    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        t_start.record(stream)
        for i in range(K):
            step(i)
        t_end.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
    ms = t_start.elapsed_time(t_end)
    job_fl = fl_f + fl_b  # every rank's FLOPs (the sharded ranks' work differs)
    if world > 1:
        tt = torch.tensor([ms], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
        ms = float(tt.item())
        ff = torch.tensor([job_fl], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(ff, op=torch.distributed.ReduceOp.SUM)
        job_fl = float(ff.item())
    ms_step = ms / K
    value = job_fl / (ms_step * 1e-3) / 1e12
    fwd_ms = sum(fb[i].elapsed_time(fe[i]) for i in range(K)) / K
    bwd_ms = 0.0 if w.fwd_only else sum(bb[i].elapsed_time(be[i]) for i in range(K)) / K

    # end to end through the public API from pinned host buffers: every step
    # copies its inputs in and its results out.  Two device buffer sets and
    # two copy streams pipeline the steps, so that step i's results travel
    # to the host while step i + 1's inputs travel to the device (PCIe is
    # full duplex) and the kernels run between them.
    hq, hk, hv, hdo = (t.pin_memory() for t in (batch.q, batch.k, batch.v, batch.dout))
    hoffs = torch.tensor(batch.seq_offsets, dtype=torch.int32).pin_memory()
    hnts = torch.tensor(batch.num_targets, dtype=torch.int32).pin_memory()
    hout = [torch.empty(q.shape, dtype=torch.bfloat16).pin_memory() for _ in range(4)]
    sets = [dict(q=q, k=k, v=v, dout=dout, offs=offs, nts=nts, out=out, dq=dq, dk=dk, dv=dv)]
    sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
    in_names = ["q", "k", "v", "dout", "offs", "nts"]
    out_names = ["out", "dq", "dk", "dv"]
    if w.fwd_only:
        in_names, out_names = ["q", "k", "v", "offs", "nts"], ["out"]
    hsrc = dict(q=hq, k=hk, v=hv, dout=hdo, offs=hoffs, nts=hnts)
    if args.rab:  # the timestamps are per-token inputs too
        hsrc["ts"] = kw["timestamps"].cpu().pin_memory()
        for S in sets:
            S["ts"] = torch.empty_like(kw["timestamps"])
        in_names.append("ts")
    kw_e = {n: x for n, x in kw.items() if n != "timestamps"}
    h2d = sum(hsrc[n].numel() * hsrc[n].element_size() for n in in_names)
    d2h = sum(hout[j].numel() * hout[j].element_size() for j in range(len(out_names)))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def step_on(S):
        ts = dict(timestamps=S["ts"]) if "ts" in S else {}
        sla.hstu_sla_fwd(S["q"], S["k"], S["v"], S["offs"], S["nts"], out=S["out"],
                         workspace=ws_f, **kw_e, **ts)
        if not w.fwd_only:
            sla.hstu_sla_bwd(S["dout"], S["q"], S["k"], S["v"], S["offs"], S["nts"], dq=S["dq"],
                             dk=S["dk"], dv=S["dv"], workspace=ws_b, **kw_e, **ts)

    def e2e_run(n, start):
        """n pipelined steps after `start` (an event on the compute stream);
        returns the event of the last result copy."""
        ev = lambda: torch.cuda.Event()  # noqa: E731
        e_in, e_cmp, e_out = [], [], []
        s_in.wait_event(start)
        s_out.wait_event(start)
        for i in range(n):
            S = sets[i % 2]
            if i >= 2:
                s_in.wait_event(e_cmp[i - 2])  # set i % 2's inputs are free
            with torch.cuda.stream(s_in):
                for nm in in_names:
                    S[nm].copy_(hsrc[nm], non_blocking=True)
            e_in.append(ev())
            e_in[i].record(s_in)
            stream.wait_event(e_in[i])
            if i >= 2:
                stream.wait_event(e_out[i - 2])  # set i % 2's results are on the host
            step_on(S)
            e_cmp.append(ev())
            e_cmp[i].record(stream)
            s_out.wait_event(e_cmp[i])
            with torch.cuda.stream(s_out):
                for j, nm in enumerate(out_names):
                    hout[j].copy_(S[nm], non_blocking=True)
            e_out.append(ev())
            e_out[i].record(s_out)
        return e_out[-1]

    E = max(2, args.e2e_steps)
    warm = torch.cuda.Event()
    warm.record(stream)
    stream.wait_event(e2e_run(2, warm))
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    stream.wait_event(e2e_run(E, e0))
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / E
    # the pipelined steps read the same inputs: their last results equal the
    # device-timed loop's (forward and dK are deterministic)
    if not torch.equal(hout[0], out.cpu()) or \
            (not w.fwd_only and not torch.equal(hout[2], dk.cpu())):
        raise RuntimeError("end-to-end results differ from the device-timed loop's")
    if world > 1:
        tt = torch.tensor([e2e_ms], device=dev, dtype=torch.float64)
        torch.distributed.all_reduce(tt, op=torch.distributed.ReduceOp.MAX)
        e2e_ms = float(tt.item())

    if rank != 0:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return

    peaks, peak_src = _peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    clk = clocks.summary()
    dom = "bwd" if bwd_ms > fwd_ms else "fwd"
    dom_ms = bwd_ms if dom == "bwd" else fwd_ms
    dom_fl = fl_b if dom == "bwd" else fl_f
    dom_bytes = (F.bwd_bytes if dom == "bwd" else F.fwd_bytes)(T, H, d)
    roof = roofline(dom_fl, dom_bytes, dom_ms, peaks, peak_src, clk)
    roof.update(kernel=KERNEL_NAMES[dom], traffic=_traffic(dom, w.name))
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if args.strong else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, jagged lengths drawn per workload recipe)",
        "config": dict(_config(w, batch), **(
            {"relative_attention_bias": {"pos_buckets": 32, "time_buckets": 32}}
            if args.rab else {}), **({"sharding": shard_info} if shard_info else {})),
        "bwd_prepare": ("side stream, beside the forward" if overlap else
                        "inside the backward call") if not w.fwd_only else None,
        "pct_of_peak": 100.0 * value / world / peak,
        "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
        "fwd_tflops": fl_f / (fwd_ms * 1e-3) / 1e12 if fwd_ms else None,
        "bwd_tflops": fl_b / (bwd_ms * 1e-3) / 1e12 if bwd_ms else None,
        "roofline": roof,
        "e2e": {"value": job_fl / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": K * (LAUNCHES_PER_STEP["fwd"] +
                             (0 if w.fwd_only else LAUNCHES_PER_STEP["bwd"])),
        "clocks": clk,
    }
    if w.fwd_only:
        # M-FALCON candidate scoring on the same batch: only the query tiles that
        # hold candidates (history K/V as the cache); FLOPs over candidate pairs
        cp = F.candidate_pairs(batch.lengths, batch.num_targets, w.contextual_len, w.K1, w.K2)
        cev = new_events(2)
        for _ in range(3):
            sla.hstu_sla_fwd(q, k, v, offs, nts, out=out, workspace=ws_f, candidates_only=True, **kw)
        torch.cuda.synchronize()
        cev[0].record(stream)
        for _ in range(K):
            sla.hstu_sla_fwd(q, k, v, offs, nts, out=out, workspace=ws_f, candidates_only=True, **kw)
        cev[1].record(stream)
        torch.cuda.synchronize()
        c_ms = cev[0].elapsed_time(cev[1]) / K
        line["candidate_scoring"] = {
            "ms_per_call": c_ms, "candidate_rows": int(batch.num_targets.sum()),
            "candidate_pairs_per_head": cp,
            "tflops": F.fwd_flops(cp, H, d) / (c_ms * 1e-3) / 1e12,
            "speedup_vs_full_forward": ms_step / c_ms}
    if world == 1 and not args.no_cpu_baseline:
        rab_o = None
        if args.rab:  # the same tables and timestamps, in the oracle's types
            rab_o = dict(timestamps=kw["timestamps"].cpu().numpy().astype(np.int64),
                         rab_pos=kw["rab_pos"].cpu().numpy().astype(np.float64),
                         rab_time=kw["rab_time"].cpu().numpy().astype(np.float64))
        line["cpu_baseline"] = cpu_baseline(batch, rab=rab_o)
    print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
