#!/usr/bin/env python
"""Benchmark of the DSA forward path on B200: 128K-token prefill tokens/s
(headline) and batch-64 paged decode tokens/s, each with its roofline fraction.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One process per GPU (torchrun for N > 1). The path has no cross-GPU exchange:
each rank runs its own full workload (independent sequences), so scaling is
weak and `value` is the tokens of all ranks divided by the slowest rank's time.
Rank 0 prints one JSON line.

A prefill step is one dsa_forward over L=131072 tokens (indexer -> top-k ->
sparse attention) with every input already resident in HBM; the inputs are far
larger than L2 (q alone is 19.3 GB). A decode step is one dsa_forward over 64
sequences; L2 is flushed before every decode step, outside the timed events.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DSA prefill tokens/s at 128K and decode tokens/s (1 B200) + % of roofline"

DECODE_WL = 4


# ----------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16": d["bf16_tflops"],
                "bf16_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


def measure_fp8_peak(n=8192, reps=10, sustain_s=3.0):
    """Dense FP8 (e4m3 x e4m3 -> bf16, f32 accumulate) tensor throughput of this
    GPU, measured with the library GEMM torch._scaled_mm on n^3 (2 n^3 flops):
    best of `reps` single calls (burst) and ~sustain_s seconds of calls back to
    back (sustained, the figure for a kernel timed inside a long step). Both
    the default and the fast-accumulation GEMM are tried; the faster counts."""
    a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn).t()   # column-major
    one = torch.ones((), device="cuda")
    flops = 2.0 * n ** 3
    best = {}
    for fast in (False, True):
        def mm():
            return torch._scaled_mm(a, b, one, one, out_dtype=torch.bfloat16,
                                    use_fast_accum=fast)
        for _ in range(3):
            mm()
        torch.cuda.synchronize()
        t = []
        for _ in range(reps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            mm()
            e1.record()
            torch.cuda.synchronize()
            t.append(e0.elapsed_time(e1))
        burst_ms = min(t)
        iters = max(10, int(sustain_s * 1e3 / burst_ms))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            mm()
        e1.record()
        torch.cuda.synchronize()
        sus_ms = e0.elapsed_time(e1) / iters
        best[fast] = (flops / (burst_ms * 1e-3) / 1e12, flops / (sus_ms * 1e-3) / 1e12)
    fast = max(best, key=lambda f: best[f][0])
    del a, b
    torch.cuda.empty_cache()
    return {"fp8_tflops": best[fast][0], "fp8_tflops_sustained": best[fast][1],
            "how": f"torch._scaled_mm e4m3 {n}^3, bf16 out, use_fast_accum={fast}: best of "
                   f"{reps} (burst) and ~{sustain_s:.0f} s back to back (sustained)",
            "default_accum_tflops": best[False][0], "fast_accum_tflops": best[True][0]}


def kernel_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes of `kernel` on `workload` from the committed ncu
    summary, or None when it was captured on another workload or the kernel's
    source changed since the capture."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel)
    if not d or d.get("workload") != workload:
        return None
    src = os.path.join(ROOT, "sparse_attention_long_tcgen05_b200", "csrc", d["source"])
    if not os.path.exists(src):
        return None
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return d["bytes_per_launch"] if sha == d.get("source_sha") else None


class Clocks:
    """nvidia-smi sampling of SM clock and throttle reasons while timing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
              "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            self.proc.wait()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        with open(self.path) as f:
            lines = f.readlines()
        os.unlink(self.path)
        return self.parse(lines)

    @staticmethod
    def parse(lines):
        """Summary of `nvidia-smi --format=csv,noheader,nounits` lines of FIELDS:
        median SM clock under load (utilisation >= 50 %, else all samples), the
        maximum clock, the throttle reasons seen active, the largest power."""
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        rows = [[x.strip() for x in line.split(",")] for line in lines]
        rows = [r for r in rows if len(r) >= 10]
        if not rows:
            return None
        loaded = [r for r in rows if (num(r[4]) or 0) >= 50] or rows
        sm = [num(r[1]) for r in loaded if num(r[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i in range(4)
                          if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": num(loaded[0][2]), "reasons": reasons,
                "samples_under_load": len(loaded),
                "power_w_max": max((num(r[3]) or 0) for r in loaded)}


# Throttle reasons that reject a timed region (sw_power_cap is kept and noted).
REJECTING_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")


def clock_rejected(c):
    """Whether a clock summary rejects its timed region: a slowdown reason was
    active, or the SM clock sat well below its maximum with no reason given
    (a clock lock left by another process)."""
    if not c:
        return False
    if any(r in c["reasons"] for r in REJECTING_REASONS):
        return True
    sm, mx = c.get("sm_mhz"), c.get("sm_max_mhz")
    return bool(sm and mx and not c["reasons"] and sm < 0.85 * mx)


def any_rank(flag, world):
    """True on every rank if `flag` is true on any (all ranks must call it)."""
    if world == 1:
        return bool(flag)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([1 if flag else 0], dtype=torch.int32, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return bool(t.item())


def dist_env():
    """(world, rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def dist_setup():
    """One process per GPU: NCCL over the node's GPUs, or gloo on a host
    without one (the host logic below is the same)."""
    world, rank, local = dist_env()
    cuda = torch.cuda.is_available()
    if cuda:
        torch.cuda.set_device(local)
    if world > 1:
        import datetime
        kw = {"device_id": torch.device("cuda", local)} if cuda else {}
        torch.distributed.init_process_group("nccl" if cuda else "gloo",
                                             timeout=datetime.timedelta(seconds=300), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, units_per_rank: float, ms: float) -> float:
    """Whole-job throughput: every rank processes `units_per_rank` in a step,
    the step takes `ms` on the slowest rank."""
    return world * units_per_rank / (ms * 1e-3)


def timed(fn, steps, warmup, world, pre=None):
    """Average ms per call of fn() over `steps` calls, CUDA events on the
    current stream, warm-up first, barrier + synchronize on both sides, max
    over ranks. `pre` (untimed) runs before every call when given."""
    for _ in range(warmup):
        if pre:
            pre()
        fn()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    if pre is None:
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / steps
    else:
        total = 0.0
        for _ in range(steps):
            pre()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            total += a.elapsed_time(b)
        ms = total / steps
    barrier(world)
    torch.cuda.synchronize()
    return max_over_ranks(ms, world)


def pinned_copy(t: torch.Tensor) -> torch.Tensor:
    h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
    h.copy_(t)
    return h


def attention_pairs(L, k):
    """Selected (query, key) pairs of a causal prefill: sum_t min(k, t+1)."""
    m = min(k, L)
    return m * (m + 1) // 2 + (L - m) * k


# ----------------------------------------------------------------- our arm

def run_ours(args, world, rank, local):
    from sparse_attention_long_tcgen05_b200 import _build
    if rank == 0 or not os.path.exists(_build.LIB):
        _build.build()
    barrier(world)
    from sparse_attention_long_tcgen05_b200 import dsa
    from sparse_attention_long_tcgen05_b200.inputs import WORKLOADS, make_prefill, make_decode

    peaks = load_peaks()
    if args.decode_only:    # profiling aid: the decode step alone
        dwl = WORKLOADS[DECODE_WL]
        if args.decode_ctx_max:
            import dataclasses
            dwl = dataclasses.replace(dwl, name=f"decode_B64_ctx{args.decode_ctx_max}",
                                      ctx_min=min(dwl.ctx_min, args.decode_ctx_max // 2),
                                      ctx_max=args.decode_ctx_max)
        return {"decode": run_decode(args, world, rank, local, peaks, dsa, make_decode, dwl)}
    wl = next(w for w in WORKLOADS.values() if w.name == args.workload)
    L, k = wl.L, wl.k
    inp = make_prefill(wl, device="cuda", seed=rank)
    ind = dsa.indexer_in(inp.q_idx, inp.k_idx, inp.w, inp.q_scale, inp.k_scale)
    att = dsa.attn_in(inp.q, inp.kv, wl.scale, wl.D_V)
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, ind, att, 0, 0, k))
    idx = torch.empty(L, k, dtype=torch.int32, device="cuda")
    out = torch.empty(L, wl.H, wl.D_V, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(L, wl.H, device="cuda")

    def fwd():
        dsa.dsa_forward(ind, att, k, idx, out, lse, ws)

    def sel():
        dsa.dsa_select(ind, k, idx, ws)

    def attn():
        dsa.dsa_sparse_mqa_fwd(att, idx, k, out, lse)

    # the indexer alone, launched over the same blocks of query rows as the
    # fused selection (each block's rows against keys 0..last row of the block)
    sel_bytes = dsa.dsa_workspace_size(dsa.DSA_OP_SELECT, ind, None, 0, 0, k)
    chunk = max(1, min(L, sel_bytes // (L * 4)))
    rows_all = torch.arange(L, dtype=torch.int32, device="cuda")
    blocks = [(q0, min(chunk, L - q0)) for q0 in range(0, L, chunk)]
    ws_f = ws[: (sel_bytes // 4) * 4].view(torch.float32)

    def indexer_alone():
        for q0, rows in blocks:
            cols = q0 + rows
            dsa.dsa_indexer_scores(ind, rows_all[q0:q0 + rows], rows,
                                   ws_f[: rows * cols].view(rows, cols), cols)

    def measure():
        with Clocks(local) as clk:
            n0 = dsa.dsa_launch_counter()
            t = timed(fwd, args.steps, args.warmup, world)
            n = dsa.dsa_launch_counter() - n0
        return t, n, clk.summary()

    ms, launches, clocks = measure()
    # a timed region that any rank saw throttled (or clock-locked) is timed
    # once more on every rank; the line keeps the second and shows the first
    if any_rank(clock_rejected(clocks), world):
        first = clocks
        ms, launches, clocks = measure()
        clocks = dict(clocks or {}, remeasured_after=first)
    st = dsa.dsa_check_status()
    if st != 0:
        raise RuntimeError(f"device status {dsa.status_string(st)}")
    # launches counted above include the warm-up calls: scale to the timed ones
    per_call = launches / (args.steps + args.warmup)
    ms_sel = timed(sel, args.steps, 1, world)
    ms_attn = timed(attn, args.steps, 1, world)
    ms_idx = timed(indexer_alone, args.steps, 1, world)
    st = dsa.dsa_check_status()
    if st != 0:
        raise RuntimeError(f"device status {dsa.status_string(st)}")
    fp8 = measure_fp8_peak() if not args.skip_fp8_peak else None
    fp8_sus = fp8["fp8_tflops_sustained"] if fp8 else 2.0 * peaks["bf16_sustained"]
    fp8_note = ("FP8 dense sustained, measured in this run (torch._scaled_mm)" if fp8 else
                f"2 x bf16 dense sustained ({peaks['source']}; nominal FP8/bf16 ratio)")

    idx_flops = 2.0 * wl.H_I * wl.d_I * (L * (L + 1) / 2)
    attn_flops = 2.0 * wl.H * (wl.D_K + wl.D_V) * attention_pairs(L, k)
    idx_tf = idx_flops / (ms_idx * 1e-3) / 1e12
    sel_tf = idx_flops / (ms_sel * 1e-3) / 1e12
    attn_tf = attn_flops / (ms_attn * 1e-3) / 1e12
    stages = {
        "select_ms": ms_sel, "select_fp8_tflops": sel_tf,
        "indexer_ms": ms_idx, "indexer_launches": len(blocks), "indexer_rows_per_launch": chunk,
        "indexer_fp8_tflops": idx_tf,
        "indexer_frac_fp8_sustained": idx_tf / fp8_sus,
        "indexer_frac_fp8_nominal_2x_bf16_sustained": idx_tf / (2.0 * peaks["bf16_sustained"]),
        "topk_ms_estimate": ms_sel - ms_idx,
        "attention_ms": ms_attn, "attention_bf16_tflops": attn_tf,
        "attention_frac_bf16_sustained": attn_tf / peaks["bf16_sustained"],
        "indexer_flops": idx_flops, "attention_flops": attn_flops,
    }
    rooflines = {
        "indexer_fp8_kernel": {
            "bound": "tensor", "achieved": idx_tf, "peak": fp8_sus, "unit": "TFLOP/s",
            "frac": idx_tf / fp8_sus, "peak_note": fp8_note,
            "algorithmic": "2*64*128 FP8 flops per (t, s<=t) pair, L(L+1)/2 pairs",
            "launches": len(blocks), "ms": ms_idx,
            "traffic": kernel_traffic("indexer_fp8_kernel", wl.name)},
        "sparse_mqa_bf16_kernel": {
            "bound": "tensor", "achieved": attn_tf, "peak": peaks["bf16_sustained"],
            "unit": "TFLOP/s", "frac": attn_tf / peaks["bf16_sustained"],
            "peak_note": f"bf16 dense sustained ({peaks['source']})",
            "algorithmic": "2*128*(576+512) bf16 flops per selected (t, key) pair",
            "launches": 1, "ms": ms_attn,
            "traffic": kernel_traffic("sparse_mqa_bf16_kernel", wl.name)},
    }
    # the headline roofline is that of the kernel with the largest share of the step
    dom = "indexer_fp8_kernel" if ms_idx > ms_attn else "sparse_mqa_bf16_kernel"
    roof = dict(rooflines[dom], kernel=dom)

    curve = None
    if not args.skip_curve:
        curve = cost_vs_position(dsa, inp, wl, k, world, peaks)
    kl = None
    if not args.skip_kl:
        kl = indexer_kl_signal(dsa, inp, wl, ind, att, ws, idx, out, lse, k, world, peaks)
    bwd = None
    if not args.skip_bwd:
        bwd = attention_backward(dsa, wl, att, idx, out, lse, k, world, peaks)
        rooflines["sparse_mqa_bwd_kernel"] = {
            "bound": "tensor", "achieved": bwd["bf16_tflops"], "peak": peaks["bf16_sustained"],
            "unit": "TFLOP/s", "frac": bwd["frac_bf16_sustained"],
            "peak_note": f"bf16 dense sustained ({peaks['source']})",
            "algorithmic": "2*128*(2*576+576+2*512) bf16 flops per selected (t, key) pair",
            "launches": 1, "ms": bwd["ms"],
            "traffic": kernel_traffic("sparse_mqa_bwd_kernel", wl.name)}

    # ------------------------------------------------------------ e2e (host buffers)
    e2e = None
    if not args.skip_e2e:
        try:
            e2e = prefill_e2e(dsa, inp, ind, att, ws, idx, out, lse, k, args, world)
        except Exception as ex:  # pinned-memory limits on the host
            e2e = {"value": None, "unit": "tokens/s", "error": str(ex)[:200]}

    # ------------------------------------------------------------ cpu baseline
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        cpu = oracle_prefill_rate(inp, wl, budget_s=args.cpu_budget)

    value_tok = job_rate(world, L, ms)
    res = {
        "metric": METRIC, "value": value_tok, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3+bf16 (f32 accumulate)", "data": "synthetic",
        "config": workload_config(wl, world),
        "roofline": roof, "rooflines": rooflines, "fp8_peak": fp8, "stages": stages,
        "cpu_baseline": cpu, "e2e": e2e, "cost_vs_position": curve, "indexer_kl": kl,
        "attention_backward": bwd,
        "gpu_launches": int(round(per_call * args.steps)),
        "clocks": clocks,
    }
    del inp, out, idx, lse, ws
    torch.cuda.empty_cache()
    if not args.skip_decode:
        res["decode"] = run_decode(args, world, rank, local, peaks, dsa, make_decode,
                                   WORKLOADS[DECODE_WL])
    return res


def cost_vs_position(dsa, inp, wl, k, world, peaks, block=4096, steps=2,
                     positions=(4096, 8192, 16384, 32768, 65536, 98304, 131072)):
    """Prefill cost per token position: for each P, the block of `block`
    queries at positions P-block .. P-1 against keys 0..P-1 (a chunk of the
    prefill), timed once through dsa_forward (indexer -> top-k -> sparse
    attention) and once through dsa_dense_mqa_fwd (dense causal attention, the
    baseline DSA replaces), on the same inputs. ms per block of queries."""
    out = torch.empty(block, wl.H, wl.D_V, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(block, wl.H, device="cuda")
    idx = torch.empty(block, k, dtype=torch.int32, device="cuda")
    pts = []
    for P in positions:
        if P > wl.L or P < block:
            continue
        off = P - block
        ind = dsa.indexer_in(inp.q_idx[off:P], inp.k_idx[:P], inp.w[off:P], inp.q_scale[off:P],
                             inp.k_scale[:P])
        att = dsa.attn_in(inp.q[off:P], inp.kv[:P], wl.scale, wl.D_V)
        ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, ind, att, 0, 0, k))
        ms_dsa = timed(lambda: dsa.dsa_forward(ind, att, k, idx, out, lse, ws), steps, 1, world)
        ms_dense = timed(lambda: dsa.dsa_dense_mqa_fwd(att, out, lse), steps, 1, world)
        st = dsa.dsa_check_status()
        if st != 0:
            raise RuntimeError(f"device status {dsa.status_string(st)}")
        keys = block * (off + 1) + block * (block - 1) // 2          # sum of (t + 1)
        dense_tf = 2.0 * wl.H * (wl.D_K + wl.D_V) * keys / (ms_dense * 1e-3) / 1e12
        pts.append({"position": P, "dsa_ms": ms_dsa, "dense_ms": ms_dense,
                    "dense_over_dsa": ms_dense / ms_dsa, "dense_bf16_tflops": dense_tf,
                    "dense_frac_bf16_sustained": dense_tf / peaks["bf16_sustained"]})
        del ws
    return {"block_queries": block, "unit": "ms per block of queries", "points": pts,
            "how": "queries P-block..P-1 against keys 0..P-1 of the 128K inputs; dsa = "
                   "dsa_forward (indexer, top-k, sparse attention), dense = dsa_dense_mqa_fwd"}


def indexer_kl_signal(dsa, inp, wl, ind, att, ws, idx, out, lse, k, world, peaks, steps=2):
    """The indexer's KL training signal over the whole prefill (what a sparse
    training step adds to the forward): the selection with its kept scores
    (dsa_select_scored) and the signal (dsa_indexer_kl) from the forward's lse.
    The KL kernel recomputes q.k for all 128 heads and 576 dims of every
    selected pair: 2 * 128 * 576 flops per pair."""
    L = wl.L
    sel = torch.empty(L, k, device="cuda")
    loss = torch.empty(L, device="cuda")
    grad = torch.empty(L, k, device="cuda")
    dsa.dsa_forward(ind, att, k, idx, out, lse, ws)
    ms_sel = timed(lambda: dsa.dsa_select_scored(ind, k, idx, sel, ws), steps, 1, world)
    ms_kl = timed(lambda: dsa.dsa_indexer_kl(att, idx, k, lse, sel, loss, grad), steps, 1, world)
    st = dsa.dsa_check_status()
    if st != 0:
        raise RuntimeError(f"device status {dsa.status_string(st)}")
    flops = 2.0 * wl.H * wl.D_K * attention_pairs(L, k)
    tf = flops / (ms_kl * 1e-3) / 1e12
    res = {"select_scored_ms": ms_sel, "indexer_kl_ms": ms_kl, "kl_bf16_tflops": tf,
           "kl_frac_bf16_sustained": tf / peaks["bf16_sustained"],
           "mean_loss": float(loss.mean()),
           "how": "dsa_select_scored + dsa_indexer_kl over the 128K prefill, lse from dsa_forward"}
    del sel, loss, grad
    return res


def attention_backward(dsa, wl, att, idx, out, lse, k, world, peaks, steps=2):
    """Gradient of the sparse attention over the 128K prefill's own selection
    (the main model's side of a sparse training step): dsa_sparse_mqa_bwd with
    a seeded upstream gradient, given the forward's out and lse. Per selected
    (t, key) pair it recomputes the logits and dP and forms the query, key and
    value gradients: 2*128*(576 + 512 + 576 + 576 + 512) flops."""
    from sparse_attention_long_tcgen05_b200.inputs import make_grad_out
    L = wl.L
    d_out = make_grad_out(L, wl.H, wl.D_V, device="cuda", seed=71)
    dq = torch.empty(L, wl.H, wl.D_K, dtype=torch.bfloat16, device="cuda")
    dkv = torch.zeros(L, wl.D_K, device="cuda")
    delta = torch.empty(L, wl.H, 2, device="cuda")
    ms = timed(lambda: dsa.dsa_sparse_mqa_bwd(att, idx, k, out, lse, d_out, dq, dkv, delta),
               steps, 1, world)
    st = dsa.dsa_check_status()
    if st != 0:
        raise RuntimeError(f"device status {dsa.status_string(st)}")
    flops = 2.0 * wl.H * (2 * wl.D_K + wl.D_K + 2 * wl.D_V) * attention_pairs(L, k)
    tf = flops / (ms * 1e-3) / 1e12
    del d_out, dq, dkv, delta
    return {"ms": ms, "bf16_tflops": tf, "frac_bf16_sustained": tf / peaks["bf16_sustained"],
            "flops": flops, "launches": 2,
            "how": "dsa_sparse_mqa_bwd (row-dot kernel for D, then the tcgen05 backward) over "
                   "the 128K selection of dsa_forward; dkv accumulated in fp32"}


def profile_backward(L: int):
    """The attention backward alone on an L-token prefill of the 128K
    workload's shapes (seeded inputs; selection from random_selection), one
    warm-up launch and three timed ones: the command the backward's ncu
    summaries are taken with."""
    import dataclasses
    from sparse_attention_long_tcgen05_b200 import dsa
    from sparse_attention_long_tcgen05_b200.inputs import (WORKLOADS, make_grad_out,
                                                           make_prefill, random_selection)
    wl = dataclasses.replace(WORKLOADS[3], name=f"prefill_L{L}", L=L)
    k = wl.k
    inp = make_prefill(wl, device="cuda", seed=0)
    idx = random_selection(L, L, k, device="cuda", seed=70)
    d_out = make_grad_out(L, wl.H, wl.D_V, device="cuda", seed=71)
    att = dsa.attn_in(inp.q, inp.kv, wl.scale, wl.D_V)
    out = torch.empty(L, wl.H, wl.D_V, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(L, wl.H, device="cuda")
    dsa.dsa_sparse_mqa_fwd(att, idx, k, out, lse)
    dq = torch.empty(L, wl.H, wl.D_K, dtype=torch.bfloat16, device="cuda")
    dkv = torch.zeros(L, wl.D_K, device="cuda")
    delta = torch.empty(L, wl.H, 2, device="cuda")
    run = lambda: dsa.dsa_sparse_mqa_bwd(att, idx, k, out, lse, d_out, dq, dkv, delta)
    ms = timed(run, 3, 1, 1)
    st = dsa.dsa_check_status()
    if st != 0:
        raise RuntimeError(f"device status {dsa.status_string(st)}")
    pairs = int((idx >= 0).sum())
    tf = 2.0 * wl.H * (2 * wl.D_K + wl.D_K + 2 * wl.D_V) * pairs / (ms * 1e-3) / 1e12
    return {"profile": "attention_backward", "L": L, "k": k, "ms": ms, "pairs": pairs,
            "bf16_tflops": tf}


def prefill_e2e(dsa, inp, ind, att, ws, idx, out, lse, k, args, world, n_chunks=8):
    """Same metric through the public calls with HOST buffers: every step copies
    all of its inputs from pinned host memory and reads the attention output and
    lse back, and the copies overlap the kernels. The indexer-side inputs and the
    latent cache go up first; q (19.3 GB at 128K) streams up in n_chunks row
    chunks on a copy stream while dsa_select runs; dsa_sparse_mqa_fwd then runs
    chunk by chunk as each chunk's q lands (the chunk's queries are the suffix
    of the first c1 keys, so positions are unchanged), and each chunk's output
    goes back on a second copy stream while the next chunk computes."""
    wl = inp.wl
    L = wl.L
    small = [inp.q_idx, inp.q_scale, inp.k_idx, inp.k_scale, inp.w, inp.kv]
    host_small = [pinned_copy(t) for t in small]
    host_q = pinned_copy(inp.q)
    host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    host_lse = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    bounds = [(L * c // n_chunks, L * (c + 1) // n_chunks) for c in range(n_chunks)]
    atts = [dsa.attn_in(inp.q[c0:c1], inp.kv[:c1], wl.scale, wl.D_V) for c0, c1 in bounds]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def step():
        comp = torch.cuda.current_stream()
        go = torch.cuda.Event()
        go.record(comp)
        ev_small, ev_q, ev_o = torch.cuda.Event(), [], []
        with torch.cuda.stream(s_in):
            s_in.wait_event(go)
            for h, d in zip(host_small, small):
                d.copy_(h, non_blocking=True)
            ev_small.record(s_in)
            for c0, c1 in bounds:
                inp.q[c0:c1].copy_(host_q[c0:c1], non_blocking=True)
                ev_q.append(torch.cuda.Event())
                ev_q[-1].record(s_in)
        comp.wait_event(ev_small)
        dsa.dsa_select(ind, k, idx, ws)
        for c, (c0, c1) in enumerate(bounds):
            comp.wait_event(ev_q[c])
            dsa.dsa_sparse_mqa_fwd(atts[c], idx[c0:c1], k, out[c0:c1], lse[c0:c1])
            ev_o.append(torch.cuda.Event())
            ev_o[-1].record(comp)
        with torch.cuda.stream(s_out):
            for c, (c0, c1) in enumerate(bounds):
                s_out.wait_event(ev_o[c])
                host_out[c0:c1].copy_(out[c0:c1], non_blocking=True)
                host_lse[c0:c1].copy_(lse[c0:c1], non_blocking=True)
            done = torch.cuda.Event()
            done.record(s_out)
        comp.wait_event(done)

    ms = timed(step, args.e2e_steps, 1, world)
    h2d = sum(t.numel() * t.element_size() for t in host_small) + \
        host_q.numel() * host_q.element_size()
    d2h = host_out.numel() * host_out.element_size() + host_lse.numel() * 4
    return {"value": job_rate(world, L, ms), "unit": "tokens/s", "ms_per_step": ms,
            "steps": args.e2e_steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "how": f"pinned host buffers; dsa_select + {n_chunks} chunked dsa_sparse_mqa_fwd "
                   "calls, host<->device copies on two copy streams overlapping the kernels"}


def workload_config(wl, world):
    """The `config` object of a prefill line, shared by both arms."""
    q_gb = wl.L * wl.H * wl.D_K * 2 / 1e9
    return {"workload": wl.name, "L": wl.L, "k": wl.k, "H_I": wl.H_I, "d_I": wl.d_I,
            "H": wl.H, "d_qk": wl.D_K, "d_v": wl.D_V, "seed": "rank",
            "l2": f"inputs larger than L2 (q alone {q_gb:.1f} GB)",
            "parallelism": f"replicas x{world} (independent sequences)"}


def oracle_prefill_rate(inp, wl, budget_s=15.0, rows_cap=None):
    """The CPU oracle as it stands on a bounded sample of query rows of the same
    workload (uniform rows, so the mean prefix is ~L/2): tokens/s = rows/wall."""
    import numpy as np
    from oracle import dsa_oracle as O
    from sparse_attention_long_tcgen05_b200.inputs import sample_rows
    try:
        from threadpoolctl import threadpool_info
        cores = max((p.get("num_threads") or 0) for p in threadpool_info()) or os.cpu_count()
    except Exception:
        cores = os.cpu_count()
    rows = sample_rows(wl.L, 512, seed=1)
    rng = np.random.default_rng(2)
    rng.shuffle(rows)
    k_deq = O.dequantize(inp.k_idx.cpu().numpy(), inp.k_scale.cpu().numpy())
    kv = inp.kv.cpu()
    done = 0
    t0 = time.time()
    for t in rows:
        if time.time() - t0 > budget_s or (rows_cap and done >= rows_cap):
            break
        q_deq = O.dequantize(inp.q_idx[t].cpu().numpy()[None], inp.q_scale[t:t + 1].cpu().numpy())
        sc = O.indexer_row(q_deq[0], k_deq[: t + 1], inp.w[t].double().cpu().numpy())
        sel = O.topk_row(sc, t, wl.k)
        sel = sel[sel >= 0]
        keys = kv[torch.from_numpy(sel).long()].double().numpy()
        O.attend(inp.q[t].double().cpu().numpy(), keys, keys[:, : wl.D_V], wl.scale)
        done += 1
    wall = time.time() - t0
    return {"value": done / wall, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{done} uniformly drawn query rows of {wl.name} "
                      f"(indexer+top-k+attention per row, float64), {wall:.1f} s wall"}


def run_decode(args, world, rank, local, peaks, dsa, make_decode, wl):
    inp = make_decode(wl, device="cuda", seed=rank)
    lay = dsa.paged_layout(inp.block_table, inp.ctx_lens, inp.num_pages)
    ind = dsa.indexer_in(inp.q_idx, inp.k_cache, inp.w, inp.q_scale, inp.k_cache_scale.view(-1),
                         kv=lay)
    att = dsa.attn_in(inp.q, inp.kv_cache, wl.scale, wl.D_V, kv_layout=lay)
    B, k = inp.q.shape[0], wl.k
    ws = dsa.workspace(dsa.dsa_workspace_size(dsa.DSA_OP_FORWARD, ind, att, 0, 0, k))
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    out = torch.empty(B, wl.H, wl.D_V, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, wl.H, device="cuda")
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    flush_buf = torch.empty(2 * l2 // 4 + 1024, dtype=torch.float32, device="cuda")

    def flush():
        flush_buf.fill_(1.0)

    def fwd():
        dsa.dsa_forward(ind, att, k, idx, out, lse, ws)

    def sel():
        dsa.dsa_select(ind, k, idx, ws)

    def attn():
        dsa.dsa_sparse_mqa_fwd(att, idx, k, out, lse)

    steps = max(args.steps, 10)
    ms = timed(fwd, steps, args.warmup, world, pre=flush)
    ms_sel = timed(sel, steps, 1, world, pre=flush)
    ms_attn = timed(attn, steps, 1, world, pre=flush)
    ctx = inp.ctx_lens.long()
    n_sel = torch.clamp(ctx, max=k)
    scan_bytes = float((ctx * (wl.d_I + 4)).sum())
    gather_bytes = float((n_sel * wl.D_K * 2).sum())
    qo_bytes = B * (wl.H * wl.D_K * 2 + wl.H * wl.D_V * 2 + wl.H * 4 + wl.H_I * wl.d_I +
                    wl.H_I * 4 + 4)
    step_bytes = scan_bytes + gather_bytes + qo_bytes
    hbm = peaks["hbm_gbs"]
    sel_gbs = (scan_bytes + B * (wl.H_I * wl.d_I + wl.H_I * 4)) / (ms_sel * 1e-3) / 1e9
    attn_gbs = (gather_bytes + B * (wl.H * wl.D_K * 2 + wl.H * wl.D_V * 2)) / (ms_attn * 1e-3) / 1e9
    step_gbs = step_bytes / (ms * 1e-3) / 1e9
    # e2e: the caches stay resident; per step the new query tensors go up and
    # the attention output comes back
    e2e = None
    if not args.skip_e2e:
        dev_in = [inp.q_idx, inp.q_scale, inp.w, inp.q, inp.ctx_lens, inp.block_table]
        host_in = [pinned_copy(t) for t in dev_in]
        host_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()

        def step():
            for h, d in zip(host_in, dev_in):
                d.copy_(h, non_blocking=True)
            fwd()
            host_out.copy_(out, non_blocking=True)
        ms_e2e = timed(step, steps, 1, world, pre=flush)
        e2e = {"value": job_rate(world, B, ms_e2e), "unit": "tokens/s", "ms_per_step": ms_e2e,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in host_in),
               "d2h_bytes_per_step": host_out.numel() * host_out.element_size()}
    return {
        "workload": wl.name, "value": job_rate(world, B, ms), "unit": "tokens/s",
        "ms_per_step": ms, "steps": steps, "l2": "flushed before every step (untimed)",
        "mean_ctx": float(ctx.float().mean()),
        "roofline": {"kernel": "whole decode step", "bound": "hbm", "achieved": step_gbs,
                     "peak": hbm, "unit": "GB/s", "frac": step_gbs / hbm,
                     "algorithmic_bytes_per_step": step_bytes, "traffic": None},
        "rooflines": {
            # the sparse gather: every selected latent row once (1152 B) + q in, O out
            "sparse_mqa_bf16_kernel": {
                "bound": "hbm", "achieved": attn_gbs, "peak": hbm, "unit": "GB/s",
                "frac": attn_gbs / hbm, "ms": ms_attn,
                "algorithmic_bytes": gather_bytes + B * (wl.H * wl.D_K * 2 + wl.H * wl.D_V * 2),
                "algorithmic": "sum_b min(k, ctx_b) * 1152 B + q (147 KB) + O (131 KB) per "
                               "sequence",
                "traffic": kernel_traffic("sparse_mqa_bf16_kernel", wl.name)},
            # the key-cache scan of the indexer (+ its top-k): every cached key's
            # e4m3 row and scale once, q_I and w in
            "select (indexer_fp8_kernel + topk_kernel)": {
                "bound": "hbm", "achieved": sel_gbs, "peak": hbm, "unit": "GB/s",
                "frac": sel_gbs / hbm, "ms": ms_sel,
                "algorithmic_bytes": scan_bytes + B * (wl.H_I * wl.d_I + wl.H_I * 4),
                "algorithmic": "sum_b ctx_b * 132 B + q_I (8 KB) + w (256 B) per sequence",
                "traffic": kernel_traffic("indexer_fp8_kernel", wl.name)},
        },
        "stages": {"select_ms": ms_sel, "select_gbs": sel_gbs, "select_frac_hbm": sel_gbs / hbm,
                   "attention_ms": ms_attn, "attention_gbs": attn_gbs,
                   "attention_frac_hbm": attn_gbs / hbm},
        "e2e": e2e,
    }


# ----------------------------------------------------------------- reference arm

def run_reference(args, world, rank):
    """The oracle as it stands on the host cores: each step is a bounded sample
    of query rows of the same workload; tokens/s = rows / wall time, and
    ms_per_step the mean wall time of a timed step (a sample, not the whole
    workload)."""
    from sparse_attention_long_tcgen05_b200.inputs import WORKLOADS, make_prefill
    wl = next(w for w in WORKLOADS.values() if w.name == args.workload)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_prefill(wl, device=dev, seed=0)   # input generation only, untimed
    rates, walls = [], []
    for i in range(args.warmup + args.steps):
        t0 = time.time()
        r = oracle_prefill_rate(inp, wl, budget_s=args.ref_step_s)
        if i >= args.warmup:
            rates.append(r)
            walls.append(time.time() - t0)
    value = statistics.mean(r["value"] for r in rates)
    cpu = dict(rates[-1])
    cpu["value"] = value
    cpu["sample"] = (f"{args.steps} steps of ~{args.ref_step_s:.0f} s, each "
                     + rates[-1]["sample"])
    return {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * statistics.mean(walls),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": workload_config(wl, world),
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="prefill_L131072",
                    choices=["prefill_L4096", "prefill_L32768_needle", "prefill_L131072"],
                    help="prefill workload of the headline line (smaller ones for profiling)")
    ap.add_argument("--skip-decode", action="store_true")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode step (profiling aid; no headline value)")
    ap.add_argument("--decode-ctx-max", type=int, default=0,
                    help="with --decode-only: a smaller decode (context lengths up to this) "
                         "for multi-pass profiling")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-bwd", action="store_true",
                    help="skip the sparse attention backward record")
    ap.add_argument("--skip-kl", action="store_true",
                    help="skip the indexer KL training-signal measurement")
    ap.add_argument("--skip-curve", action="store_true",
                    help="skip the prefill cost-vs-position curve (DSA against dense)")
    ap.add_argument("--skip-fp8-peak", action="store_true",
                    help="do not measure the FP8 GEMM peak (the indexer is then reported "
                         "against 2 x the bf16 peak)")
    ap.add_argument("--profile-bwd", type=int, default=0, metavar="L",
                    help="run only the attention backward on an L-token prefill (seeded "
                         "inputs, random_selection), warm-up then 3 timed launches: a "
                         "profiling aid with no headline value")
    ap.add_argument("--e2e-steps", type=int, default=4)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-step-s", type=float, default=10.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        # the oracle on the host cores: rank 0 alone, no process group
        world, rank, _ = dist_env()
        if rank != 0:
            return
        print(json.dumps(run_reference(args, world, rank)), flush=True)
        return
    if args.profile_bwd:
        print(json.dumps(profile_backward(args.profile_bwd)), flush=True)
        return
    world, rank, local = dist_setup()
    res = run_ours(args, world, rank, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
