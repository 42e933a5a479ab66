#!/usr/bin/env python
"""Benchmark of the 4-bit FlashAttention forward hot path on B200.

One step = one pass of the hot path over one batch of the prefill workload
(Smooth-QK scale + FP4 quantize of Q, K, V, then the 4-bit attention forward);
the Smooth-QK calibration is offline and untimed.  The split-KV decode row is
measured in the same run on its own workload and reported under "decode".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Rank 0 prints one JSON line.  Multi-GPU: one process per GPU (torchrun); the
path has no data exchange, so each rank runs its own batch (weak scaling) and
the value is all ranks' work over the max-over-ranks device time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_quantized_flashattention_smooth_b200 import workloads as W  # noqa: E402

METRIC = "4-bit attention fwd TFLOPS and % of dense FP4 peak; decode KV GB/s vs HBM"
FP4_OVER_BF16 = 4.0   # nominal dense ratio: 9 PFLOP/s FP4 / 2.25 PFLOP/s BF16
L2_FLUSH_BYTES = 256 << 20


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sust=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, src="fallback")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    def __init__(self, index: int):
        import tempfile
        log_dir = os.environ.get("HIFA4_CLOCK_LOG_DIR", tempfile.gettempdir())
        self.path = os.path.join(log_dir, f"hifa4_clocks_rank{index}.csv")
        os.makedirs(os.path.dirname(self.path), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(index), f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                       "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.p = None

    def stop(self):
        if self.p is None:
            return None
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except Exception:
            self.p.kill()
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
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
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "samples": len(sm), "reasons": sorted(reasons)}


def dist_setup(n_gpus: int, backend: str = "nccl"):
    """One process per GPU (torchrun env).  backend "gloo" runs the same
    plumbing on CPU (tests)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return rank, world, local


def _coll_device():
    import torch.distributed as dist
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def allmax(x: float, world) -> float:
    """Max over ranks (device time of a multi-GPU step is the slowest rank's)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], device=_coll_device(), dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, ms_per_rank: float, world: int) -> float:
    """Whole-job throughput: the units all ranks processed (each its own batch,
    no exchange) over the max-over-ranks time, per second."""
    return units_per_rank * world / (allmax(ms_per_rank, world) * 1e-3)


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws its own batch of the workload."""
    return seed + 1000 * rank


# ------------------------------------------------------------ our arm -----
class PrefillSetup:
    """Device-resident inputs of one prefill workload (this rank's batch):
    raw Q, K, V, the Smooth-QK scales (offline, untimed) and the quantized
    buffers the timed step writes."""

    def __init__(self, w, fmt, rank=0, alpha=0.5, inputs=None):
        import bit_quantized_flashattention_smooth_b200 as h
        self.w, self.fmt = w, fmt
        wr = W.Workload(**{**w.__dict__, "seed": rank_seed(w.seed, rank)})   # each rank its own batch
        self.host = inputs if inputs is not None else W.make_prefill(wr)
        dev = torch.device("cuda")
        self.qd, self.kd, self.vd = (t.to(dev) for t in self.host)
        self.s, self.inv = h.calibrate_smooth_qk(self.qd[:, :, : w.n_cal], self.kd[:, :, : w.n_cal], w.n_cal,
                                                 alpha=alpha)
        self.z = h.alloc_qkv(w.B, w.Hq, w.Hkv, w.N, w.d, fmt, dev)
        self.o = torch.empty((w.B, w.Hq, w.N, w.d), device=dev, dtype=W.torch_dtype(w.dtype))
        self.scale = 1.0 / math.sqrt(w.d)

    def quantize(self):
        import bit_quantized_flashattention_smooth_b200 as h
        h.quantize_qkv(self.qd, self.kd, self.vd, self.s, self.inv, self.fmt, out=self.z)

    def attention(self, mode, tau=0.0):
        import bit_quantized_flashattention_smooth_b200 as h
        h.attn_fwd(self.z, self.scale, self.w.causal, mode, self.w.block_n, out=self.o, rescale_threshold=tau)


def time_step(setup, mode, steps, warmup, tau=0.0, world=1, clocks=False):
    """One step = the quantize launch, then the attention launch; L2 flushed
    between timed steps (outside the step's events).  Returns per-step device
    ms of the step, the attention and the quantize (means over `steps`)."""
    import bit_quantized_flashattention_smooth_b200 as h
    flush = L2Flush()
    for _ in range(warmup):
        flush()
        setup.quantize()
        setup.attention(mode, tau)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    sampler = ClockSampler(torch.cuda.current_device()) if clocks else None
    barrier(world)
    torch.cuda.synchronize()
    t_wall = time.perf_counter()
    for i in range(steps):
        flush()
        e0, e1, e2 = ev[i]
        e0.record(stream)
        setup.quantize()
        e1.record(stream)
        setup.attention(mode, tau)
        e2.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    wall = time.perf_counter() - t_wall
    clk = sampler.stop() if sampler else None
    dev_err = h.device_error()
    if dev_err:
        raise RuntimeError(f"device error word {dev_err:#x}")
    return dict(step_ms=sum(a.elapsed_time(c) for a, b, c in ev) / steps,
                attn_ms=sum(b.elapsed_time(c) for a, b, c in ev) / steps,
                quant_ms=sum(a.elapsed_time(b) for a, b, c in ev) / steps, clocks=clk, wall=wall)


def run_prefill(args, rank, world):
    """The headline: the workload's step timed over args.steps, then the same
    step end to end through the C ABI with host buffers."""
    import bit_quantized_flashattention_smooth_b200 as h
    w = W.WORKLOADS[args.workload]
    fmt = h.NVFP4 if args.fmt == "nvfp4" else h.MXFP4
    mode = h.PREORDER if args.mode == "preorder" else h.INCONSISTENT
    st = PrefillSetup(w, fmt, rank)
    t = time_step(st, mode, args.steps, args.warmup, args.rescale_threshold, world, clocks=True)
    step_ms_max = allmax(t["step_ms"], world)
    attn_ms_max = allmax(t["attn_ms"], world)
    flops = W.prefill_flops(w)

    # ---- end to end through the C ABI with host buffers (pinned) ----
    qh, kh, vh = (x.pin_memory() for x in st.host)
    oh = torch.empty(st.o.shape, dtype=st.o.dtype).pin_memory()
    stream = torch.cuda.current_stream()

    def e2e_step():
        st.qd.copy_(qh, non_blocking=True); st.kd.copy_(kh, non_blocking=True); st.vd.copy_(vh, non_blocking=True)
        st.quantize()
        st.attention(mode, args.rescale_threshold)
        oh.copy_(st.o, non_blocking=True)

    n_e2e = max(3, min(args.steps, args.e2e_steps))
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_s.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    e_e.record(stream)
    torch.cuda.synchronize()
    e2e_ms = allmax(e_s.elapsed_time(e_e) / n_e2e, world)
    h2d = sum(x.numel() * x.element_size() for x in st.host)
    d2h = st.o.numel() * st.o.element_size()
    st.quantize()      # the comparisons read Q-hat, K-hat, V-hat (untimed)
    return dict(w=w, fmt=fmt, mode=mode, step_ms=step_ms_max, attn_ms=attn_ms_max, quant_ms=t["quant_ms"],
                flops=flops, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, clocks=t["clocks"], wall=t["wall"],
                launches=2 * args.steps, setup=st, n_e2e=n_e2e)


def _phat_grid(device):
    return torch.tensor([0, .5, 1, 1.5, 2, 3, 4, 6], dtype=torch.float64, device=device)


def _ue4m3_values(device):
    e = torch.arange(128, device=device)
    ex, mant = (e >> 3) & 15, (e & 7).double()
    return torch.where(ex == 0, mant * 2.0 ** -9, (1 + mant / 8) * torch.pow(2.0, ex.double() - 7))


def tile_epsilon_gpu(setup, mode, batches=None):
    """Per-tile normalizer error of the kernel (the pages measure it per
    attention tile): sum(P-hat) / sum(P) - 1 over the 128 rows x BN keys of
    every visited tile, from the kernel's own P-hat dump and sums of P.  The
    dump holds B*Hq*N*ceil(N/BN) tiles, so large workloads run it on a few
    batches (`batches`) and reduce it in 128-row chunks."""
    import bit_quantized_flashattention_smooth_b200 as h
    w, z = setup.w, setup.z
    if batches is not None:
        z = h.QuantizedQKV(z.q_codes[:batches], z.q_scales[:batches], z.k_codes[:batches], z.k_scales[:batches],
                           z.vt_codes[:batches], z.vt_scales[:batches], batches, z.Hq, z.Hkv, z.N, z.d, z.fmt)
    _, dump = h.attn_fwd_dump(z, setup.scale, w.causal, mode, w.block_n, sum_p=True)
    beta = h.beta_of(z.fmt)
    dev = dump.codes.device
    grid = _phat_grid(dev)
    # sum of the two E2M1 values of a code byte (keys 2i and 2i+1 share a block)
    b = torch.arange(256, device=dev)
    pair_sum = (grid[b & 7] + grid[(b >> 4) & 7]).float()
    if z.fmt == h.NVFP4:
        sd_tab = (_ue4m3_values(dev) * 2.0 ** h.P_PRESCALE_LOG2).float()
    B, H, N, nkt = dump.m.shape
    nq = (N + 127) // 128
    eps_all = []
    for qt in range(nq):
        r0, r1 = qt * 128, min(N, qt * 128 + 128)
        codes = dump.codes[:, :, r0:r1]                                   # [B,H,R,nkt,BN/2]
        blk = pair_sum[codes.long()].view(B, H, r1 - r0, nkt, w.block_n // beta, beta // 2).sum(-1)
        sc = dump.scales[:, :, r0:r1].long()
        sd = sd_tab[sc.clamp(max=127)] if z.fmt == h.NVFP4 else torch.pow(2.0, sc.float() - 127)
        sph = (blk.double() * sd.double()).sum(-1)                       # [B,H,R,nkt]
        vis = torch.isfinite(dump.m[:, :, r0:r1])
        num = torch.where(vis, sph, 0.0).sum(2)
        den = torch.where(vis, dump.sum_p[:, :, r0:r1].double(), 0.0).sum(2)
        eps_all.append((num / den - 1.0)[den > 0])
    eps = torch.cat(eps_all)
    q = eps.float().quantile(torch.tensor([0.1, 0.9], device=dev)) if eps.numel() < (1 << 24) else None
    return dict(tiles=int(eps.numel()), median=float(eps.median()), frac_negative=float((eps < 0).double().mean()),
                p10=float(q[0]) if q is not None else None, p90=float(q[1]) if q is not None else None,
                batches=z.B)


def measure_config(name, fmt_name, mode_name, steps, warmup, alpha=0.5, want_eps=False):
    """One config of the path timed alone (quantize + attention, L2 flushed),
    with its throughput against the FP4 peak and the softmax ceiling."""
    import bit_quantized_flashattention_smooth_b200 as h
    w = W.WORKLOADS[name]
    fmt = h.NVFP4 if fmt_name == "nvfp4" else h.MXFP4
    mode = h.PREORDER if mode_name == "preorder" else h.INCONSISTENT
    st = PrefillSetup(w, fmt, alpha=alpha)
    t = time_step(st, mode, steps, warmup)
    flops = W.prefill_flops(w)
    rec = {"workload": name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "causal": w.causal,
           "format": fmt_name, "normalizer": mode_name, "alpha": alpha, "block_n": w.block_n, "steps": steps,
           "step_ms": t["step_ms"], "attn_ms": t["attn_ms"], "quantize_ms": t["quant_ms"],
           "step_tflops": flops / (t["step_ms"] * 1e-3) / 1e12, "attn_tflops": flops / (t["attn_ms"] * 1e-3) / 1e12,
           "tokens_per_s": w.B * w.N / (t["step_ms"] * 1e-3)}
    if want_eps:
        rec["epsilon_tile"] = tile_epsilon_gpu(st, mode)
        o, lph, lp = h.attn_fwd(st.z, st.scale, w.causal, mode, w.block_n, out_dtype=W.torch_dtype(w.dtype),
                                debug=True)
        e = (lph / lp - 1.0).flatten()
        rec["epsilon_row"] = {"median": float(e.median()), "frac_negative": float((e < 0).float().mean())}
    return rec, st


def deviation_by_rows(o4, ex, N):
    """Deviation of the 4-bit output from exact attention on the first,
    middle and last 128-row query tile and overall."""
    out = {}
    for label, (r0, r1) in (("first_tile", (0, min(128, N))), ("middle_tile", (N // 2, min(N, N // 2 + 128))),
                            ("last_tile", (max(0, N - 128), N)), ("all", (0, N))):
        a, b = o4[:, r0:r1].float(), ex[:, r0:r1]
        out[label] = {"rows": [r0, r1], "max_abs_rel": float((a - b).abs().max() / b.abs().max()),
                      "cosine": float(torch.nn.functional.cosine_similarity(a.flatten(), b.flatten(), dim=0))}
    return out


class L2Flush:
    """Between timed launches: write a buffer larger than L2 (evicting the
    inputs), then read a second one, so that the dirty lines of the write are
    written back here and not inside the next timed kernel."""

    def __init__(self, dev="cuda"):
        self.w = torch.empty(L2_FLUSH_BYTES, device=dev, dtype=torch.uint8)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, device=dev, dtype=torch.int32)

    def __call__(self):
        self.w.zero_()
        self.r.max()


def time_ms(fn, n=30):
    """Mean device time of fn over n launches after 3 warm-ups, L2 flushed
    before each (CUDA events on the current stream)."""
    flush = L2Flush()
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    tot = 0.0
    for _ in range(n):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1)
    return tot / n


def exact_attention_rows(q, k, v, causal, scale, heads):
    """fp32 softmax attention of the given heads on the unquantized inputs
    (the 'exact BF16 attention' the 4-bit output is compared with)."""
    B, Hq, N, d = q.shape
    G = Hq // k.shape[1]
    mask = torch.ones(N, N, dtype=torch.bool, device=q.device).tril() if causal else None
    out = []
    for hh in heads:
        sc = (q[0, hh].float() @ k[0, hh // G].float().T) * scale
        if mask is not None:
            sc = sc.masked_fill(~mask, float("-inf"))
        out.append(torch.softmax(sc, dim=-1) @ v[0, hh // G].float())
    return torch.stack(out)


def comparisons(res):
    """Outside the timed region, on the headline workload: the in-house BF16
    kernel and the cuDNN BF16 attention on the same (unsmoothed,
    unquantized) inputs, the deviation of the 4-bit output from exact
    attention by query-tile range, the normalizer error of both modes per row
    and per tile (Theorem 1), lazy rescaling and the Smooth-QK sweep."""
    import bit_quantized_flashattention_smooth_b200 as h
    st = res["setup"]
    w, z = st.w, st.z
    qd, kd, vd = st.qd, st.kd, st.vd
    scale = st.scale
    out = {"workload": w.name}
    qb, kb, vb = qd.to(torch.bfloat16), kd.to(torch.bfloat16), vd.to(torch.bfloat16)
    attn_ms = res["attn_ms"]
    ob = None
    if w.d in (64, 128, 256) and w.N % 8 == 0:
        vt = h.bf16_transpose_v(vb)
        ob = h.bf16_attn_fwd(qb, kb, vt, scale, w.causal)
        ms = time_ms(lambda: h.bf16_attn_fwd(qb, kb, vt, scale, w.causal, out=ob), n=10)
        out["bf16_inhouse"] = {"ms": ms, "tflops": res["flops"] / (ms * 1e-3) / 1e12,
                               "fp4_speedup": ms / attn_ms, "kernel": "attn_fwd_bf16 (tcgen05 kind::f16)"}
        del vt
    try:
        import torch.nn.functional as F
        from torch.nn.attention import SDPBackend, sdpa_kernel
        G = w.Hq // w.Hkv
        kk, vv = kb.repeat_interleave(G, dim=1), vb.repeat_interleave(G, dim=1)
        with sdpa_kernel(SDPBackend.CUDNN_ATTENTION):
            ms = time_ms(lambda: F.scaled_dot_product_attention(qb, kk, vv, is_causal=w.causal, scale=scale), n=10)
        out["bf16_cudnn_sdpa"] = {"ms": ms, "tflops": res["flops"] / (ms * 1e-3) / 1e12,
                                  "fp4_speedup": ms / attn_ms, "note": "library kernel, context only"}
        del kk, vv
    except Exception as e:  # context only
        out["bf16_cudnn_sdpa"] = {"error": str(e)[:120]}
    # deviation from exact attention (4 heads of batch 0), by query-tile range
    heads = list(range(min(4, w.Hq)))
    ex = exact_attention_rows(qd, kd, vd, w.causal, scale, heads)
    dev = {"heads": heads, "fp4": deviation_by_rows(st.o[0, heads], ex, w.N)}
    if ob is not None:
        dev["bf16_inhouse"] = deviation_by_rows(ob[0, heads], ex, w.N)
    out["deviation_from_exact"] = dev
    # normalizer error: eps_row = l_Phat / l_P - 1 per row; per tile, sum(P-hat)
    # / sum(P) - 1 over each 128-row x BN tile (the pages' unit of measurement)
    odt = W.torch_dtype(w.dtype)
    o_pre, lph, lp = h.attn_fwd(z, scale, w.causal, h.PREORDER, w.block_n, out_dtype=odt, debug=True)
    o_inc = h.attn_fwd(z, scale, w.causal, h.INCONSISTENT, w.block_n, out_dtype=odt)
    eps = (lph / lp - 1.0).flatten()
    a, b = o_inc[0, heads].float().flatten(1), o_pre[0, heads].float().flatten(1)
    scale_err = ((a * b).sum(1) / (b * b).sum(1) - 1.0)
    out["epsilon"] = {"row_median": float(eps.median()), "row_frac_negative": float((eps < 0).float().mean()),
                      "preorder_output_scale_error": 0.0,
                      "inconsistent_output_scale_error_median_over_heads": float(scale_err.median())}
    del o_pre, o_inc, lph, lp
    try:
        out["epsilon"]["tile_inconsistent"] = tile_epsilon_gpu(st, h.INCONSISTENT, batches=1)
    except Exception as e:  # measurement only
        out["epsilon"]["tile_inconsistent"] = {"error": str(e)[:160]}
    # Lazy running-max updates (FlashAttention-4's conditional rescaling; the
    # paper states the exact recurrence, tau = 0): time and deviation from
    # exact attention against the exact recurrence, same harness and heads
    lazy = []
    o_t = torch.empty_like(st.o)
    for tau in (0.0, 1.0, 3.0):
        fn = lambda: h.attn_fwd(z, scale, w.causal, h.PREORDER, w.block_n, out=o_t, rescale_threshold=tau)
        ms = time_ms(fn, n=10)
        fn()
        o4t = o_t[0, heads].float()
        lazy.append({"rescale_threshold": tau, "ms": ms, "tflops": res["flops"] / (ms * 1e-3) / 1e12,
                     "max_abs_rel": float((o4t - ex).abs().max() / ex.abs().max()),
                     "cosine": float(torch.nn.functional.cosine_similarity(o4t.flatten(), ex.flatten(), dim=0))})
    for rec in lazy:
        rec["speedup_vs_exact_recurrence"] = lazy[0]["ms"] / rec["ms"]
    out["lazy_rescale"] = lazy
    del o_t
    # Smooth-QK migration strength and the applicability gate: deviation of
    # the 4-bit output from exact attention (same 4 heads) and eps per setting
    sweep = []
    for label, alpha, enable in (("off", 0.5, 0), ("alpha=0", 0.0, 1), ("alpha=0.25", 0.25, 1),
                                 ("alpha=0.5", 0.5, 1), ("alpha=0.75", 0.75, 1), ("gate, alpha=0.5", 0.5, h.GATE)):
        s_a, inv_a = h.calibrate_smooth_qk(qd[:, :, : w.n_cal], kd[:, :, : w.n_cal], w.n_cal, alpha=alpha,
                                           enable=enable)
        h.quantize_qkv(qd, kd, vd, s_a, inv_a, res["fmt"], out=z)
        oa, lpa, lpp = h.attn_fwd(z, scale, w.causal, h.PREORDER, w.block_n, out_dtype=odt, debug=True)
        o4a = oa[0, heads].float()
        ea = (lpa / lpp - 1.0).flatten()
        sweep.append({"setting": label, "heads_smoothed": int((s_a != 1.0).any(dim=1).sum()),
                      "max_abs_rel": float((o4a - ex).abs().max() / ex.abs().max()),
                      "cosine": float(torch.nn.functional.cosine_similarity(o4a.flatten(), ex.flatten(), dim=0)),
                      "eps_median": float(ea.median())})
        del oa, lpa, lpp
    out["smooth_qk_sweep"] = sweep
    st.quantize()      # restore the headline's quantized inputs
    return out


def q_mean_comparison():
    """The Q-Mean auxiliary (a reading: the pages name it only) on the
    Q-offset workload and on qwen3 (no offsets), both formats: the time of each
    stage (L2 flushed) and the deviation of the output from exact attention
    (heads 0-3, by query-tile range), with and without the auxiliary."""
    import bit_quantized_flashattention_smooth_b200 as h
    out = []
    for name in ("qwen3_qmean", "qwen3_prefill"):
        w = W.WORKLOADS[name]
        q, k, v = (t.cuda() for t in W.make_prefill(w))
        s, inv = h.calibrate_smooth_qk(q[:, :, : w.n_cal], k[:, :, : w.n_cal], w.n_cal)
        mu = h.calibrate_q_mean(q[:, :, : w.n_cal], s, w.n_cal)
        scale = 1.0 / math.sqrt(w.d)
        heads = list(range(4))
        ex = exact_attention_rows(q, k, v, w.causal, scale, heads)
        for fmt_name, fmt in (("nvfp4", h.NVFP4), ("mxfp4", h.MXFP4)):
            z = h.alloc_qkv(w.B, w.Hq, w.Hkv, w.N, w.d, fmt)
            o = torch.empty((w.B, w.Hq, w.N, w.d), device="cuda", dtype=W.torch_dtype(w.dtype))
            rec = {"workload": name, "format": fmt_name}
            h.quantize_qkv(q, k, v, s, inv, fmt, out=z)
            rec["plain"] = {"quantize_ms": time_ms(lambda: h.quantize_qkv(q, k, v, s, inv, fmt, out=z), n=20),
                            "attn_ms": time_ms(lambda: h.attn_fwd(z, scale, w.causal, h.PREORDER, w.block_n, out=o),
                                               n=20)}
            rec["plain"]["deviation"] = deviation_by_rows(o[0, heads], ex, w.N)
            h.quantize_qkv(q, k, v, s, inv, fmt, out=z, q_mu=mu)
            bias = h.q_mean_bias(z, mu)
            rec["q_mean"] = {
                "quantize_ms": time_ms(lambda: h.quantize_qkv(q, k, v, s, inv, fmt, out=z, q_mu=mu), n=20),
                "bias_ms": time_ms(lambda: h.q_mean_bias(z, mu), n=20),
                "attn_ms": time_ms(lambda: h.attn_fwd(z, scale, w.causal, h.PREORDER, w.block_n, out=o,
                                                      qk_bias=bias), n=20)}
            rec["q_mean"]["deviation"] = deviation_by_rows(o[0, heads], ex, w.N)
            out.append(rec)
            del z, o, bias
        del q, k, v, ex
        torch.cuda.empty_cache()
    return out


def traffic_record(kernel, workload, fmt, block_n, launch_path="fused"):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of
    one ncu capture, from profiles/traffic.json, if the kernel source still has
    the hash recorded with it (else None: the counters are stale)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "bit_quantized_flashattention_smooth_b200", "csrc", kernel.replace("_fp4", "") + ".cu")
    if not os.path.exists(path) or not os.path.exists(src):
        return None
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    for rec in json.load(open(path)):
        if (rec.get("kernel") == kernel and rec.get("workload") == workload and rec.get("format") == fmt and
                rec.get("block_n") == block_n and rec.get("path", "two-launch") == launch_path and
                rec.get("source_sha256_16") == digest):
            return rec["bytes_per_launch"]
    return None


def fp4_probe_peak():
    """Dense FP4 tensor throughput of back-to-back block-scaled MMAs (the
    repo's fp4_mma_probe): 128x256x256 NVFP4 products on 8 CTAs per SM-wave."""
    import bit_quantized_flashattention_smooth_b200 as h
    n, k, reps = 256, 256, 4000
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    ctas = sms
    ac = torch.randint(0, 256, (128, k // 2), dtype=torch.uint8, device="cuda")
    bc = torch.randint(0, 256, (n, k // 2), dtype=torch.uint8, device="cuda")
    asc = torch.full((h.scale_bytes(128, k, h.NVFP4),), 0x38, dtype=torch.uint8, device="cuda")
    bsc = torch.full((h.scale_bytes(n, k, h.NVFP4),), 0x38, dtype=torch.uint8, device="cuda")
    out = torch.empty((128, n), device="cuda")
    h.fp4_mma_probe(ac, asc, bc, bsc, n, k, h.NVFP4, 10, ctas, out)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    h.fp4_mma_probe(ac, asc, bc, bsc, n, k, h.NVFP4, reps, ctas, out)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    return 2.0 * 128 * n * k * reps * ctas / (ms * 1e-3) / 1e12


def cpu_baseline(w, fmt, mode, prefill_inputs=None, budget_s=15.0):
    """The oracle, as it stands, on the host cores, on a bounded sample of the
    workload: the quantization of batch 0 (all of its Q, K and V), then the
    attention of the last query rows of batch 0, all heads, with as many rows
    (up to one 128-row tile) as fit the time budget."""
    import oracle
    q, k, v = prefill_inputs if prefill_inputs is not None else W.make_prefill(w)
    qn, kn, vn = q[:1].float().numpy(), k[:1].float().numpy(), v[:1].float().numpy()
    s, inv = oracle.calibrate(qn, kn, w.n_cal)
    t0 = time.perf_counter()
    qz = oracle.quantize_qkv(qn, kn, vn, s, inv, fmt)
    t_q = time.perf_counter() - t0
    probe = 4
    t0 = time.perf_counter()
    oracle.attention(qz, w.N, fmt, 1 / math.sqrt(w.d), w.causal, mode, w.block_n, rows=(w.N - probe, w.N))
    per_row = (time.perf_counter() - t0) / probe
    rows = int(max(probe, min(128, (budget_s - t_q) / max(per_row, 1e-9))))
    t0 = time.perf_counter()
    oracle.attention(qz, w.N, fmt, 1 / math.sqrt(w.d), w.causal, mode, w.block_n, rows=(w.N - rows, w.N))
    dt = time.perf_counter() - t0 + t_q
    pairs = sum((i + 1) if w.causal else w.N for i in range(w.N - rows, w.N))
    flops = 4.0 * w.Hq * w.d * pairs
    return dict(value=flops / dt / 1e12, unit="TFLOPS", cores=oracle.threads(), kind="oracle",
                sample=f"batch 0 of {w.name}: oracle quantize of all its Q/K/V ({t_q:.1f} s) plus the attention "
                       f"of its last {rows} query rows, all {w.Hq} heads ({flops / 1e9:.2f} GFLOP, {dt:.1f} s "
                       f"in total); TFLOPS over the sample")


def run_decode(args):
    """Split-KV decode over the NVFP4 cache of the decode workload; returns
    achieved KV GB/s (algorithmic cache bytes / kernel time)."""
    import bit_quantized_flashattention_smooth_b200 as h
    w = W.WORKLOADS["split_decode"]
    dev = torch.device("cuda")
    kv, B, Hkv, Hq, d = w.N, w.B, w.Hkv, w.Hq, w.d
    q, k, v, qcal, kcal = W.make_decode_device(w, dev)
    s, inv = h.calibrate_smooth_qk(qcal, kcal, w.n_cal)
    cache = h.quantize_kv(k, v, inv, h.NVFP4, Hq=Hq)
    del k, v
    splits = h.default_splits(B, Hkv, kv)
    ws = torch.empty(h.decode_workspace_bytes(B, Hq, d, splits), device=dev, dtype=torch.uint8)
    o = torch.empty((B, Hq, d), device=dev, dtype=torch.bfloat16)
    flush = L2Flush(dev)
    for _ in range(3):
        h.attn_decode(q, s, cache, kv, None, h.PREORDER, splits, ws, o)
    torch.cuda.synchronize()
    n = max(5, min(args.steps, 50))
    tot = 0.0
    for _ in range(n):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        h.attn_decode(q, s, cache, kv, None, h.PREORDER, splits, ws, o)
        e1.record()
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1)
    ms = tot / n
    kv_bytes = (cache.k_codes.numel() + cache.k_scales.numel() + cache.vt_codes.numel() + cache.vt_scales.numel())
    # appending one token per sequence to an appendable cache of the same
    # shape (its cost does not depend on the cache contents)
    del cache
    acache, tail = h.alloc_appendable_kv_cache(B, Hq, Hkv, kv + 128, d, h.NVFP4)
    kn = torch.randn((B, Hkv, 1, d), device=dev).to(torch.bfloat16)
    vn = torch.randn((B, Hkv, 1, d), device=dev).to(torch.bfloat16)
    append_ms = time_ms(lambda: h.kv_cache_append(acache, tail, kn, vn, inv, kv), n=20)
    return dict(ms=ms, bytes=kv_bytes, gbs=kv_bytes / (ms * 1e-3) / 1e9, splits=splits, append_ms=append_ms)


# ------------------------------------------------------- reference arm ----
def run_reference(args, rank, world):
    """The CPU oracle timed on the host cores on bounded samples of the same
    workload (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    w = W.WORKLOADS[args.workload]
    fmt = 0 if args.fmt == "nvfp4" else 1
    mode = 0 if args.mode == "preorder" else 1
    q, k, v = W.make_prefill(w)
    qn, kn, vn = q[:1].float().numpy(), k[:1].float().numpy(), v[:1].float().numpy()
    s, inv = oracle.calibrate(qn, kn, w.n_cal)
    qz = oracle.quantize_qkv(qn, kn, vn, s, inv, fmt)
    # one step = attention of `rows` query rows (from the last tile) of all heads
    total_budget = 90.0
    rows = 8
    t0 = time.perf_counter()
    oracle.attention(qz, w.N, fmt, 1 / math.sqrt(w.d), w.causal, mode, w.block_n, rows=(w.N - rows, w.N))
    per_row = (time.perf_counter() - t0) / rows
    rows = int(max(1, min(128, total_budget / max(1, args.steps + args.warmup) / per_row)))
    for _ in range(args.warmup):
        oracle.attention(qz, w.N, fmt, 1 / math.sqrt(w.d), w.causal, mode, w.block_n, rows=(w.N - rows, w.N))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.attention(qz, w.N, fmt, 1 / math.sqrt(w.d), w.causal, mode, w.block_n, rows=(w.N - rows, w.N))
    dt = time.perf_counter() - t0
    pairs = sum((i + 1) if w.causal else w.N for i in range(w.N - rows, w.N))
    flops = 4.0 * w.Hq * w.d * pairs * args.steps
    val = flops / dt / 1e12
    return dict(value=val, ms=dt / args.steps * 1e3,
                sample=f"per step: oracle attention of the last {rows} query rows of batch 0, all {w.Hq} heads, "
                       f"of {w.name}")


def profile_target(args, launches: int = 5):
    """A short run of one kernel for an ncu capture: inputs built, then
    `launches` launches of the target (skip the first with -s in ncu)."""
    import bit_quantized_flashattention_smooth_b200 as h
    w = W.WORKLOADS[args.workload]
    if args.profile_batches:
        # a smaller capture of the same workload: its first batches (same
        # shapes and value distributions; traffic scales with the batch)
        w = W.Workload(**{**w.__dict__, "B": min(w.B, args.profile_batches)})
    fmt = h.NVFP4 if args.fmt == "nvfp4" else h.MXFP4
    mode = h.PREORDER if args.mode == "preorder" else h.INCONSISTENT
    dev = torch.device("cuda")
    if args.profile == "decode":
        wd = W.WORKLOADS["split_decode"]
        q, k, v, qcal, kcal = W.make_decode_device(wd, dev)
        s, inv = h.calibrate_smooth_qk(qcal, kcal, wd.n_cal)
        cache = h.quantize_kv(k, v, inv, h.NVFP4, Hq=wd.Hq)
        del k, v
        splits = h.default_splits(wd.B, wd.Hkv, wd.N)
        ws = torch.empty(h.decode_workspace_bytes(wd.B, wd.Hq, wd.d, splits), device=dev, dtype=torch.uint8)
        o = torch.empty((wd.B, wd.Hq, wd.d), device=dev, dtype=torch.bfloat16)
        fn = lambda: h.attn_decode(q, s, cache, wd.N, None, h.PREORDER, splits, ws, o)  # noqa: E731
    else:
        q, k, v = W.make_prefill(w)
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        s, inv = h.calibrate_smooth_qk(qd[:, :, : w.n_cal], kd[:, :, : w.n_cal], w.n_cal)
        z = h.quantize_qkv(qd, kd, vd, s, inv, fmt)
        scale = 1.0 / math.sqrt(w.d)
        if args.profile == "quantize":
            if args.path == "fused":
                kvz = h.quantize_kv(kd, vd, inv, fmt, Hq=w.Hq)
                fn = lambda: h.quantize_kv(kd, vd, inv, fmt, Hq=w.Hq, out=kvz)  # noqa: E731
            else:
                fn = lambda: h.quantize_qkv(qd, kd, vd, s, inv, fmt, out=z)  # noqa: E731
        elif args.profile == "attn":
            o = torch.empty((w.B, w.Hq, w.N, w.d), device=dev, dtype=W.torch_dtype(w.dtype))
            if args.path == "fused":
                kvz = h.quantize_kv(kd, vd, inv, fmt, Hq=w.Hq)
                fn = lambda: h.attn_fwd_fused(qd, s, kvz, scale, w.causal, mode, w.block_n, out=o)  # noqa: E731
            else:
                fn = lambda: h.attn_fwd(z, scale, w.causal, mode, w.block_n, out=o)  # noqa: E731
        else:
            qb, kb = qd.to(torch.bfloat16), kd.to(torch.bfloat16)
            vt = h.bf16_transpose_v(vd.to(torch.bfloat16))
            ob = torch.empty_like(qb)
            fn = lambda: h.bf16_attn_fwd(qb, kb, vt, scale, w.causal, out=ob)  # noqa: E731
    for _ in range(launches):
        fn()
    torch.cuda.synchronize()
    if h.device_error():
        raise RuntimeError("device error word set")
    print(json.dumps({"profile": args.profile, "workload": w.name if args.profile != "decode" else "split_decode",
                      "B": w.B, "launches": launches}), flush=True)


def measure_all_configs(args, pk, headline):
    """Every config of the path in one run (the headline's workload is
    reported by the headline itself): time, TFLOP/s, tokens/s and roofline
    fractions; epsilon per row and per tile where the normalizer modes are
    compared."""
    import bit_quantized_flashattention_smooth_b200 as h
    fp4_peak = pk["bf16"] * FP4_OVER_BF16
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    mufu = 16.0 * sms * 1965.0 * 1e6
    plan = [("tiny_mha", "nvfp4", "preorder", 0.5, False), ("tiny_mha", "nvfp4", "inconsistent", 0.5, True),
            ("qwen3_prefill", "nvfp4", "preorder", 0.5, False), ("qwen3_prefill", "mxfp4", "preorder", 0.5, False),
            ("qwen3_prefill", "nvfp4", "inconsistent", 0.5, True),
            ("gemma2_prefill", "nvfp4", "preorder", 0.5, False), ("gemma2_prefill", "nvfp4", "inconsistent", 0.5, True),
            ("gemma2_prefill", "nvfp4", "preorder", 0.25, True)]
    out = []
    for name, fmt, mode, alpha, eps in plan:
        try:
            rec, st = measure_config(name, fmt, mode, args.config_steps, 5, alpha=alpha, want_eps=eps)
            rec["frac_fp4_peak"] = rec["attn_tflops"] / fp4_peak
            rec["frac_mufu_ceiling"] = W.exp_count(st.w) / (rec["attn_ms"] * 1e-3) / mufu
            if mode == "preorder" and alpha == 0.5 and fmt == "nvfp4":
                w = st.w
                qb, kb = st.qd.to(torch.bfloat16), st.kd.to(torch.bfloat16)
                vt = h.bf16_transpose_v(st.vd.to(torch.bfloat16))
                ob = h.bf16_attn_fwd(qb, kb, vt, st.scale, w.causal)
                ms = time_ms(lambda: h.bf16_attn_fwd(qb, kb, vt, st.scale, w.causal, out=ob), n=10)
                rec["bf16_inhouse_ms"] = ms
                rec["fp4_speedup_vs_bf16_inhouse"] = ms / rec["attn_ms"]
                del qb, kb, vt, ob
            out.append(rec)
            del st
            torch.cuda.empty_cache()
        except Exception as e:  # measurement only
            out.append({"workload": name, "format": fmt, "normalizer": mode, "alpha": alpha, "error": str(e)[:200]})
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="long_prefill")
    ap.add_argument("--fmt", default="nvfp4", choices=["nvfp4", "mxfp4"])
    ap.add_argument("--mode", default="preorder", choices=["preorder", "inconsistent"])
    ap.add_argument("--rescale-threshold", type=float, default=0.0,
                    help="lazy running-max threshold tau (0 = the exact online recurrence)")
    ap.add_argument("--path", default="two-launch", choices=["fused", "two-launch"],
                    help="fused: K/V quantize + attention with Smooth-QK and Q quantization in the kernel "
                         "(--profile only); two-launch: Q/K/V quantize + attention")
    ap.add_argument("--block-n", type=int, default=0, help="key tile (0 = the workload's)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--config-steps", type=int, default=50, help="timed steps of each entry of `configs`")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-probe", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--no-compare", action="store_true", help="skip the BF16 / exact / epsilon comparisons")
    ap.add_argument("--profile", choices=["attn", "quantize", "decode", "bf16"], default=None,
                    help="run only this kernel a few times (for an ncu capture) and exit")
    ap.add_argument("--profile-batches", type=int, default=0,
                    help="--profile on the first B batches of the workload (a smaller capture)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    # the reference arm is the CPU oracle: its ranks need no GPU (gloo plumbing)
    rank, world, local = dist_setup(args.gpus, "gloo" if args.impl == "reference" else "nccl")
    if args.block_n:
        W.WORKLOADS[args.workload] = W.Workload(**{**W.WORKLOADS[args.workload].__dict__, "block_n": args.block_n})
    w = W.WORKLOADS[args.workload]
    config = {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "causal": w.causal,
              "format": args.fmt, "normalizer": args.mode, "block_n": w.block_n, "path": "two-launch",
              "rescale_threshold": args.rescale_threshold,
              "l2": "flushed between timed steps (256 MiB write, then 256 MiB read); inputs also exceed L2",
              "parallelism": f"replicas x{world}"}

    if args.profile:
        profile_target(args)
        return

    if args.impl == "reference":
        ref = run_reference(args, rank, world)
        if rank == 0:
            import oracle
            line = {"metric": METRIC, "value": ref["value"], "unit": "TFLOPS", "n_gpus": world,
                    "steps": args.steps, "warmup": args.warmup, "ms_per_step": ref["ms"],
                    "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                    "data": "synthetic", "config": config, "impl": "reference",
                    "cpu_baseline": {"value": ref["value"], "unit": "TFLOPS", "cores": oracle.threads(),
                                     "kind": "oracle", "sample": ref["sample"]},
                    "e2e": {"value": ref["value"], "unit": "TFLOPS", "h2d_bytes_per_step": 0,
                            "d2h_bytes_per_step": 0}}
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    pk = peaks()
    res = run_prefill(args, rank, world)
    value = weak_scaling_value(res["flops"], res["step_ms"], world) / 1e12
    attn_tflops = res["flops"] / (res["attn_ms"] * 1e-3) / 1e12
    fp4_peak = pk["bf16"] * FP4_OVER_BF16
    extra = {}
    if rank == 0 and not args.no_probe:
        try:
            extra["fp4_probe_tflops"] = fp4_probe_peak()
        except Exception as e:  # measurement only
            extra["fp4_probe_error"] = str(e)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["step_ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp4-e2m1 (fp32 accumulate / softmax)", "data": "synthetic",
        "config": config,
        "roofline": {"bound": "tensor", "kernel": "attn_fwd_fp4", "achieved": attn_tflops, "peak": fp4_peak,
                     "unit": "TFLOP/s", "frac": attn_tflops / fp4_peak, "traffic": None,
                     "peak_note": f"{pk['src']} bf16 burst {pk['bf16']} TFLOP/s x nominal FP4/BF16 ratio 4"},
        "attn_ms": res["attn_ms"], "quantize_ms": res["quant_ms"],
        "e2e": {"value": res["flops"] * world / (res["e2e_ms"] * 1e-3) / 1e12, "unit": "TFLOPS",
                "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"], "steps": res["n_e2e"]},
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
    }
    line.update(extra)
    if "fp4_probe_tflops" in extra:
        line["roofline"]["frac_of_probe_peak"] = attn_tflops / extra["fp4_probe_tflops"]
    line["tokens_per_s"] = w.B * w.N * world / (res["step_ms"] * 1e-3)
    # the softmax's own ceiling: every score needs one 2^x, and the MUFU unit
    # gives 16 per clock per SM (at the median SM clock seen while timing)
    clk_mhz = (res["clocks"] or {}).get("sm_mhz") or 1965.0
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    n_exp = W.exp_count(w)
    line["roofline_softmax"] = {"bound": "alu", "unit": "exp2/s", "achieved": n_exp / (res["attn_ms"] * 1e-3),
                                "peak": 16.0 * sms * clk_mhz * 1e6, "exp2_per_launch": n_exp,
                                "frac": n_exp / (res["attn_ms"] * 1e-3) / (16.0 * sms * clk_mhz * 1e6),
                                "note": "MUFU ex2 ceiling: 16/clk/SM x SMs x median SM clock"}
    tr = traffic_record("attn_fwd_fp4", w.name, args.fmt, w.block_n, "two-launch")
    if tr is not None:
        line["roofline"]["traffic"] = tr
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, res["fmt"], res["mode"], res["setup"].host)
    if rank == 0 and not args.no_compare:
        try:
            line["comparisons"] = comparisons(res)
        except Exception as e:  # measurement only
            line["comparisons"] = {"error": str(e)[:200]}
    del res
    torch.cuda.empty_cache()
    if rank == 0 and not args.no_configs:
        line["configs"] = measure_all_configs(args, pk, w.name)
        try:
            line["q_mean"] = q_mean_comparison()
        except Exception as e:  # measurement only
            line["q_mean"] = {"error": str(e)[:200]}
    if not args.no_decode:
        try:
            decode = run_decode(args)
            line["decode"] = {"workload": "split_decode", "kv_gbs": decode["gbs"], "ms": decode["ms"],
                              "kv_bytes": decode["bytes"], "hbm_peak_gbs": pk["hbm"],
                              "frac": decode["gbs"] / pk["hbm"], "frac_of_8tbs_spec": decode["gbs"] / 8000.0,
                              "splits": decode["splits"], "append_one_token_ms": decode["append_ms"],
                              "tokens_per_s": W.WORKLOADS["split_decode"].B / (decode["ms"] * 1e-3)}
        except Exception as e:
            line["decode"] = {"error": str(e)[:200]}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
