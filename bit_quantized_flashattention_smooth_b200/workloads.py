"""Seeded synthetic workloads (inputs only; no quantization or attention math).

Both the CUDA path and the CPU oracle take their inputs from here.  The module
holds shapes, random draws, rotary position embedding of the synthetic Q/K and
the outlier-channel pattern -- the preparation of "post-RoPE Q and K" that the
paper's Smooth-QK acts on ("HiFA4: Training-Free 4-bit FlashAttention on Ascend
HIF4 NPUs for LLM Inference", Abstract para 2) -- and nothing of the method.

Recipes (one per workload):
  tiny_mha       B1 H2 N256 d64 non-causal fp16; Q,K,V ~ N(0,1); K channels
                 60..63 replaced by +20|z|; calibration tokens 0..63; BN 64.
  qwen3_prefill  B1 Hq32 Hkv8 d128 N4096 causal bf16; Q,K ~ N(0,1) with the
                 three lowest-frequency RoPE pairs of K (channels 61-63 and
                 125-127) replaced by +15|z| before RoPE (NeoX rotate-half,
                 theta 1e6, positions 0..N-1); V ~ N(0,1).
  gemma2_prefill B1 Hq16 Hkv8 d256 N8192 causal bf16; as above with theta 1e4
                 and the four lowest-frequency pairs (124-127, 252-255) x10.
  long_prefill   B8 Hq32 Hkv8 d128 N16384 causal bf16; Q ~ N(0,1); K i.i.d.
                 Student-t (nu=3) in every channel; RoPE theta 1e6; V ~ N(0,1);
                 calibration tokens 0..255.
  qwen3_qmean    qwen3_prefill's shapes and K, with seed 5 and a per-channel
                 offset in Q: channels 58-60 (the first halves of the next
                 three lowest-frequency RoPE pairs, beside K's outliers) get +8
                 before RoPE, so after the slow rotation they carry a
                 near-constant channel mean (the case the Q-Mean auxiliary
                 addresses).
  split_decode   B64 Hq32 Hkv8 d128, KV length 32768, one query; K,V ~ N(0,1)
                 with qwen3_prefill's outlier pattern and RoPE; the calibration
                 set is a 256-token slice of K plus an independent 256-token Q
                 draw; the query sits at position 32768.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int            # query/key length (prefill) or KV length (decode)
    d: int
    causal: bool
    dtype: str        # "bf16" | "fp16"
    seed: int
    n_cal: int
    block_n: int
    theta: float | None
    outlier_channels: tuple = field(default_factory=tuple)
    outlier_scale: float = 0.0
    k_dist: str = "normal"   # "normal" | "student_t3"
    decode: bool = False
    q_offset_channels: tuple = field(default_factory=tuple)
    q_offset: float = 0.0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


def _lowfreq_pairs(d: int, npairs: int) -> tuple:
    half = d // 2
    lo = list(range(half - npairs, half))
    return tuple(lo + [c + half for c in lo])


WORKLOADS = {
    "tiny_mha": Workload("tiny_mha", 1, 2, 2, 256, 64, False, "fp16", 0, 64, 64, None,
                         (60, 61, 62, 63), 20.0),
    "qwen3_prefill": Workload("qwen3_prefill", 1, 32, 8, 4096, 128, True, "bf16", 1, 256, 64, 1e6,
                              _lowfreq_pairs(128, 3), 15.0),
    "gemma2_prefill": Workload("gemma2_prefill", 1, 16, 8, 8192, 256, True, "bf16", 2, 256, 128, 1e4,
                               _lowfreq_pairs(256, 4), 10.0),
    "long_prefill": Workload("long_prefill", 8, 32, 8, 16384, 128, True, "bf16", 3, 256, 64, 1e6,
                             (), 0.0, "student_t3"),
    "qwen3_qmean": Workload("qwen3_qmean", 1, 32, 8, 4096, 128, True, "bf16", 5, 256, 64, 1e6,
                            _lowfreq_pairs(128, 3), 15.0, q_offset_channels=(58, 59, 60), q_offset=8.0),
    "split_decode": Workload("split_decode", 64, 32, 8, 32768, 128, False, "bf16", 4, 256, 128, 1e6,
                             _lowfreq_pairs(128, 3), 15.0, decode=True),
}


def torch_dtype(name: str):
    return torch.bfloat16 if name == "bf16" else torch.float16


def rope_neox(x: np.ndarray, theta: float, pos0: int = 0) -> np.ndarray:
    """Rotate-half RoPE on the last axis of x [..., T, d] (float32)."""
    T, d = x.shape[-2:]
    half = d // 2
    inv_freq = theta ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = np.arange(pos0, pos0 + T, dtype=np.float64)[:, None] * inv_freq[None, :]
    cos = np.cos(ang).astype(np.float32)
    sin = np.sin(ang).astype(np.float32)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def rope_torch(x: torch.Tensor, theta: float, pos0: int = 0) -> torch.Tensor:
    """rope_neox for a float32 torch tensor [..., T, d] on any device."""
    T, d = x.shape[-2:]
    half = d // 2
    inv_freq = theta ** (-torch.arange(half, dtype=torch.float64, device=x.device) * 2.0 / d)
    ang = torch.arange(pos0, pos0 + T, dtype=torch.float64, device=x.device)[:, None] * inv_freq[None, :]
    cos, sin = torch.cos(ang).float(), torch.sin(ang).float()
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1)


def make_decode_device(w: Workload, device="cuda"):
    """The decode recipe drawn on the device with a seeded torch generator (the
    full-size cache is 2 x 4 GiB of bf16; a host draw would dominate a run).
    Returns (q [B,Hq,d], k, v [B,Hkv,kv,d], q_cal [B,Hq,n_cal,d], k_cal)."""
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    kv, B = w.N, w.B
    k = torch.randn((B, w.Hkv, kv, w.d), generator=g, device=device, dtype=torch.float32)
    for c in w.outlier_channels:
        k[..., c] = w.outlier_scale * k[..., c].abs()
    k = rope_torch(k, w.theta).to(torch_dtype(w.dtype))
    v = torch.randn((B, w.Hkv, kv, w.d), generator=g, device=device, dtype=torch.float32).to(torch_dtype(w.dtype))
    q = rope_torch(torch.randn((B, w.Hq, 1, w.d), generator=g, device=device), w.theta, pos0=kv)
    q_cal = rope_torch(torch.randn((B, w.Hq, w.n_cal, w.d), generator=g, device=device), w.theta)
    n_cal = min(w.n_cal, kv)
    return (q[:, :, 0].to(torch_dtype(w.dtype)), k, v, q_cal[:, :, :n_cal].to(torch_dtype(w.dtype)),
            k[:, :, :n_cal].contiguous())


def _draw_k(rng, shape, w: Workload) -> np.ndarray:
    if w.k_dist == "student_t3":
        return rng.standard_t(3, size=shape).astype(np.float32)
    k = rng.standard_normal(shape, dtype=np.float32)
    for c in w.outlier_channels:
        k[..., c] = w.outlier_scale * np.abs(k[..., c])
    return k


def _round(x: np.ndarray, dtype: str) -> torch.Tensor:
    """fp32 -> bf16/fp16 with round-to-nearest-even (torch's cast)."""
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch_dtype(dtype))


def make_prefill(w: Workload, N: int | None = None, B: int | None = None):
    """Returns (q, k, v) as CPU torch tensors of w.dtype, shapes [B,H,N,d]."""
    N = w.N if N is None else N
    B = w.B if B is None else B
    rng = np.random.Generator(np.random.PCG64(w.seed))
    q = rng.standard_normal((B, w.Hq, N, w.d), dtype=np.float32)
    for c in w.q_offset_channels:
        q[..., c] += np.float32(w.q_offset)
    k = _draw_k(rng, (B, w.Hkv, N, w.d), w)
    v = rng.standard_normal((B, w.Hkv, N, w.d), dtype=np.float32)
    if w.theta is not None:
        # rope_torch on the host equals rope_neox bit for bit (the same fp32
        # operations, element by element) and runs on all host threads
        q = rope_torch(torch.from_numpy(q), w.theta).numpy()
        k = rope_torch(torch.from_numpy(k), w.theta).numpy()
    return _round(q, w.dtype), _round(k, w.dtype), _round(v, w.dtype)


def make_decode(w: Workload, kv_len: int | None = None, B: int | None = None):
    """Returns (q [B,Hq,d], k_cache, v_cache [B,Hkv,kv,d], q_cal [B,Hq,256,d],
    k_cal [B,Hkv,256,d]) as CPU torch tensors of w.dtype."""
    kv = w.N if kv_len is None else kv_len
    B = w.B if B is None else B
    rng = np.random.Generator(np.random.PCG64(w.seed))
    k = _draw_k(rng, (B, w.Hkv, kv, w.d), w)
    v = rng.standard_normal((B, w.Hkv, kv, w.d), dtype=np.float32)
    q = rng.standard_normal((B, w.Hq, 1, w.d), dtype=np.float32)
    q_cal = rng.standard_normal((B, w.Hq, w.n_cal, w.d), dtype=np.float32)
    if w.theta is not None:
        k = rope_neox(k, w.theta)
        q = rope_neox(q, w.theta, pos0=kv)
        q_cal = rope_neox(q_cal, w.theta)
    n_cal = min(w.n_cal, kv)
    k_cal = k[:, :, :n_cal]
    return (_round(q[:, :, 0], w.dtype), _round(k, w.dtype), _round(v, w.dtype),
            _round(q_cal[:, :, :n_cal], w.dtype), _round(k_cal, w.dtype))


def attended_pairs(N: int, causal: bool) -> int:
    return N * (N + 1) // 2 if causal else N * N


def exp_count(w: Workload) -> float:
    """2^x evaluations of the softmax: one per attended query-key pair."""
    return float(w.B * w.Hq * attended_pairs(w.N, w.causal))


def prefill_flops(w: Workload, N: int | None = None, B: int | None = None) -> float:
    """4 * B * Hq * d * (attended query-key pairs): QK^T and PV multiply-adds."""
    N = w.N if N is None else N
    B = w.B if B is None else B
    return 4.0 * B * w.Hq * w.d * attended_pairs(N, w.causal)
