"""Python binding of the B200 4-bit FlashAttention library (libhifa4.so).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``csrc/`` behind the C ABI of ``include/hifa4.h``.  PyTorch provides device
memory and the current stream.  There is no CPU fallback: if the in-tree
library is missing, every call raises.

Method: "HiFA4: Training-Free 4-bit FlashAttention on Ascend HIF4 NPUs for LLM
Inference", Abstract paras 1-2 (Smooth-QK, 4-bit QK^T and PV GEMMs, online
softmax, P-Reordering).
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhifa4.so")

NVFP4, MXFP4 = 0, 1
PREORDER, INCONSISTENT = 0, 1
BF16, FP16 = 0, 1
P_PRESCALE_LOG2 = -8

_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported", 3: "CUDA error", 4: "timeout"}
_lib = None

ABI_FUNCTIONS = (
    "hifa4_codes_bytes", "hifa4_scale_bytes", "hifa4_calibrate_smooth_qk", "hifa4_quantize_qkv",
    "hifa4_quantize_kv", "hifa4_calibrate_q_mean", "hifa4_quantize_qkv_qmean", "hifa4_q_mean_bias",
    "hifa4_attn_fwd_qmean",
    "hifa4_attn_fwd", "hifa4_attn_fwd_ex", "hifa4_attn_fwd_dump", "hifa4_attn_fwd_fused", "hifa4_decode_workspace_size", "hifa4_decode_default_splits", "hifa4_attn_decode",
    "hifa4_decode_noalloc_max_bytes", "hifa4_attn_decode_noalloc",
    "hifa4_fp4_mma_probe", "hifa4_convert_probe", "hifa4_div6_probe", "hifa4_exp2_poly_probe", "hifa4_e2m1_map_probe", "hifa4_bf16_attn_fwd", "hifa4_bf16_transpose_v", "hifa4_wait_timeout_probe", "hifa4_kv_cache_append", "hifa4_attn_decode_cache", "hifa4_status_string", "hifa4_last_error",
    "hifa4_device_error",
)


class HiFA4Error(RuntimeError):
    pass


def lib():
    """Load the in-tree CUDA library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise HiFA4Error(f"CUDA library not built: {LIB_PATH} (run __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, i64, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        L.hifa4_codes_bytes.argtypes = [i64, i]; L.hifa4_codes_bytes.restype = sz
        L.hifa4_scale_bytes.argtypes = [i64, i, i]; L.hifa4_scale_bytes.restype = sz
        L.hifa4_calibrate_smooth_qk.argtypes = [vp, vp, i, i, i, i, i, i, i, f, i, vp, vp, vp]
        L.hifa4_quantize_qkv.argtypes = [vp, vp, vp, i, i, i, i, i, i, vp, vp, i, vp, vp, vp, vp, vp, vp, vp]
        L.hifa4_quantize_kv.argtypes = [vp, vp, i, i, i, i, i, vp, i, vp, vp, vp, vp, vp]
        L.hifa4_calibrate_q_mean.argtypes = [vp, i, i, i, i, i, i, i, vp, vp, vp]
        L.hifa4_quantize_qkv_qmean.argtypes = [vp, vp, vp, i, i, i, i, i, i, vp, vp, vp, i, vp, vp, vp, vp, vp, vp,
                                               vp]
        L.hifa4_q_mean_bias.argtypes = [vp, vp, vp, i, i, i, i, i, i, vp, vp]
        L.hifa4_attn_fwd_qmean.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, vp, i, vp, f,
                                           vp]
        L.hifa4_attn_fwd.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, vp, i, vp, vp, vp, vp]
        L.hifa4_attn_fwd_ex.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, vp, i, vp, vp, vp, f,
                                        vp]
        L.hifa4_attn_fwd_dump.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, vp, i, f, vp, vp, vp,
                                          vp, vp]
        L.hifa4_attn_fwd_fused.argtypes = [vp, i, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, vp, i, vp, vp, vp,
                                           f, vp]
        L.hifa4_decode_workspace_size.argtypes = [i, i, i, i]; L.hifa4_decode_workspace_size.restype = sz
        L.hifa4_decode_default_splits.argtypes = [i, i, i, i]; L.hifa4_decode_default_splits.restype = i
        L.hifa4_attn_decode.argtypes = [vp, i, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i,
                                        ctypes.POINTER(ctypes.c_int), vp, sz, vp, i, vp]
        L.hifa4_decode_noalloc_max_bytes.argtypes = []; L.hifa4_decode_noalloc_max_bytes.restype = sz
        L.hifa4_attn_decode_noalloc.argtypes = [vp, i, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i,
                                                ctypes.POINTER(ctypes.c_int), vp, i, vp]
        L.hifa4_fp4_mma_probe.argtypes = [vp, vp, vp, vp, i, i, i, i, i, vp, vp]
        L.hifa4_convert_probe.argtypes = [vp, i64, vp, vp, vp]
        L.hifa4_div6_probe.argtypes = [ctypes.c_uint32, ctypes.c_uint32, vp, vp, vp]
        L.hifa4_exp2_poly_probe.argtypes = [vp, i64, vp, vp]
        L.hifa4_e2m1_map_probe.argtypes = [vp, i64, vp, vp, vp]
        L.hifa4_bf16_attn_fwd.argtypes = [vp, vp, vp, i, i, i, i, i, f, i, vp, vp, vp]
        L.hifa4_bf16_transpose_v.argtypes = [vp, i, i, i, i, vp, vp]
        L.hifa4_wait_timeout_probe.argtypes = [vp, vp]
        L.hifa4_kv_cache_append.argtypes = [vp, vp, i, i, i, i, i, vp, i, i, i, vp, vp, vp, vp, vp, vp]
        L.hifa4_attn_decode_cache.argtypes = [vp, i, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, i,
                                              ctypes.POINTER(ctypes.c_int), vp, sz, vp, i, f, vp]
        L.hifa4_status_string.argtypes = [i]; L.hifa4_status_string.restype = ctypes.c_char_p
        L.hifa4_last_error.argtypes = []; L.hifa4_last_error.restype = ctypes.c_char_p
        L.hifa4_device_error.argtypes = []; L.hifa4_device_error.restype = ctypes.c_uint
        for name in ABI_FUNCTIONS:
            getattr(L, name).restype = getattr(L, name).restype or ctypes.c_int
        _lib = L
    return _lib


def _check(st: int, what: str):
    if st != 0:
        msg = lib().hifa4_last_error().decode(errors="replace")
        raise HiFA4Error(f"{what}: {_STATUS.get(st, st)}: {msg}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float16:
        return FP16
    raise HiFA4Error(f"unsupported dtype {t.dtype}")


def pad128(n: int) -> int:
    return (n + 127) // 128 * 128


def beta_of(fmt: int) -> int:
    return 16 if fmt == NVFP4 else 32


def scale_bytes(rows: int, k: int, fmt: int) -> int:
    return int(lib().hifa4_scale_bytes(rows, k, fmt))


def device_error() -> int:
    """Synchronizes, returns and clears the device error word (0 = fine)."""
    return int(lib().hifa4_device_error())


# --------------------------------------------------------------- calibrate ---
GATE = 2   # calibrate_smooth_qk(enable=GATE): per-head applicability gate


def calibrate_smooth_qk(q: torch.Tensor, k: torch.Tensor, n_cal: int, alpha: float = 0.5,
                        enable: bool | int = True):
    """q [B,Hq,T,d], k [B,Hkv,T,d] (cuda, bf16/fp16) -> (s, inv_s) [Hkv,d] float32.
    enable: False / True, or GATE for the per-head applicability gate."""
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    q = q.contiguous(); k = k.contiguous()
    s = torch.empty((Hkv, d), device=q.device, dtype=torch.float32)
    inv = torch.empty_like(s)
    _check(lib().hifa4_calibrate_smooth_qk(_ptr(q), _ptr(k), _dt(q), B, Hq, Hkv, n_cal, T, d, float(alpha),
                                           int(enable), _ptr(s), _ptr(inv), _stream()),
           "calibrate_smooth_qk")
    return s, inv


# ---------------------------------------------------------------- quantize ---
@dataclass
class QuantizedQKV:
    """4-bit Q-hat, K-hat, V-hat^T in the library layouts (include/hifa4.h)."""
    q_codes: torch.Tensor
    q_scales: torch.Tensor
    k_codes: torch.Tensor
    k_scales: torch.Tensor
    vt_codes: torch.Tensor
    vt_scales: torch.Tensor
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    fmt: int

    @property
    def Np(self) -> int:
        return pad128(self.N)


def alloc_qkv(B, Hq, Hkv, N, d, fmt, device="cuda") -> QuantizedQKV:
    Np = pad128(N)
    u8 = dict(device=device, dtype=torch.uint8)
    sq = scale_bytes(N, d, fmt)
    sv = scale_bytes(d, Np, fmt)
    return QuantizedQKV(
        torch.empty((B, Hq, Np, d // 2), **u8), torch.empty((B, Hq, sq), **u8),
        torch.empty((B, Hkv, Np, d // 2), **u8), torch.empty((B, Hkv, sq), **u8),
        torch.empty((B, Hkv, d, Np // 2), **u8), torch.empty((B, Hkv, sv), **u8),
        B, Hq, Hkv, N, d, fmt)


def quantize_qkv(q, k, v, s=None, inv_s=None, fmt: int = NVFP4, out: QuantizedQKV | None = None,
                 q_mu: torch.Tensor | None = None):
    """Fused Smooth-QK scale + block quantization.  q [B,Hq,N,d], k/v [B,Hkv,N,d].
    q_mu [Hq,d] (calibrate_q_mean): the Q-Mean auxiliary, subtracted from the
    smoothed query (hifa4_quantize_qkv_qmean)."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    q = q.contiguous(); k = k.contiguous(); v = v.contiguous()
    z = out if out is not None else alloc_qkv(B, Hq, Hkv, N, d, fmt, q.device)
    if q_mu is not None:
        _check(lib().hifa4_quantize_qkv_qmean(_ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hq, Hkv, N, d, _ptr(s),
                                              _ptr(inv_s), _ptr(q_mu), fmt, _ptr(z.q_codes), _ptr(z.q_scales),
                                              _ptr(z.k_codes), _ptr(z.k_scales), _ptr(z.vt_codes),
                                              _ptr(z.vt_scales), _stream()), "quantize_qkv_qmean")
        return z
    _check(lib().hifa4_quantize_qkv(_ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hq, Hkv, N, d, _ptr(s), _ptr(inv_s),
                                    fmt, _ptr(z.q_codes), _ptr(z.q_scales), _ptr(z.k_codes), _ptr(z.k_scales),
                                    _ptr(z.vt_codes), _ptr(z.vt_scales), _stream()), "quantize_qkv")
    return z


def calibrate_q_mean(q: torch.Tensor, s: torch.Tensor | None, n_cal: int, Hkv: int | None = None) -> torch.Tensor:
    """Q-Mean auxiliary: the per-channel mean of the smoothed query over the
    calibration tokens.  q [B,Hq,T,d] (cuda), s [Hkv,d] or None -> mu [Hq,d]."""
    B, Hq, T, d = q.shape
    Hkv = s.shape[0] if s is not None else (Hkv or Hq)
    q = q.contiguous()
    mu = torch.empty((Hq, d), device=q.device, dtype=torch.float32)
    _check(lib().hifa4_calibrate_q_mean(_ptr(q), _dt(q), B, Hq, Hkv, n_cal, T, d, _ptr(s), _ptr(mu), _stream()),
           "calibrate_q_mean")
    return mu


def q_mean_bias(z: QuantizedQKV, q_mu: torch.Tensor) -> torch.Tensor:
    """The Q-Mean score term mu . K-hat per key: [B,Hq,Np] float32."""
    bias = torch.empty((z.B, z.Hq, z.Np), device=z.k_codes.device, dtype=torch.float32)
    _check(lib().hifa4_q_mean_bias(_ptr(z.k_codes), _ptr(z.k_scales), _ptr(q_mu), z.B, z.Hq, z.Hkv, z.N, z.d, z.fmt,
                                   _ptr(bias), _stream()), "q_mean_bias")
    return bias


def alloc_kv_cache(B, Hq, Hkv, kv_len, d, fmt, device="cuda") -> QuantizedQKV:
    """A 4-bit KV cache (no Q buffers)."""
    Np = pad128(kv_len)
    u8 = dict(device=device, dtype=torch.uint8)
    empty = torch.empty(0, **u8)
    return QuantizedQKV(empty, empty,
                        torch.empty((B, Hkv, Np, d // 2), **u8), torch.empty((B, Hkv, scale_bytes(kv_len, d, fmt)), **u8),
                        torch.empty((B, Hkv, d, Np // 2), **u8), torch.empty((B, Hkv, scale_bytes(d, Np, fmt)), **u8),
                        B, Hq, Hkv, kv_len, d, fmt)


def alloc_appendable_kv_cache(B, Hq, Hkv, capacity, d, fmt, dtype=torch.bfloat16, device="cuda"):
    """An empty 4-bit KV cache for `capacity` tokens (zeroed, as the append
    contract requires) and its V tail buffer [B, Hkv, beta, d]."""
    z = alloc_kv_cache(B, Hq, Hkv, capacity, d, fmt, device)
    for t in (z.k_codes, z.k_scales, z.vt_codes, z.vt_scales):
        t.zero_()
    beta = 16 if fmt == NVFP4 else 32
    return z, torch.zeros((B, Hkv, beta, d), device=device, dtype=dtype)


def kv_cache_append(cache: QuantizedQKV, v_tail: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                    inv_s: torch.Tensor | None, pos: int):
    """Append tokens [pos, pos + T) (k_new, v_new [B, Hkv, T, d]) to an appendable cache."""
    B, Hkv, T, d = k_new.shape
    k_new = k_new.contiguous(); v_new = v_new.contiguous()
    _check(lib().hifa4_kv_cache_append(_ptr(k_new), _ptr(v_new), _dt(k_new), B, Hkv, T, d, _ptr(inv_s), cache.fmt,
                                       int(pos), cache.N, _ptr(cache.k_codes), _ptr(cache.k_scales),
                                       _ptr(cache.vt_codes), _ptr(cache.vt_scales), _ptr(v_tail), _stream()),
           "kv_cache_append")


def quantize_kv(k, v, inv_s=None, fmt: int = NVFP4, Hq: int | None = None, out: QuantizedQKV | None = None):
    """Quantize K (scaled by inv_s) and V into a 4-bit KV cache."""
    B, Hkv, N, d = k.shape
    k = k.contiguous(); v = v.contiguous()
    z = out if out is not None else alloc_kv_cache(B, Hq or Hkv, Hkv, N, d, fmt, k.device)
    _check(lib().hifa4_quantize_kv(_ptr(k), _ptr(v), _dt(k), B, Hkv, N, d, _ptr(inv_s), fmt, _ptr(z.k_codes),
                                   _ptr(z.k_scales), _ptr(z.vt_codes), _ptr(z.vt_scales), _stream()), "quantize_kv")
    return z


# --------------------------------------------------------------- attention ---
def attn_fwd(z: QuantizedQKV, softmax_scale: float | None = None, causal: bool = True, mode: int = PREORDER,
             block_n: int = 128, out_dtype=torch.bfloat16, return_lse: bool = False, debug: bool = False,
             out: torch.Tensor | None = None, rescale_threshold: float = 0.0, qk_bias: torch.Tensor | None = None):
    """4-bit attention forward.  Returns O [B,Hq,N,d] (and lse / debug sums).
    rescale_threshold > 0 updates the running max lazily (hifa4_attn_fwd_ex).
    qk_bias [B,Hq,Np] (q_mean_bias): the Q-Mean score term (hifa4_attn_fwd_qmean)."""
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(z.d)
    dev = z.q_codes.device
    o = out if out is not None else torch.empty((z.B, z.Hq, z.N, z.d), device=dev, dtype=out_dtype)
    lse = torch.empty((z.B, z.Hq, z.N), device=dev, dtype=torch.float32) if return_lse else None
    if qk_bias is not None:
        if debug:
            raise HiFA4Error("attn_fwd: the Q-Mean forward has no debug sums")
        _check(lib().hifa4_attn_fwd_qmean(_ptr(z.q_codes), _ptr(z.q_scales), _ptr(z.k_codes), _ptr(z.k_scales),
                                          _ptr(z.vt_codes), _ptr(z.vt_scales), _ptr(qk_bias), z.B, z.Hq, z.Hkv, z.N,
                                          z.d, z.fmt, float(softmax_scale), int(bool(causal)), int(mode),
                                          int(block_n), _ptr(o), _dt(o), _ptr(lse), float(rescale_threshold),
                                          _stream()), "attn_fwd_qmean")
        return (o, lse) if return_lse else o
    lph = torch.empty((z.B, z.Hq, z.N), device=dev, dtype=torch.float32) if debug else None
    lp = torch.empty((z.B, z.Hq, z.N), device=dev, dtype=torch.float32) if debug else None
    _check(lib().hifa4_attn_fwd_ex(_ptr(z.q_codes), _ptr(z.q_scales), _ptr(z.k_codes), _ptr(z.k_scales),
                                   _ptr(z.vt_codes), _ptr(z.vt_scales), z.B, z.Hq, z.Hkv, z.N, z.d, z.fmt,
                                   float(softmax_scale), int(bool(causal)), int(mode), int(block_n), _ptr(o),
                                   _dt(o), _ptr(lse), _ptr(lph), _ptr(lp), float(rescale_threshold), _stream()),
           "attn_fwd")
    res = [o]
    if return_lse:
        res.append(lse)
    if debug:
        res += [lph, lp]
    return res[0] if len(res) == 1 else tuple(res)


@dataclass
class PhatDump:
    """Quantized attention weights of one forward, as fed to the PV MMA
    (hifa4_attn_fwd_dump): codes [B,Hq,N,nkt,BN/2] packed E2M1, scales
    [B,Hq,N,nkt,BN/beta], m [B,Hq,N,nkt] running max after each key tile,
    sum_p [B,Hq,N,nkt] (or None) sum of P of each tile."""
    codes: torch.Tensor
    scales: torch.Tensor
    m: torch.Tensor
    sum_p: torch.Tensor | None


def attn_fwd_dump(z: QuantizedQKV, softmax_scale: float | None = None, causal: bool = True, mode: int = PREORDER,
                  block_n: int = 128, out_dtype=torch.bfloat16, rescale_threshold: float = 0.0,
                  sum_p: bool = False):
    """Forward plus the P-hat dump.  sum_p=True selects the softmax variant
    that forms P (as the debug normalizers do) and records sum(P) per tile.
    Returns (O, PhatDump); unvisited tiles hold zeros (m: NaN)."""
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(z.d)
    dev = z.q_codes.device
    nkt = (z.N + block_n - 1) // block_n
    beta = beta_of(z.fmt)
    o = torch.empty((z.B, z.Hq, z.N, z.d), device=dev, dtype=out_dtype)
    codes = torch.zeros((z.B, z.Hq, z.N, nkt, block_n // 2), device=dev, dtype=torch.uint8)
    scales = torch.zeros((z.B, z.Hq, z.N, nkt, block_n // beta), device=dev, dtype=torch.uint8)
    m = torch.full((z.B, z.Hq, z.N, nkt), float("nan"), device=dev, dtype=torch.float32)
    sp = torch.zeros((z.B, z.Hq, z.N, nkt), device=dev, dtype=torch.float32) if sum_p else None
    _check(lib().hifa4_attn_fwd_dump(_ptr(z.q_codes), _ptr(z.q_scales), _ptr(z.k_codes), _ptr(z.k_scales),
                                     _ptr(z.vt_codes), _ptr(z.vt_scales), z.B, z.Hq, z.Hkv, z.N, z.d, z.fmt,
                                     float(softmax_scale), int(bool(causal)), int(mode), int(block_n), _ptr(o),
                                     _dt(o), float(rescale_threshold), _ptr(codes), _ptr(scales), _ptr(m), _ptr(sp),
                                     _stream()), "attn_fwd_dump")
    return o, PhatDump(codes, scales, m, sp)


def attn_fwd_fused(q: torch.Tensor, s: torch.Tensor | None, kv: QuantizedQKV, softmax_scale: float | None = None,
                   causal: bool = True, mode: int = PREORDER, block_n: int = 128, out_dtype=torch.bfloat16,
                   return_lse: bool = False, debug: bool = False, out: torch.Tensor | None = None,
                   rescale_threshold: float = 0.0):
    """Prefill forward with Smooth-QK and Q quantization inside the attention
    kernel: q [B,Hq,N,d] raw (bf16/fp16), s [Hkv,d] or None, kv = quantize_kv(k, v, 1/s).
    Equals quantize_qkv + attn_fwd bit for bit."""
    B, Hq, N, d = q.shape
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    q = q.contiguous()
    dev = q.device
    o = out if out is not None else torch.empty((B, Hq, N, d), device=dev, dtype=out_dtype)
    lse = torch.empty((B, Hq, N), device=dev, dtype=torch.float32) if return_lse else None
    lph = torch.empty((B, Hq, N), device=dev, dtype=torch.float32) if debug else None
    lp = torch.empty((B, Hq, N), device=dev, dtype=torch.float32) if debug else None
    _check(lib().hifa4_attn_fwd_fused(_ptr(q), _dt(q), _ptr(s), _ptr(kv.k_codes), _ptr(kv.k_scales),
                                      _ptr(kv.vt_codes), _ptr(kv.vt_scales), B, Hq, kv.Hkv, N, d, kv.fmt,
                                      float(softmax_scale), int(bool(causal)), int(mode), int(block_n), _ptr(o),
                                      _dt(o), _ptr(lse), _ptr(lph), _ptr(lp), float(rescale_threshold), _stream()),
           "attn_fwd_fused")
    res = [o]
    if return_lse:
        res.append(lse)
    if debug:
        res += [lph, lp]
    return res[0] if len(res) == 1 else tuple(res)


# ------------------------------------------------------------------ decode ---
def decode_workspace_bytes(B, Hq, d, num_splits) -> int:
    return int(lib().hifa4_decode_workspace_size(B, Hq, d, num_splits))


def default_splits(B, Hkv, kv_len, block_n=128) -> int:
    return int(lib().hifa4_decode_default_splits(B, Hkv, kv_len, block_n))


def attn_decode(q: torch.Tensor, s: torch.Tensor | None, cache: QuantizedQKV, kv_len: int | None = None,
                softmax_scale: float | None = None, mode: int = PREORDER, num_splits: int = 0,
                workspace: torch.Tensor | None = None, out: torch.Tensor | None = None, out_dtype=torch.bfloat16,
                rescale_threshold: float = 0.0):
    """Split-KV decode of q [B,Hq,d] over the 4-bit cache.  Returns (O, splits_used).
    rescale_threshold > 0 updates each split's running max lazily."""
    B, Hq, d = q.shape
    kv = cache.N if kv_len is None else kv_len
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    if num_splits == 0:
        num_splits = default_splits(B, cache.Hkv, kv)
    ws_bytes = decode_workspace_bytes(B, Hq, d, num_splits)
    if workspace is None:
        workspace = torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
    o = out if out is not None else torch.empty((B, Hq, d), device=q.device, dtype=out_dtype)
    used = ctypes.c_int(0)
    q = q.contiguous()
    # the cache's layout is that of its capacity cache.N; decode reads kv tokens
    _check(lib().hifa4_attn_decode_cache(_ptr(q), _dt(q), _ptr(s), _ptr(cache.k_codes), _ptr(cache.k_scales),
                                         _ptr(cache.vt_codes), _ptr(cache.vt_scales), B, Hq, cache.Hkv, kv, cache.N,
                                         d, cache.fmt, float(softmax_scale), int(mode), 128, int(num_splits),
                                         ctypes.byref(used), _ptr(workspace), workspace.numel(), _ptr(o), _dt(o),
                                         float(rescale_threshold), _stream()), "attn_decode")
    return o, used.value


def attn_decode_noalloc(q: torch.Tensor, s: torch.Tensor | None, cache: QuantizedQKV, kv_len: int | None = None,
                        softmax_scale: float | None = None, mode: int = PREORDER, num_splits: int = 0,
                        out: torch.Tensor | None = None, out_dtype=torch.bfloat16):
    """Split-KV decode that allocates nothing on the device: the split partials
    live in the library's own scratch (for callers that may not allocate).
    Returns (O, splits_used)."""
    B, Hq, d = q.shape
    kv = cache.N if kv_len is None else kv_len
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    o = out if out is not None else torch.empty((B, Hq, d), device=q.device, dtype=out_dtype)
    used = ctypes.c_int(0)
    q = q.contiguous()
    _check(lib().hifa4_attn_decode_noalloc(_ptr(q), _dt(q), _ptr(s), _ptr(cache.k_codes), _ptr(cache.k_scales),
                                           _ptr(cache.vt_codes), _ptr(cache.vt_scales), B, Hq, cache.Hkv, kv, d,
                                           cache.fmt, float(softmax_scale), int(mode), 128, int(num_splits),
                                           ctypes.byref(used), _ptr(o), _dt(o), _stream()), "attn_decode_noalloc")
    return o, used.value


# ------------------------------------------------------------- measurement ---
def fp4_mma_probe(a_codes, a_scales, b_codes, b_scales, n: int, k: int, fmt: int, repeats: int = 1,
                  ctas: int = 1, out: torch.Tensor | None = None):
    d = out if out is not None else torch.empty((128, n), device=a_codes.device, dtype=torch.float32)
    _check(lib().hifa4_fp4_mma_probe(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), n, k, fmt,
                                     repeats, ctas, _ptr(d), _stream()), "fp4_mma_probe")
    return d


def div6_probe(lo_bits: int, hi_bits: int):
    """(mismatch count, first failing bit pattern) of the fast fl32(a/6)."""
    cnt = torch.zeros(1, dtype=torch.int64, device="cuda")
    first = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    _check(lib().hifa4_div6_probe(lo_bits, hi_bits, _ptr(cnt), _ptr(first), _stream()), "div6_probe")
    return int(cnt.item()), int(first.item()) & 0xFFFFFFFF


def wait_timeout_probe():
    """Run the bounded-wait failure path once; returns (wait succeeded, abort flag)."""
    st = torch.zeros(2, dtype=torch.int32, device="cuda")
    _check(lib().hifa4_wait_timeout_probe(_ptr(st), _stream()), "wait_timeout_probe")
    torch.cuda.synchronize()
    return bool(st[0].item()), int(st[1].item())


def bf16_transpose_v(v: torch.Tensor) -> torch.Tensor:
    """V [B, Hkv, N, d] bf16 -> V^T [B, Hkv, d, N] (the BF16 kernel's layout)."""
    v = v.contiguous()
    B, H, N, d = v.shape
    vt = torch.empty((B, H, d, N), device=v.device, dtype=torch.bfloat16)
    _check(lib().hifa4_bf16_transpose_v(_ptr(v), B, H, N, d, _ptr(vt), _stream()), "bf16_transpose_v")
    return vt


def bf16_attn_fwd(q: torch.Tensor, k: torch.Tensor, vt: torch.Tensor, softmax_scale: float | None = None,
                  causal: bool = True, return_lse: bool = False, out: torch.Tensor | None = None):
    """Plain BF16 attention (the unquantized baseline).  q [B,Hq,N,d], k [B,Hkv,N,d], vt [B,Hkv,d,N] bf16."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(d)
    o = out if out is not None else torch.empty_like(q)
    lse = torch.empty((B, Hq, N), device=q.device, dtype=torch.float32) if return_lse else None
    _check(lib().hifa4_bf16_attn_fwd(_ptr(q), _ptr(k), _ptr(vt), B, Hq, Hkv, N, d, float(softmax_scale), int(causal),
                                     _ptr(o), _ptr(lse) if lse is not None else None, _stream()), "bf16_attn_fwd")
    return (o, lse) if return_lse else o


def exp2_poly_probe(y: torch.Tensor) -> torch.Tensor:
    """The prefill kernel's FMA-pipe 2^y (for y <= 0) applied element-wise."""
    y = y.contiguous().float()
    out = torch.empty_like(y)
    _check(lib().hifa4_exp2_poly_probe(_ptr(y), y.numel(), _ptr(out), _stream()), "exp2_poly_probe")
    return out


def e2m1_map_probe(y: torch.Tensor):
    """E2M1 codes of 2^y from the exponential-free code argument and from the
    MUFU 2^y (one code per byte each)."""
    y = y.contiguous().float()
    cm = torch.empty(y.shape, device=y.device, dtype=torch.uint8)
    ce = torch.empty(y.shape, device=y.device, dtype=torch.uint8)
    _check(lib().hifa4_e2m1_map_probe(_ptr(y), y.numel(), _ptr(cm), _ptr(ce), _stream()), "e2m1_map_probe")
    return cm, ce


def convert_probe(x: torch.Tensor):
    x = x.contiguous().float()
    e2 = torch.empty(x.shape, device=x.device, dtype=torch.uint8)
    e4 = torch.empty(x.shape, device=x.device, dtype=torch.uint8)
    _check(lib().hifa4_convert_probe(_ptr(x), x.numel(), _ptr(e2), _ptr(e4), _stream()), "convert_probe")
    return e2, e4
