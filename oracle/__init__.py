"""CPU oracle for the 4-bit FlashAttention forward (Smooth-QK + P-Reordering).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with the CUDA library and the CUDA library never
calls it; the product path fails loudly when its own extension is missing.

The arithmetic lives in ``hifa4_oracle.c`` (plain C, fp64 outside the 4-bit
format decisions, which are made in IEEE fp32 as the written specification
fixes them).  This module only builds that file with gcc and marshals numpy
arrays.  Sources: "HiFA4: Training-Free 4-bit FlashAttention on Ascend HIF4
NPUs for LLM Inference", Abstract paragraphs 1-3; OCP MX v1.0 (E2M1, E8M0);
NVIDIA NVFP4 (16 x E2M1 + UE4M3).

Parity unpinned: the magnitude of the normalizer error epsilon (the paper's
-0.064 comes from a real Qwen3-8B trace that is not available here).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hifa4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libhifa4_oracle.so")
_lock = threading.Lock()
_lib = None

NVFP4, MXFP4 = 0, 1
PREORDER, INCONSISTENT = 0, 1
# oracle-only test knobs: P-hat = P, and fp64 scores/probabilities
VAR_NO_PQUANT, VAR_EXACT = 1, 2
# P-hat global prescale for NVFP4: g_P = 2^P_PRESCALE_LOG2 (a reading; the
# pages leave the HIF4 P-hat scale undefined).
P_PRESCALE_LOG2 = -8


def beta_of(fmt: int) -> int:
    return 16 if fmt == NVFP4 else 32


def pad128(n: int) -> int:
    return (n + 127) // 128 * 128


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    with _lock:
        if (not force and os.path.exists(_LIB_PATH)
                and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
            return _LIB_PATH
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
               "-fopenmp", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB_PATH)
        return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        path = build()
        L = ctypes.CDLL(path)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        i, i64, f, d = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_double
        L.or_threads.restype = i
        L.or_e2m1_encode.argtypes = [f]; L.or_e2m1_encode.restype = ctypes.c_uint8
        L.or_e2m1_decode.argtypes = [ctypes.c_uint8]; L.or_e2m1_decode.restype = d
        L.or_ue4m3_encode.argtypes = [f]; L.or_ue4m3_encode.restype = ctypes.c_uint8
        L.or_ue4m3_decode.argtypes = [ctypes.c_uint8]; L.or_ue4m3_decode.restype = d
        L.or_ue8m0_decode.argtypes = [ctypes.c_uint8]; L.or_ue8m0_decode.restype = d
        L.or_mx_exponent.argtypes = [f]; L.or_mx_exponent.restype = i
        L.or_encode_array.argtypes = [f32p, i64, u8p, u8p]
        L.or_quant_block_nvfp4.argtypes = [f32p, i, f, u8p]; L.or_quant_block_nvfp4.restype = ctypes.c_uint8
        L.or_quant_block_mxfp4.argtypes = [f32p, i, u8p]; L.or_quant_block_mxfp4.restype = ctypes.c_uint8
        L.or_quantize_rows.argtypes = [f32p, i64, i, i, f, u8p, u8p]
        L.or_sf_tiled_offset.argtypes = [i64, i, i]; L.or_sf_tiled_offset.restype = i64
        L.or_sf_tile.argtypes = [u8p, i64, i, u8p, i64]
        L.or_calibrate.argtypes = [f32p, f32p, i, i, i, i, i, i, d, i, f32p, f32p]
        L.or_calibrate_q_mean.argtypes = [f32p, i, i, i, i, i, i, f32p, f32p]
        L.or_quantize_qkv.argtypes = [f32p, f32p, f32p, i, i, i, i, i, f32p, f32p, i,
                                      u8p, u8p, u8p, u8p, u8p, u8p, f32p]
        L.or_attention.argtypes = [u8p, u8p, u8p, u8p, u8p, u8p, i, i, i, i, i, i, d, i, i,
                                   i, i, f64p, f64p, f64p, f64p, u8p, u8p, f64p, f64p,
                                   f32p, f32p, f32p, i, i, i, f, f32p]
        L.or_split_len.argtypes = [i, i, i]; L.or_split_len.restype = i
        L.or_decode.argtypes = [f32p, f32p, u8p, u8p, u8p, u8p, i, i, i, i, i, i, d, i, i, i,
                                i, f64p, f64p, i, f]
        _lib = L
    return _lib


def threads() -> int:
    return int(lib().or_threads())


def _p(a, ct):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


# ---------------------------------------------------------------- formats ---
def e2m1_encode(x) -> np.ndarray:
    x = _f32(x).ravel()
    f = lib().or_e2m1_encode
    return np.array([f(float(v)) for v in x], dtype=np.uint8)


def e2m1_decode(codes) -> np.ndarray:
    f = lib().or_e2m1_decode
    return np.array([f(int(c)) for c in np.asarray(codes).ravel()], dtype=np.float64)


def ue4m3_encode(t) -> np.ndarray:
    t = _f32(t).ravel()
    f = lib().or_ue4m3_encode
    return np.array([f(float(v)) for v in t], dtype=np.uint8)


def ue4m3_decode(codes) -> np.ndarray:
    f = lib().or_ue4m3_decode
    return np.array([f(int(c)) for c in np.asarray(codes).ravel()], dtype=np.float64)


def ue8m0_decode(codes) -> np.ndarray:
    f = lib().or_ue8m0_decode
    return np.array([f(int(c)) for c in np.asarray(codes).ravel()], dtype=np.float64)


def encode_array(x):
    """(E2M1(x), UE4M3(|x|)) element-wise, as uint8 arrays."""
    x = _f32(x).ravel()
    e2 = np.zeros(x.size, np.uint8)
    e4 = np.zeros(x.size, np.uint8)
    lib().or_encode_array(_p(x, ctypes.c_float), x.size, _p(e2, ctypes.c_uint8), _p(e4, ctypes.c_uint8))
    return e2, e4


def mx_exponent(amax: float) -> int:
    return int(lib().or_mx_exponent(float(amax)))


def quantize_rows(x, fmt: int, g: float = 1.0):
    """x [rows, K] -> (codes [rows, K/2] packed, scales [rows, K/beta] plain)."""
    x = _f32(x)
    rows, K = x.shape
    beta = beta_of(fmt)
    codes = np.zeros((rows, K // 2), np.uint8)
    sc = np.zeros((rows, K // beta), np.uint8)
    lib().or_quantize_rows(_p(x, ctypes.c_float), rows, K, fmt, float(g),
                           _p(codes, ctypes.c_uint8), _p(sc, ctypes.c_uint8))
    return codes, sc


def unpack_codes(codes: np.ndarray) -> np.ndarray:
    """[..., K/2] packed bytes -> [..., K] 4-bit codes (low nibble first)."""
    c = np.asarray(codes, dtype=np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = c & 15
    out[..., 1::2] = c >> 4
    return out


def dequantize_rows(codes, scales, fmt: int, g: float = 1.0) -> np.ndarray:
    """Plain numpy dequantization (fp64) of packed codes with plain scales."""
    beta = beta_of(fmt)
    c = unpack_codes(codes).astype(np.int64)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float64)
    mag = grid[c & 7] * np.where(c & 8, -1.0, 1.0)
    sc = np.asarray(scales).astype(np.int64)
    if fmt == NVFP4:
        sdv = ue4m3_decode(np.arange(128))
        sd = (sdv[np.minimum(sc, 127)] * g).astype(np.float32).astype(np.float64)
    else:
        sd = np.ldexp(1.0, sc - 127)
    return mag * np.repeat(sd, beta, axis=-1)


def sf_tile(plain: np.ndarray, rows_padded: int | None = None) -> np.ndarray:
    """Plain [rows, nb] scales -> tiled byte layout (rows padded to 128)."""
    plain = np.ascontiguousarray(plain, dtype=np.uint8)
    rows, nb = plain.shape
    rp = rows_padded if rows_padded is not None else pad128(rows)
    nkc = (nb + 3) // 4
    out = np.zeros((rp // 128) * nkc * 512, np.uint8)
    lib().or_sf_tile(_p(plain, ctypes.c_uint8), rows, nb, _p(out, ctypes.c_uint8), rp)
    return out


def sf_tiled_bytes(rows: int, nb: int) -> int:
    return (pad128(rows) // 128) * ((nb + 3) // 4) * 512


# ------------------------------------------------------------ calibration ---
GATE = 2   # calibrate(enable=GATE): the per-head applicability gate


def calibrate(q, k, n_cal: int, alpha: float = 0.5, enable=True):
    """q [B,Hq,T,d], k [B,Hkv,T,d] (float) -> (s, inv_s) [Hkv, d] float32.
    enable: False / True, or GATE (smoothing per kv head only where its
    largest K channel amax exceeds 8 x the channel median)."""
    q = _f32(q); k = _f32(k)
    B, Hq, T, d = q.shape
    Hkv = k.shape[1]
    s = np.zeros((Hkv, d), np.float32)
    inv = np.zeros((Hkv, d), np.float32)
    lib().or_calibrate(_p(q, ctypes.c_float), _p(k, ctypes.c_float), B, Hq, Hkv, n_cal, T, d,
                       float(alpha), int(enable), _p(s, ctypes.c_float), _p(inv, ctypes.c_float))
    return s, inv


def calibrate_q_mean(q, s, n_cal: int):
    """Q-Mean auxiliary (a reading; the pages name it only): the per-channel
    mean of the smoothed query over the calibration tokens, q [B,Hq,T,d],
    s [Hkv,d] or None -> mu [Hq,d] float32."""
    q = _f32(q)
    B, Hq, T, d = q.shape
    s32 = _f32(s) if s is not None else None
    Hkv = s32.shape[0] if s32 is not None else Hq
    mu = np.zeros((Hq, d), np.float32)
    lib().or_calibrate_q_mean(_p(q, ctypes.c_float), B, Hq, Hkv, n_cal, T, d,
                              _p(s32, ctypes.c_float) if s32 is not None else None, _p(mu, ctypes.c_float))
    return mu


# ------------------------------------------------------------- quantize ---
def quantize_qkv(q, k, v, s=None, inv_s=None, fmt: int = NVFP4, q_mu=None):
    """Fused Smooth-QK scale + block quantization; plain scale layouts.
    q_mu [Hq,d]: the Q-Mean auxiliary, subtracted from the smoothed query.

    Returns dict with q_codes [B,Hq,Np,d/2], q_sc [B,Hq,Np,d/beta],
    k_codes, k_sc (Hkv), vt_codes [B,Hkv,d,Np/2], vt_sc [B,Hkv,d,Np/beta].
    """
    q = _f32(q); k = _f32(k); v = _f32(v)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    beta = beta_of(fmt)
    Np = pad128(N)
    out = dict(
        q_codes=np.zeros((B, Hq, Np, d // 2), np.uint8), q_sc=np.zeros((B, Hq, Np, d // beta), np.uint8),
        k_codes=np.zeros((B, Hkv, Np, d // 2), np.uint8), k_sc=np.zeros((B, Hkv, Np, d // beta), np.uint8),
        vt_codes=np.zeros((B, Hkv, d, Np // 2), np.uint8), vt_sc=np.zeros((B, Hkv, d, Np // beta), np.uint8))
    s_keep = (_f32(s) if s is not None else None, _f32(inv_s) if inv_s is not None else None)
    sp = _p(s_keep[0], ctypes.c_float) if s_keep[0] is not None else None
    ip = _p(s_keep[1], ctypes.c_float) if s_keep[1] is not None else None
    mu = _f32(q_mu) if q_mu is not None else None
    lib().or_quantize_qkv(_p(q, ctypes.c_float), _p(k, ctypes.c_float), _p(v, ctypes.c_float),
                          B, Hq, Hkv, N, d, sp, ip, fmt,
                          *[_p(out[n], ctypes.c_uint8) for n in
                            ("q_codes", "q_sc", "k_codes", "k_sc", "vt_codes", "vt_sc")],
                          _p(mu, ctypes.c_float) if mu is not None else None)
    return out


def tile_scales(qz: dict) -> dict:
    """Plain scale arrays of quantize_qkv -> the tiled layouts, per head."""
    out = {}
    for name in ("q_sc", "k_sc", "vt_sc"):
        a = qz[name]
        lead = a.shape[:-2]
        rows, nb = a.shape[-2:]
        flat = a.reshape(-1, rows, nb)
        out[name] = np.stack([sf_tile(t) for t in flat]).reshape(lead + (-1,))
    return out


# ------------------------------------------------------------ attention ---
def attention(qz: dict, N: int, fmt: int = NVFP4, softmax_scale: float | None = None,
              causal: bool = True, mode: int = PREORDER, BN: int = 128,
              pexp: int = P_PRESCALE_LOG2, rows=None, dump_phat: bool = False,
              variant: int = 0, tau: float = 0.0, raw: dict | None = None, q_mu=None):
    """Oracle forward over the quantized tensors of quantize_qkv.

    Returns dict O [B,Hq,N,d] fp64, lse, l_phat, l_p [B,Hq,N]; optional P-hat
    dump (codes, scales, running max and the per-tile sums of P-hat and P).
    rows=(begin, end) restricts the query rows computed (other rows of the
    outputs stay NaN).  tau > 0: the running max moves only when a tile's max
    exceeds it by more than tau (lazy rescaling).  raw: test-only ablation,
    {"q"|"k"|"v": float array} in [B,H,N,d] replacing the dequantized operand.
    q_mu [Hq,d]: the Q-Mean auxiliary; every score gets back mu . k of its key.
    """
    qc, qs = qz["q_codes"], qz["q_sc"]
    B, Hq, Np, dh = qc.shape
    d = dh * 2
    Hkv = qz["k_codes"].shape[1]
    if softmax_scale is None:
        softmax_scale = 1.0 / np.sqrt(d)
    r0, r1 = (0, N) if rows is None else rows
    O = np.full((B, Hq, N, d), np.nan)
    lse = np.full((B, Hq, N), np.nan)
    lph = np.full((B, Hq, N), np.nan)
    lp = np.full((B, Hq, N), np.nan)
    ntiles = (N + BN - 1) // BN
    beta = beta_of(fmt)
    if BN % beta:
        raise ValueError(f"key tile {BN} is not a multiple of the P-hat block {beta}")
    pd = np.zeros((B, Hq, N, ntiles * BN), np.uint8) if dump_phat else None
    psd = np.zeros((B, Hq, N, ntiles * BN // beta), np.uint8) if dump_phat else None
    md = np.full((B, Hq, N, ntiles), np.nan) if dump_phat else None
    ts = np.full((B, Hq, N, ntiles, 2), np.nan) if dump_phat else None
    raw = raw or {}
    rq, rk, rv = (None if raw.get(n) is None else _f32(raw[n]) for n in ("q", "k", "v"))
    arrs = [np.ascontiguousarray(qz[n]) for n in ("q_codes", "q_sc", "k_codes", "k_sc", "vt_codes", "vt_sc")]
    mu = _f32(q_mu) if q_mu is not None else None
    lib().or_attention(*[_p(a, ctypes.c_uint8) for a in arrs], B, Hq, Hkv, N, d, fmt,
                       float(softmax_scale), int(causal), int(mode), int(BN), int(pexp),
                       _p(O, ctypes.c_double), _p(lse, ctypes.c_double), _p(lph, ctypes.c_double),
                       _p(lp, ctypes.c_double), _p(pd, ctypes.c_uint8), _p(psd, ctypes.c_uint8),
                       _p(md, ctypes.c_double), _p(ts, ctypes.c_double), _p(rq, ctypes.c_float),
                       _p(rk, ctypes.c_float), _p(rv, ctypes.c_float), int(r0), int(r1), int(variant), float(tau),
                       _p(mu, ctypes.c_float) if mu is not None else None)
    res = dict(O=O, lse=lse, l_phat=lph, l_p=lp)
    if dump_phat:
        res["phat_codes"] = pd
        res["phat_sc"] = psd
        res["m_tiles"] = md
        res["tile_sum_phat"] = ts[..., 0]
        res["tile_sum_p"] = ts[..., 1]
    return res


def tile_epsilon(sum_phat: np.ndarray, sum_p: np.ndarray, BM: int = 128) -> np.ndarray:
    """Normalizer error of each attention tile (a reading: the pages measure
    epsilon per tile without defining it): for the BM query rows x BN keys of
    tile (b, h, query tile, key tile), sum of P-hat over sum of P, minus one.
    Inputs are the per-row, per-key-tile sums [B,H,N,nkt] of attention(...,
    dump_phat=True), each relative to its row's running max at that tile;
    rows the oracle did not compute (NaN) and tiles with no visible key are
    left out.  Returns [B,H,ceil(N/BM),nkt] with NaN where a tile is empty."""
    B, H, N, nkt = sum_p.shape
    nq = (N + BM - 1) // BM
    pad = nq * BM - N
    sph = np.nan_to_num(np.pad(sum_phat, ((0, 0), (0, 0), (0, pad), (0, 0))), nan=0.0)
    sp = np.nan_to_num(np.pad(sum_p, ((0, 0), (0, 0), (0, pad), (0, 0))), nan=0.0)
    a = sph.reshape(B, H, nq, BM, nkt).sum(axis=3)
    b = sp.reshape(B, H, nq, BM, nkt).sum(axis=3)
    with np.errstate(invalid="ignore", divide="ignore"):
        return np.where(b > 0, a / b - 1.0, np.nan)


def split_len(kv_len: int, num_splits: int, BN: int) -> int:
    return int(lib().or_split_len(kv_len, num_splits, BN))


def decode(q, s, cache: dict, kv_len: int, fmt: int = NVFP4, softmax_scale: float | None = None,
           mode: int = PREORDER, BN: int = 128, num_splits: int = 1,
           pexp: int = P_PRESCALE_LOG2, variant: int = 0, tau: float = 0.0):
    """Split-KV decode: q [B,Hq,d] float, cache = quantize_qkv output (N=kv_len).
    tau: lazy running-max threshold of each split, as in attention()."""
    q = _f32(q)
    B, Hq, d = q.shape
    Hkv = cache["k_codes"].shape[1]
    if BN % beta_of(fmt):
        raise ValueError(f"key tile {BN} is not a multiple of the P-hat block {beta_of(fmt)}")
    if softmax_scale is None:
        softmax_scale = 1.0 / np.sqrt(d)
    O = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    s32 = _f32(s) if s is not None else None
    arrs = [np.ascontiguousarray(cache[n]) for n in ("k_codes", "k_sc", "vt_codes", "vt_sc")]
    lib().or_decode(_p(q, ctypes.c_float), _p(s32, ctypes.c_float) if s32 is not None else None,
                    *[_p(a, ctypes.c_uint8) for a in arrs], B, Hq, Hkv, kv_len, d, fmt,
                    float(softmax_scale), int(mode), int(BN), int(num_splits), int(pexp),
                    _p(O, ctypes.c_double), _p(lse, ctypes.c_double), int(variant), float(tau))
    return dict(O=O, lse=lse)
