"""A second, loop-only implementation of the written specification, for tiny
shapes.  It shares no code with the C oracle: element and scale rounding come
from the ml_dtypes library casts (float4_e2m1fn, float8_e4m3fn), everything
else is spelled out with Python loops over rows, key tiles, blocks and keys.

Used only to pin the oracle (tests/test_oracle_attention.py).
"""
from __future__ import annotations

import math

import ml_dtypes
import numpy as np

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def e2m1(y: float) -> int:
    """RNE to E2M1 with saturation (ml_dtypes' cast saturates); sign kept."""
    return int(np.array([y], np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8)[0]) & 15


def e2m1_val(c: int) -> float:
    v = GRID[c & 7]
    return -v if c & 8 else v


def ue4m3(t: float) -> int:
    """RNE to E4M3 with saturation at 448 (clamp first: ml_dtypes does not saturate)."""
    t = min(float(np.float32(t)), 448.0)
    return int(np.array([t], np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)[0])


def ue4m3_val(c: int) -> float:
    return float(np.array([c], np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)[0])


def nvfp4_block(x, g: float):
    x = [np.float32(v) for v in x]
    amax = np.float32(0.0)
    for v in x:
        amax = max(amax, np.float32(abs(v)))
    t = np.float32(np.float32(amax / np.float32(6.0)) / np.float32(g))
    sc = ue4m3(t)
    sd = np.float32(np.float32(ue4m3_val(sc)) * np.float32(g))
    if sd == 0:
        return [0] * len(x), sc, [0.0] * len(x)
    inv = np.float32(np.float32(1.0) / sd)
    codes = [e2m1(float(np.float32(v * inv))) for v in x]
    return codes, sc, [e2m1_val(c) * float(sd) for c in codes]


def mxfp4_block(x):
    x = [np.float32(v) for v in x]
    amax = max(float(abs(v)) for v in x)
    if amax == 0.0:
        E = -127
    else:
        E = math.floor(math.log2(amax)) - 2
        # guard the float log2 at exact powers of two
        while 2.0 ** (E + 2) > amax:
            E -= 1
        while 2.0 ** (E + 3) <= amax:
            E += 1
        E = max(-127, min(127, E))
    codes = [e2m1(float(np.float32(float(v) * 2.0 ** (-E)))) for v in x]
    return codes, E + 127, [e2m1_val(c) * 2.0 ** E for c in codes]


def quantize_vec(x, fmt: int, g: float = 1.0):
    beta = 16 if fmt == 0 else 32
    codes, scales, deq = [], [], []
    for b0 in range(0, len(x), beta):
        blk = x[b0:b0 + beta]
        c, s, dq = nvfp4_block(blk, g) if fmt == 0 else mxfp4_block(blk)
        codes += c
        scales.append(s)
        deq += dq
    return codes, scales, deq


def pack(codes):
    return [codes[i] | (codes[i + 1] << 4) for i in range(0, len(codes), 2)]


def quantize_qkv(q, k, v, s, inv_s, fmt):
    """Same layouts as the oracle (plain scales, rows padded to 128)."""
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    beta = 16 if fmt == 0 else 32
    Np = (N + 127) // 128 * 128
    out = dict(q_codes=np.zeros((B, Hq, Np, d // 2), np.uint8), q_sc=np.zeros((B, Hq, Np, d // beta), np.uint8),
               k_codes=np.zeros((B, Hkv, Np, d // 2), np.uint8), k_sc=np.zeros((B, Hkv, Np, d // beta), np.uint8),
               vt_codes=np.zeros((B, Hkv, d, Np // 2), np.uint8), vt_sc=np.zeros((B, Hkv, d, Np // beta), np.uint8))
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            for t in range(Np):
                row = [float(np.float32(q[b, hq, t, c]) * np.float32(s[h, c])) if t < N else 0.0 for c in range(d)]
                c_, s_, _ = quantize_vec(row, fmt)
                out["q_codes"][b, hq, t] = pack(c_)
                out["q_sc"][b, hq, t] = s_
        for h in range(Hkv):
            for t in range(Np):
                row = [float(np.float32(k[b, h, t, c]) * np.float32(inv_s[h, c])) if t < N else 0.0 for c in range(d)]
                c_, s_, _ = quantize_vec(row, fmt)
                out["k_codes"][b, h, t] = pack(c_)
                out["k_sc"][b, h, t] = s_
            for c in range(d):
                row = [float(v[b, h, t, c]) if t < N else 0.0 for t in range(Np)]
                c_, s_, _ = quantize_vec(row, fmt)
                out["vt_codes"][b, h, c] = pack(c_)
                out["vt_sc"][b, h, c] = s_
    return out


def _deq_row(codes_row, sc_row, fmt):
    beta = 16 if fmt == 0 else 32
    out = []
    for i in range(len(codes_row) * 2):
        byte = int(codes_row[i // 2])
        c = byte & 15 if i % 2 == 0 else byte >> 4
        sc = int(sc_row[i // beta])
        sd = ue4m3_val(sc) if fmt == 0 else 2.0 ** (sc - 127)
        out.append(e2m1_val(c) * sd)
    return out


def attention(qz, N, fmt, softmax_scale, causal, mode, BN, pexp=-8, tau=0.0, tile_sums=False):
    """Returns O [B,Hq,N,d] (fp64) and (l_phat, l_p).  tau: the running max
    moves to the tile max only when that exceeds fl32(m + tau).  tile_sums:
    also return [B,Hq,N,nkt,2], the sum of P-hat and of P over each key tile
    a row visits (NaN for the tiles past its last visible key)."""
    qc = qz["q_codes"]
    B, Hq, Np, dh = qc.shape
    d = dh * 2
    Hkv = qz["k_codes"].shape[1]
    G = Hq // Hkv
    beta = 16 if fmt == 0 else 32
    g = 2.0 ** pexp if fmt == 0 else 1.0
    c_log2 = softmax_scale * 1.4426950408889634074
    O = np.zeros((B, Hq, N, d))
    LPH = np.zeros((B, Hq, N))
    LP = np.zeros((B, Hq, N))
    TS = np.full((B, Hq, N, (N + BN - 1) // BN, 2), np.nan)
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            K = [_deq_row(qz["k_codes"][b, h, t], qz["k_sc"][b, h, t], fmt) for t in range(N)]
            VT = [_deq_row(qz["vt_codes"][b, h, c], qz["vt_sc"][b, h, c], fmt) for c in range(d)]
            for i in range(N):
                qrow = _deq_row(qz["q_codes"][b, hq, i], qz["q_sc"][b, hq, i], fmt)
                m, lph, lp = -math.inf, 0.0, 0.0
                acc = [0.0] * d
                last = i + 1 if causal else N
                for j0 in range(0, last, BN):
                    xs = []
                    for key in range(j0, j0 + BN):
                        if key < last:
                            sdot = 0.0
                            for c in range(d):
                                sdot += qrow[c] * K[key][c]
                            xs.append(float(np.float32(sdot * c_log2)))
                        else:
                            xs.append(None)
                    mt = max(x for x in xs if x is not None)
                    m_new = mt if mt > float(np.float32(m) + np.float32(tau)) else m
                    alpha = 0.0 if m == -math.inf else math.exp2(m - m_new)
                    P = []
                    for x in xs:
                        if x is None:
                            P.append(0.0)
                        else:
                            p = float(np.float32(math.exp2(x - m_new)))
                            P.append(0.0 if p < 2.0 ** -126 else p)
                    Ph = []
                    for b0 in range(0, BN, beta):
                        blk = P[b0:b0 + beta]
                        _, _, dq = nvfp4_block(blk, g) if fmt == 0 else mxfp4_block(blk)
                        Ph += dq
                    sp = 0.0
                    sph = 0.0
                    for kk in range(BN):
                        sp += P[kk]
                        sph += Ph[kk]
                    TS[b, hq, i, j0 // BN] = (sph, sp)
                    lp = alpha * lp + sp
                    lph = alpha * lph + sph
                    for c in range(d):
                        a = 0.0
                        for kk in range(BN):
                            if Ph[kk] != 0.0:
                                a += Ph[kk] * VT[c][j0 + kk]
                        acc[c] = alpha * acc[c] + a
                    m = m_new
                l = lph if mode == 0 else lp
                O[b, hq, i] = [a / l for a in acc]
                LPH[b, hq, i] = lph
                LP[b, hq, i] = lp
    if tile_sums:
        return O, LPH, LP, TS
    return O, LPH, LP
