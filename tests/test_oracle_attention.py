"""Pins of the oracle's quantize / attention / decode layer (no GPU).

Each test checks the oracle against something other than itself: a second,
loop-only implementation (tests/bruteforce.py), textbook softmax attention,
closed-form identities of the method ("HiFA4: Training-Free 4-bit
FlashAttention on Ascend HIF4 NPUs for LLM Inference", Abstract para 2:
Smooth-QK is an equivalent rescaling; P-Reordering normalizes by the same
P-hat that feeds the PV GEMM; Theorem 1's error is a coherent output scaling),
and the sign of epsilon given by the announcement abstract ("net
probability-mass loss").  The magnitude of epsilon is parity unpinned.
"""
import itertools

import numpy as np
import pytest

import oracle
from tests import bruteforce

GRID = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])


def _inputs(B, Hq, Hkv, N, d, seed, outlier=True):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hq, N, d)).astype(np.float32)
    k = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    if outlier:
        k[..., d - 2:] = 12 * np.abs(k[..., d - 2:])
    return q, k, v


def _dequant_all(qz, fmt):
    out = {}
    for name, sc in (("q", "q_sc"), ("k", "k_sc"), ("vt", "vt_sc")):
        c = qz[name + "_codes"]
        out[name] = oracle.dequantize_rows(c.reshape(-1, c.shape[-1]), qz[sc].reshape(-1, qz[sc].shape[-1]),
                                           fmt).reshape(c.shape[:-1] + (c.shape[-1] * 2,))
    return out


def _textbook(qd, kd, vd, N, scale, causal, G):
    """softmax(Q K^T * scale) V in fp64 over the given (dequantized) tensors."""
    B, Hq = qd.shape[:2]
    O = np.zeros((B, Hq, N, qd.shape[-1]))
    for b in range(B):
        for hq in range(Hq):
            h = hq // G
            S = qd[b, hq, :N] @ kd[b, h, :N].T * scale
            if causal:
                S = np.where(np.tril(np.ones((N, N), bool)), S, -np.inf)
            S = S - S.max(-1, keepdims=True)
            P = np.exp(S)
            O[b, hq] = (P / P.sum(-1, keepdims=True)) @ vd[b, h, :N]
    return O


@pytest.mark.parametrize("fmt", [oracle.NVFP4, oracle.MXFP4])
def test_quantize_equals_bruteforce(fmt):
    B, Hq, Hkv, N, d = 1, 4, 2, 40, 64
    q, k, v = _inputs(B, Hq, Hkv, N, d, 10 + fmt)
    s, inv = oracle.calibrate(q, k, n_cal=16, alpha=0.5)
    ours = oracle.quantize_qkv(q, k, v, s, inv, fmt)
    ref = bruteforce.quantize_qkv(q, k, v, s, inv, fmt)
    for name in ours:
        assert np.array_equal(ours[name], ref[name]), name


CASES = [
    # (fmt, N, d, BN, causal, G, mode)
    (oracle.NVFP4, 16, 16, 16, True, 1, oracle.PREORDER),
    (oracle.NVFP4, 48, 32, 16, True, 2, oracle.PREORDER),
    (oracle.NVFP4, 48, 32, 32, False, 2, oracle.INCONSISTENT),
    (oracle.NVFP4, 64, 16, 32, True, 1, oracle.INCONSISTENT),
    (oracle.MXFP4, 40, 32, 32, True, 2, oracle.PREORDER),
    (oracle.MXFP4, 64, 32, 32, False, 1, oracle.INCONSISTENT),
]


@pytest.mark.parametrize("fmt,N,d,BN,causal,G,mode", CASES)
def test_attention_equals_bruteforce(fmt, N, d, BN, causal, G, mode):
    Hkv = 1
    q, k, v = _inputs(1, G * Hkv, Hkv, N, d, 20 + N + d)
    s, inv = oracle.calibrate(q, k, n_cal=8, alpha=0.5)
    qz = oracle.quantize_qkv(q, k, v, s, inv, fmt)
    scale = 1 / np.sqrt(d)
    ours = oracle.attention(qz, N, fmt, scale, causal, mode, BN)
    O, lph, lp = bruteforce.attention(qz, N, fmt, scale, causal, mode, BN)
    np.testing.assert_allclose(ours["O"], O, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(ours["l_phat"], lph, rtol=1e-13)
    np.testing.assert_allclose(ours["l_p"], lp, rtol=1e-13)


@pytest.mark.parametrize("causal,BN,G", [(True, 16, 2), (False, 32, 1), (True, 64, 4)])
def test_quant_off_is_textbook_softmax(causal, BN, G):
    """P quantizer replaced by the identity and fp64 scores: the tiled online
    recurrence must equal two-pass softmax attention over the same Q,K,V."""
    N, d = 72, 32
    q, k, v = _inputs(2, 2 * G, 2, N, d, 30 + BN)
    qz = oracle.quantize_qkv(q, k, v, None, None, oracle.NVFP4)
    deq = _dequant_all(qz, oracle.NVFP4)
    scale = 0.3
    res = oracle.attention(qz, N, oracle.NVFP4, scale, causal, oracle.PREORDER, BN,
                           variant=oracle.VAR_NO_PQUANT | oracle.VAR_EXACT)
    vd = np.swapaxes(deq["vt"], -1, -2)
    ref = _textbook(deq["q"], deq["k"], vd, N, scale, causal, G)
    np.testing.assert_allclose(res["O"], ref, rtol=1e-12, atol=1e-13)
    # the inconsistent normalizer is the same thing when P-hat = P
    res2 = oracle.attention(qz, N, oracle.NVFP4, scale, causal, oracle.INCONSISTENT, BN,
                            variant=oracle.VAR_NO_PQUANT | oracle.VAR_EXACT)
    np.testing.assert_allclose(res2["O"], ref, rtol=1e-12, atol=1e-13)


def _lossless_qk(B, Hq, Hkv, N, d, rng):
    """Q, K whose every 16-block is grid values x 2^e with a +-6 entry, so
    NVFP4 quantization is exact; also pow2 Smooth-QK scales constant per
    16-channel block that keep it exact."""
    def make(H):
        vals = rng.choice(np.concatenate([GRID, -GRID]), (B, H, N, d))
        vals[..., ::16] = 6.0
        e = rng.integers(-3, 3, (B, H, N, d // 16))
        return (vals * np.repeat(2.0 ** e, 16, axis=-1)).astype(np.float32)
    q, k = make(Hq), make(Hkv)
    s = np.repeat(2.0 ** rng.integers(-2, 3, (Hkv, d // 16)), 16, axis=-1).astype(np.float32)
    return q, k, s


def test_smooth_qk_is_equivalent_rescaling():
    rng = np.random.default_rng(5)
    B, Hq, Hkv, N, d = 1, 4, 2, 40, 32
    q, k, s = _lossless_qk(B, Hq, Hkv, N, d, rng)
    v = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    inv = (1.0 / s).astype(np.float32)
    qz_s = oracle.quantize_qkv(q, k, v, s, inv, oracle.NVFP4)
    qz_1 = oracle.quantize_qkv(q, k, v, None, None, oracle.NVFP4)
    deq = _dequant_all(qz_s, oracle.NVFP4)
    G = Hq // Hkv
    # Q is scaled by s of its kv head (head hq -> hq // G), K by 1/s
    for hq in range(Hq):
        np.testing.assert_array_equal(deq["q"][0, hq, :N], q[0, hq] * s[hq // G])
    for h in range(Hkv):
        np.testing.assert_array_equal(deq["k"][0, h, :N], k[0, h] * inv[h])
    # QK^T is unchanged, so the whole forward is bit-identical
    for mode in (oracle.PREORDER, oracle.INCONSISTENT):
        a = oracle.attention(qz_s, N, oracle.NVFP4, 0.25, True, mode, 16)
        b = oracle.attention(qz_1, N, oracle.NVFP4, 0.25, True, mode, 16)
        np.testing.assert_array_equal(a["O"], b["O"])


@pytest.mark.parametrize("fmt,BN", [(oracle.NVFP4, 16), (oracle.NVFP4, 64), (oracle.MXFP4, 32)])
def test_preorder_two_pass_identity(fmt, BN):
    """P-Reordering: O = sum_j w_j P-hat_j V-hat / sum_j w_j sum(P-hat_j),
    w_j = 2^(m_j - m_final), rebuilt from the P-hat codes the online pass used."""
    N, d, G = 100, 32, 2
    q, k, v = _inputs(1, G, 1, N, d, 40 + BN)
    s, inv = oracle.calibrate(q, k, n_cal=16)
    qz = oracle.quantize_qkv(q, k, v, s, inv, fmt)
    res = oracle.attention(qz, N, fmt, 1 / np.sqrt(d), True, oracle.PREORDER, BN, dump_phat=True)
    beta = oracle.beta_of(fmt)
    g = 2.0 ** oracle.P_PRESCALE_LOG2 if fmt == oracle.NVFP4 else 1.0
    vd = np.swapaxes(_dequant_all(qz, fmt)["vt"], -1, -2)[0, 0]
    for hq in range(G):
        for i in (0, 17, 63, 64, 99):
            ntl = i // BN + 1
            codes = res["phat_codes"][0, hq, i, :ntl * BN]
            sc = res["phat_sc"][0, hq, i, :ntl * BN // beta]
            grid = GRID[codes & 7]
            if fmt == oracle.NVFP4:
                sd = (oracle.ue4m3_decode(sc) * g).astype(np.float32).astype(np.float64)
            else:
                sd = 2.0 ** (sc.astype(np.float64) - 127)
            phat = grid * np.repeat(sd, beta)
            m = res["m_tiles"][0, hq, i, :ntl]
            w = np.repeat(2.0 ** (m - m[-1]), BN)
            num = (w * phat) @ vd[:ntl * BN]
            den = np.sum(w * phat)
            np.testing.assert_allclose(res["O"][0, hq, i], num / den, rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(res["l_phat"][0, hq, i], den, rtol=1e-12)


@pytest.mark.parametrize("fmt", [oracle.NVFP4, oracle.MXFP4])
def test_theorem1_coherent_scaling_and_sign(fmt):
    """Inconsistent normalizer: O_incons[r,:] = (l_phat / l_p) O_reord[r,:]
    exactly (same numerator), i.e. one scale per row across all channels;
    the error eps = l_phat / l_p - 1 is a net probability-mass loss."""
    N, d, G = 256, 64, 2
    q, k, v = _inputs(1, G, 1, N, d, 50)
    s, inv = oracle.calibrate(q, k, n_cal=64)
    qz = oracle.quantize_qkv(q, k, v, s, inv, fmt)
    a = oracle.attention(qz, N, fmt, 1 / np.sqrt(d), True, oracle.PREORDER, 64)
    b = oracle.attention(qz, N, fmt, 1 / np.sqrt(d), True, oracle.INCONSISTENT, 64)
    ratio = a["l_phat"] / a["l_p"]
    np.testing.assert_allclose(b["O"], a["O"] * ratio[..., None], rtol=1e-12, atol=1e-14)
    eps = ratio - 1
    assert np.median(eps) < 0, np.median(eps)


def test_decode_single_split_equals_last_causal_row():
    B, Hq, Hkv, N, d = 2, 4, 2, 200, 64
    q, k, v = _inputs(B, Hq, Hkv, N, d, 60)
    s, inv = oracle.calibrate(q, k, n_cal=32)
    qz = oracle.quantize_qkv(q, k, v, s, inv, oracle.NVFP4)
    for mode in (oracle.PREORDER, oracle.INCONSISTENT):
        pre = oracle.attention(qz, N, oracle.NVFP4, 1 / 8, True, mode, 64, rows=(N - 1, N))
        dec = oracle.decode(q[:, :, N - 1], s, qz, N, oracle.NVFP4, 1 / 8, mode, 64, num_splits=1)
        np.testing.assert_array_equal(dec["O"], pre["O"][:, :, N - 1])
        np.testing.assert_allclose(dec["lse"], pre["lse"][:, :, N - 1], rtol=1e-15)


@pytest.mark.parametrize("splits", [1, 3, 7])
def test_decode_split_combine_exact_when_quant_off(splits):
    B, Hq, Hkv, N, d = 1, 4, 2, 300, 32
    q, k, v = _inputs(B, Hq, Hkv, N, d, 70)
    qz = oracle.quantize_qkv(q, k, v, None, None, oracle.NVFP4)
    deq = _dequant_all(qz, oracle.NVFP4)
    # the decode query is quantized like a Q row; take it from a one-row quantize
    qq = oracle.quantize_qkv(q[:, :, N - 1:N], k[:, :, :1], v[:, :, :1], None, None, oracle.NVFP4)
    qd = _dequant_all(qq, oracle.NVFP4)["q"][:, :, :1]
    res = oracle.decode(q[:, :, N - 1], None, qz, N, oracle.NVFP4, 0.2, oracle.PREORDER, 32,
                        num_splits=splits, variant=oracle.VAR_NO_PQUANT | oracle.VAR_EXACT)
    vd = np.swapaxes(deq["vt"], -1, -2)
    for b, hq in itertools.product(range(B), range(Hq)):
        h = hq // (Hq // Hkv)
        sc = qd[b, hq, 0] @ deq["k"][b, h, :N].T * 0.2
        p = np.exp(sc - sc.max())
        ref = p @ vd[b, h, :N] / p.sum()
        np.testing.assert_allclose(res["O"][b, hq], ref, rtol=1e-12, atol=1e-13)


# ------------------------------------------------------- lazy rescaling ---
# The running max may be updated lazily (the conditional rescaling of
# FlashAttention-4): it moves to a tile's max x_t only when x_t exceeds
# fl32(m + tau).  Pins: a loop-only second implementation bit for bit, exact
# softmax attention when quantization is off (the stale max cancels), the
# P-Reordering two-pass identity, and the rule's own invariants on the dumps.

LAZY_CASES = [
    # (fmt, N, d, BN, causal, G, mode, tau)
    (oracle.NVFP4, 64, 16, 16, True, 1, oracle.PREORDER, 3.0),
    (oracle.NVFP4, 48, 32, 16, False, 2, oracle.INCONSISTENT, 1.5),
    (oracle.MXFP4, 64, 32, 32, True, 2, oracle.PREORDER, 8.0),
    (oracle.MXFP4, 40, 32, 32, False, 1, oracle.INCONSISTENT, 2.0),
]


@pytest.mark.parametrize("fmt,N,d,BN,causal,G,mode,tau", LAZY_CASES)
def test_lazy_rescale_equals_bruteforce(fmt, N, d, BN, causal, G, mode, tau):
    q, k, v = _inputs(1, G, 1, N, d, 80 + N + d)
    s, inv = oracle.calibrate(q, k, n_cal=8, alpha=0.5)
    qz = oracle.quantize_qkv(q, k, v, s, inv, fmt)
    scale = 2.5 / np.sqrt(d)            # wide scores: the max both moves and stays stale
    ours = oracle.attention(qz, N, fmt, scale, causal, mode, BN, tau=tau)
    O, lph, lp = bruteforce.attention(qz, N, fmt, scale, causal, mode, BN, tau=tau)
    np.testing.assert_allclose(ours["O"], O, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(ours["l_phat"], lph, rtol=1e-13)
    np.testing.assert_allclose(ours["l_p"], lp, rtol=1e-13)
    # the lazy path changed the result (it is exercised by this input)
    exact = oracle.attention(qz, N, fmt, scale, causal, mode, BN)
    assert not np.array_equal(exact["O"], ours["O"])


@pytest.mark.parametrize("tau", [0.5, 3.0, 8.0])
@pytest.mark.parametrize("causal,BN", [(True, 16), (False, 32)])
def test_lazy_rescale_quant_off_is_textbook_softmax(tau, causal, BN):
    """Without quantization a stale max cancels between O and l: exact
    softmax attention for any threshold, both normalizers."""
    N, d, G = 72, 32, 2
    q, k, v = _inputs(1, 2 * G, 2, N, d, 90 + BN)
    qz = oracle.quantize_qkv(q, k, v, None, None, oracle.NVFP4)
    deq = _dequant_all(qz, oracle.NVFP4)
    scale = 0.6
    ref = _textbook(deq["q"], deq["k"], np.swapaxes(deq["vt"], -1, -2), N, scale, causal, G)
    for mode in (oracle.PREORDER, oracle.INCONSISTENT):
        res = oracle.attention(qz, N, oracle.NVFP4, scale, causal, mode, BN,
                               variant=oracle.VAR_NO_PQUANT | oracle.VAR_EXACT, tau=tau)
        np.testing.assert_allclose(res["O"], ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("fmt,tau", [(oracle.NVFP4, 3.0), (oracle.MXFP4, 6.0)])
def test_lazy_rescale_rule_and_two_pass_identity(fmt, tau):
    """On the dumps: m moves only to a tile max above fl32(m + tau) and never
    down; P-hat reaches above 1 under a stale max (but not past the bound
    2^tau rounded up to the grid); and O is the P-Reordering two-pass sum
    over the per-tile P-hat weighted by 2^(m_j - m_final)."""
    N, d, G = 128, 32, 2
    BN = 2 * oracle.beta_of(fmt)
    q, k, v = _inputs(1, G, 1, N, d, 95)
    s, inv = oracle.calibrate(q, k, n_cal=16)
    qz = oracle.quantize_qkv(q, k, v, s, inv, fmt)
    scale = 2.0 / np.sqrt(d)
    res = oracle.attention(qz, N, fmt, scale, True, oracle.PREORDER, BN, dump_phat=True, tau=tau)
    beta = oracle.beta_of(fmt)
    g = 2.0 ** oracle.P_PRESCALE_LOG2 if fmt == oracle.NVFP4 else 1.0
    vd = np.swapaxes(_dequant_all(qz, fmt)["vt"], -1, -2)[0, 0]
    stale = above_one = 0
    for hq in range(G):
        for i in range(N):
            ntl = i // BN + 1
            m = res["m_tiles"][0, hq, i, :ntl]
            assert np.all(np.diff(m) >= 0)
            for j in range(1, ntl):
                if m[j] != m[j - 1]:
                    assert m[j] > np.float32(np.float32(m[j - 1]) + np.float32(tau))
            codes = res["phat_codes"][0, hq, i, :ntl * BN]
            sc = res["phat_sc"][0, hq, i, :ntl * BN // beta]
            if fmt == oracle.NVFP4:
                sd = (oracle.ue4m3_decode(sc) * g).astype(np.float32).astype(np.float64)
            else:
                sd = 2.0 ** (sc.astype(np.float64) - 127)
            phat = GRID[codes & 7] * np.repeat(sd, beta)
            # P <= 2^tau, and P-hat rounds a block's max by at most its scale step
            assert phat.max() <= 2.0 ** tau * (1.125 if fmt == oracle.NVFP4 else 1.5)
            above_one += int(phat.max() > 1.0)
            stale += int(np.any(np.diff(m) == 0))
            w = np.repeat(2.0 ** (m - m[-1]), BN)
            num = (w * phat) @ vd[:ntl * BN]
            den = np.sum(w * phat)
            np.testing.assert_allclose(res["O"][0, hq, i], num / den, rtol=1e-12, atol=1e-14)
    assert stale > 0 and above_one > 0


@pytest.mark.parametrize("fmt", [oracle.NVFP4, oracle.MXFP4])
def test_lazy_rescale_zero_threshold_is_exact_recurrence(fmt):
    """tau = 0 moves the max whenever it rises: the exact recurrence."""
    N, d = 96, 32
    q, k, v = _inputs(1, 2, 1, N, d, 97)
    qz = oracle.quantize_qkv(q, k, v, None, None, fmt)
    a = oracle.attention(qz, N, fmt, 0.4, True, oracle.PREORDER, 32, dump_phat=True)
    b = oracle.attention(qz, N, fmt, 0.4, True, oracle.PREORDER, 32, dump_phat=True, tau=0.0)
    np.testing.assert_array_equal(a["O"], b["O"])
    # and that recurrence's max is the running maximum of the tile maxima
    m = a["m_tiles"][0, 0, N - 1]
    assert np.all(np.diff(m) >= 0) and np.all(np.isfinite(m))


@pytest.mark.parametrize("splits", [1, 3])
def test_lazy_decode_split_combine_exact_when_quant_off(splits):
    B, Hq, Hkv, N, d = 1, 4, 2, 300, 32
    q, k, v = _inputs(B, Hq, Hkv, N, d, 71)
    qz = oracle.quantize_qkv(q, k, v, None, None, oracle.NVFP4)
    deq = _dequant_all(qz, oracle.NVFP4)
    qq = oracle.quantize_qkv(q[:, :, N - 1:N], k[:, :, :1], v[:, :, :1], None, None, oracle.NVFP4)
    qd = _dequant_all(qq, oracle.NVFP4)["q"][:, :, :1]
    res = oracle.decode(q[:, :, N - 1], None, qz, N, oracle.NVFP4, 0.5, oracle.PREORDER, 32,
                        num_splits=splits, variant=oracle.VAR_NO_PQUANT | oracle.VAR_EXACT, tau=3.0)
    vd = np.swapaxes(deq["vt"], -1, -2)
    for b, hq in itertools.product(range(B), range(Hq)):
        h = hq // (Hq // Hkv)
        sc = qd[b, hq, 0] @ deq["k"][b, h, :N].T * 0.5
        p = np.exp(sc - sc.max())
        np.testing.assert_allclose(res["O"][b, hq], p @ vd[b, h, :N] / p.sum(), rtol=1e-12, atol=1e-13)


def test_lazy_rescale_threshold_is_strict_and_fp32():
    """The rule on crafted scores: with NVFP4-exact Q and K (a single 6 in
    each Q row, a single 3 or 6 in a key row) and c = 1, tile 0's max is 18
    and tile 1's is 36.  tau = 18 keeps the max (36 > fl32(18 + 18) is
    false: the comparison is strict); tau = 17.9995 moves it (fl32(18 +
    17.9995) < 36); tau = 0 moves it."""
    N, d, BN = 32, 16, 16
    q = np.zeros((1, 1, N, d), np.float32)
    q[..., 0] = 6.0
    k = np.zeros((1, 1, N, d), np.float32)
    k[0, 0, 0, 0] = 3.0          # tile 0: score 18
    k[0, 0, 16, 0] = 6.0         # tile 1: score 36
    v = np.random.default_rng(3).standard_normal((1, 1, N, d)).astype(np.float32)
    qz = oracle.quantize_qkv(q, k, v, None, None, oracle.NVFP4)
    deq = _dequant_all(qz, oracle.NVFP4)
    assert deq["q"][0, 0, 0, 0] == 6.0 and deq["k"][0, 0, 0, 0] == 3.0 and deq["k"][0, 0, 16, 0] == 6.0
    scale = 1.0 / 1.4426950408889634          # c = scale * log2(e) = 1 up to fp64 rounding
    for tau, moved in ((18.0, False), (17.9995, True), (0.0, True)):
        res = oracle.attention(qz, N, oracle.NVFP4, scale, False, oracle.PREORDER, BN, dump_phat=True, tau=tau)
        m = res["m_tiles"][0, 0, 5]
        assert m[0] == 18.0 and m[1] == (36.0 if moved else 18.0), (tau, m)


def test_lazy_decode_single_split_equals_last_causal_row():
    """With one split, decode under the lazy rule is the last causal prefill
    row under the same rule, exactly (the rule is per row and per tile)."""
    B, Hq, Hkv, N, d = 1, 4, 2, 200, 64
    q, k, v = _inputs(B, Hq, Hkv, N, d, 61)
    s, inv = oracle.calibrate(q, k, n_cal=32)
    qz = oracle.quantize_qkv(q, k, v, s, inv, oracle.NVFP4)
    for tau in (1.0, 3.0):
        pre = oracle.attention(qz, N, oracle.NVFP4, 0.5, True, oracle.PREORDER, 64, rows=(N - 1, N), tau=tau)
        dec = oracle.decode(q[:, :, N - 1], s, qz, N, oracle.NVFP4, 0.5, oracle.PREORDER, 64, num_splits=1, tau=tau)
        np.testing.assert_array_equal(dec["O"], pre["O"][:, :, N - 1])


# ---------------------------------------------------------- per-tile epsilon ---
# The pages report the normalizer error per attention tile ("all 3.6M measured
# attention tiles exhibit net probability-mass loss", the arXiv announcement
# abstract) without defining it.  The reading: over the 128 query rows x BN
# keys of a tile, sum(P-hat) / sum(P) - 1, each row's terms taken against its
# running max at that tile (the same P and P-hat that enter l_phat and l_p).


@pytest.mark.parametrize("fmt,N,d,BN,causal,G,mode", CASES[:4] + CASES[5:])
def test_tile_sums_equal_bruteforce(fmt, N, d, BN, causal, G, mode):
    q, k, v = _inputs(1, G, 1, N, d, 20 + N + d)
    s, inv = oracle.calibrate(q, k, n_cal=8, alpha=0.5)
    qz = oracle.quantize_qkv(q, k, v, s, inv, fmt)
    scale = 1 / np.sqrt(d)
    ours = oracle.attention(qz, N, fmt, scale, causal, mode, BN, dump_phat=True)
    _, _, _, ts = bruteforce.attention(qz, N, fmt, scale, causal, mode, BN, tile_sums=True)
    np.testing.assert_allclose(ours["tile_sum_phat"], ts[..., 0], rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(ours["tile_sum_p"], ts[..., 1], rtol=1e-13, atol=1e-300)


@pytest.mark.parametrize("fmt,BN,tau", [(oracle.NVFP4, 16, 0.0), (oracle.MXFP4, 32, 0.0), (oracle.NVFP4, 32, 3.0)])
def test_tile_sums_rebuild_the_normalizers(fmt, BN, tau):
    """Both normalizers are the per-tile sums carried to the final max:
    l = sum_j 2^(m_j - m_last) sum_tile_j, for l_phat and l_p alike."""
    N, d, G = 150, 32, 2
    q, k, v = _inputs(1, G, 1, N, d, 70 + BN)
    s, inv = oracle.calibrate(q, k, n_cal=16)
    qz = oracle.quantize_qkv(q, k, v, s, inv, fmt)
    res = oracle.attention(qz, N, fmt, 1 / np.sqrt(d), True, oracle.PREORDER, BN, dump_phat=True, tau=tau)
    for hq in range(G):
        for i in (0, 31, 32, 100, 149):
            ntl = i // BN + 1
            m = res["m_tiles"][0, hq, i, :ntl]
            w = 2.0 ** (m - m[-1])
            np.testing.assert_allclose(np.sum(w * res["tile_sum_phat"][0, hq, i, :ntl]), res["l_phat"][0, hq, i],
                                       rtol=1e-12)
            np.testing.assert_allclose(np.sum(w * res["tile_sum_p"][0, hq, i, :ntl]), res["l_p"][0, hq, i],
                                       rtol=1e-12)
            assert np.all(np.isnan(res["tile_sum_p"][0, hq, i, ntl:]))


def test_tile_epsilon_zero_without_p_quantizer_and_negative_with_it():
    """With P-hat = P every tile's error is exactly 0; with the quantizer the
    typical tile loses probability mass (the sign of the pages' finding)."""
    N, d, G = 384, 64, 2
    q, k, v = _inputs(1, G, 1, N, d, 80)
    s, inv = oracle.calibrate(q, k, n_cal=64)
    qz = oracle.quantize_qkv(q, k, v, s, inv, oracle.NVFP4)
    off = oracle.attention(qz, N, oracle.NVFP4, 1 / np.sqrt(d), True, oracle.PREORDER, 64, dump_phat=True,
                           variant=oracle.VAR_NO_PQUANT)
    e_off = oracle.tile_epsilon(off["tile_sum_phat"], off["tile_sum_p"])
    fin = np.isfinite(e_off)
    # causal, 3 query tiles of 128 rows x 64-key tiles: 2 + 4 + 6 visited tiles per head
    assert fin.sum() == G * (2 + 4 + 6)
    assert np.all(e_off[fin] == 0.0)
    on = oracle.attention(qz, N, oracle.NVFP4, 1 / np.sqrt(d), True, oracle.PREORDER, 64, dump_phat=True)
    e_on = oracle.tile_epsilon(on["tile_sum_phat"], on["tile_sum_p"])
    assert np.array_equal(np.isfinite(e_on), fin)
    assert np.median(e_on[fin]) < 0


def test_tile_epsilon_aggregation_by_hand():
    """tile_epsilon sums 128-row groups of the per-row terms; checked on a
    hand-made array with a ragged last group and an empty tile."""
    sph = np.zeros((1, 1, 130, 2))
    sp = np.zeros((1, 1, 130, 2))
    sph[0, 0, :128, 0], sp[0, 0, :128, 0] = 0.5, 1.0          # tile (0, 0): 64 / 128 - 1
    sph[0, 0, 128:, 0], sp[0, 0, 128:, 0] = 3.0, 2.0          # tile (1, 0): 6 / 4 - 1
    sph[0, 0, 5, 1], sp[0, 0, 5, 1] = np.nan, np.nan          # tile (0, 1): not computed -> empty
    sph[0, 0, 129, 1], sp[0, 0, 129, 1] = 1.0, 4.0            # tile (1, 1): 1 / 4 - 1
    e = oracle.tile_epsilon(sph, sp)
    assert e.shape == (1, 1, 2, 2)
    assert e[0, 0, 0, 0] == -0.5 and e[0, 0, 1, 0] == 0.5 and e[0, 0, 1, 1] == -0.75
    assert np.isnan(e[0, 0, 0, 1])


def test_raw_operand_ablation_is_textbook_attention():
    """The test-only raw operands replace the dequantized Q, K and V: with all
    three raw, the P quantizer off and fp64 scores, the oracle is textbook
    softmax attention of the raw tensors (pins the raw layouts and GQA map)."""
    B, G, Hkv, N, d = 2, 2, 2, 90, 32
    q, k, v = _inputs(B, G * Hkv, Hkv, N, d, 90)
    qz = oracle.quantize_qkv(q, k, v, None, None, oracle.NVFP4)
    res = oracle.attention(qz, N, oracle.NVFP4, 0.2, True, oracle.PREORDER, 32,
                           variant=oracle.VAR_NO_PQUANT | oracle.VAR_EXACT, raw=dict(q=q, k=k, v=v))
    ref = _textbook(q.astype(np.float64), k.astype(np.float64), v.astype(np.float64), N, 0.2, True, G)
    np.testing.assert_allclose(res["O"], ref, rtol=1e-12, atol=1e-13)
    # one raw operand at a time changes the result (each is really used)
    base = oracle.attention(qz, N, oracle.NVFP4, 0.2, True, oracle.PREORDER, 32)["O"]
    for name, arr in (("q", q), ("k", k), ("v", v)):
        o = oracle.attention(qz, N, oracle.NVFP4, 0.2, True, oracle.PREORDER, 32, raw={name: arr})["O"]
        assert not np.allclose(o, base, rtol=1e-6, atol=0), name
