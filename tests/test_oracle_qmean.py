"""Pins of the oracle's Q-Mean auxiliary (no GPU).

The pages name "the adopted Q-Mean auxiliary" ("HiFA4: Training-Free 4-bit
FlashAttention on Ascend HIF4 NPUs for LLM Inference", Abstract para 3) and
nothing more.  The reading built here: subtract the per-channel calibration
mean mu of the smoothed query before it is quantized, and give every score
back the rank-one term mu . k of its key.  What pins it:
- the mean itself: a closed form (constant channels) and a brute-force mean;
- mu = 0 changes nothing, bit for bit;
- without quantization the scores are unchanged, (q - mu) . k + mu . k = q . k:
  the recurrence in fp64 gives textbook attention either way (a dropped bias,
  a wrong sign or a bias from the wrong head fails this);
- on a query with channel offsets the 4-bit Q-hat with the mean removed is
  closer to the smoothed query than without.
"""
import numpy as np

import oracle


def _rng(seed=0):
    return np.random.default_rng(seed)


def test_q_mean_closed_form_and_brute_force():
    rng = _rng(1)
    B, Hq, Hkv, T, d, n_cal = 2, 4, 2, 96, 64, 48
    q = rng.standard_normal((B, Hq, T, d)).astype(np.float32)
    s = rng.uniform(0.25, 4.0, (Hkv, d)).astype(np.float32)
    # channel 5 of every head constant 3 over the calibration tokens: mu = fl32(3 * s)
    q[:, :, :n_cal, 5] = 3.0
    mu = oracle.calibrate_q_mean(q, s, n_cal)
    G = Hq // Hkv
    for hq in range(Hq):
        assert mu[hq, 5] == np.float32(3.0) * s[hq // G, 5]
    # brute force: the fp64 mean of fl32(q * s) over (b, t < n_cal)
    qs = (q[:, :, :n_cal] * np.repeat(s, G, axis=0)[None, :, None, :]).astype(np.float32)
    ref = qs.astype(np.float64).mean(axis=(0, 2))
    np.testing.assert_allclose(mu, ref, rtol=2e-7, atol=1e-9)
    # without smoothing it is the plain channel mean
    mu1 = oracle.calibrate_q_mean(q, None, n_cal)
    np.testing.assert_allclose(mu1, q[:, :, :n_cal].astype(np.float64).mean(axis=(0, 2)), rtol=2e-7, atol=1e-9)


def _problem(seed=2, N=160, d=64, offset=0.0):
    rng = _rng(seed)
    B, Hq, Hkv = 1, 4, 2
    q = rng.standard_normal((B, Hq, N, d)).astype(np.float32)
    q[..., 3:9] += np.float32(offset)
    k = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    return q, k, v


def test_zero_mean_changes_nothing():
    q, k, v = _problem()
    s, inv = oracle.calibrate(q, k, 64)
    for fmt in (oracle.NVFP4, oracle.MXFP4):
        a = oracle.quantize_qkv(q, k, v, s, inv, fmt)
        b = oracle.quantize_qkv(q, k, v, s, inv, fmt, q_mu=np.zeros((4, 64), np.float32))
        for n in a:
            assert np.array_equal(a[n], b[n]), n
        oa = oracle.attention(a, 160, fmt, BN=64)["O"]
        ob = oracle.attention(b, 160, fmt, BN=64, q_mu=np.zeros((4, 64), np.float32))["O"]
        assert np.array_equal(oa, ob)


def test_scores_unchanged_without_quantization():
    """With P-hat = P, fp64 scores and raw operands, Q-Mean leaves attention
    as it is.  The query values are multiples of 1/16 and the calibration
    count a power of two, so mu and q - mu are exact in fp32 and the two runs
    differ only by fp64 rounding."""
    rng = _rng(3)
    B, Hq, Hkv, N, d, n_cal = 1, 4, 2, 192, 64, 64
    q = (np.round(rng.standard_normal((B, Hq, N, d)) * 16) / 16).astype(np.float32)
    q[..., 10:14] += 5.0
    k = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, N, d)).astype(np.float32)
    mu = oracle.calibrate_q_mean(q, None, n_cal)
    G = Hq // Hkv
    assert np.array_equal((q - mu[None, :, None, :]).astype(np.float64),
                          q.astype(np.float64) - mu[None, :, None, :].astype(np.float64))
    qz = oracle.quantize_qkv(q, k, v, None, None, oracle.NVFP4)
    var = oracle.VAR_NO_PQUANT | oracle.VAR_EXACT
    plain = oracle.attention(qz, N, oracle.NVFP4, BN=64, variant=var, raw=dict(q=q, k=k, v=v))["O"]
    qm = oracle.attention(qz, N, oracle.NVFP4, BN=64, variant=var,
                          raw=dict(q=q - mu[None, :, None, :], k=k, v=v), q_mu=mu)["O"]
    np.testing.assert_allclose(qm, plain, rtol=0, atol=1e-12)
    # and both are textbook softmax attention
    for hq in range(Hq):
        S = q[0, hq].astype(np.float64) @ k[0, hq // G].astype(np.float64).T / np.sqrt(d)
        S = np.where(np.tril(np.ones((N, N), bool)), S, -np.inf)
        P = np.exp(S - S.max(-1, keepdims=True))
        ref = (P / P.sum(-1, keepdims=True)) @ v[0, hq // G].astype(np.float64)
        np.testing.assert_allclose(qm[0, hq], ref, rtol=0, atol=1e-12)
    # dropping the term, or adding it with the wrong sign, moves the result
    off = oracle.attention(qz, N, oracle.NVFP4, BN=64, variant=var,
                           raw=dict(q=q - mu[None, :, None, :], k=k, v=v))["O"]
    neg = oracle.attention(qz, N, oracle.NVFP4, BN=64, variant=var,
                           raw=dict(q=q - mu[None, :, None, :], k=k, v=v), q_mu=-mu)["O"]
    assert np.abs(off - plain).max() > 1e-3 and np.abs(neg - plain).max() > 1e-3


def test_mean_removal_shrinks_the_query_quantization_error():
    q, k, v = _problem(seed=4, N=200, offset=6.0)
    s, inv = oracle.calibrate(q, k, 128)
    mu = oracle.calibrate_q_mean(q, s, 128)
    qs = q * np.repeat(s, 2, axis=0)[None, :, None, :]
    for fmt in (oracle.NVFP4, oracle.MXFP4):
        a = oracle.quantize_qkv(q, k, v, s, inv, fmt)
        b = oracle.quantize_qkv(q, k, v, s, inv, fmt, q_mu=mu)
        da = oracle.dequantize_rows(a["q_codes"], a["q_sc"], fmt)[:, :, :200]
        db = oracle.dequantize_rows(b["q_codes"], b["q_sc"], fmt)[:, :, :200] + mu[None, :, None, :]
        ea = np.linalg.norm(da - qs) / np.linalg.norm(qs)
        eb = np.linalg.norm(db - qs) / np.linalg.norm(qs)
        assert eb < 0.8 * ea, (fmt, ea, eb)
        # padding rows (200..255) stay zero codes
        assert not b["q_codes"][:, :, 200:].any() and not b["q_sc"][:, :, 200:].any()
