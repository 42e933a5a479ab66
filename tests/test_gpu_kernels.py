"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Codes and scales must match bit for bit; outputs must satisfy
|dO| <= 1e-2 max|O| + 1e-3 elementwise and cosine >= 0.9999."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

h = None


@pytest.fixture(scope="module", autouse=True)
def _lib():
    global h
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_quantized_flashattention_smooth_b200 as mod
    mod.lib()
    h = mod
    yield
    assert h.device_error() == 0, "a kernel gave up a bounded wait"


# ------------------------------------------------------------ conversions ---
def _sweep():
    rng = np.random.default_rng(0)
    vals = []
    for e in range(-14, 10):
        m = rng.integers(0, 1 << 23, 20000, dtype=np.int64)
        vals.append((((e + 127) << 23) | m).astype(np.uint32).view(np.float32))
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    e4 = oracle.ue4m3_decode(np.arange(127)).astype(np.float32)
    e4m = ((e4[:-1].astype(np.float64) + e4[1:]) / 2).astype(np.float32)
    base = np.concatenate(vals + [grid, mids, e4, e4m, np.array([0, 447, 448, 464, 500, 1e30, 2.0 ** -10], np.float32)])
    nb = np.concatenate([base, np.nextafter(base, np.float32(np.inf)), np.nextafter(base, np.float32(0))])
    return np.concatenate([nb, -nb]).astype(np.float32)


def test_hw_conversions_match_written_rounding():
    x = _sweep()
    e2_gpu, e4_gpu = h.convert_probe(torch.from_numpy(x).cuda())
    e2_ref, e4_ref = oracle.encode_array(x)
    e2_gpu = U.to_np(e2_gpu).astype(np.uint8)
    bad = np.nonzero(e2_gpu != e2_ref)[0]
    assert bad.size == 0, f"E2M1: {bad.size} mismatches e.g. x={x[bad[:8]]} gpu={e2_gpu[bad[:8]]} ref={e2_ref[bad[:8]]}"
    pos = ~np.signbit(x)   # scales are encoded from |amax| >= +0
    e4_gpu = U.to_np(e4_gpu).astype(np.uint8)
    bad = np.nonzero((e4_gpu != e4_ref) & pos)[0]
    assert bad.size == 0, f"E4M3: {bad.size} mismatches e.g. x={x[bad[:8]]} gpu={e4_gpu[bad[:8]]} ref={e4_ref[bad[:8]]}"


def test_hw_conversions_exhaustive():
    """Every finite fp32 bit pattern, in 16 chunks of 2^28: the E2M1
    conversion the kernels use equals the oracle's written encoder, and the
    UE4M3 scale conversion equals it on every non-negative finite value (NaN
    and infinities are outside the encoders' domain)."""
    chunk = 1 << 28
    for start in range(0, 1 << 32, chunk):
        s0 = start if start < (1 << 31) else start - (1 << 32)     # the same bits as int32
        x = torch.arange(s0, s0 + chunk, dtype=torch.int32, device="cuda").view(torch.float32)
        e2_gpu, e4_gpu = h.convert_probe(x)
        e2_gpu = e2_gpu.cpu().numpy()
        e4_gpu = e4_gpu.cpu().numpy()
        del x
        xn = np.arange(start, start + chunk, dtype=np.uint64).astype(np.uint32).view(np.float32)
        e2_ref, e4_ref = oracle.encode_array(xn)
        fin = np.isfinite(xn)
        bad = np.nonzero((e2_gpu != e2_ref) & fin)[0]
        assert bad.size == 0, (f"E2M1: {bad.size} mismatches in chunk {start:#x}, e.g. bits "
                               f"{xn[bad[:4]].view(np.uint32)} gpu={e2_gpu[bad[:4]]} ref={e2_ref[bad[:4]]}")
        pos = fin & ~np.signbit(xn)
        bad = np.nonzero((e4_gpu != e4_ref) & pos)[0]
        assert bad.size == 0, (f"UE4M3: {bad.size} mismatches in chunk {start:#x}, e.g. bits "
                               f"{xn[bad[:4]].view(np.uint32)} gpu={e4_gpu[bad[:4]]} ref={e4_ref[bad[:4]]}")


def test_fast_div6_is_ieee_division():
    """The P-hat scale path computes fl32(amax/6) without a division; it must
    equal IEEE division for zero and every float in [2^-122, 2^20] (quotients
    that are normal), and the variant with g_P = 2^-8 folded into its
    constants must equal 2^8 times that quotient over the same range.  Below
    2^-122 the scale code is 0 either way: the
    quotient times 2^8 is under 2^-116, far below half the smallest UE4M3
    subnormal."""
    n, first = h.div6_probe(0x02800000, 0x49800000)
    assert n == 0, f"{n} mismatches, first at bits {first:#x}"
    n0, _ = h.div6_probe(0, 1)
    assert n0 == 0


def test_exp2_polynomial_error_bound():
    """The FMA-pipe 2^y: relative error within the fitted bound (2.9e-6 in
    fp32 Horner form, checked here against fp64 with a 4e-6 margin) over the
    whole range a probability can take, exactly 1 at y = 0, exactly 0 from
    y = -127 down (and for -inf, the masked score), and below 2^-126 no value
    larger than 2^-126."""
    g = torch.Generator().manual_seed(7)
    y = torch.cat([-126.0 * torch.rand(1 << 20, generator=g), -torch.rand(1 << 16, generator=g),
                   torch.tensor([0.0, -0.5, -1.0, -126.0, -126.49, -126.51, -127.0, -130.0, -1e30, -float("inf")])])
    out = U.to_np(h.exp2_poly_probe(y.cuda())).astype(np.float64)
    yd = y.double().numpy()
    ref = np.exp2(yd)
    sel = yd >= -126.0
    rel = np.abs(out[sel] / ref[sel] - 1.0)
    assert rel.max() < 4e-6, f"max rel err {rel.max():.3e} at y={yd[sel][rel.argmax()]}"
    assert out[yd == 0.0].tolist() == [1.0]
    assert np.all(out[yd <= -127.0] == 0.0)
    assert np.all(out[yd < -126.0] < 2.0 ** -126) and np.all(out >= 0.0)


def test_exponential_free_code_decisions():
    """The exponential-free P-hat code argument takes every E2M1 decision
    that the written encoder takes on fl32(2^y): over a dense sweep of
    log2-domain values, at y = -2 (the 0.25 tie, code 0), for -inf, and
    near each rounding edge y* = log2(midpoint) it may differ only within
    1e-6 of y* (the MUFU 2^y has the same kind of window)."""
    g = torch.Generator().manual_seed(9)
    mids = np.log2(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]))
    near = (mids[:, None] + np.linspace(-2e-5, 2e-5, 4001)[None, :]).ravel()
    y = torch.cat([torch.rand(1 << 21, generator=g) * 13.5 - 10.0, torch.from_numpy(near).float(),
                   torch.tensor([-2.0, -1.0, 0.0, 1.0, 2.0, 3.0, 3.5, -8.0, -9.5, -1e30, -float("inf")])])
    cm, ce = h.e2m1_map_probe(y.cuda())
    cm, ce = U.to_np(cm).astype(np.uint8), U.to_np(ce).astype(np.uint8)
    yd = y.double().numpy()
    ref, _ = oracle.encode_array(np.exp2(yd).astype(np.float32))
    window = np.min(np.abs(yd[:, None] - mids[None, :]), axis=1) < 1e-6
    bad = (cm != ref) & ~window
    assert not bad.any(), f"{bad.sum()} code mismatches, first at y={yd[bad][0]!r}"
    assert np.all(cm[yd == -2.0] == 0) and np.all(cm[np.isneginf(yd)] == 0)
    # inside the windows both device paths stay within a few decisions
    assert np.sum(cm != ref) <= np.sum(ce != ref) + 64, (np.sum(cm != ref), np.sum(ce != ref))


def test_bounded_wait_gives_up_and_reports():
    """A wait that nothing completes ends after its limit with the abort flag
    and the timeout bit set, the kernel returns, and the context stays usable
    (no trap, no hang)."""
    assert h.device_error() == 0
    ok, flag = h.wait_timeout_probe()
    assert not ok and flag == 1
    assert h.device_error() & 8           # read and cleared
    assert h.device_error() == 0
    n, _ = h.div6_probe(0x3F800000, 0x3F801000)
    assert n == 0


# --------------------------------------------------------------- FP4 MMA ---
@pytest.mark.parametrize("fmt", [oracle.NVFP4, oracle.MXFP4])
@pytest.mark.parametrize("n,k", [(128, 128), (64, 128), (256, 256), (128, 256)])
def test_fp4_mma_tile_layouts(fmt, n, k):
    rng = np.random.default_rng(n + k + fmt)
    beta = oracle.beta_of(fmt)
    ac = rng.integers(0, 256, (128, k // 2), dtype=np.uint8)
    bc = rng.integers(0, 256, (n, k // 2), dtype=np.uint8)
    lo, hi = (0x28, 0x48) if fmt == oracle.NVFP4 else (120, 134)
    asc = rng.integers(lo, hi, (128, k // beta), dtype=np.uint8)
    bsc = rng.integers(lo, hi, (n, k // beta), dtype=np.uint8)
    A = oracle.dequantize_rows(ac, asc, fmt)
    Bm = oracle.dequantize_rows(bc, bsc, fmt)
    ref = A @ Bm.T
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    d = h.fp4_mma_probe(dev(ac), dev(oracle.sf_tile(asc)), dev(bc), dev(oracle.sf_tile(bsc)), n, k, fmt, 1, 1)
    got = U.to_np(d)
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-5 * np.abs(ref).max())
    d3 = h.fp4_mma_probe(dev(ac), dev(oracle.sf_tile(asc)), dev(bc), dev(oracle.sf_tile(bsc)), n, k, fmt, 3, 2)
    np.testing.assert_allclose(U.to_np(d3), 3 * ref, rtol=1e-5, atol=3e-5 * np.abs(ref).max())


# ---------------------------------------------------- calibrate + quantize ---
QUANT_CASES = [
    # B, Hq, Hkv, N, d, fmt, dtype
    (1, 2, 2, 256, 64, oracle.NVFP4, torch.float16),
    (1, 4, 2, 200, 128, oracle.NVFP4, torch.bfloat16),
    (2, 4, 1, 130, 256, oracle.MXFP4, torch.bfloat16),
    (1, 8, 2, 300, 64, oracle.MXFP4, torch.float16),
    (1, 2, 2, 1, 128, oracle.NVFP4, torch.bfloat16),
    (1, 4, 4, 520, 256, oracle.NVFP4, torch.bfloat16),
    (2, 4, 2, 333, 128, oracle.MXFP4, torch.float16),
    (3, 2, 1, 77, 64, oracle.NVFP4, torch.bfloat16),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,fmt,dtype", QUANT_CASES)
def test_calibrate_and_quantize_bit_exact(B, Hq, Hkv, N, d, fmt, dtype):
    q, k, v = U.synthetic(B, Hq, Hkv, N, d, seed=N + d, dtype=dtype)
    n_cal = min(N, 64)
    s_ref, inv_ref = oracle.calibrate(q.float().numpy(), k.float().numpy(), n_cal=n_cal, alpha=0.5)
    s, inv = h.calibrate_smooth_qk(q.cuda(), k.cuda(), n_cal=n_cal, alpha=0.5)
    s_g, inv_g = U.to_np(s), U.to_np(inv)
    np.testing.assert_allclose(s_g, s_ref, rtol=2 ** -22)
    # quantize with the oracle's scales on both sides, then compare bytes
    z = h.quantize_qkv(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(s_ref).cuda(),
                       torch.from_numpy(inv_ref).cuda(), fmt)
    qz, tiled = U.oracle_quantize(q, k, v, s_ref, inv_ref, fmt)
    for name in ("q_codes", "k_codes", "vt_codes"):
        g = U.to_np(getattr(z, name)).astype(np.uint8)
        assert np.array_equal(g, qz[name]), (name, int(np.sum(g != qz[name])))
    for name in ("q_sc", "k_sc", "vt_sc"):
        g = U.to_np(getattr(z, name.replace("_sc", "_scales"))).astype(np.uint8)
        assert np.array_equal(g, tiled[name]), (name, int(np.sum(g != tiled[name])))


def test_calibration_gate_matches_oracle():
    """The per-head applicability gate: the GPU decision and scales equal the
    oracle's for heads with and without K outliers."""
    B, Hq, Hkv, N, d = 1, 8, 4, 128, 128
    q, k, v = U.synthetic(B, Hq, Hkv, N, d, seed=17, dtype=torch.bfloat16, outlier=0.0)
    k = k.clone()
    k[:, 1, :, 5] *= 30       # head 1: one strong outlier channel
    k[:, 3, :, 77] *= 12
    for alpha in (0.5, 0.25):
        s_ref, inv_ref = oracle.calibrate(q.float().numpy(), k.float().numpy(), n_cal=64, alpha=alpha,
                                          enable=oracle.GATE)
        s, inv = h.calibrate_smooth_qk(q.cuda(), k.cuda(), n_cal=64, alpha=alpha, enable=h.GATE)
        np.testing.assert_allclose(U.to_np(s), s_ref, rtol=2 ** -22)
        np.testing.assert_allclose(U.to_np(inv), inv_ref, rtol=2 ** -22)
        on = [not np.all(s_ref[hh] == 1.0) for hh in range(Hkv)]
        assert on[1] and on[3] and not on[0] and not on[2], on


# -------------------------------------------------------------- attention ---
ATTN_CASES = [
    # B, Hq, Hkv, N, d, causal, BN, fmt, mode, dtype
    (1, 2, 2, 256, 64, False, 64, oracle.NVFP4, oracle.PREORDER, torch.float16),
    (1, 2, 2, 256, 64, False, 64, oracle.NVFP4, oracle.INCONSISTENT, torch.float16),
    (1, 4, 1, 200, 128, True, 128, oracle.NVFP4, oracle.PREORDER, torch.bfloat16),
    (1, 4, 2, 384, 128, True, 64, oracle.MXFP4, oracle.PREORDER, torch.bfloat16),
    (1, 2, 2, 300, 64, False, 128, oracle.MXFP4, oracle.INCONSISTENT, torch.bfloat16),
    (1, 4, 2, 130, 256, True, 128, oracle.NVFP4, oracle.INCONSISTENT, torch.bfloat16),
    (2, 2, 1, 257, 256, False, 128, oracle.MXFP4, oracle.PREORDER, torch.bfloat16),
    (1, 2, 2, 1, 128, True, 128, oracle.NVFP4, oracle.PREORDER, torch.bfloat16),
    (1, 8, 2, 512, 128, True, 128, oracle.NVFP4, oracle.PREORDER, torch.bfloat16),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,BN,fmt,mode,dtype", ATTN_CASES)
def test_attention_matches_oracle(B, Hq, Hkv, N, d, causal, BN, fmt, mode, dtype):
    q, k, v = U.synthetic(B, Hq, Hkv, N, d, seed=7 * N + d, dtype=dtype)
    s_ref, inv_ref = oracle.calibrate(q.float().numpy(), k.float().numpy(), n_cal=min(N, 64))
    z = h.quantize_qkv(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(s_ref).cuda(),
                       torch.from_numpy(inv_ref).cuda(), fmt)
    qz, _ = U.oracle_quantize(q, k, v, s_ref, inv_ref, fmt)
    scale = 1.0 / math.sqrt(d)
    ref = oracle.attention(qz, N, fmt, scale, causal, mode, BN)
    o, lse, lph, lp = h.attn_fwd(z, scale, causal, mode, BN, out_dtype=dtype, return_lse=True, debug=True)
    ok, err, bound, cos = U.compare_out(U.to_np(o), ref["O"])
    assert ok, f"max|dO|={err:.3e} bound={bound:.3e} cos={cos:.6f}"
    np.testing.assert_allclose(U.to_np(lse), ref["lse"], rtol=1e-3, atol=1e-2)
    np.testing.assert_allclose(U.to_np(lph), ref["l_phat"], rtol=2e-2)
    np.testing.assert_allclose(U.to_np(lp), ref["l_p"], rtol=2e-3)


def test_theorem1_coherence_on_gpu():
    """Inconsistent vs P-Reordering outputs differ by one scale per row, equal
    to l_phat / l_p, with net probability-mass loss (eps < 0)."""
    B, Hq, Hkv, N, d = 1, 4, 2, 512, 128
    q, k, v = U.synthetic(B, Hq, Hkv, N, d, seed=99)
    z = h.quantize_qkv(q.cuda(), k.cuda(), v.cuda(), None, None, oracle.NVFP4)
    o_r, lph, lp = h.attn_fwd(z, None, True, oracle.PREORDER, 128, out_dtype=torch.float16, debug=True)
    o_i = h.attn_fwd(z, None, True, oracle.INCONSISTENT, 128, out_dtype=torch.float16)
    o_r, o_i = U.to_np(o_r).astype(np.float64), U.to_np(o_i).astype(np.float64)
    ratio = U.to_np(lph) / U.to_np(lp)
    pred = o_r * ratio[..., None]
    assert np.max(np.abs(o_i - pred)) <= 2e-3 * np.max(np.abs(o_r)) + 1e-3
    eps = ratio - 1
    assert np.median(eps) < 0


# ----------------------------------------------------------------- decode ---
DECODE_CASES = [
    # B, Hq, Hkv, kv_len, fmt, mode, splits, q dtype
    (2, 8, 2, 1000, oracle.NVFP4, oracle.PREORDER, 3, torch.bfloat16),
    (2, 8, 2, 1000, oracle.NVFP4, oracle.INCONSISTENT, 1, torch.bfloat16),
    (1, 8, 1, 777, oracle.MXFP4, oracle.PREORDER, 4, torch.float16),
    (3, 4, 2, 2048, oracle.MXFP4, oracle.INCONSISTENT, 0, torch.bfloat16),
    (1, 2, 2, 129, oracle.NVFP4, oracle.PREORDER, 2, torch.bfloat16),
]


@pytest.mark.parametrize("B,Hq,Hkv,kv,fmt,mode,splits,qdt", DECODE_CASES)
def test_decode_matches_oracle(B, Hq, Hkv, kv, fmt, mode, splits, qdt):
    d = 128
    _, k, v = U.synthetic(B, Hq, Hkv, kv, d, seed=kv + Hq, dtype=torch.bfloat16)
    g = np.random.Generator(np.random.PCG64(kv))
    q = torch.from_numpy(g.standard_normal((B, Hq, d), dtype=np.float32)).to(qdt)
    qcal = torch.from_numpy(g.standard_normal((B, Hq, 64, d), dtype=np.float32)).to(torch.bfloat16)
    s_ref, inv_ref = oracle.calibrate(qcal.float().numpy(), k[:, :, :64].float().numpy(), n_cal=64)
    cache = h.quantize_kv(k.cuda(), v.cuda(), torch.from_numpy(inv_ref).cuda(), fmt, Hq=Hq)
    # cache bytes equal the oracle's
    qz, tiled = U.oracle_quantize(torch.zeros((B, Hkv, kv, d)), k, v, np.ones_like(s_ref), inv_ref, fmt)
    assert np.array_equal(U.to_np(cache.k_codes).astype(np.uint8), qz["k_codes"])
    assert np.array_equal(U.to_np(cache.vt_codes).astype(np.uint8), qz["vt_codes"])
    assert np.array_equal(U.to_np(cache.k_scales).astype(np.uint8), tiled["k_sc"])
    assert np.array_equal(U.to_np(cache.vt_scales).astype(np.uint8), tiled["vt_sc"])
    o, used = h.attn_decode(q.cuda(), torch.from_numpy(s_ref).cuda(), cache, kv, 1 / math.sqrt(d), mode, splits,
                            out_dtype=torch.float32 if False else torch.bfloat16)
    ref = oracle.decode(q.float().numpy(), s_ref, qz, kv, fmt, 1 / math.sqrt(d), mode, 128, num_splits=used)
    ok, err, bound, cos = U.compare_out(U.to_np(o), ref["O"])
    assert ok, f"splits={used} max|dO|={err:.3e} bound={bound:.3e} cos={cos:.6f}"
