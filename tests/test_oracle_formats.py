"""Pins of the oracle's format layer against library routines, closed forms and
exhaustive enumeration (no GPU)."""
import math

import ml_dtypes
import numpy as np
import pytest

import oracle

GRID = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])


def _sweep_fp32(lo_exp, hi_exp, per_binade=4096, seed=0):
    """fp32 values spanning binades [2^lo, 2^hi): all midpoints of the E2M1
    and E4M3 grids +- 1 ulp, plus random mantissas in every binade."""
    rng = np.random.default_rng(seed)
    vals = []
    for e in range(lo_exp, hi_exp):
        m = rng.integers(0, 1 << 23, per_binade, dtype=np.int64)
        bits = ((e + 127) << 23) | m
        vals.append(bits.astype(np.uint32).view(np.float32))
    vals = np.concatenate(vals)
    return np.concatenate([vals, -vals])


def _neighbours(x):
    x = np.asarray(x, np.float32)
    return np.concatenate([x, np.nextafter(x, np.float32(np.inf)), np.nextafter(x, np.float32(-np.inf))])


def test_e2m1_against_ml_dtypes():
    mids = (GRID[:-1] + GRID[1:]) / 2
    x = np.concatenate([_sweep_fp32(-12, 5), _neighbours(mids), _neighbours(-mids), _neighbours(GRID),
                        np.array([0.0, -0.0, 6.0, 7.99, 8.0, 1e30, -1e30, 1e-40], np.float32)]).astype(np.float32)
    lib = oracle.lib()
    ours = np.array([lib.or_e2m1_encode(float(v)) for v in x], np.uint8)
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, e.g. x={x[bad[:5]]} ours={ours[bad[:5]]} ref={ref[bad[:5]]}"


def test_e2m1_tie_table_and_roundtrip():
    # RNE ties go to the even code (OCP MX v1.0 rounding): 0.25->0, 0.75->1, 1.25->1,
    # 1.75->2, 2.5->2, 3.5->4, 5->4; saturation at 6.
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0, 7.0: 6.0, 100.0: 6.0}
    for x, want in ties.items():
        c = oracle.e2m1_encode([x])[0]
        assert oracle.e2m1_decode([c])[0] == want, x
        c = oracle.e2m1_encode([-x])[0]
        assert oracle.e2m1_decode([c])[0] == -want, -x
    for code in range(16):
        v = oracle.e2m1_decode([code])[0]
        if code == 8:
            assert oracle.e2m1_encode([-0.0])[0] == 8
        else:
            assert oracle.e2m1_encode([v])[0] == code
    # negative values that round to zero keep the sign bit
    assert oracle.e2m1_encode([-0.1])[0] == 8


def test_ue4m3_against_ml_dtypes():
    vals = np.array([oracle.ue4m3_decode([c])[0] for c in range(127)])
    mids = (vals[:-1] + vals[1:]) / 2
    x = np.concatenate([np.abs(_sweep_fp32(-14, 9)), _neighbours(mids), _neighbours(vals[1:]),
                        np.array([0.0, 2.0 ** -10, 1.5 * 2.0 ** -10, 448.0, 463.99], np.float32)])
    x = x[(x >= 0) & (x < 464)].astype(np.float32)
    lib = oracle.lib()
    ours = np.array([lib.or_ue4m3_encode(float(v)) for v in x], np.uint8)
    ref = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches e.g. {x[bad[:5]]}: {ours[bad[:5]]} vs {ref[bad[:5]]}"


def test_ue4m3_saturation_and_decode():
    assert list(oracle.ue4m3_encode([448, 464, 500, 1e9])) == [0x7E] * 4
    assert oracle.ue4m3_decode([0x7E])[0] == 448.0
    assert oracle.ue4m3_decode([1])[0] == 2.0 ** -9       # smallest subnormal
    assert oracle.ue4m3_decode([8])[0] == 2.0 ** -6       # smallest normal
    ref = np.arange(127, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    assert np.array_equal(oracle.ue4m3_decode(np.arange(127)), ref)


def test_ue8m0_decode_and_mx_exponent_property():
    assert oracle.ue8m0_decode([127])[0] == 1.0
    assert oracle.ue8m0_decode([0])[0] == 2.0 ** -127
    ref = np.arange(255, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    assert np.array_equal(oracle.ue8m0_decode(np.arange(255)), ref)
    # defining property (OCP MX: emax of E2M1 is 2): after the shift by 2^-E the
    # block maximum lands in the top binade [4, 8) of E2M1, unless clamped.
    rng = np.random.default_rng(1)
    for amax in np.concatenate([rng.lognormal(0, 20, 2000), [1.0, 4.0, 6.0, 8.0, 2.0 ** -120, 3e38]]).astype(np.float32):
        E = oracle.mx_exponent(float(amax))
        y = float(amax) * 2.0 ** (-E)
        if -127 < E < 127:
            assert 4.0 <= y < 8.0, (amax, E)
    assert oracle.mx_exponent(0.0) == -127
    assert oracle.mx_exponent(2.0 ** -140) == -127


def test_nvfp4_block_exact_roundtrip():
    # A block of grid values times a power of two whose max is 6*2^e has
    # t = amax/6 = 2^e exactly, so the scale is exact and every code round-trips.
    rng = np.random.default_rng(2)
    for e in range(-9, 8):
        vals = rng.choice(np.concatenate([GRID, -GRID]), 16)
        vals[rng.integers(16)] = 6.0
        x = (vals * 2.0 ** e).astype(np.float32)
        codes, sc = oracle.quantize_rows(x[None, :], oracle.NVFP4)
        deq = oracle.dequantize_rows(codes, sc, oracle.NVFP4)[0]
        assert np.array_equal(deq, x.astype(np.float64)), e
        assert oracle.ue4m3_decode(sc[0])[0] == 2.0 ** e


def test_nvfp4_error_bound_and_zero_block():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((512, 64)).astype(np.float32) * np.exp(rng.uniform(-8, 5, (512, 1))).astype(np.float32)
    codes, sc = oracle.quantize_rows(x, oracle.NVFP4)
    deq = oracle.dequantize_rows(codes, sc, oracle.NVFP4)
    # Per block: the decoded scale sd is within 1/16 (half an E4M3 ulp) of
    # amax/6, so x/sd stays within 6*17/16 and the rounding error is at most
    # half of the widest grid step (2), i.e. |x - deq| <= sd.  Blocks whose
    # scale underflows (amax/6 <= 2^-10) quantize to zero.
    amax = np.abs(x).reshape(512, 4, 16).max(-1)
    sd = oracle.ue4m3_decode(sc.ravel()).reshape(sc.shape)
    err = np.abs(x - deq).reshape(512, 4, 16).max(-1)
    live = sc != 0
    normal = sc >= 8
    assert np.all(np.abs(sd[normal] / (amax[normal] / 6) - 1) <= 1 / 16 + 1e-7)
    # inside the grid the error is at most half a step (<= sd); above 6*sd
    # (subnormal scales only) the element saturates to 6*sd
    assert np.all(err[live] <= np.maximum(sd[live], amax[live] - 6 * sd[live]))
    assert np.all(err[normal] <= sd[normal])
    assert np.all(amax[~live] / 6 <= 2.0 ** -10)
    assert np.all(deq.reshape(512, 4, 16)[~live] == 0)
    z = np.zeros((1, 16), np.float32)
    codes, sc = oracle.quantize_rows(z, oracle.NVFP4)
    assert sc[0, 0] == 0 and np.all(codes == 0)
    # a block whose scale underflows to zero gives all-zero codes
    tiny = np.full((1, 16), 2.0 ** -20, np.float32)
    codes, sc = oracle.quantize_rows(tiny, oracle.NVFP4)
    assert sc[0, 0] == 0 and np.all(codes == 0)


def test_mxfp4_block_exact_roundtrip_and_clip():
    rng = np.random.default_rng(4)
    for E in (-127, -60, -3, 0, 5, 100):
        vals = rng.choice(np.concatenate([GRID, -GRID]), 32)
        vals[0] = 4.0   # max in [4, 8) -> shared exponent E
        x = (vals * 2.0 ** E).astype(np.float32)
        if not np.all(np.isfinite(x)) or np.any((x != 0) & (np.abs(x) < 2.0 ** -149)):
            continue
        codes, sc = oracle.quantize_rows(x[None, :], oracle.MXFP4)
        assert int(sc[0, 0]) == E + 127
        assert np.array_equal(oracle.dequantize_rows(codes, sc, oracle.MXFP4)[0], x.astype(np.float64))
    # values in [6, 8) after the shift clip to 6
    x = np.full((1, 32), 7.5, np.float32)
    codes, sc = oracle.quantize_rows(x, oracle.MXFP4)
    assert int(sc[0, 0]) == 127 and np.all(oracle.unpack_codes(codes) == 7)


def test_packing_low_nibble_first():
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 6.0    # code 7 in the low nibble of byte 0
    x[0, 1] = -0.5   # code 9 in the high nibble of byte 0
    x[0, 3] = 1.0    # code 2 in the high nibble of byte 1
    codes, sc = oracle.quantize_rows(x, oracle.NVFP4)
    assert oracle.ue4m3_decode(sc[0])[0] == 1.0
    assert codes[0, 0] == (7 | (9 << 4)) and codes[0, 1] == (2 << 4)


def test_tiled_scale_layout():
    # Defined map: 512-byte chunk (row//128, block//4); inside it byte
    # (row%32)*16 + ((row%128)//32)*4 + block%4.
    lib = oracle.lib()
    assert lib.or_sf_tiled_offset(0, 0, 2) == 0
    assert lib.or_sf_tiled_offset(1, 0, 2) == 16
    assert lib.or_sf_tiled_offset(32, 0, 2) == 4
    assert lib.or_sf_tiled_offset(33, 5, 2) == 512 + 16 + 4 + 1
    assert lib.or_sf_tiled_offset(130, 7, 2) == 2 * 512 + 512 + 2 * 16 + 3
    rows, nb = 256, 8
    plain = np.arange(rows * nb, dtype=np.int64).reshape(rows, nb) % 251
    tiled = oracle.sf_tile(plain.astype(np.uint8))
    offs = np.array([[lib.or_sf_tiled_offset(r, b, 2) for b in range(nb)] for r in range(rows)])
    assert len(set(offs.ravel().tolist())) == rows * nb          # injective
    assert offs.max() < tiled.size
    assert np.array_equal(tiled[offs], plain.astype(np.uint8))


def test_calibration_closed_form():
    B, Hq, Hkv, T, d = 2, 4, 2, 8, 16
    q = np.full((B, Hq, T, d), 0.5, np.float32)
    k = np.full((B, Hkv, T, d), 0.5, np.float32)
    # group 1 (q heads 2, 3), channel 5: aK = 16 (batch 1, token 6), aQ = 4 (head 3, token 6)
    k[1, 1, 6, 5] = -16.0
    q[0, 3, 6, 5] = 4.0
    q[1, 3, 7, 5] = 99.0      # beyond n_cal=7: ignored
    s, inv = oracle.calibrate(q, k, n_cal=7, alpha=0.5)
    assert s[1, 5] == 2.0 and inv[1, 5] == 0.5      # sqrt(16)/sqrt(4)
    assert s[0, 5] == 1.0                            # both amax 0.5
    s2, _ = oracle.calibrate(q, k, n_cal=7, alpha=0.25)
    assert s2[1, 5] == np.float32(16 ** 0.25 / 4 ** 0.75)
    s3, inv3 = oracle.calibrate(q, k, n_cal=7, alpha=0.5, enable=False)
    assert np.all(s3 == 1.0) and np.all(inv3 == 1.0)
    k[0, 0, 0, 0] = 1e30       # clamp at 2^16
    s4, _ = oracle.calibrate(q, k, n_cal=7, alpha=1.0)
    assert s4[0, 0] == 2.0 ** 16


def test_applicability_gate():
    """The gate (a reading: smoothing on for a kv head only if its largest K
    channel amax exceeds 8 times the channel median) on hand-built amax
    patterns: each head's scales are either exactly the ungated ones or all
    ones, and the decision flips right at the threshold."""
    B, Hq, Hkv, T, d = 1, 4, 2, 4, 16
    q = np.full((B, Hq, T, d), 1.0, np.float32)
    k = np.zeros((B, Hkv, T, d), np.float32)
    # head 0: channel amax 1..16 except channel 15 = 8 * median + a hair -> on
    # head 1: channel amax 1..16 with channel 15 = exactly 8 * median -> off
    base = np.arange(1, d + 1, dtype=np.float32)          # median (8 + 9) / 2 = 8.5
    for h in range(Hkv):
        k[0, h, 0, :] = base
    k[0, 0, 0, 15] = np.nextafter(np.float32(68.0), np.float32(1e9))
    k[0, 1, 0, 15] = 68.0
    s_on, inv_on = oracle.calibrate(q, k, n_cal=T, alpha=0.5, enable=True)
    s_g, inv_g = oracle.calibrate(q, k, n_cal=T, alpha=0.5, enable=oracle.GATE)
    assert np.array_equal(s_g[0], s_on[0]) and np.array_equal(inv_g[0], inv_on[0])
    assert np.all(s_g[1] == 1.0) and np.all(inv_g[1] == 1.0)
    assert not np.all(s_on[1] == 1.0)        # the ungated scales do differ from 1 there
    # an outlier-free layer keeps every head off
    k2 = np.ones((B, Hkv, T, d), np.float32)
    s2, _ = oracle.calibrate(q, k2, n_cal=T, alpha=0.5, enable=oracle.GATE)
    assert np.all(s2 == 1.0)
