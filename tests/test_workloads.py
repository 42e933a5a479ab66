"""The seeded synthetic inputs follow the stated recipe (no GPU): shapes and
dtypes of the five workloads, determinism per seed, the K outlier channels
(positive, scaled, on the lowest-frequency RoPE pairs), the rotate-half RoPE
(norm-preserving per pair, identity at position 0, the numpy and torch
versions agree), the Student-t K of the long-context workload, and the FLOP
and exponential counts the bench divides by."""
import numpy as np
import pytest
import torch

from bit_quantized_flashattention_smooth_b200 import workloads as W


@pytest.mark.parametrize("name,shape,dtype", [
    ("tiny_mha", (1, 2, 2, 256, 64), torch.float16),
    ("qwen3_prefill", (1, 32, 8, 4096, 128), torch.bfloat16),
    ("gemma2_prefill", (1, 16, 8, 8192, 256), torch.bfloat16),
    ("long_prefill", (8, 32, 8, 16384, 128), torch.bfloat16),
    ("split_decode", (64, 32, 8, 32768, 128), torch.bfloat16),
    ("qwen3_qmean", (1, 32, 8, 4096, 128), torch.bfloat16),
])
def test_workload_table(name, shape, dtype):
    w = W.WORKLOADS[name]
    assert (w.B, w.Hq, w.Hkv, w.N, w.d) == shape
    assert W.torch_dtype(w.dtype) == dtype
    assert w.Hq % w.Hkv == 0


def test_prefill_draw_is_seeded_and_shaped():
    w = W.WORKLOADS["qwen3_prefill"]
    q, k, v = W.make_prefill(w, N=256)
    q2, k2, v2 = W.make_prefill(w, N=256)
    assert q.shape == (1, 32, 256, 128) and k.shape == (1, 8, 256, 128) and v.shape == k.shape
    assert q.dtype == torch.bfloat16
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    w2 = W.Workload(**{**w.__dict__, "seed": w.seed + 1000})
    q3, _, _ = W.make_prefill(w2, N=256)
    assert not torch.equal(q, q3)


def test_outlier_channels_on_low_frequency_pairs():
    w = W.WORKLOADS["qwen3_prefill"]
    assert w.outlier_channels == (61, 62, 63, 125, 126, 127)
    _, k, _ = W.make_prefill(w, N=512)
    kf = k.float()
    out = list(w.outlier_channels)
    rest = [c for c in range(w.d) if c not in out]
    # 15 |z| before RoPE; the lowest-frequency pairs barely rotate over 512 tokens
    assert kf[..., out].mean() > 10.0
    assert kf[..., rest].abs().mean() < 1.0
    assert (kf[:, :, 0, out] >= 0).all()                # position 0: RoPE is the identity
    tiny = W.WORKLOADS["tiny_mha"]
    _, kt, _ = W.make_prefill(tiny)
    assert (kt[..., 60:64].float() >= 0).all() and kt[..., 60:64].float().mean() > 12.0


def test_rope_is_rotate_half_and_norm_preserving():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, 3, 40, 16)).astype(np.float32)
    y = W.rope_neox(x, 1e4)
    np.testing.assert_array_equal(y[..., 0, :], x[..., 0, :])
    n_x = x[..., :8] ** 2 + x[..., 8:] ** 2
    n_y = y[..., :8].astype(np.float64) ** 2 + y[..., 8:].astype(np.float64) ** 2
    np.testing.assert_allclose(n_y, n_x, rtol=1e-5)
    yt = W.rope_torch(torch.from_numpy(x), 1e4).numpy()
    np.testing.assert_allclose(yt, y, rtol=1e-6, atol=1e-6)
    # position p of a unit vector on pair 0 rotates by p radians (inv_freq[0] = 1)
    e = np.zeros((1, 5, 16), np.float32)
    e[..., 0] = 1.0
    r = W.rope_neox(e, 1e4)
    np.testing.assert_allclose(r[0, :, 0], np.cos(np.arange(5)), atol=1e-6)
    np.testing.assert_allclose(r[0, :, 8], np.sin(np.arange(5)), atol=1e-6)


def test_long_context_k_is_heavy_tailed():
    w = W.WORKLOADS["long_prefill"]
    _, k, _ = W.make_prefill(w, N=256, B=1)
    kf = k.float().flatten()
    kurt = float(((kf - kf.mean()) ** 4).mean() / kf.var() ** 2)
    assert kurt > 6.0               # a normal draw has 3; Student-t(3) has no finite fourth moment
    assert w.outlier_channels == ()


def test_work_counts():
    w = W.WORKLOADS["qwen3_prefill"]
    assert W.attended_pairs(4096, True) == 4096 * 4097 // 2
    assert W.prefill_flops(w) == 4 * 1 * 32 * 128 * (4096 * 4097 // 2)
    assert abs(W.prefill_flops(w) / 1e9 - 137.4) < 0.1
    assert W.exp_count(w) == 32 * 4096 * 4097 // 2
    assert W.attended_pairs(256, False) == 256 * 256


@pytest.mark.parametrize("name", ["qwen3_prefill", "gemma2_prefill", "long_prefill"])
def test_prefill_recipe_uses_exact_rope(name):
    """make_prefill (host torch RoPE) equals the numpy recipe bit for bit."""
    w = W.WORKLOADS[name]
    q, k, v = W.make_prefill(w, N=300, B=1)
    rng = np.random.Generator(np.random.PCG64(w.seed))
    qn = rng.standard_normal((1, w.Hq, 300, w.d), dtype=np.float32)
    kn = W._draw_k(rng, (1, w.Hkv, 300, w.d), w)
    vn = rng.standard_normal((1, w.Hkv, 300, w.d), dtype=np.float32)
    qn, kn = W.rope_neox(qn, w.theta), W.rope_neox(kn, w.theta)
    for a, b in ((q, qn), (k, kn), (v, vn)):
        assert torch.equal(a, torch.from_numpy(b).to(W.torch_dtype(w.dtype)))


def test_q_offset_channels_carry_a_near_constant_mean():
    """qwen3_qmean: +8 on Q channels 58-60 before RoPE; those pairs barely
    rotate, so the channels keep a mean near 8 (the other channels near 0),
    and K keeps qwen3_prefill's outliers on channels 61-63 / 125-127."""
    w = W.WORKLOADS["qwen3_qmean"]
    q, k, _ = W.make_prefill(w, N=512)
    qf = q.float()
    m = qf[..., 58:61].mean(dim=(0, 1, 2))
    assert torch.all((m > 7.5) & (m < 8.5)), m
    rest = [c for c in range(w.d) if c not in (58, 59, 60)]
    assert qf[..., rest].mean(dim=(0, 1, 2)).abs().max() < 0.3
    assert k.float()[..., [61, 62, 63]].mean() > 10.0
    w0 = W.WORKLOADS["qwen3_prefill"]
    q0, _, _ = W.make_prefill(w0, N=512)
    assert q0.float()[..., 58:61].mean().abs() < 0.2
