"""Appendable 4-bit KV cache: any sequence of appends gives, bit for bit, the
one-shot quantization of the whole sequence (hifa4_quantize_kv) and the
oracle's quantization of the zero-padded sequence; decode over it equals
decode over the one-shot cache and the oracle's split decode (exact and
lazily rescaled running max)."""
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
    assert h.device_error() == 0


def _inputs(B, Hkv, L, d, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    k = (torch.randn((B, Hkv, L, d), generator=g, device="cuda") * 2).to(torch.bfloat16)
    v = torch.randn((B, Hkv, L, d), generator=g, device="cuda").to(torch.bfloat16)
    inv_s = torch.exp2(torch.rand((Hkv, d), generator=g, device="cuda") * 4 - 2).float()
    return k, v, inv_s


def _one_shot(k, v, inv_s, cap, fmt):
    """hifa4_quantize_kv of the sequence zero-padded to the capacity (the
    append contract: tokens not yet written are 0)."""
    B, Hkv, L, d = k.shape
    kp = torch.zeros((B, Hkv, cap, d), device="cuda", dtype=k.dtype)
    vp = torch.zeros_like(kp)
    kp[:, :, :L] = k
    vp[:, :, :L] = v
    return h.quantize_kv(kp, vp, inv_s, fmt)


@pytest.mark.parametrize("fmt", [oracle.NVFP4, oracle.MXFP4])
@pytest.mark.parametrize("d,chunks", [
    (128, [200, 1, 1, 5, 13, 17, 3, 32, 100, 61]),
    (64, [1] * 40 + [7, 90]),
    (256, [128, 33, 16, 15, 1]),
])
def test_appends_equal_one_shot_quantization(fmt, d, chunks):
    B, Hkv, Hq, cap = 2, 2, 8, 640
    L = sum(chunks)
    k, v, inv_s = _inputs(B, Hkv, L, d, seed=d + fmt)
    cache, tail = h.alloc_appendable_kv_cache(B, Hq, Hkv, cap, d, fmt)
    pos = 0
    for T in chunks:
        h.kv_cache_append(cache, tail, k[:, :, pos:pos + T], v[:, :, pos:pos + T], inv_s, pos)
        pos += T
        ref = _one_shot(k[:, :, :pos], v[:, :, :pos], inv_s, cap, fmt)
        for name in ("k_codes", "k_scales", "vt_codes", "vt_scales"):
            a, b = getattr(cache, name), getattr(ref, name)
            assert torch.equal(a, b), f"{name} after {pos} tokens: {int((a != b).sum())} bytes differ"
    # the final cache against the oracle's quantizer on the zero-padded
    # sequence (the append contract: tokens not yet written are 0)
    kp = np.zeros((B, Hkv, cap, d), np.float32)
    vp = np.zeros_like(kp)
    kp[:, :, :L] = k.float().cpu().numpy()
    vp[:, :, :L] = v.float().cpu().numpy()
    oz = oracle.quantize_qkv(np.zeros_like(kp), kp, vp, None, inv_s.cpu().numpy(), fmt)
    ot = oracle.tile_scales(oz)
    assert np.array_equal(U.to_np(cache.k_codes).astype(np.uint8), oz["k_codes"])
    assert np.array_equal(U.to_np(cache.vt_codes).astype(np.uint8), oz["vt_codes"])
    assert np.array_equal(U.to_np(cache.k_scales).astype(np.uint8), ot["k_sc"])
    assert np.array_equal(U.to_np(cache.vt_scales).astype(np.uint8), ot["vt_sc"])


def test_decode_over_appended_cache():
    B, Hkv, Hq, d, cap, fmt = 3, 2, 8, 128, 1000, oracle.NVFP4
    k, v, inv_s = _inputs(B, Hkv, 700, d, seed=5)
    cache, tail = h.alloc_appendable_kv_cache(B, Hq, Hkv, cap, d, fmt)
    g = torch.Generator(device="cuda").manual_seed(6)
    q = torch.randn((B, Hq, d), generator=g, device="cuda").to(torch.bfloat16)
    pos = 0
    for T in (300, 1, 99, 300):
        h.kv_cache_append(cache, tail, k[:, :, pos:pos + T], v[:, :, pos:pos + T], inv_s, pos)
        pos += T
        o_app, _ = h.attn_decode(q, None, cache, kv_len=pos)
        one = h.quantize_kv(k[:, :, :pos], v[:, :, :pos], inv_s, fmt, Hq=Hq)
        o_one, _ = h.attn_decode(q, None, one)
        assert torch.equal(o_app, o_one), f"decode over {pos} appended tokens differs"


@pytest.mark.parametrize("fmt,mode,tau", [(oracle.NVFP4, oracle.PREORDER, 0.0), (oracle.NVFP4, oracle.PREORDER, 3.0),
                                          (oracle.MXFP4, oracle.INCONSISTENT, 0.0), (oracle.MXFP4, oracle.PREORDER, 3.0)])
def test_decode_cache_matches_oracle(fmt, mode, tau):
    """hifa4_attn_decode_cache over an appended cache against the oracle's
    split decode of the same tokens, at the kernel's split count, with the
    exact (tau = 0) and the lazily updated (tau = 3) running max."""
    B, Hkv, Hq, d, cap = 2, 2, 8, 128, 1200
    k, v, inv_s = _inputs(B, Hkv, 1100, d, seed=21 + fmt)
    s = (1.0 / inv_s).float()
    cache, tail = h.alloc_appendable_kv_cache(B, Hq, Hkv, cap, d, fmt)
    g = torch.Generator(device="cuda").manual_seed(22)
    q = torch.randn((B, Hq, d), generator=g, device="cuda").to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    pos = 0
    for T in (700, 1, 250, 149):
        h.kv_cache_append(cache, tail, k[:, :, pos:pos + T], v[:, :, pos:pos + T], inv_s, pos)
        pos += T
        o, used = h.attn_decode(q, s, cache, kv_len=pos, softmax_scale=scale, mode=mode, num_splits=3,
                                rescale_threshold=tau)
        kn = k[:, :, :pos].float().cpu().numpy()
        vn = v[:, :, :pos].float().cpu().numpy()
        oz = oracle.quantize_qkv(np.zeros_like(kn), kn, vn, None, inv_s.cpu().numpy(), fmt)
        ref = oracle.decode(q.float().cpu().numpy(), s.cpu().numpy(), oz, pos, fmt, scale, mode, 128,
                            num_splits=used, tau=tau)
        ok, err, bound, cos = U.compare_out(U.to_np(o), ref["O"])
        assert ok, f"{pos} tokens, splits={used}: max|dO|={err:.3e} bound={bound:.3e} cos={cos:.6f}"
