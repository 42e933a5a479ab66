"""The fused prefill path (Smooth-QK scaling and Q quantization inside the
attention kernel) against the two-launch path (hifa4_quantize_qkv, then
hifa4_attn_fwd_ex): the in-kernel Q-hat follows the same rules, so O, lse and
the debug normalizers must be bit-identical; the two-launch path is itself
held to the oracle by test_gpu_kernels and test_gpu_fullsize."""
import math

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


FUSED_CASES = [
    # B, Hq, Hkv, N, d, causal, BN, fmt, mode, dtype, smooth, tau
    (1, 2, 2, 256, 64, False, 64, oracle.NVFP4, oracle.PREORDER, torch.float16, True, 0.0),
    (1, 4, 1, 200, 128, True, 128, oracle.NVFP4, oracle.INCONSISTENT, torch.bfloat16, True, 0.0),
    (1, 4, 2, 384, 128, True, 64, oracle.MXFP4, oracle.PREORDER, torch.bfloat16, True, 0.0),
    (1, 2, 2, 300, 64, False, 128, oracle.MXFP4, oracle.INCONSISTENT, torch.bfloat16, False, 0.0),
    (1, 4, 2, 130, 256, True, 128, oracle.NVFP4, oracle.PREORDER, torch.bfloat16, True, 3.0),
    (2, 2, 1, 257, 256, False, 128, oracle.MXFP4, oracle.PREORDER, torch.float16, True, 0.0),
    (1, 2, 2, 1, 128, True, 128, oracle.NVFP4, oracle.PREORDER, torch.bfloat16, True, 0.0),
    (2, 8, 2, 520, 128, True, 64, oracle.NVFP4, oracle.PREORDER, torch.bfloat16, True, 3.0),
    (1, 4, 2, 77, 64, True, 64, oracle.MXFP4, oracle.PREORDER, torch.bfloat16, True, 0.0),
]


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal,BN,fmt,mode,dtype,smooth,tau", FUSED_CASES)
def test_fused_equals_two_launch_path(B, Hq, Hkv, N, d, causal, BN, fmt, mode, dtype, smooth, tau):
    q, k, v = U.synthetic(B, Hq, Hkv, N, d, seed=13 * N + d, dtype=dtype)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    s = inv = None
    if smooth:
        s, inv = h.calibrate_smooth_qk(q, k, n_cal=min(N, 64))
    z = h.quantize_qkv(q, k, v, s, inv, fmt)
    scale = 1.0 / math.sqrt(d)
    ref = h.attn_fwd(z, scale, causal, mode, BN, out_dtype=dtype, return_lse=True, debug=True,
                     rescale_threshold=tau)
    kv = h.quantize_kv(k, v, inv, fmt, Hq=Hq)
    got = h.attn_fwd_fused(q, s, kv, scale, causal, mode, BN, out_dtype=dtype, return_lse=True, debug=True,
                           rescale_threshold=tau)
    for a, b, name in zip(got, ref, ("O", "lse", "l_phat", "l_p")):
        assert torch.equal(a, b), name


def test_fused_full_size_and_repeatable():
    """The 32-head 4096-token causal prefill, NVFP4, 64-key tiles."""
    q, k, v = U.synthetic(1, 32, 8, 4096, 128, seed=21)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    s, inv = h.calibrate_smooth_qk(q, k, n_cal=256)
    z = h.quantize_qkv(q, k, v, s, inv, oracle.NVFP4)
    ref = h.attn_fwd(z, None, True, oracle.PREORDER, 64)
    kv = h.quantize_kv(k, v, inv, oracle.NVFP4, Hq=32)
    o = h.attn_fwd_fused(q, s, kv, None, True, oracle.PREORDER, 64)
    assert torch.equal(o, ref)
    for _ in range(5):
        assert torch.equal(h.attn_fwd_fused(q, s, kv, None, True, oracle.PREORDER, 64), o)
