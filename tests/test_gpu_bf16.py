"""The in-house BF16 attention kernel (the unquantized baseline the 4-bit
path is measured against) against a plain PyTorch fp32 reference of the same
op: softmax(Q K^T * scale, causal top-left) V on the bf16 inputs."""
import math

import pytest
import torch

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


def _reference(q, k, v, causal, scale):
    """fp32 attention per head (GQA by head index // G); returns O and the
    base-2 log-sum-exp of the scaled scores."""
    B, Hq, N, d = q.shape
    G = Hq // k.shape[1]
    o = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    mask = torch.ones(N, N, dtype=torch.bool, device=q.device).tril() if causal else None
    for b in range(B):
        for hh in range(Hq):
            s = (q[b, hh].float() @ k[b, hh // G].float().T) * scale
            if mask is not None:
                s = s.masked_fill(~mask, float("-inf"))
            lse[b, hh] = torch.logsumexp(s, dim=-1) / math.log(2.0)
            o[b, hh] = torch.softmax(s, dim=-1) @ v[b, hh // G].float()
    return o, lse


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [
    (1, 2, 2, 256, 64, False),      # the tiny MHA shape
    (1, 4, 2, 200, 128, True),      # GQA, ragged last query and key tiles
    (2, 2, 1, 136, 64, True),       # two batches, one row past a query tile
    (1, 4, 2, 320, 256, True),      # d = 256 (one CTA per SM), ragged
    (1, 32, 8, 4096, 128, True),    # the 32-head 4096-token causal prefill
])
def test_bf16_attention_matches_fp32_reference(B, Hq, Hkv, N, d, causal):
    g = torch.Generator(device="cuda").manual_seed(11)
    q = torch.randn((B, Hq, N, d), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((B, Hkv, N, d), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((B, Hkv, N, d), generator=g, device="cuda").to(torch.bfloat16)
    vt = h.bf16_transpose_v(v)
    assert torch.equal(vt, v.transpose(-1, -2).contiguous())
    scale = 1.0 / math.sqrt(d)
    o, lse = h.bf16_attn_fwd(q, k, vt, scale, causal, return_lse=True)
    torch.cuda.synchronize()
    ref_o, ref_lse = _reference(q, k, v, causal, scale)
    ok, err, bound, cos = U.compare_out(U.to_np(o.float()), U.to_np(ref_o))
    assert ok, f"max|dO|={err:.3e} bound={bound:.3e} cos={cos:.6f}"
    torch.testing.assert_close(lse, ref_lse, rtol=1e-4, atol=1e-4)


def test_bf16_attention_repeatable():
    """Bit-identical outputs over repeated launches (no pipeline race)."""
    g = torch.Generator(device="cuda").manual_seed(12)
    q = torch.randn((1, 32, 4096, 128), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((1, 8, 4096, 128), generator=g, device="cuda").to(torch.bfloat16)
    vt = h.bf16_transpose_v(torch.randn((1, 8, 4096, 128), generator=g, device="cuda").to(torch.bfloat16))
    o0 = h.bf16_attn_fwd(q, k, vt)
    for _ in range(10):
        assert torch.equal(h.bf16_attn_fwd(q, k, vt), o0)
