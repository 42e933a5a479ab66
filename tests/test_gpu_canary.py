"""Out-of-bounds writes: every output of quantize, prefill, decode and the
BF16 kernel is a view at the start of a larger buffer whose tail holds a
canary pattern; after the launches the tail must be untouched."""
import math

import pytest
import torch

import oracle
from bit_quantized_flashattention_smooth_b200 import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

h = None
TAIL = 4096


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


class Canary:
    """Tensors carved from the front of buffers with a 4 KiB patterned tail."""

    def __init__(self):
        self.bufs = []

    def empty(self, shape, dtype):
        n = math.prod(shape)
        esz = torch.empty((), dtype=dtype).element_size()
        raw = torch.empty(n * esz + TAIL, device="cuda", dtype=torch.uint8)
        raw[n * esz:] = 0xA5
        self.bufs.append((raw, n * esz))
        return raw[: n * esz].view(dtype).view(shape)

    def check(self):
        torch.cuda.synchronize()
        for raw, used in self.bufs:
            tail = raw[used:]
            assert bool((tail == 0xA5).all()), f"{int((tail != 0xA5).sum())} tail bytes overwritten"


def _quantized(cn, B, Hq, Hkv, N, d, fmt):
    Np = h.pad128(N)
    sq, sv = h.scale_bytes(N, d, fmt), h.scale_bytes(d, Np, fmt)
    u8 = torch.uint8
    return h.QuantizedQKV(cn.empty((B, Hq, Np, d // 2), u8), cn.empty((B, Hq, sq), u8),
                          cn.empty((B, Hkv, Np, d // 2), u8), cn.empty((B, Hkv, sq), u8),
                          cn.empty((B, Hkv, d, Np // 2), u8), cn.empty((B, Hkv, sv), u8), B, Hq, Hkv, N, d, fmt)


@pytest.mark.parametrize("B,Hq,Hkv,N,d,fmt,BN", [
    (1, 4, 2, 200, 128, oracle.NVFP4, 64),
    (2, 2, 1, 130, 64, oracle.MXFP4, 128),
    (1, 2, 2, 257, 256, oracle.NVFP4, 128),
])
def test_prefill_writes_stay_in_bounds(B, Hq, Hkv, N, d, fmt, BN):
    q, k, v = U.synthetic(B, Hq, Hkv, N, d, seed=5 * N + d, dtype=torch.bfloat16)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    cn = Canary()
    s, inv = h.calibrate_smooth_qk(q, k, min(N, 64))
    z = h.quantize_qkv(q, k, v, s, inv, fmt, out=_quantized(cn, B, Hq, Hkv, N, d, fmt))
    o = cn.empty((B, Hq, N, d), torch.bfloat16)
    for mode in (oracle.PREORDER, oracle.INCONSISTENT):
        h.attn_fwd(z, 1.0 / math.sqrt(d), True, mode, BN, out=o)
    cn.check()


def test_bf16_writes_stay_in_bounds():
    g = torch.Generator(device="cuda").manual_seed(3)
    q = torch.randn((1, 4, 200, 128), generator=g, device="cuda").to(torch.bfloat16)
    k = torch.randn((1, 2, 200, 128), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((1, 2, 200, 128), generator=g, device="cuda").to(torch.bfloat16)
    cn = Canary()
    vt = cn.empty((1, 2, 128, 200), torch.bfloat16)
    h.lib().hifa4_bf16_transpose_v(h._ptr(v), 1, 2, 200, 128, h._ptr(vt), h._stream())
    o = cn.empty((1, 4, 200, 128), torch.bfloat16)
    h.bf16_attn_fwd(q, k, vt, out=o)
    cn.check()


def test_decode_writes_stay_in_bounds():
    B, Hq, Hkv, kv, d = 3, 8, 2, 1000, 128
    g = torch.Generator(device="cuda").manual_seed(4)
    k = torch.randn((B, Hkv, kv, d), generator=g, device="cuda").to(torch.bfloat16)
    v = torch.randn((B, Hkv, kv, d), generator=g, device="cuda").to(torch.bfloat16)
    q = torch.randn((B, Hq, d), generator=g, device="cuda").to(torch.bfloat16)
    cache = h.quantize_kv(k, v, None, oracle.NVFP4, Hq=Hq)
    splits = h.default_splits(B, Hkv, kv)
    cn = Canary()
    ws = cn.empty((h.decode_workspace_bytes(B, Hq, d, splits),), torch.uint8)
    o = cn.empty((B, Hq, d), torch.bfloat16)
    h.attn_decode(q, None, cache, kv, None, oracle.PREORDER, splits, ws, o)
    cn.check()
