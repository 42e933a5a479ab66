"""The decode entry point that allocates nothing (hifa4_attn_decode_noalloc),
for callers that are handed only input and output buffers and may not
allocate device memory themselves.  Its output must agree with the ordinary
decode entry point (caller-provided workspace) within the parity tolerance,
on two calls in a row, since every call reuses the library's one scratch
array.  This file is collected last on purpose."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def test_noalloc_decode_matches_workspace_decode():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_quantized_flashattention_smooth_b200 as h
    L = h.lib()
    B, Hq, Hkv, kv, d = 2, 8, 2, 1500, 128
    _, k, v = U.synthetic(B, Hq, Hkv, kv, d, seed=11)
    g = np.random.Generator(np.random.PCG64(12))
    q = torch.from_numpy(g.standard_normal((B, Hq, d), dtype=np.float32)).to(torch.bfloat16).cuda()
    s, inv = h.calibrate_smooth_qk(q[:, :, None, :].expand(B, Hq, 8, d).contiguous(), k[:, :, :8].cuda(), 8)
    cache = h.quantize_kv(k.cuda(), v.cuda(), inv, h.NVFP4, Hq=Hq)
    scale = 1.0 / math.sqrt(d)
    ref, used_ref = h.attn_decode(q, s, cache, kv, scale, h.PREORDER, 3)
    outs = []
    for _ in range(2):
        o = torch.empty((B, Hq, d), device="cuda", dtype=torch.bfloat16)
        used = ctypes.c_int(0)
        st = L.hifa4_attn_decode_noalloc(
            ctypes.c_void_p(q.data_ptr()), h.BF16, ctypes.c_void_p(s.data_ptr()),
            ctypes.c_void_p(cache.k_codes.data_ptr()), ctypes.c_void_p(cache.k_scales.data_ptr()),
            ctypes.c_void_p(cache.vt_codes.data_ptr()), ctypes.c_void_p(cache.vt_scales.data_ptr()),
            B, Hq, Hkv, kv, d, h.NVFP4, scale, h.PREORDER, 128, 3, ctypes.byref(used),
            ctypes.c_void_p(o.data_ptr()), h.BF16, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, L.hifa4_last_error()
        assert used.value == used_ref
        torch.cuda.synchronize()
        outs.append(o)
        ok, err, bound, cos = U.compare_out(U.to_np(o), U.to_np(ref))
        assert ok, f"max|dO|={err:.3e} bound={bound:.3e} cos={cos:.6f}"
    ok, err, bound, cos = U.compare_out(U.to_np(outs[1]), U.to_np(outs[0]))
    assert ok
    # a call that needs more than the library's scratch is refused, not run
    big_B = int(L.hifa4_decode_noalloc_max_bytes() // (Hq * (d + 2) * 4)) + 1
    st = L.hifa4_attn_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), h.BF16, None, ctypes.c_void_p(cache.k_codes.data_ptr()),
        ctypes.c_void_p(cache.k_scales.data_ptr()), ctypes.c_void_p(cache.vt_codes.data_ptr()),
        ctypes.c_void_p(cache.vt_scales.data_ptr()), big_B, Hq, Hkv, kv, d, h.NVFP4, scale, h.PREORDER, 128, 1,
        None, ctypes.c_void_p(outs[0].data_ptr()), h.BF16, None)
    assert st == 1 and b"scratch" in L.hifa4_last_error()
    assert h.device_error() == 0
