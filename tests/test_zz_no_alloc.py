"""The decode entry point that allocates nothing (hifa4_attn_decode_noalloc),
for callers that are handed only input and output buffers and may not
allocate device memory themselves (a plugin or custom operator inside a
framework whose allocator owns the device memory, or a serving loop where an
allocation could block).  Its output must agree with the ordinary decode
entry point (caller-provided workspace) within the parity tolerance, on calls
in a row that solve different problems, since every call reuses the
library's one scratch array.  This file is collected last on purpose."""
import ctypes
import math

import numpy as np
import pytest
import torch

from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _problem(h, B, Hq, Hkv, kv, d, fmt, seed):
    _, k, v = U.synthetic(B, Hq, Hkv, kv, d, seed=seed)
    g = np.random.Generator(np.random.PCG64(seed + 1))
    q = torch.from_numpy(g.standard_normal((B, Hq, d), dtype=np.float32)).to(torch.bfloat16).cuda()
    s, inv = h.calibrate_smooth_qk(q[:, :, None, :].expand(B, Hq, 8, d).contiguous(), k[:, :, :8].cuda(), 8)
    cache = h.quantize_kv(k.cuda(), v.cuda(), inv, fmt, Hq=Hq)
    return q, s, cache


def _noalloc(L, h, q, s, cache, kv, mode, splits):
    B, Hq, d = q.shape
    o = torch.empty((B, Hq, d), device="cuda", dtype=torch.bfloat16)
    used = ctypes.c_int(0)
    st = L.hifa4_attn_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), h.BF16, ctypes.c_void_p(s.data_ptr()),
        ctypes.c_void_p(cache.k_codes.data_ptr()), ctypes.c_void_p(cache.k_scales.data_ptr()),
        ctypes.c_void_p(cache.vt_codes.data_ptr()), ctypes.c_void_p(cache.vt_scales.data_ptr()),
        B, Hq, cache.Hkv, kv, d, cache.fmt, 1.0 / math.sqrt(d), mode, 128, splits, ctypes.byref(used),
        ctypes.c_void_p(o.data_ptr()), h.BF16, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, L.hifa4_last_error()
    torch.cuda.synchronize()
    return o, used.value


def test_noalloc_decode_matches_workspace_decode():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import bit_quantized_flashattention_smooth_b200 as h
    L = h.lib()
    d = 128
    # two different problems in a row (shape, data, format, normalizer, split
    # count): the second call must not see anything the first left behind
    cases = [((2, 8, 2, 1500), h.NVFP4, h.PREORDER, 3, 11),
             ((3, 16, 4, 2300), h.MXFP4, h.INCONSISTENT, 0, 31),
             ((1, 8, 1, 700), h.NVFP4, h.PREORDER, 2, 41)]
    for (B, Hq, Hkv, kv), fmt, mode, splits, seed in cases:
        q, s, cache = _problem(h, B, Hq, Hkv, kv, d, fmt, seed)
        ref, used_ref = h.attn_decode(q, s, cache, kv, 1.0 / math.sqrt(d), mode, splits)
        o, used = _noalloc(L, h, q, s, cache, kv, mode, splits)
        assert used == used_ref
        ok, err, bound, cos = U.compare_out(U.to_np(o), U.to_np(ref))
        assert ok, f"B={B} kv={kv} fmt={fmt} mode={mode}: max|dO|={err:.3e} bound={bound:.3e} cos={cos:.6f}"
    # a call that needs more than the library's scratch is refused, not run
    q, s, cache = _problem(h, 1, 8, 2, 300, d, h.NVFP4, 51)
    big_B = int(L.hifa4_decode_noalloc_max_bytes() // (8 * (d + 2) * 4)) + 1
    o = torch.empty((1, 8, d), device="cuda", dtype=torch.bfloat16)
    st = L.hifa4_attn_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), h.BF16, None, ctypes.c_void_p(cache.k_codes.data_ptr()),
        ctypes.c_void_p(cache.k_scales.data_ptr()), ctypes.c_void_p(cache.vt_codes.data_ptr()),
        ctypes.c_void_p(cache.vt_scales.data_ptr()), big_B, 8, 2, 300, d, h.NVFP4, 1.0 / math.sqrt(d), h.PREORDER,
        128, 1, None, ctypes.c_void_p(o.data_ptr()), h.BF16, None)
    assert st == 1 and b"scratch" in L.hifa4_last_error()
    assert h.device_error() == 0
