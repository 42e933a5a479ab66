"""The C-ABI library loads, exports every symbol include/hifa4.h declares, and
validates arguments on the host (no GPU work is launched by these calls)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    from bit_quantized_flashattention_smooth_b200 import build as b
    b.build()
    import bit_quantized_flashattention_smooth_b200 as h
    return h.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "hifa4.h")).read()
    return sorted(set(re.findall(r"HIFA4_API\s+[\w\s\*]+?\b(hifa4_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    import bit_quantized_flashattention_smooth_b200 as h
    assert set(h.ABI_FUNCTIONS) == set(names)


def test_size_helpers(L):
    import bit_quantized_flashattention_smooth_b200 as h
    assert L.hifa4_codes_bytes(200, 128) == 256 * 64
    # Q rows N=200 -> 256 rows = 2 row groups; d=128 NVFP4 -> 8 blocks -> 2 chunks
    assert h.scale_bytes(200, 128, h.NVFP4) == 2 * 2 * 512
    assert h.scale_bytes(200, 128, h.MXFP4) == 2 * 1 * 512
    assert h.scale_bytes(64, 4096, h.NVFP4) == 1 * 64 * 512      # V^T of d=64, Np=4096
    assert h.decode_workspace_bytes(2, 8, 128, 4) == 2 * 8 * 4 * 130 * 4
    assert 1 <= h.default_splits(64, 8, 32768) <= 256


def test_host_validation_without_gpu(L):
    import bit_quantized_flashattention_smooth_b200 as h
    nul = None
    fake = ctypes.c_void_p(16)   # never dereferenced: validation fails first
    # d = 96 unsupported
    st = L.hifa4_attn_fwd(fake, fake, fake, fake, fake, fake, 1, 2, 2, 128, 96, 0, 0.1, 1, 0, 128, fake, 0,
                          nul, nul, nul, nul)
    assert st == 2 and b"d=96" in L.hifa4_last_error()
    # Hq not a multiple of Hkv
    st = L.hifa4_quantize_qkv(fake, fake, fake, 0, 1, 6, 4, 128, 128, nul, nul, 0, fake, fake, fake, fake,
                              fake, fake, nul)
    assert st == 1
    # misaligned pointer
    bad = ctypes.c_void_p(24)
    st = L.hifa4_attn_fwd(fake, fake, fake, fake, bad, fake, 1, 2, 2, 128, 128, 0, 0.1, 1, 0, 128, fake, 0,
                          nul, nul, nul, nul)
    assert st == 1 and b"aligned" in L.hifa4_last_error()
    # bad block size / null output
    st = L.hifa4_attn_fwd(fake, fake, fake, fake, fake, fake, 1, 2, 2, 128, 128, 0, 0.1, 1, 0, 96, fake, 0,
                          nul, nul, nul, nul)
    assert st == 2
    st = L.hifa4_attn_fwd(fake, fake, fake, fake, fake, fake, 1, 2, 2, 128, 128, 0, 0.1, 1, 0, 128, nul, 0,
                          nul, nul, nul, nul)
    assert st == 1
    # lazy rescale threshold: [0, 3] for NVFP4 (P-hat scale range), [0, 8] for MXFP4, NaN refused
    for fmt, tau in ((0, 3.5), (0, -1.0), (1, 8.5), (0, float("nan"))):
        st = L.hifa4_attn_fwd_ex(fake, fake, fake, fake, fake, fake, 1, 2, 2, 128, 128, fmt, 0.1, 1, 0, 128, fake,
                                 0, nul, nul, nul, ctypes.c_float(tau), nul)
        assert st == 1 and b"rescale_threshold" in L.hifa4_last_error(), (fmt, tau)
    used0 = ctypes.c_int(0)
    st = L.hifa4_attn_decode_cache(fake, 0, nul, fake, fake, fake, fake, 1, 8, 2, 1024, 1024, 128, 0, 0.1, 0, 128,
                                   0, ctypes.byref(used0), fake, 1 << 20, fake, 0, ctypes.c_float(4.0), nul)
    assert st == 1 and b"rescale_threshold" in L.hifa4_last_error()
    # fused path: Q dtype, null pointers and tile checks as the unfused entry
    st = L.hifa4_attn_fwd_fused(fake, 7, nul, fake, fake, fake, fake, 1, 2, 2, 128, 128, 0, 0.1, 1, 0, 128, fake, 0,
                                nul, nul, nul, ctypes.c_float(0.0), nul)
    assert st == 1 and b"dtype" in L.hifa4_last_error()
    st = L.hifa4_attn_fwd_fused(nul, 0, nul, fake, fake, fake, fake, 1, 2, 2, 128, 128, 0, 0.1, 1, 0, 128, fake, 0,
                                nul, nul, nul, ctypes.c_float(0.0), nul)
    assert st == 1
    st = L.hifa4_attn_fwd_fused(fake, 0, nul, fake, fake, fake, fake, 1, 2, 2, 128, 256, 0, 0.1, 1, 0, 64, fake, 0,
                                nul, nul, nul, ctypes.c_float(0.0), nul)
    assert st == 2
    # decode: d must be 128, workspace required
    used = ctypes.c_int(0)
    st = L.hifa4_attn_decode(fake, 0, nul, fake, fake, fake, fake, 1, 8, 2, 1024, 64, 0, 0.1, 0, 128, 0,
                             ctypes.byref(used), fake, 1 << 20, fake, 0, nul)
    assert st == 2
    st = L.hifa4_attn_decode(fake, 0, nul, fake, fake, fake, fake, 1, 8, 2, 1024, 128, 0, 0.1, 0, 128, 0,
                             ctypes.byref(used), nul, 0, fake, 0, nul)
    assert st == 1
    assert L.hifa4_status_string(2) == b"unsupported configuration"


def test_q_mean_entry_points_validate_on_the_host(L):
    """The Q-Mean auxiliary's four entry points refuse bad arguments before
    any launch: null or misaligned pointers, d = 256 in the forward, more
    than 8 query heads per kv head for the score terms, bad calibration
    counts."""
    nul = None
    fake = ctypes.c_void_p(16)
    bad = ctypes.c_void_p(24)
    # calibration: n_cal outside (0, ld_tok], null output
    st = L.hifa4_calibrate_q_mean(fake, 0, 1, 4, 2, 0, 64, 128, nul, fake, nul)
    assert st == 1 and b"n_cal" in L.hifa4_last_error()
    st = L.hifa4_calibrate_q_mean(fake, 0, 1, 4, 2, 32, 64, 128, nul, nul, nul)
    assert st == 1
    # quantize with the mean: q_mu required and aligned
    st = L.hifa4_quantize_qkv_qmean(fake, fake, fake, 0, 1, 4, 2, 128, 128, nul, nul, nul, 0, fake, fake, fake,
                                    fake, fake, fake, nul)
    assert st == 1 and b"q_mu" in L.hifa4_last_error()
    st = L.hifa4_quantize_qkv_qmean(fake, fake, fake, 0, 1, 4, 2, 128, 128, nul, nul, bad, 0, fake, fake, fake,
                                    fake, fake, fake, nul)
    assert st == 1 and b"q_mu" in L.hifa4_last_error()
    # score terms: at most 8 query heads per kv head
    st = L.hifa4_q_mean_bias(fake, fake, fake, 1, 16, 1, 128, 128, 0, fake, nul)
    assert st == 2 and b"8 query heads" in L.hifa4_last_error()
    st = L.hifa4_q_mean_bias(fake, fake, fake, 4096, 32, 8, 128, 128, 0, fake, nul)
    assert st == 2 and b"65535" in L.hifa4_last_error()
    # forward: d = 256 refused, terms required and aligned
    st = L.hifa4_attn_fwd_qmean(fake, fake, fake, fake, fake, fake, fake, 1, 2, 2, 128, 256, 0, 0.1, 1, 0, 128,
                                fake, 0, nul, ctypes.c_float(0.0), nul)
    assert st == 2 and b"d=256" in L.hifa4_last_error()
    st = L.hifa4_attn_fwd_qmean(fake, fake, fake, fake, fake, fake, bad, 1, 2, 2, 128, 128, 0, 0.1, 1, 0, 128,
                                fake, 0, nul, ctypes.c_float(0.0), nul)
    assert st == 1 and b"aligned" in L.hifa4_last_error()
    st = L.hifa4_attn_fwd_qmean(fake, fake, fake, fake, fake, fake, nul, 1, 2, 2, 128, 128, 0, 0.1, 1, 0, 128,
                                fake, 0, nul, ctypes.c_float(0.0), nul)
    assert st == 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import bit_quantized_flashattention_smooth_b200 as h
    monkeypatch.setattr(h, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(h, "_lib", None)
    with pytest.raises(h.HiFA4Error):
        h.lib()
