"""bench.py's host-side bookkeeping (no GPU): the DRAM traffic record is
used only for the kernel source it was measured on and for the launch path
it was measured with."""
import hashlib
import json
import os

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _write(tmp_path, recs):
    d = tmp_path / "profiles"
    d.mkdir()
    (d / "traffic.json").write_text(json.dumps(recs))


def test_traffic_record_matches_source_hash_and_path(tmp_path, monkeypatch):
    src = os.path.join(ROOT, "bit_quantized_flashattention_smooth_b200", "csrc", "attn_fwd.cu")
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    base = {"kernel": "attn_fwd_fp4", "workload": "qwen3_prefill", "format": "nvfp4", "block_n": 64,
            "bytes_per_launch": 123}
    fake_root = tmp_path
    (fake_root / "bit_quantized_flashattention_smooth_b200" / "csrc").mkdir(parents=True)
    (fake_root / "bit_quantized_flashattention_smooth_b200" / "csrc" / "attn_fwd.cu").write_bytes(open(src, "rb").read())
    _write(fake_root, [{**base, "path": "two-launch", "source_sha256_16": digest}])
    monkeypatch.setattr(bench, "ROOT", str(fake_root))
    assert bench.traffic_record("attn_fwd_fp4", "qwen3_prefill", "nvfp4", 64, "two-launch") == 123
    # another launch path, tile width or a changed source: no record
    assert bench.traffic_record("attn_fwd_fp4", "qwen3_prefill", "nvfp4", 64, "fused") is None
    assert bench.traffic_record("attn_fwd_fp4", "qwen3_prefill", "nvfp4", 128, "two-launch") is None
    (fake_root / "bit_quantized_flashattention_smooth_b200" / "csrc" / "attn_fwd.cu").write_text("// changed\n")
    assert bench.traffic_record("attn_fwd_fp4", "qwen3_prefill", "nvfp4", 64, "two-launch") is None

