"""Where the 4-bit path's deviation from exact attention comes from (no GPU).

The 4-bit forward quantizes three operands: Q-hat and K-hat (the scores),
P-hat (the attention weights) and V-hat.  On the qwen3 prefill workload (first,
middle and last 128-row query tiles of 8 query heads) the oracle is run with
each quantizer switched off in turn -- raw Smooth-QK'd Q and K for the scores,
P-hat = P, raw V -- and with all three off, and compared with exact fp64
softmax attention of the unquantized inputs.  With everything off the oracle is
exact attention up to the fp32 rounding of scores and probabilities, which pins
the ablation plumbing; each single ablation must not move the result away from
exact attention.  The measured numbers are printed (and quoted in the design
notes).  Source of the three quantized GEMM operands: "HiFA4: Training-Free
4-bit FlashAttention on Ascend HIF4 NPUs for LLM Inference", Abstract paras
1-2.
"""
import numpy as np
import pytest

import oracle
from bit_quantized_flashattention_smooth_b200 import workloads as W

ROWS = {"first": (0, 128), "middle": (2048, 2176), "last": (3968, 4096)}
HQ, HKV = 8, 2            # query heads 0..7 and their two kv heads (G = 4)


def _exact(q, k, v, r0, r1, scale):
    """fp64 causal softmax attention of rows [r0, r1) of every head."""
    G = q.shape[1] // k.shape[1]
    out = np.zeros((q.shape[1], r1 - r0, q.shape[-1]))
    for hq in range(q.shape[1]):
        S = q[0, hq, r0:r1].astype(np.float64) @ k[0, hq // G, :r1].astype(np.float64).T * scale
        mask = np.arange(r1)[None, :] <= np.arange(r0, r1)[:, None]
        S = np.where(mask, S, -np.inf)
        S -= S.max(-1, keepdims=True)
        P = np.exp(S)
        out[hq] = (P / P.sum(-1, keepdims=True)) @ v[0, hq // G, :r1].astype(np.float64)
    return out


def _metrics(o, ex):
    return (float(np.abs(o - ex).max() / np.abs(ex).max()),
            float(np.sum(o * ex) / (np.linalg.norm(o) * np.linalg.norm(ex))))


@pytest.mark.slow
def test_quantizer_ablation_on_qwen3_rows(capsys):
    w = W.WORKLOADS["qwen3_prefill"]
    q, k, v = W.make_prefill(w)
    q = q[:, :HQ].float().numpy()
    k = k[:, :HKV].float().numpy()
    v = v[:, :HKV].float().numpy()
    s, inv = oracle.calibrate(q[:, :, : w.n_cal], k[:, :, : w.n_cal], w.n_cal)
    qz = oracle.quantize_qkv(q, k, v, s, inv, oracle.NVFP4)
    scale = 1.0 / np.sqrt(w.d)
    G = HQ // HKV
    # the scores' raw operands: Smooth-QK'd Q and K in fp32, as they enter
    # the quantizer (Q K^T is unchanged by the rescale in exact arithmetic)
    q_s = (q * np.repeat(s, G, axis=0)[None, :, None, :]).astype(np.float32)
    k_s = (k * inv[None, :, None, :]).astype(np.float32)
    variants = {
        "4-bit (the method)": dict(),
        "scores unquantized": dict(raw=dict(q=q_s, k=k_s)),
        "P-hat = P": dict(variant=oracle.VAR_NO_PQUANT),
        "V unquantized": dict(raw=dict(v=v)),
        "all unquantized": dict(raw=dict(q=q_s, k=k_s, v=v), variant=oracle.VAR_NO_PQUANT),
    }
    table = {}
    for label, (r0, r1) in ROWS.items():
        ex = _exact(q, k, v, r0, r1, scale)
        for name, kw in variants.items():
            o = oracle.attention(qz, w.N, oracle.NVFP4, scale, True, oracle.PREORDER, w.block_n, rows=(r0, r1),
                                 **kw)["O"][0, :, r0:r1]
            table[(label, name)] = _metrics(o, ex)
    with capsys.disabled():
        print("\ndeviation from exact attention (max|dO|/max|O|, cosine), qwen3 heads 0-7:")
        for name in variants:
            print(f"  {name:22s} " + "  ".join(f"{lab}: {table[(lab, name)][0]:.4f} {table[(lab, name)][1]:.5f}"
                                                 for lab in ROWS))
    for lab in ROWS:
        full = table[(lab, "4-bit (the method)")][1]
        # everything off: exact attention up to fp32 scores and probabilities
        assert table[(lab, "all unquantized")][1] > 0.999999, lab
        for name in ("scores unquantized", "P-hat = P", "V unquantized"):
            assert table[(lab, name)][1] >= full - 1e-4, (lab, name, table[(lab, name)][1], full)
