"""Writes tests/golden/oracle_tiny.json: the oracle's outputs on a small seeded
case (both formats, both normalizer modes, exact and lazy running max), so that
any later change to the oracle's arithmetic shows up as a diff of this file.
Calls only oracle/; run `python tests/golden/make_golden.py` from the repo root
after a deliberate change, and name in the commit the passage (or its reading)
that justifies it."""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402

CASES = [
    # fmt, mode, tau
    (oracle.NVFP4, oracle.PREORDER, 0.0),
    (oracle.NVFP4, oracle.INCONSISTENT, 0.0),
    (oracle.MXFP4, oracle.PREORDER, 0.0),
    (oracle.NVFP4, oracle.PREORDER, 3.0),
]
B, HQ, HKV, N, D, BN = 1, 2, 1, 48, 32, 16
ROWS = (0, 17, 47)


def inputs():
    rng = np.random.default_rng(2026)
    q = rng.standard_normal((B, HQ, N, D)).astype(np.float32)
    k = rng.standard_normal((B, HKV, N, D)).astype(np.float32)
    v = rng.standard_normal((B, HKV, N, D)).astype(np.float32)
    k[..., -2:] = 12 * np.abs(k[..., -2:])
    return q, k, v


def compute():
    q, k, v = inputs()
    s, inv = oracle.calibrate(q, k, n_cal=16, alpha=0.5)
    out = {"shape": [B, HQ, HKV, N, D], "block_n": BN, "rows": list(ROWS), "cases": []}
    for fmt, mode, tau in CASES:
        qz = oracle.quantize_qkv(q, k, v, s, inv, fmt)
        r = oracle.attention(qz, N, fmt, 1.0 / np.sqrt(D), True, mode, 32 if fmt == oracle.MXFP4 else BN, tau=tau)
        out["cases"].append({
            "fmt": int(fmt), "mode": int(mode), "tau": tau,
            "O": [[r["O"][0, h, i].tolist() for i in ROWS] for h in range(HQ)],
            "lse": [[float(r["lse"][0, h, i]) for i in ROWS] for h in range(HQ)],
        })
    return out


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json")
    with open(path, "w") as f:
        json.dump(compute(), f, indent=0)
        f.write("\n")
    print("wrote", path)
