"""Write the oracle regression fixture tests/golden/oracle_tiny_d4_T10.json.

The pages print no worked numeric example, so the stored values here are the
oracle's own output on a tiny seeded input (d_k = d_v = 4, T = 10, H = 2); they
guard against unintended edits to the oracle, and are not a pin of the oracle's
correctness (tests/test_oracle.py holds those).  This script calls only oracle/.
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402


def main():
    rng = np.random.default_rng(2025)
    B, T, H, d = 1, 10, 2, 4
    q = rng.standard_normal((B, T, H, d))
    k = rng.standard_normal((B, T, H, d))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, d))
    la = -np.log1p(np.exp(rng.standard_normal((B, T, H, d))))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H))))
    h0 = rng.standard_normal((B, H, d, d))
    o, hT = oracle.recurrent(q, k, v, la, beta, h0)
    out = {
        "source": "oracle.recurrent on a seeded numpy input (default_rng(2025)); written by make_golden.py",
        "inputs": {"q": q.tolist(), "k": k.tolist(), "v": v.tolist(), "log_alpha": la.tolist(),
                   "beta": beta.tolist(), "h0": h0.tolist()},
        "o": o.tolist(), "h_T": hT.tolist(),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_d4_T10.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=0)
    print(path)


if __name__ == "__main__":
    main()
