"""Write oracle_tiny_fp32.json: the fp64 oracle's decode output on the seeded
tiny fp32 workload (B1, 2 heads, D64, S256, d16, k64).  Calls only oracle/ and
workloads/.  Run from the repository root:  python tests/golden/make_oracle_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import get_workload, generators as gen  # noqa: E402


def compute():
    w = get_workload("tiny-fp32")
    inp = gen.decode_inputs(w)
    P = np.stack([oracle.pca_basis(c)[0] for c in inp["calib"]]).astype(np.float32).astype(np.float64)
    K_hat = oracle.rotate_keys(inp["keys64"], P, w.dtype)
    r = oracle.loki_decode(inp["q64"], K_hat, inp["values64"], P, w.seq_len, w.d, w.k)
    dense = oracle.dense_decode(inp["q64"], K_hat, inp["values64"], P, w.seq_len)
    return w, r, dense


def main():
    w, r, dense = compute()
    doc = {
        "workload": w.name, "d": w.d, "k": w.k,
        "written_by": "tests/golden/make_oracle_golden.py (oracle only)",
        "idx": r["idx"].tolist(),
        "out": [[[float(f"{x:.17g}") for x in row] for row in b] for b in r["out"]],
        "dense_out": [[[float(f"{x:.17g}") for x in row] for row in b] for b in dense],
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_fp32.json"), "w") as f:
        json.dump(doc, f, indent=0)


if __name__ == "__main__":
    main()
