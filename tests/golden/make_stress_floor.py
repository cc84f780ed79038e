"""Writes stress_lse_floor.json: the LSE error floor of FP16 attention
operands on the massive-activation workload (HF discussion #26 on
RecursiveSI/flint, massive activations), over every query row.

The floor is the largest |lse(q~, k~ rounded to FP16) - lse(exact)| of the
FP64 oracle: what any kernel that feeds FP16 normalised Q/K to its QK^T
product carries at best.  Only the oracle is called.

    python tests/golden/make_stress_floor.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
import workloads as W  # noqa: E402


def main():
    w = W.make("stress_full_4x8192_pad")
    rows = np.arange(w.T)
    _, exact = oracle.attn_fwd_workload(w, rows=rows)
    _, fp16 = oracle.attn_fwd_workload(w, rows=rows, qk_round=2)
    _, bf16 = oracle.attn_fwd_workload(w, rows=rows, qk_round=1)
    fin = np.isfinite(exact)
    rec = dict(workload=w.name, rows=int(w.T),
               lse_floor_fp16=float(np.abs(fp16[fin] - exact[fin]).max()),
               lse_floor_bf16=float(np.abs(bf16[fin] - exact[fin]).max()),
               note="oracle with normalised, rotated Q/K rounded to FP16 (BF16) vs exact FP64, all rows")
    with open(os.path.join(HERE, "stress_lse_floor.json"), "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    print(rec)


if __name__ == "__main__":
    main()
