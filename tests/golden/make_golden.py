"""Writes tests/golden/tiny_oracle.json from the CPU oracle alone.

The pages print no worked numeric example, so this file is a regression record of the
oracle on the tiny workload (B=1, H=1, L=256, D=64, fp16, 64x64 tiles, INT8, bitmask routing
with Bernoulli(0.25) FP16 bits); it never takes a value from the CUDA path.
Run: python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
from workloads import CONFIGS, make_workload  # noqa: E402


def main():
    w = CONFIGS["tiny"]
    t = make_workload(w)
    mask = oracle.build_mask(w.B, w.H, w.nqt, w.nkt, w.group_tiles, w.p_fp16, w.mask_seed)
    r = oracle.attention(t.q, t.k, t.v, bm=w.bm, bn=w.bn, mask=mask, group_tiles=w.group_tiles,
                         fmt=w.fmt, want_codes=True)
    sel = [(0, 0, i, d) for i, d in [(0, 0), (17, 5), (63, 63), (64, 0), (128, 31), (255, 63)]]
    out = {
        "_about": __doc__.strip().splitlines()[0],
        "workload": "tiny",
        "mask": [str(int(x)) for x in mask.reshape(-1)],
        "route": r["route"].reshape(-1).tolist(),
        "q_scales": [float(x) for x in r["q_scales"].reshape(-1)],
        "k_scales": [float(x) for x in r["k_scales"].reshape(-1)],
        "q_code_sum": int(r["q_codes"].view(np.int8).astype(np.int64).sum()),
        "k_code_sum": int(r["k_codes"].view(np.int8).astype(np.int64).sum()),
        "lse": [float(x) for x in r["lse"].reshape(-1)],
        "o_samples": [[list(s), float(r["o"][s])] for s in sel],
        "o_abs_sum": float(np.abs(r["o"]).sum()),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
