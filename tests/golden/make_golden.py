"""Writes tests/golden/tiny_oracle.json from the fp64 oracle (oracle/ only).

The pages print no numeric MLA result, so the stored values are the oracle's
own, on the seeded 'tiny' workload (B=1, Sq=1, H=16, L=256, bf16 N(0,1)):
all 16 LSE values and 64 sampled output elements, and the same for its FP8
cache (tiny_fp8_oracle.json).  The fixtures guard the oracle against silent drift; its correctness rests on the pins in
tests/oracle_pins.py.  Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from mla_decode_attention_11_b200 import workloads as W  # noqa: E402


def main():
    w = W.WORKLOADS["tiny"]
    q, kv, sl = W.generate(w)
    out, lse = oracle.mla_decode(q, kv, sl, w.scale)
    rng = np.random.default_rng(2024)
    idx = np.sort(rng.choice(out.size, size=64, replace=False))
    gold = {
        "workload": w.name,
        "note": "written by tests/golden/make_golden.py from oracle/ only",
        "lse": [float(x) for x in lse.reshape(-1)],
        "out_index": [int(i) for i in idx],
        "out_value": [float(x) for x in out.reshape(-1)[idx]],
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json"), "w") as f:
        json.dump(gold, f, indent=1)

    # the same workload over its FP8 (E4M3) cache
    q8, codes, ks, sl8 = W.generate_fp8(w)
    out8, lse8 = oracle.mla_decode_fp8(q8, codes, ks, sl8, w.scale)
    gold8 = {
        "workload": w.name,
        "kv_scale": ks,
        "note": "written by tests/golden/make_golden.py from oracle/ only (FP8 cache)",
        "lse": [float(x) for x in lse8.reshape(-1)],
        "out_index": [int(i) for i in idx],
        "out_value": [float(x) for x in out8.reshape(-1)[idx]],
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_fp8_oracle.json"), "w") as f:
        json.dump(gold8, f, indent=1)


if __name__ == "__main__":
    main()
