"""Write tests/golden/oracle_tiny.json from the oracle (and only the oracle).

Run: python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from mla_flash_attention_attn_b200 import workloads as W  # noqa: E402


def main():
    w = W.make("v2lite_decode", n_kv=24, n_head=2, n_pad=5)
    out = oracle.attention(w.q[0], w.kcache[0], mask=w.mask[0], scale=w.scale)
    rec = {
        "what": "oracle output, v2lite_decode recipe at n_kv=24, n_head=2, n_pad=5, seed 1002",
        "writer": "tests/golden/make_golden.py (calls only oracle/ and the generators)",
        "rows": 2,
        "cols_sampled": [0, 1, 17, 255, 511],
        "values": [[repr(float(out[r, c])) for c in (0, 1, 17, 255, 511)] for r in range(2)],
    }
    with open(os.path.join(HERE, "oracle_tiny.json"), "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
