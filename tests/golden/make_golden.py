"""Writes the stored expected values under tests/golden/ (oracle only).

The pages print no numeric worked example, so every stored value here comes
from the fp64 oracle (``oracle/``) on a seeded synthetic input; nothing comes
from the CUDA path. Run:  python tests/golden/make_golden.py
"""

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from exact_attention_151_b200.inputs import WORKLOADS, bits, make_qkv  # noqa: E402


def main():
    w = WORKLOADS["small_b1h2n256d64"]
    q, k, v = make_qkv(w)
    rows = [(0, h, i) for h in range(w.H) for i in list(range(0, w.N, 17)) + [w.N - 1]]
    o, lse = oracle.attention_rows(bits(q), bits(k), bits(v), w.softmax_scale, w.causal, w.dtype, rows)
    doc = {
        "what": "oracle O and LSE rows for the small configuration B=1 H=2 N=256 D=64 bf16 N(0,1) seed 0, "
                "scale 1/sqrt(64), non-causal; inputs from exact_attention_151_b200.inputs.make_qkv",
        "source": "oracle/attention_oracle.cpp (fp64 definition); written by tests/golden/make_golden.py",
        "workload": w.name,
        "rows": rows,
        "o": [[float.hex(float(x)) for x in r] for r in o],
        "lse": [float.hex(float(x)) for x in lse],
    }
    with open(os.path.join(HERE, "small_b1h2n256d64_rows.json"), "w") as f:
        json.dump(doc, f, indent=0)


if __name__ == "__main__":
    main()
