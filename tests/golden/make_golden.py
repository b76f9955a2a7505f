"""Writes the oracle regression fixture ``tiny_oracle.json`` for the tiny fp32 layer workload.

Calls only the oracle and the seeded input generator; nothing here comes from the CUDA path.
Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402


def main():
    cfg = synth.CONFIGS["tiny"]
    inp = synth.make_inputs(cfg)
    tokens = np.array([0, 1, 2, 127, 255], np.int32)
    f = oracle.forward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, cfg.dtype, tokens=tokens)
    doc = {
        "what": "oracle outputs for the tiny fp32 layer (T=256,H=64,E=4,k=2,F=256, dropless, seed 1)",
        "writer": "tests/golden/make_golden.py (oracle + synth only)",
        "topk_idx": f.routing.topk_idx.tolist(),
        "topk_w_first8": f.routing.topk_w[:8].tolist(),
        "expert_counts": f.disp.expert_counts.tolist(),
        "aux": f.aux,
        "z": f.z,
        "tokens": tokens.tolist(),
        "out_rows": f.out.tolist(),
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json"), "w") as fh:
        json.dump(doc, fh)


if __name__ == "__main__":
    main()
