"""The oracle still reproduces its committed regression fixture (written by tests/golden/make_golden.py)."""
import json
import os

import numpy as np

import oracle
import synth

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_oracle.json")


def test_tiny_fixture():
    doc = json.load(open(GOLD))
    cfg = synth.CONFIGS["tiny"]
    inp = synth.make_inputs(cfg)
    f = oracle.forward(inp.x, inp.Wg, inp.bg, inp.W1, inp.b1, inp.W2, inp.b2, cfg.k, cfg.CF, cfg.dtype,
                       tokens=np.array(doc["tokens"], np.int32))
    assert f.routing.topk_idx.tolist() == doc["topk_idx"]
    np.testing.assert_allclose(f.routing.topk_w[:8], doc["topk_w_first8"], rtol=1e-14)
    assert f.disp.expert_counts.tolist() == doc["expert_counts"]
    assert abs(f.aux - doc["aux"]) <= 1e-14 * abs(doc["aux"]) and abs(f.z - doc["z"]) <= 1e-14 * abs(doc["z"])
    np.testing.assert_allclose(f.out, doc["out_rows"], rtol=1e-12, atol=1e-14)
