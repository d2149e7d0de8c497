"""Regression guard: the oracle still produces its stored tiny-case values."""
import json
import os
import sys

import numpy as np

import oracle

sys.path.insert(0, os.path.join(os.path.dirname(__file__), "golden"))
from make_golden import case  # noqa: E402


def test_tiny_layer_regression():
    with open(os.path.join(os.path.dirname(__file__), "golden", "tiny_layer.json")) as fh:
        g = json.load(fh)
    c = case()
    fwd = oracle.layer_fwd(c["x"], c["W13"], c["W2"], logits=c["logits"], k=c["k"])
    bwd = oracle.layer_bwd(fwd, c["dy"], c["x"], c["W13"], c["W2"])
    assert fwd["topk_idx"].tolist() == g["topk_idx"]
    assert fwd["offsets"].tolist() == g["offsets"]
    assert fwd["slot"].tolist() == g["slot"]
    for name, got in (("gates", fwd["gates"]), ("y", fwd["y"]), ("dx", bwd["dx"]),
                      ("d_logits", bwd["d_logits"])):
        assert np.allclose(got, np.array(g[name]), rtol=1e-12, atol=1e-14), name
    assert np.isclose(bwd["dW2"].sum(), g["dW2_sum"], rtol=1e-12)
    assert np.isclose(bwd["dW13"].sum(), g["dW13_sum"], rtol=1e-12)
