"""Write tests/golden/tiny_layer.json from the oracle alone (regression fixture).

The Olmo-core 3 pages print no worked numeric example of the MoE layer, so the
only stored values here are the oracle's own, on a seeded 6-token, 4-expert, top-2
case; they guard the oracle against accidental change.  Run:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402


def case():
    rng = np.random.default_rng(2026)
    T, d, E, k, f = 6, 8, 4, 2, 4
    x = np.round(rng.standard_normal((T, d)), 3)
    W13 = np.round(rng.standard_normal((E, 2 * f, d)) * 0.3, 3)
    W2 = np.round(rng.standard_normal((E, d, f)) * 0.3, 3)
    L = np.round(rng.standard_normal((T, E)), 3).astype(np.float32)
    dy = np.round(rng.standard_normal((T, d)), 3)
    return dict(T=T, d=d, E=E, k=k, f=f, x=x, W13=W13, W2=W2, logits=L, dy=dy)


def main():
    c = case()
    fwd = oracle.layer_fwd(c["x"], c["W13"], c["W2"], logits=c["logits"], k=c["k"])
    bwd = oracle.layer_bwd(fwd, c["dy"], c["x"], c["W13"], c["W2"])
    out = dict(
        note="written by tests/golden/make_golden.py from oracle/ only",
        topk_idx=fwd["topk_idx"].tolist(), gates=fwd["gates"].tolist(),
        offsets=fwd["offsets"].tolist(), slot=fwd["slot"].tolist(),
        y=fwd["y"].tolist(), dx=bwd["dx"].tolist(), d_logits=bwd["d_logits"].tolist(),
        dW2_sum=float(bwd["dW2"].sum()), dW13_sum=float(bwd["dW13"].sum()))
    with open(os.path.join(HERE, "tiny_layer.json"), "w") as fh:
        json.dump(out, fh, indent=1)


if __name__ == "__main__":
    main()
