"""Writes tests/golden/kda_tiny.json: a tiny fixed KDA case and the oracle's outputs (o, the
final state, and the transition of the whole sequence).

The pages about the model print no worked numeric example for KDA, so this fixture is
a regression pin only: its inputs are small exact decimals chosen here, and its
expected values come from the fp64 oracle (this script calls nothing but ``oracle``).
Regenerate only when a change to the oracle's arithmetic is justified by the pages.
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)
import oracle  # noqa: E402


def case():
    T, H, dk, dv = 5, 1, 4, 3
    q = np.array([[0.5, 0.5, 0.5, 0.5], [0.6, 0.0, 0.8, 0.0], [0.0, 1.0, 0.0, 0.0],
                  [0.0, 0.6, 0.0, 0.8], [0.5, -0.5, 0.5, -0.5]]).reshape(T, H, dk)
    k = np.array([[1.0, 0.0, 0.0, 0.0], [0.0, 0.6, 0.8, 0.0], [0.5, 0.5, 0.5, 0.5],
                  [0.0, 0.0, 0.0, 1.0], [0.8, 0.0, 0.0, 0.6]]).reshape(T, H, dk)
    v = np.array([[1.0, -2.0, 0.5], [0.25, 1.5, -1.0], [2.0, 0.0, 1.0], [-0.5, 0.75, 0.125],
                  [1.0, 1.0, -1.0]]).reshape(T, H, dv)
    g = np.array([[-0.1, -0.2, -0.05, -0.5], [-0.1, -0.3, -0.01, -1.0], [-0.2, -0.2, -0.2, -0.2],
                  [0.0, -0.05, -0.4, -0.1], [-0.3, -0.1, -0.02, -0.6]]).reshape(T, H, dk)
    beta = np.array([0.5, 0.25, 0.75, 0.9, 0.1]).reshape(T, H)
    h0 = np.array([[0.1, 0.0, -0.1], [0.2, 0.3, 0.0], [0.0, -0.2, 0.1], [0.05, 0.05, 0.05]]
                  ).reshape(1, H, dk, dv)
    return dict(q=q, k=k, v=v, g=g, beta=beta, h0=h0, scale=0.5)


if __name__ == "__main__":
    c = case()
    o, ht = oracle.kda_fwd(c["q"], c["k"], c["v"], c["g"], c["beta"], c["scale"], c["h0"])
    m = oracle.transition(c["k"], c["g"], c["beta"])
    out = {k: np.asarray(v).tolist() for k, v in c.items() if k != "scale"}
    out.update(scale=c["scale"], o=o.tolist(), ht=ht.tolist(), m=m.tolist())
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "kda_tiny.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)
