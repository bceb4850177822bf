"""Writes tests/golden/tiny_case.json from the CPU oracle alone.

Run from the repository root:  python tests/golden/make_golden.py
The inputs are drawn here with a fixed NumPy seed; every expected value comes
from oracle.rkl_oracle (nothing from the CUDA path).
"""
import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
from oracle import rkl_oracle as O  # noqa: E402


def main():
    rs = np.random.RandomState(4242)
    B, Sm1, H, V = 2, 3, 4, 6
    h_s = np.round(rs.normal(size=(B * Sm1, H)), 3)
    h_t = np.round(rs.normal(size=(B * Sm1, H)), 3)
    W_s = np.round(rs.normal(size=(V, H)), 3)
    W_t = np.round(rs.normal(size=(V, H)), 3)
    mask = np.array([[0, 1, 1], [1, 0, 1]], dtype=np.uint8)
    red = O.REDUCE_SEQ_MEAN_NESTED
    out = O.forward(h_s, W_s, h_t, W_t, mask, red)
    dH, dW = O.backward(h_s, W_s, h_t, W_t, mask, red)
    g = {
        "note": "oracle outputs for a tiny hidden-payload case, nested per-sequence mean",
        "reduction": red,
        "inputs": {"h_s": h_s.tolist(), "h_t": h_t.tolist(), "W_s": W_s.tolist(),
                   "W_t": W_t.tolist(), "mask": mask.tolist()},
        "loss_tok": out["loss_tok"].tolist(), "loss": out["loss"],
        "dH_s": dH.tolist(), "dW_s": dW.tolist(),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_case.json")
    with open(path, "w") as f:
        json.dump(g, f, indent=1)


if __name__ == "__main__":
    main()
