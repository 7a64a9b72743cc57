"""Writes oracle_small.json: the fp64 oracle's outputs on one tiny hand-picked input.

The pages print no worked example, so nothing here comes from them.  The fixture is a
regression record of the oracle, written by this script from ``oracle/`` alone: a change
to the oracle's arithmetic shows up as a mismatch in tests/test_golden.py and has to be
justified (and the fixture rewritten) on purpose.  It is not a pin; the pins are in
tests/pins.py.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402

G_MIN = -5.0


def fixture_inputs():
    """B1 T5 H1 d4, dyadic values (exact in float32)."""
    q = np.array([[1, 0, 0, 0], [0, 1, 0, 0], [0.5, 0.5, 0, 0], [0, 0, 1, 0], [0.25, -0.5, 0.5, 0.25]],
                 np.float32)
    k = np.array([[0, 1, 0, 0], [1, 0, 0, 0], [0.5, 0, 0.5, 0], [0, 0, 0, 1], [0.5, 0.5, -0.5, 0.5]], np.float32)
    v = np.array([[1, 2, 0, -1], [0.5, 0, 1, 0], [-1, 0.25, 0, 2], [0, 1, 1, 1], [2, -1, 0.5, 0]], np.float32)
    a = np.array([[0, 1, -1, 2], [-2, 0, 0.5, 1], [4, -4, 0, 0], [1, 1, 1, 1], [-8, 8, 0.25, -0.25]], np.float32)
    beta = np.array([0.5, 0.25, 0.75, 1.0, 0.125], np.float32)
    dO = np.array([[1, 0, 0, 0], [0, -1, 0, 0], [0.5, 0.5, 0.5, 0.5], [0, 0, 2, 0], [-1, 1, -1, 1]], np.float32)
    S0 = (np.arange(16, dtype=np.float64).reshape(4, 4) - 7.5) / 8.0
    dST = np.eye(4) * 0.5
    shape = lambda x: x.reshape(1, 5, 1, -1)  # noqa: E731
    return dict(q=shape(q), k=shape(k), v=shape(v), a=shape(a), beta=beta.reshape(1, 5, 1), dO=shape(dO),
                S0=S0.reshape(1, 1, 4, 4), dST=dST.reshape(1, 1, 4, 4))


def compute():
    x = fixture_inputs()
    args = (x["q"], x["k"], x["v"], x["a"], x["beta"])
    o, S_T = oracle.recurrence(*args, G_MIN, S0=x["S0"])
    g = oracle.backward(*args, x["dO"], G_MIN, S0=x["S0"], dST=x["dST"])
    out = {"g": oracle.gate(x["a"], G_MIN).astype(np.float64), "o": o, "S_T": S_T}
    out.update({k: v for k, v in g.items()})
    return {k: np.asarray(v, np.float64).tolist() for k, v in out.items()}


if __name__ == "__main__":
    data = {"about": "fp64 oracle outputs (gate, recurrence, backward) for fixture_inputs() of "
                     "make_golden.py, g_min = -5; written by make_golden.py from oracle/ only",
            "g_min": G_MIN, "values": compute()}
    with open(os.path.join(HERE, "oracle_small.json"), "w") as f:
        json.dump(data, f, indent=1)
