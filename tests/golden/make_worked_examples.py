"""Writes worked_examples.json: hand-derived closed-form values that pin the oracle.

The EntmaxKV pages print no worked example, so each value below is derived by
hand from a textbook closed form (cited per entry) and evaluated with Python's
math module.  Nothing here calls the CUDA library or the oracle.
Run:  python tests/golden/make_worked_examples.py
"""
import json
import math
import os

s7 = math.sqrt(7.0)
EXAMPLES = {
    "_about": "Hand-derived worked examples used to pin the oracle. The EntmaxKV pages print no "
              "worked example, so every entry cites the closed form it was derived from; values "
              "were computed from those closed forms with Python's math module, not by the oracle.",
    "entmax": [
        {"name": "sparsemax three entries", "alpha": 2.0, "x": [1.0, 0.5, 0.0], "tau": 0.25,
         "p": [0.75, 0.25, 0.0],
         "cite": "alpha = 2 entmax is sparsemax, the Euclidean projection onto the simplex "
                 "(Martins and Astudillo 2016, Prop. 1): support {1,2}, tau = (1.0 + 0.5 - 1)/2"},
        {"name": "sparsemax tie", "alpha": 2.0, "x": [0.3, 0.3], "tau": -0.2, "p": [0.5, 0.5],
         "cite": "both entries in the support: 2 (0.3 - tau) = 1"},
        {"name": "1.5-entmax two entries", "alpha": 1.5, "x": [0.5, 0.0], "tau": (1.0 - s7) / 4.0,
         "p": [((1.0 + s7) / 4.0) ** 2, ((s7 - 1.0) / 4.0) ** 2],
         "cite": "both entries in the support: (0.5 - tau)^2 + tau^2 = 1, i.e. "
                 "2 tau^2 - tau - 0.75 = 0, smaller root (1 - sqrt 7)/4"},
        {"name": "1.5-entmax one-hot", "alpha": 1.5, "x": [1.5, 0.2, 0.1], "tau": 0.5,
         "p": [1.0, 0.0, 0.0],
         "cite": "support {1}: (1.5 - tau)^2 = 1 gives tau = 0.5 >= 0.2, so the other entries get zero"},
        {"name": "1.5-entmax uniform", "alpha": 1.5, "x": [0.0, 0.0, 0.0, 0.0], "tau": -0.5,
         "p": [0.25, 0.25, 0.25, 0.25],
         "cite": "all four equal entries in the support: 4 tau^2 = 1, smaller root -1/2"},
    ],
    "gauss_g": [
        {"alpha": 2.0, "m": 0.0, "s": 1.0, "tau": 0.0, "g": 1.0 / math.sqrt(2.0 * math.pi),
         "cite": "E[X_+] for X ~ N(0,1) is phi(0) = 1/sqrt(2 pi)"},
        {"alpha": 1.5, "m": 0.0, "s": 1.0, "tau": 0.0, "g": 0.5,
         "cite": "E[X_+^2] for X ~ N(0,1) is half of E[X^2] = 1/2 by symmetry"},
        {"alpha": 2.0, "m": 1.0, "s": 0.0, "tau": 0.25, "g": 0.75, "cite": "a point mass: (1 - 0.25)_+"},
        {"alpha": 1.5, "m": 1.0, "s": 0.0, "tau": 0.25, "g": 0.5625,
         "cite": "a point mass: (1 - 0.25)_+^2"},
        {"alpha": 2.0, "m": 0.0, "s": 2.0, "tau": 0.0, "g": 2.0 / math.sqrt(2.0 * math.pi),
         "cite": "E[X_+] for X ~ N(0, 4) is 2 phi(0)"},
    ],
    "z_table": [
        {"n": 1, "z": 0.0, "cite": "one token: the page maximum is the token itself"},
        {"n": 2, "z": math.sqrt(2.0 * math.log(2.0)), "cite": "sqrt(2 ln 2)"},
        {"n": 64, "z": math.sqrt(2.0 * math.log(64.0)), "cite": "sqrt(2 ln 64)"},
    ],
    "welford": [
        {"tokens": [1.0, 2.0, 4.0], "mean": 7.0 / 3.0, "var": 14.0 / 9.0,
         "cite": "population variance ((4/3)^2 + (1/3)^2 + (5/3)^2) / 3 = 14/9"},
    ],
    "bbox": [
        {"q": [1.0, -2.0], "kmin": [0.0, -1.0], "kmax": [2.0, 3.0], "scale": 1.0, "ub": 4.0,
         "corner_key": [2.0, -1.0],
         "cite": "max over the box of q.k picks k_max where q >= 0 and k_min where q < 0: "
                 "1*2 + (-2)*(-1) = 4, attained by the corner (2, -1)"},
    ],
}

if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "worked_examples.json")
    with open(out, "w") as f:
        json.dump(EXAMPLES, f, indent=1)
    print("wrote", out)
