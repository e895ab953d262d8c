"""Write ``exact_small.json``: tiny problems solved in exact rational arithmetic.

The pages print no worked numeric example of the recurrence, so the stored
values here are the exact real results of its definition (Prizma "seq/delta.py"
module docstring: S_t = alpha_t S_{t-1} + u_t k_t^T, u_t = beta_t (v_t - alpha_t
S_{t-1} k_t), pre-write read o_t = S_{t-1} q_t; tiny_gdn/fugue.py
``BidirectionalGatedDeltaNet2`` docstring for the post-write read q_t^T S_t).
They are computed only through ``oracle.exact`` (product-of-transitions form in
``fractions.Fraction``).  Regenerate with ``python tests/golden/make_exact_golden.py``.
"""
from __future__ import annotations

import json
import os
import sys
from fractions import Fraction as F

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle.exact import forward_exact  # noqa: E402

# integer vectors in R^3 with integer length (so L2 normalisation stays rational)
PYTH3 = [(1, 2, 2), (2, 1, 2), (2, 2, 1), (2, 3, 6), (3, 6, 2), (6, 2, 3), (1, 4, 8),
         (4, 4, 7), (2, 6, 9), (0, 3, 4), (4, 0, 3), (-1, 2, -2), (2, -3, 6), (-6, 2, 3)]


def fs(x):
    return [str(v) for v in x] if isinstance(x, (list, tuple)) else str(x)


def case_post_plain():
    q = [[1, 0, 2], [0, 1, -1], [2, 1, 0], [1, 1, 1], [-1, 0, 1]]
    k = [[1, 2, 0], [0, 1, 1], [1, -1, 1], [2, 0, -1], [1, 1, 0]]
    v = [[1, -2], [3, 0], [0, 1], [-1, 1], [2, 2]]
    alpha = [F(1, 2), F(3, 4), F(7, 8), F(1), F(5, 8)]
    beta = [F(1, 3), F(1, 2), F(2, 3), F(1, 4), F(3, 5)]
    H0 = [[F(1, 10), 0], [0, F(-1, 5)], [F(1, 4), F(1, 8)]]
    return dict(name="post_plain_T5_dk3_dv2", read_mode="post", scale="1/2", qk_l2norm=False,
                q=q, k=k, v=v, alpha=alpha, beta=beta, H0=H0)


def case_pre_l2norm():
    q = [list(PYTH3[i]) for i in (0, 3, 6, 9, 12, 1)]
    k = [list(PYTH3[i]) for i in (4, 7, 10, 13, 2, 5)]
    v = [[1, 0, -1], [2, 1, 0], [0, -3, 1], [1, 1, 1], [-2, 0, 2], [0, 1, 0]]
    alpha = [F(9, 10), F(1, 2), F(3, 4), F(1), F(2, 3), F(4, 5)]
    beta = [F(1, 2), F(3, 2), F(1, 4), F(19, 10), F(1), F(2, 5)]  # beta up to 2 (negative eigenvalues)
    H0 = [[0, F(1, 3), 0], [F(-1, 2), 0, F(1, 7)], [0, 0, F(1, 9)]]
    return dict(name="pre_l2norm_T6_dk3_dv3", read_mode="pre", scale="1", qk_l2norm=True,
                q=q, k=k, v=v, alpha=alpha, beta=beta, H0=H0)


def case_repeated_key_floor():
    T = 6
    q = [list(PYTH3[i]) for i in range(T)]
    k = [list(PYTH3[3])] * T
    v = [[i + 1, -i] for i in range(T)]
    alpha = [F(1, 2)] * T
    beta = [F(1, 2), F(1, 3), F(1), F(1, 4), F(2, 3), F(1, 5)]
    H0 = [[0, 0], [0, 0], [0, 0]]
    return dict(name="post_repeated_key_alpha_half_T6", read_mode="post", scale="1/3",
                qk_l2norm=True, q=q, k=k, v=v, alpha=alpha, beta=beta, H0=H0)


def main():
    cases = []
    for c in (case_post_plain(), case_pre_l2norm(), case_repeated_key_floor()):
        o, HT = forward_exact(c["q"], c["k"], c["v"], c["alpha"], c["beta"], c["H0"],
                              read_mode=c["read_mode"], scale=F(c["scale"]),
                              qk_l2norm=c["qk_l2norm"])
        cases.append({
            "name": c["name"], "read_mode": c["read_mode"], "scale": c["scale"],
            "qk_l2norm": c["qk_l2norm"],
            "q": [fs(r) for r in c["q"]], "k": [fs(r) for r in c["k"]],
            "v": [fs(r) for r in c["v"]], "alpha": fs(c["alpha"]), "beta": fs(c["beta"]),
            "H0": [fs(r) for r in c["H0"]],
            "o": [fs(r) for r in o], "H_final": [fs(r) for r in HT],
        })
    doc = {
        "source": "exact rational values of the gated delta-rule definition (Prizma seq/delta.py "
                  "module docstring; tiny_gdn/fugue.py BidirectionalGatedDeltaNet2 docstring for "
                  "the post-write read); the pages print no numeric worked example",
        "state_layout": "H = S^T, [dk][dv]",
        "cases": cases,
    }
    with open(os.path.join(HERE, "exact_small.json"), "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
