"""Writes tests/golden/exact_tiny.json: exact rational outputs of the KATA
causal forward on tiny integer inputs, computed by oracle/exact.py (Python
Fractions; no floating point).  The pages print no worked example, so these
fixtures pin the definition (gist.science summary of "Kernelized Linear
Attention: Breaking the Capacity Wall with Symmetric Cones", Technical summary
2.1 and 2.2) by exact arithmetic instead.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle.exact import forward_exact, forward_exact_mg  # noqa: E402

CASES = [
    # name, q, k, v (one head; T x d lists of small integers)
    ("T4_d2", [[1, 0], [1, 1], [0, 2], [-1, 1]], [[1, 1], [2, -1], [0, 1], [1, 3]],
     [[1, -2], [3, 0], [-1, 1], [2, 2]]),
    ("T5_d3_zero_query", [[1, 2, 0], [0, 0, 0], [1, -1, 1], [2, 0, -1], [0, 1, 1]],
     [[1, 0, 1], [0, 1, 0], [1, 1, -1], [-2, 1, 0], [1, -1, 2]],
     [[1], [-1], [2], [0], [3]]),
    ("T3_d1", [[2], [-1], [3]], [[1], [-2], [1]], [[4, -1], [0, 2], [1, 1]]),
]


# KATA-Mg cases (gist.science summary 2.3, "Variantes"; the reading of the
# design notes): name, g, q, k, v.  The first one is checkable by hand: with
# g = 2 each coordinate is its own factor, so the weights are q_1^2 k_1^2 +
# q_2^2 k_2^2: row 0 has weight 1 + 4 = 5, so y_0 = v_0 = 1; row 1 has weights
# 1 + 1 = 2 (key 0) and 4 + 1 = 5 (key 1), so y_1 = (2 * 1 + 5 * 3) / 7 = 17/7
# (one factor would give (q.k)^2 = 4 and 1, and y_1 = 7/5).
MG_CASES = [
    ("T2_d2_g2_by_hand", 2, [[1, 2], [1, 1]], [[1, 1], [2, -1]], [[1], [3]]),
    ("T5_d4_g2", 2, [[1, 0, 2, -1], [0, 1, 1, 1], [2, -1, 0, 0], [1, 1, -1, 2], [0, 0, 0, 1]],
     [[1, 2, 0, 1], [-1, 1, 1, 0], [0, 0, 2, 1], [1, -1, 1, 1], [2, 0, -1, 1]],
     [[1, -1], [2, 0], [0, 3], [-2, 1], [1, 1]]),
    ("T4_d6_g3", 3, [[1, 0, 1, 1, 0, -1], [0, 2, 0, 1, 1, 0], [1, 1, 1, 1, 1, 1], [0, 0, 0, 0, 2, 1]],
     [[1, 1, 0, 0, 1, 0], [0, 1, -1, 2, 0, 1], [1, 0, 0, 1, 1, -1], [2, -1, 1, 0, 0, 1]],
     [[1], [-1], [4], [2]]),
]


def main():
    out = []
    for name, q, k, v in CASES:
        y = forward_exact(q, k, v)
        out.append({"name": name, "q": q, "k": k, "v": v,
                    "y": [[f"{x.numerator}/{x.denominator}" for x in row] for row in y]})
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "exact_tiny.json")
    with open(path, "w") as f:
        json.dump({"source": "oracle/exact.py (Fractions) via tests/golden/make_golden.py",
                   "cases": out}, f, indent=1)
    print("wrote", path)
    out = []
    for name, g, q, k, v in MG_CASES:
        y = forward_exact_mg(q, k, v, g)
        out.append({"name": name, "g": g, "q": q, "k": k, "v": v,
                    "y": [[f"{x.numerator}/{x.denominator}" for x in row] for row in y]})
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "exact_mg_tiny.json")
    with open(path, "w") as f:
        json.dump({"source": "oracle/exact.py forward_exact_mg (Fractions) via "
                             "tests/golden/make_golden.py", "cases": out}, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
