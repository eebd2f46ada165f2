"""Writes the hand-derived closed-form fixtures in this folder.

The values come from closed-form mathematics written out below (no oracle
call, no GPU): the inverse p-th root of [[2, 1], [1, 2]] from its
eigendecomposition, and the first Shampoo step for a rank-1 gradient.
Run from the repository root: ``python tests/golden/derive_closed_forms.py``.
"""
import json
import os

HERE = os.path.dirname(os.path.abspath(__file__))


def main():
    r4 = 3 ** -0.25
    r2 = 3 ** -0.5
    root = {
        "what": "Exact inverse p-th root of A = [[2,1],[1,2]] with eps = 0, derived by hand",
        "citation": "\"Shampoo optimizer\" notes, simplified matrix-case listing (L^(-1/4)); "
                    "SOAP abstract excerpt (1/2 power). Values from the eigendecomposition "
                    "A = Q diag(3, 1) Q^T, Q = [[1,1],[1,-1]]/sqrt(2), so A^(-1/p) = "
                    "1/2 [[3^(-1/p)+1, 3^(-1/p)-1],[3^(-1/p)-1, 3^(-1/p)+1]]",
        "A": [[2.0, 1.0], [1.0, 2.0]],
        "eps": 0.0,
        "cases": [
            {"p": 4, "X": [[(r4 + 1) / 2, (r4 - 1) / 2], [(r4 - 1) / 2, (r4 + 1) / 2]]},
            {"p": 2, "X": [[(r2 + 1) / 2, (r2 - 1) / 2], [(r2 - 1) / 2, (r2 + 1) / 2]]},
        ],
    }
    step = {
        "what": "First Shampoo step from zero statistics for the rank-1 gradient "
                "G = u v^T, u = (3, 4), v = (1, 0)",
        "citation": "\"Shampoo optimizer\" notes, simplified matrix-case listing "
                    "(L += G G^T, R += G^T G, W -= eta L^(-1/4) G R^(-1/4)); podcast transcript "
                    "'Preconditioned optimization without the full matrix cost', cue 20. "
                    "Hand derivation: L + eps I has eigenvalues 25 + 11 = 36 on u/|u| and 11 "
                    "elsewhere, R + eps I likewise on v, so L^(-1/4) G R^(-1/4) = "
                    "5 * 36^(-1/4) * 36^(-1/4) * (u/5) v^T = (5/6) (u/5) v^T",
        "G": [[3.0, 0.0], [4.0, 0.0]],
        "eps": 11.0,
        "p": 4,
        "lr": 0.5,
        "beta_values": [1.0, 0.9, 0.0],
        "P": [[0.5, 0.0], [2.0 / 3.0, 0.0]],
        "W1_from_zero": [[-0.25, 0.0], [-1.0 / 3.0, 0.0]],
    }
    with open(os.path.join(HERE, "inverse_root_2x2.json"), "w") as f:
        json.dump(root, f, indent=1)
    with open(os.path.join(HERE, "first_step_rank1.json"), "w") as f:
        json.dump(step, f, indent=1)


if __name__ == "__main__":
    main()
