"""Write oracle_small_case.json: a seeded regression case for the oracle.

Calls only the oracle (and the seeded input generators); nothing here comes
from the CUDA path.  Re-run only when the oracle's arithmetic changes for a
reason stated in the commit message.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from ternary_weight_bit_bitlinear_b200 import inputs  # noqa: E402


def main():
    M, K, N = 16, 48, 3
    W = inputs.latent_weights(M, K, seed=4242).numpy()
    x = inputs.activations(N, K, seed=4243, outlier_count=2).numpy()
    out = oracle.bitlinear(W, x)
    case = {
        "_about": "Seeded small layer (M=16, K=48, N=3) through the oracle; written by make_golden.py.",
        "M": M, "K": K, "N": N,
        "W": [float(v) for v in W.ravel()],
        "x": [float(v) for v in x.ravel()],
        "alpha": float(out["alpha"]),
        "packed": [int(v) for v in out["packed"].ravel()],
        "q": [int(v) for v in out["q"].ravel()],
        "acc": [int(v) for v in out["acc"].ravel()],
        "y": [float(v) for v in out["y"].ravel()],
    }
    with open(os.path.join(HERE, "oracle_small_case.json"), "w") as f:
        json.dump(case, f)


if __name__ == "__main__":
    main()
