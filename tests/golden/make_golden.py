"""Writes ``exact_tiny.json``: exact rational results of tiny RDA problems.

The stored values come from ``oracle.exact`` only (exact ``Fraction``
arithmetic of the token-sequential recurrence, cross-checked here against the
hand-expanded closed form before anything is written).  The inputs are small
dyadic rationals, so every alpha is exactly ``2**-m`` and log(alpha) is
``-m ln 2``.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import random
import sys
from fractions import Fraction

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import exact  # noqa: E402


def _rand_frac(rng, den=8, lo=-8, hi=8):
    return Fraction(rng.randint(lo, hi), den)


def make_case(seed, T, Dk, Dv, with_s0, with_gamma):
    rng = random.Random(seed)
    q = [[_rand_frac(rng) for _ in range(Dk)] for _ in range(T)]
    k = [[_rand_frac(rng) for _ in range(Dk)] for _ in range(T)]
    v = [[_rand_frac(rng) for _ in range(Dv)] for _ in range(T)]
    alpha_exp = [rng.randint(0, 2) for _ in range(T)]            # alpha = 2^-m
    alpha = [Fraction(1, 2 ** m) for m in alpha_exp]
    beta = [Fraction(rng.randint(0, 4), 4) for _ in range(T)]
    gamma = [Fraction(rng.randint(2, 6), 4) for _ in range(T)] if with_gamma else None
    S0 = ([[_rand_frac(rng) for _ in range(Dk)] for _ in range(Dv)] if with_s0 else None)
    outs, S = exact.sequential(q, k, v, alpha, beta, S0=S0, gamma=gamma)
    assert S == exact.closed_form(k, v, alpha, beta, S0=S0, gamma=gamma)
    enc = lambda m: [[str(x) for x in r] for r in m]
    return {
        "seed": seed, "T": T, "Dk": Dk, "Dv": Dv,
        "q": enc(q), "k": enc(k), "v": enc(v),
        "alpha_log2": [-m for m in alpha_exp],
        "beta": [str(x) for x in beta],
        "gamma": None if gamma is None else [str(x) for x in gamma],
        "S0": None if S0 is None else enc(S0),
        "out": enc(outs),
        "S_final": enc(S),
    }


def main():
    cases = [
        make_case(11, 1, 1, 1, False, False),
        make_case(12, 3, 2, 2, True, False),
        make_case(13, 5, 3, 2, True, True),
        make_case(14, 8, 4, 4, True, True),
        make_case(15, 8, 4, 3, False, True),
        make_case(16, 6, 2, 4, True, False),
    ]
    doc = {
        "what": "exact rational results of the RDA gated delta rule on tiny inputs",
        "source": "oracle.exact.sequential, checked equal to oracle.exact.closed_form",
        "layout": "per case: q,k [T][Dk], v [T][Dv], S0 and S_final [Dv][Dk] (math "
                  "orientation), out [T][Dv]; alpha = 2**alpha_log2",
        "cases": cases,
    }
    with open(os.path.join(HERE, "exact_tiny.json"), "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
