"""Writes the exact rational KDA fixtures in this folder.

Calls only oracle/exact.py (the definition as an explicit product of rational
matrices, exact arithmetic). Run from the repository root:
    python tests/golden/make_golden.py
Each fixture records its inputs and the exact outputs o_t and states S_t as
"p/q" strings. Citation: Kimi K3 technical FAQ (runpod.io), "What is KDA, and
why does a serving engineer care?" -- delta-rule recurrence with a per-channel
forget gate and a d_k x d_v state, in the standard gated-delta form
S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
o_t = S_t^T q_t / sqrt(d_k). The pages print no worked example; these are
hand-chosen rational cases.
"""
from __future__ import annotations

import json
import sys
from fractions import Fraction as F
from pathlib import Path

ROOT = Path(__file__).resolve().parents[2]
sys.path.insert(0, str(ROOT))
from oracle.exact import kda_exact  # noqa: E402

HERE = Path(__file__).resolve().parent


def s(x):
    return f"{x.numerator}/{x.denominator}"


def mat(m):
    return [[s(x) for x in row] for row in m]


# All inputs are dyadic rationals, so q, k, v, beta and S_0 are exact in fp32
# (the oracles' input type); only g = log(alpha) is rounded when it is formed.
# Unit-norm dyadic keys: (1/2)(+-1, +-1, +-1, +-1) and signed basis vectors.
UNIT_KEYS = [
    [F(1, 2), F(1, 2), F(1, 2), F(1, 2)],
    [F(1, 2), F(-1, 2), F(1, 2), F(-1, 2)],
    [F(0), F(1), F(0), F(0)],
    [F(-1, 2), F(-1, 2), F(1, 2), F(1, 2)],
    [F(1, 2), F(1, 2), F(1, 2), F(1, 2)],
    [F(0), F(0), F(0), F(-1)],
    [F(1, 2), F(-1, 2), F(-1, 2), F(1, 2)],
    [F(1), F(0), F(0), F(0)],
]


def case(name, keys, alpha, beta, q, v, s0, note):
    T = len(keys)
    o, S = kda_exact(q, keys, v, alpha, beta, s0, F(1, 2))
    return {
        "name": name,
        "note": note,
        "citation": "Kimi K3 technical FAQ (runpod.io), 'What is KDA, and why does a serving "
                    "engineer care?'; standard gated-delta form of the recurrence",
        "T": T, "dk": 4, "dv": 4, "scale": "1/2",
        "q": mat(q), "k": mat(keys), "v": mat(v), "alpha": mat(alpha),
        "beta": [s(b) for b in beta], "s0": mat(s0),
        "o": mat(o), "states": [mat(St) for St in S],
    }


def main():
    T = 8
    alpha = [[F(1, 1) if (t + c) % 4 == 0 else F(9 + ((t * 3 + c) % 5), 16) for c in range(4)]
             for t in range(T)]
    beta = [F(1, 2), F(3, 4), F(1, 8), F(7, 8), F(5, 8), F(1, 1), F(13, 16), F(3, 8)]
    q = [[F(((t * 5 + c * 3) % 7) - 3, 4) for c in range(4)] for t in range(T)]
    v = [[F(((t * 7 + c * 2) % 9) - 4, 4) for c in range(4)] for t in range(T)]
    zero = [[F(0)] * 4 for _ in range(4)]
    s0 = [[F(((i * 4 + j) % 7) - 3, 8) for j in range(4)] for i in range(4)]
    gen_keys = [[F(((t * 3 + c * 5) % 11) - 5, 8) for c in range(4)] for t in range(T)]
    cases = [
        case("unit_keys_zero_state", UNIT_KEYS, alpha, beta, q, v, zero,
             "unit-norm keys, mixed gates (alpha = 1 on some channels), S_0 = 0"),
        case("unit_keys_state", UNIT_KEYS, alpha, beta, q, v, s0,
             "unit-norm keys, mixed gates, nonzero S_0"),
        case("generic_keys_state", gen_keys, alpha, beta, q, v, s0,
             "keys not normalised (the definition does not need it), nonzero S_0"),
    ]
    out = HERE / "exact_product_T8_d4.json"
    out.write_text(json.dumps({"generator": "tests/golden/make_golden.py",
                               "cases": cases}, indent=1))
    print("wrote", out)


if __name__ == "__main__":
    main()
