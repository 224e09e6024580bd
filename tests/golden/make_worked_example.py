"""Writes worked_example_G2_T3_L2.json: a MoDA forward and backward whose
every value is an exact rational (or a rational multiple of ln 2), computed
here with Fraction arithmetic straight from the operator's definition (paper
summary of arXiv 2603.15619, section 3.4 "The Unified Operator": one softmax
scaled by 1/sqrt(d) over the causal keys j <= t and the token's own L depth
rows; query head h reads KV head floor(h / G), "moda-attention 0.1.0" PyPI
page, "Key Design Choices").  It imports neither the oracle nor the library.

Construction.  d = 16, so the scale 1/sqrt(d) is exactly 1/4.  Every query
is q = 4 ln2 * e0 and every key is k0 * e0 for a small integer k0, so each
score is s = ln2 * k0 and each softmax weight is 2**k0 / Z with Z an
integer.  Value rows are one-hot per attended item (sequence key j -> e_j,
depth row t*L + l -> e_(T + t*L + l)), so an output row lists its weights.
The backward reads dO[h, t] = e0 + e_(T + t*L) (plain FlashAttention-style
reading: D = rowsum(dO * O), dS = P * (dO v^T - D), dq = scale * sum dS k,
dk = scale * sum dS q, dv = sum P dO, the depth gradients token-local).
Since q = 4 ln2 e0 and scale = 1/4, dk and dkd equal ln2 * (sum of dS) in
dimension 0; they are stored as that rational coefficient of ln 2.

Run:  python tests/golden/make_worked_example.py
"""
import json
import os
from fractions import Fraction as F

B, Hq, Hk, T, L, d = 1, 4, 2, 3, 2, 16
G = Hq // Hk
SCALE = F(1, 4)
# exponent k0 of every key, per KV head: sequence keys j = 0..T-1 and depth
# rows in token-major order t*L + l
K_SEQ = {0: [0, 1, 2], 1: [2, 0, 1]}
K_DEP = {0: [1, 0, 2, 1, 0, 0], 1: [0, 2, 1, 1, 2, 0]}


def onehot(i):
    v = [F(0)] * d
    v[i] = F(1)
    return v


def main():
    O = [[[None] * T for _ in range(Hq)]]
    Z = [[[None] * T for _ in range(Hq)]]
    dQ0 = [[[F(0)] * T for _ in range(Hq)]]
    dK0 = [[[F(0)] * T for _ in range(Hk)]]            # coefficient of ln 2, dimension 0
    dV = [[[[F(0)] * d for _ in range(T)] for _ in range(Hk)]]
    dKd0 = [[[F(0)] * (T * L) for _ in range(Hk)]]     # coefficient of ln 2, dimension 0
    dVd = [[[[F(0)] * d for _ in range(T * L)] for _ in range(Hk)]]
    for h in range(Hq):
        kv = h // G
        for t in range(T):
            # attended items: (kind, index, k0, value row)
            items = [("seq", j, K_SEQ[kv][j], onehot(j)) for j in range(t + 1)]
            items += [("dep", t * L + l, K_DEP[kv][t * L + l], onehot(T + t * L + l)) for l in range(L)]
            z = sum(F(2) ** k for _, _, k, _ in items)
            p = [F(2) ** k / z for _, _, k, _ in items]
            o = [sum(pi * v[c] for pi, (_, _, _, v) in zip(p, items)) for c in range(d)]
            O[0][h][t], Z[0][h][t] = o, z
            do = onehot(0)
            do[T + t * L] += 1
            Drow = sum(a * b for a, b in zip(do, o))
            for pi, (kind, idx, k, v) in zip(p, items):
                ds = pi * (sum(a * b for a, b in zip(do, v)) - Drow)
                dQ0[0][h][t] += SCALE * ds * k                  # k = k0 * e0
                if kind == "seq":
                    dK0[0][kv][idx] += ds                       # scale * 4 ln2 = ln2
                    for c in range(d):
                        dV[0][kv][idx][c] += pi * do[c]
                else:
                    dKd0[0][kv][idx] += ds
                    for c in range(d):
                        dVd[0][kv][idx][c] += pi * do[c]

    def s(x):
        if isinstance(x, list):
            return [s(y) for y in x]
        return str(x)

    out = {
        "source": "operator definition (paper summary of arXiv 2603.15619, section 3.4); "
                  "GQA head map floor(h/G) (moda-attention PyPI page, Key Design Choices); "
                  "exact Fraction arithmetic, tests/golden/make_worked_example.py",
        "shape": {"B": B, "Hq": Hq, "Hk": Hk, "T": T, "L": L, "d": d},
        "q_dim0_over_ln2": 4,
        "k0_seq": [K_SEQ[k] for k in range(Hk)],
        "k0_dep": [K_DEP[k] for k in range(Hk)],
        "v": "sequence key j -> e_j; depth row t*L+l -> e_(T+t*L+l)",
        "dO": "e0 + e_(T+t*L) for every head and token",
        "O": s(O), "Z": s(Z),
        "dQ_dim0": s(dQ0), "dK_dim0_over_ln2": s(dK0), "dV": s(dV),
        "dKd_dim0_over_ln2": s(dKd0), "dVd": s(dVd),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "worked_example_G2_T3_L2.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")
    print(path)


if __name__ == "__main__":
    main()
