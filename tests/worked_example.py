"""Loader of the worked example in tests/golden (exact values from the
operator's definition, written by tests/golden/make_worked_example.py): its
inputs as float64 arrays (token-major depth) and its expected outputs."""
import json
import math
import os
from fractions import Fraction

import numpy as np

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "worked_example_G2_T3_L2.json")
LN2 = math.log(2.0)


def _num(a):
    return np.vectorize(lambda s: float(Fraction(s)), otypes=[np.float64])(np.array(a, dtype=object))


def load():
    """Inputs (float64, token-major depth) and expected outputs."""
    g = json.load(open(GOLD))
    s = g["shape"]
    B, Hq, Hk, T, L, d = s["B"], s["Hq"], s["Hk"], s["T"], s["L"], s["d"]
    Q = np.zeros((B, Hq, T, d))
    Q[..., 0] = g["q_dim0_over_ln2"] * LN2
    K = np.zeros((B, Hk, T, d))
    V = np.zeros((B, Hk, T, d))
    Kd = np.zeros((B, Hk, T * L, d))
    Vd = np.zeros((B, Hk, T * L, d))
    for kv in range(Hk):
        for j in range(T):
            K[0, kv, j, 0] = g["k0_seq"][kv][j]
            V[0, kv, j, j] = 1.0
        for r in range(T * L):
            Kd[0, kv, r, 0] = g["k0_dep"][kv][r]
            Vd[0, kv, r, T + r] = 1.0
    dO = np.zeros((B, Hq, T, d))
    dO[..., 0] = 1.0
    for t in range(T):
        dO[:, :, t, T + t * L] += 1.0
    exp = {"O": _num(g["O"]), "LSE": np.log(_num(g["Z"]))}
    for name, key, shp, ln2 in (("dQ", "dQ_dim0", Q.shape, False), ("dK", "dK_dim0_over_ln2", K.shape, True),
                                ("dKd", "dKd_dim0_over_ln2", Kd.shape, True)):
        a = np.zeros(shp)
        a[..., 0] = _num(g[key]) * (LN2 if ln2 else 1.0)
        exp[name] = a
    exp["dV"] = _num(g["dV"])
    exp["dVd"] = _num(g["dVd"])
    return dict(shape=s, Q=Q, K=K, V=V, Kd=Kd, Vd=Vd, dO=dO), exp
