"""Writes roots_2x2.json: inverse p-th roots of 2x2 matrices [[a, b], [b, a]]
from their closed form.

The matrix has eigenvectors (1, 1)/sqrt(2) and (1, -1)/sqrt(2) with
eigenvalues a + b and a - b, so (A + eps I)^{-1/p} = [[h, k], [k, h]] with
u = (a + b + eps)^{-1/p}, v = (a - b + eps)^{-1/p}, h = (u + v)/2,
k = (u - v)/2.  Nothing here calls the oracle or the CUDA library: the
values are the closed form itself, written out in plain Python floats.
The pages ("Scalable Second Order Optimization for Deep Learning") print no
worked example; these cases pin the oracle's root to the mathematics.
"""
import json
import os

CASES = [(2.0, 1.0, 0.0, 4), (2.0, 1.0, 0.0, 2), (5.0, -3.0, 1e-6, 4),
         (1e-4, 5e-5, 1e-6, 4), (3.0, 0.0, 0.5, 8)]

out = []
for a, b, eps, p in CASES:
    u = (a + b + eps) ** (-1.0 / p)
    v = (a - b + eps) ** (-1.0 / p)
    h, k = (u + v) / 2.0, (u - v) / 2.0
    out.append({"A": [[a, b], [b, a]], "eps": eps, "p": p, "X": [[h, k], [k, h]]})

path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "roots_2x2.json")
with open(path, "w") as f:
    json.dump({"source": "closed form of the 2x2 symmetric root; see make_roots_2x2.py",
               "cases": out}, f, indent=1)
