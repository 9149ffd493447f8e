"""Write tests/golden/brute_tiny.json: an exact rational worked example.

The pages print no worked numeric example, so the stored values come from the
exact brute force in ``oracle/brute.py`` (closed product of the affine maps
A_t = alpha_t (I - beta_t k_t k_t^T); no floating point anywhere).  This script
calls only ``oracle/``.  Regenerate with:  python tests/golden/make_golden.py
"""
import json
import os
import sys
from fractions import Fraction

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
from oracle import brute  # noqa: E402

F = Fraction
q = [[F(1, 2), F(-1, 4), F(3, 4)], [F(0), F(1), F(-1, 2)], [F(1, 4), F(1, 4), F(1, 2)],
     [F(-3, 4), F(1, 2), F(0)]]
k = [[F(1), F(0), F(0)], [F(1, 2), F(1, 2), F(-1, 2)], [F(0), F(3, 4), F(1, 4)],
     [F(-1, 4), F(0), F(1)]]
v = [[F(1), F(-2)], [F(1, 2), F(3, 2)], [F(-1), F(0)], [F(2), F(1, 4)]]
alpha = [F(1), F(3, 4), F(1, 2), F(7, 8)]
beta = [F(1, 2), F(3, 2), F(1), F(1, 4)]
S0 = [[F(1, 8), F(0), F(-1, 4)], [F(0), F(1, 2), F(1, 8)]]  # d_v x d_k

o, S_T = brute.solve(q, k, v, alpha, beta, S0)
s = lambda m: [[str(x) for x in row] for row in m]
out = {
    "source": "exact closed product of the delta-rule affine maps (oracle/brute.py); "
              "update of 'DeltaNet Attention' (class docstring) with the per-token decay "
              "of 'linear_attention' (LinearAttention)",
    "q": s(q), "k": s(k), "v": s(v), "alpha": [str(a) for a in alpha],
    "beta": [str(b) for b in beta], "S0": s(S0), "o": s(o), "S_T": s(S_T),
}
path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "brute_tiny.json")
with open(path, "w") as fh:
    json.dump(out, fh, indent=1)
print("wrote", path)
