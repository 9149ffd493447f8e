"""Write tests/golden/brute_tiny.json and brute_channel_gates.json: exact rational examples.

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

# Per-key-channel gates ("linear_attention", ChannelGates) and the state after every two
# tokens: the same tokens, one decay per key channel, each prefix solved exactly.
alpha_c = [[F(1), F(1, 2), F(3, 4)], [F(7, 8), F(1), F(1, 4)], [F(1, 2), F(5, 8), F(1)],
           [F(3, 4), F(3, 8), F(7, 8)]]
o_c, S_c = brute.solve(q, k, v, alpha_c, beta, S0)
prefix = [brute.solve(q[:e], k[:e], v[:e], alpha_c[:e], beta[:e], S0)[1] for e in (2, 4)]
out_c = {
    "source": "exact closed product of A_t = diag(alpha_t) (I - beta_t k_t k_t^T) "
              "(oracle/brute.py); per-key-channel gates of 'linear_attention' (ChannelGates); "
              "states after tokens 2 and 4",
    "q": s(q), "k": s(k), "v": s(v), "alpha": s(alpha_c), "beta": [str(b) for b in beta],
    "S0": s(S0), "o": s(o_c), "S_T": s(S_c), "S_after": [s(m) for m in prefix],
}
path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "brute_channel_gates.json")
with open(path, "w") as fh:
    json.dump(out_c, fh, indent=1)
print("wrote", path)
