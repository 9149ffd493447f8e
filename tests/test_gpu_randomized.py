"""Seeded randomized GPU parity of the prefill against the fp64 oracle.

Each case draws one small problem from the space the library supports and checks every output
and final state: input dtype, head dimension, GQA group, fixed-length or varlen batches (with
empty and ragged sequences), decay on/off, beta up to 2, initial state on/off, scale, q/k L2
normalisation by the kernel (inputs rescaled row by row), fp32 or bf16 output.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_59_b200 as dr
import oracle
from gated_delta_rule_59_b200 import inputs
from _parity import metric_for

pytestmark = pytest.mark.gpu

N_CASES = 24


def draw(i):
    rng = np.random.default_rng(5000 + i)
    dtype = torch.bfloat16 if rng.random() < 0.7 else torch.float32
    d = int(rng.choice([128, 128, 64, 32]))
    Hqk = int(rng.choice([1, 2, 4]))
    Hv = Hqk * int(rng.choice([1, 2]))
    varlen = rng.random() < 0.3
    if varlen:
        lens = [int(x) for x in rng.integers(0, 300, int(rng.integers(1, 6)))]
        lens[int(rng.integers(0, len(lens)))] = int(rng.integers(1, 300))  # one non-empty
        cu = inputs.cu_from_lengths(lens)
        B, T = 1, cu[-1]
    else:
        cu = None
        B, T = int(rng.integers(1, 4)), int(rng.integers(1, 300))
    return dict(dtype=dtype, d=d, Hqk=Hqk, Hv=Hv, B=B, T=T, cu=cu,
                gated=bool(rng.random() < 0.8), beta_max=float(rng.choice([1.0, 2.0])),
                state_std=float(rng.choice([0.0, 0.05])),
                scale=float(rng.choice([1.0, d ** -0.5])), l2n=bool(rng.random() < 0.3),
                out=torch.bfloat16 if (dtype == torch.bfloat16 and rng.random() < 0.2)
                else torch.float32, seed=7000 + i)


@pytest.mark.parametrize("i", range(N_CASES))
def test_random_prefill_case(cuda_device, i):
    c = draw(i)
    p = inputs.prefill(c["B"], c["T"], c["Hqk"], c["Hv"], c["d"], c["d"], c["dtype"],
                       gated=c["gated"], beta_max=c["beta_max"], state_std=c["state_std"],
                       seed=c["seed"], cu_seqlens=c["cu"])
    q, k = p.q, p.k
    if c["l2n"]:
        gen = torch.Generator().manual_seed(c["seed"] + 1)
        q = (q.float() * torch.empty(q.shape[:-1] + (1,)).uniform_(0.3, 3.0, generator=gen)
             ).to(c["dtype"]).contiguous()
        k = (k.float() * torch.empty(k.shape[:-1] + (1,)).uniform_(0.3, 3.0, generator=gen)
             ).to(c["dtype"]).contiguous()
    dev = cuda_device
    f = lambda t: None if t is None else t.to(dev)
    o, st = dr.chunk_fwd(f(q), f(k), f(p.v), f(p.g), f(p.beta), f(p.state_in), f(p.cu_seqlens),
                         scale=c["scale"], out_dtype=c["out"], qk_l2norm=c["l2n"])
    torch.cuda.synchronize()
    assert dr.device_status() == 0
    ro, rs = oracle.run(q, k, p.v, p.g, p.beta, p.state_in, p.cu_seqlens, scale=c["scale"],
                        qk_l2norm=c["l2n"])
    metric, tol = metric_for(c["dtype"])
    if c["out"] == torch.bfloat16:
        # a bf16 output also carries its storage rounding (half an ulp, 2^-8 relative at most),
        # allowed explicitly as in test_bf16_output_dtype
        err = np.abs(o.double().cpu().numpy() - ro) - 2.0 ** -8 * np.abs(ro)
        eo = float(np.max(err) / np.sqrt(np.mean(ro ** 2)))
    else:
        eo = metric(o.cpu(), ro)
    es = metric(st.cpu(), rs)
    assert eo <= tol and es <= tol, (c, eo, es)
