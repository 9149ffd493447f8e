"""GPU parity of the fused decode step (dr_recurrent_step) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import gated_delta_rule_59_b200 as dr
import oracle
from gated_delta_rule_59_b200 import inputs
from _parity import TOL_BF16, TOL_F32, metric_for, rel_max, rel_rms, to64

pytestmark = pytest.mark.gpu


def run_steps(state0, steps, dev, scale=1.0, out_dtype=torch.float32):
    state = state0.to(dev).contiguous()
    outs = []
    for st in steps:
        s = st.to(dev)
        outs.append(dr.recurrent_step(s.q, s.k, s.v, s.g, s.beta, state, scale=scale,
                                      out_dtype=out_dtype).cpu())
    torch.cuda.synchronize()
    assert dr.device_status() == 0
    return outs, state.cpu()


def oracle_steps(state0, steps, scale=1.0):
    st = to64(state0)
    outs = []
    for s in steps:
        o, st = oracle.step(s.q, s.k, s.v, s.g, s.beta, st, scale=scale)
        outs.append(o)
    return outs, st


def test_decode_gated_workload_64_steps(cuda_device):
    """Gated decode: B=256, H=32, d=128, bf16 q/k/v, beta in (0,2), 64 steps in place."""
    state0, steps = inputs.decode_config(n_steps=64)
    outs, state = run_steps(state0, steps, cuda_device)
    ref_o, ref_s = oracle_steps(state0, steps)
    worst = max(rel_rms(o, r) for o, r in zip(outs, ref_o))
    assert worst <= TOL_BF16, worst
    assert rel_rms(state, ref_s) <= TOL_BF16


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 64), (64, 64), (128, 32), (128, 128)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_shapes_and_dtypes(cuda_device, dk, dv, dtype):
    B, Hqk, Hv = 5, 2, 4
    state0 = inputs.decode_state(B, Hv, dk, dv, std=0.3, seed=dk * 7 + dv)
    steps = inputs.decode_steps(B, Hqk, Hv, dk, dv, 6, dtype, True, 2.0, seed=dk + dv)
    outs, state = run_steps(state0, steps, cuda_device, scale=0.7)
    ref_o, ref_s = oracle_steps(state0, steps, scale=0.7)
    metric, tol = metric_for(dtype)
    for o, r in zip(outs, ref_o):
        assert metric(o, r) <= tol
    assert metric(state, ref_s) <= tol


def test_decode_degenerate_cases(cuda_device):
    B, H, d = 3, 2, 64
    state0 = inputs.decode_state(B, H, d, d, std=1.0, seed=5)
    st = inputs.decode_steps(B, H, H, d, d, 1, torch.float32, True, 1.0, seed=9)[0]
    # beta = 0: pure decay;  g = None: no decay
    zero_beta = inputs.DecodeStep(st.q, st.k, st.v, st.g, torch.zeros_like(st.beta))
    outs, state = run_steps(state0, [zero_beta], cuda_device)
    expect = np.exp(to64(st.g))[:, :, None, None] * to64(state0)
    assert rel_max(state, expect) <= TOL_F32
    no_gate = inputs.DecodeStep(st.q, st.k, st.v, None, st.beta)
    outs, state = run_steps(state0, [no_gate], cuda_device)
    ref_o, ref_s = oracle_steps(state0, [no_gate])
    assert rel_max(state, ref_s) <= TOL_F32 and rel_max(outs[0], ref_o[0]) <= TOL_F32


def test_decode_bf16_output(cuda_device):
    state0, steps = inputs.decode_config(n_steps=2, B=8)
    outs, _ = run_steps(state0, steps, cuda_device, out_dtype=torch.bfloat16)
    ref_o, _ = oracle_steps(state0, steps)
    for o, r in zip(outs, ref_o):
        assert o.dtype == torch.bfloat16
        # bf16 storage of the output adds at most half an ulp (2^-8 relative) per element
        err = np.abs(to64(o) - r) - 2.0 ** -8 * np.abs(r)
        assert np.max(err) / np.sqrt(np.mean(r ** 2)) <= TOL_BF16


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_decode_qk_l2norm_option(cuda_device, dtype):
    """DR_QK_L2NORM on decode: rescaled q/k rows (one all-zero k) normalised in the kernel."""
    state0, steps = inputs.decode_config(n_steps=4, B=16)
    gen = torch.Generator().manual_seed(5)
    new = []
    for i, s in enumerate(steps):
        cq = torch.empty(s.q.shape[:-1] + (1,)).uniform_(0.2, 5.0, generator=gen)
        ck = torch.empty(s.k.shape[:-1] + (1,)).uniform_(0.2, 5.0, generator=gen)
        q = (s.q.float() * cq).to(dtype)
        k = (s.k.float() * ck).to(dtype)
        if i == 1:
            k[3] = 0.0
        new.append(inputs.DecodeStep(q.contiguous(), k.contiguous(), s.v.to(dtype), s.g, s.beta))
    state = state0.to(cuda_device).contiguous()
    outs = []
    for s in new:
        d = s.to(cuda_device)
        outs.append(dr.recurrent_step(d.q, d.k, d.v, d.g, d.beta, state, scale=0.125,
                                      qk_l2norm=True).cpu())
    torch.cuda.synchronize()
    assert dr.device_status() == 0
    st = to64(state0)
    for s, o in zip(new, outs):
        ro, st = oracle.step(s.q, s.k, s.v, s.g, s.beta, st, scale=0.125, qk_l2norm=True)
        metric, tol = metric_for(dtype)
        assert metric(o, ro) <= tol
    metric, tol = metric_for(dtype)
    assert metric(state.cpu(), st) <= tol
