"""GPU parity of per-key-channel gates (DR_GATE_PER_CHANNEL) against the fp64 oracle.

g [.., Hv, dk]: one log decay per key channel (the "linear_attention" page's
ChannelGates).  Prefill runs the CUDA-core kernel for every dtype; decode the fused
step kernel.  Gates are drawn per channel and then stretched by per-channel factors up
to 40, so that channels decay at very different rates (some almost forget every
chunk, some keep nearly everything).
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_59_b200 as dr
import oracle
from gated_delta_rule_59_b200 import inputs
from _parity import TOL_BF16, metric_for, rel_max, rel_rms, to64, unit_slice

pytestmark = pytest.mark.gpu


def stretched(g, seed):
    """g times a per-(head, channel) factor in [1, 40]: strongly channel-dependent decay."""
    gen = torch.Generator().manual_seed(seed)
    f = torch.empty(g.shape[-2:]).uniform_(0.0, 1.0, generator=gen)
    return (g * (1.0 + 39.0 * f ** 3)).contiguous()


def problem(B, T, Hqk, Hv, d, dtype, seed, cu=None):
    p = inputs.prefill(B, T, Hqk, Hv, d, d, dtype, gated=True, state_std=0.05, seed=seed,
                       cu_seqlens=cu, channel_gates=True)
    return inputs.Prefill(p.q, p.k, p.v, stretched(p.g, seed), p.beta, p.state_in,
                          p.cu_seqlens, p.name)


def check(p, dev, qk_l2norm=False, scale=1.0, chunk_states=False):
    d = p.to(dev)
    res = dr.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.state_in, d.cu_seqlens, scale=scale,
                       qk_l2norm=qk_l2norm, output_chunk_states=chunk_states)
    torch.cuda.synchronize()
    assert dr.device_status() == 0
    ref = oracle.run(p.q, p.k, p.v, p.g, p.beta, p.state_in, p.cu_seqlens, scale=scale,
                     qk_l2norm=qk_l2norm, chunk_len=dr.CHUNK if chunk_states else 0)
    metric, tol = metric_for(p.q.dtype)
    errs = [metric(x.cpu(), r) for x, r in zip(res, ref) if r.size]
    assert max(errs) <= tol, errs
    return errs


def test_kernel_choice():
    assert dr.prefill_kernel(torch.bfloat16, 128, 128, channel_gates=True) == "simt_f32"
    assert dr.prefill_kernel(torch.bfloat16, 128, 128) == "tc_bf16"


@pytest.mark.parametrize("dtype,d,T,group", [(torch.float32, 64, 150, 2),
                                             (torch.float32, 128, 97, 1),
                                             (torch.bfloat16, 128, 200, 2),
                                             (torch.bfloat16, 32, 64, 1)])
def test_prefill_channel_gates(cuda_device, dtype, d, T, group):
    check(problem(2, T, 2, 2 * group, d, dtype, seed=600 + T + d), cuda_device)


def test_prefill_channel_gates_varlen(cuda_device):
    cu = inputs.cu_from_lengths([0, 5, 64, 1, 0, 129, 200, 63])
    check(problem(1, cu[-1], 2, 4, 128, torch.bfloat16, seed=610, cu=cu), cuda_device)


def test_prefill_channel_gates_with_l2norm_and_chunk_states(cuda_device):
    p = problem(2, 140, 1, 2, 64, torch.float32, seed=620)
    check(p, cuda_device, qk_l2norm=True, scale=0.125, chunk_states=True)


def test_equal_channels_match_the_scalar_gate(cuda_device):
    """Channel gates that repeat the scalar gate give the scalar path's result (fp32, both
    through the CUDA-core kernel; the decays enter the sums differently, so up to rounding)."""
    p = inputs.prefill(1, 150, 1, 2, 64, 64, torch.float32, gated=True, state_std=0.05,
                       seed=630)
    d = p.to(cuda_device)
    gc = d.g[..., None].expand(-1, -1, -1, 64).contiguous()
    o1, s1 = dr.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.state_in, None)
    o2, s2 = dr.chunk_fwd(d.q, d.k, d.v, gc, d.beta, d.state_in, None)
    torch.cuda.synchronize()
    assert rel_max(o2.cpu(), o1.cpu()) <= 1e-5 and rel_max(s2.cpu(), s1.cpu()) <= 1e-5


def test_prefill_channel_gates_workload_sampled_units(cuda_device):
    """The benchmarked shape (B=2 T=8192 Hqk=16 -> Hv=32 d=128 bf16) with channel gates."""
    p = inputs.prefill(2, 8192, 16, 32, 128, 128, torch.bfloat16, gated=True, state_std=0.02,
                       seed=640, channel_gates=True)
    d = p.to(cuda_device)
    o, st = dr.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.state_in, None)
    torch.cuda.synchronize()
    assert dr.device_status() == 0
    o, st = o.cpu(), st.cpu()
    for n, h in [(0, 3), (1, 29)]:
        args, (b, t0, t1) = unit_slice(p, n, h)  # g keeps its channel axis: [1, T, 1, dk]
        ro, rs = oracle.run(*args)
        assert rel_rms(o[b:b + 1, t0:t1, h:h + 1], ro) <= TOL_BF16
        assert rel_rms(st[n:n + 1, h:h + 1], rs) <= TOL_BF16


@pytest.mark.parametrize("dtype,d,l2n", [(torch.float32, 64, False), (torch.float32, 128, True),
                                         (torch.bfloat16, 128, False), (torch.bfloat16, 32, True)])
def test_decode_channel_gates(cuda_device, dtype, d, l2n):
    B, Hqk, Hv = 6, 2, 4
    state0 = inputs.decode_state(B, Hv, d, d, std=0.3, seed=650 + d)
    steps = inputs.decode_steps(B, Hqk, Hv, d, d, 5, dtype, True, 2.0, seed=651 + d,
                                channel_gates=True)
    steps = [inputs.DecodeStep(s.q, s.k, s.v, stretched(s.g, 7 + i), s.beta)
             for i, s in enumerate(steps)]
    state = state0.to(cuda_device).contiguous()
    ref_s = to64(state0)
    metric, tol = metric_for(dtype)
    for s in steps:
        sd = s.to(cuda_device)
        o = dr.recurrent_step(sd.q, sd.k, sd.v, sd.g, sd.beta, state, scale=0.5, qk_l2norm=l2n)
        ro, ref_s = oracle.step(s.q, s.k, s.v, s.g, s.beta, ref_s, scale=0.5, qk_l2norm=l2n)
        torch.cuda.synchronize()
        assert metric(o.cpu(), ro) <= tol
    assert dr.device_status() == 0
    assert metric(state.cpu(), ref_s) <= tol
