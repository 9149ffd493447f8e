"""GPU parity of the chunk-state output of dr_chunk_fwd against the fp64 oracle.

The state after every 64 tokens of each sequence and after its last token (the
intermediate states the "linear_attention" page's recurrent route exposes), from both prefill
kernels (the CTA-pair tensor-core kernel for bf16 d=128, the CUDA-core kernel
otherwise), fixed-length and varlen, with and without in-kernel q/k L2 normalisation.
Storing them must leave o and the final state as they are without it.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_59_b200 as dr
import oracle
from gated_delta_rule_59_b200 import inputs
from _parity import TOL_BF16, metric_for, rel_max, rel_rms, to64, unit_slice

pytestmark = pytest.mark.gpu


def run_both(p, dev, out_dtype=torch.float32, qk_l2norm=False, scale=1.0):
    d = p.to(dev)
    args = (d.q, d.k, d.v, d.g, d.beta, d.state_in, d.cu_seqlens)
    o0, s0 = dr.chunk_fwd(*args, scale=scale, out_dtype=out_dtype, qk_l2norm=qk_l2norm)
    o1, s1, cs = dr.chunk_fwd(*args, scale=scale, out_dtype=out_dtype, qk_l2norm=qk_l2norm,
                              output_chunk_states=True)
    torch.cuda.synchronize()
    assert dr.device_status() == 0
    return (o0.cpu(), s0.cpu()), (o1.cpu(), s1.cpu(), cs.cpu())


def check(p, dev, out_dtype=torch.float32, qk_l2norm=False, scale=1.0):
    (o0, s0), (o1, s1, cs) = run_both(p, dev, out_dtype, qk_l2norm, scale)
    ro, rs, rcs = oracle.run(p.q, p.k, p.v, p.g, p.beta, p.state_in, p.cu_seqlens, scale=scale,
                             qk_l2norm=qk_l2norm, chunk_len=dr.CHUNK)
    assert tuple(cs.shape) == rcs.shape
    metric, tol = metric_for(p.q.dtype)
    ecs = metric(cs, rcs) if rcs.size else 0.0
    assert ecs <= tol, ecs
    # the output and the final state are those of the call without chunk states
    assert rel_max(o1.float(), o0.float()) <= 1e-6 and rel_max(s1, s0) <= 1e-6
    # each sequence's last row is its final state (stored from the same registers)
    B, T = p.q.shape[:2]
    cu = None if p.cu_seqlens is None else p.cu_seqlens.tolist()
    bases, _ = oracle.chunk_rows(cu, B, T, dr.CHUNK)
    lens = [T] * B if cu is None else [b - a for a, b in zip(cu[:-1], cu[1:])]
    for n, ln in enumerate(lens):
        if ln > 0:
            last = bases[n] + (ln + dr.CHUNK - 1) // dr.CHUNK - 1
            assert torch.equal(cs[last], s1[n]), n
    return ecs


@pytest.mark.parametrize("dtype,d,T,out_dtype", [(torch.bfloat16, 128, 200, torch.float32),
                                                 (torch.bfloat16, 128, 128, torch.bfloat16),
                                                 (torch.bfloat16, 128, 1, torch.float32),
                                                 (torch.bfloat16, 64, 130, torch.float32),
                                                 (torch.float32, 64, 97, torch.float32),
                                                 (torch.float32, 128, 64, torch.float32)])
def test_chunk_states_fixed_length(cuda_device, dtype, d, T, out_dtype):
    p = inputs.prefill(2, T, 2, 4, d, d, dtype, gated=True, state_std=0.02, seed=500 + T + d)
    check(p, cuda_device, out_dtype=out_dtype)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64)])
def test_chunk_states_varlen(cuda_device, dtype, d):
    lens = [0, 5, 64, 1, 0, 129, 200, 63]
    cu = inputs.cu_from_lengths(lens)
    p = inputs.prefill(1, cu[-1], 2, 4, d, d, dtype, gated=True, state_std=0.02, seed=510 + d,
                       cu_seqlens=cu)
    check(p, cuda_device)


def test_chunk_states_with_qk_l2norm(cuda_device):
    p = inputs.prefill(2, 150, 2, 4, 128, 128, torch.bfloat16, gated=True, state_std=0.02,
                       seed=520)
    check(p, cuda_device, qk_l2norm=True, scale=128 ** -0.5)


def test_chunk_states_caller_buffer_and_zero_tokens(cuda_device):
    p = inputs.prefill(1, 100, 1, 2, 128, 128, torch.bfloat16, gated=True, state_std=0.02,
                       seed=530).to(cuda_device)
    buf = torch.full((2, 2, 128, 128), float("nan"), device=cuda_device)
    o, st, cs = dr.chunk_fwd(p.q, p.k, p.v, p.g, p.beta, p.state_in, None, chunk_states=buf)
    torch.cuda.synchronize()
    assert cs is buf and not torch.isnan(buf).any() and torch.equal(buf[1], st[0])
    with pytest.raises(ValueError):
        dr.chunk_fwd(p.q, p.k, p.v, p.g, p.beta, p.state_in, None, chunk_states=buf[:1])
    z = inputs.prefill(2, 0, 1, 2, 128, 128, torch.bfloat16, gated=True, state_std=0.02,
                       seed=531).to(cuda_device)
    o, st, cs = dr.chunk_fwd(z.q, z.k, z.v, z.g, z.beta, z.state_in, None,
                             output_chunk_states=True)
    torch.cuda.synchronize()
    assert dr.device_status() == 0 and cs.shape == (0, 2, 128, 128)
    assert torch.equal(st, z.state_in)


def test_chunk_states_gated_prefill_workload_sampled_units(cuda_device):
    """B=2 T=8192 Hqk=16 -> Hv=32 d=128 bf16 (the benchmarked launch) with its 2 x 128 chunk
    states per head; sampled units against the oracle's chunk states."""
    p = inputs.config(2)
    d = p.to(cuda_device)
    o, st, cs = dr.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.state_in, None,
                             output_chunk_states=True)
    torch.cuda.synchronize()
    assert dr.device_status() == 0
    nt = p.q.shape[1] // dr.CHUNK
    assert cs.shape == (2 * nt, 32, 128, 128)
    for n, h in [(0, 5), (1, 30)]:
        args, _ = unit_slice(p, n, h)
        _, _, rcs = oracle.run(*args, chunk_len=dr.CHUNK)
        got = cs[n * nt:(n + 1) * nt, h:h + 1].cpu()
        e = rel_rms(got, rcs)
        assert e <= TOL_BF16, (n, h, e)
        # every stored row, not just the whole tensor, stays within the bound of its own size
        for j in (0, nt // 2, nt - 1):
            assert rel_rms(got[j], rcs[j]) <= TOL_BF16, (n, h, j)
