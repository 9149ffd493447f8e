"""GPU parity of the chunked prefill (dr_chunk_fwd) against the fp64 oracle.

Small cases are compared element by element over every output; the full-size
workloads are compared on whole sampled (sequence, head) units, which the
oracle recomputes one by one.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_59_b200 as dr
import oracle
from gated_delta_rule_59_b200 import inputs
from _parity import TOL_BF16, TOL_F32, metric_for, rel_max, rel_rms, to64, unit_slice

pytestmark = pytest.mark.gpu


def gpu_run(p, dev, scale=1.0, out_dtype=torch.float32, with_state=True):
    d = p.to(dev)
    o, st = dr.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.state_in, d.cu_seqlens, scale=scale,
                         output_final_state=with_state, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert dr.device_status() == 0
    return o.cpu(), None if st is None else st.cpu()


def check_full(p, dev, scale=1.0):
    o, st = gpu_run(p, dev, scale)
    ro, rs = oracle.run(p.q, p.k, p.v, p.g, p.beta, p.state_in, p.cu_seqlens, scale=scale)
    metric, tol = metric_for(p.q.dtype)
    eo, es = metric(o, ro), metric(st, rs)
    assert eo <= tol and es <= tol, (eo, es)
    return eo, es


def test_plain_deltanet_fp32_workload(cuda_device):
    """B=1 T=64 H=2 d=16 fp32, g = 0, zero initial state: max rel error <= 1e-4."""
    check_full(inputs.config(0), cuda_device)


@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
@pytest.mark.parametrize("d", [64, 128])
def test_bf16_ragged_lengths(cuda_device, T, d):
    p = inputs.prefill(2, T, 2, 4, d, d, torch.bfloat16, gated=True, state_std=0.02,
                       seed=T * 10 + d)
    check_full(p, cuda_device)


@pytest.mark.parametrize("dk,dv", [(16, 16), (32, 32), (64, 128), (128, 64), (16, 128)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_head_dims(cuda_device, dk, dv, dtype):
    p = inputs.prefill(1, 97, 1, 2, dk, dv, dtype, gated=True, state_std=0.1, seed=dk + 3 * dv)
    check_full(p, cuda_device, scale=dk ** -0.5)


def _rescaled_rows(x, seed, zero_token=None):
    """Rows (last axis) multiplied by random positive factors, one token zeroed; same dtype."""
    gen = torch.Generator().manual_seed(seed)
    c = torch.empty(x.shape[:-1] + (1,)).uniform_(0.2, 5.0, generator=gen)
    y = x.float() * c
    if zero_token is not None:
        y[:, zero_token] = 0.0
    return y.to(x.dtype).contiguous()


@pytest.mark.parametrize("dtype,d,T,group", [(torch.bfloat16, 128, 200, 2),
                                             (torch.bfloat16, 128, 64, 1),
                                             (torch.bfloat16, 64, 130, 2),
                                             (torch.float32, 64, 97, 1)])
def test_qk_l2norm_option(cuda_device, dtype, d, T, group):
    """DR_QK_L2NORM: q/k rows rescaled (one token all zero) and normalised by the kernel,
    against the oracle normalising the same inputs in fp64; scale = d^-1/2."""
    p = inputs.prefill(2, T, 2, 2 * group, d, d, dtype, gated=True, state_std=0.02,
                       seed=300 + T + d)
    q = _rescaled_rows(p.q, 1, zero_token=T // 3)
    k = _rescaled_rows(p.k, 2, zero_token=T // 2)
    scale = d ** -0.5
    dev = cuda_device
    o, st = dr.chunk_fwd(q.to(dev), k.to(dev), p.v.to(dev), p.g.to(dev), p.beta.to(dev),
                         p.state_in.to(dev), None, scale=scale, qk_l2norm=True)
    torch.cuda.synchronize()
    assert dr.device_status() == 0
    ro, rs = oracle.run(q, k, p.v, p.g, p.beta, p.state_in, None, scale=scale, qk_l2norm=True)
    metric, tol = metric_for(dtype)
    eo, es = metric(o.cpu(), ro), metric(st.cpu(), rs)
    assert eo <= tol and es <= tol, (eo, es)


def test_many_units_several_cluster_waves(cuda_device):
    """B=3, Hv=32: 96 (sequence, head) units = 192 CTAs of 2-CTA clusters, more than one wave
    on 148 SMs; every output and final state against the oracle."""
    p = inputs.prefill(3, 150, 16, 32, 128, 128, torch.bfloat16, gated=True, state_std=0.02,
                       seed=77)
    check_full(p, cuda_device)


@pytest.mark.parametrize("group", [1, 2, 4])
def test_gqa_groups(cuda_device, group):
    p = inputs.prefill(1, 130, 2, 2 * group, 128, 128, torch.bfloat16, gated=True,
                       state_std=0.02, seed=40 + group)
    check_full(p, cuda_device)


def test_degenerate_gates_and_betas(cuda_device):
    base = inputs.prefill(1, 150, 1, 2, 64, 64, torch.float32, gated=True, state_std=0.5, seed=77)
    # beta = 0: outputs read the decayed initial state, state = e^{sum g} state_in
    p = inputs.Prefill(base.q, base.k, base.v, base.g, torch.zeros_like(base.beta),
                       base.state_in, None)
    check_full(p, cuda_device)
    # beta near 2 (negative eigenvalue regime) and very negative gates
    p = inputs.Prefill(base.q, base.k, base.v, base.g * 60.0, torch.full_like(base.beta, 1.999),
                       base.state_in, None)
    check_full(p, cuda_device)
    # g = 0 given explicitly equals g absent
    pz = inputs.Prefill(base.q, base.k, base.v, torch.zeros_like(base.g), base.beta, base.state_in, None)
    pn = inputs.Prefill(base.q, base.k, base.v, None, base.beta, base.state_in, None)
    oz, sz = gpu_run(pz, cuda_device)
    on, sn = gpu_run(pn, cuda_device)
    assert torch.equal(oz, on) and torch.equal(sz, sn)


def test_varlen_with_empty_and_ragged_sequences(cuda_device):
    lens = [0, 5, 64, 1, 0, 129, 200, 63]
    cu = inputs.cu_from_lengths(lens)
    p = inputs.prefill(1, cu[-1], 2, 4, 128, 128, torch.bfloat16, gated=True, state_std=0.02,
                       seed=91, cu_seqlens=cu)
    check_full(p, cuda_device)
    # empty sequences return their initial state untouched
    _, st = gpu_run(p, cuda_device)
    assert torch.equal(st[0], p.state_in[0]) and torch.equal(st[4], p.state_in[4])


def test_varlen_equals_separate_calls(cuda_device):
    lens = [70, 33, 128]
    cu = inputs.cu_from_lengths(lens)
    p = inputs.prefill(1, cu[-1], 1, 2, 64, 64, torch.float32, gated=True, state_std=0.1,
                       seed=92, cu_seqlens=cu)
    o, st = gpu_run(p, cuda_device)
    for n in range(len(lens)):
        a, b = cu[n], cu[n + 1]
        pn = inputs.Prefill(p.q[:, a:b], p.k[:, a:b], p.v[:, a:b], p.g[:, a:b], p.beta[:, a:b],
                            p.state_in[n:n + 1], None)
        on, sn = gpu_run(pn, cuda_device)
        assert rel_max(on, o[:, a:b]) <= 1e-6 and rel_max(sn, st[n:n + 1]) <= 1e-6


def test_state_carry_split_equals_unsplit(cuda_device):
    p = inputs.prefill(2, 300, 1, 1, 128, 128, torch.bfloat16, gated=True, state_std=0.02, seed=93)
    o, st = gpu_run(p, cuda_device)
    cut = 130
    p1 = inputs.Prefill(p.q[:, :cut].contiguous(), p.k[:, :cut].contiguous(), p.v[:, :cut].contiguous(),
                        p.g[:, :cut].contiguous(), p.beta[:, :cut].contiguous(), p.state_in, None)
    o1, s1 = gpu_run(p1, cuda_device)
    p2 = inputs.Prefill(p.q[:, cut:].contiguous(), p.k[:, cut:].contiguous(), p.v[:, cut:].contiguous(),
                        p.g[:, cut:].contiguous(), p.beta[:, cut:].contiguous(), s1, None)
    o2, s2 = gpu_run(p2, cuda_device)
    ro, rs = oracle.run(p.q, p.k, p.v, p.g, p.beta, p.state_in)
    assert rel_rms(torch.cat([o1, o2], 1), ro) <= TOL_BF16
    assert rel_rms(s2, rs) <= TOL_BF16


def test_state_in_is_read_only_and_no_state_out(cuda_device):
    p = inputs.prefill(1, 100, 1, 2, 64, 64, torch.bfloat16, gated=True, state_std=0.02, seed=94)
    d = p.to(cuda_device)
    keep = d.state_in.clone()
    o, st = dr.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, d.state_in, output_final_state=False)
    torch.cuda.synchronize()
    assert st is None and torch.equal(keep, d.state_in)
    ro, _ = oracle.run(p.q, p.k, p.v, p.g, p.beta, p.state_in)
    assert rel_rms(o.cpu(), ro) <= TOL_BF16


def test_zero_tokens_copies_state(cuda_device):
    p = inputs.prefill(3, 0, 1, 2, 64, 64, torch.bfloat16, gated=True, state_std=0.1, seed=95)
    _, st = gpu_run(p, cuda_device)
    assert torch.equal(st, p.state_in)
    p0 = inputs.prefill(3, 0, 1, 2, 64, 64, torch.bfloat16, gated=True, seed=95)
    _, st0 = gpu_run(p0, cuda_device)
    assert torch.count_nonzero(st0) == 0


def test_malformed_cu_seqlens_reported_on_device(cuda_device):
    p = inputs.prefill(1, 50, 1, 1, 64, 64, torch.bfloat16, gated=True, seed=96,
                       cu_seqlens=[0, 30, 20, 50])
    d = p.to(cuda_device)
    dr.chunk_fwd(d.q, d.k, d.v, d.g, d.beta, None, d.cu_seqlens)
    assert dr.device_status() == 2  # DR_ERR_SHAPE, and the context stays usable
    assert dr.device_status() == 0


def test_bf16_output_dtype(cuda_device):
    p = inputs.prefill(1, 200, 2, 4, 128, 128, torch.bfloat16, gated=True, state_std=0.02, seed=97)
    o, st = gpu_run(p, cuda_device, out_dtype=torch.bfloat16)
    ro, rs = oracle.run(p.q, p.k, p.v, p.g, p.beta, p.state_in)
    assert o.dtype == torch.bfloat16
    err = np.abs(to64(o) - ro) - 2.0 ** -8 * np.abs(ro)  # allow bf16 storage rounding
    assert np.max(err) / np.sqrt(np.mean(ro ** 2)) <= TOL_BF16
    assert rel_rms(st, rs) <= TOL_BF16


# ---------------------------------------------------------------- full-size workloads


def check_units(p, dev, units, o=None, st=None):
    if o is None:
        o, st = gpu_run(p, dev)
    worst = 0.0
    for n, h in units:
        args, (b, t0, t1) = unit_slice(p, n, h)
        ro, rs = oracle.run(*args)
        eo = rel_rms(o[b:b + 1, t0:t1, h:h + 1], ro)
        es = rel_rms(st[n:n + 1, h:h + 1], rs)
        assert eo <= TOL_BF16 and es <= TOL_BF16, (n, h, eo, es)
        worst = max(worst, eo, es)
    return worst


def test_deltanet_layer_workload_full(cuda_device):
    """B=4 T=2048 H=16 d=64 bf16, g = 0: every output against the oracle."""
    check_full(inputs.config(1), cuda_device)


def test_gated_prefill_workload_sampled_units(cuda_device):
    """B=2 T=8192 Hqk=16 -> Hv=32 d=128 bf16 (the benchmarked launch), sampled units."""
    p = inputs.config(2)
    check_units(p, cuda_device, [(0, 0), (0, 17), (1, 31), (1, 8)])


def test_varlen_long_context_workload_sampled_units(cuda_device):
    """8 sequences of 512..16384 tokens + one of 65536, H=16 d=128, sampled units."""
    p = inputs.config(4)
    n_seqs = p.cu_seqlens.numel() - 1
    check_units(p, cuda_device, [(0, 3), (3, 15), (n_seqs - 2, 0), (n_seqs - 1, 9)])
