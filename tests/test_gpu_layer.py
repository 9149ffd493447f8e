"""GPU parity of the steps either side of the rule against ``oracle/layer.py``.

dr_short_conv_silu (causal depthwise convolution + SiLU, with conv state and varlen) and
dr_norm_gate (RMSNorm / LayerNorm per head + SiLU output gate): fp32 element by element
within 1e-4 of the largest reference value, bf16 within 2e-2 of the reference RMS (plus
the bf16 storage rounding of a bf16 output); the convolution's carried state is exact.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_59_b200 as dr
from gated_delta_rule_59_b200 import inputs
from oracle import layer
from _parity import TOL_BF16, TOL_F32, rel_max, to64

pytestmark = pytest.mark.gpu


def err_bf16(x, ref, out_bf16):
    x, ref = to64(x), to64(ref)
    e = np.abs(x - ref) - (2.0 ** -8 * np.abs(ref) if out_bf16 else 0.0)
    return float(np.max(e) / np.sqrt(np.mean(ref ** 2)))


def check(x, ref, dtype, out_dtype):
    if dtype == torch.float32 and out_dtype == torch.float32:
        assert rel_max(x, ref) <= TOL_F32
    else:
        assert err_bf16(x, ref, out_dtype == torch.bfloat16) <= TOL_BF16


@pytest.mark.parametrize("dtype,out_dtype", [(torch.float32, torch.float32),
                                             (torch.bfloat16, torch.bfloat16),
                                             (torch.bfloat16, torch.float32)])
@pytest.mark.parametrize("K", [1, 2, 4, 8])
def test_conv_fixed_length(cuda_device, dtype, out_dtype, K):
    gen = torch.Generator().manual_seed(700 + K)
    B, T, H, d = 2, 75, 3, 64
    x = torch.randn((B, T, H, d), generator=gen).to(dtype)
    w = torch.randn((H, d, K), generator=gen) * 0.5
    s0 = torch.randn((B, H, d, K - 1), generator=gen)
    y, st = dr.short_conv_silu(x.to(cuda_device), w.to(cuda_device), s0.to(cuda_device),
                               out_dtype=out_dtype)
    torch.cuda.synchronize()
    ry, rs = layer.short_conv_silu(x, w, s0)
    check(y.cpu(), ry, dtype, out_dtype)
    assert np.array_equal(to64(st.cpu()), rs)  # the inputs themselves, exactly


def test_conv_varlen_and_state_carry(cuda_device):
    gen = torch.Generator().manual_seed(710)
    lens = [0, 3, 64, 1, 0, 129, 40]
    cu = inputs.cu_from_lengths(lens)
    T, H, d, K = cu[-1], 2, 128, 4
    x = torch.randn((1, T, H, d), generator=gen)
    w = torch.randn((H, d, K), generator=gen) * 0.5
    s0 = torch.randn((len(lens), H, d, K - 1), generator=gen)
    cut = torch.tensor(cu, dtype=torch.int32)
    dev = cuda_device
    y, st = dr.short_conv_silu(x.to(dev), w.to(dev), s0.to(dev), cut.to(dev))
    torch.cuda.synchronize()
    assert dr.device_status() == 0
    ry, rs = layer.short_conv_silu(x, w, s0, np.array(cu))
    assert rel_max(y.cpu(), ry) <= TOL_F32
    assert np.array_equal(to64(st.cpu()), rs)
    # split one sequence in two calls, state carried on the device: same outputs
    a = torch.randn((1, 50, H, d), generator=gen).to(dev)
    w_ = w.to(dev)
    y_all, s_all = dr.short_conv_silu(a, w_)
    y1, s1 = dr.short_conv_silu(a[:, :17].contiguous(), w_)
    y2, s2 = dr.short_conv_silu(a[:, 17:].contiguous(), w_, s1)
    torch.cuda.synchronize()
    assert rel_max(torch.cat([y1, y2], 1).cpu(), y_all.cpu()) <= 1e-6
    assert torch.equal(s2, s_all)


def test_conv_in_place_state_and_zero_tokens(cuda_device):
    gen = torch.Generator().manual_seed(720)
    H, d, K = 1, 32, 4
    w = (torch.randn((H, d, K), generator=gen) * 0.5).to(cuda_device)
    s = torch.randn((2, H, d, K - 1), generator=gen).to(cuda_device)
    s_ref = s.clone()
    # zero tokens: the state is the history itself
    x0 = torch.empty((2, 0, H, d), device=cuda_device)
    y0, st0 = dr.short_conv_silu(x0, w, s)
    torch.cuda.synchronize()
    assert y0.numel() == 0 and torch.equal(st0, s_ref)
    # two tokens, state updated in place through the raw call
    x = torch.randn((2, 2, H, d), generator=gen).to(cuda_device)
    y = torch.empty_like(x)
    rc = dr.lib().dr_short_conv_silu(
        dr._ptr(x), 0, dr._ptr(w), K, dr._ptr(s), dr._ptr(s), None, 0, 2, 2, H * d,
        dr._ptr(y), 0, dr._stream(cuda_device))
    torch.cuda.synchronize()
    assert rc == 0
    ry, rs = layer.short_conv_silu(x.cpu(), w.cpu(), s_ref.cpu())
    assert rel_max(y.cpu(), ry) <= TOL_F32 and np.array_equal(to64(s.cpu()), rs)


@pytest.mark.parametrize("kind", ["rms", "layer"])
@pytest.mark.parametrize("dtype,zdtype,out_dtype,dv", [(torch.float32, torch.float32, torch.float32, 128),
                                                       (torch.float32, torch.bfloat16, torch.bfloat16, 128),
                                                       (torch.bfloat16, None, torch.bfloat16, 64),
                                                       (torch.float32, torch.float32, torch.float32, 48),
                                                       (torch.float32, None, torch.float32, 16)])
def test_norm_gate(cuda_device, kind, dtype, zdtype, out_dtype, dv):
    gen = torch.Generator().manual_seed(730 + dv)
    o = (torch.randn((2, 33, 4, dv), generator=gen) * 3.0).to(dtype)
    wt = torch.rand(dv, generator=gen) + 0.5
    bs = torch.randn(dv, generator=gen) if kind == "layer" else None
    z = None if zdtype is None else (torch.randn(o.shape, generator=gen) * 2.0).to(zdtype)
    dev = cuda_device
    y = dr.norm_gate(o.to(dev), wt.to(dev), None if bs is None else bs.to(dev),
                     None if z is None else z.to(dev), kind=kind, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ref = layer.norm_gate(o, wt, bs, z, kind=kind)
    check(y.cpu(), ref, dtype if zdtype in (None, torch.float32) else torch.bfloat16, out_dtype)


def test_norm_gate_in_place(cuda_device):
    gen = torch.Generator().manual_seed(740)
    o = torch.randn((3, 10, 2, 128), generator=gen)
    wt = torch.rand(128, generator=gen) + 0.5
    z = torch.randn(o.shape, generator=gen)
    d = o.to(cuda_device)
    y = dr.norm_gate(d, wt.to(cuda_device), z=z.to(cuda_device), y=d)
    torch.cuda.synchronize()
    assert y.data_ptr() == d.data_ptr()
    assert rel_max(d.cpu(), layer.norm_gate(o, wt, None, z)) <= TOL_F32


def test_mixer_on_device_equals_oracle(cuda_device):
    """conv + SiLU -> rule with in-kernel L2 norm -> RMSNorm + gate, all on the device, against
    the oracle's composed mixer (fp32, CUDA-core prefill)."""
    gen = torch.Generator().manual_seed(750)
    B, T, Hqk, Hv, d, K = 1, 90, 1, 2, 64, 4
    qx, kx = torch.randn((2, B, T, Hqk, d), generator=gen)
    vx = torch.randn((B, T, Hv, d), generator=gen)
    wq, wk = torch.randn((2, Hqk, d, K), generator=gen) * 0.5
    wv = torch.randn((Hv, d, K), generator=gen) * 0.5
    g = torch.log(torch.rand((B, T, Hv), generator=gen) * 0.5 + 0.5)
    beta = torch.rand((B, T, Hv), generator=gen)
    z = torch.randn((B, T, Hv, d), generator=gen)
    dev = cuda_device
    D = lambda t: t.contiguous().to(dev)
    q, _ = dr.short_conv_silu(D(qx), D(wq))
    k, _ = dr.short_conv_silu(D(kx), D(wk))
    v, _ = dr.short_conv_silu(D(vx), D(wv))
    o, st = dr.chunk_fwd(q, k, v, D(g), D(beta), None, None, scale=d ** -0.5, qk_l2norm=True)
    out = dr.norm_gate(o, torch.ones(d, device=dev), z=D(z))
    torch.cuda.synchronize()
    assert dr.device_status() == 0
    ref, rst, _ = layer.mixer(qx, kx, vx, wq, wk, wv, g, beta, scale=d ** -0.5, z=z)
    assert rel_max(out.cpu(), ref) <= TOL_F32 and rel_max(st.cpu(), rst) <= TOL_F32
