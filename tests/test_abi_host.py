"""Host-only checks of the C ABI: the library loads and exports every symbol the
header declares, and argument errors come back as status codes before any
launch (so these run without a GPU).
"""
import ctypes
import os
import re

import pytest

import gated_delta_rule_59_b200 as dr
from gated_delta_rule_59_b200 import build as drbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dr.h")


@pytest.fixture(scope="module")
def L():
    drbuild.build()
    return dr.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dr_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert {"dr_chunk_fwd", "dr_recurrent_step", "dr_status_string", "dr_get_device_status",
            "dr_version"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"libdr.so does not export {n}"


def test_only_abi_symbols_are_exported(L):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", dr.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert exported == set(declared_functions())


def test_version_and_status_strings(L):
    assert L.dr_version() >= 100
    for code in range(8):
        assert len(L.dr_status_string(code)) > 0
    assert L.dr_status_string(99) == b"unknown status"


P16 = ctypes.c_void_p(0x10000)  # aligned fake device pointers: never dereferenced
P4 = ctypes.c_void_p(0x10004)


def chunk(L, q=P16, k=P16, v=P16, g=None, beta=P16, s_in=None, cu=None, n_seqs=0, B=1, T=8,
          Hqk=1, Hv=1, dk=64, dv=64, dt=1, scale=1.0, o=P16, odt=0, s_out=None, cs=None,
          flags=0):
    return L.dr_chunk_fwd(q, k, v, g, beta, s_in, cu, n_seqs, B, T, Hqk, Hv, dk, dv, dt, scale,
                          o, odt, s_out, cs, flags, None)


def step(L, q=P16, k=P16, v=P16, g=None, beta=P16, state=P16, B=2, Hqk=1, Hv=1, dk=64, dv=64,
         dt=1, scale=1.0, o=P16, odt=0, flags=0):
    return L.dr_recurrent_step(q, k, v, g, beta, state, B, Hqk, Hv, dk, dv, dt, scale, o, odt,
                               flags, None)


def test_chunk_fwd_argument_errors(L):
    assert chunk(L, dt=7) == 3
    assert chunk(L, odt=-1) == 3
    assert chunk(L, T=-1) == 2
    assert chunk(L, Hqk=3, Hv=4) == 2
    assert chunk(L, Hqk=0) == 2
    assert chunk(L, cu=P16, B=2, n_seqs=1) == 2
    assert chunk(L, cu=P16, B=1, n_seqs=-1) == 2
    assert chunk(L, dk=96) == 5
    assert chunk(L, dv=256) == 5
    assert chunk(L, scale=float("nan")) == 5
    assert chunk(L, q=None) == 1
    assert chunk(L, beta=None) == 1
    assert chunk(L, o=None) == 1
    assert chunk(L, q=ctypes.c_void_p(0x10008)) == 4
    assert chunk(L, s_in=ctypes.c_void_p(0x10004)) == 4
    assert chunk(L, g=ctypes.c_void_p(0x10002)) == 4
    assert chunk(L, cs=ctypes.c_void_p(0x10008)) == 4
    assert chunk(L, cs=P16, B=0) == 0
    # option bits: DR_QK_L2NORM (1) is known, any other bit is unsupported
    assert chunk(L, flags=4) == 5
    assert chunk(L, flags=0x80000001) == 5
    # DR_GATE_PER_CHANNEL (2) needs g
    assert chunk(L, flags=2) == 1
    assert chunk(L, flags=3, g=None) == 1
    assert chunk(L, flags=2, B=0) == 0
    assert chunk(L, B=0, flags=1) == 0
    # nothing to do: no sequences => OK without touching the device
    assert chunk(L, B=0) == 0
    assert chunk(L, cu=P16, n_seqs=0) == 0
    # no tokens needs no q/k/v/beta/o, but still validates the rest
    assert chunk(L, B=0, q=None, k=None, v=None, beta=None, o=None) == 0


def test_recurrent_step_argument_errors(L):
    assert step(L, dt=5) == 3
    assert step(L, B=-1) == 2
    assert step(L, Hqk=2, Hv=3) == 2
    assert step(L, dk=48) == 5
    assert step(L, state=None) == 1
    assert step(L, v=None) == 1
    assert step(L, o=ctypes.c_void_p(0x10004)) == 4
    assert step(L, g=ctypes.c_void_p(0x10001)) == 4
    assert step(L, flags=4) == 5
    assert step(L, flags=2) == 1
    assert step(L, flags=2, B=0) == 0
    assert step(L, B=0, flags=1) == 0
    assert step(L, B=0) == 0


def test_conv_and_norm_argument_errors(L):
    conv = lambda x=P16, xd=1, w=P16, K=4, si=None, so=None, cu=None, n=0, B=1, T=8, C=16, \
        y=P16, yd=1: L.dr_short_conv_silu(x, xd, w, K, si, so, cu, n, B, T, C, y, yd, None)
    assert conv(xd=5) == 3
    assert conv(K=0) == 2 and conv(C=0) == 2 and conv(T=-1) == 2
    assert conv(K=9) == 5
    assert conv(cu=P16, B=2, n=1) == 2
    assert conv(cu=P16, n=0) == 2  # tokens but no sequence
    assert conv(x=None) == 1 and conv(w=None) == 1 and conv(y=None) == 1
    assert conv(x=ctypes.c_void_p(0x10001)) == 4
    assert conv(w=ctypes.c_void_p(0x10002)) == 4
    assert conv(B=0) == 0 and conv(B=0, x=None, y=None) == 0
    norm = lambda o=P16, od=0, w=P16, b=None, z=None, zd=0, rows=4, dv=64, kind=0, eps=1e-6, \
        y=P16, yd=0: L.dr_norm_gate(o, od, w, b, z, zd, rows, dv, kind, eps, y, yd, None)
    assert norm(od=4) == 3 and norm(z=P16, zd=9) == 3
    assert norm(rows=-1) == 2 and norm(dv=0) == 2
    assert norm(dv=129) == 5 and norm(kind=2) == 5 and norm(eps=-1.0) == 5
    assert norm(eps=float("nan")) == 5
    assert norm(o=None) == 1 and norm(w=None) == 1 and norm(y=None) == 1
    assert norm(o=ctypes.c_void_p(0x10002)) == 4
    assert norm(rows=0, o=None) == 0


def test_chunk_state_rows():
    assert dr.CHUNK == 64
    hdr = open(HEADER).read()
    assert int(re.search(r"#define DR_CHUNK (\d+)", hdr).group(1)) == dr.CHUNK
    assert int(re.search(r"#define DR_QK_L2NORM (\d+)u", hdr).group(1)) == dr.QK_L2NORM
    assert int(re.search(r"#define DR_GATE_PER_CHANNEL (\d+)u", hdr).group(1)) == dr.GATE_PER_CHANNEL
    assert re.search(r"DR_NORM_RMS = (\d+), DR_NORM_LAYER = (\d+)", hdr).groups() == (
        str(dr.NORM_KINDS["rms"]), str(dr.NORM_KINDS["layer"]))
    assert dr.chunk_state_rows(None, 3, 130) == 9
    assert dr.chunk_state_rows(None, 2, 0) == 0
    assert dr.chunk_state_rows([0, 64, 64, 65, 200], 1, 200) == 1 + 0 + 1 + 3
    # a decreasing (malformed) step counts no rows, as the kernels count it
    assert dr.chunk_state_rows([0, 100, 50, 200], 1, 200) == 2 + 0 + 3
    import oracle
    for cu in ([0, 5, 5, 12], [0, 64, 129, 129, 300]):
        assert dr.chunk_state_rows(cu, 1, cu[-1]) == oracle.chunk_rows(cu, 1, cu[-1], 64)[1]


def test_binding_rejects_cpu_tensors():
    import torch

    q = torch.zeros(1, 4, 1, 16)
    with pytest.raises(ValueError):
        dr.chunk_fwd(q, q, q, None, torch.zeros(1, 4, 1))


def test_product_path_has_no_fallback():
    """The binding never imports the oracle or any CPU implementation."""
    import ast

    pkg = os.path.join(ROOT, "gated_delta_rule_59_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            tree = ast.parse(open(os.path.join(pkg, fn)).read())
            for node in ast.walk(tree):
                if isinstance(node, (ast.Import, ast.ImportFrom)):
                    mods = [a.name for a in node.names] if isinstance(node, ast.Import) else [node.module or ""]
                    assert not any(m.split(".")[0] == "oracle" for m in mods), fn
