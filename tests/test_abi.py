"""The C-ABI library without a GPU: it loads, exports every entry point that
include/rtp.h declares, and rejects bad arguments on the host (before any CUDA
call)."""
import ctypes
import os
import re

import pytest

from long_context_sparse_rtp_b200 import build, rtp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return rtp.lib()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "rtp.h")).read()
    return sorted(set(re.findall(r"RTP_API\s+[\w\s\*]*?\b(rtp_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    # and nothing else leaks out of the library besides the C entry points
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", rtp.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert exported == set(names)


def test_status_strings(L):
    assert rtp.rtp_status_string(0) == "RTP_OK"
    assert rtp.rtp_status_string(4) == "RTP_ERR_WORKSPACE_TOO_SMALL"
    assert rtp.rtp_status_string(99) == "RTP_ERR_UNKNOWN"
    assert rtp.rtp_version() == "0.1.0"


def _shape(B=1, Lq=64, Lk=64, H=8, Hkv=2, D=128, q_pos0=0):
    return rtp.Shape(B, Lq, Lk, H, Hkv, D, q_pos0)


def _v(addr=0x10000, sb=64 * 8 * 128, sl=8 * 128):
    return rtp.View(ctypes.c_void_p(addr), sb, sl)


def test_workspace_sizes(L):
    role = (ctypes.c_uint8 * 4)(1, 0, 0, 0)
    s = _shape(B=8, Lq=1, Lk=131072, H=32, Hkv=4, q_pos0=131071)
    dec = L.rtp_workspace_size(rtp.OP_SPARSE_DECODE, ctypes.byref(s), role, 0)
    # scores (8 rows x 128K fp32) dominate: at least 4 MB per row of 8 heads x 8 batches
    assert dec >= 8 * 8 * 131072 * 4
    assert L.rtp_workspace_size(rtp.OP_TOPP_SELECT, ctypes.byref(s), role, 0) == 256
    loc = L.rtp_workspace_size(rtp.OP_LOCAL, ctypes.byref(s), role, 0)
    assert loc > 256
    bad = _shape(D=64)
    assert L.rtp_workspace_size(rtp.OP_SPARSE_DECODE, ctypes.byref(bad), role, 0) == 256


def test_host_side_errors(L):
    role = (ctypes.c_uint8 * 2)(1, 0)
    s = _shape()
    ws = ctypes.c_void_p(0x20000)
    f = ctypes.c_void_p(0x30000)
    # D != 128
    bad = _shape(D=64)
    assert L.rtp_topp_select(ctypes.byref(bad), role, 0, _v(), _v(), ctypes.c_float(0.9), f, f, f,
                             None, ws, 1 << 20, None) == 2
    # p outside [0, 1]
    for p in (-0.1, 1.5, float("nan")):
        assert L.rtp_topp_select(ctypes.byref(s), role, 0, _v(), _v(), ctypes.c_float(p), f, f, f,
                                 None, ws, 1 << 20, None) == 1
    # null shape / null role
    assert L.rtp_topp_select(None, role, 0, _v(), _v(), ctypes.c_float(0.9), f, f, f, None, ws,
                             1 << 20, None) == 1
    assert L.rtp_topp_select(ctypes.byref(s), None, 0, _v(), _v(), ctypes.c_float(0.9), f, f, f,
                             None, ws, 1 << 20, None) == 1
    # null outputs
    assert L.rtp_topp_select(ctypes.byref(s), role, 0, _v(), _v(), ctypes.c_float(0.9), None, f,
                             f, None, ws, 1 << 20, None) == 1
    # workspace too small
    assert L.rtp_topp_select(ctypes.byref(s), role, 0, _v(sb=64 * 4 * 16, sl=4 * 16),
                             _v(sb=64 * 4 * 16, sl=4 * 16), ctypes.c_float(0.9), f, f, f, None,
                             ws, 16, None) == 4
    # misaligned view
    assert L.rtp_topp_select(ctypes.byref(s), role, 0, _v(addr=0x10002, sb=64 * 4 * 16,
                                                          sl=4 * 16),
                             _v(sb=64 * 4 * 16, sl=4 * 16), ctypes.c_float(0.9), f, f, f, None,
                             ws, 1 << 20, None) == 3
    # causal: query rows past the key rows
    s2 = _shape(Lq=64, Lk=32)
    assert L.rtp_local_attn(ctypes.byref(s2), role, 16, 4, _v(), _v(), _v(), ctypes.c_float(0.1),
                            _v(), None, ws, 1 << 20, None) == 1
    # window < 1, negative sinks, bad scale
    assert L.rtp_local_attn(ctypes.byref(s), role, 0, 4, _v(), _v(), _v(), ctypes.c_float(0.1),
                            _v(), None, ws, 1 << 20, None) == 1
    assert L.rtp_local_attn(ctypes.byref(s), role, 16, -1, _v(), _v(), _v(), ctypes.c_float(0.1),
                            _v(), None, ws, 1 << 20, None) == 1
    assert L.rtp_dense_attn(ctypes.byref(s), _v(), _v(), _v(), ctypes.c_float(-1.0), _v(), None,
                            ws, 1 << 20, None) == 1
    # H not a multiple of Hkv, role value out of range
    s3 = _shape(H=7, Hkv=2)
    assert L.rtp_dense_attn(ctypes.byref(s3), _v(), _v(), _v(), ctypes.c_float(0.1), _v(), None,
                            ws, 1 << 20, None) == 1
    role_bad = (ctypes.c_uint8 * 2)(2, 0)
    assert L.rtp_local_attn(ctypes.byref(s), role_bad, 16, 4, _v(), _v(), _v(),
                            ctypes.c_float(0.1), _v(), None, ws, 1 << 20, None) == 1
    # decode needs Lq == 1
    assert L.rtp_sparse_attn_decode(ctypes.byref(s), role, 0, _v(), _v(), _v(), _v(), _v(),
                                    ctypes.c_float(0.9), ctypes.c_float(0.1), _v(), None, None,
                                    None, None, None, ws, 1 << 30, None) == 1
    # k16 layout flag must be 0 or 1
    assert L.rtp_index_scores(ctypes.byref(s), role, 2, _v(), _v(), f, f, _v(), _v(), None) == 1
    # null workspace for the status read
    assert L.rtp_get_device_status(None, None) == 1
    # nothing to do is not an error
    s0 = _shape(B=0)
    assert L.rtp_dense_attn(ctypes.byref(s0), _v(), _v(), _v(), ctypes.c_float(0.1), _v(), None,
                            None, 0, None) == 0


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(rtp, "_lib", None)
    monkeypatch.setattr(rtp, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        rtp.lib()


def test_product_never_reaches_the_oracle(L):
    """The oracle is test infrastructure: no module of the package imports it,
    and librtp.so neither links the oracle's library nor carries its symbols."""
    import ast
    import subprocess
    pkg = os.path.join(ROOT, "long_context_sparse_rtp_b200")
    for name in sorted(os.listdir(pkg)):
        if not name.endswith(".py"):
            continue
        tree = ast.parse(open(os.path.join(pkg, name)).read())
        for node in ast.walk(tree):
            if isinstance(node, ast.Import):
                assert all(a.name.split(".")[0] != "oracle" for a in node.names), name
            elif isinstance(node, ast.ImportFrom):
                assert (node.module or "").split(".")[0] != "oracle", name
    deps = subprocess.run(["ldd", rtp.LIB_PATH], capture_output=True, text=True).stdout
    assert "orc" not in deps
    syms = subprocess.run(["nm", "-D", rtp.LIB_PATH], capture_output=True, text=True).stdout
    assert not any(ln.split()[-1].startswith("orc_") for ln in syms.splitlines() if ln.split())
