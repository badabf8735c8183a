"""The local-head decode entry point that allocates nothing.

Some callers cannot give the library a workspace: they run under a memory
allocator they do not own (a host framework's fixed pool, a plugin interface
that hands over only inputs and outputs) or in a phase where device allocation
is not allowed.  rtp_local_attn_decode_noalloc keeps its scratch in a fixed
8 MiB device array instead.  These tests call it through the C ABI and check it
against rtp_local_attn, which takes a caller workspace, on two calls in a row,
and against the fp64 oracle's sink + window attention.
This file is collected last on purpose, so that a run stopping at the first
failure has run every other test before it.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_rtp_b200 import build, rtp, synth
from rtp_check import LSE_ABS, bits, check_outputs


def _args(inp, q_pos0):
    q, k, v = inp["q"], inp["k"], inp["v"]
    B, _, H, _ = q.shape
    shape = rtp.Shape(B, 1, k.shape[1], H, k.shape[2], 128, q_pos0)
    return q, k, v, shape


def test_rejects_shapes_beyond_the_scratch_array():
    """Host-side check, nothing enqueued: 400 batch entries x 3 local kv heads
    need at least one 8448-byte partial each, ~10 MB, more than the 8 MiB array."""
    build.build()
    L = rtp.lib()
    shape = rtp.Shape(400, 1, 9000, 32, 4, 128, 8999)
    role = (ctypes.c_uint8 * 4)(1, 0, 0, 0)
    v = rtp.View(ctypes.c_void_p(0x10000), 9000 * 4 * 128, 4 * 128)
    vq = rtp.View(ctypes.c_void_p(0x10000), 32 * 128, 32 * 128)
    code = L.rtp_local_attn_decode_noalloc(ctypes.byref(shape), role, 8192, 4, vq, v, v,
                                           ctypes.c_float(0.088), vq, None, None)
    assert rtp.STATUS[code] == "RTP_ERR_SCRATCH_LIMIT"


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    L = rtp.lib()
    w = synth.WORKLOADS["decode_128k_b8"]
    inp = synth.make_inputs(w, "cuda", L=6000, B=2)
    q, k, v, shape = _args(inp, 5999)
    role = inp["kv_role"]
    scale = 1.0 / math.sqrt(128)
    # reference: the workspace entry point
    o_ref, lse_ref = rtp.rtp_local_attn(q, k, v, role, window=w.window, n_sink=w.n_sink,
                                        q_pos0=5999)
    torch.cuda.synchronize()
    loc = w.local_q_heads()
    rarr = (ctypes.c_uint8 * len(role))(*[int(x) for x in role])
    outs = []
    for _ in range(2):  # two calls in a row share the scratch array
        o = torch.zeros_like(q)
        lse = torch.full((q.shape[0], q.shape[2], 1), float("nan"), device=q.device)
        code = L.rtp_local_attn_decode_noalloc(
            ctypes.byref(shape), rarr, w.window, w.n_sink, rtp.view(q), rtp.view(k), rtp.view(v),
            ctypes.c_float(scale), rtp.view(o), ctypes.c_void_p(lse.data_ptr()),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert code == 0, rtp.STATUS.get(code, code)
        torch.cuda.synchronize()
        outs.append((o, lse))
    rows = np.array([(b, 0, h) for b in range(q.shape[0]) for h in loc])
    orc = oracle.local_rows(bits(q), bits(k), bits(v), rows, H=w.H, Hkv=w.Hkv, q_pos0=5999,
                            window=w.window, n_sink=w.n_sink, scale=scale)
    for o, lse in outs:
        a = o[:, 0, loc].float().cpu().numpy().reshape(-1, 128)
        b = o_ref[:, 0, loc].float().cpu().numpy().reshape(-1, 128)
        check_outputs(a, b.astype(np.float64), "no-alloc local decode")
        np.testing.assert_allclose(lse[:, loc].cpu().numpy(), lse_ref[:, loc].cpu().numpy(),
                                   atol=2e-2, rtol=0)
        check_outputs(a, orc["o"], "no-alloc local decode vs the oracle")
        assert np.abs(lse[:, loc, 0].cpu().numpy().reshape(-1) - orc["lse"]).max() <= LSE_ABS
