"""GPU parity of the window-only local-head cache ([FASB §Local Head Attention
Pattern]: at decode the local heads keep only the sink tokens and the sliding
window, so their cache is O(window)).

A ring cache is filled from a prefill, then decode tokens are appended one by
one, far more of them than the ring has rows, so the window wraps around the
ring several times.  Every step's local-head output must equal rtp_local_attn
over the full cache bit for bit (the ring visits the same keys in the same
order), and sampled steps must match the fp64 oracle (max-abs <= 2e-2, mean-abs
<= 2e-3, lse within 2e-2).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_rtp_b200 import (local_ring_alloc, rtp_local_attn,
                                          rtp_local_attn_decode_ring, rtp_local_ring_write, synth)
from rtp_check import LSE_ABS, bits, check_outputs

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)
W = synth.WORKLOADS


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from long_context_sparse_rtp_b200 import build
    build.build()


def run_ring(L, L0, window, n_sink, B=2, check_every=100):
    """Cache of L positions; the ring is written from the first L0 (a prefill),
    then positions L0 .. L-1 are appended and decoded one at a time."""
    w = W["decode_128k_b8"]
    inp = synth.make_inputs(w, "cuda", L=L, B=B)
    k, v, role = inp["k"], inp["v"], inp["kv_role"]
    # one query per step: the generator's decode query, rolled per step so each
    # step attends with a different query
    q_all = torch.randn(L - L0, B, 1, w.H, 128, generator=torch.Generator("cuda").manual_seed(7),
                        device="cuda").to(torch.bfloat16)
    kr, vr = local_ring_alloc(B, role, window=window, n_sink=n_sink, device="cuda")
    assert kr.shape == (B, n_sink + window, 3, 128)
    rtp_local_ring_write(k[:, :L0], v[:, :L0], kr, vr, role, window=window, n_sink=n_sink,
                         pos0=0, H=w.H)
    loc = w.local_q_heads()
    kb, vb = bits(k), bits(v)
    checked = 0
    for step, P in enumerate(range(L0, L)):
        q = q_all[step]
        rtp_local_ring_write(k[:, P:P + 1], v[:, P:P + 1], kr, vr, role, window=window,
                             n_sink=n_sink, pos0=P, H=w.H)
        o1, l1 = rtp_local_attn_decode_ring(q, kr, vr, role, window=window, n_sink=n_sink, pos=P)
        o2, l2 = rtp_local_attn(q, k[:, :P + 1], v[:, :P + 1], role, window=window,
                                n_sink=n_sink, q_pos0=P)
        assert torch.equal(o1[:, :, loc], o2[:, :, loc]), P
        assert torch.equal(l1[:, loc], l2[:, loc]), P
        if step % check_every == 0 or P == L - 1:
            rows = np.array([(b, 0, h) for b in range(B) for h in loc])
            r = oracle.local_rows(bits(q), kb[:, :P + 1], vb[:, :P + 1], rows, H=w.H, Hkv=w.Hkv,
                                  q_pos0=P, window=window, n_sink=n_sink, scale=SCALE)
            og = o1.float().cpu().numpy()
            lg = l1.cpu().numpy()
            check_outputs(np.stack([og[b, 0, h] for (b, _, h) in rows]), r["o"], f"ring P={P}")
            assert np.abs(np.array([lg[b, h, 0] for (b, _, h) in rows]) - r["lse"]).max() <= LSE_ABS
            checked += 1
    torch.cuda.synchronize()
    return checked


def test_ring_wraps_small_window():
    """Window 256 + 4 sinks: 1200 appends wrap the 256-row ring four times; the
    prefill part is shorter than the sinks plus the window, so the first steps
    also cover a ring that is not full yet."""
    assert run_ring(L=1300, L0=100, window=256, n_sink=4, check_every=50) >= 20


def test_ring_wraps_decode_window():
    """The decode workload's window (4096 + 4 sinks) on a 16K cache: the ring is
    written from a 6K prefill, then 10K appends wrap it about 2.5 times."""
    assert run_ring(L=16384, L0=6000, window=4096, n_sink=4, check_every=1000) >= 10


def test_ring_no_sinks_and_one_token_window():
    """Edge cases: no sink tokens; a one-token window (the query's own key)."""
    run_ring(L=300, L0=1, window=1, n_sink=0, check_every=60)
    run_ring(L=300, L0=10, window=37, n_sink=0, check_every=60)
