"""The seeded input generator (no GPU): RoPE property, determinism, shapes."""
import numpy as np
import torch

from long_context_sparse_rtp_b200 import synth


def test_rope_depends_only_on_offset():
    """Eq. 1/2 of the RoPE section of the paper-graph-ui summary: after the
    rotation, q_m . k_n depends on the content and on m - n only."""
    g = torch.Generator().manual_seed(0)
    q = torch.randn(1, 1, 128, generator=g)
    k = torch.randn(1, 1, 128, generator=g)
    def dot(m, n):
        return float((synth.rope(q, m) * synth.rope(k, n)).double().sum())
    for m, n, shift in [(10, 3, 1000), (5000, 17, 12345), (100, 100, 77777)]:
        assert abs(dot(m, n) - dot(m + shift, n + shift)) < 2e-3
    # and it is not position-free: a different offset changes the score
    assert abs(dot(10, 3) - dot(10, 4)) > 1e-3


def test_rope_is_a_rotation():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(64, 2, 128, generator=g)
    y = synth.rope(x, 123)
    torch.testing.assert_close(y.norm(dim=-1), x.norm(dim=-1), rtol=1e-5, atol=1e-5)


def test_make_inputs_deterministic_and_shaped():
    w = synth.WORKLOADS["prefill_2k"]
    a = synth.make_inputs(w, "cpu", L=256)
    b = synth.make_inputs(w, "cpu", L=256)
    for key in ("q", "k", "v", "Wq16", "Wk16"):
        assert torch.equal(a[key], b[key])
    assert a["q"].shape == (1, 256, 8, 128) and a["k"].shape == (1, 256, 2, 128)
    assert a["Wq16"].shape == (4, 128, 16)
    assert list(a["kv_role"]) == [1, 0]
    d = synth.make_inputs(synth.WORKLOADS["decode_128k_b8"], "cpu", L=512, B=2)
    assert d["q"].shape == (2, 1, 32, 128) and d["k"].shape == (2, 512, 4, 128)
    assert d["q_pos0"] == 511 and d["Lq"] == 1


def test_needles_raise_indexer_scores():
    """A planted needle key scores far above the background for its query."""
    w = synth.WORKLOADS["decode_128k_b8"]
    inp = synth.make_inputs(w, "cpu", L=4096, B=2)
    Wq = inp["Wq16"].double()
    Wk = inp["Wk16"].double()
    q = inp["q"].double()
    k = inp["k"].double()
    hits = 0
    for b in range(2):
        for slot in range(w.H_ret):
            q16 = q[b, 0, slot] @ Wq[slot]
            s = (k[b, :, 0] @ Wk[slot]) @ q16
            z = (s - s.mean()) / s.std()
            hits += int((z > 3).sum())
    assert hits > 20
