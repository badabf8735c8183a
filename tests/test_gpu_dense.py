"""GPU parity of the dense causal baseline (rtp_dense_attn) and of the
summary's own prefill (retrieval heads dense, local heads sparse) against the
fp64 oracle.

The dense kernel is the denominator of every speed-up this library reports, so
it is checked against the oracle directly, not only against other CUDA paths:
every key 0..P of every head ([FASB §Dynamic Top-p Selection Mechanism], the
attention formula with S = all causal keys).  Tolerances: max-abs <= 2e-2 and
mean-abs <= 2e-3 on O (bf16 in, fp32 accumulation), lse within 2e-2.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_rtp_b200 import (rtp_dense_attn, rtp_index_scores, rtp_layer_prefill,
                                          synth)
from rtp_check import LSE_ABS, bits, check_outputs
from test_gpu_prefill import check_projection, run_prefill

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)
W = synth.WORKLOADS


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from long_context_sparse_rtp_b200 import build
    build.build()


def check_dense_rows(q, k, v, o, lse, positions, q_pos0, what):
    """Every head of the sampled query rows `positions` (indices into q's rows)
    against oracle.dense_rows; only those rows travel to the host."""
    B, _, H, _ = q.shape
    Hkv = k.shape[2]
    pidx = torch.as_tensor(np.asarray(positions), device=q.device)
    qb = bits(q[:, pidx])
    kb, vb = bits(k), bits(v)
    og = o[:, pidx].float().cpu().numpy()
    lg = lse[:, :, pidx].cpu().numpy()
    errs, lerr = [], 0.0
    for x, i in enumerate(positions):
        rows = np.array([(b, 0, h) for b in range(B) for h in range(H)])
        r = oracle.dense_rows(qb[:, x:x + 1], kb, vb, rows, H=H, Hkv=Hkv,
                              q_pos0=int(q_pos0 + i), scale=SCALE)
        errs.append((np.stack([og[b, x, h] for (b, _, h) in rows]), r["o"]))
        lerr = max(lerr, float(np.abs(np.array([lg[b, h, x] for (b, _, h) in rows])
                                      - r["lse"]).max()))
    mx, mean = check_outputs(np.concatenate([a for a, _ in errs]),
                             np.concatenate([b for _, b in errs]), what)
    assert lerr <= LSE_ABS, (what, lerr)
    return mx, mean, lerr


@pytest.mark.parametrize("L", [1, 63, 65, 130, 1000])
def test_dense_prefill_every_row(L):
    """Causal prefill, batch 2, 8 q / 2 kv heads: every row of every head,
    lengths that fill no tile, cross a 64-key half-tile and a 128-key tile."""
    inp = synth.make_inputs(W["prefill_2k"], "cuda", L=L, B=2)
    q, k, v = inp["q"], inp["k"], inp["v"]
    o, lse = rtp_dense_attn(q, k, v)
    torch.cuda.synchronize()
    check_dense_rows(q, k, v, o, lse, list(range(L)), 0, f"dense prefill L={L}")


def _edge_rows(L, rng, n_random):
    edge = [0, 1, 2, 63, 64, 65, 127, 128, 129, 255, 256, 1023, 1024, L // 2, L - 129,
            L - 128, L - 127, L - 2, L - 1]
    return sorted(set(int(x) for x in edge + list(rng.integers(0, L, n_random))
                      if 0 <= x < L))


@pytest.mark.slow
@pytest.mark.parametrize("name", ["prefill_32k", "prefill_128k"])
def test_dense_prefill_full_size_sampled_rows(name):
    """The 32K and 128K workloads at full length, all 32 heads, on the first,
    last and tile-edge rows plus a seeded random sample."""
    w = W[name]
    inp = synth.make_inputs(w, "cuda")
    q, k, v = inp["q"], inp["k"], inp["v"]
    o, lse = rtp_dense_attn(q, k, v)
    torch.cuda.synchronize()
    rows = _edge_rows(w.L, np.random.default_rng(40), 6)
    check_dense_rows(q, k, v, o, lse, rows, 0, f"dense prefill {name}")


@pytest.mark.parametrize("L", [1, 4100, 131072])
def test_dense_decode(L):
    """One query row per batch entry at position L - 1 against the whole cache,
    every query head (split-KV over the full range, then the split merge); the
    128K case is the decode workload's full batch of 8."""
    B = 8 if L == 131072 else 2
    inp = synth.make_inputs(W["decode_128k_b8"], "cuda", L=L, B=B)
    q, k, v = inp["q"], inp["k"], inp["v"]
    o, lse = rtp_dense_attn(q, k, v, q_pos0=L - 1)
    torch.cuda.synchronize()
    check_dense_rows(q, k, v, o, lse, [0], L - 1, f"dense decode L={L}")


def test_dense_retrieval_prefill_pages_mode():
    """The summary's own prefill: retrieval heads attend to every causal key,
    local heads to sinks + window, with the indexer on pre-RoPE vectors building
    the k16 cache for decode.  The 2K workload, every row of every head, against
    the oracle (dense rows on retrieval heads, local rows on local heads); the
    retrieval heads equal the top-p path at p = 1 bit for bit."""
    w = W["prefill_2k"]
    L = 2048
    inp = synth.make_inputs(w, "cuda", L=L, indexer_input="pre")
    q, k, v, Wq, Wk, role = (inp[x] for x in ("q", "k", "v", "Wq16", "Wk16", "kv_role"))
    res = rtp_layer_prefill(q, k, v, Wq, Wk, role, p=w.p, window=w.window, n_sink=w.n_sink,
                            retrieval="dense", q_idx=inp["q_idx"], k_idx=inp["k_idx"])
    ref = rtp_layer_prefill(q, k, v, Wq, Wk, role, p=1.0, window=w.window, n_sink=w.n_sink,
                            q_idx=inp["q_idx"], k_idx=inp["k_idx"])
    torch.cuda.synchronize()
    assert res["sel"] is None and res["q16"] is None
    assert torch.equal(res["o"], ref["o"]) and torch.equal(res["lse"], ref["lse"])
    assert torch.equal(res["k16"], ref["k16"])
    # the k16 cache is the projection of the pre-RoPE keys
    kib, Wkb = bits(inp["k_idx"]), bits(Wk)
    ret, loc = w.retrieval_q_heads(), w.local_q_heads()
    k16g = bits(res["k16"])
    for s, h in enumerate(ret):
        check_projection(k16g[0, :, s], kib[0, :, h // w.G], Wkb[s])
    qb, kb, vb = bits(q), bits(k), bits(v)
    og = res["o"].float().cpu().numpy()
    lg = res["lse"].cpu().numpy()
    rows = np.array([(0, i, h) for i in range(L) for h in ret])
    rd = oracle.dense_rows(qb, kb, vb, rows, H=w.H, Hkv=w.Hkv, q_pos0=0, scale=SCALE)
    check_outputs(np.stack([og[0, i, h] for (_, i, h) in rows]), rd["o"], "retrieval dense")
    assert np.abs(np.array([lg[0, h, i] for (_, i, h) in rows]) - rd["lse"]).max() <= LSE_ABS
    lrows = np.array([(0, i, h) for i in range(L) for h in loc])
    rl = oracle.local_rows(qb, kb, vb, lrows, H=w.H, Hkv=w.Hkv, q_pos0=0, window=w.window,
                           n_sink=w.n_sink, scale=SCALE)
    check_outputs(np.stack([og[0, i, h] for (_, i, h) in lrows]), rl["o"], "local")


def test_pre_rope_indexer_prefill_topp():
    """Exact top-p prefill with the indexer on pre-RoPE q, k and attention on
    post-RoPE q, k: the full parity protocol (projection, selection, outputs)
    on the 2K workload, every row."""
    run_prefill(W["prefill_2k"], 2048, 0.9, indexer_input="pre")


def test_index_scores_keys_only():
    """k16 alone (no query rows) equals the k16 half of a joint projection."""
    w = W["prefill_2k"]
    inp = synth.make_inputs(w, "cuda", L=500)
    q, k, Wq, Wk, role = (inp[x] for x in ("q", "k", "Wq16", "Wk16", "kv_role"))
    _, k16a = rtp_index_scores(q, k, Wq, Wk, role)
    _, k16b = rtp_index_scores(None, k, Wq, Wk, role, H=w.H)
    torch.cuda.synchronize()
    assert torch.equal(k16a, k16b)


def check_local_rows(q, k, v, o, lse, role, window, n_sink, q_pos0, what):
    """Every local head of every query row against oracle.local_rows."""
    B, Lq, H, _ = q.shape
    Hkv = k.shape[2]
    G = H // Hkv
    loc = [h for h in range(H) if role[h // G] == 0]
    qb, kb, vb = bits(q), bits(k), bits(v)
    og = o.float().cpu().numpy()
    lg = lse.cpu().numpy()
    got, ref, lerr = [], [], 0.0
    for i in range(Lq):
        rows = np.array([(b, 0, h) for b in range(B) for h in loc])
        r = oracle.local_rows(qb[:, i:i + 1], kb, vb, rows, H=H, Hkv=Hkv, q_pos0=q_pos0 + i,
                              window=window, n_sink=n_sink, scale=SCALE)
        got.append(np.stack([og[b, i, h] for (b, _, h) in rows]))
        ref.append(r["o"])
        lerr = max(lerr, float(np.abs(np.array([lg[b, h, i] for (b, _, h) in rows])
                                      - r["lse"]).max()))
    check_outputs(np.concatenate(got), np.concatenate(ref), what)
    assert lerr <= LSE_ABS, (what, lerr)


@pytest.mark.parametrize("Lq", [77, 256, 333])
def test_chunked_prefill_dense_every_row(Lq):
    """A prefill chunk: Lq query rows at positions 300 .. 300 + Lq - 1 over a
    cache of 300 + Lq keys, batch 2.  The kernel holds 256 query rows per CTA as
    two 128-row tiles: 77 rows leave the second tile empty, 333 leave the last
    CTA's second tile part-filled, and position 300 is not tile-aligned."""
    q_pos0 = 300
    inp = synth.make_inputs(W["prefill_2k"], "cuda", L=q_pos0 + Lq, B=2)
    q = inp["q"][:, q_pos0:].contiguous()
    k, v = inp["k"], inp["v"]
    o, lse = rtp_dense_attn(q, k, v, q_pos0=q_pos0)
    torch.cuda.synchronize()
    check_dense_rows(q, k, v, o, lse, list(range(Lq)), q_pos0, f"dense chunk Lq={Lq}")


@pytest.mark.parametrize("window,n_sink", [(5, 0), (100, 4), (200, 130), (700, 0)])
def test_chunked_prefill_local_every_row(window, n_sink):
    """Sinks + sliding window on a prefill chunk (300 rows at positions 300 ..
    599 over 600 keys, batch 2): windows narrower than a tile, sinks that span
    more than one 128-key tile, a window wider than the whole cache, no sinks."""
    from long_context_sparse_rtp_b200 import rtp_local_attn
    q_pos0, Lq = 300, 300
    w = W["prefill_2k"]
    inp = synth.make_inputs(w, "cuda", L=q_pos0 + Lq, B=2)
    q = inp["q"][:, q_pos0:].contiguous()
    k, v, role = inp["k"], inp["v"], inp["kv_role"]
    o, lse = rtp_local_attn(q, k, v, role, window=window, n_sink=n_sink, q_pos0=q_pos0)
    torch.cuda.synchronize()
    check_local_rows(q, k, v, o, lse, [int(x) for x in role], window, n_sink, q_pos0,
                     f"local chunk window={window} sinks={n_sink}")
