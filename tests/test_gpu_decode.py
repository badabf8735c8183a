"""GPU parity: one decode token (retrieval heads: exact top-p over the k16
cache + union gather; local heads: sinks + window) against the fp64 oracle,
plus GPU self-consistency (decode == last prefill row, p = 1 == dense,
window >= L == dense, bitwise-repeatable runs)."""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_rtp_b200 import (rtp_dense_attn, rtp_index_scores, rtp_layer_decode,
                                          rtp_layer_prefill, rtp_local_attn,
                                          rtp_sparse_attn_decode, rtp_sparse_attn_prefill,
                                          rtp_topp_select, synth)
from rtp_check import (LSE_ABS, bits, check_outputs, check_row_outputs, check_row_selection,
                       gpu_kept, row_reference,
                       oracle_k16, row_scores)

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)
W = synth.WORKLOADS


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from long_context_sparse_rtp_b200 import build
    build.build()


def gpu_decode(inp, w, p, per_kv=False):
    q, k, v = inp["q"], inp["k"], inp["v"]
    Wq, Wk = inp["Wq16"], inp["Wk16"]
    if per_kv:
        Wk = Wk[[s for s in range(0, w.H_ret, w.G)]].contiguous()
    role = inp["kv_role"]
    q16, k16 = rtp_index_scores(inp.get("q_idx", q), inp.get("k_idx", k), Wq, Wk, role,
                                k16_per_kv_head=int(per_kv))
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], w.H, 1, dtype=torch.float32, device=q.device)
    _, _, sel = rtp_sparse_attn_decode(q, k, v, q16, k16, role, p, k16_per_kv_head=int(per_kv),
                                       o=o, lse=lse)
    rtp_local_attn(q, k, v, role, window=w.window, n_sink=w.n_sink, q_pos0=k.shape[1] - 1, o=o,
                   lse=lse)
    torch.cuda.synchronize()
    return q16, k16, o, lse, sel, Wk


def run_decode(w, L, B, p, per_kv=False, seed=None, indexer_input="post"):
    if seed is not None:
        w = w.with_(seed=seed)
    inp = synth.make_inputs(w, "cuda", L=L, B=B, indexer_input=indexer_input)
    q16, k16, o, lse, sel, Wk = gpu_decode(inp, w, p, per_kv)
    p = float(np.float32(p))
    qb, kb, vb = bits(inp["q"]), bits(inp["k"]), bits(inp["v"])
    qib = bits(inp["q_idx"]) if "q_idx" in inp else qb
    kib = bits(inp["k_idx"]) if "k_idx" in inp else kb
    Wqb, Wkb = bits(inp["Wq16"]), bits(Wk)
    q16g, k16g = bits(q16), bits(k16)
    sel = {key: val.cpu().numpy() for key, val in sel.items()}
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    ret, loc = w.retrieval_q_heads(), w.local_q_heads()
    k16slot = [s // w.G for s in range(w.H_ret)] if per_kv else list(range(w.H_ret))
    P = L - 1
    rows = np.array([(b, 0, h) for b in range(B) for h in ret])
    slots = np.array([s for b in range(B) for s in range(len(ret))])
    ks = np.array(k16slot)[slots]
    # (ii) selection on the GPU's q16/k16
    r2 = oracle.retrieval_rows(qb, kb, vb, q16g, k16g, rows, slots, ks, H=w.H, Hkv=w.Hkv,
                               q_pos0=P, p=p, scale=SCALE, want_sel=True)
    n_band = 0
    kept = []
    for r, (b, _, h) in enumerate(rows):
        s = slots[r]
        s64 = row_scores(q16g[b, 0, s], k16g[b, :, k16slot[s]], P)
        n_band += check_row_selection(s64, p, r2["t"][r], r2["sel"][r], float(sel["thr"][b, s]),
                                      int(sel["jtie"][b, s]), int(sel["count"][b, s]),
                                      float(sel["mass"][b, s]))
        kept.append(gpu_kept(q16g[b, 0, s], k16g[b, :, k16slot[s]], P, float(sel["thr"][b, s]),
                             int(sel["jtie"][b, s]), int(sel["count"][b, s]), p))
    # (iii) end to end with the oracle's own projections
    q16o = np.zeros_like(q16g)
    for b in range(B):
        for s, h in enumerate(ret):
            q16o[b, 0, s] = oracle.project(qib[b, 0, h][None], Wqb[s])[0][0]
    k16o = oracle_k16(kib, Wkb, w, per_kv)
    r3 = oracle.retrieval_rows(qb, kb, vb, q16o, k16o, rows, slots, ks, H=w.H, Hkv=w.Hkv,
                               q_pos0=P, p=p, scale=SCALE, want_sel=True)
    og = np.stack([o[b, 0, h] for (b, _, h) in rows])
    o_ref, lse_ref, ref_ok, e2e_ok = [], [], [], []
    for r, (b, _, h) in enumerate(rows):
        g = h // w.G
        a, l_, ok, ok2 = row_reference(qb[b, 0, h], kb[b, :P + 1, g], vb[b, :P + 1, g], kept[r],
                                       r2["sel"][r], r2["o"][r], r2["lse"][r], r3["sel"][r],
                                       SCALE)
        o_ref.append(a)
        lse_ref.append(l_)
        ref_ok.append(ok)
        e2e_ok.append(ok2)
    stats = check_row_outputs(og, np.stack(o_ref), ref_ok, r3["o"], e2e_ok,
                              f"retrieval decode L={L} B={B} p={p}")
    lg = np.array([lse[b, h, 0] for (b, _, h) in rows])
    assert np.abs(lg - np.array(lse_ref))[np.array(ref_ok)].max(initial=0.0) <= LSE_ABS
    if loc:
        lrows = np.array([(b, 0, h) for b in range(B) for h in loc])
        rl = oracle.local_rows(qb, kb, vb, lrows, H=w.H, Hkv=w.Hkv, q_pos0=P, window=w.window,
                               n_sink=w.n_sink, scale=SCALE)
        check_outputs(np.stack([o[b, 0, h] for (b, _, h) in lrows]), rl["o"], "local decode")
        assert np.abs(np.array([lse[b, h, 0] for (b, _, h) in lrows]) - rl["lse"]).max() <= LSE_ABS
    return dict(n_band=n_band, stats=stats)


@pytest.mark.parametrize("L", [1, 5, 1023, 1025, 4100, 8192])
@pytest.mark.parametrize("p", [0.0, 0.9, 0.95, 1.0])
def test_decode_small(L, p):
    run_decode(W["decode_128k_b8"], L, 2, p)


def test_decode_per_kv_k16():
    run_decode(W["decode_128k_b8"], 6000, 2, 0.95, per_kv=True)


def test_decode_pre_rope_indexer():
    """The indexer projects the pre-RoPE q, k (the summary's projection input)
    while attention uses the post-RoPE ones; the oracle takes the same split."""
    run_decode(W["decode_128k_b8"], 6000, 2, 0.95, indexer_input="pre")


@pytest.mark.parametrize("H", [4, 8, 16, 64])
@pytest.mark.parametrize("per_kv", [False, True])
def test_decode_head_groups(H, per_kv):
    """G = H / 4 query heads per kv head in {1, 2, 4, 16}, k16 per query head or per kv head."""
    run_decode(W["decode_128k_b8"].with_(H=H), 3000, 2, 0.9, per_kv=per_kv)


def test_decode_128k_batch8_full():
    """The full 128K x batch-8 decode workload: every row of every head, and at
    most one of its 64 retrieval rows left out of either output check."""
    st = run_decode(W["decode_128k_b8"], 131072, 8, 0.95)["stats"]
    assert st["skip_ref"] <= 1 and st["skip_e2e"] <= 1, st


def test_decode_equals_last_prefill_row():
    w = W["prefill_2k"]
    L = 777
    inp = synth.make_inputs(w, "cuda", L=L)
    q, k, v, Wq, Wk, role = (inp[x] for x in ("q", "k", "v", "Wq16", "Wk16", "kv_role"))
    pre = rtp_layer_prefill(q, k, v, Wq, Wk, role, p=0.9, window=w.window, n_sink=w.n_sink)
    # decode of the last row through the layer API (writes the new k16 row into the cache)
    k16_cache = pre["k16"].clone()
    k16_cache[:, L - 1] = 0
    dec = rtp_layer_decode(q[:, L - 1:], k[:, L - 1:], k, v, k16_cache, Wq, Wk, role, pos=L - 1,
                           p=0.9, window=w.window, n_sink=w.n_sink)
    torch.cuda.synchronize()
    assert torch.equal(k16_cache, pre["k16"])
    # both phases score a key by one 16-term tensor-core dot product of the same
    # bf16 q16 and k16 with fp32 accumulation (decode's other slots add exact
    # zeros), so they see identical scores; each sums fixed-point masses on its
    # own bin grid, which agree to ~1e-6 relative, so the cut could move only
    # for a row whose cumulative mass passes p * Z within that margin (none of
    # these rows): the same row gets the same threshold, tie index and count
    for key in ("thr", "jtie", "count"):
        assert torch.equal(dec["sel"][key], pre["sel"][key][:, :, L - 1]), key
    torch.testing.assert_close(dec["o"][:, 0].float(), pre["o"][:, L - 1].float(), atol=2e-2,
                               rtol=0)


def test_p1_equals_dense_and_wide_window_equals_dense():
    w = W["prefill_2k"]
    inp = synth.make_inputs(w, "cuda", L=1111)
    q, k, v, Wq, Wk, role = (inp[x] for x in ("q", "k", "v", "Wq16", "Wk16", "kv_role"))
    dense, dlse = rtp_dense_attn(q, k, v)
    sp = rtp_layer_prefill(q, k, v, Wq, Wk, role, p=1.0, window=1111, n_sink=0)
    torch.cuda.synchronize()
    torch.testing.assert_close(sp["o"].float(), dense.float(), atol=0, rtol=0)
    torch.testing.assert_close(sp["lse"], dlse, atol=0, rtol=0)
    # decode flavour
    d = synth.make_inputs(W["decode_128k_b8"], "cuda", L=3000, B=2)
    q, k, v = d["q"], d["k"], d["v"]
    o1, l1 = rtp_dense_attn(q, k, v, q_pos0=2999)
    o2 = torch.empty_like(q)
    rtp_local_attn(q, k, v, [0, 0, 0, 0], window=5000, n_sink=0, q_pos0=2999, o=o2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_repeatable_bitwise():
    w = W["prefill_2k"]
    inp = synth.make_inputs(w, "cuda", L=1500)
    args = [inp[x] for x in ("q", "k", "v", "Wq16", "Wk16", "kv_role")]
    a = rtp_layer_prefill(*args, p=0.9, window=w.window, n_sink=w.n_sink)
    b = rtp_layer_prefill(*args, p=0.9, window=w.window, n_sink=w.n_sink)
    torch.cuda.synchronize()
    for key in ("o", "lse", "q16", "k16"):
        assert torch.equal(a[key], b[key]), key
    for key in ("thr", "jtie", "count", "mass"):
        assert torch.equal(a["sel"][key], b["sel"][key]), key
    d = synth.make_inputs(W["decode_128k_b8"], "cuda", L=20000, B=2)
    r1 = gpu_decode(d, W["decode_128k_b8"], 0.95)
    r2 = gpu_decode(d, W["decode_128k_b8"], 0.95)
    assert torch.equal(r1[2], r2[2]) and torch.equal(r1[3], r2[3])
    for key in ("thr", "jtie", "count", "mass"):
        assert torch.equal(r1[4][key], r2[4][key]), key


def test_decode_graph_matches_eager():
    """DecodeGraph replays the same kernels as the eager layer call."""
    from long_context_sparse_rtp_b200 import DecodeGraph
    w = W["decode_128k_b8"]
    d = synth.make_inputs(w, "cuda", L=5000, B=2)
    q, k, v, Wq, Wk, role = (d[x] for x in ("q", "k", "v", "Wq16", "Wk16", "kv_role"))
    _, k16 = rtp_index_scores(q, k, Wq, Wk, role)
    eager = rtp_layer_decode(q, k[:, 4999:], k, v, k16.clone(), Wq, Wk, role, pos=4999, p=w.p,
                             window=w.window, n_sink=w.n_sink)
    g = DecodeGraph(k, v, k16, Wq, Wk, role, H=w.H, pos=4999, p=w.p, window=w.window,
                    n_sink=w.n_sink)
    g.q.copy_(q)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(g.o, eager["o"])
        assert torch.equal(g.lse, eager["lse"])
    hq = q.cpu().pin_memory()
    hk = k[:, 4999:].cpu().pin_memory()
    hv = v[:, 4999:].cpu().pin_memory()
    ho = torch.empty_like(hq).pin_memory()
    for _ in range(2):  # captures the copies with the step, then replays that graph
        ho.zero_()
        g.step(hq, hk, hv, ho)
        torch.cuda.synchronize()
        assert torch.equal(ho, eager["o"].cpu())
    ho2 = torch.empty_like(hq).pin_memory()  # other buffers: copies around the graph
    g.step(hq, hk, hv, ho2)
    torch.cuda.synchronize()
    assert torch.equal(ho2, eager["o"].cpu())


def test_decode_all_scores_equal_beyond_candidate_cap():
    """W_q16 = 0 with a 9000-token cache: every key ties, so the crossing bin
    holds more keys than one sort resolves (4096) and the row takes the radix
    refinement over the stored scores; the cut is the ceil(p * N)-th index."""
    w = W["decode_128k_b8"]
    L = 9000
    inp = synth.make_inputs(w, "cuda", L=L, B=2)
    inp["Wq16"] = torch.zeros_like(inp["Wq16"])
    for p in (0.5, 0.95):
        _, _, o, lse, sel, _ = gpu_decode(inp, w, p)
        n = int(np.maximum(1, np.ceil(float(np.float32(p)) * L)))
        assert np.all(sel["count"].cpu().numpy() == n)
        assert np.all(sel["jtie"].cpu().numpy() == n - 1)
        assert np.all(sel["thr"].cpu().numpy() == 0.0)
