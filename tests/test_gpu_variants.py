"""GPU parity of the decode selection variants against the fp64 oracle:
static top-k ([FASB §5 Experimental Analysis], the method's fixed-budget
variant) and block-level approximate top-p ([FASB §Hardware-Aware Fast Top-p
Decoding Kernel], steps 1-5), both through rtp_sparse_attn_decode_select.

Protocol, per retrieval row:
 (i)   the scores the call returns are the GPU's fp32 indexer scores: each
       within the fp32 accumulation bound 17 u sum |q16||k16| of the fp64 dot
       product of the GPU's own q16, k16;
 (ii)  the oracle's rule run on those very fp32 scores gives the GPU's
       selection: top-k bit for bit (thr, jtie, count and the kept set, since
       the cut is decided on integer counts); block top-p block for block,
       except that a row whose running bin mass passes p within 1e-5 relative
       may take the neighbouring bin (the GPU sums exp in fp32, the oracle in
       fp64);
 (iii) outputs: max-abs <= 2e-2, mean-abs <= 2e-3 against the oracle's exact
       attention over the GPU's kept keys (known exactly from (ii)), lse within
       2e-2; end to end against the oracle with its own projections on the rows
       whose kept set differs from the GPU's by at most 1e-3 of the attention
       mass (a key near the cut or a block max near a bin edge may go either
       way), with the share of such rows bounded.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_rtp_b200 import (rtp_index_scores, rtp_sparse_attn_decode,
                                          rtp_sparse_attn_decode_select, synth)
from rtp_check import (LSE_ABS, SEL_BAND, _mass_share, bits, check_outputs, f64, oracle_k16,
                       report)

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)
W = synth.WORKLOADS
MARGIN = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from long_context_sparse_rtp_b200 import build
    build.build()


def _block_mask_bits(words, nb):
    w = np.asarray(words, np.int64) & 0xFFFFFFFF
    bitsv = (w[:, None] >> np.arange(32)[None, :]) & 1
    return bitsv.reshape(-1)[:nb].astype(bool)


def run_variant(select, L, B, *, p=0.95, top_k=4096, w=None, per_kv=False, max_e2e_skip=0.05):
    w = W["decode_128k_b8"] if w is None else w
    inp = synth.make_inputs(w, "cuda", L=L, B=B)
    q, k, v, Wq, Wk, role = (inp[x] for x in ("q", "k", "v", "Wq16", "Wk16", "kv_role"))
    if per_kv:
        Wk = Wk[[s for s in range(0, w.H_ret, w.G)]].contiguous()
    q16, k16 = rtp_index_scores(q, k, Wq, Wk, role, k16_per_kv_head=int(per_kv))
    o = torch.zeros_like(q)
    o, lse, sel = rtp_sparse_attn_decode_select(q, k, v, q16, k16, role, select, p=p,
                                                top_k=top_k, k16_per_kv_head=int(per_kv), o=o,
                                                want_scores=True)
    torch.cuda.synchronize()
    P = L - 1
    n = P + 1
    pf = float(np.float32(p))
    qb, kb, vb = bits(q), bits(k), bits(v)
    q16g, k16g = bits(q16), bits(k16)
    Wqb, Wkb = bits(Wq), bits(Wk)
    sc = sel["scores"].cpu().numpy().astype(np.float64)
    cnt = sel["count"].cpu().numpy()
    thr = sel["thr"].cpu().numpy()
    jt = sel["jtie"].cpu().numpy()
    bm = sel["block_mask"].cpu().numpy() if "block_mask" in sel else None
    og = o.float().cpu().numpy()
    lg = lse.cpu().numpy()
    ret = w.retrieval_q_heads()
    k16slot = [s // w.G for s in range(w.H_ret)] if per_kv else list(range(w.H_ret))
    k16o = oracle_k16(kb, Wkb, w, per_kv)
    nb = (n + 63) // 64
    o_gpu, o_ref, o_e2e, e2e_ok, lse_err, n_margin = [], [], [], [], 0.0, 0
    for b in range(B):
        for s, h in enumerate(ret):
            g = h // w.G
            s32 = sc[b, s]
            # (i) the returned scores are the GPU's indexer scores
            qv, kv = f64(q16g[b, 0, s]), f64(k16g[b, :n, k16slot[s]])
            s64 = kv @ qv
            bound = 17 * 2.0 ** -24 * (np.abs(kv) @ np.abs(qv))
            assert np.all(np.abs(s32 - s64) <= bound), (b, s)
            # (ii) the oracle's rule on the same fp32 scores
            if select == "topk":
                r = oracle.topk(s32, top_k)
                kept = r["sel"]
                assert cnt[b, s] == r["count"] == min(top_k, n)
                if top_k >= n:
                    assert thr[b, s] == -math.inf and jt[b, s] == n - 1
                else:
                    assert float(thr[b, s]) == r["t"] and jt[b, s] == r["jtie"], (b, s)
                # on the fp64 scores of the same q16/k16: equal outside the band
                r64 = oracle.topk(s64, top_k)
                if top_k < n:
                    band = np.abs(s64 - r64["t"]) <= SEL_BAND * max(abs(r64["t"]), 1.0)
                    assert np.array_equal(kept[~band], r64["sel"][~band]), (b, s)
            else:
                r = oracle.block_topp(s32, pf)
                got = _block_mask_bits(bm[b, s], nb)
                if not np.array_equal(got, r["bsel"]):
                    alt = [oracle.block_topp(s32, pf * (1 + d))["bsel"] for d in (-MARGIN, MARGIN)]
                    assert any(np.array_equal(got, a) for a in alt), (b, s)
                    n_margin += 1
                kept = np.repeat(got, 64)[:n]
                assert cnt[b, s] == int(kept.sum())
            # (iii) outputs over the GPU's kept keys
            idx = np.nonzero(kept)[0]
            oa, la = oracle.attend(qb[b, 0, h], kb[b, :n, g], vb[b, :n, g], idx, SCALE)
            o_gpu.append(og[b, 0, h])
            o_ref.append(oa)
            lse_err = max(lse_err, abs(float(lg[b, h, 0]) - la))
            # end to end: the oracle's own projections and fp64 scores
            q16o = oracle.project(qb[b, 0, h][None], Wqb[s])[0][0]
            so = oracle.scores(q16o, k16o[b, :n, k16slot[s]])
            ko = (oracle.topk(so, top_k)["sel"] if select == "topk"
                  else oracle.block_topp(so, pf)["sel"])
            ok = _mass_share(qb[b, 0, h], kb[b, :n, g], vb[b, :n, g], kept ^ ko, kept | ko,
                             SCALE) <= 1e-3
            e2e_ok.append(ok)
            o_e2e.append(oracle.attend(qb[b, 0, h], kb[b, :n, g], vb[b, :n, g],
                                       np.nonzero(ko)[0], SCALE)[0])
    o_gpu, o_ref, o_e2e = np.stack(o_gpu), np.stack(o_ref), np.stack(o_e2e)
    e2e_ok = np.array(e2e_ok)
    mx, mean = check_outputs(o_gpu, o_ref, f"{select} vs oracle on the GPU's kept keys")
    assert lse_err <= LSE_ABS, lse_err
    assert (~e2e_ok).sum() <= max(2, max_e2e_skip * len(e2e_ok)), int((~e2e_ok).sum())
    check_outputs(o_gpu[e2e_ok], o_e2e[e2e_ok], f"{select} vs oracle end to end")
    # the local heads are not touched
    loc = w.local_q_heads()
    assert not og[:, 0, loc].any()
    stats = dict(rows=len(e2e_ok), skip_e2e=int((~e2e_ok).sum()), max_abs=mx, mean_abs=mean,
                 margin_rows=n_margin)
    report(f"decode {select} L={L} B={B} p={p} k={top_k}", stats)
    return dict(sel=sel, o=o, lse=lse, stats=stats, inp=inp, q16=q16, k16=k16)


@pytest.mark.parametrize("L", [1, 65, 4100])
@pytest.mark.parametrize("k", [1, 64, 4096])
def test_topk_small(L, k):
    run_variant("topk", L, 2, top_k=k)


@pytest.mark.parametrize("L", [1, 65, 4100, 9000])
@pytest.mark.parametrize("p", [0.0, 0.9, 0.95, 1.0])
def test_block_topp_small(L, p):
    run_variant("block_topp", L, 2, p=p)


def test_topk_many_candidates():
    """k inside a crowd: 20K keys with k = 10000, so the radix levels run before
    the final sort (more than 4096 keys share the first digits)."""
    run_variant("topk", 20000, 2, top_k=10000)


@pytest.mark.parametrize("select", ["topk", "block_topp"])
def test_variants_head_groups_and_per_kv(select):
    run_variant(select, 3000, 2, w=W["decode_128k_b8"].with_(H=16), per_kv=True)


@pytest.mark.parametrize("select", ["topk", "block_topp"])
def test_variants_128k_batch8_full(select):
    """The 128K x batch-8 decode workload, every retrieval row."""
    run_variant(select, 131072, 8)


def test_select_topp_equals_decode():
    """RTP_SELECT_TOPP is rtp_sparse_attn_decode, bit for bit."""
    w = W["decode_128k_b8"]
    inp = synth.make_inputs(w, "cuda", L=7000, B=2)
    q, k, v, Wq, Wk, role = (inp[x] for x in ("q", "k", "v", "Wq16", "Wk16", "kv_role"))
    q16, k16 = rtp_index_scores(q, k, Wq, Wk, role)
    o1, l1, s1 = rtp_sparse_attn_decode(q, k, v, q16, k16, role, w.p)
    o2, l2, s2 = rtp_sparse_attn_decode_select(q, k, v, q16, k16, role, "topp", p=w.p)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    torch.testing.assert_close(l1, l2, atol=0, rtol=0, equal_nan=True)  # local heads: unwritten
    for key in ("thr", "jtie", "count", "mass"):
        assert torch.equal(s1[key], s2[key]), key


def test_all_equal_scores_topk_and_block():
    """W_q16 = 0: every score is 0.  Top-k keeps the k lowest indices; block
    top-p puts every block in one bin (hi == lo) and keeps them all."""
    w = W["decode_128k_b8"]
    inp = synth.make_inputs(w, "cuda", L=9000, B=2)
    q, k, v, Wk, role = (inp[x] for x in ("q", "k", "v", "Wk16", "kv_role"))
    Wq = torch.zeros_like(inp["Wq16"])
    q16, k16 = rtp_index_scores(q, k, Wq, Wk, role)
    _, _, s = rtp_sparse_attn_decode_select(q, k, v, q16, k16, role, "topk", top_k=5000)
    _, _, bsel = rtp_sparse_attn_decode_select(q, k, v, q16, k16, role, "block_topp", p=0.5)
    torch.cuda.synchronize()
    assert bool((s["count"] == 5000).all()) and bool((s["jtie"] == 4999).all())
    assert bool((s["thr"] == 0.0).all())
    assert bool((bsel["count"] == 9000).all())


def test_recall_against_exact_topp():
    """Reported, not a pass/fail bar beyond sanity: on the 128K decode workload,
    the share of the exact top-p kept keys (and of their indexer mass) that
    block top-p and top-k (k = 4096) keep."""
    w = W["decode_128k_b8"]
    inp = synth.make_inputs(w, "cuda", L=32768, B=4)
    q, k, v, Wq, Wk, role = (inp[x] for x in ("q", "k", "v", "Wq16", "Wk16", "kv_role"))
    q16, k16 = rtp_index_scores(q, k, Wq, Wk, role)
    _, _, ex = rtp_sparse_attn_decode_select(q, k, v, q16, k16, role, "topp", p=w.p,
                                             want_scores=True)
    _, _, bl = rtp_sparse_attn_decode_select(q, k, v, q16, k16, role, "block_topp", p=w.p)
    _, _, tk = rtp_sparse_attn_decode_select(q, k, v, q16, k16, role, "topk", top_k=4096)
    torch.cuda.synchronize()
    s = ex["scores"]
    j = torch.arange(s.shape[-1], device=s.device)
    exact = (s > ex["thr"][..., None]) | ((s == ex["thr"][..., None]) & (j <= ex["jtie"][..., None]))
    topk = (s > tk["thr"][..., None]) | ((s == tk["thr"][..., None]) & (j <= tk["jtie"][..., None]))
    wb = bl["block_mask"].to(torch.int64) & 0xFFFFFFFF
    blk = ((wb[..., :, None] >> torch.arange(32, device=s.device)) & 1).flatten(-2)
    block = blk[..., j // 64].bool()
    wgt = torch.exp(s - s.max(dim=-1, keepdim=True).values)
    out = {}
    for name, m in (("block_topp", block), ("topk", topk)):
        tok = float(((m & exact).sum() / exact.sum()).item())
        mass = float(((wgt * m).sum(-1) / wgt.sum(-1)).mean().item())
        out[name] = dict(token_recall=tok, mass_kept=mass, keys=float(m.sum(-1).float().mean()))
        assert 0.0 < tok <= 1.0
    out["topp"] = dict(keys=float(exact.sum(-1).float().mean()))
    report("recall vs exact top-p, decode 32K x 4, p=0.95, k=4096", out)
    assert out["block_topp"]["mass_kept"] >= w.p - 1e-3   # whole bins: at least p


def test_topk_scores_outside_histogram_range():
    """W_q16 scaled by 64: scores spread far beyond the score pass's absolute
    bins ([-256, 256)), so the row is flagged and top-k takes its generic radix
    path over all keys; the cut is still exact (checked against the oracle on
    the same fp32 scores)."""
    w = W["decode_128k_b8"]
    inp = synth.make_inputs(w, "cuda", L=6000, B=2)
    q, k, v, Wk, role = (inp[x] for x in ("q", "k", "v", "Wk16", "kv_role"))
    Wq = (inp["Wq16"].float() * 64).to(torch.bfloat16)
    q16, k16 = rtp_index_scores(q, k, Wq, Wk, role)
    _, _, s = rtp_sparse_attn_decode_select(q, k, v, q16, k16, role, "topk", top_k=700,
                                            want_scores=True)
    torch.cuda.synchronize()
    sc = s["scores"].cpu().numpy().astype(np.float64)
    assert np.abs(sc).max() > 256
    for b in range(2):
        for r in range(w.H_ret):
            o = oracle.topk(sc[b, r], 700)
            assert float(s["thr"][b, r]) == o["t"] and int(s["jtie"][b, r]) == o["jtie"]
            assert int(s["count"][b, r]) == 700
