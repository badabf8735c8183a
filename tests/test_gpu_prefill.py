"""GPU parity: causal prefill of one mixed layer against the fp64 oracle.

Stage by stage:
 (i)   q16/k16 projections equal the oracle's bf16 values, or sit one bf16 ulp
       away where the exact value lies within fp32-accumulation distance of a
       rounding midpoint;
 (ii)  the top-p selection, re-derived by the oracle from the GPU's own q16/k16,
       matches outside the threshold band and the GPU cut is a valid top-p cut;
 (iii) outputs match the oracle run end to end (its own projections).
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_rtp_b200 import (rtp_index_scores, rtp_layer_prefill, rtp_topp_select,
                                          synth)
from rtp_check import (LSE_ABS, SEL_BAND, bits, check_outputs, check_row_outputs,
                       check_row_selection, f64, gpu_kept, oracle_k16, oracle_q16,
                       row_reference, row_scores)

pytestmark = pytest.mark.gpu

SCALE = 1.0 / math.sqrt(128)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from long_context_sparse_rtp_b200 import build
    build.build()


def check_projection(gpu_bits, x_bits_rows, W_bits):
    """(i) for one slot: gpu_bits [n,16], x_bits_rows [n,128], W [128,16]."""
    ref, pre = oracle.project(x_bits_rows, W_bits)
    diff = np.nonzero(gpu_bits != ref)
    if diff[0].size == 0:
        return 0
    g = f64(gpu_bits[diff])
    # fp32 accumulation of 128 products: |sum_fp32 - exact| <= 128 u sum|x_d W_dc|; the bf16
    # rounding adds at most half an ulp of the result (ulp = 2^-7 relative, 2^-133 floor)
    bound = 128 * 2.0 ** -24 * (np.abs(f64(x_bits_rows)) @ np.abs(f64(W_bits)))[diff]
    ulp = np.maximum(np.abs(g) * 2.0 ** -7, 2.0 ** -133)
    assert np.all(np.abs(g - pre[diff]) <= bound + 0.5 * ulp)
    assert diff[0].size <= max(4, gpu_bits.size // 200)
    return diff[0].size


def run_prefill(w, L, p, B=1, positions=None, per_kv=False, check_proj=True, seed=None,
                indexer_input="post"):
    """indexer_input="pre": the indexer projects the pre-RoPE draws (q_idx, k_idx)
    while attention runs on the post-RoPE q, k; the oracle follows the same split."""
    if seed is not None:
        w = w.with_(seed=seed)
    inp = synth.make_inputs(w, "cuda", L=L, B=B, indexer_input=indexer_input)
    q, k, v = inp["q"], inp["k"], inp["v"]
    qi, ki = inp.get("q_idx", q), inp.get("k_idx", k)
    Wq, Wk = inp["Wq16"], inp["Wk16"]
    if per_kv:  # one indexer key per retrieval kv head: the first query head's W_k16
        Wk = Wk[[s for s in range(0, w.H_ret, w.G)]].contiguous()
    role = inp["kv_role"]
    res = rtp_layer_prefill(q, k, v, Wq, Wk, role, p=p, window=w.window, n_sink=w.n_sink,
                            k16_per_kv_head=int(per_kv), q_idx=inp.get("q_idx"),
                            k_idx=inp.get("k_idx"))
    torch.cuda.synchronize()
    if positions is None:
        positions = np.arange(L)
    positions = np.asarray(sorted(set(int(x) for x in positions)))
    # only the sampled query rows travel to the host
    pidx = torch.as_tensor(positions, device=q.device)
    kb, vb = bits(k), bits(v)
    kib = kb if ki is k else bits(ki)
    Wqb, Wkb = bits(Wq), bits(Wk)
    qs, q16s = bits(q[:, pidx]), bits(res["q16"][:, pidx])
    qis = qs if qi is q else bits(qi[:, pidx])
    k16g = bits(res["k16"])
    sel = {key: val[:, :, pidx].cpu().numpy() for key, val in res["sel"].items()}
    o = res["o"][:, pidx].float().cpu().numpy()
    lse = res["lse"][:, :, pidx].cpu().numpy()
    ret, loc = w.retrieval_q_heads(), w.local_q_heads()
    p = float(np.float32(p))  # the C ABI takes p as fp32
    k16slot = [s // w.G for s in range(w.H_ret)] if per_kv else list(range(w.H_ret))

    # (i) projections
    if check_proj:
        for b in range(B):
            for s, h in enumerate(ret):
                check_projection(q16s[b, :, s], qis[b, :, h], Wqb[s])
            for s in sorted(set(k16slot)):
                g = ret[s * (w.G if per_kv else 1)] // w.G
                check_projection(k16g[b, :, s], kib[b, :, g], Wkb[s])
    k16o = oracle_k16(kib, Wkb, w, per_kv)

    n_band, o_ret_g, o_ret_a, o_ret_o, o_loc_g, o_loc_o = 0, [], [], [], [], []
    ref_ok, e2e_ok = [], []
    lse_err = 0.0
    for b in range(B):
        for x, i in enumerate(positions):
            rows = np.array([(0, 0, h) for h in ret])
            q1, q16_1 = qs[b:b + 1, x:x + 1], q16s[b:b + 1, x:x + 1]
            kb1, vb1, k16g1 = kb[b:b + 1], vb[b:b + 1], k16g[b:b + 1]
            # (ii) selection on the GPU's q16/k16
            r2 = oracle.retrieval_rows(q1, kb1, vb1, q16_1, k16g1, rows, np.arange(len(ret)),
                                       np.array(k16slot), H=w.H, Hkv=w.Hkv, q_pos0=int(i), p=p,
                                       scale=SCALE, want_sel=True)
            # (iii) end to end with the oracle's own projections
            q16o = np.stack([oracle.project(qis[b, x, h][None], Wqb[s])[0][0]
                             for s, h in enumerate(ret)])[None, None]
            r3 = oracle.retrieval_rows(q1, kb1, vb1, q16o, k16o[b:b + 1], rows,
                                       np.arange(len(ret)), np.array(k16slot), H=w.H, Hkv=w.Hkv,
                                       q_pos0=int(i), p=p, scale=SCALE, want_sel=True)
            for s, h in enumerate(ret):
                s64 = row_scores(q16s[b, x, s], k16g[b, :, k16slot[s]], int(i))
                t_g, jt_g = float(sel["thr"][b, s, x]), int(sel["jtie"][b, s, x])
                n_band += check_row_selection(s64, p, r2["t"][s], r2["sel"][s], t_g, jt_g,
                                              int(sel["count"][b, s, x]),
                                              float(sel["mass"][b, s, x]))
                g = h // w.G
                kept = gpu_kept(q16s[b, x, s], k16g[b, :, k16slot[s]], int(i), t_g, jt_g,
                                int(sel["count"][b, s, x]), p)
                o_ref, lse_ref, ok, ok2 = row_reference(
                    qs[b, x, h], kb[b, :i + 1, g], vb[b, :i + 1, g], kept, r2["sel"][s],
                    r2["o"][s], r2["lse"][s], r3["sel"][s], SCALE)
                o_ret_a.append(o_ref)
                ref_ok.append(ok)
                e2e_ok.append(ok2)
                if ok:
                    lse_err = max(lse_err, abs(float(lse[b, h, x]) - lse_ref))
            o_ret_o.append(r3["o"])
            o_ret_g.append(o[b, x, ret])
            if loc:
                rl = oracle.local_rows(q1, kb1, vb1, np.array([(0, 0, h) for h in loc]), H=w.H,
                                       Hkv=w.Hkv, q_pos0=int(i), window=w.window,
                                       n_sink=w.n_sink, scale=SCALE)
                o_loc_o.append(rl["o"])
                o_loc_g.append(o[b, x, loc])
                lse_err = max(lse_err, float(np.abs(lse[b, loc, x] - rl["lse"]).max()))
    stats = check_row_outputs(np.concatenate(o_ret_g), np.stack(o_ret_a), ref_ok,
                              np.concatenate(o_ret_o), e2e_ok,
                              f"retrieval prefill {w.name} L={L} B={B} p={p}")
    if loc:
        check_outputs(np.concatenate(o_loc_g), np.concatenate(o_loc_o), "local heads")
    assert lse_err <= LSE_ABS, lse_err
    return dict(n_band=n_band, res=res, inp=inp, stats=stats)


W = synth.WORKLOADS


def test_prefill_2k_full():
    """The 2K workload, every row of every head."""
    run_prefill(W["prefill_2k"], 2048, 0.9)


@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 130, 1000])
@pytest.mark.parametrize("p", [0.0, 0.5, 0.9, 1.0])
def test_prefill_ragged_and_limits(L, p):
    run_prefill(W["prefill_2k"], L, p, check_proj=(p == 0.5))


def test_prefill_batch2_per_kv_k16():
    run_prefill(W["prefill_2k"], 700, 0.9, B=2, per_kv=True)


@pytest.mark.parametrize("p", [0.8, 0.9, 0.95, 0.99])
def test_prefill_temperature_sweep(p):
    """The 32K workload's generator (per-query temperature, 2 retrieval kv heads)
    at 4K rows, sampled positions."""
    rng = np.random.default_rng(1)
    pos = np.concatenate([np.arange(8), np.arange(4096 - 8, 4096), rng.integers(0, 4096, 48)])
    run_prefill(W["prefill_32k"], 4096, p, positions=pos, check_proj=False)


def test_prefill_multihop_and_group_needles():
    rng = np.random.default_rng(2)
    pos = np.concatenate([[0, 1, 4095, 4096, 4097, 8191], rng.integers(0, 8192, 32)])
    run_prefill(W["prefill_128k"], 8192, 0.95, positions=pos, check_proj=False)
    run_prefill(W["prefill_1m"], 8192, 0.95, positions=pos, check_proj=False)


def test_prefill_all_scores_equal():
    """W_q16 = 0: every indexer score is 0, so every key ties; the kept set is the
    ceil(p * N) lowest indices."""
    w = W["prefill_2k"]
    inp = synth.make_inputs(w, "cuda", L=300)
    Wq = torch.zeros_like(inp["Wq16"])
    for p in (0.0, 0.37, 0.9):
        res = rtp_layer_prefill(inp["q"], inp["k"], inp["v"], Wq, inp["Wk16"], inp["kv_role"],
                                p=p, window=w.window, n_sink=w.n_sink)
        cnt = res["sel"]["count"].cpu().numpy()
        jt = res["sel"]["jtie"].cpu().numpy()
        N = np.arange(1, 301)
        expect = np.maximum(1, np.ceil(float(np.float32(p)) * N)).astype(int)
        assert np.array_equal(cnt[0, 0], expect)
        assert np.array_equal(jt[0, 0], expect - 1)
        assert np.all(res["sel"]["thr"].cpu().numpy() == 0.0)


def test_prefill_all_scores_equal_deep():
    """W_q16 = 0 at 10K rows: every key ties, so rows past 8128 keys take the
    level-1 sub-bins (one sub-bin holds every key), the composite-key digits
    through the identical score bits, and the index bits; the kept set is still
    the ceil(p * N) lowest indices."""
    w = W["prefill_2k"]
    L = 10000
    inp = synth.make_inputs(w, "cuda", L=L)
    Wq = torch.zeros_like(inp["Wq16"])
    N = np.arange(1, L + 1)
    for p in (0.37, 0.95):
        res = rtp_layer_prefill(inp["q"], inp["k"], inp["v"], Wq, inp["Wk16"], inp["kv_role"],
                                p=p, window=w.window, n_sink=w.n_sink)
        torch.cuda.synchronize()
        cnt = res["sel"]["count"].cpu().numpy()
        jt = res["sel"]["jtie"].cpu().numpy()
        expect = np.maximum(1, np.ceil(float(np.float32(p)) * N)).astype(int)
        for s in range(cnt.shape[1]):
            assert np.array_equal(cnt[0, s], expect), s
            assert np.array_equal(jt[0, s], expect - 1), s
        assert np.all(res["sel"]["thr"].cpu().numpy() == 0.0)


def _select_small_workspace(q16, k16, kv_role, p, H):
    """rtp_topp_select through the C ABI with a workspace of only the status
    word: the parked candidate lists are off."""
    from long_context_sparse_rtp_b200 import rtp as R
    B, Lq, n_ret = q16.shape[0], q16.shape[1], q16.shape[2]
    out = dict(thr=torch.empty(B, n_ret, Lq, dtype=torch.float32, device="cuda"),
               jtie=torch.empty(B, n_ret, Lq, dtype=torch.int32, device="cuda"),
               count=torch.empty(B, n_ret, Lq, dtype=torch.int32, device="cuda"),
               mass=torch.empty(B, n_ret, Lq, dtype=torch.float32, device="cuda"))
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    shp = R._shape(B, Lq, k16.shape[1], H, len(kv_role), 0)
    rc = R.lib().rtp_topp_select(ctypes.byref(shp), R._role(kv_role), 0, R.view(q16, 16),
                                 R.view(k16, 16), ctypes.c_float(p), R._ptr(out["thr"]),
                                 R._ptr(out["jtie"]), R._ptr(out["count"]), R._ptr(out["mass"]),
                                 R._ptr(ws), ws.numel(), R._stream())
    assert rc == 0, rc
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32)[0]) == 0  # the device status word
    return out


@pytest.mark.parametrize("p", [0.95, 0.99])
def test_select_without_list_workspace(p):
    """With a workspace too small for the candidate lists, every dense crossing
    range is refined by further sweeps instead of a parked list; the selection
    is the same, bit for bit."""
    w = W["prefill_128k"]
    inp = synth.make_inputs(w, "cuda", L=6000)
    role = inp["kv_role"]
    q16, k16 = rtp_index_scores(inp["q"], inp["k"], inp["Wq16"], inp["Wk16"], role)
    full = rtp_topp_select(q16, k16, role, p, H=w.H)
    small = _select_small_workspace(q16, k16, role, p, w.H)
    for key in ("thr", "jtie", "count", "mass"):
        assert torch.equal(small[key], full[key]), key
    # every key tied: each row's crossing range holds all its keys
    wz = torch.zeros_like(inp["Wq16"])
    q16z, _ = rtp_index_scores(inp["q"][:, :3000], inp["k"][:, :3000], wz, inp["Wk16"], role)
    k16z = k16[:, :3000].contiguous()
    full = rtp_topp_select(q16z, k16z, role, p, H=w.H)
    small = _select_small_workspace(q16z, k16z, role, p, w.H)
    for key in ("thr", "jtie", "count", "mass"):
        assert torch.equal(small[key], full[key]), key
    N = np.arange(1, 3001)
    expect = np.maximum(1, np.ceil(float(np.float32(p)) * N)).astype(int)
    assert np.array_equal(small["count"][0, 0].cpu().numpy(), expect)


def test_single_key_sets_return_that_value_row():
    """A kept set of one key makes the softmax weight exactly 1, so the output
    is that key's V row bit for bit: p = 0 keeps only the top-scoring key (the
    lowest index among equal maxima) on the retrieval heads, and a window of one
    token without sinks keeps the query's own key on the local heads."""
    w = W["prefill_2k"]
    L = 777
    inp = synth.make_inputs(w, "cuda", L=L)
    q, k, v, role = inp["q"], inp["k"], inp["v"], inp["kv_role"]
    res = rtp_layer_prefill(q, k, v, inp["Wq16"], inp["Wk16"], role, p=0.0, window=1, n_sink=0)
    torch.cuda.synchronize()
    sel = res["sel"]
    assert bool((sel["count"] == 1).all())
    jt = sel["jtie"].long()                                   # [B, H_ret, L]
    ret, loc = w.retrieval_q_heads(), w.local_q_heads()
    o = res["o"]
    for s, h in enumerate(ret):
        g = h // w.G
        assert torch.equal(o[0, :, h], v[0, jt[0, s], g]), h
        # the kept key is a causal argmax of the indexer scores, the lowest index
        # among equal maxima: checked in fp64 up to the selection band, since the
        # GPU compares fp32 scores
        sc = (res["q16"][0, :, s].double() @ res["k16"][0, :, s].double().T)
        idx = torch.arange(L, device="cuda")
        sc = sc.masked_fill(idx[None, :] > idx[:, None], float("-inf"))
        best = sc.max(dim=1).values
        mine = sc.gather(1, jt[0, s][:, None])[:, 0]
        band = SEL_BAND * best.abs().clamp(min=1.0)
        assert bool((best - mine <= band).all())
        before = sc.masked_fill(idx[None, :] >= jt[0, s][:, None], float("-inf"))
        assert bool((before.max(dim=1).values < mine + band).all())
    for h in loc:
        assert torch.equal(o[0, :, h], v[0, :, h // w.G]), h
