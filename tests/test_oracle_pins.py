"""Pins for the fp64 CPU oracle (no GPU).

Each pin checks the oracle against something other than itself: a value
worked by hand (tests/golden), a closed form, a special case that reduces to a
plain numpy formula, brute force over all subsets, or an invariant the rule
implies.  Rules are from the paper-graph-ui summary of "Full Attention Strikes
Back" (arXiv 2605.16928): §Low-Dimensional Projection Mechanism, §Dynamic
Top-p Selection Mechanism (Eq. 5), §Local Head Attention Pattern.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32_to_bf16_bits_exact(x):
    """bf16 bits of values already exactly representable in bf16."""
    b = np.asarray(x, np.float32).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "value not representable in bf16"
    return (b >> 16).astype(np.uint16)


def rand_bf16(rng, shape, scale=1.0):
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)  # truncation: any bf16 pattern will do


# ---------------------------------------------------------------- bf16 rounding

@pytest.mark.parametrize("x,bits", [
    (1.0, 0x3F80),
    (1.0 + 2**-8, 0x3F80),              # halfway 1 .. 1+2^-7: tie to even (1.0)
    (1.0 + 3 * 2**-8, 0x3F82),          # halfway 1+2^-7 .. 1+2^-6: tie to even
    (1.0 + 2**-8 + 2**-30, 0x3F81),     # just above halfway: up
    (-2.5, 0xC020),
    (0.0, 0x0000),
    (2.0**-133, 0x0001),                # smallest subnormal
    (2.0**-134, 0x0000),                # halfway 0 .. 2^-133: tie to even (0)
    (3 * 2.0**-134, 0x0002),            # halfway 2^-133 .. 2^-132: tie to even
    ((2 - 2**-7) * 2.0**127, 0x7F7F),   # largest finite
    (2.0**128 * (1 - 2**-9), 0x7F80),   # halfway max .. 2^128: even -> overflow to inf
    (-1e300, 0xFF80),
])
def test_bf16_round_known(x, bits):
    assert int(oracle.bf16_round(np.array([x]))[0]) == bits


def test_bf16_round_is_nearest_even():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))
    r = oracle.bf16_round(x)
    v = oracle.bf16_bits_to_f64(r)
    # neighbours one bf16 ulp either side
    up = oracle.bf16_bits_to_f64(r + 1)
    dn = oracle.bf16_bits_to_f64(r - 1)
    err = np.abs(x - v)
    assert np.all(err <= np.abs(x - up))
    assert np.all(err <= np.abs(x - dn))
    tie = (err == np.abs(x - up)) | (err == np.abs(x - dn))
    assert np.all((r[tie] & 1) == 0)


# ---------------------------------------------------------------- projection + scores

def test_project_exact_integers():
    rng = np.random.default_rng(2)
    x = rng.integers(-2, 3, size=(37, 128)).astype(np.float64)
    W = rng.integers(-1, 2, size=(128, 16)).astype(np.float64) / 8
    out, pre = oracle.project(f32_to_bf16_bits_exact(x), f32_to_bf16_bits_exact(W))
    ref = x @ W                                   # exact: small dyadic rationals
    assert np.array_equal(pre, ref)
    assert np.array_equal(oracle.bf16_bits_to_f64(out), ref)


def test_project_random_matches_numpy():
    rng = np.random.default_rng(3)
    xb = rand_bf16(rng, (200, 128))
    Wb = rand_bf16(rng, (128, 16), 1 / math.sqrt(128))
    out, pre = oracle.project(xb, Wb)
    ref = oracle.bf16_bits_to_f64(xb) @ oracle.bf16_bits_to_f64(Wb)
    np.testing.assert_allclose(pre, ref, rtol=1e-13, atol=1e-13)
    assert np.array_equal(out, oracle.bf16_round(pre))


def test_scores_match_numpy():
    rng = np.random.default_rng(4)
    q = rand_bf16(rng, (16,))
    k = rand_bf16(rng, (300, 16))
    s = oracle.scores(q, k)
    ref = oracle.bf16_bits_to_f64(k) @ oracle.bf16_bits_to_f64(q)
    np.testing.assert_allclose(s, ref, rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------- top-p

def _golden_topp():
    cases = []
    with open(os.path.join(GOLDEN, "topp_hand.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            _, s, p, kept = (c.strip() for c in line.split("|"))
            cases.append((np.array(s.split(), float), float(p), [int(t) for t in kept.split()]))
    return cases


@pytest.mark.parametrize("s,p,kept", _golden_topp())
def test_topp_golden(s, p, kept):
    r = oracle.topp(s, p)
    assert list(np.nonzero(r["sel"])[0]) == kept
    assert r["count"] == len(kept)


def _brute_force_topp(s, p):
    """All subsets: the smallest size whose best subset reaches p*Z; among the
    subsets of that size reaching p*Z, the one that is best under (score desc,
    index asc) compared element by element after sorting."""
    n = len(s)
    w = np.exp(s - s.max())
    Z = w.sum()
    for size in range(1, n + 1):
        best = None
        for sub in itertools.combinations(range(n), size):
            if w[list(sub)].sum() >= p * Z * (1 - 1e-12):
                key = sorted(((-s[j], j) for j in sub))
                if best is None or key < best[0]:
                    best = (key, sub)
        if best is not None:
            return sorted(best[1])
    return list(range(n))


def test_topp_brute_force_small():
    rng = np.random.default_rng(5)
    checked = 0
    for trial in range(300):
        n = int(rng.integers(1, 12))
        if trial % 3 == 0:   # many exact ties
            s = rng.integers(-3, 4, size=n).astype(float) * 0.5
        else:
            s = rng.standard_normal(n) * rng.uniform(0.2, 4)
        p = float(rng.choice([0.0, 0.3, 0.5, 0.8, 0.9, 0.95, 0.99, rng.uniform()]))
        r = oracle.topp(s, p)
        got = list(np.nonzero(r["sel"])[0])
        ref = _brute_force_topp(s, p)
        w = np.exp(s - s.max())
        # the brute force's 1e-12 slack only matters when a prefix lands on p*Z
        if abs(np.sort(w)[::-1].cumsum() / w.sum() - p).min() < 1e-9:
            continue
        assert got == ref, (s, p, got, ref)
        checked += 1
    assert checked > 250


def test_topp_limits_and_invariants():
    rng = np.random.default_rng(6)
    for _ in range(50):
        n = int(rng.integers(1, 400))
        s = rng.standard_normal(n) * rng.uniform(0.1, 8)
        if n > 3:
            s[rng.integers(0, n)] = s.max()          # a tie at the max
        # p -> 0: exactly the argmax, lowest index among equal maxima
        r0 = oracle.topp(s, 0.0)
        assert r0["count"] == 1 and r0["sel"][int(np.argmax(s))]
        r1 = oracle.topp(s, 1.0)
        assert r1["count"] == n and r1["sel"].all()
        prev = None
        w = np.exp(s - s.max())
        Z = w.sum()
        for p in (0.1, 0.5, 0.8, 0.9, 0.95, 0.99):
            r = oracle.topp(s, p)
            sel = r["sel"]
            if prev is not None:
                assert np.all(sel >= prev)            # monotone in p
            prev = sel
            mass = w[sel].sum()
            assert mass >= p * Z * (1 - 1e-12)
            # dropping the last kept key falls below p*Z
            order = sorted(np.nonzero(sel)[0], key=lambda j: (-s[j], j))
            assert mass - w[order[-1]] < p * Z * (1 + 1e-12)
            # descriptor: kept <=> s > t or (s == t and j <= jtie)
            j = np.arange(n)
            desc = (s > r["t"]) | ((s == r["t"]) & (j <= r["jtie"]))
            assert np.array_equal(desc, sel)
            assert abs(r["mass_frac"] - mass / Z) < 1e-12


def test_topp_cut_above_the_never_kept_point():
    """A key below m - ln(N / ((1 - p) Z)) is never kept: the N keys below that
    point weigh less than (1 - p) Z together, so the keys above it already
    reach p Z and the shortest prefix stops before them (Eq. 5's minimality).
    The prefill selection sizes its first histogram range by this bound (Z
    taken from below, which only widens it).  Rows include heavy and flat
    score spreads and keys packed just under the bound."""
    rng = np.random.default_rng(11)
    for trial in range(120):
        n = int(rng.integers(2, 3000))
        s = rng.standard_normal(n) * rng.uniform(0.2, 8)
        p = float(rng.choice([0.0, 0.5, 0.8, 0.9, 0.95, 0.99]))
        m = s.max()
        Z = np.exp(s - m).sum()
        bound = m - math.log(n / ((1 - p) * Z)) if p < 1 else -math.inf
        if trial % 4 == 0 and np.isfinite(bound):
            # half the keys just below the bound: the cut must still stay above
            lo = rng.random(n) < 0.5
            lo[int(np.argmax(s))] = False
            s[lo] = bound - rng.uniform(1e-9, 1e-3, lo.sum())
            m = s.max()
            Z = np.exp(s - m).sum()
            bound = m - math.log(n / ((1 - p) * Z))
        r = oracle.topp(s, p)
        assert r["t"] >= bound, (n, p, r["t"], bound)
        assert not r["sel"][s < bound].any()


def test_topp_all_equal_scores():
    for n in (1, 7, 100):
        s = np.zeros(n)
        for p in (0.0, 0.3, 0.9, 1.0):
            r = oracle.topp(s, p)
            expect = max(1, math.ceil(p * n - 1e-9)) if p < 1 else n
            assert r["count"] == expect
            assert list(np.nonzero(r["sel"])[0]) == list(range(expect))
            assert r["jtie"] == expect - 1


# ---------------------------------------------------------------- attention

def _golden_attend():
    cases = []
    with open(os.path.join(GOLDEN, "attend_hand.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            case, sset, ent, lse = (c.strip() for c in line.split("|"))
            exp = np.zeros(128)
            for e in ent.split():
                d, val = e.split(":")
                exp[int(d)] = float(val)
            cases.append((int(case), [int(t) for t in sset.split()], exp, float(lse)))
    return cases


@pytest.mark.parametrize("case,sset,expect,lse", _golden_attend())
def test_attend_golden(case, sset, expect, lse):
    q = np.zeros(128)
    K = np.zeros((3, 128))
    V = np.zeros((3, 128))
    if case in (1, 2):
        q[0] = 1
        K[0, 0] = 1
        V[0, 0] = 4
        V[1, 1] = 8
        scale = math.log(3)
    else:
        q[5] = 2
        K[0, 5], K[1, 5] = 1, -1
        for j in range(3):
            V[j, 7] = j + 1
        scale = math.log(2) / 2
    o, l = oracle.attend(f32_to_bf16_bits_exact(q), f32_to_bf16_bits_exact(K),
                         f32_to_bf16_bits_exact(V), np.array(sset), scale)
    np.testing.assert_allclose(o, expect, rtol=1e-14, atol=1e-14)
    assert abs(l - lse) < 1e-14


def _numpy_causal_attention(q, K, V, mask, scale):
    """Textbook masked softmax attention written with numpy matrix ops."""
    logits = (q @ K.T) * scale
    logits = np.where(mask, logits, -np.inf)
    mx = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - mx)
    den = w.sum(axis=1, keepdims=True)
    return (w @ V) / den, (mx + np.log(den))[:, 0]


def _small_layer(rng, B=1, L=40, H=4, Hkv=2):
    q = rand_bf16(rng, (B, L, H, 128))
    k = rand_bf16(rng, (B, L, Hkv, 128))
    v = rand_bf16(rng, (B, L, Hkv, 128))
    return q, k, v


def test_dense_rows_match_numpy():
    rng = np.random.default_rng(7)
    B, L, H, Hkv = 2, 40, 4, 2
    q, k, v = _small_layer(rng, B, L, H, Hkv)
    rows = np.array([(b, i, h) for b in range(B) for i in range(L) for h in range(H)])
    scale = 1 / math.sqrt(128)
    r = oracle.dense_rows(q, k, v, rows, H=H, Hkv=Hkv, q_pos0=0, scale=scale)
    qf, kf, vf = (oracle.bf16_bits_to_f64(x) for x in (q, k, v))
    causal = np.tril(np.ones((L, L), bool))
    for b in range(B):
        for h in range(H):
            g = h // (H // Hkv)
            o, lse = _numpy_causal_attention(qf[b, :, h], kf[b, :, g], vf[b, :, g], causal, scale)
            sel = (rows[:, 0] == b) & (rows[:, 2] == h)
            np.testing.assert_allclose(r["o"][sel], o, rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(r["lse"][sel], lse, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("window,n_sink", [(1, 0), (1, 4), (5, 0), (7, 3), (64, 4)])
def test_local_rows_match_masks(window, n_sink):
    rng = np.random.default_rng(8)
    L, H, Hkv = 48, 2, 1
    q, k, v = _small_layer(rng, 1, L, H, Hkv)
    rows = np.array([(0, i, h) for i in range(L) for h in range(H)])
    scale = 0.1
    r = oracle.local_rows(q, k, v, rows, H=H, Hkv=Hkv, q_pos0=0, window=window,
                          n_sink=n_sink, scale=scale)
    qf, kf, vf = (oracle.bf16_bits_to_f64(x) for x in (q, k, v))
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    mask = (j <= i) & ((j < n_sink) | (j > i - window))     # explicit brute-force mask
    for h in range(H):
        o, lse = _numpy_causal_attention(qf[0, :, h], kf[0, :, 0], vf[0, :, 0], mask, scale)
        sel = rows[:, 2] == h
        np.testing.assert_allclose(r["o"][sel], o, rtol=1e-12, atol=1e-12)
    if window == 1 and n_sink == 0:
        # a single key: the output is that key's value row, exactly
        for rr, (b, i_, h) in enumerate(rows):
            assert np.array_equal(r["o"][rr], vf[0, i_, 0])


def test_local_set_brute():
    for P in range(0, 30):
        for W in (1, 2, 5, 40):
            for ns in (0, 1, 4):
                got = oracle.local_set(P, W, ns)
                ref = [j for j in range(P + 1) if j < ns or P - j < W]
                assert list(got) == ref


def _retrieval_setup(rng, L=64, H=4, Hkv=2, B=1):
    q, k, v = _small_layer(rng, B, L, H, Hkv)
    G = H // Hkv
    ret_heads = list(range(G))              # kv head 0 retrieval
    Wq = rand_bf16(rng, (G, 128, 16), 1 / math.sqrt(128))
    Wk = rand_bf16(rng, (G, 128, 16), 1 / math.sqrt(128))
    q16 = np.zeros((B, L, G, 16), np.uint16)
    k16 = np.zeros((B, L, G, 16), np.uint16)
    for b in range(B):
        for slot, h in enumerate(ret_heads):
            q16[b, :, slot] = oracle.project(q[b, :, h], Wq[slot])[0]
            k16[b, :, slot] = oracle.project(k[b, :, 0], Wk[slot])[0]
    rows = np.array([(b, i, h) for b in range(B) for i in range(L) for h in ret_heads])
    slot = rows[:, 2]
    return q, k, v, q16, k16, rows, slot


def test_retrieval_p1_is_dense_and_p0_is_argmax():
    rng = np.random.default_rng(9)
    L, H, Hkv = 64, 4, 2
    q, k, v, q16, k16, rows, slot = _retrieval_setup(rng, L, H, Hkv)
    scale = 1 / math.sqrt(128)
    r1 = oracle.retrieval_rows(q, k, v, q16, k16, rows, slot, slot, H=H, Hkv=Hkv,
                               q_pos0=0, p=1.0, scale=scale)
    d = oracle.dense_rows(q, k, v, rows, H=H, Hkv=Hkv, q_pos0=0, scale=scale)
    np.testing.assert_allclose(r1["o"], d["o"], rtol=1e-12, atol=1e-12)
    assert np.array_equal(r1["count"], rows[:, 1] + 1)
    r0 = oracle.retrieval_rows(q, k, v, q16, k16, rows, slot, slot, H=H, Hkv=Hkv,
                               q_pos0=0, p=0.0, scale=scale, want_sel=True)
    vf = oracle.bf16_bits_to_f64(v)
    for rr, (b, i, h) in enumerate(rows):
        s = oracle.bf16_bits_to_f64(k16[b, :i + 1, slot[rr]]) @ oracle.bf16_bits_to_f64(q16[b, i, slot[rr]])
        j = int(np.argmax(s))
        assert r0["count"][rr] == 1 and r0["sel"][rr][j]
        assert np.array_equal(r0["o"][rr], vf[b, j, 0])        # softmax over one key


def test_decode_row_equals_last_prefill_row():
    rng = np.random.default_rng(10)
    L, H, Hkv = 50, 4, 2
    q, k, v, q16, k16, rows, slot = _retrieval_setup(rng, L, H, Hkv)
    scale = 1 / math.sqrt(128)
    pre = oracle.retrieval_rows(q, k, v, q16, k16, rows, slot, slot, H=H, Hkv=Hkv,
                                q_pos0=0, p=0.9, scale=scale)
    last = rows[:, 1] == L - 1
    drows = rows[last].copy()
    drows[:, 1] = 0
    dec = oracle.retrieval_rows(q[:, L - 1:], k, v, q16[:, L - 1:], k16, drows,
                                slot[last], slot[last], H=H, Hkv=Hkv, q_pos0=L - 1,
                                p=0.9, scale=scale)
    for key in ("o", "lse", "t", "jtie", "count", "mass_frac"):
        assert np.array_equal(dec[key], pre[key][last]), key
    loc_pre = oracle.local_rows(q, k, v, rows[last], H=H, Hkv=Hkv, q_pos0=0, window=8,
                                n_sink=2, scale=scale)
    loc_dec = oracle.local_rows(q[:, L - 1:], k, v, drows, H=H, Hkv=Hkv, q_pos0=L - 1,
                                window=8, n_sink=2, scale=scale)
    assert np.array_equal(loc_pre["o"], loc_dec["o"])


def test_retrieval_rows_match_composition():
    """The row driver equals scores -> topp -> attend composed by hand, with the
    selection taken from brute-force sort in numpy."""
    rng = np.random.default_rng(11)
    L, H, Hkv = 48, 4, 2
    q, k, v, q16, k16, rows, slot = _retrieval_setup(rng, L, H, Hkv)
    scale = 1 / math.sqrt(128)
    p = 0.8
    r = oracle.retrieval_rows(q, k, v, q16, k16, rows, slot, slot, H=H, Hkv=Hkv,
                              q_pos0=0, p=p, scale=scale, want_sel=True)
    qf, kf, vf = (oracle.bf16_bits_to_f64(x) for x in (q, k, v))
    for rr, (b, i, h) in enumerate(rows):
        s = oracle.bf16_bits_to_f64(k16[b, :i + 1, slot[rr]]) @ oracle.bf16_bits_to_f64(q16[b, i, slot[rr]])
        order = np.lexsort((np.arange(i + 1), -s))
        w = np.exp(s - s.max())
        c = np.cumsum(w[order])
        kcount = int(np.searchsorted(c, p * w.sum(), side="left")) + 1
        kept = np.sort(order[:kcount])
        assert list(np.nonzero(r["sel"][rr])[0]) == list(kept)
        mask = np.zeros((1, i + 1), bool)
        mask[0, kept] = True
        o, lse = _numpy_causal_attention(qf[b, i:i + 1, h], kf[b, :i + 1, 0], vf[b, :i + 1, 0],
                                         mask, scale)
        np.testing.assert_allclose(r["o"][rr], o[0], rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- static top-k
# [FASB §5 Experimental Analysis]: the method's fixed-budget variant keeps the k
# highest-scoring keys (k = 4096 there); ties go to the lower index, the order the
# top-p rule uses.

@pytest.mark.parametrize("seed", range(6))
def test_topk_equals_sorted_prefix(seed):
    """Against numpy's lexsort of (score desc, index asc): the first k keys."""
    rng = np.random.default_rng(200 + seed)
    n = int(rng.integers(1, 40))
    s = rng.integers(-3, 4, n).astype(float)  # many exact ties
    order = np.lexsort((np.arange(n), -s))
    for k in (1, 2, 5, n - 1, n, n + 3):
        if k < 1:
            continue
        r = oracle.topk(s, k)
        want = np.zeros(n, bool)
        want[order[:min(k, n)]] = True
        assert np.array_equal(r["sel"], want), (k, s)
        assert r["count"] == min(k, n)
        last = order[min(k, n) - 1]
        assert r["jtie"] == last and r["t"] == s[last]


def test_topk_special_cases():
    s = np.array([0.5, 2.0, 2.0, -1.0, 2.0])
    r = oracle.topk(s, 1)
    assert list(np.nonzero(r["sel"])[0]) == [1]          # argmax, lowest index
    r = oracle.topk(s, 2)
    assert list(np.nonzero(r["sel"])[0]) == [1, 2]       # tie at the cut: lower index
    assert oracle.topk(s, 99)["sel"].all()               # k >= n: every key
    z = oracle.topk(np.zeros(10), 4)                     # all equal: the first k indices
    assert list(np.nonzero(z["sel"])[0]) == [0, 1, 2, 3] and z["jtie"] == 3


# ---------------------------------------------------------------- block top-p
# [FASB §Hardware-Aware Fast Top-p Decoding Kernel], steps 1-5.

def _golden_block_topp():
    cases = []
    with open(os.path.join(GOLDEN, "block_topp_hand.txt")) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            _, spec, p, blocks = (c.strip() for c in line.split("|"))
            s = np.concatenate([np.full(int(c), float(v))
                                for v, c in (run.split("*") for run in spec.split())])
            cases.append((s, float(p), [int(t) for t in blocks.split()]))
    return cases


@pytest.mark.parametrize("s,p,blocks", _golden_block_topp())
def test_block_topp_golden(s, p, blocks):
    r = oracle.block_topp(s, p)
    assert list(np.nonzero(r["bsel"])[0]) == blocks
    n = s.size
    assert r["count"] == sum(min(64, n - 64 * b) for b in blocks)
    assert np.array_equal(np.nonzero(r["sel"])[0],
                          np.concatenate([np.arange(64 * b, min(64 * b + 64, n)) for b in blocks]))


def _block_brute_force(s, p, block=64):
    """With every block alone in its histogram bin, the selection is the shortest
    prefix of blocks ranked by their max (descending) whose summed softmax mass
    reaches p of the total: computed here block by block, with no histogram."""
    nb = (s.size + block - 1) // block
    m = s.max()
    mass = np.array([np.exp(s[b * block:(b + 1) * block] - m).sum() for b in range(nb)])
    mx = np.array([s[b * block:(b + 1) * block].max() for b in range(nb)])
    order = np.argsort(-mx, kind="stable")
    keep = np.zeros(nb, bool)
    acc = 0.0
    for b in order:
        keep[b] = True
        acc += mass[b]
        if acc >= p * mass.sum():
            break
    return keep


@pytest.mark.parametrize("seed", range(8))
def test_block_topp_brute_force_distinct_bins(seed):
    rng = np.random.default_rng(300 + seed)
    nb = int(rng.integers(2, 7))
    n = 64 * (nb - 1) + int(rng.integers(1, 65))           # a short last block
    # block maxima at least 3 bins apart: every block in its own bin
    tops = rng.permutation(np.linspace(0.0, 8.0, nb))
    s = np.empty(n)
    for b in range(nb):
        blk = slice(64 * b, min(64 * b + 64, n))
        w = blk.stop - blk.start
        s[blk] = tops[b] - rng.uniform(0.0, 3.0, w)
        s[blk.start + int(rng.integers(0, w))] = tops[b]
    for p in (0.0, 0.3, 0.6, 0.9, 0.95, 0.999):
        r = oracle.block_topp(s, p)
        assert len(set(r["bin"])) == nb
        assert np.array_equal(r["bsel"], _block_brute_force(s, p)), (p, r["bin"])


@pytest.mark.parametrize("seed", range(4))
def test_block_topp_invariants(seed):
    """p >= 1 keeps every block; p = 0 keeps exactly the top bin's blocks; the
    selection grows with p; the kept softmax mass reaches p; the block holding
    the argmax key is always kept."""
    rng = np.random.default_rng(400 + seed)
    n = int(rng.integers(65, 3000))
    s = rng.standard_normal(n) * 4.0
    r1 = oracle.block_topp(s, 1.0)
    assert r1["bsel"].all() and r1["count"] == n and abs(r1["mass_frac"] - 1.0) < 1e-12
    r0 = oracle.block_topp(s, 0.0)
    assert np.array_equal(r0["bsel"], r0["bin"] == 255)
    prev = None
    for p in np.linspace(0.0, 1.0, 21):
        r = oracle.block_topp(s, p)
        assert r["bsel"][int(np.argmax(s)) // 64]
        assert r["mass_frac"] >= p - 1e-12
        if prev is not None:
            assert np.all(r["bsel"] >= prev)
        prev = r["bsel"]
