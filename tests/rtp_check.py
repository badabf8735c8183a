"""Shared checks for the GPU-vs-oracle parity tests.

Tolerances:

* selection: the kept set of every retrieval row equals the oracle's, except for
  keys whose indexer score lies within SEL_BAND (relative, floor 1) of the row
  threshold -- the oracle's or the GPU's own.  In addition the GPU threshold must
  be a valid top-p cut under the oracle's fp64 masses: the mass strictly above it
  stays below p and the mass at or above it reaches p, both up to MASS_EPS (the
  GPU computes exp and the scores in fp32);
* outputs: max-abs <= 2e-2 and mean-abs <= 2e-3 against the oracle's fp64
  output (bf16 inputs, fp32 accumulation on the GPU); lse within 2e-2.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from long_context_sparse_rtp_b200 import synth

SEL_BAND = 1e-5
MASS_EPS = 1e-5
SCORE_SLACK = 2e-6
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_ABS = 2e-2


def bits(t: torch.Tensor) -> np.ndarray:
    return synth.bits(t)


def f64(b: np.ndarray) -> np.ndarray:
    return oracle.bf16_bits_to_f64(b)


def check_row_selection(s64, p, t_orc, sel_orc, t_gpu, jtie_gpu, count_gpu, mass_gpu=None):
    """One retrieval row.  s64: fp64 indexer scores of keys 0..P computed from the
    GPU's q16/k16.  Returns the number of keys inside the tolerance band."""
    n = s64.size
    j = np.arange(n)
    if p >= 1.0:
        assert t_gpu == -math.inf and count_gpu == n and jtie_gpu == n - 1
        return 0
    sel_gpu = (s64 > t_gpu) | ((s64 == t_gpu) & (j <= jtie_gpu))
    band = np.abs(s64 - t_orc) <= SEL_BAND * max(abs(t_orc), 1.0)
    band |= np.abs(s64 - t_gpu) <= SEL_BAND * max(abs(t_gpu), 1.0)
    out = ~band
    bad = np.nonzero(sel_gpu[out] != sel_orc[out])[0]
    assert bad.size == 0, (
        f"selection differs outside the band at keys {j[out][bad][:8]} "
        f"(t_orc={t_orc!r}, t_gpu={t_gpu!r}, count gpu={count_gpu} orc={int(sel_orc.sum())})")
    n_out = int(sel_gpu[out].sum())
    assert n_out <= count_gpu <= n_out + int(band.sum()), (count_gpu, n_out, int(band.sum()))
    # the GPU cut is a valid top-p cut under fp64 masses
    w = np.exp(s64 - s64.max())
    Z = w.sum()
    slack = SCORE_SLACK * max(abs(t_gpu), 1.0)
    above = w[s64 > t_gpu + slack].sum() / Z
    at_or_above = w[s64 >= t_gpu - slack].sum() / Z
    assert above < p + MASS_EPS, (above, p)
    assert at_or_above >= p - MASS_EPS, (at_or_above, p)
    if mass_gpu is not None:
        m_lo = w[sel_gpu & out].sum() / Z
        m_hi = m_lo + w[band].sum() / Z
        assert m_lo - MASS_EPS <= mass_gpu <= m_hi + MASS_EPS, (mass_gpu, m_lo, m_hi)
    return int(band.sum())


def check_outputs(o_gpu: np.ndarray, o_orc: np.ndarray, what: str):
    if o_gpu.size == 0:
        return 0.0, 0.0
    err = np.abs(o_gpu.astype(np.float64) - o_orc)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= O_MAX_ABS, f"{what}: max-abs {mx:.3e}"
    assert mean <= O_MEAN_ABS, f"{what}: mean-abs {mean:.3e}"
    return mx, mean


def gpu_kept(q16_row_bits, k16_bits, P, t_gpu, jtie_gpu, count_gpu, p):
    """The GPU's kept set of one row, as far as fp64 arithmetic can tell it.

    The GPU keeps key j if its fp32 score s32_j > t or (s32_j == t and j <=
    jtie), where t = s32 of key jtie.  |s32_j - s64_j| <= 17 u sum_d |q_d k_jd|
    (16 products exact in fp32, 15 additions, one rounding; u = 2^-24), so a key
    whose fp64 score differs from the tie key's by more than both bounds is
    decided; the undecided rest (the tie key among them, always kept) is filled
    with count - (decided kept) keys.  Returns (mask over 0..P, amb) where amb
    is None when that fill is forced (none or all of the undecided rest) and
    otherwise the mask of undecided keys, in which the choice shown (score desc,
    index asc) may differ from the GPU's."""
    n = P + 1
    if p >= 1.0:
        return np.ones(n, bool), None
    q = f64(q16_row_bits)
    k = f64(k16_bits[:n])
    s64 = k @ q
    bound = 17 * 2.0 ** -24 * (np.abs(k) @ np.abs(q))
    c = int(jtie_gpu)
    gap = s64 - s64[c]
    tol = bound + bound[c]
    above = gap > tol
    und = ~above & (gap >= -tol)
    need = int(count_gpu) - int(above.sum())
    n_und = int(und.sum())
    assert 1 <= need <= n_und, (need, n_und)
    mask = above.copy()
    if need == n_und:
        mask |= und
        return mask, None
    mask[c] = True
    if need == 1:
        return mask, None
    j = np.nonzero(und & (np.arange(n) != c))[0]
    order = j[np.lexsort((j, -s64[j]))]
    mask[order[:need - 1]] = True
    return mask, und


E2E_MASS = 1e-3


def _mass_share(q_bits, K_bits, V_bits, part, whole, scale):
    """Attention-mass share of the keys `part` among the keys `whole` (masks)."""
    if not part.any():
        return 0.0
    _, l_part = oracle.attend(q_bits, K_bits, V_bits, np.nonzero(part)[0], scale)
    _, l_whole = oracle.attend(q_bits, K_bits, V_bits, np.nonzero(whole)[0], scale)
    return math.exp(l_part - l_whole)


def row_reference(q_bits, K_bits, V_bits, kept, sel_same, o_same, lse_same, sel_e2e, scale):
    """References for one retrieval row.  kept = gpu_kept(...).

    (o_ref, lse_ref, ok): the oracle's exact attention over the GPU's own kept
    set (taken from the oracle run on the GPU's q16/k16 when its kept set is the
    same, else attended directly).  ok is False only when that set is not
    forced by fp64 arithmetic (gpu_kept's amb) and its undecided keys carry more
    than E2E_MASS of the attention mass, so that the GPU may have attended to a
    set that differs from the reconstruction in a way that matters.
    e2e_ok: whether the oracle run end to end (its own projections) may serve as
    a second reference: its kept set differs from the GPU's by keys whose share
    of the attention mass (over the union of both sets) is at most E2E_MASS.
    Keys near the cut carry little mass except in rows with few kept keys, where
    a legitimate one-key difference changes the output by O(1)."""
    mask, amb = kept
    if np.array_equal(mask, sel_same):
        o_ref, lse_ref = o_same, lse_same
    else:
        o_ref, lse_ref = oracle.attend(q_bits, K_bits, V_bits, np.nonzero(mask)[0], scale)
    ok = amb is None or _mass_share(q_bits, K_bits, V_bits, amb, mask | amb, scale) <= E2E_MASS
    e2e_ok = _mass_share(q_bits, K_bits, V_bits, mask ^ sel_e2e, mask | sel_e2e,
                         scale) <= E2E_MASS
    return o_ref, lse_ref, ok, e2e_ok


def check_row_outputs(o_gpu, o_ref, ref_ok, o_e2e, e2e_ok, what, max_skip=0.05):
    """Output parity of retrieval rows: against the oracle's attention over the
    GPU's own kept set (o_ref) on every row where that set is known (ref_ok),
    and against the oracle run end to end on its own projections where its kept
    set carries the same mass up to E2E_MASS (e2e_ok).  The share of rows left
    out of either check is bounded."""
    n = len(o_gpu)
    ref_ok = np.asarray(ref_ok, bool)
    e2e_ok = np.asarray(e2e_ok, bool)
    assert (~ref_ok).sum() <= max(2, max_skip * n), (int((~ref_ok).sum()), n)
    assert (~e2e_ok).sum() <= max(2, max_skip * n), (int((~e2e_ok).sum()), n)
    r1 = check_outputs(o_gpu[ref_ok], o_ref[ref_ok], what + " vs oracle on the GPU's kept sets")
    r2 = check_outputs(o_gpu[e2e_ok], o_e2e[e2e_ok], what + " vs oracle end to end")
    stats = dict(rows=n, skip_ref=int((~ref_ok).sum()), skip_e2e=int((~e2e_ok).sum()),
                 max_abs=r1[0], mean_abs=r1[1], e2e_max_abs=r2[0], e2e_mean_abs=r2[1])
    report(what, stats)
    return stats


def report(what, stats):
    """Append one JSON line of parity statistics to $RTP_PARITY_LOG (if set)."""
    import json
    import os
    path = os.environ.get("RTP_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(dict(what=what, **stats)) + "\n")


def oracle_k16(k_bits, Wk_bits, w: synth.Workload, per_kv: bool = False):
    """Oracle projection of every key row for every k16 slot: [B, Lk, H_k16, 16]."""
    B, Lk = k_bits.shape[0], k_bits.shape[1]
    ret = w.retrieval_q_heads()
    if per_kv:
        kvs = sorted(w.ret_kv)
    else:
        kvs = [h // w.G for h in ret]
    out = np.empty((B, Lk, len(kvs), 16), np.uint16)
    for b in range(B):
        for s, g in enumerate(kvs):
            out[b, :, s] = oracle.project(k_bits[b, :, g], Wk_bits[s])[0]
    return out


def oracle_q16(q_bits, Wq_bits, w: synth.Workload):
    B, Lq = q_bits.shape[0], q_bits.shape[1]
    ret = w.retrieval_q_heads()
    out = np.empty((B, Lq, len(ret), 16), np.uint16)
    for b in range(B):
        for s, h in enumerate(ret):
            out[b, :, s] = oracle.project(q_bits[b, :, h], Wq_bits[s])[0]
    return out


def row_scores(q16_bits_row, k16_bits, P):
    """fp64 indexer scores of keys 0..P: k16_bits [Lk, 16] (one slot)."""
    return f64(k16_bits[:P + 1]) @ f64(q16_bits_row)
