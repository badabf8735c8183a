"""bench.py's host-side arithmetic (no GPU): the algorithmic bytes behind the
decode roofline, the profile lookup that supplies `traffic`, the peaks."""
import json
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from long_context_sparse_rtp_b200 import synth  # noqa: E402


def test_decode_bytes_closed_forms():
    """k16: one 16-dim bf16 row per (batch, key, retrieval query head); local:
    K and V rows of the sink + window span for every (batch, local kv head);
    gathered: K and V rows of the kept union; small: q, o, the new k/v rows and
    the k16 row appends."""
    w = synth.WORKLOADS["decode_128k_b8"]
    B, L = 8, 131072
    st = dict(w=w, q=torch.empty(B, 1, w.H, 128, device="meta"), L=L)
    union = 19180
    got = bench.decode_bytes(st, union)
    assert got["k16"] == B * L * w.H_ret * 16 * 2 == 268435456
    n_loc_kv = w.Hkv - len(w.ret_kv)
    assert got["local"] == B * n_loc_kv * (w.window + w.n_sink) * 2 * 128 * 2 == 50380800
    assert got["gather"] == union * 2 * 128 * 2
    assert got["total"] == got["k16"] + got["local"] + got["gather"] + got["small"]
    # a cache shorter than the window reads only the keys it has
    st_short = dict(st, L=1000)
    assert bench.decode_bytes(st_short, 0)["local"] == B * n_loc_kv * 1000 * 2 * 128 * 2


def test_profiled_traffic_matches_source_hash(tmp_path, monkeypatch):
    # the committed summary names the source it was taken from
    t = bench.profiled_traffic("dec_score_decode_128k_b8.md")
    assert t is None or t > 268435456  # read once: at least the k16 bytes
    # a summary whose source changed since gives no traffic
    prof = tmp_path / "profiles"
    prof.mkdir()
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    (prof / "x.md").write_text("traffic_bytes_per_launch: 1234\n"
                               "source: k.cu sha256 prefix 0000000000000000\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic("x.md") is None
    import hashlib
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (prof / "x.md").write_text(f"traffic_bytes_per_launch: 1234\nsource: k.cu sha256 prefix {sha}\n")
    assert bench.profiled_traffic("x.md") == 1234
    assert bench.profiled_traffic("missing.md") is None


def test_peaks_measured_or_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.peaks()["src"] == "fallback"
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        dict(hbm_gbs=6549.1, bf16_tflops=1628.0, bf16_tflops_sustained=1372.6)))
    pk = bench.peaks()
    assert pk["src"] == "measured" and pk["hbm"] == 6549.1 and pk["bf16_sus"] == 1372.6


def test_one_rank_reduction_and_seeds():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    seeds = {bench.rank_seed(7, r) for r in range(8)}
    assert len(seeds) == 8  # every rank draws its own replica


def test_warmup_below_three_is_refused(monkeypatch):
    monkeypatch.setattr(sys, "argv", ["bench.py", "--warmup", "2"])
    with pytest.raises(SystemExit):
        bench.main()


def test_dense_decode_leg_bookkeeping(monkeypatch):
    """The dense-decode baseline leg: one rtp_dense_attn call per step with the
    query at the last cache position, and the K/V bytes of every kv head."""
    import long_context_sparse_rtp_b200 as pkg
    B, L, H, Hkv = 8, 131072, 32, 4
    st = dict(q=torch.empty(B, 1, H, 128, device="meta"),
              k=torch.empty(B, L, Hkv, 128, device="meta"),
              v=torch.empty(B, L, Hkv, 128, device="meta"), L=L)
    calls = []

    def fake_dense(q, k, v, *, q_pos0, o, lse):
        calls.append((q_pos0, tuple(o.shape), tuple(lse.shape)))

    def fake_time_steps(fn, steps, warmup, world, flush):
        for _ in range(warmup + steps):
            fn()
        return 0.35 * steps, None

    monkeypatch.setattr(pkg, "rtp_dense_attn", fake_dense)
    monkeypatch.setattr(bench, "time_steps", fake_time_steps)

    class Args:
        steps, warmup = 4, 3

    r = bench.bench_decode_dense(dict(st=st, flush=None), Args)
    assert r["bytes"] == B * L * Hkv * 128 * 2 * 2 == 2147483648
    assert abs(r["ms_step"] - 0.35) < 1e-12
    assert calls == [(L - 1, (B, 1, H, 128), (B, H, 1))] * 7


def test_attention_pair_counts_against_brute_force():
    """The roofline pair counts: the sink + window rule summed over rows, and
    the 128 x 128 tiles the causal / local schedules visit, against explicit
    enumeration on small sizes."""
    import numpy as np
    for L, W, S in [(1, 1, 0), (5, 3, 1), (300, 37, 4), (1000, 256, 4), (700, 1000, 0)]:
        brute = sum(len([j for j in range(P + 1) if j < S or j > P - W]) for P in range(L))
        assert bench.local_pairs(L, W, S) == brute
    for L, W, S in [(1, 1, 0), (200, 64, 4), (1000, 256, 4), (1300, 300, 130)]:
        nb = (L + 127) // 128
        dense = local = 0
        for rb in range(nb):
            P0, Pl = rb * 128, min(L, rb * 128 + 128) - 1
            for t in range(Pl // 128 + 1):
                dense += 1
                keys = range(t * 128, t * 128 + 128)
                # a tile is visited iff some row of the block keeps some key of it
                if any(j <= P and (j < S or j > P - W) for P in range(P0, Pl + 1) for j in keys):
                    local += 1
        assert bench.tile_pairs(L) == dense * 128 * 128
        assert bench.tile_pairs(L, W, S) == local * 128 * 128, (L, W, S)
