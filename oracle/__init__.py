"""Plain fp64 CPU oracle for the RTPurbo attention hot path.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; never by the product package.  The
arithmetic lives in ``rtp_oracle.c`` (plain C, fp64, OpenMP over independent
rows); this module compiles it with gcc and marshals numpy arrays.  It shares no
code with the CUDA library.

bf16 tensors travel as their raw 16-bit patterns (``numpy.uint16``).

What each function follows (the paper-graph-ui summary page of "Full Attention
Strikes Back: Transferring Full Attention into Sparse within Hundred Training
Steps", arXiv 2605.16928, cited by section):

* ``project``     -- §Low-Dimensional Projection Mechanism (16-dim W^Q, W^K),
                     rounded once to bf16 (the indexer's quantisation point).
* ``scores``      -- same section, the score s(m, n) = q16_m . k16_n.
* ``topp``        -- §Dynamic Top-p Selection Mechanism, Eq. 5 (softmax of the
                     indexer scores, smallest highest-score prefix reaching p);
                     ties go to the lower index.
* ``attend``      -- same section, exact softmax attention over the kept set
                     with the 1/sqrt(d_h) scale.
* ``topk``        -- §5 Experimental Analysis, the method's static top-k
                     variant (k = 4096): the k highest scores, ties to the
                     lower index.
* ``block_topp``  -- §Hardware-Aware Fast Top-p Decoding Kernel, steps 1-5:
                     64-key blocks reduced to (max, log-sum-exp), a 256-bin
                     histogram over the block maxima, a walk down the bins to
                     mass p, whole blocks selected.
* ``local_set``   -- §Local Head Attention Pattern (sinks + sliding window).
* ``retrieval_rows`` / ``local_rows`` / ``dense_rows`` -- the above per row.

Every function is pinned by tests in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rtp_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "liborc.so")
_lib = None

D = 128
R = 16


def build(force: bool = False) -> str:
    """Compile rtp_oracle.c into oracle/_build/liborc.so (gcc, -O2, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
           "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.orc_double_to_bf16.restype = ctypes.c_uint16
        _lib.orc_double_to_bf16.argtypes = [ctypes.c_double]
        _lib.orc_bf16_to_double.restype = ctypes.c_double
        _lib.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        _lib.orc_local_set.restype = ctypes.c_int64
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 patterns (pure numpy; no rounding involved)."""
    u = _c(bits, np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bits, round-to-nearest-even (the oracle's rounding)."""
    lib = _load()
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    lib.orc_bf16_round_array(_p(x), ctypes.c_int64(x.size), _p(out))
    return out


def project(x_bits: np.ndarray, W_bits: np.ndarray):
    """x [n,128] bf16 bits, W [128,16] bf16 bits -> (bf16 bits [n,16], fp64 pre-rounding [n,16])."""
    lib = _load()
    x = _c(x_bits, np.uint16).reshape(-1, D)
    W = _c(W_bits, np.uint16).reshape(D, R)
    n = x.shape[0]
    out = np.empty((n, R), np.uint16)
    pre = np.empty((n, R), np.float64)
    lib.orc_project_rows(_p(x), ctypes.c_int64(n), ctypes.c_int64(D), _p(W),
                         _p(out), ctypes.c_int64(R), _p(pre))
    return out, pre


def scores(q16_bits: np.ndarray, k16_bits: np.ndarray) -> np.ndarray:
    """q16 [16], k16 [n,16] (bf16 bits) -> fp64 scores [n]."""
    lib = _load()
    q = _c(q16_bits, np.uint16).reshape(R)
    k = _c(k16_bits, np.uint16).reshape(-1, R)
    s = np.empty(k.shape[0], np.float64)
    lib.orc_scores(_p(q), _p(k), ctypes.c_int64(k.shape[0]), ctypes.c_int64(R), _p(s))
    return s


def topp(s: np.ndarray, p: float) -> dict:
    """Top-P of one row of scores.  Returns sel (bool [n]), t, jtie, count, mass_frac, Z, m."""
    lib = _load()
    s = _c(s, np.float64).reshape(-1)
    n = s.size
    if n < 1:
        raise ValueError("top-p needs at least one key")
    sel = np.empty(n, np.uint8)
    t = ctypes.c_double()
    Z = ctypes.c_double()
    m = ctypes.c_double()
    mf = ctypes.c_double()
    jt = ctypes.c_int64()
    cnt = ctypes.c_int64()
    lib.orc_topp(_p(s), ctypes.c_int64(n), ctypes.c_double(p), _p(sel),
                 ctypes.byref(t), ctypes.byref(jt), ctypes.byref(cnt),
                 ctypes.byref(mf), ctypes.byref(Z), ctypes.byref(m))
    return dict(sel=sel.astype(bool), t=t.value, jtie=jt.value, count=cnt.value,
                mass_frac=mf.value, Z=Z.value, m=m.value)


def topk(s: np.ndarray, k: int) -> dict:
    """Static top-k of one row of scores.  Returns sel (bool [n]), t, jtie, count."""
    lib = _load()
    s = _c(s, np.float64).reshape(-1)
    n = s.size
    if n < 1 or k < 1:
        raise ValueError("top-k needs at least one key and k >= 1")
    sel = np.empty(n, np.uint8)
    t = ctypes.c_double()
    jt = ctypes.c_int64()
    cnt = ctypes.c_int64()
    lib.orc_topk(_p(s), ctypes.c_int64(n), ctypes.c_int64(k), _p(sel), ctypes.byref(t),
                 ctypes.byref(jt), ctypes.byref(cnt))
    return dict(sel=sel.astype(bool), t=t.value, jtie=jt.value, count=cnt.value)


def block_topp(s: np.ndarray, p: float, block: int = 64, nbins: int = 256) -> dict:
    """Block-level approximate top-p of one row of scores.  Returns bsel (bool
    [nb]), bin (int [nb]), kstar, sel (bool [n], the kept tokens), count,
    mass_frac (kept share of the token softmax mass)."""
    lib = _load()
    s = _c(s, np.float64).reshape(-1)
    n = s.size
    if n < 1:
        raise ValueError("block top-p needs at least one key")
    nb = (n + block - 1) // block
    bsel = np.empty(nb, np.uint8)
    bins = np.empty(nb, np.int64)
    ks = ctypes.c_int64()
    cnt = ctypes.c_int64()
    mf = ctypes.c_double()
    lib.orc_block_topp(_p(s), ctypes.c_int64(n), ctypes.c_double(p), ctypes.c_int64(block),
                       ctypes.c_int64(nbins), _p(bsel), _p(bins), ctypes.byref(ks),
                       ctypes.byref(cnt), ctypes.byref(mf))
    bsel = bsel.astype(bool)
    return dict(bsel=bsel, bin=bins, kstar=ks.value, sel=np.repeat(bsel, block)[:n],
                count=cnt.value, mass_frac=mf.value)


def attend(q_bits, K_bits, V_bits, idx, scale: float):
    """Exact attention of one query over the key rows idx (ascending). Returns (o fp64 [128], lse)."""
    lib = _load()
    q = _c(q_bits, np.uint16).reshape(D)
    K = _c(K_bits, np.uint16).reshape(-1, D)
    V = _c(V_bits, np.uint16).reshape(-1, D)
    idx = _c(idx, np.int64).reshape(-1)
    if idx.size < 1:
        raise ValueError("attention needs at least one key")
    o = np.empty(D, np.float64)
    lse = ctypes.c_double()
    lib.orc_attend(_p(q), _p(K), ctypes.c_int64(D), _p(V), ctypes.c_int64(D),
                   _p(idx), ctypes.c_int64(idx.size), ctypes.c_double(scale),
                   _p(o), ctypes.byref(lse))
    return o, lse.value


def local_set(P: int, window: int, n_sink: int) -> np.ndarray:
    lib = _load()
    idx = np.empty(P + 1, np.int64)
    n = lib.orc_local_set(ctypes.c_int64(P), ctypes.c_int64(window),
                          ctypes.c_int64(n_sink), _p(idx))
    return idx[:n].copy()


def _dims(B, Lq, Lk, H, Hkv, q_pos0):
    return np.array([B, Lq, Lk, H, Hkv, q_pos0], np.int64)


def retrieval_rows(q, k, v, q16, k16, rows, row_hq16, row_hk16, *, H, Hkv,
                   q_pos0, p, scale, want_sel=False):
    """Retrieval-head rows end to end on the given q16/k16.

    q [B,Lq,H,128], k/v [B,Lk,Hkv,128], q16 [B,Lq,Hq16,16], k16 [B,Lk,Hk16,16]
    (bf16 bits).  rows: int array [n,3] of (b, i, h).  row_hq16/row_hk16: the
    head slot of each row in q16 / k16.  Returns a dict with o [n,128], lse,
    t, jtie, count, mass_frac and (want_sel) a list of bool masks over 0..P.
    """
    lib = _load()
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    q16 = _c(q16, np.uint16)
    k16 = _c(k16, np.uint16)
    B, Lq = q.shape[0], q.shape[1]
    Lk = k.shape[1]
    rows = _c(rows, np.int64).reshape(-1, 3)
    n = rows.shape[0]
    rb, ri, rh = (_c(rows[:, c], np.int64) for c in range(3))
    hq = _c(row_hq16, np.int64).reshape(n)
    hk = _c(row_hk16, np.int64).reshape(n)
    o = np.empty((n, D), np.float64)
    lse = np.empty(n, np.float64)
    t = np.empty(n, np.float64)
    jt = np.empty(n, np.int64)
    cnt = np.empty(n, np.int64)
    mf = np.empty(n, np.float64)
    sel = sel_off = None
    if want_sel:
        lens = q_pos0 + ri + 1
        sel_off = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
        sel = np.zeros(int(lens.sum()), np.uint8)
    lib.orc_retrieval_rows(
        _p(_dims(B, Lq, Lk, H, Hkv, q_pos0)), _p(q), _p(k), _p(v),
        _p(q16), ctypes.c_int64(q16.shape[2]), _p(k16), ctypes.c_int64(k16.shape[2]),
        ctypes.c_int64(n), _p(rb), _p(ri), _p(rh), _p(hq), _p(hk),
        ctypes.c_double(p), ctypes.c_double(scale), _p(o), _p(lse), _p(t),
        _p(jt), _p(cnt), _p(mf),
        _p(sel) if want_sel else None, _p(sel_off) if want_sel else None)
    out = dict(o=o, lse=lse, t=t, jtie=jt, count=cnt, mass_frac=mf)
    if want_sel:
        out["sel"] = [sel[sel_off[r]:sel_off[r] + q_pos0 + ri[r] + 1].astype(bool)
                      for r in range(n)]
    return out


def local_rows(q, k, v, rows, *, H, Hkv, q_pos0, window, n_sink, scale):
    """Local-head rows (sinks + window).  Returns dict(o [n,128], lse [n])."""
    lib = _load()
    q = _c(q, np.uint16)
    k = _c(k, np.uint16)
    v = _c(v, np.uint16)
    B, Lq = q.shape[0], q.shape[1]
    Lk = k.shape[1]
    rows = _c(rows, np.int64).reshape(-1, 3)
    n = rows.shape[0]
    rb, ri, rh = (_c(rows[:, c], np.int64) for c in range(3))
    o = np.empty((n, D), np.float64)
    lse = np.empty(n, np.float64)
    lib.orc_local_rows(_p(_dims(B, Lq, Lk, H, Hkv, q_pos0)), _p(q), _p(k), _p(v),
                       ctypes.c_int64(n), _p(rb), _p(ri), _p(rh),
                       ctypes.c_int64(window), ctypes.c_int64(n_sink),
                       ctypes.c_double(scale), _p(o), _p(lse))
    return dict(o=o, lse=lse)


def dense_rows(q, k, v, rows, *, H, Hkv, q_pos0, scale):
    """Dense causal rows: every key 0..P (the local set with an unbounded window)."""
    Lk = np.asarray(k).shape[1]
    return local_rows(q, k, v, rows, H=H, Hkv=Hkv, q_pos0=q_pos0,
                      window=Lk + q_pos0 + 1, n_sink=0, scale=scale)
