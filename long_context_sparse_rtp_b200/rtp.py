"""Thin Python binding of librtp.so (ctypes).

Argument marshalling only: every step of the layer runs in the CUDA library.
torch provides device memory and the current stream.  The functions carry the
C entry points' names; see include/rtp.h for the exact contracts.

If the shared library is missing or cannot be loaded this module raises on
first use -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librtp.so")

RTP_OK = 0
STATUS = {0: "RTP_OK", 1: "RTP_ERR_INVALID_ARG", 2: "RTP_ERR_UNSUPPORTED",
          3: "RTP_ERR_ALIGNMENT", 4: "RTP_ERR_WORKSPACE_TOO_SMALL", 5: "RTP_ERR_CUDA",
          6: "RTP_ERR_DEVICE_TIMEOUT", 7: "RTP_ERR_SCRATCH_LIMIT"}
OP_INDEX_SCORES, OP_TOPP_SELECT, OP_SPARSE_PREFILL, OP_SPARSE_DECODE, OP_LOCAL, OP_DENSE = range(6)
SELECT_TOPP, SELECT_BLOCK_TOPP, SELECT_TOPK = range(3)
SELECT = {"topp": SELECT_TOPP, "block_topp": SELECT_BLOCK_TOPP, "topk": SELECT_TOPK}


class RtpError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Lq", ctypes.c_int32), ("Lk", ctypes.c_int32),
                ("H", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32),
                ("q_pos0", ctypes.c_int64)]


class View(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("stride_b", ctypes.c_int64),
                ("stride_l", ctypes.c_int64)]


_lib = None
_lock = threading.Lock()


def lib():
    """Load librtp.so (raises if it is not built)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is not built; run `python -m long_context_sparse_rtp_b200.build`")
                L = ctypes.CDLL(LIB_PATH)
                V, S, P = View, ctypes.POINTER(Shape), ctypes.c_void_p
                i32, f32, sz = ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
                L.rtp_workspace_size.restype = sz
                L.rtp_workspace_size.argtypes = [ctypes.c_int, S, P, i32]
                L.rtp_workspace_init.argtypes = [P, sz, P]
                L.rtp_index_scores.argtypes = [S, P, i32, V, V, P, P, V, V, P]
                L.rtp_topp_select.argtypes = [S, P, i32, V, V, f32, P, P, P, P, P, sz, P]
                L.rtp_sparse_attn_prefill.argtypes = [S, P, i32, V, V, V, V, V, P, P, f32, V, P,
                                                      P, sz, P]
                L.rtp_sparse_attn_decode.argtypes = [S, P, i32, V, V, V, V, V, f32, f32, V, P,
                                                     P, P, P, P, P, sz, P]
                L.rtp_sparse_attn_decode_select.argtypes = [S, P, i32, V, V, V, V, V, i32, f32,
                                                            i32, f32, V, P, P, P, P, P, P, P,
                                                            P, sz, P]
                L.rtp_local_attn.argtypes = [S, P, i32, i32, V, V, V, f32, V, P, P, sz, P]
                L.rtp_local_ring_write.argtypes = [S, P, i32, i32, V, V, V, V, P]
                L.rtp_local_attn_decode_ring.argtypes = [S, P, i32, i32, V, V, V, f32, V, P, P,
                                                         sz, P]
                L.rtp_dense_attn.argtypes = [S, V, V, V, f32, V, P, P, sz, P]
                L.rtp_local_attn_decode_noalloc.argtypes = [S, P, i32, i32, V, V, V, f32, V, P, P]
                L.rtp_probe_ex2.argtypes = [i32, i32, P, P]
                L.rtp_status_string.restype = ctypes.c_char_p
                L.rtp_status_string.argtypes = [ctypes.c_int]
                L.rtp_get_device_status.argtypes = [P, P]
                L.rtp_version.restype = ctypes.c_char_p
                for fn in ("rtp_workspace_init", "rtp_index_scores", "rtp_topp_select",
                           "rtp_sparse_attn_prefill", "rtp_sparse_attn_decode",
                           "rtp_sparse_attn_decode_select", "rtp_local_attn",
                           "rtp_local_ring_write", "rtp_local_attn_decode_ring", "rtp_probe_ex2", "rtp_dense_attn", "rtp_get_device_status",
                           "rtp_local_attn_decode_noalloc"):
                    getattr(L, fn).restype = ctypes.c_int
                _lib = L
    return _lib


def _check(fn: str, code: int):
    if code != RTP_OK:
        raise RtpError(fn, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def view(t: torch.Tensor | None, width: int = 128) -> View:
    """[B][L][heads][width] tensor -> rtp_view (heads x width contiguous per row)."""
    if t is None:
        return View(None, 0, 0)
    if t.dim() != 4 or t.stride(3) != 1 or t.stride(2) != width:
        raise ValueError("expected a [B, L, heads, width] tensor with contiguous heads*width")
    return View(ctypes.c_void_p(t.data_ptr()), t.stride(0), t.stride(1))


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _role(kv_role):
    arr = (ctypes.c_uint8 * len(kv_role))(*[int(x) for x in kv_role])
    return arr


def _shape(B, Lq, Lk, H, Hkv, q_pos0):
    return Shape(B, Lq, Lk, H, Hkv, 128, q_pos0)


# --------------------------------------------------------------------- workspaces
_ws_cache: dict = {}


def workspace(op: int, shape: Shape, role, k16_per_kv: int, device, stream=None) -> torch.Tensor:
    """A zero-initialised workspace of the size the library asks for, cached per
    (device, op) and grown on demand.  The binding's convenience functions share
    it, so they must not run concurrently on several streams; callers that need
    that pass their own workspace through the C ABI."""
    need = lib().rtp_workspace_size(op, ctypes.byref(shape), role, k16_per_kv)
    key = (str(torch.device(device)), op)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def rtp_workspace_size(op: int, shape: Shape, kv_role, k16_per_kv_head: int = 0) -> int:
    return lib().rtp_workspace_size(op, ctypes.byref(shape), _role(kv_role), k16_per_kv_head)


def rtp_status_string(code: int) -> str:
    return lib().rtp_status_string(code).decode()


def rtp_probe_ex2(blocks: int, iters: int, out: torch.Tensor, stream=None) -> None:
    """The ex2-rate probe kernel (blocks x 256 threads x iters x 8 ex2)."""
    _check("rtp_probe_ex2", lib().rtp_probe_ex2(blocks, iters, _ptr(out), _stream(stream)))


def rtp_version() -> str:
    return lib().rtp_version().decode()


def rtp_get_device_status(ws: torch.Tensor, stream=None) -> int:
    return lib().rtp_get_device_status(_ptr(ws), _stream(stream))


def rtp_check_device(device=None, stream=None) -> None:
    """Reads (and clears) the device status word of every workspace the binding
    holds for `device`; raises RtpError if a kernel recorded an error since the
    last check (a bounded wait that ran out, or an internal consistency check).
    Synchronises the stream."""
    dev = str(torch.device(device if device is not None else "cuda"))
    if dev == "cuda":
        dev = f"cuda:{torch.cuda.current_device()}"
    for (d, op), ws in list(_ws_cache.items()):
        if d != dev:
            continue
        where = int(ws[4:8].view(torch.int32).item())
        code = rtp_get_device_status(ws, stream)
        if code != RTP_OK:
            raise RtpError(f"device status of op {op} (site {where})", code)


# --------------------------------------------------------------------- entry points
def _n_ret(kv_role, G):
    return int(sum(int(x) for x in kv_role)) * G


def rtp_index_scores(q, k, Wq16, Wk16, kv_role, *, q16=None, k16=None, k16_per_kv_head=0,
                     H=None, stream=None):
    """16-dim indexer projections.  q [B,Lq,H,128] (or None), k [B,Lk,Hkv,128] (or None;
    then pass H, the query head count).
    Returns (q16 [B,Lq,H_ret,16], k16 [B,Lk,H_k16,16]); pass q16/k16 to write in place."""
    ref = q if q is not None else k
    B = ref.shape[0]
    H = q.shape[2] if q is not None else H
    Hkv = len(kv_role)
    if H is None:
        raise ValueError("pass q or H for the head count")
    G = H // Hkv
    n_ret = _n_ret(kv_role, G)
    H_k16 = int(sum(int(x) for x in kv_role)) if k16_per_kv_head else n_ret
    Lq = q.shape[1] if q is not None else 0
    Lk = k.shape[1] if k is not None else 0
    dev = ref.device
    if q is not None and q16 is None:
        q16 = torch.empty(B, Lq, n_ret, 16, dtype=torch.bfloat16, device=dev)
    if k is not None and k16 is None:
        k16 = torch.empty(B, Lk, H_k16, 16, dtype=torch.bfloat16, device=dev)
    shp = _shape(B, Lq, Lk, H, Hkv, 0)
    _check("rtp_index_scores", lib().rtp_index_scores(
        ctypes.byref(shp), _role(kv_role), k16_per_kv_head, view(q), view(k),
        _ptr(Wq16), _ptr(Wk16), view(q16, 16), view(k16, 16), _stream(stream)))
    return q16, k16


def rtp_topp_select(q16, k16, kv_role, p, *, H, q_pos0=0, k16_per_kv_head=0, want_mass=True,
                    stream=None):
    """Exact top-p per retrieval row.  Returns dict(thr, jtie, count, mass) of [B,H_ret,Lq]."""
    B, Lq, n_ret = q16.shape[0], q16.shape[1], q16.shape[2]
    Lk = k16.shape[1]
    Hkv = len(kv_role)
    dev = q16.device
    thr = torch.empty(B, n_ret, Lq, dtype=torch.float32, device=dev)
    jtie = torch.empty(B, n_ret, Lq, dtype=torch.int32, device=dev)
    count = torch.empty(B, n_ret, Lq, dtype=torch.int32, device=dev)
    mass = torch.empty(B, n_ret, Lq, dtype=torch.float32, device=dev) if want_mass else None
    shp = _shape(B, Lq, Lk, H, Hkv, q_pos0)
    role = _role(kv_role)
    ws = workspace(OP_TOPP_SELECT, shp, role, k16_per_kv_head, dev, stream)
    _check("rtp_topp_select", lib().rtp_topp_select(
        ctypes.byref(shp), role, k16_per_kv_head, view(q16, 16), view(k16, 16),
        ctypes.c_float(p), _ptr(thr), _ptr(jtie), _ptr(count), _ptr(mass), _ptr(ws),
        ws.numel(), _stream(stream)))
    return dict(thr=thr, jtie=jtie, count=count, mass=mass)


def rtp_sparse_attn_prefill(q, k, v, q16, k16, thr, jtie, kv_role, *, scale=None, q_pos0=0,
                            k16_per_kv_head=0, o=None, lse=None, stream=None):
    """Exact attention over the kept sets (retrieval heads).  Returns (o, lse).
    thr = jtie = None keeps every causal key (p >= 1) on the dense tile schedule;
    q16/k16 may then be None."""
    B, Lq, H, _ = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    dev = q.device
    if o is None:
        o = torch.zeros_like(q)
    if lse is None:
        lse = torch.full((B, H, Lq), float("nan"), dtype=torch.float32, device=dev)
    scale = 1.0 / (128 ** 0.5) if scale is None else scale
    shp = _shape(B, Lq, Lk, H, Hkv, q_pos0)
    role = _role(kv_role)
    ws = workspace(OP_SPARSE_PREFILL, shp, role, k16_per_kv_head, dev, stream)
    _check("rtp_sparse_attn_prefill", lib().rtp_sparse_attn_prefill(
        ctypes.byref(shp), role, k16_per_kv_head, view(q), view(k), view(v), view(q16, 16),
        view(k16, 16), _ptr(thr), _ptr(jtie), ctypes.c_float(scale), view(o), _ptr(lse),
        _ptr(ws), ws.numel(), _stream(stream)))
    return o, lse


def rtp_sparse_attn_decode(q, k_cache, v_cache, q16, k16_cache, kv_role, p, *, scale=None,
                           q_pos0=None, k16_per_kv_head=0, o=None, lse=None, want_sel=True,
                           stream=None):
    """One decode step for the retrieval heads.  q [B,1,H,128].
    Returns (o, lse, dict(thr, jtie, count, mass) of [B,H_ret])."""
    B, Lq, H, _ = q.shape
    Lk, Hkv = k_cache.shape[1], k_cache.shape[2]
    dev = q.device
    n_ret = q16.shape[2]
    q_pos0 = Lk - 1 if q_pos0 is None else q_pos0
    if o is None:
        o = torch.zeros_like(q)
    if lse is None:
        lse = torch.full((B, H, 1), float("nan"), dtype=torch.float32, device=dev)
    sel = None
    if want_sel:
        sel = dict(thr=torch.empty(B, n_ret, dtype=torch.float32, device=dev),
                   jtie=torch.empty(B, n_ret, dtype=torch.int32, device=dev),
                   count=torch.empty(B, n_ret, dtype=torch.int32, device=dev),
                   mass=torch.empty(B, n_ret, dtype=torch.float32, device=dev))
    scale = 1.0 / (128 ** 0.5) if scale is None else scale
    shp = _shape(B, Lq, Lk, H, Hkv, q_pos0)
    role = _role(kv_role)
    ws = workspace(OP_SPARSE_DECODE, shp, role, k16_per_kv_head, dev, stream)
    g = (lambda key: _ptr(sel[key])) if sel else (lambda key: None)
    _check("rtp_sparse_attn_decode", lib().rtp_sparse_attn_decode(
        ctypes.byref(shp), role, k16_per_kv_head, view(q), view(k_cache), view(v_cache),
        view(q16, 16), view(k16_cache, 16), ctypes.c_float(p), ctypes.c_float(scale), view(o),
        _ptr(lse), g("thr"), g("jtie"), g("count"), g("mass"), _ptr(ws), ws.numel(),
        _stream(stream)))
    return o, lse, sel


def rtp_sparse_attn_decode_select(q, k_cache, v_cache, q16, k16_cache, kv_role, select, *,
                                  p=0.95, top_k=4096, scale=None, q_pos0=None,
                                  k16_per_kv_head=0, o=None, lse=None, want_scores=False,
                                  want_sel=True, stream=None):
    """One decode step for the retrieval heads with selection rule `select`
    ("topp", "block_topp" or "topk").  Returns (o, lse, sel) with sel a dict of
    [B, H_ret] tensors (thr, jtie, count, mass; thr/jtie unwritten for
    block_topp), plus block_mask [B, H_ret, words] int32 (block_topp) and
    scores [B, H_ret, P + 1] fp32 (want_scores)."""
    B, Lq, H, _ = q.shape
    Lk, Hkv = k_cache.shape[1], k_cache.shape[2]
    dev = q.device
    n_ret = q16.shape[2]
    q_pos0 = Lk - 1 if q_pos0 is None else q_pos0
    N = q_pos0 + 1
    mode = SELECT[select]
    if o is None:
        o = torch.zeros_like(q)
    if lse is None:
        lse = torch.full((B, H, 1), float("nan"), dtype=torch.float32, device=dev)
    sel = {}
    if want_sel:
        sel = dict(thr=torch.full((B, n_ret), float("nan"), dtype=torch.float32, device=dev),
                   jtie=torch.full((B, n_ret), -1, dtype=torch.int32, device=dev),
                   count=torch.empty(B, n_ret, dtype=torch.int32, device=dev),
                   mass=torch.empty(B, n_ret, dtype=torch.float32, device=dev))
        words = ((N + 63) // 64 + 31) // 32
        if mode == SELECT_BLOCK_TOPP:
            sel["block_mask"] = torch.zeros(B, n_ret, words, dtype=torch.int32, device=dev)
    if want_scores:
        sel["scores"] = torch.empty(B, n_ret, N, dtype=torch.float32, device=dev)
    scale = 1.0 / (128 ** 0.5) if scale is None else scale
    shp = _shape(B, Lq, Lk, H, Hkv, q_pos0)
    role = _role(kv_role)
    ws = workspace(OP_SPARSE_DECODE, shp, role, k16_per_kv_head, dev, stream)
    _check("rtp_sparse_attn_decode_select", lib().rtp_sparse_attn_decode_select(
        ctypes.byref(shp), role, k16_per_kv_head, view(q), view(k_cache), view(v_cache),
        view(q16, 16), view(k16_cache, 16), mode, ctypes.c_float(p), int(top_k),
        ctypes.c_float(scale), view(o), _ptr(lse), _ptr(sel.get("thr")), _ptr(sel.get("jtie")),
        _ptr(sel.get("count")), _ptr(sel.get("mass")), _ptr(sel.get("block_mask")),
        _ptr(sel.get("scores")), _ptr(ws), ws.numel(), _stream(stream)))
    return o, lse, sel


def rtp_local_attn(q, k, v, kv_role, *, window, n_sink, scale=None, q_pos0=0, o=None,
                   lse=None, stream=None):
    """Sink + sliding-window attention on the local heads (prefill or Lq == 1 decode)."""
    B, Lq, H, _ = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    dev = q.device
    if o is None:
        o = torch.zeros_like(q)
    if lse is None:
        lse = torch.full((B, H, Lq), float("nan"), dtype=torch.float32, device=dev)
    scale = 1.0 / (128 ** 0.5) if scale is None else scale
    shp = _shape(B, Lq, Lk, H, Hkv, q_pos0)
    role = _role(kv_role)
    ws = workspace(OP_LOCAL, shp, role, 0, dev, stream)
    _check("rtp_local_attn", lib().rtp_local_attn(
        ctypes.byref(shp), role, window, n_sink, view(q), view(k), view(v),
        ctypes.c_float(scale), view(o), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return o, lse


def local_ring_alloc(B, kv_role, *, window, n_sink, device):
    """Zeroed (k_ring, v_ring) of [B, n_sink + window, n_local_kv, 128] bf16."""
    n_lkv = sum(1 for x in kv_role if int(x) == 0)
    shape = (B, n_sink + window, n_lkv, 128)
    return (torch.zeros(shape, dtype=torch.bfloat16, device=device),
            torch.zeros(shape, dtype=torch.bfloat16, device=device))


def rtp_local_ring_write(k, v, k_ring, v_ring, kv_role, *, window, n_sink, pos0=0, H=None,
                         stream=None):
    """Copy the local kv heads of k, v [B, n, Hkv, 128] (row i = position pos0 + i)
    into the ring cache; only the sinks and the last `window` positions land."""
    B, n, Hkv, _ = k.shape
    H = Hkv if H is None else H
    shp = _shape(B, n, n, H, Hkv, pos0)
    _check("rtp_local_ring_write", lib().rtp_local_ring_write(
        ctypes.byref(shp), _role(kv_role), window, n_sink, view(k), view(v), view(k_ring),
        view(v_ring), _stream(stream)))


def rtp_local_attn_decode_ring(q, k_ring, v_ring, kv_role, *, window, n_sink, pos, scale=None,
                               o=None, lse=None, stream=None):
    """Local heads of one decode token at position `pos` from the ring cache."""
    B, Lq, H, _ = q.shape
    Hkv = len(kv_role)
    if o is None:
        o = torch.zeros_like(q)
    if lse is None:
        lse = torch.full((B, H, 1), float("nan"), dtype=torch.float32, device=q.device)
    scale = 1.0 / (128 ** 0.5) if scale is None else scale
    shp = _shape(B, 1, pos + 1, H, Hkv, pos)
    role = _role(kv_role)
    ws = workspace(OP_LOCAL, shp, role, 0, q.device, stream)
    _check("rtp_local_attn_decode_ring", lib().rtp_local_attn_decode_ring(
        ctypes.byref(shp), role, window, n_sink, view(q), view(k_ring), view(v_ring),
        ctypes.c_float(scale), view(o), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return o, lse


def rtp_dense_attn(q, k, v, *, scale=None, q_pos0=0, o=None, lse=None, stream=None):
    """Dense causal attention baseline on every head."""
    B, Lq, H, _ = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    dev = q.device
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Lq), dtype=torch.float32, device=dev)
    scale = 1.0 / (128 ** 0.5) if scale is None else scale
    shp = _shape(B, Lq, Lk, H, Hkv, q_pos0)
    role = _role([0] * Hkv)
    ws = workspace(OP_DENSE, shp, role, 0, dev, stream)
    _check("rtp_dense_attn", lib().rtp_dense_attn(
        ctypes.byref(shp), view(q), view(k), view(v), ctypes.c_float(scale), view(o),
        _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)))
    return o, lse


def rtp_local_attn_decode_noalloc(q, k, v, kv_role, *, window, n_sink, scale=None, q_pos0=None,
                                  o=None, lse=None, stream=None):
    """Local-head decode (Lq == 1) that allocates nothing inside the library: its
    scratch is a fixed 8 MiB device array.  For callers that cannot provide a
    workspace.  Calls that overlap on the GPU race on that array."""
    B, Lq, H, _ = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    q_pos0 = Lk - 1 if q_pos0 is None else q_pos0
    if o is None:
        o = torch.zeros_like(q)
    if lse is None:
        lse = torch.full((B, H, Lq), float("nan"), dtype=torch.float32, device=q.device)
    scale = 1.0 / (128 ** 0.5) if scale is None else scale
    shp = _shape(B, Lq, Lk, H, Hkv, q_pos0)
    _check("rtp_local_attn_decode_noalloc", lib().rtp_local_attn_decode_noalloc(
        ctypes.byref(shp), _role(kv_role), window, n_sink, view(q), view(k), view(v),
        ctypes.c_float(scale), view(o), _ptr(lse), _stream(stream)))
    return o, lse
