"""One mixed attention layer through the C ABI, in call order.

prefill:  rtp_index_scores -> rtp_topp_select -> rtp_sparse_attn_prefill
          (retrieval heads) and rtp_local_attn (local heads) into one output;
          or, retrieval="dense", the k16 projection and dense attention on the
          retrieval heads (every causal key) with the same local heads.
decode:   rtp_index_scores on the new token (q16 + k16 append into the cache)
          -> rtp_sparse_attn_decode (retrieval heads) and rtp_local_attn (local
          heads, Lq = 1) into one output.
Only sequencing and buffer allocation happen here; every step runs in librtp.so.
"""
from __future__ import annotations

import torch

from .rtp import (rtp_index_scores, rtp_local_attn, rtp_local_attn_decode_ring,
                  rtp_local_ring_write, rtp_sparse_attn_decode, rtp_sparse_attn_decode_select,
                  rtp_sparse_attn_prefill, rtp_topp_select)


def rtp_layer_prefill(q, k, v, Wq16, Wk16, kv_role, *, p, window, n_sink, scale=None,
                      k16_per_kv_head=0, stream=None, retrieval="topp", q_idx=None,
                      k_idx=None):
    """Causal prefill of one layer.  Returns dict(o, lse, q16, k16, sel).

    retrieval="topp": exact top-p selection and sparse attention on the retrieval
    heads.  retrieval="dense": the retrieval heads attend to every causal key
    (the summary's own prefill, where only the local heads are sparse); the
    k16 cache the decode steps need is still projected, q16 and sel are None.
    q_idx/k_idx: the indexer's inputs when they differ from q/k (pre-RoPE
    vectors, the summary's projection input); attention always uses q/k."""
    H = q.shape[2]
    q_idx = q if q_idx is None else q_idx
    k_idx = k if k_idx is None else k_idx
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], H, q.shape[1], dtype=torch.float32, device=q.device)
    if retrieval == "dense":
        _, k16 = rtp_index_scores(None, k_idx, Wq16, Wk16, kv_role, H=H,
                                  k16_per_kv_head=k16_per_kv_head, stream=stream)
        rtp_sparse_attn_prefill(q, k, v, None, None, None, None, kv_role, scale=scale,
                                k16_per_kv_head=k16_per_kv_head, o=o, lse=lse, stream=stream)
        rtp_local_attn(q, k, v, kv_role, window=window, n_sink=n_sink, scale=scale, o=o,
                       lse=lse, stream=stream)
        return dict(o=o, lse=lse, q16=None, k16=k16, sel=None)
    if retrieval != "topp":
        raise ValueError("retrieval must be 'topp' or 'dense'")
    q16, k16 = rtp_index_scores(q_idx, k_idx, Wq16, Wk16, kv_role,
                                k16_per_kv_head=k16_per_kv_head, stream=stream)
    sel = rtp_topp_select(q16, k16, kv_role, p, H=H, k16_per_kv_head=k16_per_kv_head,
                          stream=stream)
    rtp_sparse_attn_prefill(q, k, v, q16, k16, sel["thr"], sel["jtie"], kv_role, scale=scale,
                            k16_per_kv_head=k16_per_kv_head, o=o, lse=lse, stream=stream)
    rtp_local_attn(q, k, v, kv_role, window=window, n_sink=n_sink, scale=scale, o=o, lse=lse,
                   stream=stream)
    return dict(o=o, lse=lse, q16=q16, k16=k16, sel=sel)


def rtp_layer_decode(q, k_new, k_cache, v_cache, k16_cache, Wq16, Wk16, kv_role, *, pos, p,
                     window, n_sink, scale=None, k16_per_kv_head=0, stream=None, o=None,
                     lse=None, want_sel=True, q_idx=None, k_new_idx=None, select="topp",
                     top_k=4096, local_ring=None, v_new=None):
    """One decode token at position `pos` (the caches already hold its k/v row;
    its k16 row is written here).  Returns dict(o, lse, q16, sel).
    q_idx/k_new_idx: the indexer's inputs when they differ from q/k_new
    (pre-RoPE vectors).  select: "topp" (exact top-p), "block_topp" or "topk"
    (top_k keys).  local_ring=(k_ring, v_ring): the local heads read a
    window-only ring cache instead of k_cache / v_cache; the new token's local
    rows (k_new, and v_new or row `pos` of v_cache) are appended to it here."""
    H = q.shape[2]
    if o is None:
        o = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[0], H, 1, dtype=torch.float32, device=q.device)
    main = torch.cuda.current_stream(q.device) if stream is None else stream
    # the local heads depend on nothing the retrieval heads compute: side stream
    side = _side_stream(q.device)
    side.wait_stream(main)
    kc, vc = k_cache[:, :pos + 1], v_cache[:, :pos + 1]
    if local_ring is None:
        rtp_local_attn(q, kc, vc, kv_role, window=window, n_sink=n_sink, scale=scale,
                       q_pos0=pos, o=o, lse=lse, stream=side)
    else:
        kr, vr = local_ring
        vn = v_cache[:, pos:pos + 1] if v_new is None else v_new
        rtp_local_ring_write(k_new, vn, kr, vr, kv_role, window=window, n_sink=n_sink, pos0=pos,
                             H=H, stream=side)
        rtp_local_attn_decode_ring(q, kr, vr, kv_role, window=window, n_sink=n_sink, pos=pos,
                                   scale=scale, o=o, lse=lse, stream=side)
    k16_row = k16_cache[:, pos:pos + 1]
    q16, _ = rtp_index_scores(q if q_idx is None else q_idx,
                              k_new if k_new_idx is None else k_new_idx, Wq16, Wk16, kv_role,
                              k16=k16_row,
                              k16_per_kv_head=k16_per_kv_head, stream=stream)
    if select == "topp":
        _, _, sel = rtp_sparse_attn_decode(q, kc, vc, q16, k16_cache[:, :pos + 1], kv_role, p,
                                           scale=scale, q_pos0=pos,
                                           k16_per_kv_head=k16_per_kv_head, o=o, lse=lse,
                                           want_sel=want_sel, stream=stream)
    else:
        _, _, sel = rtp_sparse_attn_decode_select(q, kc, vc, q16, k16_cache[:, :pos + 1],
                                                  kv_role, select, p=p, top_k=top_k,
                                                  scale=scale, q_pos0=pos,
                                                  k16_per_kv_head=k16_per_kv_head, o=o, lse=lse,
                                                  want_sel=want_sel, stream=stream)
    main.wait_stream(side)
    return dict(o=o, lse=lse, q16=q16, sel=sel)


_side_streams: dict = {}


def _side_stream(device):
    key = str(torch.device(device))
    s = _side_streams.get(key)
    if s is None:
        s = torch.cuda.Stream(device=device)
        _side_streams[key] = s
    return s


class DecodeGraph:
    """One decode step of the layer captured once in a CUDA graph and replayed.

    The step (indexer projection of the new token with its k16 append, exact
    top-p and gathered attention on the retrieval heads, sink+window attention on
    the local heads) issues several kernels; replaying them as one graph removes
    the per-launch host cost.  Inputs live in fixed device buffers: `q`
    [B, 1, H, 128] and row `pos` of the k/v caches; outputs in `o`, `lse`.
    """

    def __init__(self, k_cache, v_cache, k16_cache, Wq16, Wk16, kv_role, *, H, pos, p, window,
                 n_sink, scale=None, k16_per_kv_head=0, trace=False, select="topp", top_k=4096,
                 local_ring=None):
        B = k_cache.shape[0]
        dev = k_cache.device
        self.k_cache, self.v_cache, self.pos = k_cache, v_cache, pos
        self.q = torch.zeros(B, 1, H, 128, dtype=torch.bfloat16, device=dev)
        self.o = torch.empty_like(self.q)
        self.lse = torch.empty(B, H, 1, dtype=torch.float32, device=dev)
        args = (self.q, k_cache[:, pos:pos + 1], k_cache, v_cache, k16_cache, Wq16, Wk16, kv_role)
        kw = dict(pos=pos, p=p, window=window, n_sink=n_sink, scale=scale,
                  k16_per_kv_head=k16_per_kv_head, o=self.o, lse=self.lse, want_sel=False,
                  select=select, top_k=top_k, local_ring=local_ring)
        self._call = lambda: rtp_layer_decode(*args, **kw)
        self._call()                      # eager once: workspaces and buffers exist
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        if trace:  # the library's kernel-trace events become nodes of this graph
            from .rtp import lib
            lib().rtp_trace_reset()
            lib().rtp_trace_enable(1)
        try:
            with torch.cuda.graph(self.graph, capture_error_mode="thread_local"):
                self._call()
        finally:
            if trace:
                lib().rtp_trace_enable(0)

    def replay(self):
        self.graph.replay()

    def _io(self, q_host, k_host, v_host, o_host):
        """The three input copies run concurrently (two on helper streams), then
        the step, then the output copy."""
        pos = self.pos
        main = torch.cuda.current_stream()
        if not hasattr(self, "_copy_streams"):
            self._copy_streams = [torch.cuda.Stream(device=self.q.device) for _ in range(2)]
        for cs in self._copy_streams:
            cs.wait_stream(main)
        with torch.cuda.stream(self._copy_streams[0]):
            self.k_cache[:, pos:pos + 1].copy_(k_host, non_blocking=True)
        with torch.cuda.stream(self._copy_streams[1]):
            self.v_cache[:, pos:pos + 1].copy_(v_host, non_blocking=True)
        self.q.copy_(q_host, non_blocking=True)
        for cs in self._copy_streams:
            main.wait_stream(cs)
        self._call()
        o_host.copy_(self.o, non_blocking=True)

    def step(self, q_host, k_host, v_host, o_host):
        """Copy the new token in from (pinned) host buffers, run, copy o out.

        For one set of pinned host buffers the copies are captured together with
        the step into a second graph (built on the first call with those
        buffers), so a step is one graph launch; other host buffers take the
        copies one by one around the step's graph."""
        bufs = (q_host, k_host, v_host, o_host)
        key = tuple(t.data_ptr() for t in bufs)
        pinned = all(t.is_pinned() for t in bufs)
        if pinned and getattr(self, "_io_key", None) == key:
            self._io_graph.replay()
            return o_host
        if pinned and getattr(self, "_io_key", None) is None:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, capture_error_mode="thread_local"):
                self._io(*bufs)
            self._io_graph, self._io_key = g, key
            self._io_graph.replay()
            return o_host
        pos = self.pos
        self.q.copy_(q_host, non_blocking=True)
        self.k_cache[:, pos:pos + 1].copy_(k_host, non_blocking=True)
        self.v_cache[:, pos:pos + 1].copy_(v_host, non_blocking=True)
        self.graph.replay()
        o_host.copy_(self.o, non_blocking=True)
        return o_host
