"""One mixed attention layer through the C ABI, in call order.

prefill:  rtp_index_scores -> rtp_topp_select -> rtp_sparse_attn_prefill
          (retrieval heads) and rtp_local_attn (local heads) into one output.
decode:   rtp_index_scores on the new token (q16 + k16 append into the cache)
          -> rtp_sparse_attn_decode (retrieval heads) and rtp_local_attn (local
          heads, Lq = 1) into one output.
Only sequencing and buffer allocation happen here; every step runs in librtp.so.
"""
from __future__ import annotations

import torch

from .rtp import (rtp_index_scores, rtp_local_attn, rtp_sparse_attn_decode,
                  rtp_sparse_attn_prefill, rtp_topp_select)


def rtp_layer_prefill(q, k, v, Wq16, Wk16, kv_role, *, p, window, n_sink, scale=None,
                      k16_per_kv_head=0, stream=None):
    """Causal prefill of one layer.  Returns dict(o, lse, q16, k16, sel)."""
    H = q.shape[2]
    q16, k16 = rtp_index_scores(q, k, Wq16, Wk16, kv_role, k16_per_kv_head=k16_per_kv_head,
                                stream=stream)
    sel = rtp_topp_select(q16, k16, kv_role, p, H=H, k16_per_kv_head=k16_per_kv_head,
                          stream=stream)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], H, q.shape[1], dtype=torch.float32, device=q.device)
    rtp_sparse_attn_prefill(q, k, v, q16, k16, sel["thr"], sel["jtie"], kv_role, scale=scale,
                            k16_per_kv_head=k16_per_kv_head, o=o, lse=lse, stream=stream)
    rtp_local_attn(q, k, v, kv_role, window=window, n_sink=n_sink, scale=scale, o=o, lse=lse,
                   stream=stream)
    return dict(o=o, lse=lse, q16=q16, k16=k16, sel=sel)


def rtp_layer_decode(q, k_new, k_cache, v_cache, k16_cache, Wq16, Wk16, kv_role, *, pos, p,
                     window, n_sink, scale=None, k16_per_kv_head=0, stream=None):
    """One decode token at position `pos` (the caches already hold its k/v row;
    its k16 row is written here).  Returns dict(o, lse, q16, sel)."""
    H = q.shape[2]
    k16_row = k16_cache[:, pos:pos + 1]
    q16, _ = rtp_index_scores(q, k_new, Wq16, Wk16, kv_role, k16=k16_row,
                              k16_per_kv_head=k16_per_kv_head, stream=stream)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[0], H, 1, dtype=torch.float32, device=q.device)
    kc, vc = k_cache[:, :pos + 1], v_cache[:, :pos + 1]
    _, _, sel = rtp_sparse_attn_decode(q, kc, vc, q16, k16_cache[:, :pos + 1], kv_role, p,
                                       scale=scale, q_pos0=pos, k16_per_kv_head=k16_per_kv_head,
                                       o=o, lse=lse, stream=stream)
    rtp_local_attn(q, kc, vc, kv_role, window=window, n_sink=n_sink, scale=scale, q_pos0=pos,
                   o=o, lse=lse, stream=stream)
    return dict(o=o, lse=lse, q16=q16, sel=sel)
