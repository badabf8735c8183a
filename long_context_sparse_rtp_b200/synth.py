"""Seeded synthetic inputs shaped like the paper's Qwen3-30B-A3B-class layer.

This module only draws inputs; it holds none of the method's arithmetic (no
projection, score, selection or attention).  The tests, the benchmark and the
oracle-side checks all draw their inputs here.

Recipe (common to every workload):

* q, k, v ~ N(0, 1) drawn as fp32 pre-RoPE vectors, in fixed chunks of
  ``CHUNK`` positions from one torch generator seeded with the workload seed;
* optional per-query temperature tau ~ logU[0.5, 4]: q <- q / tau;
* RoPE with base 1e6 on q and k, rotating the interleaved pairs (2c, 2c+1) by
  pos * base^(-2c/128) (the block-diagonal R(m) of the summary page's section
  on RoPE-induced compressibility, Eq. 1), angles in fp64;
* W_q16, W_k16 ~ N(0, 1/128), one pair per retrieval query head;
* planted needles ("+4 sigma alignment"): for retrieval head h let
  M_h = W_q16[h] W_k16[h]^T, u_h the unit top eigenvector of (M_h + M_h^T)/2
  with eigenvalue lambda_h, sigma_h = ||M_h||_F (the score spread of unit
  Gaussian q, k).  A needle adds a_h u_h to a post-RoPE key and to the
  post-RoPE queries it targets, with a_h^2 lambda_h = 4 sigma_h, which raises
  that pair's indexer score by about 4 sigma;
* everything is rounded to bf16 once at the end.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np
import torch

D = 128
R = 16
ROPE_BASE = 1.0e6
CHUNK = 8192


@dataclass(frozen=True)
class Workload:
    name: str
    phase: str              # "prefill" or "decode"
    B: int
    L: int                  # prefill: sequence length; decode: cache length incl. the new token
    H: int
    Hkv: int
    ret_kv: tuple           # kv heads whose query heads are retrieval heads
    window: int
    n_sink: int
    p: float
    needles: str            # "residue8" | "uniform64" | "chain4" | "group64" | "none"
    temperature: bool
    seed: int
    p_sweep: tuple = ()

    @property
    def G(self) -> int:
        return self.H // self.Hkv

    @property
    def H_ret(self) -> int:
        return len(self.ret_kv) * self.G

    def kv_role(self) -> np.ndarray:
        role = np.zeros(self.Hkv, np.uint8)
        role[list(self.ret_kv)] = 1
        return role

    def retrieval_q_heads(self) -> list:
        return [g * self.G + j for g in sorted(self.ret_kv) for j in range(self.G)]

    def local_q_heads(self) -> list:
        ret = set(self.retrieval_q_heads())
        return [h for h in range(self.H) if h not in ret]

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # 2K causal prefill, GQA 4, kv0 retrieval, kv1 local (256 + 4 sinks), p = 0.9
    "prefill_2k": Workload("prefill_2k", "prefill", 1, 2048, 8, 2, (0,), 256, 4,
                           0.9, "residue8", False, 0),
    # one decode token against a 128K cache, batch 8, 1 retrieval + 3 local kv heads
    "decode_128k_b8": Workload("decode_128k_b8", "decode", 8, 131072, 32, 4, (0,),
                               4096, 4, 0.95, "uniform64", False, 2),
    # 32K causal prefill, 2 of 4 kv heads retrieval, per-query temperature, p swept
    "prefill_32k": Workload("prefill_32k", "prefill", 1, 32768, 32, 4, (0, 1), 2048,
                            4, 0.9, "none", True, 3, (0.8, 0.9, 0.95, 0.99)),
    # 128K causal prefill, multi-hop (4-key chains per 4096-row query group)
    "prefill_128k": Workload("prefill_128k", "prefill", 1, 131072, 32, 4, (0,), 4096,
                             4, 0.95, "chain4", False, 4),
    # 1M causal prefill, needles per 4096-row query group
    "prefill_1m": Workload("prefill_1m", "prefill", 1, 1048576, 32, 4, (0,), 4096,
                           4, 0.95, "group64", False, 5),
}


def _rope_(x: torch.Tensor, pos0) -> None:
    """In-place RoPE on x [n, heads, 128] (fp32) for positions pos0 .. pos0+n-1,
    or for the n positions of a 1-D tensor `pos0`."""
    n = x.shape[0]
    c = torch.arange(D // 2, device=x.device, dtype=torch.float64)
    theta = ROPE_BASE ** (-2.0 * c / D)
    if isinstance(pos0, torch.Tensor):
        pos = pos0.to(device=x.device, dtype=torch.float64)
    else:
        pos = torch.arange(pos0, pos0 + n, device=x.device, dtype=torch.float64)
    ang = pos[:, None] * theta[None, :]
    cos = torch.cos(ang).to(torch.float32)[:, None, :]
    sin = torch.sin(ang).to(torch.float32)[:, None, :]
    a = x[..., 0::2].clone()
    b = x[..., 1::2].clone()
    x[..., 0::2] = a * cos - b * sin
    x[..., 1::2] = a * sin + b * cos


def rope(x: torch.Tensor, pos0: int) -> torch.Tensor:
    """Out-of-place RoPE on [n, heads, 128] (for tests of the generator)."""
    y = x.to(torch.float32).clone()
    _rope_(y, pos0)
    return y


def _needle_dirs(Wq: np.ndarray, Wk: np.ndarray):
    """Per retrieval head: unit top eigenvector u, and the amplitude a."""
    dirs, amps = [], []
    for h in range(Wq.shape[0]):
        M = Wq[h] @ Wk[h].T
        Ms = 0.5 * (M + M.T)
        lam, vec = np.linalg.eigh(Ms)
        u = vec[:, -1]
        sigma = float(np.linalg.norm(M))
        a = math.sqrt(4.0 * sigma / float(lam[-1]))
        dirs.append(u)
        amps.append(a)
    return np.stack(dirs), np.array(amps)


def make_inputs(w: Workload, device="cpu", L: int | None = None, B: int | None = None,
                indexer_input: str = "post"):
    """Draw one workload's tensors.

    Returns a dict: q [B,Lq,H,128], k/v [B,Lk,Hkv,128], Wq16 [H_ret,128,16],
    Wk16 [H_ret,128,16] (all bf16 on ``device``), kv_role (numpy uint8 [Hkv]),
    and the ints Lq, Lk, q_pos0.

    indexer_input="pre" also returns q_idx [B,Lq,H,128] and k_idx
    [B,Lk,Hkv,128]: the same draws before RoPE (bf16), for an indexer that
    projects pre-RoPE vectors as the summary's projection section describes.
    The needles are then planted in those pre-RoPE vectors, and the planted rows
    of q, k are the RoPE of the planted pre-RoPE rows, so the indexer sees the
    +4 sigma uplift exactly and attention sees its rotated form.
    """
    if indexer_input not in ("post", "pre"):
        raise ValueError("indexer_input must be 'post' or 'pre'")
    pre = indexer_input == "pre"
    L = w.L if L is None else L
    B = w.B if B is None else B
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed)
    if w.phase == "decode":
        Lq, Lk, q_pos0 = 1, L, L - 1
    else:
        Lq, Lk, q_pos0 = L, L, 0
    H, Hkv, H_ret = w.H, w.Hkv, w.H_ret

    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=dev, dtype=torch.float32)

    Wq = randn(H_ret, D, R) / math.sqrt(D)
    Wk = randn(H_ret, D, R) / math.sqrt(D)
    Wq = Wq.to(torch.bfloat16)
    Wk = Wk.to(torch.bfloat16)

    q = torch.empty(B, Lq, H, D, dtype=torch.bfloat16, device=dev)
    k = torch.empty(B, Lk, Hkv, D, dtype=torch.bfloat16, device=dev)
    v = torch.empty(B, Lk, Hkv, D, dtype=torch.bfloat16, device=dev)
    q_idx = torch.empty_like(q) if pre else None
    k_idx = torch.empty_like(k) if pre else None

    rng = np.random.default_rng(w.seed + 1000)
    Wq_np = Wq.float().cpu().numpy().astype(np.float64)
    Wk_np = Wk.float().cpu().numpy().astype(np.float64)
    u, amp = _needle_dirs(Wq_np, Wk_np) if w.needles != "none" else (None, None)
    ret_heads = w.retrieval_q_heads()
    G = w.G
    # needle plan: lists of (b, key position, retrieval slot) and (b, q row, slot)
    key_adds, q_adds = [], []
    if w.needles == "residue8":
        for slot in range(H_ret):
            cnt = min(8, max(Lk - 4, 0))
            pos = rng.choice(np.arange(4, Lk), size=cnt, replace=False) if cnt else []
            for gidx, n in enumerate(pos):
                key_adds.append((0, int(n), slot))
                rows = np.arange(Lq)
                rows = rows[(rows % 8 == gidx) & (rows + q_pos0 > n)]
                q_adds.append((0, rows, slot))
    elif w.needles == "uniform64":
        for b in range(B):
            for slot in range(H_ret):
                cnt = min(int(rng.integers(0, 65)), max(Lk - 1, 0))
                pos = rng.choice(Lk - 1, size=cnt, replace=False) if cnt else []
                for n in pos:
                    key_adds.append((b, int(n), slot))
                if cnt:
                    q_adds.append((b, np.arange(Lq), slot))
    elif w.needles in ("chain4", "group64"):
        gsz = 4096
        for gi, start in enumerate(range(0, Lq, gsz)):
            slot = gi % H_ret
            rows = np.arange(start, min(start + gsz, Lq))
            if start + q_pos0 < 1:
                continue
            if w.needles == "group64":
                cnt = int(rng.integers(0, 65))
                pos = rng.choice(start + q_pos0, size=min(cnt, start + q_pos0), replace=False)
                for n in pos:
                    key_adds.append((0, int(n), slot))
                if cnt:
                    q_adds.append((0, rows, slot))
            else:
                hi = start + q_pos0
                prev_rows = rows
                for _ in range(4):
                    if hi < 1:
                        break
                    n = int(rng.integers(0, hi))
                    key_adds.append((0, n, slot))
                    q_adds.append((0, prev_rows, slot))
                    prev_rows = np.array([n - q_pos0]) if n - q_pos0 >= 0 else np.array([], np.int64)
                    hi = n

    for b in range(B):
        for c0 in range(0, Lq, CHUNK):
            n = min(CHUNK, Lq - c0)
            x = randn(n, H, D)
            if w.temperature:
                tau = torch.exp(torch.empty(n, H, 1, device=dev).uniform_(
                    math.log(0.5), math.log(4.0), generator=gen))
                x = x / tau
            if pre:
                q_idx[b, c0:c0 + n] = x.to(torch.bfloat16)
            _rope_(x, q_pos0 + c0)
            q[b, c0:c0 + n] = x.to(torch.bfloat16)
        for c0 in range(0, Lk, CHUNK):
            n = min(CHUNK, Lk - c0)
            x = randn(n, Hkv, D)
            if pre:
                k_idx[b, c0:c0 + n] = x.to(torch.bfloat16)
            _rope_(x, c0)
            k[b, c0:c0 + n] = x.to(torch.bfloat16)
            v[b, c0:c0 + n] = randn(n, Hkv, D).to(torch.bfloat16)

    if key_adds or q_adds:
        ut = torch.tensor(u * amp[:, None], dtype=torch.float32, device=dev)
        for b, n, slot in key_adds:
            g = ret_heads[slot] // G
            if pre:
                k_idx[b, n, g] = (k_idx[b, n, g].float() + ut[slot]).to(torch.bfloat16)
                y = k_idx[b, n:n + 1, g:g + 1].float()
                _rope_(y, n)
                k[b, n, g] = y[0, 0].to(torch.bfloat16)
            else:
                k[b, n, g] = (k[b, n, g].float() + ut[slot]).to(torch.bfloat16)
        for b, rows, slot in q_adds:
            if len(rows) == 0:
                continue
            h = ret_heads[slot]
            ridx = torch.as_tensor(np.asarray(rows), device=dev, dtype=torch.long)
            if pre:
                q_idx[b, ridx, h] = (q_idx[b, ridx, h].float() + ut[slot]).to(torch.bfloat16)
                y = q_idx[b, ridx, h].float()[:, None, :]
                _rope_(y, ridx + q_pos0)
                q[b, ridx, h] = y[:, 0].to(torch.bfloat16)
            else:
                q[b, ridx, h] = (q[b, ridx, h].float() + ut[slot]).to(torch.bfloat16)

    out = dict(q=q, k=k, v=v, Wq16=Wq, Wk16=Wk, kv_role=w.kv_role(),
               Lq=Lq, Lk=Lk, q_pos0=q_pos0)
    if pre:
        out.update(q_idx=q_idx, k_idx=k_idx)
    return out


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
