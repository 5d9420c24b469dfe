"""Seeded synthetic inputs for decode and prefill (shared by tests, bench and smoke).

This module only draws inputs: random tensors, planted heavy-hitter keys, page
tables. It holds none of the method's arithmetic (no scoring, selection or
attention), so both the CUDA path and the fp64 oracle can consume its output.

Recipe (the pages give workload shapes in prose only; where they leave a detail
open, the plainest reading is taken and stated here):
* Q, K, V ~ N(0, 1), stored bf16.
* One shared index projection W_idx [d, r] ~ N(0, 1/d); index keys
  k_idx = bf16(K_bf16 @ W_idx), index queries q_idx = bf16(Q_bf16 @ W_idx).
* Heavy hitters are planted in K only: K[pos] = bf16(amp * q_hat + N(0, 0.1^2)),
  q_hat the unit vector of the mean query of the kv group (decode: the group's G
  query heads; prefill: the group's heads over all positions). Positions are
  drawn without replacement by one of: ``uniform``, ``zipf`` (block index with
  P(j) ~ (j+1)^-a, offset uniform inside the block), ``runs`` (runs of
  consecutive tokens at non-overlapping random starts).
* Paged caches use a pool [num_pages, Hkv, 64, d] with num_pages = B * nb and a
  page table that is a seeded random permutation of the pages, reshaped [B, nb].
  Index keys stay contiguous [B, Hkv, T, r] (a separate selector cache).
* ``diffuse_odd``: queries of odd sequences are multiplied by 0.5 before the
  bf16 rounding (q_idx follows), which spreads their top-p sets.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import numpy as np
import torch

BLOCK = 64


@dataclass(frozen=True)
class Workload:
    name: str
    phase: str                      # "decode" | "prefill"
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int
    r: int = 16
    paged: bool = False
    n_sink: int = 1
    n_local: int = 2
    p: float = 0.9
    k_max: int = 16
    k_min: int = 0
    hh_count: int = 4               # planted heavy hitters per (sequence, kv head)
    hh_kind: str = "uniform"        # uniform | zipf | runs
    hh_param: float = 0.0           # zipf exponent, or run length
    amp: float = 4.0
    diffuse_odd: bool = False
    seed: int = 0
    seq_lens: Optional[tuple] = None  # per-sequence lengths (<= T); None = all T
    head_w: Optional[tuple] = None    # per-query-head weights; None = 1/G

    @property
    def G(self):
        return self.Hq // self.Hkv

    @property
    def nb(self):
        return (self.T + BLOCK - 1) // BLOCK

    def with_(self, **kw):
        return replace(self, **kw)


# The five workloads of the long-context decode / prefill study, named by shape.
WORKLOADS = {
    "decode_tiny_b1_h8_t4k": Workload(
        "decode_tiny_b1_h8_t4k", "decode", B=1, Hq=8, Hkv=2, d=64, T=4096, paged=False,
        n_sink=1, n_local=2, p=0.9, k_max=16, hh_count=4, hh_kind="uniform", amp=4.0),
    "decode_b8_h32_t32k_paged": Workload(
        "decode_b8_h32_t32k_paged", "decode", B=8, Hq=32, Hkv=8, d=128, T=32768, paged=True,
        n_sink=1, n_local=4, p=0.9, k_max=64, hh_count=32, hh_kind="uniform", amp=3.0),
    "decode_b32_h32_t128k_paged": Workload(
        "decode_b32_h32_t128k_paged", "decode", B=32, Hq=32, Hkv=8, d=128, T=131072,
        paged=True, n_sink=1, n_local=8, p=0.95, k_max=256, hh_count=64, hh_kind="zipf",
        hh_param=1.1, amp=2.5, diffuse_odd=True),
    "decode_b1_h64_t1m": Workload(
        "decode_b1_h64_t1m", "decode", B=1, Hq=64, Hkv=8, d=128, T=1048576, paged=False,
        n_sink=2, n_local=8, p=0.9, k_max=512, hh_count=128, hh_kind="runs", hh_param=8,
        amp=3.0),
    "prefill_b1_h32_t64k": Workload(
        "prefill_b1_h32_t64k", "prefill", B=1, Hq=32, Hkv=8, d=128, T=65536, paged=False,
        n_sink=1, n_local=2, p=1.0, k_max=64, hh_count=256, hh_kind="uniform", amp=3.0),
}


def _positions(rng: np.random.Generator, kind: str, count: int, T_b: int, param: float):
    """Distinct heavy-hitter token positions in [0, T_b)."""
    count = min(count, T_b)
    if kind == "uniform":
        return np.sort(rng.choice(T_b, size=count, replace=False))
    if kind == "zipf":
        nb = (T_b + BLOCK - 1) // BLOCK
        pj = (np.arange(nb) + 1.0) ** (-param)
        pj /= pj.sum()
        chosen = set()
        while len(chosen) < count:
            j = int(rng.choice(nb, p=pj))
            t = j * BLOCK + int(rng.integers(0, min(BLOCK, T_b - j * BLOCK)))
            chosen.add(t)               # a duplicate is simply redrawn
        return np.array(sorted(chosen))
    if kind == "runs":
        run = int(param)
        n_runs = max(1, count // run)
        starts = []
        while len(starts) < n_runs:
            s = int(rng.integers(0, max(1, T_b - run)))
            if all(abs(s - o) >= run for o in starts):
                starts.append(s)
        pos = np.concatenate([np.arange(s, min(s + run, T_b)) for s in sorted(starts)])
        return pos
    raise ValueError(kind)


def _normal_(t: torch.Tensor, gen: torch.Generator, chunk_rows: int = 1 << 22):
    """Fill a bf16 tensor with N(0,1) draws chunk by chunk (no large fp32 temporaries)."""
    flat = t.view(-1, t.shape[-1])
    for s in range(0, flat.shape[0], chunk_rows):
        flat[s:s + chunk_rows].normal_(generator=gen)
    return t


def _project(x: torch.Tensor, W: torch.Tensor, chunk_rows: int = 1 << 22) -> torch.Tensor:
    """bf16(x_bf16 @ W) row-chunked; x [..., d] -> [..., r]."""
    flat = x.reshape(-1, x.shape[-1])
    out = torch.empty(flat.shape[0], W.shape[1], dtype=torch.bfloat16, device=x.device)
    for s in range(0, flat.shape[0], chunk_rows):
        out[s:s + chunk_rows] = (flat[s:s + chunk_rows].float() @ W).to(torch.bfloat16)
    return out.view(*x.shape[:-1], W.shape[1])


def seq_lens_of(w: Workload):
    return list(w.seq_lens) if w.seq_lens is not None else [w.T] * w.B


def make_decode_inputs(w: Workload, device="cpu") -> dict:
    """Decode-step inputs. Returns a dict of tensors on ``device``:
    q [B,Hq,d], q_idx [B,Hq,r], k_idx [B,Hkv,T,r] (bf16); K, V contiguous
    [B,Hkv,T,d] or pooled [P,Hkv,64,d] (bf16); page_table [B,nb] int32 or None;
    seq_lens [B] int32; head_w [Hq] float32."""
    assert w.phase == "decode"
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(w.seed)
    B, Hq, Hkv, d, T, r, G, nb = w.B, w.Hq, w.Hkv, w.d, w.T, w.r, w.G, w.nb
    lens = seq_lens_of(w)

    Q = torch.randn(B, Hq, d, generator=gen, device=dev)
    if w.diffuse_odd:
        Q[1::2] *= 0.5
    q = Q.to(torch.bfloat16)
    W = torch.randn(d, r, generator=gen, device=dev) / math.sqrt(d)

    if w.paged:
        P = B * nb
        shape = (P, Hkv, BLOCK, d)
    else:
        shape = (B, Hkv, T, d)
    K = _normal_(torch.empty(shape, dtype=torch.bfloat16, device=dev), gen)
    V = _normal_(torch.empty(shape, dtype=torch.bfloat16, device=dev), gen)

    rng = np.random.default_rng(w.seed + 1000003)
    page_table = None
    if w.paged:
        page_table_np = rng.permutation(B * nb).reshape(B, nb).astype(np.int32)
        page_table = torch.from_numpy(page_table_np).to(dev)

    # heavy hitters: K = amp * q_hat + N(0, 0.1^2), at positions per (b, g)
    qf = q.float()
    for b in range(B):
        for g in range(Hkv):
            pos = _positions(rng, w.hh_kind, w.hh_count, lens[b], w.hh_param)
            if pos.size == 0:
                continue
            mean = qf[b, g * G:(g + 1) * G].mean(0)
            qhat = mean / mean.norm()
            noise = torch.randn(len(pos), d, generator=gen, device=dev) * 0.1
            rows = (w.amp * qhat[None, :] + noise).to(torch.bfloat16)
            pos_t = torch.from_numpy(pos).to(dev)
            if w.paged:
                K[page_table[b, pos_t // BLOCK].long(), g, pos_t % BLOCK] = rows
            else:
                K[b, g, pos_t] = rows

    q_idx = _project(q, W)
    if w.paged:
        idx_pool = _project(K, W)                                     # [P,Hkv,64,r]
        k_idx = idx_pool[page_table.long()]                           # [B,nb,Hkv,64,r]
        k_idx = k_idx.permute(0, 2, 1, 3, 4).reshape(B, Hkv, nb * BLOCK, r)[:, :, :T].contiguous()
        del idx_pool
    else:
        k_idx = _project(K, W)
    head_w = (torch.tensor(w.head_w, dtype=torch.float32, device=dev) if w.head_w is not None
              else torch.full((Hq,), 1.0 / G, dtype=torch.float32, device=dev))
    return dict(q=q, q_idx=q_idx, k_idx=k_idx, K=K, V=V, page_table=page_table,
                seq_lens=torch.tensor(lens, dtype=torch.int32, device=dev), head_w=head_w)


def make_prefill_inputs(w: Workload, device="cpu") -> dict:
    """Prefill inputs: Q [B,Hq,T,d], q_idx [B,Hq,T,r], K, V [B,Hkv,T,d],
    k_idx [B,Hkv,T,r] (all bf16, contiguous); head_w [Hq] float32."""
    assert w.phase == "prefill"
    dev = torch.device(device)
    gen = torch.Generator(device=dev).manual_seed(w.seed)
    B, Hq, Hkv, d, T, r, G = w.B, w.Hq, w.Hkv, w.d, w.T, w.r, w.G
    Q = _normal_(torch.empty(B, Hq, T, d, dtype=torch.bfloat16, device=dev), gen)
    W = torch.randn(d, r, generator=gen, device=dev) / math.sqrt(d)
    K = _normal_(torch.empty(B, Hkv, T, d, dtype=torch.bfloat16, device=dev), gen)
    V = _normal_(torch.empty(B, Hkv, T, d, dtype=torch.bfloat16, device=dev), gen)
    rng = np.random.default_rng(w.seed + 1000003)
    for b in range(B):
        for g in range(Hkv):
            pos = _positions(rng, w.hh_kind, w.hh_count, T, w.hh_param)
            mean = Q[b, g * G:(g + 1) * G].float().mean(dim=(0, 1))
            qhat = mean / mean.norm()
            noise = torch.randn(len(pos), d, generator=gen, device=dev) * 0.1
            K[b, g, torch.from_numpy(pos).to(dev)] = (w.amp * qhat[None, :] + noise).to(torch.bfloat16)
    q_idx = _project(Q, W)
    k_idx = _project(K, W)
    head_w = (torch.tensor(w.head_w, dtype=torch.float32, device=dev) if w.head_w is not None
              else torch.full((Hq,), 1.0 / G, dtype=torch.float32, device=dev))
    return dict(q=Q, q_idx=q_idx, k_idx=k_idx, K=K, V=V, head_w=head_w)


def logical_kv(inputs: dict, w: Workload, b: int, g: int, which: str = "K") -> torch.Tensor:
    """[T, d] logical-order rows of K or V for (b, g), following the page table."""
    X = inputs[which]
    if inputs.get("page_table") is None:
        return X[b, g]
    pt = inputs["page_table"][b].long()
    return X[pt, g].reshape(-1, X.shape[-1])[:w.T]
