"""Plain fp64 CPU oracle for dynamic block-sparse attention (decode and prefill).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The product path (``block_sparse_long_06_b200``) never imports or calls
it, and this module imports nothing from the product.

Every function takes already-widened float64 numpy arrays (bf16 inputs are
widened exactly by the caller) and computes in float64 with plain numpy. A
library matmul (``@``), ``np.maximum``, ``np.exp`` and a lexicographic sort are
the only primitives; there is no blocking, fusion or reordering beyond what the
definitions state, so each function can be read against its source.

Sources (gist.science technical summaries; cited by page title and section):

* [SpotAttention §1]  SpotAttention, Methodology §1 "selector architecture":
  the weighted-ReLU score s[q,t] = sum_h w_h ReLU(q^I_h . k^I_{h,t}).
* [SpotAttention §3]  SpotAttention, Methodology §3 "dual top-p rule":
  reserved sink prefix and recency suffix are always kept; nucleus (top-p)
  selection runs on the distribution of the remaining (residual) blocks and
  stops once the cumulative mass reaches p; a floor K_min.
* [RTPurbo §2]        Full Attention Strikes Back (RTPurbo), Methodology §2:
  a low-dimensional (r = 16) index projection of queries and keys.
* [RTPurbo §3]        RTPurbo, Methodology §3: dynamic top-p, accumulate
  attention mass until the threshold p is reached.
* [HGA mechanism §2/§4] Hierarchical Global Attention (HGA), Central mechanism
  §2 (current chunk, sink chunks and recent local chunks always visible) and
  §4 (exact token-level softmax over the routed set, no summary values).
* [PBS §1]            Sparser Block-Sparse Attention via Token Permutation
  (PBS-Attn), Methodology §1: attention output is invariant to permuting
  key/value pairs (used by the tests as an invariant).

Readings where the pages leave a step open:

* block aggregate of token scores = max over the block's tokens (and, in
  prefill, over the query block's tokens too);
* w_h = 1/G when no head weights are given; idx_scale (1/sqrt(r)) multiplies
  the head sum;
* top-p acts on the softmax of the block scores over the candidate (residual)
  set only; "reaches p" = smallest prefix whose cumulative mass is >= p, and
  the prefix has at least one block; p <= 0 keeps no dynamic block; p >= 1
  keeps every candidate (before the K_max cap);
* p is compared as the float32 value the device sees: p_hat = float(float32(p));
* K_max caps the dynamic set only; K_min (<= K_max) is a floor on it;
* equal scores order by lower block index first;
* sink and local sets that overlap are unioned; a partial last block is kept
  in the local window, and tokens at t >= T are never visible;
* the decode query sees all T cached tokens (the current one included);
* attention scale 1/sqrt(d) unless given; log-sum-exp in natural log.

Parity status: every function here is pinned by ``tests/test_oracle.py``
(hand-worked cases, library routines for special cases, invariants).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

BLOCK = 64


# --------------------------------------------------------------------------
# helpers that are plain data handling (no arithmetic of the method)
# --------------------------------------------------------------------------
def num_blocks(T: int, block: int = BLOCK) -> int:
    """Number of 64-token blocks covering T tokens (last one may be partial)."""
    return (T + block - 1) // block


def p_hat(p: float) -> float:
    """The top-p threshold as the float32 value the device compares against."""
    return float(np.float32(p))


def gather_tokens(cache: np.ndarray, page_table, b: int, g: int, token_ids, block: int = BLOCK):
    """Token rows of sequence b, kv head g, from a contiguous [B,Hkv,T,w] cache
    (page_table None) or a paged [P,Hkv,block,w] pool with page_table[b, j]."""
    token_ids = np.asarray(token_ids, dtype=np.int64)
    if page_table is None:
        return cache[b, g, token_ids]
    pages = np.asarray(page_table)[b, token_ids // block]
    return cache[pages, g, token_ids % block]


# --------------------------------------------------------------------------
# scoring  [SpotAttention §1], [RTPurbo §2]
# --------------------------------------------------------------------------
def token_scores(q_idx_heads: np.ndarray, k_idx_tokens: np.ndarray, head_w: np.ndarray,
                 idx_scale: float) -> np.ndarray:
    """u[..., t] = idx_scale * sum_h w_h * ReLU(q_idx[h] . k_idx[t]).

    q_idx_heads: [G, r] (one query) or [G, n_q, r] (several query positions).
    k_idx_tokens: [n_k, r].  head_w: [G].
    Returns [n_k] or [n_q, n_k].
    """
    dots = q_idx_heads @ k_idx_tokens.T                  # [G, n_k] or [G, n_q, n_k]
    return idx_scale * np.tensordot(head_w, np.maximum(dots, 0.0), axes=(0, 0))


def decode_block_scores(q_idx_g: np.ndarray, k_idx_g: np.ndarray, T: int, head_w: np.ndarray,
                        idx_scale: float, block: int = BLOCK) -> np.ndarray:
    """S_j = max over tokens t of block j (t < T) of u_t, for one (sequence, kv head).

    q_idx_g: [G, r] index queries of the group's heads; k_idx_g: [>=T, r] logical
    index keys. Returns S of length ceil(T/64).
    """
    u = token_scores(q_idx_g, k_idx_g[:T], head_w, idx_scale)
    nb = num_blocks(T, block)
    S = np.empty(nb, dtype=np.float64)
    for j in range(nb):
        S[j] = u[j * block:min((j + 1) * block, T)].max()
    return S


def prefill_block_scores(q_idx_g: np.ndarray, k_idx_g: np.ndarray, T: int, head_w: np.ndarray,
                         idx_scale: float, rows=None, block: int = BLOCK) -> dict:
    """S[i, j] = max over (tq in query block i, tk in key block j) of
    idx_scale * sum_h w_h ReLU(q_idx[h, tq] . k_idx[tk]), for key blocks j < i.

    q_idx_g: [G, >=T, r]; k_idx_g: [>=T, r]. Every pair (tq, tk) with j < i is
    causal, so no mask enters the score. Returns {i: S_i[0:i]} for the query
    blocks in ``rows`` (all blocks when None).
    """
    nqb = num_blocks(T, block)
    rows = range(nqb) if rows is None else rows
    out = {}
    for i in rows:
        q0, q1 = i * block, min((i + 1) * block, T)
        if i == 0:
            out[i] = np.zeros(0)
            continue
        u = token_scores(q_idx_g[:, q0:q1, :], k_idx_g[:i * block], head_w, idx_scale)  # [nq, i*64]
        S_i = np.empty(i, dtype=np.float64)
        for j in range(i):
            S_i[j] = u[:, j * block:(j + 1) * block].max()
        out[i] = S_i
    return out


# --------------------------------------------------------------------------
# selection  [SpotAttention §3], [RTPurbo §3], [HGA mechanism §2]
# --------------------------------------------------------------------------
@dataclass
class Selection:
    kept: list                     # ascending block ids (reserved ∪ dynamic)
    reserved: list                 # ascending reserved ids
    candidates: list               # ascending candidate ids
    order: list = field(default_factory=list)      # candidates ordered by (S desc, id asc)
    mass: np.ndarray = None        # mass of order[i] (softmax over candidates)
    cum: np.ndarray = None         # inclusive cumulative mass along order
    k_p: int = 0                   # top-p prefix length before the caps
    k: int = 0                     # dynamic blocks kept
    cap: int = 0                   # min(K_max, |C|)


def reserved_decode(nb: int, n_sink: int, n_local: int) -> list:
    """Sink prefix [0, n_sink) and recency suffix [nb - n_local, nb), clipped and unioned."""
    return sorted(set(range(min(n_sink, nb))) | set(range(max(0, nb - n_local), nb)))


def reserved_prefill(i: int, n_sink: int, n_local: int) -> list:
    """Current (diagonal) block i, sink blocks [0, n_sink) that are causal (<= i),
    and the n_local blocks just before i."""
    return sorted({i} | set(range(min(n_sink, i + 1))) | set(range(max(0, i - n_local), i)))


def select_dynamic(S: np.ndarray, candidates: list, p: float, k_max: int, k_min: int = 0):
    """Dual top-p on the residual candidates, capped at K_max, floored at K_min.

    Order the candidates by score descending, ties to the lower block id. The mass
    of a candidate is its softmax weight over the candidates only. k_p is the
    smallest prefix (at least one block) whose cumulative mass reaches p_hat; with
    p >= 1 every candidate; with p <= 0 none. Then k = max(min(k_p, K_max),
    min(K_min, |C|)).
    """
    C = list(candidates)
    n = len(C)
    if n == 0:
        return [], np.zeros(0), np.zeros(0), 0, 0, 0
    s = np.array([S[j] for j in C], dtype=np.float64)
    order_idx = np.lexsort((np.array(C), -s))            # primary -s (desc), then id asc
    order = [C[t] for t in order_idx]
    M = s.max()
    w = np.exp(s - M)
    mass = w[order_idx] / w.sum()
    cum = np.cumsum(mass)
    ph = p_hat(p)
    if ph <= 0.0:
        k_p = 0
    elif ph >= 1.0:
        k_p = n
    else:
        reached = np.nonzero(cum >= ph)[0]
        k_p = int(reached[0]) + 1 if reached.size else n
    cap = min(k_max, n)
    k = max(min(k_p, cap), min(k_min, n))
    return order, mass, cum, k_p, k, cap


def select_decode(S: np.ndarray, n_sink: int, n_local: int, p: float, k_max: int,
                  k_min: int = 0) -> Selection:
    """Kept blocks for one (sequence, kv head) decode row with nb = len(S) blocks."""
    nb = len(S)
    R = reserved_decode(nb, n_sink, n_local)
    Rs = set(R)
    C = [j for j in range(nb) if j not in Rs]
    order, mass, cum, k_p, k, cap = select_dynamic(S, C, p, k_max, k_min)
    kept = sorted(Rs | set(order[:k]))
    return Selection(kept, R, C, order, mass, cum, k_p, k, cap)


def select_prefill(S_i: np.ndarray, i: int, n_sink: int, n_local: int, p: float, k_max: int,
                   k_min: int = 0) -> Selection:
    """Kept key blocks for query block i; S_i holds scores of key blocks [0, i)."""
    R = reserved_prefill(i, n_sink, n_local)
    Rs = set(R)
    C = [j for j in range(i) if j not in Rs]
    order, mass, cum, k_p, k, cap = select_dynamic(S_i, C, p, k_max, k_min)
    kept = sorted(Rs | set(order[:k]))
    return Selection(kept, R, C, order, mass, cum, k_p, k, cap)


# --------------------------------------------------------------------------
# exact attention over the kept tokens  [HGA mechanism §4]
# --------------------------------------------------------------------------
def attend(q_heads: np.ndarray, K_tok: np.ndarray, V_tok: np.ndarray, scale: float):
    """Softmax attention of each query row over the given token set.

    q_heads: [G, d]; K_tok, V_tok: [n, d]. Returns o [G, d], lse [G] (natural log).
    With n = 0 the output is 0 and the lse is -inf.
    """
    G, d = q_heads.shape
    if K_tok.shape[0] == 0:
        return np.zeros((G, d)), np.full(G, -np.inf)
    s = (q_heads @ K_tok.T) * scale                       # [G, n]
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    o = (e @ V_tok) / z
    lse = (m + np.log(z))[:, 0]
    return o, lse


def kept_token_ids(kept_blocks, T: int, block: int = BLOCK) -> np.ndarray:
    """Token ids of the kept blocks that exist (t < T), in block order."""
    ids = [np.arange(j * block, min((j + 1) * block, T)) for j in kept_blocks]
    return np.concatenate(ids) if ids else np.zeros(0, dtype=np.int64)


def attend_prefill_block(q_heads_blk: np.ndarray, q_pos: np.ndarray, K_tok: np.ndarray,
                         V_tok: np.ndarray, k_pos: np.ndarray, scale: float):
    """Causal softmax attention for the query rows of one query block.

    q_heads_blk: [G, n_q, d] at positions q_pos [n_q]; keys/values at k_pos [n].
    A key is visible to a query when k_pos <= q_pos. Returns o [G, n_q, d],
    lse [G, n_q].
    """
    s = np.einsum("gqd,kd->gqk", q_heads_blk, K_tok) * scale
    visible = k_pos[None, None, :] <= q_pos[None, :, None]
    s = np.where(visible, s, -np.inf)
    m = s.max(axis=2, keepdims=True)
    e = np.where(visible, np.exp(s - m), 0.0)
    z = e.sum(axis=2, keepdims=True)
    o = np.einsum("gqk,kd->gqd", e, V_tok) / z
    lse = (m + np.log(z))[..., 0]
    return o, lse


# --------------------------------------------------------------------------
# whole rows (score -> select -> attend), as the tests consume them
# --------------------------------------------------------------------------
def decode_row(q_g, q_idx_g, k_idx_g, K_g, V_g, T, head_w, idx_scale, attn_scale,
               n_sink, n_local, p, k_max, k_min=0, kept_override=None):
    """One decode row (sequence b, kv head g).

    q_g [G,d], q_idx_g [G,r]; k_idx_g [>=T,r], K_g/V_g [>=T,d] in logical token
    order. ``kept_override`` replaces the selection (used to re-run attention on
    a device-selected set that the tie rule accepted).
    Returns dict(S, sel, o, lse).
    """
    S = decode_block_scores(q_idx_g, k_idx_g, T, head_w, idx_scale)
    sel = select_decode(S, n_sink, n_local, p, k_max, k_min)
    kept = sel.kept if kept_override is None else list(kept_override)
    ids = kept_token_ids(kept, T)
    o, lse = attend(q_g, K_g[ids], V_g[ids], attn_scale)
    return {"S": S, "sel": sel, "o": o, "lse": lse}


def prefill_rows(q_g, q_idx_g, k_idx_g, K_g, V_g, T, head_w, idx_scale, attn_scale,
                 n_sink, n_local, p, k_max, k_min=0, rows=None, kept_override=None):
    """Prefill for the query blocks ``rows`` of one (sequence, kv head).

    q_g [G,>=T,d], q_idx_g [G,>=T,r], k_idx_g [>=T,r], K_g/V_g [>=T,d].
    ``kept_override``: optional {i: kept list}. Returns {i: dict(S, sel, o, lse)}
    with o [G, n_q, d] and lse [G, n_q].
    """
    nqb = num_blocks(T)
    rows = list(range(nqb)) if rows is None else list(rows)
    S_all = prefill_block_scores(q_idx_g, k_idx_g, T, head_w, idx_scale, rows=rows)
    out = {}
    for i in rows:
        sel = select_prefill(S_all[i], i, n_sink, n_local, p, k_max, k_min)
        kept = sel.kept if kept_override is None or i not in kept_override else list(kept_override[i])
        q_pos = np.arange(i * BLOCK, min((i + 1) * BLOCK, T))
        k_pos = kept_token_ids(kept, T)
        o, lse = attend_prefill_block(q_g[:, q_pos, :], q_pos, K_g[k_pos], V_g[k_pos], k_pos,
                                      attn_scale)
        out[i] = {"S": S_all[i], "sel": sel, "o": o, "lse": lse}
    return out


def default_head_weights(G: int) -> np.ndarray:
    """w_h = 1/G for every head of the group (reading used when none are given)."""
    return np.full(G, 1.0 / G)


def default_idx_scale(r: int) -> float:
    return 1.0 / math.sqrt(r)


def default_attn_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
