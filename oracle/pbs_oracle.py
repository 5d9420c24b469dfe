"""Plain fp64 CPU oracle of block-sparse prefill over segment-permuted keys (PBS).

TEST INFRASTRUCTURE, like ``bsa_oracle``: only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s oracle legs may import it; the product never does, and this
module imports nothing from the product.

Source: "Sparser Block-Sparse Attention via Token Permutation" (PBS-Attn),
Methodology:
* §1: attention is invariant to permuting key/value pairs together, and
  equivariant to permuting queries; permuting both and inverting the output
  permutation gives the unpermuted result;
* §2: the sequence is cut into contiguous segments of S tokens; keys are permuted
  only inside their segment, so causality between segments is kept (a query of
  segment i never sees a key of a segment j > i);
* §3: the permutation of a segment sorts its keys by a global importance score in
  descending order; the importance of a key is the mean pooling of the attention
  scores that the last query block gives it; queries stay in their natural order;
* §4: block selection then works on the permuted keys.

Readings where the page leaves a step open:
* "attention scores" of the last query block = its causal softmax probabilities
  (scale 1/sqrt(d) unless given), averaged over the block's queries and the
  query heads of the kv group (one permutation per kv head);
* ties in importance order by the lower original position first;
* the block scorer stays the method's own (max over the tile of the weighted-ReLU
  index score, SpotAttention Methodology §1), applied to the permuted index keys;
  the page's mean pooling is a different scorer and is not used;
* the query block's own segment is always kept, with a per-key causal mask on the
  keys' original positions (inside a segment the permutation mixes earlier and
  later keys); the sink blocks and the n_local blocks just before the own segment
  (in permuted order) are kept too; every other block of an earlier segment is a
  candidate for the top-p / top-k rule;
* queries are not permuted, so no inverse permutation of the output is needed.

With S = 64 (one block per segment) the permutation only reorders keys inside a
block: block maxima, the reserved set and the visible token set are those of the
unpermuted prefill, so the result equals ``bsa_oracle.prefill_rows``.
"""
from __future__ import annotations

import numpy as np

from oracle import bsa_oracle as O

BLOCK = O.BLOCK


# --------------------------------------------------------------------------
# importance and permutation  [PBS §2, §3]
# --------------------------------------------------------------------------
def key_importance(q_last: np.ndarray, q_pos: np.ndarray, K: np.ndarray, scale: float):
    """Mean over the query rows of their causal softmax probabilities over the keys.

    q_last: [G, nq, d] queries of the last query block at positions q_pos [nq];
    K: [T, d] keys in natural order. A key t is visible to a query at position tq
    when t <= tq. Returns imp [T]; imp sums to 1 (every row is a distribution).
    """
    T = K.shape[0]
    s = np.einsum("gqd,kd->gqk", q_last, K) * scale                  # [G, nq, T]
    visible = np.arange(T)[None, None, :] <= q_pos[None, :, None]
    s = np.where(visible, s, -np.inf)
    m = s.max(axis=2, keepdims=True)
    e = np.where(visible, np.exp(s - m), 0.0)
    prob = e / e.sum(axis=2, keepdims=True)
    return prob.mean(axis=(0, 1))


def segment_permutation(imp: np.ndarray, seg: int) -> np.ndarray:
    """perm[p] = original position of the key at permuted position p.

    Positions are cut into segments [s * seg, (s + 1) * seg); inside a segment the
    keys are ordered by importance descending, equal importance by lower position.
    """
    T = len(imp)
    perm = np.empty(T, dtype=np.int64)
    for s0 in range(0, T, seg):
        s1 = min(s0 + seg, T)
        pos = np.arange(s0, s1)
        order = np.lexsort((pos, -imp[s0:s1]))      # primary -imp, then position
        perm[s0:s1] = pos[order]
    return perm


# --------------------------------------------------------------------------
# selection on the permuted blocks  [PBS §2, §4; SpotAttention §3]
# --------------------------------------------------------------------------
def segment_blocks(i: int, seg_blocks: int, nqb: int):
    """[b0, b1): the blocks of query block i's segment."""
    b0 = (i // seg_blocks) * seg_blocks
    return b0, min(b0 + seg_blocks, nqb)


def reserved_pbs(i: int, seg_blocks: int, nqb: int, n_sink: int, n_local: int) -> list:
    """Own segment's blocks, sink blocks [0, n_sink) up to the segment's end, and the
    n_local blocks just before the own segment."""
    b0, b1 = segment_blocks(i, seg_blocks, nqb)
    return sorted(set(range(b0, b1)) | set(range(min(n_sink, b1))) |
                  set(range(max(0, b0 - n_local), b0)))


def select_pbs(S_i: np.ndarray, i: int, seg_blocks: int, nqb: int, n_sink: int, n_local: int,
               p: float, k_max: int, k_min: int = 0) -> O.Selection:
    """Kept permuted key blocks of query block i; S_i holds the scores of blocks
    [0, b0) (the earlier segments), b0 the first block of i's segment."""
    b0, _ = segment_blocks(i, seg_blocks, nqb)
    R = reserved_pbs(i, seg_blocks, nqb, n_sink, n_local)
    Rs = set(R)
    C = [j for j in range(b0) if j not in Rs]
    order, mass, cum, k_p, k, cap = O.select_dynamic(S_i, C, p, k_max, k_min)
    kept = sorted(Rs | set(order[:k]))
    return O.Selection(kept, R, C, order, mass, cum, k_p, k, cap)


# --------------------------------------------------------------------------
# whole rows
# --------------------------------------------------------------------------
def last_block_importance(q_g, K_g, T, attn_scale):
    """Importance of every key from the last query block's rows (positions
    [64 * (nqb - 1), T)) of the group's heads."""
    ql = np.arange((O.num_blocks(T) - 1) * BLOCK, T)
    return key_importance(q_g[:, ql, :], ql, K_g[:T], attn_scale)


def pbs_prefill_rows(q_g, q_idx_g, k_idx_g, K_g, V_g, T, seg, head_w, idx_scale, attn_scale,
                     n_sink, n_local, p, k_max, k_min=0, rows=None, kept_override=None,
                     perm_override=None):
    """PBS prefill for query blocks ``rows`` of one (sequence, kv head).

    q_g [G,>=T,d], q_idx_g [G,>=T,r], k_idx_g [>=T,r], K_g/V_g [>=T,d] in natural
    order; seg = segment length in tokens (a multiple of 64). ``perm_override``
    replaces the permutation (used to re-run the steps after it on an order that a
    comparison accepted as a tie).
    Returns (perm, {i: dict(S, sel, o, lse)}): S are the scores of the permuted
    blocks [0, b0), o [G, n_q, d] and lse [G, n_q] in natural query order.
    """
    assert seg % BLOCK == 0 and seg > 0
    nqb = O.num_blocks(T)
    seg_blocks = seg // BLOCK
    rows = list(range(nqb)) if rows is None else list(rows)
    # importance from the last query block, then the segmented permutation
    if perm_override is None:
        perm = segment_permutation(last_block_importance(q_g, K_g, T, attn_scale), seg)
    else:
        perm = np.asarray(perm_override, dtype=np.int64)
    kidx_p = k_idx_g[:T][perm]
    out = {}
    for i in rows:
        b0, _ = segment_blocks(i, seg_blocks, nqb)
        q0, q1 = i * BLOCK, min((i + 1) * BLOCK, T)
        # scores of the permuted blocks of earlier segments: every key there is
        # causal for every query of block i
        if b0 > 0:
            u = O.token_scores(q_idx_g[:, q0:q1, :], kidx_p[:b0 * BLOCK], head_w, idx_scale)
            S_i = np.array([u[:, j * BLOCK:(j + 1) * BLOCK].max() for j in range(b0)])
        else:
            S_i = np.zeros(0)
        sel = select_pbs(S_i, i, seg_blocks, nqb, n_sink, n_local, p, k_max, k_min)
        kept = sel.kept if kept_override is None or i not in kept_override \
            else list(kept_override[i])
        # keys of the kept permuted blocks, masked by their original positions
        k_perm_pos = O.kept_token_ids(kept, T)
        k_orig = perm[k_perm_pos]
        q_pos = np.arange(q0, q1)
        o, lse = O.attend_prefill_block(q_g[:, q_pos, :], q_pos, K_g[k_orig], V_g[k_orig],
                                        k_orig, attn_scale)
        out[i] = {"S": S_i, "sel": sel, "o": o, "lse": lse}
    return perm, out
