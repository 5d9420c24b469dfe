"""Plain fp64 CPU oracle of two-level (block, then token-group) routing for decode.

TEST INFRASTRUCTURE, like ``bsa_oracle``: only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s oracle legs may import it; the product never does, and this
module imports nothing from the product.

Source: "Hierarchical Global Attention (HGA)", Central mechanism:
* §1: the sequence is cut into chunks of C = 64 tokens, and each chunk into groups;
* §2: level 1 routes the query to chunks by chunk summaries; level 2 routes it,
  inside the chosen chunks, to groups by group summaries; the current chunk, a few
  sink chunks and the recent local chunks are always visible;
* §4: the output is exact softmax attention over the tokens of the routed set, with
  no summary values in it.

Readings where the page leaves a step open:
* chunks are the method's 64-token blocks, and level 1 is the method's own block
  selection (sinks + local window + top-p over the candidates, capped at K_max);
* a summary score is the method's block score restricted to the tokens it covers:
  the max over those tokens of u_t = idx_scale * sum_h w_h ReLU(q_idx[h] . k_idx[t])
  (a group of gs tokens, gs dividing 64; the page's RoPE-aware mixed summaries are
  model-side and not used);
* level 2 ranks the groups of the dynamically selected blocks (not the always
  visible ones, which stay whole) by group score descending, ties to the lower
  group id, and keeps the first k_groups of them; a group past the sequence end
  does not exist;
* attention runs over every token of the always-visible blocks and of the kept
  groups (t < T).

With gs = 64 (one group per block) and k_groups >= K_max, or with k_groups at
least the number of candidate groups, level 2 keeps every selected token and the
result equals ``bsa_oracle.decode_row``.
"""
from __future__ import annotations

import numpy as np

from oracle import bsa_oracle as O

BLOCK = O.BLOCK


def group_scores(q_idx_g: np.ndarray, k_idx_g: np.ndarray, T: int, head_w: np.ndarray,
                 idx_scale: float, gs: int) -> np.ndarray:
    """Score of every group of gs tokens: the max of the token scores it covers."""
    u = O.token_scores(q_idx_g, k_idx_g[:T], head_w, idx_scale)
    ng = (T + gs - 1) // gs
    return np.array([u[k * gs:min((k + 1) * gs, T)].max() for k in range(ng)])


def select_groups(sel: O.Selection, Sg: np.ndarray, T: int, gs: int, k_groups: int):
    """Level 2: kept group ids among the groups of the dynamically selected blocks.
    Returns (candidate groups ascending, kept groups ascending)."""
    gpb = BLOCK // gs
    R = set(sel.reserved)
    dyn = [j for j in sel.kept if j not in R]
    cand = [j * gpb + k for j in dyn for k in range(gpb) if (j * gpb + k) * gs < T]
    if not cand:
        return [], []
    s = np.array([Sg[c] for c in cand])
    order = [cand[t] for t in np.lexsort((np.array(cand), -s))]
    return cand, sorted(order[:k_groups])


def routed_tokens(sel: O.Selection, kept_groups, T: int, gs: int) -> np.ndarray:
    """Token ids of the always-visible blocks and of the kept groups, ascending."""
    ids = [np.arange(j * BLOCK, min((j + 1) * BLOCK, T)) for j in sel.reserved]
    ids += [np.arange(c * gs, min((c + 1) * gs, T)) for c in kept_groups]
    return np.sort(np.concatenate(ids)) if ids else np.zeros(0, dtype=np.int64)


def hga_decode_row(q_g, q_idx_g, k_idx_g, K_g, V_g, T, head_w, idx_scale, attn_scale,
                   n_sink, n_local, p, k_max, gs, k_groups, k_min=0, kept_override=None,
                   groups_override=None):
    """One decode row (sequence b, kv head g) with two-level routing.

    Returns dict(S, sel, Sg, cand, groups, o, lse); ``kept_override`` /
    ``groups_override`` replace the level-1 / level-2 choices (to re-run attention on
    a device choice that a comparison accepted as a tie).
    """
    S = O.decode_block_scores(q_idx_g, k_idx_g, T, head_w, idx_scale)
    sel = O.select_decode(S, n_sink, n_local, p, k_max, k_min)
    if kept_override is not None:
        R = set(sel.reserved)
        sel = O.Selection(sorted(kept_override), sel.reserved, sel.candidates, sel.order,
                          sel.mass, sel.cum, sel.k_p, len(set(kept_override) - R), sel.cap)
    Sg = group_scores(q_idx_g, k_idx_g, T, head_w, idx_scale, gs)
    cand, groups = select_groups(sel, Sg, T, gs, k_groups)
    if groups_override is not None:
        groups = sorted(groups_override)
    ids = routed_tokens(sel, groups, T, gs)
    o, lse = O.attend(q_g, K_g[ids], V_g[ids], attn_scale)
    return {"S": S, "sel": sel, "Sg": Sg, "cand": cand, "groups": groups, "o": o, "lse": lse}
