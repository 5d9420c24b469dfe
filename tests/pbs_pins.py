"""Pins for the PBS oracle (oracle/pbs_oracle.py): checks against things other than
the oracle itself. Each ``check_*`` takes the PBS oracle module ``P`` and raises
AssertionError on a mismatch; ``test_pbs_oracle.py`` runs them on the real oracle,
and the planted-mistake tests require that some check fails on each mutant.

What pins what:
* hand-worked fixtures (tests/golden/pbs_hand_cases.json): importance values,
  segment permutations with ties and a ragged last segment, reserved sets;
* library routines: torch.softmax in float64 for the importance (mean of masked
  softmax rows), torch's scaled_dot_product_attention in float64 with a boolean
  mask for the attention over the original positions of the kept keys (the
  permutation invariance of PBS-Attn, Methodology §1), and for the dense limit
  (every block kept: plain causal attention);
* a special case that reduces to the pinned unpermuted oracle: one-block segments;
* structure fixed by the method: the permutation maps every segment onto itself
  (Methodology §2) and orders each segment by importance.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

from oracle import bsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cases():
    with open(os.path.join(GOLDEN, "pbs_hand_cases.json")) as f:
        return json.load(f)


def _inputs(T=64 * 7 + 21, G=2, d=16, r=16, seed=0, plant=True):
    """Small random prefill inputs in float64 (bf16-like magnitudes), with a few keys
    aligned with late queries so that importance is far from uniform."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((G, T, d))
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    if plant:
        qhat = q[:, -1, :].mean(0)
        qhat /= np.linalg.norm(qhat)
        for t in rng.choice(T, size=12, replace=False):
            K[t] = 3.0 * qhat + 0.1 * rng.standard_normal(d)
    q_idx = rng.standard_normal((G, T, r))
    k_idx = rng.standard_normal((T, r))
    return q, q_idx, k_idx, K, V


def _sdpa_masked(q_rows, K, V, allowed, scale):
    """torch SDPA in float64: q_rows [G, nq, d], allowed [nq, T] bool."""
    qt = torch.from_numpy(q_rows)[None]
    kt = torch.from_numpy(K)[None, None].expand(1, q_rows.shape[0], -1, -1)
    vt = torch.from_numpy(V)[None, None].expand(1, q_rows.shape[0], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(allowed), scale=scale)
    return o[0].numpy()


# ---------------------------------------------------------------- hand cases
def check_importance_hand(P):
    for c in _cases()["importance_cases"]:
        imp = P.key_importance(np.array(c["q_last"]), np.array(c["q_pos"]), np.array(c["K"]),
                               c["scale"])
        assert np.allclose(imp, c["imp"], rtol=0, atol=1e-14), f"{c['name']}: {imp}"


def check_permutation_hand(P):
    for c in _cases()["permutation_cases"]:
        perm = P.segment_permutation(np.array(c["imp"]), c["seg"])
        assert list(perm) == c["perm"], f"{c['name']}: {list(perm)} != {c['perm']}"


def check_reserved_hand(P):
    for c in _cases()["reserved_cases"]:
        R = P.reserved_pbs(c["i"], c["seg_blocks"], c["nqb"], c["n_sink"], c["n_local"])
        assert R == c["reserved"], f"{c['name']}: {R} != {c['reserved']}"
        S = np.zeros(max(1, c["i"]))
        sel = P.select_pbs(S, c["i"], c["seg_blocks"], c["nqb"], c["n_sink"], c["n_local"],
                           0.0, 0)
        assert sel.candidates == c["candidates"], f"{c['name']}: {sel.candidates}"


# ---------------------------------------------------------------- library routines
def check_importance_vs_torch(P):
    q, _, _, K, _ = _inputs()
    T = K.shape[0]
    ql = np.arange(T - 37, T)
    imp = P.key_importance(q[:, ql, :], ql, K, 0.25)
    s = torch.from_numpy(np.einsum("gqd,kd->gqk", q[:, ql, :], K) * 0.25)
    mask = torch.from_numpy(np.arange(T)[None, :] <= ql[:, None])
    ref = torch.softmax(s.masked_fill(~mask, float("-inf")), dim=-1).mean(dim=(0, 1)).numpy()
    assert np.allclose(imp, ref, rtol=1e-12, atol=1e-15)
    assert abs(imp.sum() - 1.0) < 1e-12


def check_attention_is_over_original_positions(P):
    """Output of every row = masked SDPA over the original positions of the keys of
    its kept permuted blocks (attention is invariant to the key order)."""
    q, q_idx, k_idx, K, V = _inputs(seed=1)
    T, G, d = K.shape[0], q.shape[0], q.shape[2]
    scale = 1.0 / math.sqrt(d)
    seg = 128
    perm, rows = P.pbs_prefill_rows(q, q_idx, k_idx, K, V, T, seg, np.full(G, 0.5), 0.25, scale,
                                    1, 1, 1.0, 2)
    for i, ref in rows.items():
        q0, q1 = i * 64, min(i * 64 + 64, T)
        keys = perm[O.kept_token_ids(ref["sel"].kept, T)]
        allowed = np.zeros((q1 - q0, T), dtype=bool)
        allowed[:, keys] = True
        allowed &= np.arange(T)[None, :] <= np.arange(q0, q1)[:, None]
        o = _sdpa_masked(q[:, q0:q1, :], K, V, allowed, scale)
        assert np.allclose(ref["o"], o, rtol=1e-10, atol=1e-12), f"row {i}"


def check_dense_limit_is_causal_attention(P):
    q, q_idx, k_idx, K, V = _inputs(seed=2)
    T, G, d = K.shape[0], q.shape[0], q.shape[2]
    scale = 1.0 / math.sqrt(d)
    _, rows = P.pbs_prefill_rows(q, q_idx, k_idx, K, V, T, 192, np.full(G, 0.5), 0.25, scale,
                                 1, 2, 1.0, 64)
    allowed = np.arange(T)[None, :] <= np.arange(T)[:, None]
    o_all = _sdpa_masked(q[:, :T, :], K, V, allowed, scale)
    for i, ref in rows.items():
        q0, q1 = i * 64, min(i * 64 + 64, T)
        assert np.allclose(ref["o"], o_all[:, q0:q1], rtol=1e-10, atol=1e-12), f"row {i}"


# ---------------------------------------------------------------- special case, structure
def check_one_block_segments_are_plain_prefill(P):
    q, q_idx, k_idx, K, V = _inputs(seed=3)
    T, G, d = K.shape[0], q.shape[0], q.shape[2]
    hw = np.array([0.3, 0.7])
    for p, k_max in ((1.0, 2), (0.6, 3)):
        _, rows = P.pbs_prefill_rows(q, q_idx, k_idx, K, V, T, 64, hw, 0.25, 1 / math.sqrt(d),
                                     1, 2, p, k_max)
        plain = O.prefill_rows(q, q_idx, k_idx, K, V, T, hw, 0.25, 1 / math.sqrt(d), 1, 2, p,
                               k_max)
        for i in rows:
            assert rows[i]["sel"].kept == plain[i]["sel"].kept, f"row {i}"
            assert np.allclose(rows[i]["S"], plain[i]["S"], rtol=1e-13, atol=0), f"row {i}"
            assert np.allclose(rows[i]["o"], plain[i]["o"], rtol=1e-12, atol=1e-14), f"row {i}"


def check_permutation_structure(P):
    q, _, _, K, _ = _inputs(seed=4)
    T = K.shape[0]
    ql = np.arange(T - 64, T)
    imp = P.key_importance(q[:, ql, :], ql, K, 0.25)
    for seg in (64, 128, 256, 1024):
        perm = P.segment_permutation(imp, seg)
        assert sorted(perm) == list(range(T)), "not a permutation"
        for s0 in range(0, T, seg):
            s1 = min(s0 + seg, T)
            block = perm[s0:s1]
            assert block.min() >= s0 and block.max() < s1, "a key left its segment"
            assert np.all(np.diff(imp[block]) <= 0), "segment not in descending importance"


def check_scores_of_permuted_blocks_brute_force(P):
    """Block scores by explicit loops over (query, key, head) on a small case: the
    keys of permuted block j are the original positions perm[64 j : 64 j + 64]."""
    q, q_idx, k_idx, K, V = _inputs(T=64 * 5 + 9, seed=5)
    T, G = K.shape[0], q.shape[0]
    hw = np.array([0.25, 0.75])
    perm, rows = P.pbs_prefill_rows(q, q_idx, k_idx, K, V, T, 128, hw, 0.5, 0.25, 1, 0, 1.0, 1,
                                    rows=[2, 3, 4])
    for i, ref in rows.items():
        b0 = (i // 2) * 2
        assert len(ref["S"]) == b0
        for j in range(b0):
            best = 0.0
            for tq in range(i * 64, min(i * 64 + 64, T)):
                for p in range(j * 64, j * 64 + 64):
                    t = int(perm[p])
                    u = 0.0
                    for h in range(G):
                        dot = sum(q_idx[h, tq, c] * k_idx[t, c] for c in range(q_idx.shape[2]))
                        u += hw[h] * max(dot, 0.0)
                    best = max(best, 0.5 * u)
            assert abs(ref["S"][j] - best) <= 1e-12 * max(1.0, best), f"S[{i},{j}]"


ALL_CHECKS = [check_scores_of_permuted_blocks_brute_force, check_importance_hand, check_permutation_hand, check_reserved_hand,
              check_importance_vs_torch, check_attention_is_over_original_positions,
              check_dense_limit_is_causal_attention, check_one_block_segments_are_plain_prefill,
              check_permutation_structure]
