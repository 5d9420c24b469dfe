"""Pins for the fp64 oracle: checks against things other than the oracle itself.

Each ``check_*`` takes an oracle module ``O`` and raises AssertionError on a
mismatch. ``test_oracle.py`` runs them on the real oracle; ``test_oracle_mutants.py``
runs them on copies of the oracle with one planted mistake each and requires
that some check fails, so a plausible slip anywhere in the oracle is caught.

What pins what:
* hand-worked fixtures under tests/golden/ (scores, block maxima, selection,
  attention), each derived by hand with its citation;
* library routines for special cases: torch's scaled_dot_product_attention in
  float64 on the CPU (dense attention when every block is kept, sink+local
  attention when p = 0, causal attention for prefill with top-k >= blocks);
* invariants stated on the pages or fixed by the mathematics: key/value
  permutation invariance (PBS-Attn, Methodology §1), nestedness of the top-p set
  in p, positive homogeneity of the ReLU score, page-table indirection.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _close(a, b, tol=1e-12, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} != {b.shape}"
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    err = np.where(both_inf, 0.0, np.abs(a - b))
    assert np.all(err <= tol * np.maximum(1.0, np.abs(b))), f"{what}: max err {err.max()}"


# ---------------------------------------------------------------- hand cases
def check_token_scores(O):
    for c in _load("score_hand_cases.json")["token_cases"]:
        u = O.token_scores(np.array(c["q_idx"]), np.array(c["k_idx"]), np.array(c["head_w"]),
                           c["idx_scale"])
        _close(u, c["u"], what=c["name"])


def check_decode_block_scores(O):
    for c in _load("score_hand_cases.json")["decode_block_cases"]:
        S = O.decode_block_scores(np.array(c["q_idx"]), np.array(c["k_idx"]), c["T"],
                                  np.array(c["head_w"]), c["idx_scale"], block=c["block"])
        _close(S, c["S"], what=c["name"])


def check_prefill_block_scores(O):
    for c in _load("score_hand_cases.json")["prefill_block_cases"]:
        S = O.prefill_block_scores(np.array(c["q_idx"]), np.array(c["k_idx"]), c["T"],
                                   np.array(c["head_w"]), c["idx_scale"], block=c["block"])
        for i, v in c["S"].items():
            _close(S[int(i)], v, what=c["name"])


def check_selection_decode(O):
    for c in _load("selection_hand_cases.json")["decode_cases"]:
        sel = O.select_decode(np.array(c["S"]), c["n_sink"], c["n_local"], c["p"], c["k_max"],
                              c["k_min"])
        assert list(sel.kept) == c["kept"], f"{c['name']}: {sel.kept} != {c['kept']}"


def check_selection_prefill(O):
    for c in _load("selection_hand_cases.json")["prefill_cases"]:
        sel = O.select_prefill(np.array(c["S_i"], dtype=np.float64), c["i"], c["n_sink"],
                               c["n_local"], c["p"], c["k_max"])
        assert list(sel.kept) == c["kept"], f"{c['name']}: {sel.kept} != {c['kept']}"


def check_attention_hand(O):
    for c in _load("attention_hand_cases.json")["cases"]:
        o, lse = O.attend(np.array(c["q"]), np.array(c["K"]), np.array(c["V"]), c["scale"])
        _close(o, c["o"], what=c["name"])
        _close(lse, c["lse"], what=c["name"])


# ------------------------------------------------------- library special cases
def _rand_decode_case(seed, G=4, d=16, r=16, T=200):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((G, d))
    q_idx = rng.standard_normal((G, r))
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    k_idx = rng.standard_normal((T, r))
    return q, q_idx, K, V, k_idx


def _sdpa(q, K, V, scale, mask=None):
    """torch SDPA in float64; q [G, n_q, d], K/V [n, d]; returns o and lse."""
    qt = torch.from_numpy(q)
    Kt = torch.from_numpy(K)[None].expand(q.shape[0], -1, -1)
    Vt = torch.from_numpy(V)[None].expand(q.shape[0], -1, -1)
    m = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, attn_mask=m, scale=scale)
    s = (qt @ Kt.transpose(-1, -2)) * scale
    if m is not None:
        s = s.masked_fill(~m, -math.inf)
    lse = torch.logsumexp(s, dim=-1)
    return o.numpy(), lse.numpy()


def check_dense_equals_sdpa(O):
    """p = 1 and K_max >= |C|: every block is kept, so decode is dense attention."""
    for seed, T in [(1, 200), (2, 64), (3, 1)]:
        q, q_idx, K, V, k_idx = _rand_decode_case(seed, T=T)
        G = q.shape[0]
        res = O.decode_row(q, q_idx, k_idx, K, V, T, O.default_head_weights(G), 0.25, 0.25,
                           n_sink=1, n_local=1, p=1.0, k_max=1000)
        o_ref, lse_ref = _sdpa(q[:, None, :], K, V, 0.25)
        _close(res["o"], o_ref[:, 0], tol=1e-12, what=f"dense o T={T}")
        _close(res["lse"], lse_ref[:, 0], tol=1e-12, what=f"dense lse T={T}")


def check_sink_local_equals_masked_sdpa(O):
    """p = 0, K_min = 0: only sink and local blocks, i.e. sink + sliding-window attention."""
    T, n_sink, n_local = 200, 1, 1         # blocks 0 and 3 (the partial last block)
    q, q_idx, K, V, k_idx = _rand_decode_case(4, T=T)
    G = q.shape[0]
    res = O.decode_row(q, q_idx, k_idx, K, V, T, O.default_head_weights(G), 0.25, 0.3,
                       n_sink=n_sink, n_local=n_local, p=0.0, k_max=8)
    t = np.arange(T)
    visible = (t < 64 * n_sink) | (t >= 64 * ((T + 63) // 64 - n_local))
    mask = np.broadcast_to(visible, (G, 1, T)).copy()
    o_ref, lse_ref = _sdpa(q[:, None, :], K, V, 0.3, mask)
    _close(res["o"], o_ref[:, 0], tol=1e-12, what="sink+local o")
    _close(res["lse"], lse_ref[:, 0], tol=1e-12, what="sink+local lse")


def check_prefill_dense_equals_causal_sdpa(O):
    """Prefill with top-k >= number of blocks and p = 1 is causal dense attention."""
    rng = np.random.default_rng(5)
    G, d, r, T = 2, 16, 16, 150
    q = rng.standard_normal((G, T, d))
    q_idx = rng.standard_normal((G, T, r))
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    k_idx = rng.standard_normal((T, r))
    out = O.prefill_rows(q, q_idx, k_idx, K, V, T, O.default_head_weights(G), 0.25, 0.2,
                         n_sink=1, n_local=1, p=1.0, k_max=64)
    causal = np.tril(np.ones((T, T), dtype=bool))
    o_ref, lse_ref = _sdpa(q, K, V, 0.2, np.broadcast_to(causal, (G, T, T)).copy())
    for i, res in out.items():
        rows = np.arange(i * 64, min(i * 64 + 64, T))
        _close(res["o"], o_ref[:, rows], tol=1e-12, what=f"prefill o block {i}")
        _close(res["lse"], lse_ref[:, rows], tol=1e-12, what=f"prefill lse block {i}")


def check_prefill_blockmask_equals_masked_sdpa(O):
    """Prefill with a small top-k: the output equals SDPA under the token mask built from
    the kept blocks and causality."""
    rng = np.random.default_rng(6)
    G, d, r, T = 2, 16, 16, 64 * 7 + 5
    q = rng.standard_normal((G, T, d))
    q_idx = rng.standard_normal((G, T, r))
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    k_idx = rng.standard_normal((T, r))
    out = O.prefill_rows(q, q_idx, k_idx, K, V, T, O.default_head_weights(G), 0.25, 0.2,
                         n_sink=1, n_local=1, p=1.0, k_max=2)
    for i, res in out.items():
        kept = res["sel"].kept
        rows = np.arange(i * 64, min(i * 64 + 64, T))
        blk_ok = np.zeros(T, dtype=bool)
        for j in kept:
            blk_ok[j * 64:min(j * 64 + 64, T)] = True
        mask = blk_ok[None, :] & (np.arange(T)[None, :] <= rows[:, None])
        o_ref, lse_ref = _sdpa(q[:, rows], K, V, 0.2, np.broadcast_to(mask, (G,) + mask.shape).copy())
        _close(res["o"], o_ref, tol=1e-12, what=f"prefill masked o block {i}")
        _close(res["lse"], lse_ref, tol=1e-12, what=f"prefill masked lse block {i}")


# ------------------------------------------------------------------ invariants
def check_kv_permutation_invariance(O):
    """PBS-Attn, Methodology §1: permuting key/value pairs together leaves the output."""
    rng = np.random.default_rng(7)
    q = rng.standard_normal((4, 32))
    K = rng.standard_normal((300, 32))
    V = rng.standard_normal((300, 32))
    perm = rng.permutation(300)
    o1, l1 = O.attend(q, K, V, 0.2)
    o2, l2 = O.attend(q, K[perm], V[perm], 0.2)
    _close(o1, o2, tol=1e-12, what="perm o")
    _close(l1, l2, tol=1e-12, what="perm lse")


def check_nested_in_p(O):
    """The dynamic set for p1 < p2 is a prefix of the set for p2 (same order)."""
    rng = np.random.default_rng(8)
    S = rng.standard_normal(40) * 2.0
    prev = None
    for p in [0.05, 0.2, 0.5, 0.8, 0.95, 0.999]:
        sel = O.select_decode(S, 2, 3, p, k_max=1000)
        dyn = sel.order[:sel.k]
        if prev is not None:
            assert dyn[:len(prev)] == prev, "top-p sets are not nested"
            assert len(dyn) >= len(prev)
        prev = dyn


def check_homogeneity(O):
    """ReLU is positively homogeneous: scaling all head weights by c > 0 scales S by c,
    which keeps the K_max (top-k) set when p >= 1."""
    rng = np.random.default_rng(9)
    q_idx = rng.standard_normal((4, 16))
    k_idx = rng.standard_normal((640, 16))
    w = np.array([0.1, 0.2, 0.3, 0.4])
    S1 = O.decode_block_scores(q_idx, k_idx, 640, w, 0.25)
    S2 = O.decode_block_scores(q_idx, k_idx, 640, 3.0 * w, 0.25)
    _close(S2, 3.0 * S1, tol=1e-12, what="homogeneity")
    a = O.select_decode(S1, 1, 1, 1.0, k_max=3).kept
    b = O.select_decode(S2, 1, 1, 1.0, k_max=3).kept
    assert a == b


def check_paged_gather(O):
    """A shuffled page table addresses the same logical tokens as a contiguous cache."""
    rng = np.random.default_rng(10)
    B, Hkv, T, w = 2, 3, 64 * 5, 8
    logical = rng.standard_normal((B, Hkv, T, w))
    nb = T // 64
    table = rng.permutation(B * nb).reshape(B, nb)
    pool = np.zeros((B * nb, Hkv, 64, w))
    for b in range(B):
        for j in range(nb):
            pool[table[b, j]] = logical[b, :, j * 64:(j + 1) * 64]
    ids = rng.integers(0, T, size=50)
    for b in range(B):
        for g in range(Hkv):
            a = O.gather_tokens(logical, None, b, g, ids)
            c = O.gather_tokens(pool, table, b, g, ids)
            assert np.array_equal(a, c)


ALL_CHECKS = [
    check_token_scores, check_decode_block_scores, check_prefill_block_scores,
    check_selection_decode, check_selection_prefill, check_attention_hand,
    check_dense_equals_sdpa, check_sink_local_equals_masked_sdpa,
    check_prefill_dense_equals_causal_sdpa, check_prefill_blockmask_equals_masked_sdpa,
    check_kv_permutation_invariance, check_nested_in_p, check_homogeneity, check_paged_gather,
]
