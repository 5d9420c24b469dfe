"""Pins for the two-level routing oracle (oracle/hga_oracle.py): checks against things
other than the oracle itself; ``test_hga_oracle.py`` runs them on the real oracle and
requires that planted mistakes in copies of it fail some of them.

What pins what:
* hand-worked fixtures (tests/golden/hga_hand_cases.json): kept groups for several
  caps, with a tie and a partial last block, and the routed token set;
* brute force: group scores by explicit loops over (token, head);
* the mathematics: a block's score is the max of its groups' scores;
* a special case that reduces to the pinned one-level oracle: one group per block
  with k_groups >= K_max, and k_groups covering every candidate group;
* a library routine: torch's scaled_dot_product_attention in float64 with a
  boolean mask over the routed tokens.
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
    with open(os.path.join(GOLDEN, "hga_hand_cases.json")) as f:
        return json.load(f)


def _row(T=64 * 9 + 21, G=4, d=32, r=16, seed=0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((G, d))
    qi = rng.standard_normal((G, r))
    ki = rng.standard_normal((T, r))
    K = rng.standard_normal((T, d))
    V = rng.standard_normal((T, d))
    return q, qi, ki, K, V


def _ranges(text):
    out = []
    for part in text.split(","):
        a, b = part.strip().split("-")
        out.extend(range(int(a), int(b) + 1))
    return out


def check_group_selection_hand(H):
    for c in _cases()["group_selection_cases"]:
        sel = O.Selection(c["kept"], c["reserved"], [])
        ng = (c["T"] + c["gs"] - 1) // c["gs"]
        Sg = np.full(ng, -1.0)
        for k, v in c["Sg"].items():
            Sg[int(k)] = v
        for kg, want in c["k_groups"].items():
            _, groups = H.select_groups(sel, Sg, c["T"], c["gs"], int(kg))
            assert list(groups) == want, f"{c['name']} k={kg}: {groups} != {want}"
        _, g2 = H.select_groups(sel, Sg, c["T"], c["gs"], 2)
        toks = H.routed_tokens(sel, g2, c["T"], c["gs"])
        assert list(toks) == _ranges(c["tokens_k2"]), f"{c['name']}: tokens"


def check_group_scores_brute_force(H):
    q, qi, ki, K, V = _row(T=64 * 3 + 5, seed=1)
    hw = np.array([0.1, 0.2, 0.3, 0.4])
    for gs in (16, 32):
        Sg = H.group_scores(qi, ki, ki.shape[0], hw, 0.25, gs)
        T = ki.shape[0]
        for k in range(len(Sg)):
            best = -np.inf
            for t in range(k * gs, min((k + 1) * gs, T)):
                u = 0.0
                for h in range(qi.shape[0]):
                    u += hw[h] * max(0.0, sum(qi[h, c] * ki[t, c] for c in range(qi.shape[1])))
                best = max(best, 0.25 * u)
            assert abs(Sg[k] - best) <= 1e-12 * max(1.0, abs(best)), f"group {k}"


def check_block_is_max_of_groups(H):
    q, qi, ki, K, V = _row(seed=2)
    T = ki.shape[0]
    hw = np.full(4, 0.25)
    S = O.decode_block_scores(qi, ki, T, hw, 0.25)
    for gs in (16, 32):
        Sg = H.group_scores(qi, ki, T, hw, 0.25, gs)
        gpb = 64 // gs
        for j in range(len(S)):
            assert S[j] == max(Sg[j * gpb:(j + 1) * gpb]), f"block {j}, gs {gs}"


def check_reduces_to_one_level(H):
    q, qi, ki, K, V = _row(seed=3)
    T, d = ki.shape[0], K.shape[1]
    hw = np.full(4, 0.25)
    for p, k_max in ((0.9, 4), (1.0, 3)):
        plain = O.decode_row(q, qi, ki, K, V, T, hw, 0.25, 1 / math.sqrt(d), 1, 2, p, k_max)
        one = H.hga_decode_row(q, qi, ki, K, V, T, hw, 0.25, 1 / math.sqrt(d), 1, 2, p, k_max,
                               64, k_max)
        allg = H.hga_decode_row(q, qi, ki, K, V, T, hw, 0.25, 1 / math.sqrt(d), 1, 2, p, k_max,
                                16, 4 * k_max)
        for r in (one, allg):
            assert r["sel"].kept == plain["sel"].kept
            assert np.allclose(r["o"], plain["o"], rtol=1e-12, atol=1e-14)
            assert np.allclose(r["lse"], plain["lse"], rtol=1e-12, atol=1e-14)


def check_attention_vs_masked_sdpa(H):
    q, qi, ki, K, V = _row(seed=4)
    T, G, d = ki.shape[0], q.shape[0], K.shape[1]
    hw = np.full(4, 0.25)
    r = H.hga_decode_row(q, qi, ki, K, V, T, hw, 0.25, 1 / math.sqrt(d), 1, 2, 0.95, 5, 16, 7)
    # the routed set from its definition: whole reserved blocks, then kept groups
    mask = np.zeros(T, dtype=bool)
    for j in r["sel"].reserved:
        mask[j * 64:min(j * 64 + 64, T)] = True
    for c in r["groups"]:
        mask[c * 16:min(c * 16 + 16, T)] = True
    assert len(r["groups"]) == min(7, len(r["cand"]))
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(K)[None, None].expand(1, G, -1, -1),
        torch.from_numpy(V)[None, None].expand(1, G, -1, -1),
        attn_mask=torch.from_numpy(mask)[None, None, None, :], scale=1 / math.sqrt(d))
    assert np.allclose(r["o"], o[0, :, 0].numpy(), rtol=1e-10, atol=1e-12)


ALL_CHECKS = [check_group_selection_hand, check_group_scores_brute_force,
              check_block_is_max_of_groups, check_reduces_to_one_level,
              check_attention_vs_masked_sdpa]
