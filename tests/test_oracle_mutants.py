"""Each planted mistake in a copy of the oracle must be caught by some pin.

The mistakes are planted in fresh copies of ``oracle/bsa_oracle.py`` on the CPU;
the real oracle is never modified. A mutant that passes every pin would mean the
pins cannot tell that slip from the method.
"""
import importlib.util
import os
import sys

import numpy as np
import pytest

from tests import oracle_pins

ORACLE_PATH = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "bsa_oracle.py")


def fresh_oracle(tag):
    spec = importlib.util.spec_from_file_location(f"bsa_oracle_mutant_{tag}", ORACLE_PATH)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod          # dataclasses look their module up here
    spec.loader.exec_module(mod)
    return mod


def m_block_mean(O):
    def decode_block_scores(q_idx_g, k_idx_g, T, head_w, idx_scale, block=64):
        u = O.token_scores(q_idx_g, k_idx_g[:T], head_w, idx_scale)
        nb = O.num_blocks(T, block)
        return np.array([u[j * block:min((j + 1) * block, T)].mean() for j in range(nb)])
    O.decode_block_scores = decode_block_scores


def m_no_relu(O):
    def token_scores(q, k, w, s):
        if q.ndim == 2:
            return s * np.tensordot(w, q @ k.T, axes=(0, 0))
        return s * np.tensordot(w, np.einsum("gqr,kr->gqk", q, k), axes=(0, 0))
    O.token_scores = token_scores


def m_reversed_weights(O):
    orig = O.token_scores
    O.token_scores = lambda q, k, w, s: orig(q, k, np.asarray(w)[::-1].copy(), s)


def m_prefill_max_per_head(O):
    def prefill_block_scores(q_idx_g, k_idx_g, T, head_w, idx_scale, rows=None, block=64):
        nqb = O.num_blocks(T, block)
        rows = range(nqb) if rows is None else rows
        out = {}
        for i in rows:
            q0, q1 = i * block, min((i + 1) * block, T)
            S_i = np.zeros(i)
            for j in range(i):
                d = np.einsum("gqr,kr->gqk", q_idx_g[:, q0:q1], k_idx_g[j * block:(j + 1) * block])
                S_i[j] = idx_scale * np.sum(head_w * np.maximum(d, 0).max(axis=(1, 2)))
            out[i] = S_i
        return out
    O.prefill_block_scores = prefill_block_scores


def m_softmax_over_all_blocks(O):
    orig = O.select_dynamic

    def select_decode(S, n_sink, n_local, p, k_max, k_min=0):
        nb = len(S)
        R = O.reserved_decode(nb, n_sink, n_local)
        C = [j for j in range(nb) if j not in set(R)]
        # mistake: masses normalised over every block, reserved ones included
        w = np.exp(S - S.max())
        mass_all = w / w.sum()
        order = sorted(C, key=lambda j: (-S[j], j))
        cum = np.cumsum([mass_all[j] for j in order])
        ph = O.p_hat(p)
        if ph <= 0:
            k_p = 0
        elif ph >= 1:
            k_p = len(C)
        else:
            hit = np.nonzero(cum >= ph)[0]
            k_p = int(hit[0]) + 1 if hit.size else len(C)
        k = max(min(k_p, min(k_max, len(C))), min(k_min, len(C)))
        return O.Selection(sorted(set(R) | set(order[:k])), R, C, order, None, cum, k_p, k, 0)
    O.select_decode = select_decode
    del orig


def m_ties_higher_first(O):
    orig = O.select_dynamic

    def select_dynamic(S, candidates, p, k_max, k_min=0):
        C = list(candidates)[::-1]
        order, mass, cum, k_p, k, cap = orig(S, C, p, k_max, k_min)
        # reorder equal scores to higher id first
        order = sorted(order, key=lambda j: (-S[j], -j))
        return order, mass, cum, k_p, k, cap
    O.select_dynamic = select_dynamic


def m_strict_greater(O):
    def select_dynamic(S, candidates, p, k_max, k_min=0):
        C = list(candidates)
        n = len(C)
        if n == 0:
            return [], np.zeros(0), np.zeros(0), 0, 0, 0
        s = np.array([S[j] for j in C])
        idx = np.lexsort((np.array(C), -s))
        order = [C[t] for t in idx]
        w = np.exp(s - s.max())
        mass = w[idx] / w.sum()
        cum = np.cumsum(mass)
        ph = O.p_hat(p)
        if ph <= 0:
            k_p = 0
        elif ph >= 1:
            k_p = n
        else:
            hit = np.nonzero(cum > ph)[0]          # mistake: strict
            k_p = int(hit[0]) + 1 if hit.size else n
        cap = min(k_max, n)
        return order, mass, cum, k_p, max(min(k_p, cap), min(k_min, n)), cap
    O.select_dynamic = select_dynamic


def m_kmax_caps_total(O):
    orig = O.select_decode

    def select_decode(S, n_sink, n_local, p, k_max, k_min=0):
        sel = orig(S, n_sink, n_local, p, k_max, k_min)
        sel.kept = sel.kept[:k_max] if len(sel.kept) > k_max else sel.kept
        return sel
    O.select_decode = select_decode


def m_p_as_float64(O):
    O.p_hat = lambda p: float(p)


def m_no_attn_scale(O):
    orig = O.attend
    O.attend = lambda q, K, V, scale: orig(q, K, V, 1.0)


def m_causal_strict(O):
    orig = O.attend_prefill_block

    def attend_prefill_block(q, q_pos, K, V, k_pos, scale):
        # mistake: a query does not see its own key (k < q instead of k <= q); the first
        # row has no key at all, so give it the previous behaviour to avoid NaN
        return orig(q, q_pos - 1 + (q_pos == q_pos.min()), K, V, k_pos, scale)
    O.attend_prefill_block = attend_prefill_block


def m_local_off_by_one(O):
    O.reserved_decode = lambda nb, n_sink, n_local: sorted(
        set(range(min(n_sink, nb))) | set(range(max(0, nb - n_local - 1), nb)))


def m_prefill_no_diagonal(O):
    O.reserved_prefill = lambda i, n_sink, n_local: sorted(
        set(range(min(n_sink, i))) | set(range(max(0, i - n_local), i)))


def m_lse_log2(O):
    orig = O.attend

    def attend(q, K, V, scale):
        o, lse = orig(q, K, V, scale)
        return o, lse / np.log(2.0)
    O.attend = attend


def m_scores_transposed_heads(O):
    """Uses the key's index dims against the wrong query head (head order rolled)."""
    orig = O.token_scores

    def token_scores(q, k, w, s):
        return orig(np.roll(q, 1, axis=0), k, w, s)
    O.token_scores = token_scores


MUTANTS = [m_block_mean, m_no_relu, m_reversed_weights, m_prefill_max_per_head,
           m_softmax_over_all_blocks, m_ties_higher_first, m_strict_greater, m_kmax_caps_total,
           m_p_as_float64, m_no_attn_scale, m_causal_strict, m_local_off_by_one,
           m_prefill_no_diagonal, m_lse_log2, m_scores_transposed_heads]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m.__name__)
def test_mutant_is_caught(mutant):
    O = fresh_oracle(mutant.__name__)
    mutant(O)
    failures = []
    for check in oracle_pins.ALL_CHECKS:
        try:
            check(O)
        except (AssertionError, ValueError, IndexError) as e:  # a pin noticed
            failures.append(check.__name__)
    assert failures, f"no pin catches {mutant.__name__}"
