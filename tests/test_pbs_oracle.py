"""The PBS oracle (segment-permuted prefill) against its pins, and planted mistakes in
copies of it that the pins must catch. CPU only."""
import importlib.util
import os
import sys

import numpy as np
import pytest

from oracle import pbs_oracle as P
from tests import pbs_pins

PBS_PATH = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "pbs_oracle.py")


@pytest.mark.parametrize("check", pbs_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_pbs_oracle_pin(check):
    check(P)


def fresh(tag):
    spec = importlib.util.spec_from_file_location(f"pbs_oracle_mutant_{tag}", PBS_PATH)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    return mod


def m_ascending(M):
    def segment_permutation(imp, seg):
        T = len(imp)
        perm = np.empty(T, dtype=np.int64)
        for s0 in range(0, T, seg):
            pos = np.arange(s0, min(s0 + seg, T))
            perm[s0:s0 + len(pos)] = pos[np.lexsort((pos, imp[s0:s0 + len(pos)]))]
        return perm
    M.segment_permutation = segment_permutation


def m_global_sort(M):
    orig = M.segment_permutation
    M.segment_permutation = lambda imp, seg: orig(imp, len(imp))


def m_ties_high_first(M):
    def segment_permutation(imp, seg):
        T = len(imp)
        perm = np.empty(T, dtype=np.int64)
        for s0 in range(0, T, seg):
            pos = np.arange(s0, min(s0 + seg, T))
            perm[s0:s0 + len(pos)] = pos[np.lexsort((-pos, -imp[s0:s0 + len(pos)]))]
        return perm
    M.segment_permutation = segment_permutation


def m_importance_max(M):
    def key_importance(q_last, q_pos, K, scale):
        T = K.shape[0]
        s = np.einsum("gqd,kd->gqk", q_last, K) * scale
        vis = np.arange(T)[None, None, :] <= q_pos[None, :, None]
        s = np.where(vis, s, -np.inf)
        e = np.where(vis, np.exp(s - s.max(axis=2, keepdims=True)), 0.0)
        return (e / e.sum(axis=2, keepdims=True)).max(axis=(0, 1))
    M.key_importance = key_importance


def m_importance_no_mask(M):
    def key_importance(q_last, q_pos, K, scale):
        s = np.einsum("gqd,kd->gqk", q_last, K) * scale
        e = np.exp(s - s.max(axis=2, keepdims=True))
        return (e / e.sum(axis=2, keepdims=True)).mean(axis=(0, 1))
    M.key_importance = key_importance


def m_importance_raw_scores(M):
    def key_importance(q_last, q_pos, K, scale):
        return (np.einsum("gqd,kd->gqk", q_last, K) * scale).mean(axis=(0, 1))
    M.key_importance = key_importance


def m_own_segment_diagonal_only(M):
    O = M.O

    def reserved_pbs(i, seg_blocks, nqb, n_sink, n_local):
        b0, _ = M.segment_blocks(i, seg_blocks, nqb)
        return sorted({i} | set(range(min(n_sink, i + 1))) | set(range(max(0, b0 - n_local), b0)))
    M.reserved_pbs = reserved_pbs


def m_local_before_block(M):
    def reserved_pbs(i, seg_blocks, nqb, n_sink, n_local):
        b0, b1 = M.segment_blocks(i, seg_blocks, nqb)
        return sorted(set(range(b0, b1)) | set(range(min(n_sink, b1))) |
                      set(range(max(0, i - n_local), i)))
    M.reserved_pbs = reserved_pbs


def m_mask_by_permuted_position(M):
    O = M.O
    orig = O.attend_prefill_block

    def pbs_rows(q_g, q_idx_g, k_idx_g, K_g, V_g, T, seg, head_w, idx_scale, attn_scale,
                 n_sink, n_local, p, k_max, k_min=0, rows=None, kept_override=None):
        # the causal mask taken on the permuted positions instead of the original ones
        saved = O.attend_prefill_block
        perm_holder = {}

        def attend(qb, q_pos, Kt, Vt, k_pos, scale):
            inv = perm_holder["inv"]
            return saved(qb, q_pos, Kt, Vt, inv[k_pos], scale)
        ql = np.arange((O.num_blocks(T) - 1) * 64, T)
        imp = M.key_importance(q_g[:, ql, :], ql, K_g[:T], attn_scale)
        perm = M.segment_permutation(imp, seg)
        inv = np.empty_like(perm)
        inv[perm] = np.arange(len(perm))
        perm_holder["inv"] = inv
        O.attend_prefill_block = attend
        try:
            return M._orig_rows(q_g, q_idx_g, k_idx_g, K_g, V_g, T, seg, head_w, idx_scale,
                                attn_scale, n_sink, n_local, p, k_max, k_min, rows, kept_override)
        finally:
            O.attend_prefill_block = saved
    M._orig_rows = M.pbs_prefill_rows
    M.pbs_prefill_rows = pbs_rows


def m_scores_unpermuted(M):
    O = M.O
    saved = M.segment_permutation

    def pbs_rows(*args, **kw):
        # block scores from the keys in natural order; attention still permuted
        real_perm = {}
        M.segment_permutation = lambda imp, seg: real_perm.setdefault("p", saved(imp, seg))
        return M._orig_rows2(*args, **kw)
    M._orig_rows2 = M.pbs_prefill_rows

    def rows_natural_scores(q_g, q_idx_g, k_idx_g, K_g, V_g, T, seg, head_w, idx_scale,
                            attn_scale, n_sink, n_local, p, k_max, k_min=0, rows=None,
                            kept_override=None):
        perm, out = M._orig_rows2(q_g, q_idx_g, k_idx_g, K_g, V_g, T, seg, head_w, idx_scale,
                                  attn_scale, n_sink, n_local, p, k_max, k_min, rows,
                                  kept_override)
        for i, r in out.items():
            b0, _ = M.segment_blocks(i, seg // 64, O.num_blocks(T))
            if b0 > 0:
                u = O.token_scores(q_idx_g[:, i * 64:min(i * 64 + 64, T), :], k_idx_g[:b0 * 64],
                                   head_w, idx_scale)
                r["S"] = np.array([u[:, j * 64:(j + 1) * 64].max() for j in range(b0)])
        return perm, out
    M.pbs_prefill_rows = rows_natural_scores


MUTANTS = [m_ascending, m_global_sort, m_ties_high_first, m_importance_max, m_importance_no_mask,
           m_importance_raw_scores, m_own_segment_diagonal_only, m_local_before_block,
           m_mask_by_permuted_position, m_scores_unpermuted]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m.__name__)
def test_pbs_mutant_is_caught(mutant):
    M = fresh(mutant.__name__)
    mutant(M)
    caught = []
    for check in pbs_pins.ALL_CHECKS:
        try:
            check(M)
        except (AssertionError, ValueError, IndexError):
            caught.append(check.__name__)
    assert caught, f"{mutant.__name__} passes every pin"
