"""The two-level routing oracle against its pins, and planted mistakes in copies of it
that the pins must catch. CPU only."""
import importlib.util
import os
import sys

import numpy as np
import pytest

from oracle import hga_oracle as H
from tests import hga_pins

HGA_PATH = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "hga_oracle.py")


@pytest.mark.parametrize("check", hga_pins.ALL_CHECKS, ids=lambda c: c.__name__)
def test_hga_oracle_pin(check):
    check(H)


def fresh(tag):
    spec = importlib.util.spec_from_file_location(f"hga_oracle_mutant_{tag}", HGA_PATH)
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    return mod


def m_group_mean(M):
    O = M.O

    def group_scores(q, k, T, w, s, gs):
        u = O.token_scores(q, k[:T], w, s)
        return np.array([u[c * gs:min((c + 1) * gs, T)].mean() for c in range((T + gs - 1) // gs)])
    M.group_scores = group_scores


def m_ties_high_first(M):
    def select_groups(sel, Sg, T, gs, k_groups):
        gpb = 64 // gs
        R = set(sel.reserved)
        cand = [j * gpb + k for j in sel.kept if j not in R for k in range(gpb) if (j * gpb + k) * gs < T]
        if not cand:
            return [], []
        s = np.array([Sg[c] for c in cand])
        order = [cand[t] for t in np.lexsort((-np.array(cand), -s))]
        return cand, sorted(order[:k_groups])
    M.select_groups = select_groups


def m_reserved_compete(M):
    def select_groups(sel, Sg, T, gs, k_groups):
        gpb = 64 // gs
        cand = [j * gpb + k for j in sel.kept for k in range(gpb) if (j * gpb + k) * gs < T]
        s = np.array([Sg[c] for c in cand])
        order = [cand[t] for t in np.lexsort((np.array(cand), -s))]
        return cand, sorted(order[:k_groups])
    M.select_groups = select_groups


def m_last_groups(M):
    def select_groups(sel, Sg, T, gs, k_groups):
        gpb = 64 // gs
        R = set(sel.reserved)
        cand = [j * gpb + k for j in sel.kept if j not in R for k in range(gpb) if (j * gpb + k) * gs < T]
        if not cand:
            return [], []
        s = np.array([Sg[c] for c in cand])
        order = [cand[t] for t in np.lexsort((np.array(cand), -s))]
        return cand, sorted(order[-k_groups:])
    M.select_groups = select_groups


def m_group_off_by_one(M):
    def routed_tokens(sel, kept_groups, T, gs):
        ids = [np.arange(j * 64, min((j + 1) * 64, T)) for j in sel.reserved]
        ids += [np.arange(c * gs + 1, min((c + 1) * gs + 1, T)) for c in kept_groups]
        return np.sort(np.concatenate(ids)) if ids else np.zeros(0, dtype=np.int64)
    M.routed_tokens = routed_tokens


def m_ghost_groups(M):
    def select_groups(sel, Sg, T, gs, k_groups):
        gpb = 64 // gs
        R = set(sel.reserved)
        cand = [j * gpb + k for j in sel.kept if j not in R for k in range(gpb)]
        Sg2 = np.concatenate([Sg, np.zeros(max(0, max(cand, default=0) + 1 - len(Sg)))])
        s = np.array([Sg2[c] for c in cand])
        order = [cand[t] for t in np.lexsort((np.array(cand), -s))]
        return cand, sorted(order[:k_groups])
    M.select_groups = select_groups


MUTANTS = [m_group_mean, m_ties_high_first, m_reserved_compete, m_last_groups,
           m_group_off_by_one, m_ghost_groups]


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda m: m.__name__)
def test_hga_mutant_is_caught(mutant):
    M = fresh(mutant.__name__)
    mutant(M)
    caught = []
    for check in hga_pins.ALL_CHECKS:
        try:
            check(M)
        except (AssertionError, ValueError, IndexError):
            caught.append(check.__name__)
    assert caught, f"{mutant.__name__} passes every pin"
