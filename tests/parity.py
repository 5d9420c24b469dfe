"""Parity helpers: run the fp64 oracle on rows of a generated workload and compare
the CUDA path's outputs with it (test infrastructure).

Bars (the decode/prefill accuracy statement of the method's target):
* block selection identical, except a near-tie at the top-p / K_max boundary:
  the oracle's competing masses differ by less than 1e-6 relative; such rows are
  reported as ties and their attention is re-checked against the oracle run on
  the device's kept set;
* attention output (fp32 copy of the normalised output) max-abs <= 2e-3 and
  relative L2 <= 1e-3 against the oracle; the bf16 output equals the
  round-to-nearest-even of that fp32 copy bit for bit; |LSE error| <= 1e-4;
* block scores (fp32 on the device) within 1e-5 relative of the oracle's.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import bsa_oracle as O

TIE_REL = 1e-6
O_MAX_ABS = 2e-3
O_REL_L2 = 1e-3
LSE_ABS = 1e-4
SCORE_REL = 1e-5


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


# ------------------------------------------------------------------ tie rule
def classify_selection(sel: O.Selection, kept_dev, tol=TIE_REL):
    """'exact' | 'tie' | 'mismatch: ...' for a device kept list against the oracle."""
    kept_dev = [int(x) for x in kept_dev]
    if sorted(kept_dev) != kept_dev or len(set(kept_dev)) != len(kept_dev):
        return "mismatch: device list not strictly ascending"
    R, C = set(sel.reserved), set(sel.candidates)
    Kd = set(kept_dev)
    if not R <= Kd:
        return f"mismatch: reserved blocks missing {sorted(R - Kd)}"
    if not Kd <= (R | C):
        return f"mismatch: blocks outside the row {sorted(Kd - R - C)}"
    Dd = Kd - R
    k = sel.k
    Do = set(sel.order[:k])
    if Dd == Do:
        return "exact"
    pos = {j: t for t, j in enumerate(sel.order)}
    mass = {j: sel.mass[pos[j]] for j in sel.order}
    kd = len(Dd)
    if kd == k:
        mb = sel.mass[k - 1]
        bad = [j for j in (Do ^ Dd) if abs(mass[j] - mb) > tol * mb]
        return "tie" if not bad else f"mismatch: blocks {sorted(Do ^ Dd)} differ (masses {[mass[j] for j in sorted(Do ^ Dd)]}, boundary {mb})"
    if abs(kd - k) == 1:
        kk = min(k, kd)
        cum = sel.cum[kk - 1] if kk >= 1 else 0.0
        return ("tie-count", kk, cum, kd)
    return f"mismatch: {kd} dynamic blocks on the device, {k} in the oracle"


def selection_verdict(sel: O.Selection, kept_dev, p: float, tol=TIE_REL):
    r = classify_selection(sel, kept_dev, tol)
    if isinstance(r, tuple):       # count differs by one: cumulative mass at the cut ~ p
        _, kk, cum, kd = r
        ph = O.p_hat(p)
        if abs(cum - ph) > tol * ph:
            return f"mismatch: count {kd} vs {sel.k} and cumulative {cum} not within tie of {ph}"
        Dd = set(int(x) for x in kept_dev) - set(sel.reserved)
        ref = set(sel.order[:kd])
        pos = {j: t for t, j in enumerate(sel.order)}
        mb = sel.mass[kd - 1] if kd >= 1 else 0.0
        bad = [j for j in (ref ^ Dd) if abs(sel.mass[pos[j]] - mb) > tol * max(mb, 1e-300)]
        return "tie" if not bad else f"mismatch: count tie but blocks {sorted(ref ^ Dd)} differ"
    return r


# ------------------------------------------------------------------ attention bars
def attention_errors(o_f32_dev, o_bf16_dev, lse_dev, o_ref, lse_ref):
    """Returns dict of error measures; o_* numpy float64 arrays of the same shape."""
    o32 = np.asarray(o_f32_dev, dtype=np.float64)
    ref = np.asarray(o_ref, dtype=np.float64)
    max_abs = float(np.max(np.abs(o32 - ref))) if o32.size else 0.0
    rel_l2 = float(np.linalg.norm(o32 - ref) / max(np.linalg.norm(ref), 1e-300)) if o32.size else 0.0
    lse_d = np.asarray(lse_dev, dtype=np.float64)
    lse_r = np.asarray(lse_ref, dtype=np.float64)
    both_inf = np.isinf(lse_d) & np.isinf(lse_r) & (np.sign(lse_d) == np.sign(lse_r))
    diff = np.abs(np.where(both_inf, 0.0, lse_d) - np.where(both_inf, 0.0, lse_r))
    lse_err = float(np.max(diff)) if lse_d.size else 0.0
    return {"max_abs": max_abs, "rel_l2": rel_l2, "lse_abs": lse_err}


def bf16_is_rne_of_f32(o_bf16: torch.Tensor, o_f32: torch.Tensor) -> bool:
    return torch.equal(o_f32.to(torch.bfloat16).view(torch.int16), o_bf16.view(torch.int16))


def check_attention(errs, what=""):
    assert errs["max_abs"] <= O_MAX_ABS, f"{what}: max abs {errs['max_abs']}"
    assert errs["rel_l2"] <= O_REL_L2, f"{what}: rel L2 {errs['rel_l2']}"
    assert errs["lse_abs"] <= LSE_ABS, f"{what}: lse err {errs['lse_abs']}"


# ------------------------------------------------------------------ decode rows
def logical_rows(X: torch.Tensor, page_table, b: int, g: int, token_ids: np.ndarray):
    """Gather logical token rows (b, g, ids) of a contiguous or paged cache (any device)."""
    ids = torch.from_numpy(np.asarray(token_ids, dtype=np.int64)).to(X.device)
    if page_table is None:
        return X[b, g, ids]
    pages = page_table[b].long()[ids // 64]
    return X[pages, g, ids % 64]


def index_heads(inputs, w, b, g, tail):
    """Index queries and weights of group g: one index head per query head, or (with
    inputs["idx_heads"] == 1) one per group, whose weight defaults to 1."""
    if inputs.get("idx_heads", 0) == 1:
        qi = f64(inputs["q_idx"][(b, slice(g, g + 1)) + tail])
        hw = np.ones(1)
        return 1, qi, hw
    G = w.G
    qi = f64(inputs["q_idx"][(b, slice(g * G, (g + 1) * G)) + tail])
    return G, qi, f64(inputs["head_w"][g * G:(g + 1) * G])


def oracle_decode_row(w, inputs, b, g, kept_override=None):
    """Oracle decode for row (b, g), gathering only the tokens it needs."""
    G = w.G
    lens = inputs["seq_lens"]
    T_b = int(lens[b])
    q_g = f64(inputs["q"][b, g * G:(g + 1) * G])
    Gi, qi_g, hw = index_heads(inputs, w, b, g, (slice(None),))
    ki_g = f64(inputs["k_idx"][b, g, :T_b])
    S = O.decode_block_scores(qi_g, ki_g, T_b, hw, 1.0 / math.sqrt(w.r))
    sel = O.select_decode(S, w.n_sink, w.n_local, w.p, w.k_max, w.k_min)
    kept = sel.kept if kept_override is None else list(kept_override)
    ids = O.kept_token_ids(kept, T_b)
    K_tok = f64(logical_rows(inputs["K"], inputs.get("page_table"), b, g, ids))
    V_tok = f64(logical_rows(inputs["V"], inputs.get("page_table"), b, g, ids))
    o, lse = O.attend(q_g, K_tok, V_tok, 1.0 / math.sqrt(w.d))
    return {"S": S, "sel": sel, "o": o, "lse": lse, "kept": kept}


def compare_decode_rows(w, inputs, step, rows, p_override=None, check_scores=True):
    """Compare a finished DecodeStep with the oracle on the given (b, g) rows.
    check_scores=False for rows the scorer skips (local heads).

    Returns a summary dict; raises AssertionError on any bar violation."""
    G = w.G
    kept = step.kept.cpu()
    cnt = step.kept_count.cpu()
    scores = step.scores.cpu()
    o = step.o.cpu()
    o32 = step.o_f32.cpu()
    lse = step.lse.cpu()
    assert bf16_is_rne_of_f32(o, o32), "bf16 output is not RNE(fp32 output)"
    summary = {"rows": 0, "ties": 0, "max_abs": 0.0, "rel_l2": 0.0, "lse_abs": 0.0,
               "score_rel": 0.0}
    for (b, g) in rows:
        ref = oracle_decode_row(w, inputs, b, g)
        nb = len(ref["S"])
        S_dev = scores[b, g, :nb].double().numpy()
        if nb and check_scores:
            rel = np.max(np.abs(S_dev - ref["S"]) / np.maximum(1.0, np.abs(ref["S"])))
            summary["score_rel"] = max(summary["score_rel"], float(rel))
            assert rel <= SCORE_REL, f"row {(b, g)}: score rel err {rel}"
        c = int(cnt[b, g])
        kd = kept[b, g, :c].tolist()
        assert all(x == -1 for x in kept[b, g, c:].tolist()), "padding is not -1"
        verdict = selection_verdict(ref["sel"], kd, w.p)
        assert not verdict.startswith("mismatch"), f"row {(b, g)}: {verdict}"
        if verdict == "tie":
            summary["ties"] += 1
            ref = oracle_decode_row(w, inputs, b, g, kept_override=kd)
        errs = attention_errors(o32[b, g * G:(g + 1) * G].double().numpy(), None,
                                lse[b, g * G:(g + 1) * G].double().numpy(), ref["o"], ref["lse"])
        check_attention(errs, f"row {(b, g)}")
        for k_ in ("max_abs", "rel_l2", "lse_abs"):
            summary[k_] = max(summary[k_], errs[k_])
        summary["rows"] += 1
    return summary


# ------------------------------------------------------------------ prefill rows
def oracle_prefill_rows(w, inputs, b, g, rows, kept_override=None):
    G = w.G
    T = w.T
    q_g = f64(inputs["q"][b, g * G:(g + 1) * G, :T])
    _, qi_g, hw = index_heads(inputs, w, b, g, (slice(0, T),))
    ki_g = f64(inputs["k_idx"][b, g, :T])
    K_g = f64(inputs["K"][b, g, :T])
    V_g = f64(inputs["V"][b, g, :T])
    return O.prefill_rows(q_g, qi_g, ki_g, K_g, V_g, T, hw, 1.0 / math.sqrt(w.r),
                          1.0 / math.sqrt(w.d), w.n_sink, w.n_local, w.p, w.k_max, w.k_min,
                          rows=rows, kept_override=kept_override)


def _check_prefill_block(w, o32, lse, b, g, i, ref, summary):
    G, T = w.G, w.T
    q0, q1 = i * 64, min(i * 64 + 64, T)
    o32_blk = o32[b, g * G:(g + 1) * G, q0:q1].double().numpy()
    lse_blk = lse[b, g * G:(g + 1) * G, q0:q1].double().numpy()
    errs = attention_errors(o32_blk, None, lse_blk, ref["o"], ref["lse"])
    check_attention(errs, f"prefill row {(b, g, i)}")
    for k_ in ("max_abs", "rel_l2", "lse_abs"):
        summary[k_] = max(summary[k_], errs[k_])
    summary["rows"] += 1


def compare_prefill_rows(w, inputs, pf, b, g, rows, check_scores=True, kept_dev=None,
                         attend_lists=None):
    """Compare a finished Prefill with the oracle on query blocks ``rows`` of (b, g).

    kept_dev: {i: list} kept lists the selection produced, when pf.kept was changed
    afterwards (default: pf.kept). attend_lists: {i: list} kept lists the attention
    is to be checked against (default: the selected set, or the device's set when
    the tie rule accepted it)."""
    kept = pf.kept.cpu()
    cnt = pf.kept_count.cpu()
    scores = pf.scores.cpu()
    o = pf.o.cpu()
    o32 = pf.o_f32.cpu()
    lse = pf.lse.cpu()
    summary = {"rows": 0, "ties": 0, "max_abs": 0.0, "rel_l2": 0.0, "lse_abs": 0.0,
               "score_rel": 0.0}
    refs = oracle_prefill_rows(w, inputs, b, g, rows)
    override = dict(attend_lists or {})
    for i, ref in refs.items():
        if i and check_scores:
            S_dev = scores[b, g, i, :i].double().numpy()
            rel = np.max(np.abs(S_dev - ref["S"]) / np.maximum(1.0, np.abs(ref["S"])))
            summary["score_rel"] = max(summary["score_rel"], float(rel))
            assert rel <= SCORE_REL, f"prefill row {(b, g, i)}: score rel err {rel}"
        if kept_dev is not None and i in kept_dev:
            kd = list(kept_dev[i])
        else:
            c = int(cnt[b, g, i])
            kd = kept[b, g, i, :c].tolist()
            assert all(x == -1 for x in kept[b, g, i, c:].tolist()), "padding is not -1"
        verdict = selection_verdict(ref["sel"], kd, w.p)
        assert not verdict.startswith("mismatch"), f"prefill row {(b, g, i)}: {verdict}"
        if verdict == "tie":
            summary["ties"] += 1
            override.setdefault(i, kd)
    if override:
        refs.update(oracle_prefill_rows(w, inputs, b, g, list(override), kept_override=override))
    for i, ref in refs.items():
        _check_prefill_block(w, o32, lse, b, g, i, ref, summary)
    G = w.G
    assert bf16_is_rne_of_f32(o[b, g * G:(g + 1) * G], o32[b, g * G:(g + 1) * G])
    return summary


# ------------------------------------------------------------------ PBS prefill rows
IMP_TIE_REL = 1e-4   # importances this close (relative) may be ordered either way


def permutation_verdict(imp, perm_dev, seg):
    """'exact' | 'tie' | 'mismatch: ...' for a device key order against the oracle's
    importances: every segment must hold its own positions, in an order whose
    importance never rises by more than IMP_TIE_REL (relative) from one key to the
    next, and keys of equal importance ordered by position."""
    perm_dev = np.asarray(perm_dev, dtype=np.int64)
    T = len(imp)
    exact = True
    for s0 in range(0, T, seg):
        s1 = min(s0 + seg, T)
        block = perm_dev[s0:s1]
        if sorted(block.tolist()) != list(range(s0, s1)):
            return f"mismatch: segment {s0} is not a permutation of its positions"
        v = imp[block]
        rise = v[1:] - v[:-1]
        tol = np.maximum(IMP_TIE_REL * np.maximum(np.abs(v[1:]), np.abs(v[:-1])), 1e-30)
        if np.any(rise > tol):
            return f"mismatch: importance rises in segment {s0}"
        eq = (v[1:] == v[:-1])
        if np.any(eq & (block[1:] < block[:-1])):
            return f"mismatch: equal importance out of position order in segment {s0}"
        order = np.lexsort((np.arange(s0, s1), -imp[s0:s1]))
        exact = exact and np.array_equal(block, np.arange(s0, s1)[order])
    return "exact" if exact else "tie"


def compare_pbs_rows(w, inputs, pbs, b, g, rows, seg):
    """Compare a finished PbsPrefill with the PBS oracle on query blocks ``rows`` of
    (b, g): key order (tie rule on importance), block scores of the earlier
    segments, kept sets (tie rule on mass), attention."""
    from oracle import pbs_oracle as P
    G, T = w.G, w.T
    q_g = f64(inputs["q"][b, g * G:(g + 1) * G, :T])
    _, qi_g, hw = index_heads(inputs, w, b, g, (slice(0, T),))
    ki_g = f64(inputs["k_idx"][b, g, :T])
    K_g = f64(inputs["K"][b, g, :T])
    V_g = f64(inputs["V"][b, g, :T])
    args = (q_g, qi_g, ki_g, K_g, V_g, T, seg, hw, 1.0 / math.sqrt(w.r), 1.0 / math.sqrt(w.d),
            w.n_sink, w.n_local, w.p, w.k_max, w.k_min)
    summary = {"rows": 0, "ties": 0, "perm": "exact", "max_abs": 0.0, "rel_l2": 0.0,
               "lse_abs": 0.0, "score_rel": 0.0}
    kp = pbs.key_pos[b, g].cpu().numpy().astype(np.int64)
    imp = P.last_block_importance(q_g, K_g, T, 1.0 / math.sqrt(w.d))
    verdict = permutation_verdict(imp, kp, seg)
    assert not verdict.startswith("mismatch"), f"key order of {(b, g)}: {verdict}"
    summary["perm"] = verdict
    perm, refs = P.pbs_prefill_rows(*args, rows=rows, perm_override=kp)
    kept = pbs.pf.kept.cpu()
    cnt = pbs.pf.kept_count.cpu()
    scores = pbs.pf.scores.cpu()
    o32 = pbs.pf.o_f32.cpu()
    lse = pbs.pf.lse.cpu()
    override = {}
    for i, ref in refs.items():
        nS = len(ref["S"])
        if nS:
            S_dev = scores[b, g, i, :nS].double().numpy()
            rel = np.max(np.abs(S_dev - ref["S"]) / np.maximum(1.0, np.abs(ref["S"])))
            summary["score_rel"] = max(summary["score_rel"], float(rel))
            assert rel <= SCORE_REL, f"PBS row {(b, g, i)}: score rel err {rel}"
        c = int(cnt[b, g, i])
        kd = kept[b, g, i, :c].tolist()
        assert all(x == -1 for x in kept[b, g, i, c:].tolist()), "padding is not -1"
        v = selection_verdict(ref["sel"], kd, w.p)
        assert not v.startswith("mismatch"), f"PBS row {(b, g, i)}: {v}"
        if v == "tie":
            summary["ties"] += 1
            override[i] = kd
    if override:
        _, more = P.pbs_prefill_rows(*args, rows=list(override), kept_override=override,
                                     perm_override=kp)
        refs.update(more)
    for i, ref in refs.items():
        _check_prefill_block(w, o32, lse, b, g, i, ref, summary)
    return summary


# ------------------------------------------------------------------ two-level (HGA) decode rows
GROUP_TIE_REL = 1e-5   # group scores this close (relative) may rank either way


def group_verdict(Sg, cand, groups_ref, groups_dev, k_groups, tol=GROUP_TIE_REL):
    """'exact' | 'tie' | 'mismatch: ...' for the device's kept groups: the right
    number of candidate groups, and any difference to the oracle's choice lies at
    the boundary score (within tol relative)."""
    Dd, Do = set(groups_dev), set(groups_ref)
    if not Dd <= set(cand):
        return f"mismatch: groups outside the candidates {sorted(Dd - set(cand))}"
    if len(Dd) != min(k_groups, len(cand)):
        return f"mismatch: {len(Dd)} groups on the device, {min(k_groups, len(cand))} expected"
    if Dd == Do:
        return "exact"
    sb = min(Sg[c] for c in Do)
    bad = [c for c in Dd ^ Do if abs(Sg[c] - sb) > tol * max(1.0, abs(sb))]
    return "tie" if not bad else f"mismatch: groups {sorted(Dd ^ Do)} differ (boundary {sb})"


def compare_hga_rows(w, inputs, step, rows, gs, k_groups):
    """Compare a finished two-level DecodeStep with the HGA oracle on (b, g) rows:
    block scores, group scores, kept blocks (tie rule on mass), kept groups (tie rule
    on score), the masks of the always-visible entries, attention."""
    from oracle import hga_oracle as H
    G = w.G
    gpb = 64 // gs
    kept, cnt = step.kept.cpu(), step.kept_count.cpu()
    scores, gsc = step.scores.cpu(), step.group_scores.cpu()
    masks = step.kept_groups.cpu()
    o, o32, lse = step.o.cpu(), step.o_f32.cpu(), step.lse.cpu()
    assert bf16_is_rne_of_f32(o, o32), "bf16 output is not RNE(fp32 output)"
    summary = {"rows": 0, "ties": 0, "group_ties": 0, "max_abs": 0.0, "rel_l2": 0.0,
               "lse_abs": 0.0, "score_rel": 0.0, "groups": 0}
    pt = inputs.get("page_table")
    for (b, g) in rows:
        T_b = int(inputs["seq_lens"][b])
        q_g = f64(inputs["q"][b, g * G:(g + 1) * G])
        _, qi_g, hw = index_heads(inputs, w, b, g, (slice(None),))
        ki_g = f64(inputs["k_idx"][b, g, :T_b])
        ids = np.arange(T_b)
        K_g = f64(logical_rows(inputs["K"], pt, b, g, ids))
        V_g = f64(logical_rows(inputs["V"], pt, b, g, ids))
        args = (q_g, qi_g, ki_g, K_g, V_g, T_b, hw, 1.0 / math.sqrt(w.r), 1.0 / math.sqrt(w.d),
                w.n_sink, w.n_local, w.p, w.k_max, gs, k_groups, w.k_min)
        ref = H.hga_decode_row(*args)
        nb = len(ref["S"])
        if nb:
            S_dev = scores[b, g, :nb].double().numpy()
            rel = np.max(np.abs(S_dev - ref["S"]) / np.maximum(1.0, np.abs(ref["S"])))
            ng = len(ref["Sg"])
            Sg_dev = gsc[b, g, :ng].double().numpy()
            grel = np.max(np.abs(Sg_dev - ref["Sg"]) / np.maximum(1.0, np.abs(ref["Sg"])))
            summary["score_rel"] = max(summary["score_rel"], float(rel), float(grel))
            assert rel <= SCORE_REL, f"row {(b, g)}: block score rel err {rel}"
            assert grel <= SCORE_REL, f"row {(b, g)}: group score rel err {grel}"
            tail = gsc[b, g, ng:nb * gpb]
            assert bool(torch.all(tail == float("-inf"))), "groups past the end are not -inf"
        c = int(cnt[b, g])
        kd = kept[b, g, :c].tolist()
        v = selection_verdict(ref["sel"], kd, w.p)
        assert not v.startswith("mismatch"), f"row {(b, g)}: {v}"
        if v == "tie":
            summary["ties"] += 1
            ref = H.hga_decode_row(*args, kept_override=kd)
        m = [int(x) & 0xffffffff for x in masks[b, g].tolist()]
        full = (1 << gpb) - 1
        R = set(ref["sel"].reserved)
        gdev = []
        for e, j in enumerate(kd):
            if j in R:
                assert m[e] == full, f"row {(b, g)}: always-visible block {j} mask {m[e]:#x}"
            else:
                assert m[e] >> gpb == 0, f"row {(b, g)}: mask {m[e]:#x} has bits past the block"
                gdev += [j * gpb + k for k in range(gpb) if (m[e] >> k) & 1]
        assert all(x == 0 for x in m[c:]), f"row {(b, g)}: masks past the count are not 0"
        gv = group_verdict(ref["Sg"], ref["cand"], ref["groups"], gdev, k_groups)
        assert not gv.startswith("mismatch"), f"row {(b, g)}: {gv}"
        if gv == "tie":
            summary["group_ties"] += 1
            ref = H.hga_decode_row(*args, kept_override=kd, groups_override=gdev)
        errs = attention_errors(o32[b, g * G:(g + 1) * G].double().numpy(), None,
                                lse[b, g * G:(g + 1) * G].double().numpy(), ref["o"], ref["lse"])
        check_attention(errs, f"row {(b, g)}")
        for k_ in ("max_abs", "rel_l2", "lse_abs"):
            summary[k_] = max(summary[k_], errs[k_])
        summary["rows"] += 1
        summary["groups"] += len(gdev)
    return summary
