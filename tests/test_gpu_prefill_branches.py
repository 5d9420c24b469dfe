"""Prefill attention branches that N(0, 1) inputs never reach, checked against the
fp64 oracle through the C ABI:

* the rescale of O in tensor memory. The kernel moves a row's running max only
  when a step's block max exceeds it by more than 8 (log2 units), and then scales
  the O rows accumulated so far, after the previous P.V has completed. On random
  inputs no row grows that much after its first kept block, so these tests plant
  keys aligned with chosen queries in later kept blocks (or raise the softmax
  scale), replay the kernel's visiting order on the fp64 scores to count the
  rescales that must happen, and require at least one;
* kept blocks that fail validation: a kept id outside [0, i] and a page id outside
  the pool. The step is skipped (its keys masked), the status bit is set, and
  every row matches the oracle run on its kept set without that block (HGA,
  Central mechanism §4: exact softmax over the tokens actually routed).
"""
import math

import numpy as np
import pytest
import torch

import block_sparse_long_06_b200 as bsa
from block_sparse_long_06_b200 import workloads as W
from oracle import bsa_oracle as O
from tests import parity

pytestmark = pytest.mark.gpu

LOG2E = 1.4426950408889634
GROWTH = 8.0   # log2 units by which a row's running max must grow before it moves


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def to_dev(inputs):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inputs.items()}


def run_prefill(w, xd, attn_scale=None, k=None, v=None, expect_status=0):
    prob = bsa.problem_for(w, head_w=xd["head_w"])
    if attn_scale is not None:
        prob.attn_scale = attn_scale
    pf = bsa.Prefill(prob)
    K = k if k is not None else bsa.contiguous_cache(xd["K"])
    V = v if v is not None else bsa.contiguous_cache(xd["V"])
    pf.run(xd["q"], xd["q_idx"], bsa.contiguous_cache(xd["k_idx"]), K, V)
    torch.cuda.synchronize()
    st = int(pf.status.item())
    assert st == expect_status, f"device status {st:#x}, expected {expect_status:#x}"
    return pf


def rescale_events(w, x, pf, b, g, rows, attn_scale, margin=1.0):
    """Replay of the kernel's order on fp64 scores for query blocks ``rows`` of (b, g):
    each row visits its kept blocks in list order, starting from max = -inf, and moves
    its max when a block's max (log2 units, causal keys only) exceeds it by more than
    8. Returns how many (row, step > 0) moves clear the threshold by more than
    ``margin`` (the kernel rescales there whatever its fp32 rounding)."""
    G, T = w.G, w.T
    kept = pf.kept.cpu()
    cnt = pf.kept_count.cpu()
    sure = 0
    for i in rows:
        q0, q1 = i * 64, min(i * 64 + 64, T)
        q = parity.f64(x["q"][b, g * G:(g + 1) * G, q0:q1])          # [G, nq, d]
        m = np.full(q.shape[:2], -np.inf)
        for jj, j in enumerate(kept[b, g, i, :int(cnt[b, g, i])].tolist()):
            k0, k1 = j * 64, min(j * 64 + 64, T)
            s = q @ parity.f64(x["K"][b, g, k0:k1]).T * (attn_scale * LOG2E)
            vis = np.arange(k0, k1)[None, None, :] <= np.arange(q0, q1)[None, :, None]
            xm = np.where(vis, s, -np.inf).max(axis=2)
            if jj > 0:
                sure += int(np.sum(np.isfinite(m) & (xm - m > GROWTH + margin)))
            m = np.where(xm > m + GROWTH, xm, m)
    return sure


def plant_growing_keys(w, x, targets, amps=(12.0, 20.0, 28.0)):
    """For each (g, i, h, tq): the key at one token of blocks i-2, i-1 and i (two local
    blocks and the diagonal, all kept, visited last and in this order) becomes
    bf16(a * q_hat), q_hat the unit query of head h at tq, with growing amplitudes a.
    A planted key scores about 1.44 a log2 units for that row, and each jump is about
    1.44 * 8 = 11.5 units above the last, so the row rescales O three times after its
    first kept block (whose max is about 3-5 units). Index keys are left as they were (the
    selection does not depend on this), so the oracle sees the same inputs."""
    G = w.G
    for (g, i, h, tq) in targets:
        assert i >= 2 and i * 64 + 1 <= tq < min(i * 64 + 64, w.T)
        qv = x["q"][0, g * G + h, tq].float()
        qhat = qv / qv.norm()
        for blk, off, a in zip((i - 2, i - 1, i), (7, 40, 1), amps):
            x["K"][0, g, blk * 64 + off] = (a * qhat).to(torch.bfloat16)


SMALL = W.Workload("small_prefill", "prefill", B=1, Hq=8, Hkv=2, d=128, T=64 * 12 + 5,
                   n_sink=1, n_local=2, p=1.0, k_max=3, hh_count=32, amp=3.0, seed=11)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 4, 8])
def test_prefill_rescale_of_o_in_tensor_memory(d, G):
    w = SMALL.with_(d=d, Hq=2 * G, Hkv=2)
    x = W.make_prefill_inputs(w, "cpu")
    targets = [(0, 4, 0, 4 * 64 + 50), (0, 9, G - 1, 9 * 64 + 17), (1, 7, G // 2, 7 * 64 + 63),
               (1, 11, 0, 11 * 64 + 3)]
    plant_growing_keys(w, x, targets)
    pf = run_prefill(w, to_dev(x))
    scale = 1.0 / math.sqrt(d)
    events = 0
    for g in range(w.Hkv):
        events += rescale_events(w, x, pf, 0, g, range(w.nb), scale)
        s = parity.compare_prefill_rows(w, x, pf, 0, g, list(range(w.nb)))
        print(f"d={d} G={G} g={g}", s)
    assert events >= 3 * len(targets), f"only {events} sure rescales"


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_rescale_with_a_large_softmax_scale(d):
    """A softmax scale of 1 (instead of 1/sqrt(d)) spreads each row's scores over tens
    of log2 units, so running maxima move often without planted keys."""
    w = SMALL.with_(d=d, T=64 * 10 + 33)
    x = W.make_prefill_inputs(w, "cpu")
    pf = run_prefill(w, to_dev(x), attn_scale=1.0)
    events = 0
    for g in range(w.Hkv):
        events += rescale_events(w, x, pf, 0, g, range(w.nb), 1.0)
        refs = parity.oracle_prefill_rows(w, x, 0, g, list(range(w.nb)))
        # the oracle at the same softmax scale
        G = w.G
        q_g = parity.f64(x["q"][0, g * G:(g + 1) * G, :w.T])
        K_g = parity.f64(x["K"][0, g, :w.T])
        V_g = parity.f64(x["V"][0, g, :w.T])
        o32 = pf.o_f32.cpu()
        lse = pf.lse.cpu()
        for i, ref in refs.items():
            kd = pf.kept[0, g, i, :int(pf.kept_count[0, g, i])].tolist()
            assert not parity.selection_verdict(ref["sel"], kd, w.p).startswith("mismatch")
            q_pos = np.arange(i * 64, min(i * 64 + 64, w.T))
            k_pos = O.kept_token_ids(kd, w.T)
            o_ref, lse_ref = O.attend_prefill_block(q_g[:, q_pos, :], q_pos, K_g[k_pos],
                                                    V_g[k_pos], k_pos, 1.0)
            errs = parity.attention_errors(o32[0, g * G:(g + 1) * G, q_pos].double().numpy(),
                                           None, lse[0, g * G:(g + 1) * G, q_pos].double().numpy(),
                                           o_ref, lse_ref)
            parity.check_attention(errs, f"scale 1, row {(g, i)}")
    assert events > 0


def test_prefill_rescale_at_64k():
    """The 64K workload with growing keys planted for rows of two kv heads."""
    w = W.WORKLOADS["prefill_b1_h32_t64k"]
    x = W.make_prefill_inputs(w, "cuda")
    targets = [(0, 100, 1, 100 * 64 + 50), (0, 1023, 3, 1023 * 64 + 10),
               (5, 600, 2, 600 * 64 + 63), (5, 67, 0, 67 * 64 + 1)]
    plant_growing_keys(w, x, targets)
    pf = run_prefill(w, x)
    events = 0
    for g in (0, 5):
        rows = sorted({t[1] for t in targets if t[0] == g} | {0, 1, 2, 3, 68, 69})
        events += rescale_events(w, x, pf, 0, g, rows, 1.0 / math.sqrt(w.d))
        s = parity.compare_prefill_rows(w, x, pf, 0, g, rows)
        print("64K planted", g, s)
    assert events >= 3 * len(targets), f"only {events} sure rescales"
    del x, pf
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ failed validation
def test_prefill_bad_kept_ids_are_skipped_and_reported():
    w = SMALL.with_(T=64 * 14 + 9, k_max=4)
    x = W.make_prefill_inputs(w, "cpu")
    xd = to_dev(x)
    prob = bsa.problem_for(w, head_w=xd["head_w"])
    pf = bsa.Prefill(prob)
    pf.select(xd["q_idx"], bsa.contiguous_cache(xd["k_idx"]))
    torch.cuda.synchronize()
    selected = {}
    for g in range(w.Hkv):
        selected[g] = {i: pf.kept[0, g, i, :int(pf.kept_count[0, g, i])].tolist()
                       for i in range(w.nb)}
    # (g, i, slot, bad id): past the diagonal, negative, far outside
    bad = [(0, 6, 1, 7), (0, 10, 0, -3), (1, 13, 2, 10 ** 6), (1, 5, 1, 14)]
    for g, i, slot, bid in bad:
        pf.kept[0, g, i, slot] = bid
    pf.attend(xd["q"], bsa.contiguous_cache(xd["K"]), bsa.contiguous_cache(xd["V"]))
    torch.cuda.synchronize()
    assert int(pf.status.item()) == bsa.BSA_DEV_BAD_KEPT
    for g in range(w.Hkv):
        lists = {}
        for gg, i, slot, bid in bad:
            if gg == g:
                lists[i] = [j for t, j in enumerate(selected[g][i]) if t != slot]
        s = parity.compare_prefill_rows(w, x, pf, 0, g, list(range(w.nb)),
                                        kept_dev=selected[g], attend_lists=lists)
        print("bad kept", g, s)


def paged_pool(X: torch.Tensor, seed: int):
    """[1, Hkv, T, d] contiguous -> ([nb, Hkv, 64, d] pool, [1, nb] shuffled page table)."""
    _, H, T, d = X.shape
    nb = (T + 63) // 64
    pt = torch.randperm(nb, generator=torch.Generator().manual_seed(seed)).to(torch.int32)
    pool = torch.zeros(nb, H, 64, d, dtype=X.dtype)
    for j in range(nb):
        n = min(64, T - j * 64)
        pool[pt[j], :, :n] = X[0, :, j * 64:j * 64 + n]
    return pool, pt.view(1, nb).contiguous()


def test_prefill_paged_cache_and_bad_page():
    w = SMALL.with_(T=64 * 12 + 40, k_max=3)
    x = W.make_prefill_inputs(w, "cpu")
    xd = to_dev(x)
    Kp, pt = paged_pool(x["K"], 3)
    Vp, _ = paged_pool(x["V"], 3)
    Kp, Vp, pt = Kp.cuda(), Vp.cuda(), pt.cuda()
    # a paged cache gives the same result as the contiguous one, bit for bit
    ref = run_prefill(w, xd)
    pg = run_prefill(w, xd, k=bsa.paged_cache(Kp, pt), v=bsa.paged_cache(Vp, pt))
    for a, b in ((ref.o, pg.o), (ref.o_f32, pg.o_f32), (ref.lse, pg.lse), (ref.kept, pg.kept)):
        assert torch.equal(a, b)
    # block 5 behind a page id outside the pool: its keys are skipped wherever it is kept
    bad_blk = 5
    pt_bad = pt.clone()
    pt_bad[0, bad_blk] = Kp.shape[0] + 1000
    pf = run_prefill(w, xd, k=bsa.paged_cache(Kp, pt_bad), v=bsa.paged_cache(Vp, pt_bad),
                     expect_status=bsa.BSA_DEV_BAD_PAGE)
    hits = 0
    for g in range(w.Hkv):
        lists = {}
        for i in range(w.nb):
            kd = pf.kept[0, g, i, :int(pf.kept_count[0, g, i])].tolist()
            if bad_blk in kd:
                lists[i] = [j for j in kd if j != bad_blk]
                hits += 1
        s = parity.compare_prefill_rows(w, x, pf, 0, g, list(range(w.nb)), attend_lists=lists)
        print("bad page", g, s)
    assert hits >= 2 * w.Hkv    # the diagonal of row 5 and the local windows of rows 6, 7
