"""Prefill block scorer through the C ABI: index-cache layouts and failed validation.

Paged and padded index-key caches must give the scores of the contiguous cache, bit for
bit, and those must match the fp64 oracle; a page id outside the pool turns every score
of that key block into -inf and sets BSA_DEV_BAD_PAGE, leaving every other score as it
was.
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


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


SMALL = W.Workload("scorer_prefill", "prefill", B=2, Hq=8, Hkv=2, d=64, T=64 * 11 + 9,
                   n_sink=1, n_local=2, p=1.0, k_max=3, hh_count=32, amp=3.0, seed=23)


def scores_for(w, xd, k_idx: bsa.Cache, expect_status=0):
    prob = bsa.problem_for(w, head_w=xd["head_w"])
    nqb = prob.nb
    scores = torch.full((w.B, w.Hkv, nqb, nqb), float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsa.bsa_score_blocks(prob, xd["q_idx"], k_idx, scores, status)
    torch.cuda.synchronize()
    assert int(status.item()) == expect_status, f"device status {int(status.item()):#x}"
    return scores


def lower(scores):
    """Entries j < i of every row (the ones the scorer defines)."""
    nqb = scores.shape[-1]
    m = torch.tril(torch.ones(nqb, nqb, dtype=torch.bool, device=scores.device), diagonal=-1)
    return scores[..., m]


def oracle_scores(w, x, b, g, rows=None):
    """{i: oracle S_i[0:i]} of (b, g)."""
    _, qi, hw = parity.index_heads(x, w, b, g, (slice(0, w.T),))
    ki = parity.f64(x["k_idx"][b, g, :w.T])
    return O.prefill_block_scores(qi, ki, w.T, hw, 1.0 / math.sqrt(w.r), rows=rows)


def check_against_oracle(w, x, scores):
    for b in range(w.B):
        for g in range(w.Hkv):
            ref = oracle_scores(w, x, b, g)
            for i, S_i in ref.items():
                if i == 0:
                    continue
                dev = scores[b, g, i, :i].double().cpu().numpy()
                rel = np.max(np.abs(dev - S_i) / np.maximum(1.0, np.abs(S_i)))
                assert rel <= parity.SCORE_REL, f"(b, g, i) = {(b, g, i)}: score rel err {rel}"


def paged_index_pool(X: torch.Tensor, seed: int):
    """[B, Hkv, T, 16] -> ([P, Hkv, 64, 16] pool, [B, nb] shuffled page table)."""
    B, H, T, r = X.shape
    nb = (T + 63) // 64
    perm = torch.randperm(B * nb, generator=torch.Generator().manual_seed(seed)).to(torch.int32)
    pool = torch.zeros(B * nb, H, 64, r, dtype=X.dtype)
    pt = perm.view(B, nb).contiguous()
    for b in range(B):
        for j in range(nb):
            n = min(64, T - j * 64)
            pool[pt[b, j], :, :n] = X[b, :, j * 64:j * 64 + n]
    return pool, pt


def padded_index_cache(X: torch.Tensor, pad: int = 8) -> bsa.Cache:
    """[B, Hkv, T, 16] -> a cache whose (block, head) records are padded by `pad`
    elements, so the block offsets are multiples of 8 but not of 16."""
    B, H, T, r = X.shape
    nb = (T + 63) // 64
    rec = 64 * r + pad
    t = torch.zeros(B, nb, H, rec, dtype=X.dtype)
    for j in range(nb):
        n = min(64, T - j * 64)
        t[:, j, :, :n * r] = X[:, :, j * 64:j * 64 + n].reshape(B, H, n * r)
    t = t.cuda()
    return bsa.Cache(t, nb * H * rec, H * rec, rec)


@pytest.mark.parametrize("G", [2, 4, 8, 16])
def test_scorer_paged_index_cache_matches_contiguous(G):
    w = SMALL.with_(Hq=2 * G)
    x = W.make_prefill_inputs(w, "cpu")
    xd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    ref = scores_for(w, xd, bsa.contiguous_cache(xd["k_idx"]))
    check_against_oracle(w, x, ref)
    pool, pt = paged_index_pool(x["k_idx"], 5)
    pg = scores_for(w, xd, bsa.paged_cache(pool.cuda(), pt.cuda()))
    assert torch.equal(lower(ref), lower(pg))


def test_scorer_bad_index_page():
    """A page id outside the pool: every score of that key block is -inf, the status says
    BSA_DEV_BAD_PAGE, and every other score is unchanged."""
    w = SMALL
    x = W.make_prefill_inputs(w, "cpu")
    xd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    pool, pt = paged_index_pool(x["k_idx"], 7)
    pool, pt = pool.cuda(), pt.cuda()
    ref = scores_for(w, xd, bsa.paged_cache(pool, pt))
    bad_b, bad_blk = 1, 4
    pt_bad = pt.clone()
    pt_bad[bad_b, bad_blk] = pool.shape[0] + 77
    sc = scores_for(w, xd, bsa.paged_cache(pool, pt_bad), expect_status=bsa.BSA_DEV_BAD_PAGE)
    nqb = sc.shape[-1]
    for b in range(w.B):
        for g in range(w.Hkv):
            for i in range(1, nqb):
                for j in range(i):
                    v, r = float(sc[b, g, i, j]), float(ref[b, g, i, j])
                    if b == bad_b and j == bad_blk:
                        assert v == float("-inf"), (b, g, i, j, v)
                    else:
                        assert v == r, (b, g, i, j, v, r)


@pytest.mark.parametrize("G", [1, 4, 8])
def test_scorer_padded_layout_matches_contiguous(G):
    """Block records padded by 8 elements (offsets that are multiples of 8 but not 16):
    oracle parity, and the contiguous cache's scores bit for bit."""
    w = SMALL.with_(Hq=2 * G)
    x = W.make_prefill_inputs(w, "cpu")
    xd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    pad = scores_for(w, xd, padded_index_cache(x["k_idx"]))
    check_against_oracle(w, x, pad)
    ref = scores_for(w, xd, bsa.contiguous_cache(xd["k_idx"]))
    assert torch.equal(lower(pad), lower(ref))


def test_scorer_full_size_sampled_rows():
    """The 64K workload: every kv head's last query block row, a middle row and an odd
    row against the oracle (rows of up to 1023 key blocks, a missing second block in the
    last key pair of odd rows)."""
    w = W.WORKLOADS["prefill_b1_h32_t64k"]
    x = W.make_prefill_inputs(w, "cuda")
    sc = scores_for(w, x, bsa.contiguous_cache(x["k_idx"]))
    rows = [w.nb - 1, w.nb // 2 + 1, 333]
    for g in range(w.Hkv):
        ref = oracle_scores(w, x, 0, g, rows=rows)
        for i in rows:
            dev = sc[0, g, i, :i].double().cpu().numpy()
            rel = np.max(np.abs(dev - ref[i]) / np.maximum(1.0, np.abs(ref[i])))
            assert rel <= parity.SCORE_REL, (g, i, rel)
