"""Compact indexer: one index head per kv group instead of one per query head
(SparDA, Main innovations §2). Through the C ABI with idx_heads = 1 (q_idx with Hkv
rows, weight 1), decode and prefill match the oracle run on the same index queries."""
import pytest
import torch

import block_sparse_long_06_b200 as bsa
from block_sparse_long_06_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def group_index_queries(q_idx, Hkv):
    """One synthetic index query per group: the bf16 mean of the group's index queries."""
    B, Hq = q_idx.shape[:2]
    G = Hq // Hkv
    return q_idx.float().reshape(B, Hkv, G, *q_idx.shape[2:]).mean(2).to(torch.bfloat16).contiguous()


@pytest.mark.parametrize("G", [4, 8])
def test_decode_one_index_head_per_group(G):
    w = W.Workload("idx1", "decode", B=2, Hq=4 * G, Hkv=4, d=128, T=64 * 37 + 11, paged=True,
                   n_sink=1, n_local=2, p=0.8, k_max=10, hh_count=8, amp=3.0, seed=13)
    x = W.make_decode_inputs(w, "cpu")
    x["q_idx"] = group_index_queries(x["q_idx"], w.Hkv)
    x["idx_heads"] = 1
    xd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    prob = bsa.problem_for(w, seq_lens=xd["seq_lens"], head_w=None)
    prob.idx_heads = 1
    step = bsa.DecodeStep(prob)
    k_idx, K, V = bsa.caches_for(xd)
    step.run(xd["q"], xd["q_idx"], k_idx, K, V)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    parity.compare_decode_rows(w, x, step, [(b, g) for b in range(w.B) for g in range(w.Hkv)])


def test_prefill_one_index_head_per_group():
    w = W.Workload("pidx1", "prefill", B=1, Hq=16, Hkv=4, d=128, T=64 * 12 + 40, n_sink=1,
                   n_local=2, p=1.0, k_max=4, hh_count=16, amp=3.0, seed=17)
    x = W.make_prefill_inputs(w, "cpu")
    x["q_idx"] = group_index_queries(x["q_idx"], w.Hkv)
    x["idx_heads"] = 1
    xd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    prob = bsa.problem_for(w, head_w=None)
    prob.idx_heads = 1
    pf = bsa.Prefill(prob)
    pf.run(xd["q"], xd["q_idx"], bsa.contiguous_cache(xd["k_idx"]), bsa.contiguous_cache(xd["K"]),
           bsa.contiguous_cache(xd["V"]))
    torch.cuda.synchronize()
    assert int(pf.status.item()) == 0
    for g in range(w.Hkv):
        parity.compare_prefill_rows(w, x, pf, 0, g, list(range(w.nb)))
