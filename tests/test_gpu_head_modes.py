"""Per-kv-head retrieval / local modes in one launch (RTPurbo, Methodology §1: most
heads are local heads that keep attention sinks plus a sliding window; a few
retrieval heads select blocks dynamically). Through the C ABI, a per-kv-head p
(p <= 0: local head) must give, row by row, the oracle's result for that head's p;
the scorers skip local heads."""
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


def to_dev(inputs, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inputs.items()}


HEAD_P = [0.9, 0.0, 0.5, -1.0]


@pytest.mark.parametrize("index_cache", ["bf16", "fp4"])
def test_decode_mixed_head_modes(index_cache):
    w = W.Workload("modes", "decode", B=2, Hq=16, Hkv=4, d=128, T=64 * 33 + 9, paged=True,
                   n_sink=1, n_local=2, p=0.9, k_max=12, hh_count=8, amp=3.0, seed=7,
                   seq_lens=(64 * 33 + 9, 64 * 20))
    x = W.make_decode_inputs(w, "cpu")
    xd = to_dev(x)
    prob = bsa.problem_for(w, seq_lens=xd["seq_lens"], head_w=xd["head_w"])
    prob.head_p = torch.tensor(HEAD_P, dtype=torch.float32, device="cuda")
    step = bsa.DecodeStep(prob)
    k_idx, K, V = bsa.caches_for(xd)
    if index_cache == "fp4":
        import numpy as np
        from oracle import index_quant as iq
        qc = bsa.contiguous_qcache(w.B, w.Hkv, w.T, bsa.IDX_FP4, device="cuda")
        bsa.bsa_quantize_index_keys(prob, k_idx, qc, step.status)
        k_idx = qc
        codes, scales, g = iq.quantize_cache(x["k_idx"].float().numpy(), x["seq_lens"].tolist(), "fp4")
        x = dict(x)
        x["k_idx"] = torch.from_numpy(iq.dequantize(codes, scales, g, "fp4"))
    step.run(xd["q"], xd["q_idx"], k_idx, K, V)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    for g, p in enumerate(HEAD_P):
        rows = [(b, g) for b in range(w.B)]
        parity.compare_decode_rows(w.with_(p=p), x, step, rows, check_scores=p > 0)
        if p <= 0:
            # a local head keeps exactly its sinks and its local window
            for b in range(w.B):
                nb = (int(x["seq_lens"][b]) + 63) // 64
                want = sorted(set(range(min(w.n_sink, nb))) | set(range(max(0, nb - w.n_local), nb)))
                c = int(step.kept_count[b, g])
                assert step.kept[b, g, :c].tolist() == want


def test_prefill_mixed_head_modes():
    w = W.Workload("pmodes", "prefill", B=1, Hq=16, Hkv=4, d=128, T=64 * 14 + 21, n_sink=1,
                   n_local=2, p=1.0, k_max=4, hh_count=16, amp=3.0, seed=11)
    x = W.make_prefill_inputs(w, "cpu")
    xd = to_dev(x)
    prob = bsa.problem_for(w, head_w=xd["head_w"])
    prob.head_p = torch.tensor([1.0, 0.0, 0.6, 0.0], dtype=torch.float32, device="cuda")
    pf = bsa.Prefill(prob)
    pf.run(xd["q"], xd["q_idx"], bsa.contiguous_cache(xd["k_idx"]), bsa.contiguous_cache(xd["K"]),
           bsa.contiguous_cache(xd["V"]))
    torch.cuda.synchronize()
    assert int(pf.status.item()) == 0
    nqb = w.nb
    for g, p in enumerate([1.0, 0.0, 0.6, 0.0]):
        parity.compare_prefill_rows(w.with_(p=p), x, pf, 0, g, list(range(nqb)),
                                    check_scores=p > 0)
