"""Block-sparse causal prefill parity on the GPU through the C ABI."""
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


def run_prefill(w, xd):
    prob = bsa.problem_for(w, head_w=xd["head_w"])
    pf = bsa.Prefill(prob)
    k_idx = bsa.contiguous_cache(xd["k_idx"])
    K = bsa.contiguous_cache(xd["K"])
    V = bsa.contiguous_cache(xd["V"])
    pf.run(xd["q"], xd["q_idx"], k_idx, K, V)
    torch.cuda.synchronize()
    assert int(pf.status.item()) == 0, f"device status {int(pf.status.item()):#x}"
    return pf


SMALL = W.Workload("small_prefill", "prefill", B=1, Hq=8, Hkv=2, d=128, T=64 * 12 + 5,
                   n_sink=1, n_local=2, p=1.0, k_max=3, hh_count=32, amp=3.0, seed=11)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T", [64 * 12 + 5, 64 * 9, 70])
def test_prefill_small_all_rows(d, T):
    w = SMALL.with_(d=d, T=T)
    x = W.make_prefill_inputs(w, "cpu")
    pf = run_prefill(w, to_dev(x))
    nqb = (T + 63) // 64
    for b in range(w.B):
        for g in range(w.Hkv):
            parity.compare_prefill_rows(w, x, pf, b, g, list(range(nqb)))


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_prefill_group_sizes(G):
    w = SMALL.with_(Hq=2 * G, Hkv=2, T=64 * 8 + 17, k_max=2)
    x = W.make_prefill_inputs(w, "cpu")
    pf = run_prefill(w, to_dev(x))
    for g in range(w.Hkv):
        parity.compare_prefill_rows(w, x, pf, 0, g, list(range(9)))


def test_prefill_dense_limit():
    """top-k >= number of blocks: every causal block kept (dense causal attention)."""
    w = SMALL.with_(k_max=64, T=64 * 10 + 3)
    x = W.make_prefill_inputs(w, "cpu")
    pf = run_prefill(w, to_dev(x))
    nqb = 11
    for i in range(nqb):
        assert int(pf.kept_count[0, 0, i]) == i + 1
    for g in range(w.Hkv):
        parity.compare_prefill_rows(w, x, pf, 0, g, list(range(nqb)))


def test_prefill_top_p_and_kmin():
    w = SMALL.with_(p=0.5, k_max=5, k_min=1, T=64 * 14)
    x = W.make_prefill_inputs(w, "cpu")
    pf = run_prefill(w, to_dev(x))
    for g in range(w.Hkv):
        parity.compare_prefill_rows(w, x, pf, 0, g, list(range(14)))


def test_prefill_full_size_rows_of_every_kv_head():
    """The 64K workload: every kv head on query blocks 0-3 (sinks and local windows
    overlap the diagonal), 67-69 (where kept(i) = min(i + 1, 68) saturates), every
    64th block and the last one."""
    w = W.WORKLOADS["prefill_b1_h32_t64k"]
    x = W.make_prefill_inputs(w, "cuda")
    pf = run_prefill(w, x)
    rows = sorted({0, 1, 2, 3, 67, 68, 69, w.nb - 1} | set(range(64, w.nb, 64)))
    total = {"rows": 0, "ties": 0}
    for g in range(w.Hkv):
        s = parity.compare_prefill_rows(w, x, pf, 0, g, rows)
        total["rows"] += s["rows"]
        total["ties"] += s["ties"]
        print("prefill 64K, kv head", g, s)
    print(f"prefill 64K: {total['rows']} rows compared, {total['ties']} ties")
    assert total["rows"] == w.Hkv * len(rows)
    # kept(i) = min(i + 1, 68) for this configuration, on every row
    kc = pf.kept_count[0].cpu()
    expect = torch.tensor([min(i + 1, 68) for i in range(w.nb)], dtype=kc.dtype)
    assert torch.equal(kc, expect.expand_as(kc))
