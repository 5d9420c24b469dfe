"""Decode parity on the GPU through the C ABI: block scores, kept sets (tie rule) and
attention outputs against the fp64 oracle, on seeded synthetic workloads."""
import math

import numpy as np
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


def run_decode(w, inputs_dev):
    prob = bsa.problem_for(w, seq_lens=inputs_dev["seq_lens"], head_w=inputs_dev["head_w"])
    step = bsa.DecodeStep(prob)
    k_idx, K, V = bsa.caches_for(inputs_dev)
    step.run(inputs_dev["q"], inputs_dev["q_idx"], k_idx, K, V)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0, f"device status {int(step.status.item()):#x}"
    return step


def all_rows(w):
    return [(b, g) for b in range(w.B) for g in range(w.Hkv)]


def test_decode_tiny_workload_all_rows():
    w = W.WORKLOADS["decode_tiny_b1_h8_t4k"]
    x = W.make_decode_inputs(w, "cpu")
    step = run_decode(w, to_dev(x))
    s = parity.compare_decode_rows(w, x, step, all_rows(w))
    assert s["rows"] == w.B * w.Hkv


SMALL = W.Workload("small", "decode", B=2, Hq=8, Hkv=2, d=128, T=64 * 40 + 37, paged=True,
                   n_sink=1, n_local=2, p=0.9, k_max=8, hh_count=8, amp=3.0, seed=3)


@pytest.mark.parametrize("p", [0.0, 0.1, 0.3, 0.5, 0.9, 1.0])
def test_decode_top_p_sweep(p):
    w = SMALL.with_(p=p, k_max=30)
    x = W.make_decode_inputs(w, "cpu")
    step = run_decode(w, to_dev(x))
    parity.compare_decode_rows(w, x, step, all_rows(w))


@pytest.mark.parametrize("T", [1, 64, 130, 4096, 64 * 70 + 1])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_lengths_and_dims(T, d):
    w = SMALL.with_(T=T, d=d, paged=False, hh_count=min(8, T))
    x = W.make_decode_inputs(w, "cpu")
    step = run_decode(w, to_dev(x))
    parity.compare_decode_rows(w, x, step, all_rows(w))


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16])
def test_decode_group_sizes(G):
    w = SMALL.with_(Hq=2 * G, Hkv=2, p=0.5, k_max=12)
    x = W.make_decode_inputs(w, "cpu")
    step = run_decode(w, to_dev(x))
    parity.compare_decode_rows(w, x, step, all_rows(w))


def test_decode_ragged_batch_and_empty_sequence():
    w = SMALL.with_(B=4, seq_lens=(64 * 40 + 37, 1000, 0, 65), p=0.7, k_max=6, k_min=2)
    x = W.make_decode_inputs(w, "cpu")
    step = run_decode(w, to_dev(x))
    rows = [(b, g) for b in (0, 1, 3) for g in range(w.Hkv)]
    parity.compare_decode_rows(w, x, step, rows)
    # the empty sequence keeps nothing and produces o = 0, lse = -inf
    assert step.kept_count[2].tolist() == [0, 0]
    assert torch.all(step.o_f32[2] == 0)
    assert torch.all(torch.isinf(step.lse[2])) and torch.all(step.lse[2] < 0)


def test_decode_unequal_head_weights():
    w = SMALL.with_(head_w=tuple(float(v) for v in np.linspace(0.05, 0.4, 8)), p=0.6, k_max=10)
    x = W.make_decode_inputs(w, "cpu")
    step = run_decode(w, to_dev(x))
    parity.compare_decode_rows(w, x, step, all_rows(w))


def test_page_table_shuffle_is_bit_identical():
    """The same logical cache behind two page tables gives bit-identical results."""
    w = SMALL.with_(p=0.6, k_max=10)
    x = W.make_decode_inputs(w, "cpu")
    xd = to_dev(x)
    s1 = run_decode(w, xd)
    out1 = [t.clone() for t in (s1.scores, s1.kept, s1.o, s1.o_f32, s1.lse)]
    # move every page to a new physical slot
    P = xd["K"].shape[0]
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(5)).to("cuda")
    K2 = torch.empty_like(xd["K"])
    V2 = torch.empty_like(xd["V"])
    K2[perm] = xd["K"]
    V2[perm] = xd["V"]
    pt2 = perm[xd["page_table"].long()].to(torch.int32).contiguous()
    xd2 = dict(xd, K=K2, V=V2, page_table=pt2)
    s2 = run_decode(w, xd2)
    out2 = (s2.scores, s2.kept, s2.o, s2.o_f32, s2.lse)
    for a, b in zip(out1, out2):
        assert torch.equal(a, b)


def test_bad_page_id_is_reported_not_trapped():
    w = SMALL.with_(B=1)
    x = W.make_decode_inputs(w, "cpu")
    xd = to_dev(x)
    xd["page_table"] = xd["page_table"].clone()
    xd["page_table"][0, 3] = 10 ** 6        # outside the pool
    prob = bsa.problem_for(w, seq_lens=xd["seq_lens"], head_w=xd["head_w"])
    step = bsa.DecodeStep(prob)
    k_idx, K, V = bsa.caches_for(xd)
    step.run(xd["q"], xd["q_idx"], k_idx, K, V)
    torch.cuda.synchronize()
    assert int(step.status.item()) & bsa.BSA_DEV_BAD_PAGE


# ---------------------------------------------------------------- full-size workloads
# Every row of every full-size decode workload: the 1M rows are the only inputs of
# the cluster selection at full size (16,374 candidates per row).
@pytest.mark.parametrize("name", ["decode_b8_h32_t32k_paged", "decode_b32_h32_t128k_paged",
                                  "decode_b1_h64_t1m"])
def test_decode_full_size_every_row(name):
    w = W.WORKLOADS[name]
    x = W.make_decode_inputs(w, "cuda")
    step = run_decode(w, x)
    s = parity.compare_decode_rows(w, x, step, all_rows(w))
    print(f"{name}: {s['rows']} rows compared, {s['ties']} ties", s)
    assert s["rows"] == w.B * w.Hkv
    # every row keeps sinks + local + at most k_max dynamic blocks
    assert int(step.kept_count.max()) <= w.n_sink + w.n_local + w.k_max
    del x, step
    torch.cuda.empty_cache()


# rows longer than 2048 candidates run the cluster selection (several CTAs per row)
LONG = W.Workload("long_rows", "decode", B=3, Hq=8, Hkv=2, d=64, T=64 * 5000 + 17, paged=False,
                  n_sink=2, n_local=3, p=0.9, k_max=300, hh_count=40, amp=3.0, seed=21,
                  seq_lens=(64 * 5000 + 17, 64 * 3000 + 5, 90))


@pytest.mark.parametrize("p,k_min", [(0.05, 0), (0.5, 4), (0.9, 0), (1.0, 0), (0.0, 7)])
def test_decode_long_rows_cluster_select(p, k_min):
    w = LONG.with_(p=p, k_min=k_min)
    x = W.make_decode_inputs(w, "cpu")
    step = run_decode(w, to_dev(x))
    parity.compare_decode_rows(w, x, step, all_rows(w))


@pytest.mark.parametrize("name", ["decode_tiny_b1_h8_t4k", "decode_b8_h32_t32k_paged"])
def test_decode_graph_matches_eager_and_oracle(name):
    """The whole host-to-host decode step as one CUDA graph launch gives the same
    bytes as the eager entry points, for the captured query and for a new query
    written into the same pinned buffers; the replayed result also passes parity."""
    w = W.WORKLOADS[name]
    x = W.make_decode_inputs(w, "cpu")
    xd = to_dev(x)
    prob = bsa.problem_for(w, seq_lens=xd["seq_lens"], head_w=xd["head_w"])
    k_idx, K, V = bsa.caches_for(xd)
    q_h, qi_h = x["q"].clone().pin_memory(), x["q_idx"].clone().pin_memory()
    eager = bsa.DecodeStep(prob)
    graphed = bsa.DecodeStep(prob)
    o_h = torch.empty(eager.o.shape, dtype=eager.o.dtype).pin_memory()
    lse_h = torch.empty(eager.lse.shape, dtype=eager.lse.dtype).pin_memory()
    g = bsa.DecodeGraph(graphed, q_h, qi_h, k_idx, K, V, o_h, lse_h)
    for trial in range(2):
        if trial == 1:   # a new query, written in place
            gen = torch.Generator().manual_seed(5)
            q_h.copy_(torch.randn(q_h.shape, generator=gen).to(q_h.dtype))
            qi_h.copy_(torch.randn(qi_h.shape, generator=gen).to(qi_h.dtype))
        eager.run(q_h.cuda(), qi_h.cuda(), k_idx, K, V)
        g.run()
        torch.cuda.synchronize()
        assert int(eager.status.item()) == 0 and int(graphed.status.item()) == 0
        assert torch.equal(o_h, eager.o.cpu())
        assert torch.equal(lse_h, eager.lse.cpu())
        assert torch.equal(graphed.kept.cpu(), eager.kept.cpu())
    x2 = dict(x, q=q_h.clone(), q_idx=qi_h.clone())
    parity.compare_decode_rows(w, x2, graphed, all_rows(w)[:4])
