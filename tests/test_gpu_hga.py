"""Two-level (block, then token-group) decode routing on the GPU through the C ABI,
against the HGA oracle ("Hierarchical Global Attention", Central mechanism §2 and
§4): block and group scores, kept blocks and kept groups (tie rules), the group
masks of the always-visible blocks, and the attention over the routed tokens."""
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


def run_hga(w, xd, gs, k_groups):
    prob = bsa.problem_for(w, seq_lens=xd["seq_lens"], head_w=xd["head_w"])
    prob.group_size, prob.k_groups = gs, k_groups
    step = bsa.DecodeStep(prob)
    k_idx, K, V = bsa.caches_for(xd)
    step.run(xd["q"], xd["q_idx"], k_idx, K, V)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0, f"device status {int(step.status.item()):#x}"
    return step


def all_rows(w):
    return [(b, g) for b in range(w.B) for g in range(w.Hkv)]


# ragged lengths: a partial last block, a one-token sequence, an empty one
SMALL = W.Workload("hga_small", "decode", B=4, Hq=8, Hkv=2, d=128, T=64 * 36 + 23, paged=True,
                   n_sink=1, n_local=2, p=0.9, k_max=10, hh_count=12, amp=3.0, seed=11,
                   seq_lens=(64 * 36 + 23, 64 * 20 + 40, 1, 0))


@pytest.mark.parametrize("k_groups", [1, 7, 1000])
@pytest.mark.parametrize("gs", [16, 32, 64])
def test_hga_small_all_rows(gs, k_groups):
    w = SMALL
    x = W.make_decode_inputs(w, "cpu")
    step = run_hga(w, to_dev(x), gs, k_groups)
    s = parity.compare_hga_rows(w, x, step, all_rows(w), gs, k_groups)
    assert s["rows"] == w.B * w.Hkv


@pytest.mark.parametrize("gs", [16, 32])
def test_hga_every_block_a_candidate(gs):
    """No local window and p = 1 with a cap above the block count: every block past
    the sink is kept at level 1, so the groups of the partial last block compete too."""
    w = SMALL.with_(n_local=0, p=1.0, k_max=64, seq_lens=(64 * 36 + 23, 64 * 20 + 7, 65, 17))
    x = W.make_decode_inputs(w, "cpu")
    step = run_hga(w, to_dev(x), gs, 9)
    parity.compare_hga_rows(w, x, step, all_rows(w), gs, 9)


@pytest.mark.parametrize("G,d", [(16, 128), (1, 64), (4, 64)])
def test_hga_group_sizes_and_dims(G, d):
    w = SMALL.with_(Hq=2 * G, Hkv=2, d=d, paged=False, p=0.7, k_max=12)
    x = W.make_decode_inputs(w, "cpu")
    step = run_hga(w, to_dev(x), 16, 11)
    parity.compare_hga_rows(w, x, step, all_rows(w), 16, 11)


def test_hga_no_groups_kept_attends_the_visible_blocks():
    w = SMALL
    x = W.make_decode_inputs(w, "cpu")
    step = run_hga(w, to_dev(x), 16, 0)
    parity.compare_hga_rows(w, x, step, all_rows(w), 16, 0)


def test_hga_whole_blocks_equal_plain_decode_bit_for_bit():
    """One group per block and k_groups >= K_max: level 2 keeps every selected
    block whole, and the kernels take the whole-block path, so the outputs are those
    of the one-level decode bit for bit."""
    w = SMALL
    xd = to_dev(W.make_decode_inputs(w, "cpu"))
    hga = run_hga(w, xd, 64, w.k_max)
    prob = bsa.problem_for(w, seq_lens=xd["seq_lens"], head_w=xd["head_w"])
    plain = bsa.DecodeStep(prob)
    k_idx, K, V = bsa.caches_for(xd)
    plain.run(xd["q"], xd["q_idx"], k_idx, K, V)
    torch.cuda.synchronize()
    assert torch.equal(hga.kept, plain.kept) and torch.equal(hga.kept_count, plain.kept_count)
    assert torch.equal(hga.o.view(torch.int16), plain.o.view(torch.int16))
    assert torch.equal(hga.lse, plain.lse)
    # group scores of one-block groups are the block scores
    nb = w.nb
    assert torch.equal(hga.group_scores[:, :, :nb], hga.scores[:, :, :nb])


def test_hga_32k_sampled_rows():
    """The 32K paged decode workload (8 sequences, 8 kv heads, K_max 64) with groups of
    16 and 96 kept groups per row: every kv head of sequences 0 and 7."""
    w = W.WORKLOADS["decode_b8_h32_t32k_paged"]
    x = W.make_decode_inputs(w, "cpu")
    step = run_hga(w, to_dev(x), 16, 96)
    rows = [(b, g) for b in (0, w.B - 1) for g in range(w.Hkv)]
    s = parity.compare_hga_rows(w, x, step, rows, 16, 96)
    assert s["groups"] > 0
    print(f"\n32K two-level rows {s['rows']}: ties {s['ties']}, group ties {s['group_ties']}, "
          f"max abs {s['max_abs']:.2e}, score rel {s['score_rel']:.2e}")
