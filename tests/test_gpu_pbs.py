"""Block-sparse prefill over a segment-permuted key order (PBS-Attn, Methodology
§1-§4) on the GPU through the C ABI, against the PBS oracle: the key order
(importance ties allowed), the block scores of earlier segments, the kept sets, and
attention with per-key causal masks in the query's own segment."""
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


def to_dev(inputs):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inputs.items()}


def run_pbs(w, xd, seg):
    prob = bsa.problem_for(w, head_w=xd["head_w"])
    prob.segment = seg
    pbs = bsa.PbsPrefill(prob)
    pbs.run(xd["q"], xd["q_idx"], bsa.contiguous_cache(xd["k_idx"]),
            bsa.contiguous_cache(xd["K"]), bsa.contiguous_cache(xd["V"]))
    torch.cuda.synchronize()
    assert int(pbs.status.item()) == 0, f"device status {int(pbs.status.item()):#x}"
    return pbs


SMALL = W.Workload("small_pbs", "prefill", B=1, Hq=8, Hkv=2, d=128, T=64 * 12 + 5,
                   n_sink=1, n_local=1, p=1.0, k_max=2, hh_count=24, amp=3.0, seed=11)


@pytest.mark.parametrize("seg", [128, 256])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 4])
def test_pbs_prefill_small_all_rows(seg, d, G):
    w = SMALL.with_(d=d, Hq=2 * G)
    x = W.make_prefill_inputs(w, "cpu")
    pbs = run_pbs(w, to_dev(x), seg)
    for g in range(w.Hkv):
        s = parity.compare_pbs_rows(w, x, pbs, 0, g, list(range(w.nb)), seg)
        print(f"seg={seg} d={d} G={G} g={g}", s)


def test_pbs_top_p_ragged_segments():
    w = SMALL.with_(T=64 * 14 + 33, p=0.5, k_max=4, k_min=1)
    x = W.make_prefill_inputs(w, "cpu")
    pbs = run_pbs(w, to_dev(x), 192)
    for g in range(w.Hkv):
        s = parity.compare_pbs_rows(w, x, pbs, 0, g, list(range(w.nb)), 192)
        print("top-p seg=192", g, s)


def test_pbs_one_block_segments_match_plain_prefill():
    """Segments of one block only reorder keys inside a block: the kept sets equal the
    unpermuted prefill's and the outputs agree within the attention tolerance."""
    w = SMALL.with_(T=64 * 10 + 7, k_max=3)
    x = W.make_prefill_inputs(w, "cpu")
    xd = to_dev(x)
    pbs = run_pbs(w, xd, 64)
    plain = bsa.Prefill(bsa.problem_for(w, head_w=xd["head_w"]))
    plain.run(xd["q"], xd["q_idx"], bsa.contiguous_cache(xd["k_idx"]),
              bsa.contiguous_cache(xd["K"]), bsa.contiguous_cache(xd["V"]))
    torch.cuda.synchronize()
    assert torch.equal(pbs.pf.kept, plain.kept)
    errs = parity.attention_errors(pbs.pf.o_f32.double().cpu().numpy(), None,
                                   pbs.pf.lse.double().cpu().numpy(),
                                   plain.o_f32.double().cpu().numpy(),
                                   plain.lse.double().cpu().numpy())
    parity.check_attention(errs, "one-block segments vs plain prefill")
    for g in range(w.Hkv):
        parity.compare_pbs_rows(w, x, pbs, 0, g, list(range(w.nb)), 64)


def test_pbs_prefill_64k_sampled_rows():
    w = W.WORKLOADS["prefill_b1_h32_t64k"]
    x = W.make_prefill_inputs(w, "cuda")
    pbs = run_pbs(w, x, 512)
    rows = [0, 1, 7, 8, 9, 100, 511, 1016, 1023]
    for g in (0, 5):
        s = parity.compare_pbs_rows(w, x, pbs, 0, g, rows, 512)
        print("PBS 64K", g, s)
    del x, pbs
    torch.cuda.empty_cache()
