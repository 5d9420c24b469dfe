"""4-bit index-key cache on the GPU through the C ABI (SpotAttention, Methodology §4):
the device quantiser reproduces the oracle's bytes exactly (integer work: bit-exact),
and decode on the quantised cache matches the oracle run on the dequantised keys
(scores, kept sets under the tie rule, attention)."""
import json
import os

import numpy as np
import pytest
import torch

import block_sparse_long_06_b200 as bsa
from block_sparse_long_06_b200 import workloads as W
from oracle import index_quant as iq
from tests import parity

pytestmark = pytest.mark.gpu
FMTS = {"fp4": bsa.IDX_FP4, "int4": bsa.IDX_INT4}


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def to_dev(inputs, device="cuda"):
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in inputs.items()}


def quantize_on_device(w, xd, fmt, paged=False):
    prob = bsa.problem_for(w, seq_lens=xd["seq_lens"], head_w=xd["head_w"])
    k_idx = bsa.contiguous_cache(xd["k_idx"])
    if paged:
        pt = xd["page_table"]
        qc = bsa.paged_qcache(pt.numel(), w.Hkv, pt, FMTS[fmt], device="cuda")
    else:
        qc = bsa.contiguous_qcache(w.B, w.Hkv, w.T, FMTS[fmt], device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    bsa.bsa_quantize_index_keys(prob, k_idx, qc, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return prob, qc


def logical_records(qc, w, page_table=None):
    rec = qc.records.cpu().numpy().reshape(-1, iq.RECORD_BYTES)
    nb = w.nb
    if page_table is None:
        return rec.reshape(w.B, w.Hkv, nb, iq.RECORD_BYTES)
    pt = page_table.cpu().numpy()
    out = np.zeros((w.B, w.Hkv, nb, iq.RECORD_BYTES), dtype=np.uint8)
    for b in range(w.B):
        for g in range(w.Hkv):
            out[b, g] = rec[pt[b] * w.Hkv + g]
    return out


def oracle_records(w, x, fmt):
    k = x["k_idx"].float().numpy()
    codes, scales, g = iq.quantize_cache(k, x["seq_lens"].tolist(), fmt)
    return iq.pack_records(codes, scales), g, codes, scales


RAGGED = W.Workload("ragged_q", "decode", B=3, Hq=8, Hkv=2, d=64, T=64 * 9 + 23, n_sink=1,
                    n_local=2, p=0.9, k_max=6, hh_count=6, amp=3.0, seed=5,
                    seq_lens=(64 * 9 + 23, 100, 0))


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
@pytest.mark.parametrize("wname", ["decode_tiny_b1_h8_t4k", "ragged"])
def test_quantiser_bit_exact(fmt, wname):
    w = RAGGED if wname == "ragged" else W.WORKLOADS[wname]
    x = W.make_decode_inputs(w, "cpu")
    _, qc = quantize_on_device(w, to_dev(x), fmt)
    ref, g, _, _ = oracle_records(w, x, fmt)
    assert np.float32(qc.gscale.item()) == g
    dev = logical_records(qc, w)
    assert np.array_equal(dev, ref), f"{int((dev != ref).sum())} bytes differ"


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
def test_quantiser_paged_bit_exact(fmt):
    w = W.WORKLOADS["decode_b8_h32_t32k_paged"].with_(B=2, T=64 * 37 + 5)
    x = W.make_decode_inputs(w, "cpu")
    _, qc = quantize_on_device(w, to_dev(x), fmt, paged=True)
    ref, g, _, _ = oracle_records(w, x, fmt)
    assert np.float32(qc.gscale.item()) == g
    assert np.array_equal(logical_records(qc, w, x["page_table"]), ref)


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
def test_quantiser_hand_derived_golden(fmt):
    G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "index_quant.json")))[fmt]
    k = torch.tensor(G["k"], dtype=torch.float32).to(torch.bfloat16)
    n = k.shape[0]
    w = W.Workload("golden", "decode", B=1, Hq=1, Hkv=1, d=64, T=n, n_sink=1, n_local=1, p=0.9,
                   k_max=1)
    xd = {"k_idx": k.reshape(1, 1, n, 16).cuda().contiguous(),
          "seq_lens": torch.tensor([n], dtype=torch.int32, device="cuda"), "head_w": None}
    _, qc = quantize_on_device(w, xd, fmt)
    assert qc.gscale.item() == G["g"]
    rec = qc.records.cpu().numpy()
    assert rec[512:512 + n].tolist() == G["scale_codes"]
    for t in range(n):
        byts = rec[8 * t:8 * t + 8]
        codes = [int(byts[c // 2] >> (4 * (c % 2))) & 15 for c in range(16)]
        assert codes == G["codes"][t], t


def run_decode_q(w, x, fmt, paged=False):
    xd = to_dev(x)
    prob, qc = quantize_on_device(w, xd, fmt, paged=paged and xd.get("page_table") is not None)
    step = bsa.DecodeStep(prob)
    _, K, V = bsa.caches_for(xd)
    step.run(xd["q"], xd["q_idx"], qc, K, V)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    # the oracle runs on the dequantised keys of the oracle's own quantiser
    _, g, codes, scales = oracle_records(w, x, fmt)
    xq = dict(x)
    xq["k_idx"] = torch.from_numpy(iq.dequantize(codes, scales, g, fmt))
    return step, xq


SMALLQ = W.Workload("smallq", "decode", B=2, Hq=8, Hkv=2, d=128, T=64 * 40 + 37, paged=True,
                    n_sink=1, n_local=2, p=0.9, k_max=8, hh_count=8, amp=3.0, seed=3)


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
@pytest.mark.parametrize("p", [0.1, 0.5, 0.9, 1.0])
def test_decode_on_quantised_cache(fmt, p):
    w = SMALLQ.with_(p=p, k_max=30)
    x = W.make_decode_inputs(w, "cpu")
    step, xq = run_decode_q(w, x, fmt, paged=True)
    rows = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    parity.compare_decode_rows(w, xq, step, rows)


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
def test_decode_on_quantised_cache_ragged_and_g8(fmt):
    for w in (RAGGED, W.Workload("g8q", "decode", B=1, Hq=64, Hkv=4, d=128, T=64 * 30, n_sink=2,
                                 n_local=3, p=0.7, k_max=12, hh_count=10, amp=3.0, seed=9)):
        x = W.make_decode_inputs(w, "cpu")
        step, xq = run_decode_q(w, x, fmt)
        rows = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
        parity.compare_decode_rows(w, xq, step, rows)


class _RowKeys:
    """Dequantised index keys of a few (b, g) rows of a full-size cache, indexable
    like the k_idx tensor by the parity helpers."""

    def __init__(self, rows):
        self.rows = rows

    def __getitem__(self, idx):
        b, g, sl = idx
        return self.rows[(b, g)][sl]


@pytest.mark.parametrize("fmt", ["fp4"])
def test_quantised_decode_full_size_sampled_rows(fmt):
    """128K, B = 32 (the bench's decode workload) on the 4-bit cache: device bytes of
    sampled rows equal the oracle's, and those rows match the oracle end to end."""
    w = W.WORKLOADS["decode_b32_h32_t128k_paged"]
    x = W.make_decode_inputs(w, "cuda")
    prob, qc = quantize_on_device(w, x, fmt)
    step = bsa.DecodeStep(prob)
    _, K, V = bsa.caches_for(x)
    step.run(x["q"], x["q_idx"], qc, K, V)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    lens = x["seq_lens"].cpu().tolist()
    g = iq.cache_gscale(x["k_idx"].float().cpu().numpy(), lens, fmt)
    assert np.float32(qc.gscale.item()) == g
    rows = [(0, 0), (5, 3), (31, 7)]
    rec = qc.records.view(w.B, w.Hkv, w.nb, iq.RECORD_BYTES)
    deq = {}
    for (b, gg) in rows:
        k = x["k_idx"][b, gg].float().cpu().numpy()
        codes, scales = iq.quantize_rows(k, g, fmt)
        nbp = w.nb * 64
        c = np.zeros((nbp, 16), dtype=np.int64)
        sc = np.zeros(nbp, dtype=np.uint8)
        c[:lens[b]], sc[:lens[b]] = codes[:lens[b]], scales[:lens[b]]
        ref = iq.pack_records(c[None, None], sc[None, None])[0, 0]
        assert np.array_equal(rec[b, gg].cpu().numpy(), ref), (b, gg)
        deq[(b, gg)] = torch.from_numpy(iq.dequantize(c, sc, g, fmt))
    xq = {k_: v for k_, v in x.items() if k_ != "k_idx"}
    xq["k_idx"] = _RowKeys(deq)
    s = parity.compare_decode_rows(w, xq, step, rows)
    print("4-bit full size", s)


@pytest.mark.parametrize("fmt", ["fp4", "int4"])
@pytest.mark.parametrize("gs", [16, 64])
def test_two_level_routing_on_quantised_cache(fmt, gs):
    """Two-level routing (HGA, Central mechanism §2) on the 4-bit cache: group scores of
    the quantised keys, kept groups and attention against the HGA oracle run on the
    dequantised keys."""
    w = SMALLQ.with_(p=0.9, k_max=12)
    x = W.make_decode_inputs(w, "cpu")
    xd = to_dev(x)
    prob, qc = quantize_on_device(w, xd, fmt, paged=True)
    prob.group_size, prob.k_groups = gs, 13
    step = bsa.DecodeStep(prob)
    _, K, V = bsa.caches_for(xd)
    step.run(xd["q"], xd["q_idx"], qc, K, V)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0
    _, g, codes, scales = oracle_records(w, x, fmt)
    xq = dict(x)
    xq["k_idx"] = torch.from_numpy(iq.dequantize(codes, scales, g, fmt))
    rows = [(b, gg) for b in range(w.B) for gg in range(w.Hkv)]
    s = parity.compare_hga_rows(w, xq, step, rows, gs, 13)
    assert s["rows"] == len(rows)
