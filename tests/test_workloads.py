"""The seeded input recipe (block_sparse_long_06_b200/workloads.py) on the CPU: determinism,
shapes, the page-table indirection, and where the heavy hitters are planted and how.

A planted key row is amp * q_hat + N(0, 0.1^2) with q_hat the unit mean query of its kv
group, so its cosine with q_hat is close to 1, while an N(0, 1) row of width d has a cosine
of about 1 / sqrt(d) with any fixed direction. The tests find the planted rows by that
cosine in logical token order (through the page table when the cache is paged).
"""
import numpy as np
import pytest
import torch

from block_sparse_long_06_b200 import workloads as W


def _cos_rows(X: torch.Tensor, u: torch.Tensor) -> torch.Tensor:
    Xf = X.float()
    return (Xf @ u) / Xf.norm(dim=-1).clamp_min(1e-12)


def _qhat_decode(x, w, b, g):
    m = x["q"][b, g * w.G:(g + 1) * w.G].float().mean(0)
    return m / m.norm()


def _planted(x, w, b, g, qhat):
    K = W.logical_kv(x, w, b, g, "K")
    return torch.nonzero(_cos_rows(K, qhat) > 0.9).flatten().numpy()


SMALL_DEC = W.WORKLOADS["decode_tiny_b1_h8_t4k"].with_(B=2, T=64 * 20 + 7, hh_count=12)


@pytest.mark.parametrize("paged", [False, True])
def test_decode_inputs_are_seeded_and_shaped(paged):
    w = SMALL_DEC.with_(paged=paged)
    a, b = W.make_decode_inputs(w), W.make_decode_inputs(w)
    for k in ("q", "q_idx", "k_idx", "K", "V", "seq_lens", "head_w"):
        assert torch.equal(a[k], b[k]), k
    c = W.make_decode_inputs(w.with_(seed=w.seed + 1))
    assert not torch.equal(a["K"], c["K"])
    assert a["q"].shape == (w.B, w.Hq, w.d) and a["q"].dtype == torch.bfloat16
    assert a["q_idx"].shape == (w.B, w.Hq, w.r)
    assert a["k_idx"].shape == (w.B, w.Hkv, w.T, w.r) and a["k_idx"].is_contiguous()
    if paged:
        assert a["K"].shape == (w.B * w.nb, w.Hkv, 64, w.d)
        pt = a["page_table"]
        assert pt.shape == (w.B, w.nb) and pt.dtype == torch.int32
        assert sorted(pt.flatten().tolist()) == list(range(w.B * w.nb))   # a permutation
    else:
        assert a["K"].shape == (w.B, w.Hkv, w.T, w.d) and a["page_table"] is None
    assert torch.allclose(a["head_w"], torch.full((w.Hq,), 1.0 / w.G))


@pytest.mark.parametrize("paged", [False, True])
def test_decode_heavy_hitters_are_planted_along_the_mean_query(paged):
    w = SMALL_DEC.with_(paged=paged, hh_kind="uniform")
    x = W.make_decode_inputs(w)
    for b in range(w.B):
        for g in range(w.Hkv):
            qhat = _qhat_decode(x, w, b, g)
            pos = _planted(x, w, b, g, qhat)
            assert len(pos) == w.hh_count, (b, g, len(pos))
            K = W.logical_kv(x, w, b, g, "K")
            # the planted rows: norm near amp, direction near q_hat
            assert torch.allclose(K[pos].float().norm(dim=-1),
                                  torch.full((len(pos),), w.amp), rtol=0.1)


def test_decode_zipf_and_runs_placements():
    # Zipf over block index: the planted blocks crowd the front of the sequence
    wz = W.WORKLOADS["decode_tiny_b1_h8_t4k"].with_(B=1, T=64 * 64, hh_count=40, hh_kind="zipf",
                                                     hh_param=1.1)
    xz = W.make_decode_inputs(wz)
    blocks = np.concatenate([_planted(xz, wz, 0, g, _qhat_decode(xz, wz, 0, g)) // 64
                             for g in range(wz.Hkv)])
    assert len(blocks) == 40 * wz.Hkv
    assert np.median(blocks) < wz.nb / 4
    # runs: hh_count / run consecutive runs of `run` tokens, non-overlapping
    wr = wz.with_(hh_kind="runs", hh_param=8, hh_count=32)
    xr = W.make_decode_inputs(wr)
    for g in range(wr.Hkv):
        pos = _planted(xr, wr, 0, g, _qhat_decode(xr, wr, 0, g))
        assert len(pos) == 32
        starts = [p for i, p in enumerate(pos) if i == 0 or pos[i - 1] != p - 1]
        lengths = np.diff(np.append([np.searchsorted(pos, s) for s in starts], len(pos)))
        assert all(l % 8 == 0 for l in lengths), lengths   # adjacent runs may touch


def test_decode_ragged_lengths_and_diffuse_odd_sequences():
    w = SMALL_DEC.with_(B=4, seq_lens=(SMALL_DEC.T, 130, 1, 64 * 3), diffuse_odd=True)
    x = W.make_decode_inputs(w)
    assert x["seq_lens"].tolist() == list(w.seq_lens)
    for b in range(w.B):
        for g in range(w.Hkv):
            pos = _planted(x, w, b, g, _qhat_decode(x, w, b, g))
            assert len(pos) == min(w.hh_count, w.seq_lens[b])
            assert pos.max() < w.seq_lens[b]
    # odd sequences: queries drawn at half scale before rounding
    n = x["q"].float().norm(dim=-1)
    ratio = float(n[1::2].mean() / n[0::2].mean())
    assert 0.4 < ratio < 0.6


def test_prefill_inputs_are_seeded_and_planted():
    w = W.Workload("wl_prefill", "prefill", B=1, Hq=8, Hkv=2, d=64, T=64 * 10 + 3, hh_count=20,
                   seed=4)
    a, b = W.make_prefill_inputs(w), W.make_prefill_inputs(w)
    for k in ("q", "q_idx", "k_idx", "K", "V", "head_w"):
        assert torch.equal(a[k], b[k]), k
    assert a["q"].shape == (w.B, w.Hq, w.T, w.d)
    assert a["q_idx"].shape == (w.B, w.Hq, w.T, w.r)
    assert a["k_idx"].shape == (w.B, w.Hkv, w.T, w.r)
    for g in range(w.Hkv):
        m = a["q"][0, g * w.G:(g + 1) * w.G].float().mean(dim=(0, 1))
        qhat = m / m.norm()
        cos = _cos_rows(a["K"][0, g], qhat)
        assert int((cos > 0.9).sum()) == w.hh_count
