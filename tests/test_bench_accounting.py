"""The bench's algorithmic byte and FLOP counts (the numerators of its roofline fractions),
checked against brute-force enumeration of what one decode step or one prefill touches.

Decode: every index key of every visible token (bf16: 16 values of 2 bytes; 4-bit: one
576-byte record per visible 64-token block), K and V of every kept block, q, q_idx, the
bf16 output and fp32 LSE, and one page-table entry per kept block in a paged cache.
Prefill: 4 * 64 * 64 * d FLOP per kept (tile, query head) (two 64x64xd products, 2 FLOP a
multiply-add), and the causal-exact count of the (query, key) pairs a causal mask leaves
visible, 4 * d FLOP per pair and head.
"""
import numpy as np
import pytest
import torch

import bench
from block_sparse_long_06_b200 import workloads as W


def _brute_decode_bytes(w, kept_count, seq_lens, fmt):
    total = 0
    kv = 0
    for b in range(w.B):
        T_b = int(seq_lens[b])
        for g in range(w.Hkv):
            if fmt == "bf16":
                total += T_b * w.r * 2                        # one index key per token
            else:
                total += ((T_b + 63) // 64) * 576              # one record per visible block
            for _ in range(int(kept_count[b, g])):
                blk = 2 * (64 * w.d * 2)                       # K and V tiles of a block
                kv += blk
                total += blk + (4 if w.paged else 0)           # + its page-table entry
    if fmt != "bf16":
        total += 4                                             # the cache scale g
    for _ in range(w.B * w.Hq):
        total += w.d * 2 + w.r * 2                             # q and q_idx of a head
        total += w.d * 2 + 4                                   # o (bf16) and lse (fp32)
    return total, kv


@pytest.mark.parametrize("fmt", ["bf16", "fp4"])
@pytest.mark.parametrize("paged", [False, True])
def test_decode_bytes_match_enumeration(fmt, paged):
    w = W.WORKLOADS["decode_tiny_b1_h8_t4k"].with_(B=3, paged=paged, T=64 * 9 + 11)
    rng = np.random.default_rng(5)
    kept = torch.from_numpy(rng.integers(0, 12, size=(w.B, w.Hkv)).astype(np.int32))
    lens = torch.tensor([w.T, 64 * 4 + 1, 64 * 7], dtype=torch.int32)
    got = bench.decode_bytes(w, kept, lens, fmt)
    want, kv = _brute_decode_bytes(w, kept, lens, fmt)
    assert got["step"] == want
    assert got["kv"] == kv
    # the attention call reads K/V, q and page ids and writes o and lse, but no index key
    idx = sum(int(lens[b]) * w.Hkv * w.r * 2 for b in range(w.B)) if fmt == "bf16" else \
        sum(((int(lens[b]) + 63) // 64) * w.Hkv * 576 for b in range(w.B)) + 4
    assert got["index_keys"] == idx
    assert got["attention"] == want - idx - w.B * w.Hq * w.r * 2


def _brute_prefill_flops(w, kept_lists):
    """kept_lists[(b, g, i)] = kept key blocks of query block i (the diagonal included)."""
    tiles = 0
    pairs = 0
    for (b, g, i), blocks in kept_lists.items():
        for j in blocks:
            tiles += 1
            for tq in range(64 * i, min(64 * (i + 1), w.T)):
                for tk in range(64 * j, min(64 * (j + 1), w.T)):
                    if tk <= tq:
                        pairs += 1
    G = w.Hq // w.Hkv
    return tiles * G * 4 * 64 * 64 * w.d, pairs * G * 4 * w.d


def test_prefill_flops_match_enumeration():
    w = W.Workload("acct_prefill", "prefill", B=1, Hq=4, Hkv=2, d=64, T=64 * 5 + 9,
                   n_sink=1, n_local=1, p=1.0, k_max=2, seed=3)
    rng = np.random.default_rng(9)
    kept_lists, kc = {}, np.zeros((w.B, w.Hkv, w.nb), dtype=np.int32)
    for b in range(w.B):
        for g in range(w.Hkv):
            for i in range(w.nb):
                others = list(rng.choice(i, size=min(i, int(rng.integers(0, 4))), replace=False)) \
                    if i > 0 else []
                kept_lists[(b, g, i)] = sorted(others) + [i]   # the diagonal is always kept
                kc[b, g, i] = len(others) + 1
    tiles, exact = bench.prefill_flops(w, torch.from_numpy(kc))
    want_tiles, want_exact = _brute_prefill_flops(w, kept_lists)
    assert tiles == want_tiles
    assert exact == want_exact
