"""Pins of the 4-bit index-key cache oracle (oracle/index_quant.py).

Source: SpotAttention, Methodology §4 (microscaled INT4/FP4 selector K cache).
Each check pins the oracle to something other than itself: a library routine
(torch's float8_e4m3fn conversion), hand-derived values (tests/golden), or a
bound that follows from the format.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import index_quant as iq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "index_quant.json")


def _bf16(x):
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def test_e4m3_round_matches_torch():
    _, vals = iq.e4m3_table()
    mids = (vals[1:] + vals[:-1]) / 2                     # every tie
    rnd = np.exp(np.random.default_rng(1).uniform(np.log(2.0 ** -12), np.log(448.0), 5000))
    xs = np.concatenate([vals, mids, rnd]).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).float().numpy()
    got = np.array([iq.e4m3_value(iq.e4m3_round(x)) for x in xs])
    assert np.array_equal(ref, got)


def test_e4m3_saturates_and_underflows():
    assert iq.e4m3_value(iq.e4m3_round(448.0)) == 448.0
    assert iq.e4m3_value(iq.e4m3_round(470.0)) == 448.0      # satfinite, not NaN
    assert iq.e4m3_value(iq.e4m3_round(1e30)) == 448.0
    assert iq.e4m3_round(2.0 ** -10) == 0                     # tie with 0 -> even (0)
    assert iq.e4m3_value(iq.e4m3_round(3 * 2.0 ** -10)) == 2.0 ** -8   # tie 1 vs 2 subnormal steps -> 2
    assert iq.e4m3_round(0.0) == 0


@pytest.mark.parametrize("fmt,cases", [
    ("fp4", [(0.0, 0), (0.25, 0), (0.2501, 1), (0.5, 1), (0.7499, 1), (0.75, 2), (1.25, 2),
             (1.2501, 3), (1.75, 4), (2.5, 4), (2.5001, 5), (3.5, 6), (5.0, 6), (5.0001, 7),
             (6.0, 7), (100.0, 7)]),
    ("int4", [(0.0, 0), (0.5, 0), (0.5001, 1), (1.5, 2), (2.5, 2), (3.5, 4), (6.5, 6), (6.5001, 7),
              (7.5, 7), (100.0, 7)]),
])
def test_magnitude_rounding_table(fmt, cases):
    for x, idx in cases:
        assert iq.magnitude_index(np.float32(x), fmt) == idx, (fmt, x)


def _golden_check(mod):
    G = json.load(open(GOLDEN))
    for fmt in ("fp4", "int4"):
        c = G[fmt]
        k = np.array(c["k"], dtype=np.float32)
        assert np.array_equal(_bf16(k), k)
        codes, scales, g = mod.quantize_cache(k[None, None], None, fmt)
        n = len(k)
        if float(g) != c["g"]:
            return False
        if scales[0, 0, :n].tolist() != c["scale_codes"]:
            return False
        if codes[0, 0, :n].tolist() != c["codes"]:
            return False
    return True


def test_golden_hand_derived():
    assert _golden_check(iq)


def test_dequantized_error_bound():
    rng = np.random.default_rng(2)
    k = _bf16(rng.standard_normal((2, 3, 200, 16)) * rng.uniform(0.01, 5.0, (2, 3, 200, 1)))
    for fmt, half_gap in (("fp4", 1.0), ("int4", 0.5)):
        codes, scales, g = iq.quantize_cache(k, [200, 137], fmt)
        deq = iq.dequantize(codes, scales, g, fmt)
        sv = np.vectorize(iq.e4m3_value)(scales) * float(g)            # t per token
        for b, T in enumerate((200, 137)):
            err = np.abs(deq[b, :, :T] - k[b, :, :T])
            # rounding to the grid costs at most half the widest gap, times t
            assert np.all(err <= half_gap * sv[b, :, :T, None] * (1 + 1e-6))
            assert np.all(deq[b, :, T:] == 0.0) and np.all(codes[b, :, T:] == 0)
        # the largest token uses the top of the E4M3 range
        assert scales.max() == 0x7E


def test_pack_records_layout():
    codes = np.zeros((1, 1, 64, 16), dtype=np.int64)
    codes[0, 0, 0] = np.arange(16)
    scales = np.zeros((1, 1, 64), dtype=np.uint8)
    scales[0, 0, 0], scales[0, 0, 63] = 0x7E, 0x11
    rec = iq.pack_records(codes, scales)
    assert rec.shape == (1, 1, 1, iq.RECORD_BYTES)
    # byte c of token 0 = code[2c] | code[2c+1] << 4
    assert rec[0, 0, 0, :8].tolist() == [0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE]
    assert rec[0, 0, 0, 512] == 0x7E and rec[0, 0, 0, 575] == 0x11


class _Mutant:
    """A copy of the oracle module with one function replaced."""

    def __init__(self, **over):
        self.__dict__.update({k: getattr(iq, k) for k in dir(iq) if not k.startswith("__")})
        self.__dict__.update(over)
        # functions look names up in their own module: rebind the ones that call others
        def quantize_token(k, g, fmt):
            k = np.asarray(k, dtype=np.float32)
            a = np.float32(np.max(np.abs(k)))
            s = np.float32(np.float32(a / np.float32(self.QMAX[fmt])) / np.float32(g))
            sc = self.e4m3_round(s)
            S = np.float32(self.e4m3_value(sc))
            codes = np.zeros(16, dtype=np.int64)
            sign = self.signs(k)
            if S == 0:
                return codes | sign, sc
            t = np.float32(S * np.float32(g))
            for c in range(16):
                codes[c] = self.magnitude_index(np.float32(abs(np.float32(k[c] / t))), fmt)
            return codes | sign, sc

        def quantize_cache(k_idx, seq_lens, fmt):
            B, Hkv, T, _ = k_idx.shape
            amax = np.float32(np.max(np.abs(k_idx.astype(np.float32))))
            g = self.gscale_of(amax, fmt)
            nb = -(-T // 64)
            codes = np.zeros((B, Hkv, nb * 64, 16), dtype=np.int64)
            scales = np.zeros((B, Hkv, nb * 64), dtype=np.uint8)
            for b in range(B):
                for h in range(Hkv):
                    for t in range(T):
                        codes[b, h, t], scales[b, h, t] = quantize_token(k_idx[b, h, t], g, fmt)
            return codes, scales, g
        self.signs = over.get("signs", lambda k: np.signbit(k).astype(np.int64) << 3)
        self.quantize_cache = quantize_cache


def _ties_away(x_abs, fmt):
    grid = iq.MAGNITUDES[fmt]
    x = float(x_abs)
    if x >= grid[-1]:
        return 7
    i = int(np.searchsorted(grid, x))
    if grid[i] == x:
        return i
    return i - 1 if x - grid[i - 1] < grid[i] - x else i


def _e4m3_floor(s):
    _, vals = iq.e4m3_table()
    return int(np.searchsorted(vals, min(float(s), 448.0), side="right") - 1)


@pytest.mark.parametrize("name,over", [
    ("magnitude ties away from zero", {"magnitude_index": _ties_away}),
    ("E4M3 scale truncated instead of rounded", {"e4m3_round": _e4m3_floor}),
    ("qmax of INT4 used for FP4", {"QMAX": {"fp4": 7.0, "int4": 7.0}}),
    ("global scale without the 448", {"gscale_of": lambda a, f: np.float32(a / np.float32(iq.QMAX[f]))}),
    ("sign of -0 dropped", {"signs": lambda k: ((k < 0).astype(np.int64)) << 3}),
])
def test_mutants_are_caught(name, over):
    assert _golden_check(iq)
    assert not _golden_check(_Mutant(**over)), name


def test_vectorised_quantiser_agrees_with_token_form():
    """quantize_rows (used on full-size caches) takes the same decisions as
    quantize_token, which the goldens and torch pin."""
    rng = np.random.default_rng(4)
    k = _bf16(rng.standard_normal((2000, 16)) * rng.uniform(1e-5, 20.0, (2000, 1)))
    k[0] = 0.0
    k[1] = 2.0 ** -20
    k[2, 5] = -0.0
    G = json.load(open(GOLDEN))
    for fmt in ("fp4", "int4"):
        g = iq.gscale_of(np.max(np.abs(k)), fmt)
        cv, sv = iq.quantize_rows(k, g, fmt)
        for n in range(len(k)):
            c, sc = iq.quantize_token(k[n], g, fmt)
            assert sc == sv[n] and np.array_equal(c, cv[n]), (fmt, n)
        gk = np.array(G[fmt]["k"], dtype=np.float32)
        cg, sg = iq.quantize_rows(gk, np.float32(G[fmt]["g"]), fmt)
        assert cg.tolist() == G[fmt]["codes"] and sg.tolist() == G[fmt]["scale_codes"]
