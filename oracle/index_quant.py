"""Plain CPU oracle of the microscaled 4-bit index-key cache.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The product path never imports or calls it, and it imports nothing
from the product.

Source: SpotAttention, Methodology §4 "quantisation": the selector's K cache
(the index keys) may be stored as microscaled INT4 or FP4, about 3.5x smaller
than bf16, while the backbone's K/V cache stays untouched. The page names the
idea and the ratio, not the format. Reading:

* a micro-block is one token's r = 16 index-key elements; it carries one FP8
  E4M3 scale (4 + 8/16 = 4.5 bits per element, 32 B -> 9 B per token = 3.56x,
  the page's "about 3.5x"); one fp32 scale g covers the whole cache so that the
  E4M3 scales stay in range;
* an element is a 4-bit sign-magnitude code: bit 3 = sign, bits 0-2 = a
  magnitude index. FP4 magnitudes are the E2M1 values (0, 0.5, 1, 1.5, 2, 3,
  4, 6) - the index is the E2M1 bit pattern; INT4 magnitudes are 0..7;
* the key of element c is  code_value(c) * e4m3_value(scale) * g.

Quantisation of one cache. Every step is float32 arithmetic with IEEE
round-to-nearest-even (numpy float32 operations), so the device quantiser, which
performs the same operations in the same order, takes the same integer
decisions. qmax = 6 (FP4) or 7 (INT4).

1. A = max |k| over every visible token (t < T_b) of every sequence and head;
   g = A / (qmax * 448) (one division by the exact constant), or 1 when A = 0.
2. Per token: a = max_c |k[c]|; s = (a / qmax) / g; the scale code is the
   E4M3 value nearest to s (ties to the even mantissa), clamped at 448.
3. S = that E4M3 value. If S = 0 every code is 0 (magnitude 0, sign of k).
   Otherwise t = S * g and, per element, x = k[c] / t; the magnitude index is
   the nearest grid magnitude to |x| (ties to the even index), clamped at the
   largest (6 or 7); the sign bit is the sign bit of k[c].
"""
from __future__ import annotations

import numpy as np

BLOCK = 64
R = 16
E4M3_MAX = 448.0
FORMATS = ("fp4", "int4")
QMAX = {"fp4": 6.0, "int4": 7.0}
MAGNITUDES = {
    "fp4": np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]),
    "int4": np.arange(8, dtype=np.float64),
}
RECORD_BYTES = BLOCK * 8 + BLOCK   # 64 tokens x 8 code bytes, then 64 scale bytes


def e4m3_table() -> tuple[np.ndarray, np.ndarray]:
    """All non-negative finite E4M3 values (bias 7, subnormals, no inf; 0x7F is
    NaN) and their byte codes, in increasing order."""
    codes, vals = [], []
    for c in range(0x7F):                       # 0x00 .. 0x7E
        e, m = c >> 3, c & 7
        v = m * 2.0 ** -9 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        codes.append(c)
        vals.append(v)
    return np.array(codes, dtype=np.uint8), np.array(vals)


_E4M3_CODES, _E4M3_VALS = e4m3_table()


def e4m3_value(code: int) -> float:
    return float(_E4M3_VALS[int(code) & 0x7F]) if (int(code) & 0x7F) != 0x7F else float("nan")


def e4m3_round(s: float) -> int:
    """Code of the E4M3 value nearest to s >= 0; ties to the even mantissa; values
    above 448 give 448 (saturating)."""
    s = float(s)
    if s >= E4M3_MAX:
        return int(_E4M3_CODES[-1])
    i = int(np.searchsorted(_E4M3_VALS, s))     # first value >= s
    if i < len(_E4M3_VALS) and _E4M3_VALS[i] == s:
        return int(_E4M3_CODES[i])
    lo, hi = i - 1, i
    dlo, dhi = s - _E4M3_VALS[lo], _E4M3_VALS[hi] - s
    if dlo < dhi:
        return int(_E4M3_CODES[lo])
    if dhi < dlo:
        return int(_E4M3_CODES[hi])
    return int(_E4M3_CODES[lo] if (_E4M3_CODES[lo] & 1) == 0 else _E4M3_CODES[hi])


def magnitude_index(x_abs: np.float32, fmt: str) -> int:
    """Nearest grid magnitude to x_abs >= 0 (ties to the even index), clamped."""
    grid = MAGNITUDES[fmt]
    x = float(x_abs)
    if x >= grid[-1]:
        return 7
    i = int(np.searchsorted(grid, x))
    if grid[i] == x:
        return i
    dlo, dhi = x - grid[i - 1], grid[i] - x
    if dlo < dhi:
        return i - 1
    if dhi < dlo:
        return i
    return i - 1 if (i - 1) % 2 == 0 else i


def gscale_of(amax: np.float32, fmt: str) -> np.float32:
    amax = np.float32(amax)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / np.float32(QMAX[fmt] * E4M3_MAX))


def quantize_token(k: np.ndarray, g: np.float32, fmt: str) -> tuple[np.ndarray, int]:
    """k: 16 float32 values (exactly the bf16 inputs). Returns the 16 codes
    (0..15, sign in bit 3) and the E4M3 scale code."""
    k = np.asarray(k, dtype=np.float32)
    a = np.float32(np.max(np.abs(k)))
    s = np.float32(np.float32(a / np.float32(QMAX[fmt])) / np.float32(g))
    sc = e4m3_round(s)
    S = np.float32(e4m3_value(sc))
    codes = np.zeros(R, dtype=np.int64)
    sign = np.signbit(k).astype(np.int64) << 3
    if S == 0:
        return codes | sign, sc
    t = np.float32(S * np.float32(g))
    for c in range(R):
        x = np.float32(k[c] / t)
        codes[c] = magnitude_index(np.float32(abs(x)), fmt)
    return codes | sign, sc


def _nearest_even(grid: np.ndarray, x: np.ndarray, top: int) -> np.ndarray:
    """Index of the grid value nearest to each x >= 0, ties to the even index,
    clamped at `top` (x beyond the grid saturates)."""
    i = np.clip(np.searchsorted(grid, x, side="left"), 1, len(grid) - 1)
    lo, hi = grid[i - 1], grid[i]
    dlo, dhi = x - lo, hi - x
    pick = np.where(dlo < dhi, i - 1, np.where(dhi < dlo, i, np.where((i - 1) % 2 == 0, i - 1, i)))
    pick = np.where(x <= grid[0], 0, pick)
    return np.where(x >= grid[-1], top, pick)


def quantize_rows(k: np.ndarray, g, fmt: str) -> tuple[np.ndarray, np.ndarray]:
    """quantize_token over many tokens at once: k [N, 16] (bf16-exact values), the
    same float32 steps elementwise. Returns codes [N, 16] and scale codes [N]."""
    k = np.asarray(k, dtype=np.float32)
    g = np.float32(g)
    a = np.max(np.abs(k), axis=1).astype(np.float32)
    s = ((a / np.float32(QMAX[fmt])).astype(np.float32) / g).astype(np.float32)
    vals64 = _E4M3_VALS
    sc_idx = _nearest_even(vals64, np.minimum(s.astype(np.float64), E4M3_MAX),
                           len(vals64) - 1)
    # ties to the even mantissa: the E4M3 table index parity is the mantissa parity
    sc = _E4M3_CODES[sc_idx]
    S = vals64[sc_idx].astype(np.float32)
    sign = np.signbit(k).astype(np.int64) << 3
    t = (S * g).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        x = np.abs((k / t[:, None]).astype(np.float32)).astype(np.float64)
    mag = _nearest_even(MAGNITUDES[fmt], np.nan_to_num(x, nan=0.0, posinf=1e30), 7)
    mag = np.where((S == 0)[:, None], 0, mag)
    return mag.astype(np.int64) | sign, sc.astype(np.uint8)


def cache_gscale(k_idx: np.ndarray, seq_lens, fmt: str) -> np.float32:
    """Step 1 alone: g from the maximum |k| over the visible tokens."""
    B, Hkv, T, _ = k_idx.shape
    lens = [T] * B if seq_lens is None else [int(x) for x in seq_lens]
    amax = np.float32(0.0)
    for b in range(B):
        if lens[b] > 0:
            amax = max(amax, np.float32(np.max(np.abs(k_idx[b, :, :lens[b]]))))
    return gscale_of(amax, fmt)


def quantize_cache(k_idx: np.ndarray, seq_lens, fmt: str):
    """k_idx [B, Hkv, T, 16] (bf16-exact values), seq_lens [B] or None.
    Returns codes [B, Hkv, nb*64, 16] int, scale codes [B, Hkv, nb*64] uint8 and g;
    tokens t >= T_b hold code 0 and scale code 0."""
    B, Hkv, T, r = k_idx.shape
    assert r == R
    lens = [T] * B if seq_lens is None else [int(x) for x in seq_lens]
    nb = -(-T // BLOCK)
    amax = np.float32(0.0)
    for b in range(B):
        if lens[b] > 0:
            amax = max(amax, np.float32(np.max(np.abs(k_idx[b, :, :lens[b]].astype(np.float32)))))
    g = gscale_of(amax, fmt)
    codes = np.zeros((B, Hkv, nb * BLOCK, R), dtype=np.int64)
    scales = np.zeros((B, Hkv, nb * BLOCK), dtype=np.uint8)
    for b in range(B):
        for h in range(Hkv):
            for t in range(lens[b]):
                codes[b, h, t], scales[b, h, t] = quantize_token(k_idx[b, h, t], g, fmt)
    return codes, scales, g


def dequantize(codes: np.ndarray, scales: np.ndarray, g, fmt: str) -> np.ndarray:
    """Keys in float64: code value * E4M3 scale * g (exact)."""
    mag = MAGNITUDES[fmt][codes & 7]
    val = np.where((codes >> 3) & 1, -mag, mag)
    sv = np.vectorize(e4m3_value)(scales).astype(np.float64)
    return val * sv[..., None] * float(g)


def pack_records(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Byte image of the cache as [B, Hkv, nb] records of 576 bytes: per block,
    64 tokens x 8 bytes (byte c = code[2c] | code[2c+1] << 4), then 64 scales."""
    B, Hkv, Tp, _ = codes.shape
    nb = Tp // BLOCK
    c = codes.reshape(B, Hkv, nb, BLOCK, 8, 2)
    byts = (c[..., 0] | (c[..., 1] << 4)).astype(np.uint8).reshape(B, Hkv, nb, BLOCK * 8)
    return np.concatenate([byts, scales.reshape(B, Hkv, nb, BLOCK)], axis=-1)
