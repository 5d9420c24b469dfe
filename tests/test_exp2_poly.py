"""The FMA-pipe exp2 of the prefill softmax: its embedded cubic matches the Remez fit,
and the emulated float32 arithmetic stays within 1e-4 relative of 2^x on [-126, 8]
(the fp16 P it feeds has a rounding of 2^-11 ~ 4.9e-4)."""
import os
import re

import numpy as np

from block_sparse_long_06_b200 import exp2_poly_fit as F

SRC = os.path.join(os.path.dirname(os.path.dirname(__file__)), "block_sparse_long_06_b200",
                   "csrc", "prefill_tc.cu")


def embedded_coeffs():
    text = open(SRC).read()
    vals = {}
    for name in ("kC0", "kC1", "kC2", "kC3"):
        m = re.search(name + r"\s*=\s*([0-9.eE+-]+)f", text)
        vals[name] = float(m.group(1))
    return [vals["kC0"], vals["kC1"], vals["kC2"], vals["kC3"]]


def test_embedded_coefficients_match_the_fit():
    c, err = F.remez_exp2()
    assert err < 8e-5
    emb = embedded_coeffs()
    assert np.allclose(np.float32(c), np.float32(emb), rtol=0, atol=2e-7)


def test_emulated_exp2_relative_error():
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001), np.linspace(-1, 1, 100001)])
    got = F.emulate_exp2_f32(x, embedded_coeffs()).astype(np.float64)
    ref = 2.0 ** x.astype(np.float32).astype(np.float64)
    ok = ref > 2.0 ** -120          # far below fp16's range the value only has to be ~0
    rel = np.abs(got[ok] / ref[ok] - 1.0)
    assert rel.max() < 1e-4
    assert np.all(got[~ok] < 1e-30) and np.all(got >= 0)
