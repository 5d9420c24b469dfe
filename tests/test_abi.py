"""The C-ABI library loads on a machine without a GPU, exports every entry point
declared in include/bsa.h, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import block_sparse_long_06_b200 as bsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "bsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(bsa_[a-z_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(bsa.LIB_PATH):
        from block_sparse_long_06_b200 import build
        build.build()
    return bsa.load_library()


def test_header_declares_the_four_steps():
    names = declared_functions()
    for n in ("bsa_score_blocks", "bsa_select_top_p", "bsa_decode", "bsa_prefill"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), f"{n} not exported"
    assert sorted(bsa.EXPORTED) == names


def _prob(**kw):
    base = dict(phase=bsa.PHASE_DECODE, B=2, Hq=8, Hkv=2, d=128, T=4096, n_sink=1, n_local=2,
                k_max=16, p=0.9)
    base.update(kw)
    return bsa.Problem(**base)


def test_max_kept(lib):
    assert bsa.bsa_max_kept(_prob()) == 1 + 2 + 16
    assert bsa.bsa_max_kept(_prob(phase=bsa.PHASE_PREFILL)) == 1 + 1 + 2 + 16


def test_workspace_size_host_only(lib):
    assert bsa.bsa_workspace_size(_prob(), bsa.OP_SCORE) == 0
    assert bsa.bsa_workspace_size(_prob(), bsa.OP_SELECT) == 0
    assert bsa.bsa_workspace_size(_prob(), bsa.OP_DECODE) > 0
    pf = _prob(phase=bsa.PHASE_PREFILL, T=1000)
    assert bsa.bsa_workspace_size(pf, bsa.OP_PREFILL) >= 2 * 2 * 1024 * 128 * 2


@pytest.mark.parametrize("kw,code", [
    (dict(Hq=6, Hkv=4), bsa.BSA_ERR_INVALID_ARG),        # Hq % Hkv != 0
    (dict(Hq=12, Hkv=4), bsa.BSA_ERR_UNSUPPORTED),       # G = 3
    (dict(d=96), bsa.BSA_ERR_UNSUPPORTED),
    (dict(r=32), bsa.BSA_ERR_UNSUPPORTED),
    (dict(k_min=5, k_max=4), bsa.BSA_ERR_INVALID_ARG),
    (dict(k_max=9000), bsa.BSA_ERR_UNSUPPORTED),
    (dict(p=float("nan")), bsa.BSA_ERR_INVALID_ARG),
    (dict(B=0), bsa.BSA_ERR_INVALID_ARG),
    (dict(T=64 * 40000), bsa.BSA_ERR_UNSUPPORTED),
    (dict(group_size=8, k_groups=4), bsa.BSA_ERR_UNSUPPORTED),     # groups of 16, 32, 64
    (dict(group_size=16, k_groups=-1), bsa.BSA_ERR_INVALID_ARG),
    (dict(group_size=16, k_groups=4, k_max=4096), bsa.BSA_ERR_UNSUPPORTED),   # > 8192 groups
])
def test_invalid_problems_rejected(lib, kw, code):
    out = ctypes.c_size_t(0)
    st = lib.bsa_workspace_size(ctypes.byref(_prob(**kw).c()), bsa.OP_DECODE, ctypes.byref(out))
    assert st == code


def test_null_pointers_rejected_before_launch(lib):
    p = _prob().c()
    st = lib.bsa_score_blocks(ctypes.byref(p), None, bsa.CCache(), None, None, None)
    assert st == bsa.BSA_ERR_INVALID_ARG
    st = lib.bsa_select_top_p(ctypes.byref(p), None, None, None, None, None)
    assert st == bsa.BSA_ERR_INVALID_ARG
    st = lib.bsa_decode(ctypes.byref(p), None, bsa.CCache(), bsa.CCache(), None, None, None, None,
                        None, None, 0, None, None)
    assert st == bsa.BSA_ERR_INVALID_ARG
    st = lib.bsa_prefill(ctypes.byref(p), None, bsa.CCache(), bsa.CCache(), None, None, None, None,
                         None, None, 0, None, None)
    assert st == bsa.BSA_ERR_INVALID_ARG   # decode problem passed to prefill


def test_status_strings(lib):
    for s in range(5):
        assert bsa.bsa_status_string(s)


def _qcache(fmt=bsa.IDX_FP4, records=0x10000, gscale=0x20000):
    return bsa.CQCache(records, gscale, 2 * 64, 1, 64, None, 0, 0, 2 * 2 * 64, fmt)


def _kcache(base=0x30000):
    return bsa.CCache(base, 2 * 4096 * 16, 64 * 16, 4096 * 16, None, 0, 0, 2 * 2 * 4096 * 16)


def test_qcache_entry_points_reject_on_host(lib):
    """Host checks of the 4-bit index-key entry points (no pointer is dereferenced)."""
    p = _prob().c()
    pf = _prob(phase=bsa.PHASE_PREFILL).c()
    # prefill problems are not supported by the 4-bit path
    assert lib.bsa_score_blocks_q(ctypes.byref(pf), 0x40000, _qcache(), 0x50000, None,
                                  None) == bsa.BSA_ERR_UNSUPPORTED
    assert lib.bsa_quantize_index_keys(ctypes.byref(pf), _kcache(), _qcache(), None,
                                       None) == bsa.BSA_ERR_UNSUPPORTED
    # unknown format, missing scale, unaligned records
    for bad in (_qcache(fmt=3), _qcache(gscale=None), _qcache(records=0x10008)):
        assert lib.bsa_score_blocks_q(ctypes.byref(p), 0x40000, bad, 0x50000, None,
                                      None) == bsa.BSA_ERR_INVALID_ARG
        assert lib.bsa_quantize_index_keys(ctypes.byref(p), _kcache(), bad, None,
                                           None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_score_blocks_q(ctypes.byref(p), None, _qcache(), 0x50000, None,
                                  None) == bsa.BSA_ERR_INVALID_ARG


def test_group_routing_rejects_on_host(lib):
    """Two-level routing: decode only, and each step needs its group buffers."""
    pf = _prob(phase=bsa.PHASE_PREFILL, group_size=16, k_groups=4).c()
    out = ctypes.c_size_t(0)
    assert lib.bsa_workspace_size(ctypes.byref(pf), bsa.OP_PREFILL,
                                  ctypes.byref(out)) == bsa.BSA_ERR_INVALID_ARG
    p = _prob(group_size=16, k_groups=4).c()          # group_scores / kept_groups null
    assert lib.bsa_score_blocks(ctypes.byref(p), 0x40000, _kcache(), 0x50000, None,
                                None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_score_blocks_q(ctypes.byref(p), 0x40000, _qcache(), 0x50000, None,
                                  None) == bsa.BSA_ERR_INVALID_ARG
    assert lib.bsa_select_top_p(ctypes.byref(p), 0x50000, 0x60000, 0x70000, None,
                                None) == bsa.BSA_ERR_INVALID_ARG
    p.group_scores = 0x80000                          # kept_groups still null
    assert lib.bsa_select_top_p(ctypes.byref(p), 0x50000, 0x60000, 0x70000, None,
                                None) == bsa.BSA_ERR_INVALID_ARG
