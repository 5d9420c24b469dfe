"""bsa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a host framework that owns every device allocation, a plugin whose
memory budget was fixed at start-up, a path where cudaMalloc would stall the
device) get the decode attention step with its split-K scratch in the library's
fixed device array instead of a workspace they would have to allocate. These
tests call it through the C ABI and compare it with bsa_decode, which takes a
caller-allocated workspace, on two calls in a row (the array keeps the previous
call's contents, which must not leak into the next result), and each call's
output with the fp64 oracle on every row.

This file is named to be collected last.
"""
import ctypes
from types import SimpleNamespace

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


def _inputs(w):
    x = W.make_decode_inputs(w, "cpu")
    return x, {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


@pytest.mark.parametrize("name,over", [
    ("decode_tiny_b1_h8_t4k", {}),
    ("decode_b8_h32_t32k_paged", dict(B=2, T=64 * 300 + 21, seq_lens=(64 * 300 + 21, 5000))),
])
def test_noalloc_matches_workspace_decode_on_two_calls(name, over):
    w = W.WORKLOADS[name].with_(**over)
    x, xd = _inputs(w)
    prob = bsa.problem_for(w, seq_lens=xd["seq_lens"], head_w=xd["head_w"])
    assert bsa.bsa_workspace_size(prob, bsa.OP_DECODE) <= bsa.NOALLOC_SCRATCH_BYTES

    # reference: score -> select -> bsa_decode with a caller-allocated workspace
    step = bsa.DecodeStep(prob)
    k_idx, K, V = bsa.caches_for(xd)
    step.run(xd["q"], xd["q_idx"], k_idx, K, V)
    torch.cuda.synchronize()
    assert int(step.status.item()) == 0

    for call in range(2):
        o = torch.full_like(step.o, float("nan"))
        lse = torch.full_like(step.lse, float("nan"))
        o32 = torch.full_like(step.o_f32, float("nan"))
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        bsa.bsa_decode_noalloc(prob, xd["q"], K, V, step.kept, step.kept_count, o, lse, o32,
                               status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, f"call {call}: device status {int(status.item()):#x}"
        errs = parity.attention_errors(o32.double().cpu().numpy(), None,
                                       lse.double().cpu().numpy(),
                                       step.o_f32.double().cpu().numpy(),
                                       step.lse.double().cpu().numpy())
        parity.check_attention(errs, f"no-alloc call {call}")
        assert parity.bf16_is_rne_of_f32(o.cpu(), o32.cpu())
        # and against the fp64 oracle, row by row
        out = SimpleNamespace(scores=step.scores, kept=step.kept, kept_count=step.kept_count,
                              o=o, o_f32=o32, lse=lse)
        rows = [(b, g) for b in range(w.B) for g in range(w.Hkv)]
        s = parity.compare_decode_rows(w, x, out, rows)
        assert s["rows"] == len(rows)


def test_noalloc_rejects_problems_beyond_the_scratch_size():
    # 1024 rows x G=16 heads x d=128 partials need more than the fixed array holds
    small = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
    prob = bsa.Problem(phase=bsa.PHASE_DECODE, B=128, Hq=128, Hkv=8, d=128, T=4096, n_sink=1,
                       n_local=2, k_max=64, p=0.9)
    assert bsa.bsa_workspace_size(prob, bsa.OP_DECODE) > bsa.NOALLOC_SCRATCH_BYTES
    cache = bsa.Cache(small, 0, 64 * 128, 0)
    lib = bsa.load_library()
    st = lib.bsa_decode_noalloc(ctypes.byref(prob.c()), ctypes.c_void_p(small.data_ptr()),
                                cache.c(), cache.c(), ctypes.c_void_p(small.data_ptr()),
                                ctypes.c_void_p(small.data_ptr()),
                                ctypes.c_void_p(small.data_ptr()),
                                ctypes.c_void_p(small.data_ptr()), None, None, None)
    assert st == bsa.BSA_ERR_WORKSPACE
