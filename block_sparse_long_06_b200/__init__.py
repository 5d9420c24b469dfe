"""Python binding of libbsa.so: dynamic block-sparse attention on B200 (sm_100a).

Thin ctypes marshalling over the C ABI in include/bsa.h. Every step of the method
runs in the library's CUDA kernels; torch only owns device memory and streams.
Importing this package does not load the library; the first call does, and it
raises if libbsa.so is missing (build it with ``python -m
block_sparse_long_06_b200.build``). There is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libbsa.so")

BSA_OK, BSA_ERR_INVALID_ARG, BSA_ERR_UNSUPPORTED, BSA_ERR_WORKSPACE, BSA_ERR_CUDA = range(5)
BSA_DEV_BAD_PAGE, BSA_DEV_BAD_KEPT, BSA_DEV_NONFINITE, BSA_DEV_TIMEOUT, BSA_DEV_FP16_RANGE = (
    0x1, 0x2, 0x4, 0x8, 0x10)
PHASE_DECODE, PHASE_PREFILL = 0, 1
OP_SCORE, OP_SELECT, OP_DECODE, OP_PREFILL, OP_PBS_PERMUTE = 0, 1, 2, 3, 4
BLOCK = 64

EXPORTED = ["bsa_max_kept", "bsa_workspace_size", "bsa_score_blocks", "bsa_select_top_p",
            "bsa_decode", "bsa_prefill", "bsa_status_string", "bsa_last_cuda_error",
            "bsa_decode_noalloc", "bsa_quantize_index_keys", "bsa_score_blocks_q",
            "bsa_pbs_permute"]
NOALLOC_SCRATCH_BYTES = 8 << 20
IDX_FP4, IDX_INT4 = 1, 2
QIDX_RECORD_BYTES = 576


class BsaError(RuntimeError):
    pass


class CCache(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("seq_stride", ctypes.c_int64),
                ("block_stride", ctypes.c_int64), ("head_stride", ctypes.c_int64),
                ("page_table", ctypes.c_void_p), ("page_table_stride", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("extent", ctypes.c_int64)]


class CQCache(ctypes.Structure):
    _fields_ = [("records", ctypes.c_void_p), ("gscale", ctypes.c_void_p),
                ("seq_stride", ctypes.c_int64), ("block_stride", ctypes.c_int64),
                ("head_stride", ctypes.c_int64), ("page_table", ctypes.c_void_p),
                ("page_table_stride", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("extent", ctypes.c_int64), ("format", ctypes.c_int32)]


class CProblem(ctypes.Structure):
    _fields_ = [("phase", ctypes.c_int32), ("B", ctypes.c_int32), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32), ("r", ctypes.c_int32),
                ("block", ctypes.c_int32), ("T", ctypes.c_int32), ("seq_lens", ctypes.c_void_p),
                ("n_sink", ctypes.c_int32), ("n_local", ctypes.c_int32),
                ("k_max", ctypes.c_int32), ("k_min", ctypes.c_int32), ("p", ctypes.c_float),
                ("idx_scale", ctypes.c_float), ("attn_scale", ctypes.c_float),
                ("head_w", ctypes.c_void_p), ("head_p", ctypes.c_void_p),
                ("idx_heads", ctypes.c_int32), ("segment", ctypes.c_int32),
                ("key_pos", ctypes.c_void_p), ("group_size", ctypes.c_int32),
                ("k_groups", ctypes.c_int32), ("group_scores", ctypes.c_void_p),
                ("kept_groups", ctypes.c_void_p)]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libbsa.so once and declare its signatures; raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise BsaError(f"{path} not found: build it with `python -m block_sparse_long_06_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(CProblem)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.bsa_max_kept.argtypes = [P]
    lib.bsa_max_kept.restype = ctypes.c_int32
    lib.bsa_workspace_size.argtypes = [P, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
    lib.bsa_workspace_size.restype = ctypes.c_int
    lib.bsa_score_blocks.argtypes = [P, vp, CCache, vp, vp, vp]
    lib.bsa_score_blocks.restype = ctypes.c_int
    lib.bsa_select_top_p.argtypes = [P, vp, vp, vp, vp, vp]
    lib.bsa_select_top_p.restype = ctypes.c_int
    for name in ("bsa_decode", "bsa_prefill"):
        f = getattr(lib, name)
        f.argtypes = [P, vp, CCache, CCache, vp, vp, vp, vp, vp, vp, sz, vp, vp]
        f.restype = ctypes.c_int
    lib.bsa_decode_noalloc.argtypes = [P, vp, CCache, CCache, vp, vp, vp, vp, vp, vp, vp]
    lib.bsa_decode_noalloc.restype = ctypes.c_int
    lib.bsa_quantize_index_keys.argtypes = [P, CCache, CQCache, vp, vp]
    lib.bsa_quantize_index_keys.restype = ctypes.c_int
    lib.bsa_score_blocks_q.argtypes = [P, vp, CQCache, vp, vp, vp]
    lib.bsa_score_blocks_q.restype = ctypes.c_int
    lib.bsa_pbs_permute.argtypes = [P, vp, CCache, CCache, CCache, vp, vp, vp, vp, vp, sz, vp, vp]
    lib.bsa_pbs_permute.restype = ctypes.c_int
    lib.bsa_status_string.argtypes = [ctypes.c_int]
    lib.bsa_status_string.restype = ctypes.c_char_p
    lib.bsa_last_cuda_error.argtypes = []
    lib.bsa_last_cuda_error.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(status: int, what: str):
    if status != BSA_OK:
        lib = load_library()
        msg = lib.bsa_status_string(status).decode()
        if status == BSA_ERR_CUDA:
            msg += ": " + lib.bsa_last_cuda_error().decode()
        raise BsaError(f"{what}: {msg} (status {status})")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


# ------------------------------------------------------------------ problem / caches
@dataclass
class Problem:
    phase: int
    B: int
    Hq: int
    Hkv: int
    d: int
    T: int
    n_sink: int
    n_local: int
    k_max: int
    p: float
    k_min: int = 0
    r: int = 16
    block: int = BLOCK
    idx_scale: float = 0.0        # 0 -> 1/sqrt(r)
    attn_scale: float = 0.0       # 0 -> 1/sqrt(d)
    seq_lens: Optional[torch.Tensor] = None   # device int32 [B] (decode)
    head_w: Optional[torch.Tensor] = None     # device float32 [Hq]
    head_p: Optional[torch.Tensor] = None     # device float32 [Hkv]: per-kv-head p (<= 0: local head)
    idx_heads: int = 0                        # 0: an index head per query head; 1: one per kv group
    segment: int = 0                          # prefill: PBS segment length in tokens (0: none)
    key_pos: Optional[torch.Tensor] = None    # prefill with segment: device int32 [B, Hkv, T]
    group_size: int = 0                       # decode: two-level routing group (16/32/64; 0: off)
    k_groups: int = 0                         # decode with group_size: kept groups per row
    group_scores: Optional[torch.Tensor] = None   # device float32 [B, Hkv, nb * 64 / group_size]
    kept_groups: Optional[torch.Tensor] = None    # device int32 [B, Hkv, max_kept] bitmasks

    @property
    def G(self):
        return self.Hq // self.Hkv

    @property
    def nb(self):
        return (self.T + BLOCK - 1) // BLOCK

    def c(self) -> CProblem:
        return CProblem(self.phase, self.B, self.Hq, self.Hkv, self.d, self.r, self.block, self.T,
                        _ptr(self.seq_lens), self.n_sink, self.n_local, self.k_max, self.k_min,
                        float(self.p), float(self.idx_scale), float(self.attn_scale),
                        _ptr(self.head_w), _ptr(self.head_p), int(self.idx_heads),
                        int(self.segment), _ptr(self.key_pos), int(self.group_size),
                        int(self.k_groups), _ptr(self.group_scores), _ptr(self.kept_groups))


@dataclass
class Cache:
    """A bf16 cache tensor (K, V or index keys) and its addressing (bsa_cache_t)."""
    tensor: torch.Tensor
    seq_stride: int
    block_stride: int
    head_stride: int
    page_table: Optional[torch.Tensor] = None
    num_pages: int = 0

    def c(self) -> CCache:
        pt = self.page_table
        return CCache(self.tensor.data_ptr(), self.seq_stride, self.block_stride, self.head_stride,
                      None if pt is None else pt.data_ptr(),
                      0 if pt is None else pt.shape[1], self.num_pages, self.tensor.numel())


def contiguous_cache(t: torch.Tensor) -> Cache:
    """[B, Hkv, T, w] contiguous bf16 tensor."""
    assert t.is_contiguous() and t.dtype == torch.bfloat16 and t.dim() == 4
    B, H, T, w = t.shape
    return Cache(t, H * T * w, BLOCK * w, T * w)


def paged_cache(pool: torch.Tensor, page_table: torch.Tensor) -> Cache:
    """[P, Hkv, 64, w] contiguous bf16 pool with a [B, nb] int32 page table."""
    assert pool.is_contiguous() and pool.dtype == torch.bfloat16 and pool.shape[2] == BLOCK
    assert page_table.dtype == torch.int32 and page_table.is_contiguous()
    P, H, _, w = pool.shape
    return Cache(pool, 0, H * BLOCK * w, BLOCK * w, page_table, P)


@dataclass
class QCache:
    """A 4-bit index-key cache (bsa_qcache_t): 576-byte records of 64 tokens, plus
    the cache scale. `records` is a uint8 tensor, `gscale` a float32 [1] tensor."""
    records: torch.Tensor
    gscale: torch.Tensor
    fmt: int
    seq_stride: int
    block_stride: int
    head_stride: int
    page_table: Optional[torch.Tensor] = None
    num_pages: int = 0

    def c(self) -> CQCache:
        pt = self.page_table
        return CQCache(self.records.data_ptr(), self.gscale.data_ptr(), self.seq_stride,
                       self.block_stride, self.head_stride, None if pt is None else pt.data_ptr(),
                       0 if pt is None else pt.shape[1], self.num_pages,
                       self.records.numel() // QIDX_RECORD_BYTES, self.fmt)


def contiguous_qcache(B: int, Hkv: int, T: int, fmt: int, device=None) -> QCache:
    """Zeroed [B, Hkv, nb] records (nb = ceil(T/64))."""
    nb = (T + BLOCK - 1) // BLOCK
    rec = torch.zeros(B * Hkv * nb * QIDX_RECORD_BYTES, dtype=torch.uint8, device=device)
    gs = torch.zeros(1, dtype=torch.float32, device=device)
    return QCache(rec, gs, fmt, Hkv * nb, 1, nb)


def paged_qcache(num_pages: int, Hkv: int, page_table: torch.Tensor, fmt: int, device=None) -> QCache:
    """Zeroed [P, Hkv] records addressed through a [B, nb] int32 page table."""
    assert page_table.dtype == torch.int32 and page_table.is_contiguous()
    rec = torch.zeros(num_pages * Hkv * QIDX_RECORD_BYTES, dtype=torch.uint8, device=device)
    gs = torch.zeros(1, dtype=torch.float32, device=device)
    return QCache(rec, gs, fmt, 0, Hkv, 1, page_table, num_pages)


# ------------------------------------------------------------------ the C entry points
def bsa_max_kept(prob: Problem) -> int:
    return load_library().bsa_max_kept(ctypes.byref(prob.c()))


def bsa_workspace_size(prob: Problem, op: int) -> int:
    out = ctypes.c_size_t(0)
    _check(load_library().bsa_workspace_size(ctypes.byref(prob.c()), op, ctypes.byref(out)),
           "bsa_workspace_size")
    return out.value


def bsa_score_blocks(prob: Problem, q_idx, k_idx: Cache, block_scores, dev_status=None,
                     stream=None):
    _check(load_library().bsa_score_blocks(ctypes.byref(prob.c()), _ptr(q_idx), k_idx.c(),
                                           _ptr(block_scores), _ptr(dev_status), _stream(stream)),
           "bsa_score_blocks")


def bsa_quantize_index_keys(prob: Problem, k_idx: Cache, out: QCache, dev_status=None,
                            stream=None):
    _check(load_library().bsa_quantize_index_keys(ctypes.byref(prob.c()), k_idx.c(), out.c(),
                                                  _ptr(dev_status), _stream(stream)),
           "bsa_quantize_index_keys")


def bsa_score_blocks_q(prob: Problem, q_idx, k_idx: QCache, block_scores, dev_status=None,
                       stream=None):
    _check(load_library().bsa_score_blocks_q(ctypes.byref(prob.c()), _ptr(q_idx), k_idx.c(),
                                             _ptr(block_scores), _ptr(dev_status), _stream(stream)),
           "bsa_score_blocks_q")


def bsa_select_top_p(prob: Problem, block_scores, kept, kept_count, dev_status=None, stream=None):
    _check(load_library().bsa_select_top_p(ctypes.byref(prob.c()), _ptr(block_scores), _ptr(kept),
                                           _ptr(kept_count), _ptr(dev_status), _stream(stream)),
           "bsa_select_top_p")


def bsa_decode(prob: Problem, q, k: Cache, v: Cache, kept, kept_count, o, lse, o_f32, workspace,
               dev_status=None, stream=None):
    _check(load_library().bsa_decode(ctypes.byref(prob.c()), _ptr(q), k.c(), v.c(), _ptr(kept),
                                     _ptr(kept_count), _ptr(o), _ptr(lse), _ptr(o_f32),
                                     _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                     _ptr(dev_status), _stream(stream)),
           "bsa_decode")


def bsa_prefill(prob: Problem, q, k: Cache, v: Cache, kept, kept_count, o, lse, o_f32, workspace,
                dev_status=None, stream=None):
    _check(load_library().bsa_prefill(ctypes.byref(prob.c()), _ptr(q), k.c(), v.c(), _ptr(kept),
                                      _ptr(kept_count), _ptr(o), _ptr(lse), _ptr(o_f32),
                                      _ptr(workspace), 0 if workspace is None else workspace.numel(),
                                      _ptr(dev_status), _stream(stream)),
           "bsa_prefill")


def bsa_decode_noalloc(prob: Problem, q, k: Cache, v: Cache, kept, kept_count, o, lse, o_f32,
                       dev_status=None, stream=None):
    """bsa_decode without a workspace argument, for callers that cannot allocate device
    memory: the split-K scratch lives in the library's fixed 8 MiB device array. Calls
    that overlap on the GPU share that array and must be serialised by the caller."""
    _check(load_library().bsa_decode_noalloc(ctypes.byref(prob.c()), _ptr(q), k.c(), v.c(),
                                             _ptr(kept), _ptr(kept_count), _ptr(o), _ptr(lse),
                                             _ptr(o_f32), _ptr(dev_status), _stream(stream)),
           "bsa_decode_noalloc")


def bsa_pbs_permute(prob: Problem, q, k: Cache, v: Cache, k_idx: Cache, k_perm, v_perm,
                    kidx_perm, key_pos, workspace, dev_status=None, stream=None):
    _check(load_library().bsa_pbs_permute(ctypes.byref(prob.c()), _ptr(q), k.c(), v.c(),
                                          k_idx.c(), _ptr(k_perm), _ptr(v_perm),
                                          _ptr(kidx_perm), _ptr(key_pos), _ptr(workspace),
                                          0 if workspace is None else workspace.numel(),
                                          _ptr(dev_status), _stream(stream)),
           "bsa_pbs_permute")


def bsa_status_string(status: int) -> str:
    return load_library().bsa_status_string(status).decode()


# ------------------------------------------------------------------ pipelines
class DecodeStep:
    """Buffers for one decode problem and the score -> select -> attend chain.

    Outputs live in this object (torch-allocated once); ``run`` enqueues the three
    entry points on the current stream and returns nothing (no host sync)."""

    def __init__(self, prob: Problem, device="cuda", keep_f32=True):
        assert prob.phase == PHASE_DECODE
        self.prob = prob
        dev = torch.device(device)
        mk = bsa_max_kept(prob)
        self.scores = torch.empty(prob.B, prob.Hkv, prob.nb, dtype=torch.float32, device=dev)
        self.kept = torch.empty(prob.B, prob.Hkv, mk, dtype=torch.int32, device=dev)
        self.kept_count = torch.empty(prob.B, prob.Hkv, dtype=torch.int32, device=dev)
        self.o = torch.empty(prob.B, prob.Hq, prob.d, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(prob.B, prob.Hq, dtype=torch.float32, device=dev)
        self.o_f32 = (torch.empty(prob.B, prob.Hq, prob.d, dtype=torch.float32, device=dev)
                      if keep_f32 else None)
        if prob.group_size > 0:   # two-level routing: group scores and kept-group masks
            prob.group_scores = torch.empty(prob.B, prob.Hkv, prob.nb * BLOCK // prob.group_size,
                                            dtype=torch.float32, device=dev)
            prob.kept_groups = torch.empty(prob.B, prob.Hkv, mk, dtype=torch.int32, device=dev)
            self.group_scores, self.kept_groups = prob.group_scores, prob.kept_groups
        ws = bsa_workspace_size(prob, OP_DECODE)
        self.workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def run(self, q, q_idx, k_idx, k: Cache, v: Cache, stream=None):
        """k_idx: a bf16 index-key Cache or a 4-bit QCache."""
        p = self.prob
        if isinstance(k_idx, QCache):
            bsa_score_blocks_q(p, q_idx, k_idx, self.scores, self.status, stream)
        else:
            bsa_score_blocks(p, q_idx, k_idx, self.scores, self.status, stream)
        bsa_select_top_p(p, self.scores, self.kept, self.kept_count, self.status, stream)
        bsa_decode(p, q, k, v, self.kept, self.kept_count, self.o, self.lse, self.o_f32,
                   self.workspace, self.status, stream)


class Prefill:
    """Buffers for one prefill problem and the score -> select -> attend chain."""

    def __init__(self, prob: Problem, device="cuda", keep_f32=True):
        assert prob.phase == PHASE_PREFILL
        self.prob = prob
        dev = torch.device(device)
        nqb = prob.nb
        mk = bsa_max_kept(prob)
        self.scores = torch.empty(prob.B, prob.Hkv, nqb, nqb, dtype=torch.float32, device=dev)
        self.kept = torch.empty(prob.B, prob.Hkv, nqb, mk, dtype=torch.int32, device=dev)
        self.kept_count = torch.empty(prob.B, prob.Hkv, nqb, dtype=torch.int32, device=dev)
        self.o = torch.empty(prob.B, prob.Hq, prob.T, prob.d, dtype=torch.bfloat16, device=dev)
        self.lse = torch.empty(prob.B, prob.Hq, prob.T, dtype=torch.float32, device=dev)
        self.o_f32 = (torch.empty(prob.B, prob.Hq, prob.T, prob.d, dtype=torch.float32, device=dev)
                      if keep_f32 else None)
        ws = bsa_workspace_size(prob, OP_PREFILL)
        self.workspace = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def select(self, q_idx, k_idx: Cache, stream=None):
        bsa_score_blocks(self.prob, q_idx, k_idx, self.scores, self.status, stream)
        bsa_select_top_p(self.prob, self.scores, self.kept, self.kept_count, self.status, stream)

    def attend(self, q, k: Cache, v: Cache, stream=None):
        bsa_prefill(self.prob, q, k, v, self.kept, self.kept_count, self.o, self.lse, self.o_f32,
                    self.workspace, self.status, stream)

    def run(self, q, q_idx, k_idx: Cache, k: Cache, v: Cache, stream=None):
        self.select(q_idx, k_idx, stream)
        self.attend(q, k, v, stream)


class PbsPrefill:
    """Block-sparse prefill over a segment-permuted key order (PBS-Attn): permute the
    keys inside segments of `prob.segment` tokens by importance, then score, select
    and attend on the permuted caches. Buffers live in this object; ``run`` enqueues
    the four entry points on the current stream."""

    def __init__(self, prob: Problem, device="cuda", keep_f32=True):
        assert prob.phase == PHASE_PREFILL and prob.segment > 0
        dev = torch.device(device)
        B, H, T, d = prob.B, prob.Hkv, prob.T, prob.d
        self.k_perm = torch.empty(B, H, T, d, dtype=torch.bfloat16, device=dev)
        self.v_perm = torch.empty(B, H, T, d, dtype=torch.bfloat16, device=dev)
        self.kidx_perm = torch.empty(B, H, T, prob.r, dtype=torch.bfloat16, device=dev)
        self.key_pos = torch.empty(B, H, T, dtype=torch.int32, device=dev)
        prob.key_pos = self.key_pos
        self.prob = prob
        ws = bsa_workspace_size(prob, OP_PBS_PERMUTE)
        self.pws = torch.empty(max(ws, 256), dtype=torch.uint8, device=dev)
        self.pf = Prefill(prob, device=device, keep_f32=keep_f32)
        self.status = self.pf.status

    def permute(self, q, k: Cache, v: Cache, k_idx: Cache, stream=None):
        bsa_pbs_permute(self.prob, q, k, v, k_idx, self.k_perm, self.v_perm, self.kidx_perm,
                        self.key_pos, self.pws, self.status, stream)

    def run(self, q, q_idx, k_idx: Cache, k: Cache, v: Cache, stream=None):
        self.permute(q, k, v, k_idx, stream)
        self.pf.run(q, q_idx, contiguous_cache(self.kidx_perm), contiguous_cache(self.k_perm),
                    contiguous_cache(self.v_perm), stream)


def problem_for(w, seq_lens: Optional[torch.Tensor] = None,
                head_w: Optional[torch.Tensor] = None) -> Problem:
    """Problem description of a synthetic workload (see workloads.Workload)."""
    phase = PHASE_DECODE if w.phase == "decode" else PHASE_PREFILL
    return Problem(phase=phase, B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, T=w.T, n_sink=w.n_sink,
                   n_local=w.n_local, k_max=w.k_max, k_min=w.k_min, p=w.p, r=w.r,
                   idx_scale=1.0 / math.sqrt(w.r), attn_scale=1.0 / math.sqrt(w.d),
                   seq_lens=seq_lens if phase == PHASE_DECODE else None, head_w=head_w)


def caches_for(inputs: dict):
    """(k_idx, K, V) caches of a generated input dict."""
    k_idx = contiguous_cache(inputs["k_idx"])
    if inputs.get("page_table") is not None:
        pt = inputs["page_table"]
        return k_idx, paged_cache(inputs["K"], pt), paged_cache(inputs["V"], pt)
    return k_idx, contiguous_cache(inputs["K"]), contiguous_cache(inputs["V"])


class DecodeGraph:
    """One decode step from host buffers as a single CUDA graph launch.

    The graph holds, on fixed device buffers: the copy of the new query (q, q_idx)
    from pinned host tensors, score -> select -> attend (the kernels keep their
    programmatic dependent-launch edges), and the copy of o and lse back into pinned
    host tensors. New queries are written into ``q_host`` / ``q_idx_host`` in place;
    ``launch`` enqueues the step, ``run`` also waits for the host outputs."""

    def __init__(self, step: DecodeStep, q_host, q_idx_host, k_idx, k: Cache, v: Cache,
                 o_host, lse_host):
        self.step, self.k_idx, self.k, self.v = step, k_idx, k, v
        self.q_host, self.q_idx_host, self.o_host, self.lse_host = q_host, q_idx_host, o_host, lse_host
        self.q_dev = torch.empty(q_host.shape, dtype=q_host.dtype, device="cuda")
        self.q_idx_dev = torch.empty(q_idx_host.shape, dtype=q_idx_host.dtype, device="cuda")
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            self._body()          # first launches (function attributes, tensor maps) uncaptured
        side.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        # "relaxed": the entry points set kernel attributes on the host while capturing
        with torch.cuda.graph(self.graph, capture_error_mode="relaxed"):
            self._body()
        torch.cuda.synchronize()

    def _body(self):
        self.q_dev.copy_(self.q_host, non_blocking=True)
        self.q_idx_dev.copy_(self.q_idx_host, non_blocking=True)
        self.step.run(self.q_dev, self.q_idx_dev, self.k_idx, self.k, self.v)
        self.o_host.copy_(self.step.o, non_blocking=True)
        self.lse_host.copy_(self.step.lse, non_blocking=True)

    def launch(self):
        self.graph.replay()

    def run(self):
        self.graph.replay()
        torch.cuda.current_stream().synchronize()


def decode_step_host(step: DecodeStep, q_host, q_idx_host, k_idx, k: Cache, v: Cache,
                     o_host, lse_host, q_dev=None, q_idx_dev=None, stream=None):
    """One decode step from host buffers: copy the new query (q, q_idx; pinned host
    tensors) to the device, run score -> select -> attend, copy o and lse back into
    the pinned host tensors, and wait for them. The KV and index-key caches stay
    resident on the device."""
    stream = torch.cuda.current_stream() if stream is None else stream
    q_dev = torch.empty(q_host.shape, dtype=q_host.dtype, device="cuda") if q_dev is None else q_dev
    q_idx_dev = (torch.empty(q_idx_host.shape, dtype=q_idx_host.dtype, device="cuda")
                 if q_idx_dev is None else q_idx_dev)
    with torch.cuda.stream(stream):
        q_dev.copy_(q_host, non_blocking=True)
        q_idx_dev.copy_(q_idx_host, non_blocking=True)
        step.run(q_dev, q_idx_dev, k_idx, k, v, stream)
        o_host.copy_(step.o, non_blocking=True)
        lse_host.copy_(step.lse, non_blocking=True)
    stream.synchronize()
