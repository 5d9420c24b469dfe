"""Benchmark: 128K-context batched decode + 64K block-sparse prefill on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one pass of the whole hot path: a decode step on the 128K workload
(index scoring -> top-p selection -> split-K sparse attention) and a block-sparse
causal prefill of the 64K workload (prefill scoring -> top-k selection -> sparse
attention). Rank 0 prints one JSON line. Under torchrun each rank runs its own
copy of the workload on its GPU (independent sequences, no data-path
collective: weak scaling); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import block_sparse_long_06_b200 as bsa                      # noqa: E402
from block_sparse_long_06_b200 import workloads as W         # noqa: E402

METRIC = "decode tokens/s & achieved HBM GB/s at 128K ctx; sparse-prefill TFLOP/s"
DECODE_WL = "decode_b32_h32_t128k_paged"
PREFILL_WL = "prefill_b1_h32_t64k"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 datasheet figures (HGX): 7.7 TB/s HBM3e, 2.25 PFLOP/s dense bf16
DATASHEET = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0}


# ---------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def peak_clock_note(peaks):
    """The SM clock the measured matmul peak was taken at, when the peaks file says."""
    c = peaks.get("clocks_under_load") or {}
    if c.get("sm_mhz_median"):
        return (f"measured peak taken at a median SM clock of {c['sm_mhz_median']:.0f} MHz "
                f"(max {c.get('sm_max_mhz', 0):.0f} MHz)")
    return None


def kernel_source_hash(files):
    """Hash of the kernel sources with comments and whitespace removed, so that a
    comment edit does not void a measurement taken on the same code."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "block_sparse_long_06_b200", "csrc", f)) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(re.sub(r"\s+", "", text).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, files, workload):
    """Per-launch DRAM bytes from the committed ncu summary, if the kernel source
    still matches the one the counters were taken on and the figure is for this
    workload; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    ent = d.get(kernel_key)
    if not ent or ent.get("source_hash") != kernel_source_hash(files):
        return None
    if ent.get("workload") != workload:
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "20", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            t0 = time.time()
            while not self.lines and time.time() - t0 < 5.0:   # sampling has started
                time.sleep(0.01)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64,
                     device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- byte / FLOP accounting
def decode_bytes(w, kept_count, seq_lens, index_cache="bf16"):
    """Algorithmic bytes of one decode step and of its attention call. Index keys:
    32 B per token in bf16; a 576-byte record per visible 64-token block (9 B per
    token) in the 4-bit formats."""
    B, Hq, Hkv, d, r = w.B, w.Hq, w.Hkv, w.d, w.r
    kc = kept_count.to(torch.int64).cpu()
    lens = seq_lens.to(torch.int64).cpu()
    kv = int(kc.sum()) * 64 * d * 2 * 2                 # K and V of every kept block
    if index_cache == "bf16":
        idx = int(lens.sum()) * Hkv * r * 2             # every index key
    else:
        idx = int(((lens + 63) // 64).sum()) * Hkv * 576 + 4
    q = B * Hq * d * 2
    q_idx = B * Hq * r * 2
    o = B * Hq * d * 2 + B * Hq * 4                     # bf16 output + fp32 lse
    pt = int(kc.sum()) * 4 if w.paged else 0            # page-table entries of kept blocks
    attn = kv + q + o + pt
    return {"step": kv + idx + q + q_idx + o + pt, "attention": attn, "index_keys": idx,
            "kv": kv}


def prefill_flops(w, kept_count):
    """(kept-tile FLOP, causal-exact FLOP) of one prefill. The first counts every kept
    64 x 64 tile whole, as the tensor cores compute it (the headline: FLOPs of the
    kept tiles); the second counts only the (query, key) pairs the causal mask leaves
    visible: half of each diagonal tile plus its diagonal, and the real rows of a
    partial last query block."""
    kc = kept_count.to(torch.int64).cpu().reshape(-1, w.nb)    # [B*Hkv, nqb]
    tiles = float(kc.sum()) * w.G * 4 * 64 * 64 * w.d
    nq = torch.tensor([min(64, w.T - 64 * i) for i in range(w.nb)], dtype=torch.int64)
    # every kept block but the diagonal is fully visible to the block's real rows
    pairs = ((kc - 1).clamp(min=0) * nq * 64).sum() + (nq * (nq + 1) // 2).sum() * kc.shape[0]
    return tiles, float(pairs) * w.G * 4 * w.d


# ---------------------------------------------------------------- our arm
def describe(w) -> str:
    """One-line description of a workload, from its fields."""
    kv = "paged KV (64-token pages)" if w.paged else "contiguous KV"
    base = f"B={w.B} Hq={w.Hq} Hkv={w.Hkv} d={w.d} T={w.T} {kv}, r={w.r}"
    if w.phase == "decode":
        return f"{base}, {w.n_sink} sink + {w.n_local} local, p={w.p}, K_max={w.k_max}"
    sel = f"top-{w.k_max}" if w.p >= 1.0 else f"p={w.p}, K_max={w.k_max}"
    return f"{base}, diagonal + {w.n_sink} sink + {w.n_local} local + {sel}"


def run_ours(args, world, rank, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    do_dec = args.phase in ("both", "decode")
    do_pf = args.phase in ("both", "prefill")
    wd = W.WORKLOADS[args.decode_workload].with_(seed=rank)
    wp = W.WORKLOADS[args.prefill_workload].with_(seed=rank)

    if do_dec:
        xd = W.make_decode_inputs(wd, dev)
        dprob = bsa.problem_for(wd, seq_lens=xd["seq_lens"], head_w=xd["head_w"])
        dstep = bsa.DecodeStep(dprob, device=dev, keep_f32=False)
        k_idx_c, K_c, V_c = bsa.caches_for(xd)
        if args.index_cache != "bf16":
            # the selector cache is quantised once, as when the keys are written
            fmt = bsa.IDX_FP4 if args.index_cache == "fp4" else bsa.IDX_INT4
            qc = bsa.contiguous_qcache(wd.B, wd.Hkv, wd.T, fmt, device=dev)
            bsa.bsa_quantize_index_keys(dprob, k_idx_c, qc, dstep.status)
            k_idx_c = qc
            torch.cuda.synchronize()
    if do_pf:
        xp = W.make_prefill_inputs(wp, dev)
        pprob = bsa.problem_for(wp, head_w=xp["head_w"])
        if args.idx_heads == 1:
            # one index head per kv group: the bf16 mean of the group's index queries
            qi = xp["q_idx"]
            xp["q_idx"] = qi.float().reshape(wp.B, wp.Hkv, wp.G, *qi.shape[2:]).mean(2) \
                .to(torch.bfloat16).contiguous()
            pprob.idx_heads, pprob.head_w = 1, None
        pf = bsa.Prefill(pprob, device=dev, keep_f32=False)
        pk_idx = bsa.contiguous_cache(xp["k_idx"])
        pK = bsa.contiguous_cache(xp["K"])
        pV = bsa.contiguous_cache(xp["V"])
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def one_step(ev=None, split=False, prefill=True):
        """One step. split=True also records an event between selection and attention
        (to time bsa_decode alone); it is left out of the step timing because an event
        there keeps the attention kernel from overlapping the selection's tail."""
        if do_dec:
            flush.zero_()                   # L2 flushed between decode steps (untimed)
        if ev:
            ev["d0"].record(stream)
        if do_dec:
            if isinstance(k_idx_c, bsa.QCache):
                bsa.bsa_score_blocks_q(dprob, xd["q_idx"], k_idx_c, dstep.scores, dstep.status)
            else:
                bsa.bsa_score_blocks(dprob, xd["q_idx"], k_idx_c, dstep.scores, dstep.status)
            bsa.bsa_select_top_p(dprob, dstep.scores, dstep.kept, dstep.kept_count, dstep.status)
        if ev and split:
            ev["a0"].record(stream)
        if do_dec:
            bsa.bsa_decode(dprob, xd["q"], K_c, V_c, dstep.kept, dstep.kept_count, dstep.o,
                           dstep.lse, None, dstep.workspace, dstep.status)
        if ev:
            ev["d1"].record(stream)
        if not prefill:
            return
        if do_pf:
            flush.zero_()                   # and before the prefill (its inputs fit in L2)
        if ev:
            ev["p0"].record(stream)
        if do_pf:
            pf.select(xp["q_idx"], pk_idx)
        if ev:
            ev["p1"].record(stream)
        if do_pf:
            pf.attend(xp["q"], pK, pV)
        if ev:
            ev["p2"].record(stream)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    st = (int(dstep.status.item()) if do_dec else 0) | (int(pf.status.item()) if do_pf else 0)
    if st:
        raise RuntimeError(f"device status {st:#x}")

    names = ("d0", "a0", "d1", "p0", "p1", "p2")
    evs = [{n: torch.cuda.Event(enable_timing=True) for n in names} for _ in range(args.steps)]
    evs_att = [{n: torch.cuda.Event(enable_timing=True) for n in names} for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device() if world == 1 else local) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for k in range(args.steps):
            one_step(evs[k])
        t_end.record(stream)
        if do_dec:                          # bsa_decode alone: the same steps, split timing
            for k in range(args.steps):
                one_step(evs_att[k], split=True, prefill=False)
        torch.cuda.synchronize()
    barrier(world)
    dec_ms = [e["d0"].elapsed_time(e["d1"]) for e in evs]
    att_ms = [e["a0"].elapsed_time(e["d1"]) for e in evs_att] if do_dec else [0.0] * args.steps
    psel_ms = [e["p0"].elapsed_time(e["p1"]) for e in evs]
    patt_ms = [e["p1"].elapsed_time(e["p2"]) for e in evs]
    total_ms = t_start.elapsed_time(t_end)

    # every rank takes the same collective steps, whatever the phase
    dec_sum = max_over_ranks(sum(dec_ms), world)
    step_ms = max_over_ranks(sum(d + ps + pa for d, ps, pa in zip(dec_ms, psel_ms, patt_ms)) /
                             args.steps, world)
    att_avg = max_over_ranks(sum(att_ms) / args.steps, world)
    patt_avg = max_over_ranks(sum(patt_ms) / args.steps, world)
    psel_avg = max_over_ranks(sum(psel_ms) / args.steps, world)
    dec_avg = dec_sum / args.steps
    hbm = peaks["hbm_gbs"]
    tflops_peak = peaks["bf16_tflops"]

    dec = pre = None
    roof_dec = roof_pf = None
    if do_dec:
        by = decode_bytes(wd, dstep.kept_count, xd["seq_lens"], args.index_cache)
        dec_sum, att_avg, dec_avg = max(dec_sum, 1e-9), max(att_avg, 1e-9), max(dec_avg, 1e-9)
        tokens_per_s = world * wd.B * args.steps / (dec_sum / 1e3)
        attn_gbs = by["attention"] / (att_avg / 1e3) / 1e9
        step_gbs = by["step"] / (dec_avg / 1e3) / 1e9
        dec = {"ms": dec_avg, "tokens_per_s": tokens_per_s, "hbm_gbs": step_gbs,
               "hbm_frac": step_gbs / hbm, "bytes_per_step": by["step"],
               "attention_ms": att_avg, "kept_blocks": int(dstep.kept_count.sum())}
        files = ["decode_attn.cu", "bsa_common.cuh", "bsa_internal.h"]
        roof_dec = {"bound": "hbm", "kernel": "bsa_decode (split-K attention + LSE merge)",
                    "achieved": attn_gbs, "peak": hbm, "unit": "GB/s", "frac": attn_gbs / hbm,
                    "peak_datasheet": DATASHEET["hbm_gbs"],
                    "frac_datasheet": attn_gbs / DATASHEET["hbm_gbs"],
                    "traffic": ncu_traffic("decode_attn", files, wd.name),
                    "peak_source": f"{peak_src} hbm_gbs (burst copy)",
                    "bytes_per_launch": by["attention"]}
    if do_pf:
        flops, flops_exact = prefill_flops(wp, pf.kept_count)
        patt_avg = max(patt_avg, 1e-9)
        pf_tflops = world * flops / (patt_avg / 1e3) / 1e12
        pre = {"select_ms": psel_avg, "attention_ms": patt_avg, "tflops": pf_tflops,
               "tensor_frac": pf_tflops / world / tflops_peak, "kept_tile_flop": flops,
               "causal_exact_flop": flops_exact,
               "causal_exact_tflops": world * flops_exact / (patt_avg / 1e3) / 1e12}
        files = ["prefill_tc.cu", "v_to_f16.cu", "tcgen05.cuh", "bsa_common.cuh",
                 "bsa_internal.h"]
        roof_pf = {"bound": "tensor", "kernel": "bsa_prefill (V->fp16 + attention)",
                   "achieved": pf_tflops / world, "peak": tflops_peak, "unit": "TFLOP/s",
                   "frac": pf_tflops / world / tflops_peak,
                   "peak_datasheet": DATASHEET["bf16_tflops"],
                   "frac_datasheet": pf_tflops / world / DATASHEET["bf16_tflops"],
                   "peak_clock": peak_clock_note(peaks),
                   "traffic": ncu_traffic("prefill_tc", files, wp.name),
                   "peak_source": f"{peak_src} bf16_tflops (burst)",
                   "flop_per_launch": flops}

    # end to end through the public API with host buffers (decode: the new query in,
    # the attention output out, every step)
    e2e = (None if args.no_e2e or not do_dec else
           run_e2e(args, dprob, dstep, xd, k_idx_c, K_c, V_c, stream, world))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and do_dec and args.index_cache == "bf16":
        cpu = cpu_baseline_decode(wd, xd, dstep, budget_s=args.cpu_budget)

    # other configurations of the path, each timed on its own (every rank runs them)
    extras = {}
    if not args.no_extras:
        if do_dec and args.index_cache == "bf16":
            qc = bsa.contiguous_qcache(wd.B, wd.Hkv, wd.T, bsa.IDX_FP4, device=dev)
            bsa.bsa_quantize_index_keys(dprob, k_idx_c, qc, dstep.status)
            extras["decode_fp4"] = time_decode(wd, xd, dprob, dstep, qc, K_c, V_c, "fp4", dev,
                                               world, args.extra_steps, peaks)
            del qc
            extras["decode_hga"] = time_hga(wd, xd, k_idx_c, K_c, V_c, dev, world,
                                            args.extra_steps, peaks, 16, 2 * wd.k_max)
            del xd, dstep, K_c, V_c, k_idx_c
            torch.cuda.empty_cache()
            for key, name in (("decode_c2", "decode_b8_h32_t32k_paged"),
                              ("decode_c4", "decode_b1_h64_t1m")):
                extras[key] = time_decode_workload(name, rank, dev, world, args.extra_steps, peaks)
        if do_pf:
            extras["prefill_pbs"] = time_pbs(wp, xp, dev, world, 256, max(3, args.extra_steps // 4),
                                             peaks)


    clocks = clk.summary()
    config = {"workload": " + ".join(w.name for w, on in ((wd, do_dec), (wp, do_pf)) if on)}
    if do_dec:
        config["decode"] = describe(wd)
        config["index_cache"] = args.index_cache
    if do_pf:
        config["prefill"] = describe(wp)
        config["index_heads_per_group"] = 1 if args.idx_heads == 1 else wp.G
    config["l2"] = ("a 256 MB buffer is written before each decode step and each prefill, "
                    "outside the timed events")
    config["parallelism"] = f"dp{world} (independent sequences per GPU)"
    # kernels per step: decode = scorer, selection, split-K attention, LSE merge;
    # prefill = scorer, selection, V->fp16, attention; then the decode-only steps
    # that time bsa_decode alone
    launches = args.steps * (4 * do_dec + 4 * do_pf) + args.steps * 4 * do_dec
    if do_dec:
        value, unit = dec["tokens_per_s"], "tokens/s"
    else:
        value, unit = pre["tflops"], "TFLOP/s"
    line = {
        "metric": METRIC,
        "value": value,
        "unit": unit,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": config,
    }
    if dec is not None:
        line["decode"] = dec
    if pre is not None:
        line["prefill"] = pre
    line["roofline"] = roof_dec if roof_dec is not None else roof_pf
    if roof_dec is not None and roof_pf is not None:
        line["roofline_prefill"] = roof_pf
    line.update(extras)
    line.update({"e2e": e2e, "gpu_launches": launches, "clocks": clocks,
                 "total_ms_events": total_ms})
    if cpu is not None:
        line["cpu_baseline"] = cpu
    return line


def time_decode(w, xd, prob, step, k_idx, K, V, index_cache, dev, world, steps, peaks):
    """Device time of the decode step (score -> select -> attend) on resident inputs,
    a 256 MB buffer written before every step (untimed); mean over `steps`, max over
    ranks."""
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        step.run(xd["q"], xd["q_idx"], k_idx, K, V)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for e0, e1 in evs:
        flush.zero_()
        e0.record(stream)
        step.run(xd["q"], xd["q_idx"], k_idx, K, V)
        e1.record(stream)
    torch.cuda.synchronize()
    st = int(step.status.item())
    ms = max_over_ranks(sum(e0.elapsed_time(e1) for e0, e1 in evs) / steps, world)
    by = decode_bytes(w, step.kept_count, xd["seq_lens"], index_cache)
    gbs = by["step"] / (ms / 1e3) / 1e9
    return {"workload": w.name, "index_cache": index_cache, "ms": ms,
            "tokens_per_s": world * w.B / (ms / 1e3), "hbm_gbs": gbs,
            "hbm_frac": gbs / peaks["hbm_gbs"], "bytes_per_step": by["step"], "steps": steps,
            "device_status": st}


def time_hga(w, xd, k_idx, K, V, dev, world, steps, peaks, gs, k_groups):
    """Decode with two-level routing (HGA): the kept blocks' best k_groups groups of gs
    tokens. Algorithmic bytes: every index key, q and the outputs, and K and V of
    the copied 16-token quarters (whole always-visible blocks, kept groups of the
    others); the intermediate block and group scores are not counted."""
    prob = bsa.problem_for(w, seq_lens=xd["seq_lens"], head_w=xd["head_w"])
    prob.group_size, prob.k_groups = gs, k_groups
    step = bsa.DecodeStep(prob, device=dev, keep_f32=False)
    out = time_decode(w, xd, prob, step, k_idx, K, V, "bf16", dev, world, steps, peaks)
    by = decode_bytes(w, step.kept_count, xd["seq_lens"], "bf16")
    m = step.kept_groups.to(torch.int64).cpu()
    quarters = sum(int(((m >> q4) & 1).sum()) for q4 in range(4)) if gs == 16 else None
    if quarters is not None:
        kv = quarters * 16 * w.d * 2 * 2
        step_bytes = by["step"] - by["kv"] + kv
        gbs = step_bytes / (out["ms"] / 1e3) / 1e9
        out.update({"bytes_per_step": step_bytes, "hbm_gbs": gbs,
                    "hbm_frac": gbs / peaks["hbm_gbs"], "kv_tokens": quarters * 16})
    out.update({"group_size": gs, "k_groups": k_groups,
                "kept_blocks": int(step.kept_count.sum())})
    del step
    torch.cuda.empty_cache()
    return out


def time_decode_workload(name, rank, dev, world, steps, peaks):
    w = W.WORKLOADS[name].with_(seed=rank)
    xd = W.make_decode_inputs(w, dev)
    prob = bsa.problem_for(w, seq_lens=xd["seq_lens"], head_w=xd["head_w"])
    step = bsa.DecodeStep(prob, device=dev, keep_f32=False)
    k_idx, K, V = bsa.caches_for(xd)
    out = time_decode(w, xd, prob, step, k_idx, K, V, "bf16", dev, world, steps, peaks)
    out["config"] = describe(w)
    del xd, step, K, V, k_idx
    torch.cuda.empty_cache()
    return out


def time_pbs(w, xp, dev, world, segment, steps, peaks):
    """Prefill over segment-permuted keys (PBS-Attn): permutation, score + select on the
    permuted index keys, attention; the kept-tile FLOP over the attention time."""
    prob = bsa.problem_for(w, head_w=xp["head_w"])
    prob.segment = segment
    pbs = bsa.PbsPrefill(prob, device=dev, keep_f32=False)
    kc, K, V = (bsa.contiguous_cache(xp["k_idx"]), bsa.contiguous_cache(xp["K"]),
                bsa.contiguous_cache(xp["V"]))
    kcp, Kp, Vp = (bsa.contiguous_cache(pbs.kidx_perm), bsa.contiguous_cache(pbs.k_perm),
                   bsa.contiguous_cache(pbs.v_perm))
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(2):
        pbs.run(xp["q"], xp["q_idx"], kc, K, V)
    evs = []
    for _ in range(steps):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        flush.zero_()
        e[0].record(stream)
        pbs.permute(xp["q"], K, V, kc)
        e[1].record(stream)
        pbs.pf.select(xp["q_idx"], kcp)
        e[2].record(stream)
        pbs.pf.attend(xp["q"], Kp, Vp)
        e[3].record(stream)
        evs.append(e)
    torch.cuda.synchronize()
    mean = lambda a, b: max_over_ranks(sum(e[a].elapsed_time(e[b]) for e in evs) / steps, world)
    perm_ms, sel_ms, att_ms = mean(0, 1), mean(1, 2), mean(2, 3)
    flops, flops_exact = prefill_flops(w, pbs.pf.kept_count)
    tf = flops / (att_ms / 1e3) / 1e12
    out = {"segment": segment, "permute_ms": perm_ms, "select_ms": sel_ms, "attention_ms": att_ms,
           "tflops": world * tf, "tensor_frac": tf / peaks["bf16_tflops"],
           "kept_tile_flop": flops, "steps": steps, "device_status": int(pbs.status.item())}
    del pbs
    torch.cuda.empty_cache()
    return out


def run_e2e(args, dprob, dstep, xd, k_idx_c, K_c, V_c, stream, world):
    """Host buffers in and out every step: the new query copied from pinned host memory,
    score -> select -> attend, o and lse copied back and waited for. The step is one
    CUDA graph launch (bsa.DecodeGraph); if capture is refused the eager entry points
    run instead, and the line says which."""
    q_h = xd["q"].cpu().pin_memory()
    qi_h = xd["q_idx"].cpu().pin_memory()
    o_h = torch.empty(dstep.o.shape, dtype=dstep.o.dtype).pin_memory()
    lse_h = torch.empty(dstep.lse.shape, dtype=dstep.lse.dtype).pin_memory()
    try:
        graph = bsa.DecodeGraph(dstep, q_h, qi_h, k_idx_c, K_c, V_c, o_h, lse_h)
        step, path = graph.run, "cuda graph (h2d copies, 4 kernels, d2h copies)"
    except (RuntimeError, bsa.BsaError) as e:
        q_d = torch.empty_like(xd["q"])
        qi_d = torch.empty_like(xd["q_idx"])
        path = f"eager entry points (graph capture failed: {str(e).splitlines()[0][:80]})"

        def step():
            bsa.decode_step_host(dstep, q_h, qi_h, k_idx_c, K_c, V_c, o_h, lse_h, q_d, qi_d)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    B = dprob.B
    return {"value": world * B * args.steps / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": q_h.numel() * 2 + qi_h.numel() * 2,
            "d2h_bytes_per_step": o_h.numel() * 2 + lse_h.numel() * 4,
            "launch": path}


# ---------------------------------------------------------------- oracle on the host
def one_thread():
    """Context in which the oracle runs on one host thread (numpy's BLAS pools limited
    to 1), so the reported core count is the number of threads that actually worked."""
    import contextlib
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(limits=1)
    except ImportError:
        return contextlib.nullcontext()


def cpu_baseline_decode(w, xd, dstep=None, budget_s=20.0, max_seqs=None):
    """Time the fp64 oracle (as it stands) on a bounded sample of decode rows of the
    workload: whole sequences (all kv heads) until ~budget_s of CPU work."""
    from oracle import bsa_oracle as O
    G, T = w.G, w.T
    pt = xd.get("page_table")
    done_seqs, t_total = 0, 0.0
    b = 0
    while b < w.B and (max_seqs is None or done_seqs < max_seqs):
        # host copies of this sequence's inputs (not timed: a CPU program would hold them)
        q = xd["q"][b].cpu()
        qi = xd["q_idx"][b].cpu()
        ki = xd["k_idx"][b].cpu()
        if pt is None:
            Kb, Vb = xd["K"][b].cpu(), xd["V"][b].cpu()
            pages = None
        else:
            pages = pt[b].long()
            Kb = xd["K"][pages].transpose(0, 1).reshape(w.Hkv, -1, w.d)[:, :T].cpu()
            Vb = xd["V"][pages].transpose(0, 1).reshape(w.Hkv, -1, w.d)[:, :T].cpu()
        hw = xd["head_w"].double().cpu().numpy()
        with one_thread():
            t0 = time.perf_counter()
            for g in range(w.Hkv):
                S = O.decode_block_scores(qi[g * G:(g + 1) * G].double().numpy(),
                                          ki[g, :T].double().numpy(), T, hw[g * G:(g + 1) * G],
                                          1.0 / math.sqrt(w.r))
                sel = O.select_decode(S, w.n_sink, w.n_local, w.p, w.k_max, w.k_min)
                ids = O.kept_token_ids(sel.kept, T)
                O.attend(q[g * G:(g + 1) * G].double().numpy(), Kb[g, ids].double().numpy(),
                         Vb[g, ids].double().numpy(), 1.0 / math.sqrt(w.d))
            t_total += time.perf_counter() - t0
        done_seqs += 1
        b += 1
        if t_total >= budget_s:
            break
    return {"value": done_seqs / t_total, "unit": "tokens/s", "cores": 1,
            "host_cores": os.cpu_count(), "kind": "oracle",
            "sample": f"{done_seqs} of {w.B} sequences of {w.name} (all {w.Hkv} kv heads each: "
                      f"score, select, attend in float64), {t_total:.1f} s"}


def run_reference(args, world, rank):
    """The oracle on the host cores, same config / metric / unit, bounded per step."""
    if rank != 0:
        return None
    wd = W.WORKLOADS[DECODE_WL]
    if torch.cuda.is_available():
        xd = W.make_decode_inputs(wd, "cuda")
    else:
        wd = wd.with_(B=2)
        xd = W.make_decode_inputs(wd, "cpu")
    per_step = []
    for k in range(args.warmup + args.steps):
        r = cpu_baseline_decode(wd, xd, budget_s=0.0, max_seqs=1)
        if k >= args.warmup:
            per_step.append(1.0 / r["value"])     # seconds for one sequence
    sec = sum(per_step)
    value = args.steps / sec
    cpu = {"value": value, "unit": "tokens/s", "cores": 1, "host_cores": os.cpu_count(),
           "kind": "oracle",
           "sample": f"one sequence (all {wd.Hkv} kv heads) of {DECODE_WL} per step"}
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": DECODE_WL, "parallelism": "host cores of rank 0"},
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=20.0)
    ap.add_argument("--phase", choices=["both", "decode", "prefill"], default="both")
    ap.add_argument("--decode-workload", default=DECODE_WL, choices=sorted(
        k for k, v in W.WORKLOADS.items() if v.phase == "decode"))
    ap.add_argument("--prefill-workload", default=PREFILL_WL, choices=sorted(
        k for k, v in W.WORKLOADS.items() if v.phase == "prefill"))
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other configurations (4-bit index cache, 32K and 1M decode, "
                         "permuted-key prefill)")
    ap.add_argument("--extra-steps", type=int, default=20)
    ap.add_argument("--idx-heads", type=int, choices=[0, 1], default=0,
                    help="prefill index heads per kv group: 0 = one per query head (the "
                         "method as configured), 1 = one per group (compact indexer)")
    ap.add_argument("--index-cache", choices=["bf16", "fp4", "int4"], default="bf16",
                    help="decode index-key cache: bf16 (the method as configured) or the "
                         "4-bit microscaled selector cache")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    world, rank, local = dist_init()
    if args.impl == "reference":
        line = run_reference(args, world, rank)
    else:
        line = run_ours(args, world, rank, local)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
