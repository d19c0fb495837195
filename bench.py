"""Benchmark: one step = KV scatter of this step's tokens + paged attention.

Default workload (N = 1): the decode batch — 64 sequences x 1 query, context
uniform in [256, 4096], Hq 32 / Hkv 8, head_dim 128, block 16, bf16 — on
which the headline HBM-bandwidth metric is quoted.  With --gpus N (launched
by torchrun, one process per GPU) every rank runs its own independent decode
batch (different seed): weak scaling, no collective on the data path; ranks
only meet at the barriers around the timed region and in one MAX reduction of
the elapsed time.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the fp64 CPU
oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "paged-attn decode HBM GB/s + prefill TFLOP/s (fraction of B200 roofline)"
WORKLOAD = ("decode_batch: 64 seqs x 1 query token, context U[256,4096], Hq 32 / Hkv 8, "
            "head_dim 128, block 16, bf16, shuffled block tables; step = scatter of the 64 new "
            "K/V rows + split-KV decode attention")


# DRAM bytes (read + write) of one decode-kernel launch on the decode batch, from
# one ncu capture (dram__bytes_read.sum + dram__bytes_write.sum), valid only
# while the decode kernel's sources hash to the recorded value.
DECODE_TRAFFIC = {"sources_sha256": "cf54aee7b0a22a80d66cd70c794b735a3de383c64b3f8f7d1c9d9bca01610ba3",
                  "bytes_per_launch": 597341355}
DECODE_SOURCES = ("decode.cu", "decode.cuh", "common.cuh", "layout.h")


def decode_sources_sha() -> str:
    h = hashlib.sha256()
    for n in DECODE_SOURCES:
        with open(os.path.join(ROOT, "paged_kv_gqa_reshape_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic():
    if DECODE_TRAFFIC["sources_sha256"] and DECODE_TRAFFIC["sources_sha256"] == decode_sources_sha():
        return DECODE_TRAFFIC["bytes_per_launch"]
    return None


def launches_per_step(case) -> int:
    """Kernels the step launches: write_kv, the plan (only when the batch has a
    multi-token query or more sequences than the decode kernel plans for
    itself), the prefill kernel if there is a multi-token query, and the
    decode kernel (always)."""
    prefill = case.max_query_len > 1
    plan = prefill or case.num_seqs > 1024
    return 1 + int(plan) + int(prefill) + 1


# ---------------------------------------------------------------------------
# algorithmic work (what the method must move / compute)
# ---------------------------------------------------------------------------

def scatter_bytes(case) -> int:
    t = int(case.k_new.shape[0])
    return t * case.num_kv_heads * case.head_dim * 2 * 4 + 8 * t


def attention_bytes(case) -> int:
    """K + V of every visible key once per KV head, plus Q, O and the tables read."""
    lens = case.seq_lens.cpu().to(torch.int64)
    kv = int(lens.sum()) * case.num_kv_heads * case.head_dim * 2 * 2
    qo = 2 * case.num_q_tokens * case.num_q_heads * case.head_dim * 2
    tables = int(((lens + case.block_size - 1) // case.block_size).sum()) * 4
    meta = 4 * (2 * case.num_seqs + 1)
    return kv + qo + tables + meta


def visible_pairs(case) -> int:
    lens = case.seq_lens.cpu().tolist()
    ql = case.query_lens.cpu().tolist()
    tot = 0
    for L, q in zip(lens, ql):
        if not case.causal:
            tot += L * q
            continue
        for i in range(q):
            tot += max(0, min(L, L - q + i + 1))
    return tot


def attention_flops(case) -> int:
    return 4 * case.head_dim * case.num_q_heads * visible_pairs(case)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.dev = device_index

    def _ids(self):
        ids = []
        try:
            u = str(torch.cuda.get_device_properties(self.dev).uuid)
            ids.append(u if u.startswith("GPU-") else "GPU-" + u)
        except Exception:
            pass
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            parts = [x.strip() for x in vis.split(",") if x.strip()]
            if self.dev < len(parts):
                ids.append(parts[self.dev])
        ids.append(str(self.dev))
        return ids

    def start(self):
        self.proc = None
        for ident in self._ids():
            try:
                probe = subprocess.run(["nvidia-smi", "-i", ident, "--query-gpu=clocks.sm",
                                        "--format=csv,noheader,nounits"],
                                       capture_output=True, text=True, timeout=20)
            except Exception:
                continue
            if probe.returncode != 0 or not probe.stdout.strip():
                continue
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", ident, "--query-gpu=" + self.FIELDS,
                     "--format=csv,noheader,nounits", "-lms", "50"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                time.sleep(0.3)  # let the first sample land before the timed region
            except Exception:
                self.proc = None
            return

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            out = ""
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


def shard_seed(rank: int) -> int:
    """Each rank attends its own, independently drawn decode batch."""
    return 1002 + rank


def max_over_ranks(ms: float, world: int, device) -> float:
    """Elapsed time of the whole job: the slowest rank's (MAX all-reduce)."""
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_step: int, steps: int, world: int, max_ms: float) -> float:
    """Throughput of all ranks together: every rank moves bytes_per_step per step."""
    return bytes_per_step * steps * world / (max_ms * 1e-3) / 1e9


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(
            d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def device_case(case, dev):
    import dataclasses
    kw = {}
    for f in dataclasses.fields(case):
        v = getattr(case, f.name)
        kw[f.name] = v.to(dev) if isinstance(v, torch.Tensor) else v
    return type(case)(**kw)


def time_varlen_component(pa, case, iters=20, warmup=3, with_scatter=False, **mods):
    """Average device time (ms) of one attention_varlen call on `case` (device
    tensors): CUDA events around back-to-back calls.  `mods` (softcap,
    alibi_slopes, mask) go to the call."""
    ws = pa.varlen_workspace(case.num_seqs, case.num_q_tokens, case.num_q_heads,
                             case.num_kv_heads, case.head_dim)
    out = torch.empty_like(case.q)
    mql, msl = case.max_query_len, case.max_seq_len

    def run():
        if with_scatter:
            pa.write_kv(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache)
        pa.attention_varlen(case.q, case.k_cache, case.v_cache, case.block_tables, case.seq_lens,
                            case.query_start_loc, case.num_kv_heads, case.scale, case.causal, out,
                            max_query_len=mql, max_seq_len=msl, workspace=ws, **mods)

    if not with_scatter:
        pa.write_kv(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache)
    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    ms = b2b_ms(run, iters)
    st, bits = pa.get_error(ws)
    if st != 0:
        raise RuntimeError(f"device error word {bits:#x}")
    return ms


def b2b_ms(fn, iters):
    """Device time (ms) per call of fn: CUDA events around `iters` back-to-back
    calls on the launching stream (no event between calls)."""
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def time_spans_component(pa, case, span_offsets, spans, iters=20, warmup=3):
    """Average device time (ms) of one attention_varlen_spans call."""
    ws = pa.varlen_workspace(case.num_seqs, case.num_q_tokens, case.num_q_heads,
                             case.num_kv_heads, case.head_dim)
    out = torch.empty_like(case.q)
    mql, msl = case.max_query_len, case.max_seq_len
    pa.write_kv(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache)

    def run():
        pa.attention_varlen_spans(case.q, case.k_cache, case.v_cache, case.block_tables,
                                  case.seq_lens, case.query_start_loc, case.num_kv_heads,
                                  case.scale, span_offsets, spans, out, max_query_len=mql,
                                  max_seq_len=msl, workspace=ws)

    for _ in range(warmup):
        run()
    torch.cuda.synchronize()
    ms = b2b_ms(run, iters)
    st, bits = pa.get_error(ws)
    if st != 0:
        raise RuntimeError(f"device error word {bits:#x}")
    return ms


def time_calls(fn, iters=20, warmup=3):
    """Device time per call (ms) of `fn`: back-to-back calls (b2b_ms)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    return b2b_ms(fn, iters)


def smallseq_weight_bytes(ss, wlen):
    """Bytes of the attention-weights output: every [batch, Hq, wlen] slot is written."""
    return ss.batch * ss.num_q_heads * wlen * 2


def smallseq_bwd_bytes(ss):
    """Algorithmic bytes of the small-seq backward: q, dout, k, v and each
    entry's saved weights read once, dq, dk, dv written once, cu_seqlens_kv."""
    total_keys = ss.k.shape[0]
    row = ss.head_dim * 2
    return (2 * ss.batch * ss.num_q_heads * row            # q, dout
            + 2 * total_keys * ss.num_kv_heads * row       # k, v
            + total_keys * ss.num_q_heads * 2              # weights of the entry's keys
            + ss.batch * ss.num_q_heads * row              # dq
            + 2 * total_keys * ss.num_kv_heads * row       # dk, dv
            + 4 * (ss.batch + 1))


def components(pa, hbm_peak, tc_peak, peak_kind):
    """Secondary single-GPU measurements on the other workloads (device time per call)."""
    res = {}
    dev = torch.device("cuda")
    vc = workloads.varlen_prefill(device=dev, keep_logical=False)
    ms = time_varlen_component(pa, vc)
    tf = attention_flops(vc) / (ms * 1e-3) / 1e12
    res["varlen_prefill"] = {"ms": round(ms, 4), "tflops": round(tf, 1),
                             "frac": round(tf / tc_peak, 3), "peak": tc_peak,
                             "unit": "TFLOP/s", "of": peak_kind}
    # the scatter alone: the same step's 17 336 new tokens into the paged caches
    ms = time_calls(lambda: pa.write_kv(vc.k_new, vc.v_new, vc.slot_mapping, vc.k_cache,
                                        vc.v_cache), iters=50)
    gbs = scatter_bytes(vc) / (ms * 1e-3) / 1e9
    res["scatter_varlen_prefill"] = {"ms": round(ms, 4), "gbs": round(gbs, 1),
                                     "frac": round(gbs / hbm_peak, 3), "unit": "GB/s",
                                     "of": peak_kind}
    del vc
    ss = workloads.smallseq_batch(device=dev)
    out = torch.empty_like(ss.q)
    ms = time_calls(lambda: pa.attention_smallseq(ss.q, ss.k, ss.v, ss.cu_seqlens_kv, ss.scale,
                                                  out))
    nbytes = (ss.k.numel() + ss.v.numel() + ss.q.numel() + out.numel()) * 2 + 4 * (ss.batch + 1)
    gbs = nbytes / (ms * 1e-3) / 1e9
    res["smallseq_batch"] = {"ms": round(ms, 4), "gbs": round(gbs, 1),
                             "frac": round(gbs / hbm_peak, 3), "unit": "GB/s", "of": peak_kind}
    # the same workload's forward with the attention-weights output, then the backward
    w = torch.empty(ss.batch, ss.num_q_heads, 16, dtype=ss.q.dtype, device=dev)
    ms = time_calls(lambda: pa.attention_smallseq(ss.q, ss.k, ss.v, ss.cu_seqlens_kv, ss.scale,
                                                  out, weights=w))
    gbs = (nbytes + smallseq_weight_bytes(ss, w.shape[2])) / (ms * 1e-3) / 1e9
    res["smallseq_fwd_weights"] = {"ms": round(ms, 4), "gbs": round(gbs, 1),
                                   "frac": round(gbs / hbm_peak, 3), "unit": "GB/s",
                                   "of": peak_kind}
    dout = torch.randn(ss.q.shape, generator=workloads._gen(1007, dev), device=dev).to(ss.q.dtype)
    dq, dk, dv = torch.empty_like(ss.q), torch.empty_like(ss.k), torch.empty_like(ss.v)
    ms = time_calls(lambda: pa.attention_smallseq_bwd(ss.q, ss.k, ss.v, dout, w,
                                                      ss.cu_seqlens_kv, ss.scale, dq, dk, dv))
    gbs = smallseq_bwd_bytes(ss) / (ms * 1e-3) / 1e9
    res["smallseq_bwd"] = {"ms": round(ms, 4), "gbs": round(gbs, 1),
                           "frac": round(gbs / hbm_peak, 3), "unit": "GB/s", "of": peak_kind}
    del ss, out, w, dout, dq, dk, dv
    # the same prefill and decode workloads with fp16 inputs
    vc16 = workloads.varlen_prefill(device=dev, keep_logical=False, dtype=torch.float16)
    ms = time_varlen_component(pa, vc16)
    tf = attention_flops(vc16) / (ms * 1e-3) / 1e12
    res["varlen_prefill_fp16"] = {"ms": round(ms, 4), "tflops": round(tf, 1),
                                  "frac": round(tf / tc_peak, 3), "peak": tc_peak,
                                  "unit": "TFLOP/s", "of": peak_kind}
    del vc16
    dc16 = workloads.decode_batch(device=dev, keep_logical=False, dtype=torch.float16)
    ms = time_varlen_component(pa, dc16, iters=50)
    gbs = attention_bytes(dc16) / (ms * 1e-3) / 1e9
    res["decode_batch_fp16"] = {"ms": round(ms, 4), "gbs": round(gbs, 1),
                                "frac": round(gbs / hbm_peak, 3), "unit": "GB/s", "of": peak_kind}
    del dc16
    # score modifiers: the prefill workload with ALiBi slopes and the TANH30
    # soft-cap (no extra bytes); the decode workload over head-major caches
    # with a shared additive mask (its [64, 4096] fp32 rows are counted)
    vc = workloads.varlen_prefill(device=dev, keep_logical=False)
    slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / vc.num_q_heads)
                           for h in range(vc.num_q_heads)], device=dev)
    ms = time_varlen_component(pa, vc, softcap=30.0, alibi_slopes=slopes)
    tf = attention_flops(vc) / (ms * 1e-3) / 1e12
    res["varlen_prefill_alibi_softcap"] = {"ms": round(ms, 4), "tflops": round(tf, 1),
                                           "frac": round(tf / tc_peak, 3), "peak": tc_peak,
                                           "unit": "TFLOP/s", "of": peak_kind}
    del vc, slopes
    dc = workloads.decode_batch(device=dev, keep_logical=False)
    hnd = dataclasses.replace(
        dc, k_cache=dc.k_cache.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3),
        v_cache=dc.v_cache.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3))
    del dc
    mlen = (hnd.max_seq_len + 3) // 4 * 4
    mask = torch.randn(hnd.num_q_tokens, mlen, generator=workloads._gen(1008, dev), device=dev)
    ms = time_varlen_component(pa, hnd, iters=50, mask=mask)
    mask_bytes = 4 * sum(int(x) for x in hnd.seq_lens.tolist())
    gbs = (attention_bytes(hnd) + mask_bytes) / (ms * 1e-3) / 1e9
    res["decode_batch_hnd_mask"] = {"ms": round(ms, 4), "gbs": round(gbs, 1),
                                    "frac": round(gbs / hbm_peak, 3), "unit": "GB/s",
                                    "of": peak_kind}
    del hnd, mask
    sc, so, sp = workloads.spans_prefill(device=dev, keep_logical=False)
    ms = time_spans_component(pa, sc, so, sp)
    pairs = workloads.spans_visible_pairs(sc.seq_lens.tolist(), sc.query_lens.tolist(),
                                          so.tolist(), sp.tolist())
    tf = 4 * sc.head_dim * sc.num_q_heads * pairs / (ms * 1e-3) / 1e12
    res["spans_prefill"] = {"ms": round(ms, 4), "tflops": round(tf, 1),
                            "frac": round(tf / tc_peak, 3), "peak": tc_peak,
                            "unit": "TFLOP/s", "of": peak_kind}
    del sc, so, sp
    mx = workloads.mixed_step(device=dev, keep_logical=False)
    ms = time_varlen_component(pa, mx, iters=10)
    nbytes = attention_bytes(mx)
    fl = attention_flops(mx)
    # serial roofline: decode bytes at the HBM peak plus prefill FLOPs at the tensor peak
    dec_bytes = sum(int(l) for l, q in zip(mx.seq_lens.tolist(), mx.query_lens.tolist()) if q == 1)
    dec_bytes *= mx.num_kv_heads * mx.head_dim * 4
    pre_fl = fl - 4 * mx.head_dim * mx.num_q_heads * sum(
        int(l) for l, q in zip(mx.seq_lens.tolist(), mx.query_lens.tolist()) if q == 1)
    t_roof = dec_bytes / (hbm_peak * 1e9) + pre_fl / (tc_peak * 1e12)
    t_max = max(dec_bytes / (hbm_peak * 1e9), pre_fl / (tc_peak * 1e12))
    res["mixed_step"] = {"ms": round(ms, 4), "roofline_ms": round(t_roof * 1e3, 4),
                         "frac_serial": round(t_roof / (ms * 1e-3), 3),
                         "frac_max": round(t_max / (ms * 1e-3), 3),
                         "decode_gb": round(dec_bytes / 1e9, 2), "prefill_tflop": round(pre_fl / 1e12, 3),
                         "of": peak_kind}
    del mx
    torch.cuda.empty_cache()
    return res


def capture_graph(fn, n):
    """A CUDA graph of n calls of fn (warmed once on a side stream first)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(n):
            fn()
    torch.cuda.synchronize()
    return g


def time_graph(fn, n, reps):
    """Average device time (ms) of one fn call: a graph of n calls replayed
    `reps` times, CUDA events around each replay."""
    g = capture_graph(fn, n)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(reps)]
    for a, b in evs:
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize()
    del g
    return statistics.mean(a.elapsed_time(b) for a, b in evs) / n


def headline_config(world: int, graph: bool) -> dict:
    """The headline workload's config, as both arms print it."""
    return {"workload": WORKLOAD, "global_batch": 64 * world, "seq_len": "256-4096",
            "parallelism": f"dp{world} (independent sequences per GPU, no collective)",
            "l2": "inputs larger than L2 (0.57 GB of K/V per step vs 126 MB L2)",
            "launch": ("one CUDA graph of the step (write_kv + attention), replayed "
                       "once per step" if graph
                       else "stream launches, one pair of library calls per step")}


def run_ours(args, rank, world, local_rank):
    import paged_kv_gqa_reshape_b200 as pa

    pa.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    hbm_peak, tc_peak, tc_sust, peak_kind = measured_peaks()

    case = workloads.decode_batch(device=dev, seed=shard_seed(rank), keep_logical=False)
    ws = pa.varlen_workspace(case.num_seqs, case.num_q_tokens, case.num_q_heads,
                             case.num_kv_heads, case.head_dim, device=dev)
    out = torch.empty_like(case.q)
    mql, msl = case.max_query_len, case.max_seq_len

    def step():
        pa.write_kv(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache,
                    workspace=ws)
        attention()

    def attention():
        pa.attention_varlen(case.q, case.k_cache, case.v_cache, case.block_tables, case.seq_lens,
                            case.query_start_loc, case.num_kv_heads, case.scale, case.causal, out,
                            max_query_len=mql, max_seq_len=msl, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, bits = pa.get_error(ws)
    if st != 0:
        raise RuntimeError(f"device error word {bits:#x} after warm-up")

    # K steps of stream launches (write_kv + attention); with --graph the step
    # is captured once as a CUDA graph and replayed once per step
    g_step = capture_graph(step, 1) if args.graph else None
    if g_step is not None:
        for _ in range(args.warmup):
            g_step.replay()
    clocks = ClockSampler(dev.index)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_start.record()
    for i in range(args.steps):
        if g_step is not None:
            g_step.replay()
        else:
            step()
    t_end.record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    st, bits = pa.get_error(ws)
    if st != 0:
        raise RuntimeError(f"device error word {bits:#x} in the timed region")
    del g_step
    # the decode kernel alone (the roofline's kernel): CUDA events around
    # back-to-back attention calls on the launching stream
    attn_ms = b2b_ms(attention, max(20, min(1000, args.steps)))

    max_ms = max_over_ranks(elapsed_ms, world, dev)
    bytes_step = scatter_bytes(case) + attention_bytes(case)
    value = whole_job_gbs(bytes_step, args.steps, world, max_ms)

    # end to end through the public API: pinned host inputs in, output back, every step
    e2e = run_e2e(pa, case, args, dev, ws, expected=out)
    e2e["ms"] = max_over_ranks(e2e["ms"], world, dev)
    e2e_value = whole_job_gbs(bytes_step, args.steps, world, e2e["ms"])

    attn_bytes = attention_bytes(case)
    achieved = attn_bytes / (attn_ms * 1e-3) / 1e9
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16; per-rank seed 1002+rank)",
        "config": headline_config(world, args.graph),
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "mode": e2e["mode"]},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                     "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                     "traffic": args.traffic if args.traffic is not None else recorded_traffic(),
                     "kernel": "decode_kernel (split-KV decode; the call launches only it), "
                               "CUDA events around back-to-back calls",
                     "peak_kind": peak_kind},
        "clocks": clk,
        "gpu_launches": launches_per_step(case) * args.steps,
    }
    return result, case


def run_single_workload(args):
    """--workload NAME (not the headline): time NAME's step on one GPU.

    Used to profile the other workloads' kernels with committed code only;
    prints one JSON line with that workload's own throughput.
    """
    import paged_kv_gqa_reshape_b200 as pa

    pa.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    hbm_peak, tc_peak, _, peak_kind = measured_peaks()
    name = args.workload
    if name == "spans_prefill":
        sc, so, sp = workloads.spans_prefill(device=dev, keep_logical=False)
        ms = time_spans_component(pa, sc, so, sp, iters=args.steps, warmup=args.warmup)
        pairs = workloads.spans_visible_pairs(sc.seq_lens.tolist(), sc.query_lens.tolist(),
                                              so.tolist(), sp.tolist())
        v = 4 * sc.head_dim * sc.num_q_heads * pairs / (ms * 1e-3) / 1e12
        return {"workload": name, "value": round(v, 2), "unit": "TFLOP/s", "ms_per_step": round(ms, 5),
                "steps": args.steps, "warmup": args.warmup, "frac": round(v / tc_peak, 4),
                "peak": tc_peak, "peak_kind": peak_kind}
    if name == "smallseq_batch":
        ss = workloads.smallseq_batch(device=dev)
        out = torch.empty_like(ss.q)

        def step():
            pa.attention_smallseq(ss.q, ss.k, ss.v, ss.cu_seqlens_kv, ss.scale, out)
        work = (ss.k.numel() + ss.v.numel() + ss.q.numel() + out.numel()) * 2 + 4 * (ss.batch + 1)
        unit, scale_div, peak = "GB/s", 1e9, hbm_peak
    elif name == "scatter_varlen":
        vc = workloads.varlen_prefill(device=dev, keep_logical=False)

        def step():
            pa.write_kv(vc.k_new, vc.v_new, vc.slot_mapping, vc.k_cache, vc.v_cache)
        work = scatter_bytes(vc)
        unit, scale_div, peak = "GB/s", 1e9, hbm_peak
    elif name == "smallseq_bwd":
        ss = workloads.smallseq_batch(device=dev)
        out = torch.empty_like(ss.q)
        w = torch.empty(ss.batch, ss.num_q_heads, 16, dtype=ss.q.dtype, device=dev)
        pa.attention_smallseq(ss.q, ss.k, ss.v, ss.cu_seqlens_kv, ss.scale, out, weights=w)
        dout = torch.randn(ss.q.shape, generator=workloads._gen(1007, dev),
                           device=dev).to(ss.q.dtype)
        dq, dk, dv = torch.empty_like(ss.q), torch.empty_like(ss.k), torch.empty_like(ss.v)

        def step():
            pa.attention_smallseq_bwd(ss.q, ss.k, ss.v, dout, w, ss.cu_seqlens_kv, ss.scale,
                                      dq, dk, dv)
        work = smallseq_bwd_bytes(ss)
        unit, scale_div, peak = "GB/s", 1e9, hbm_peak
    else:
        case = workloads.NAMED[name](device=dev, keep_logical=False) if name != "tiny_prefill" \
            else workloads.tiny_prefill(device=dev)
        ws = pa.varlen_workspace(case.num_seqs, case.num_q_tokens, case.num_q_heads,
                                 case.num_kv_heads, case.head_dim, device=dev)
        out = torch.empty_like(case.q)
        mql, msl = case.max_query_len, case.max_seq_len

        def step():
            pa.write_kv(case.k_new, case.v_new, case.slot_mapping, case.k_cache, case.v_cache,
                        workspace=ws)
            pa.attention_varlen(case.q, case.k_cache, case.v_cache, case.block_tables,
                                case.seq_lens, case.query_start_loc, case.num_kv_heads,
                                case.scale, case.causal, out, max_query_len=mql,
                                max_seq_len=msl, workspace=ws)
        if mql > 1:
            work, unit, scale_div, peak = attention_flops(case), "TFLOP/s", 1e12, tc_peak
        else:
            work = scatter_bytes(case) + attention_bytes(case)
            unit, scale_div, peak = "GB/s", 1e9, hbm_peak
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        step()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    v = work / (ms * 1e-3) / scale_div
    res = {"workload": name, "value": round(v, 2), "unit": unit, "ms_per_step": round(ms, 5),
           "steps": args.steps, "warmup": args.warmup, "frac": round(v / peak, 4),
           "peak": peak, "peak_kind": peak_kind}
    if args.timeline:
        res["timeline"] = kernel_timeline(step)
    return res


def kernel_timeline(step):
    """Start and end (µs, from the first kernel's start) of every kernel one
    call of `step` launches, from the CUDA activity records of torch.profiler:
    shows which kernels of a call ran side by side."""
    torch.cuda.synchronize()
    with torch.profiler.profile(activities=[torch.profiler.ProfilerActivity.CUDA]) as prof:
        step()
        torch.cuda.synchronize()
    ev = [e for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    if not ev:
        return []
    t0 = min(e.time_range.start for e in ev)
    return [{"kernel": e.name.split("(")[0][:80], "start_us": round(e.time_range.start - t0, 1),
             "end_us": round(e.time_range.end - t0, 1)}
            for e in sorted(ev, key=lambda e: e.time_range.start)]


def run_e2e(pa, case, args, dev, ws, expected=None):
    """The same step through the public API with host-resident inputs/outputs.

    Default (pipelined, as a serving loop runs it): each step's inputs are
    copied in on a host-to-device stream one step ahead, into one of two
    device buffers, and its output goes back on a device-to-host stream from
    one of two output buffers, so both transfers overlap the neighbouring
    steps' kernels; events order every buffer's reuse.  `--e2e-serial` runs
    copy in, kernels, copy out one after another on one stream instead (the
    only form `--graph` captures).  Either way every step copies all of its
    inputs in and its output back inside the timed region."""
    names = ["q", "k_new", "v_new", "slot_mapping", "block_tables", "seq_lens", "query_start_loc"]
    # the step's inputs packed in one pinned host buffer (each at a 256-byte
    # offset) and copied with one transfer into one device buffer, whose
    # typed views the library reads, as a serving loop stages its metadata
    offs, off = {}, 0
    for n in names:
        t = getattr(case, n)
        offs[n] = off
        off += (t.numel() * t.element_size() + 255) // 256 * 256
    host_buf = torch.empty(off, dtype=torch.uint8).pin_memory()
    for n in names:
        t = getattr(case, n)
        nbytes = t.numel() * t.element_size()
        host_buf[offs[n]:offs[n] + nbytes].copy_(t.contiguous().view(torch.uint8).view(-1).cpu())
    serial = args.e2e_serial or args.graph
    nbuf = 1 if serial else 2
    dev_bufs, devts, outs_d = [], [], []
    for _ in range(nbuf):
        buf = torch.empty(off, dtype=torch.uint8, device=dev)
        devt = {}
        for n in names:
            t = getattr(case, n)
            nbytes = t.numel() * t.element_size()
            devt[n] = buf[offs[n]:offs[n] + nbytes].view(t.dtype).view(t.shape)
        dev_bufs.append(buf)
        devts.append(devt)
        outs_d.append(torch.empty_like(case.q))
    out_h = torch.empty(case.q.shape, dtype=case.q.dtype).pin_memory()
    h2d = sum(getattr(case, n).numel() * getattr(case, n).element_size() for n in names)
    d2h = out_h.numel() * out_h.element_size()
    steps = max(1, min(args.steps, 500))
    mql, msl = case.max_query_len, case.max_seq_len  # host-side metadata, known before the step

    def kernels(b):
        devt = devts[b]
        pa.write_kv(devt["k_new"], devt["v_new"], devt["slot_mapping"], case.k_cache,
                    case.v_cache, workspace=ws)
        pa.attention_varlen(devt["q"], case.k_cache, case.v_cache, devt["block_tables"],
                            devt["seq_lens"], devt["query_start_loc"], case.num_kv_heads,
                            case.scale, case.causal, outs_d[b], max_query_len=mql,
                            max_seq_len=msl, workspace=ws)

    comp = torch.cuda.current_stream(dev)
    if serial:
        def step(i):
            dev_bufs[0].copy_(host_buf, non_blocking=True)
            kernels(0)
            out_h.copy_(outs_d[0], non_blocking=True)
    else:
        h2d_s, d2h_s = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: [torch.cuda.Event() for _ in range(nbuf)]
        staged, computed, returned = ev(), ev(), ev()
        used = [False] * nbuf

        def step(i):
            b = i % nbuf
            with torch.cuda.stream(h2d_s):
                if used[b]:
                    h2d_s.wait_event(computed[b])  # step i-2's kernels have read buffer b
                dev_bufs[b].copy_(host_buf, non_blocking=True)
                staged[b].record(h2d_s)
            comp.wait_event(staged[b])
            if used[b]:
                comp.wait_event(returned[b])  # step i-2's output has left buffer b
            kernels(b)
            computed[b].record(comp)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(computed[b])
                out_h.copy_(outs_d[b], non_blocking=True)
                returned[b].record(d2h_s)
            used[b] = True

        def drain():
            for b in range(nbuf):
                if used[b]:
                    comp.wait_event(returned[b])

    for i in range(3):
        step(i)
    if not serial:
        drain()
    torch.cuda.synchronize()
    # with --graph: one CUDA graph of the whole serial step (the host-to-device
    # copy of its inputs, the two library calls, the copy of the output back)
    g = capture_graph(lambda: step(0), 1) if args.graph else None
    if g is not None:
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    if not serial:
        h2d_s.wait_event(a)  # no copy of the timed steps starts before the first event
        d2h_s.wait_event(a)
        used = [False] * nbuf
    for i in range(steps):
        if g is not None:
            g.replay()
        else:
            step(i)
    if not serial:
        drain()  # the last outputs are back on the host before the end event
    b.record(comp)
    torch.cuda.synchronize()
    del g
    ms = a.elapsed_time(b) * args.steps / steps
    st, bits = pa.get_error(ws)
    if st != 0:
        raise RuntimeError(f"device error word {bits:#x} in the end-to-end leg")
    # the output that came back is the device-resident path's, bit for bit
    if expected is not None and not torch.equal(out_h, expected.cpu()):
        raise RuntimeError("end-to-end output differs from the device-resident step's")
    mode = ("serial: copy in, kernels, copy out on one stream" if serial else
            "pipelined: inputs copied in one step ahead on a copy stream, outputs copied "
            "back on another, two device buffers each")
    return {"ms": ms, "h2d": h2d, "d2h": d2h, "mode": mode}


# ---------------------------------------------------------------------------
# oracle legs (CPU)
# ---------------------------------------------------------------------------

def oracle_decode_sample(num_seqs, seed=1002):
    """A bounded sample of the decode workload for the CPU oracle."""
    return workloads.decode_batch(num_seqs=num_seqs, seed=seed)


class OracleDecodeStep:
    """The oracle's pass over (a window of) the decode batch: the literal cache
    write of the window's new tokens, then fp64 attention of its query rows.
    Every sequence of the decode batch has exactly one query token, token s of
    sequence s, so a window of sequences is a range of query rows."""

    def __init__(self, case):
        self.case = case
        self.kc = workloads.bf16_bits(case.k_cache).copy()
        self.vc = workloads.bf16_bits(case.v_cache).copy()
        self.q = workloads.bf16_bits(case.q)
        self.kn = workloads.bf16_bits(case.k_new)
        self.vn = workloads.bf16_bits(case.v_new)
        self.kl = workloads.bf16_bits(case.k_logical)
        self.vl = workloads.bf16_bits(case.v_logical)
        self.sm = case.slot_mapping.numpy()
        lens = case.seq_lens.to(torch.int64)
        per_seq = (lens * case.num_kv_heads * case.head_dim * 4              # K + V
                   + 2 * case.num_q_heads * case.head_dim * 2                  # q + out
                   + (lens + case.block_size - 1) // case.block_size * 4      # table
                   + 8                                                         # lengths
                   + case.num_kv_heads * case.head_dim * 2 * 4 + 8)           # scatter
        self.bytes_per_seq = per_seq.tolist()
        assert case.max_query_len == 1 and case.num_q_tokens == case.num_seqs

    def bytes(self, s0: int, n: int) -> int:
        return int(sum(self.bytes_per_seq[s0:s0 + n]))

    def run(self, s0: int = 0, n: int = None) -> float:
        import oracle
        c = self.case
        n = c.num_seqs if n is None else n
        rows = np.arange(s0, s0 + n, dtype=np.int64)
        t0 = time.perf_counter()
        oracle.write_kv(self.kn[s0:s0 + n], self.vn[s0:s0 + n], self.sm[s0:s0 + n], self.kc,
                        self.vc, c.block_size)
        oracle.attention_varlen(self.q, self.kl, self.vl, c.kv_offsets.numpy(),
                                c.seq_lens.numpy(), c.query_start_loc.numpy(), c.num_kv_heads,
                                c.scale, c.causal, rows=None if n == c.num_seqs else rows)
        return time.perf_counter() - t0


def cpu_model() -> str:
    """The host CPU's model name (first `model name` of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(budget_s=12.0):
    import oracle
    oracle.build()
    case = oracle_decode_sample(64)
    step = OracleDecodeStep(case)
    nbytes = step.bytes(0, case.num_seqs)
    times = []
    t_begin = time.perf_counter()
    while not times or (time.perf_counter() - t_begin < budget_s and len(times) < 500):
        times.append(step.run())
    gbs = nbytes * len(times) / sum(times) / 1e9
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": oracle.num_threads(),
            "cpu": cpu_model(), "kind": "oracle",
            "sample": f"the full 64-sequence decode batch (seed 1002), {len(times)} passes of "
                      f"oracle write_kv + fp64 attention ({sum(times):.1f} s)"}


def run_reference(args, rank, world, budget_s=120.0):
    """The oracle as the reference arm, on the headline workload and config.

    Each step is the oracle's pass over the 64-sequence decode batch (seed
    1002, the batch rank 0 of our arm times), or, when K such passes would
    not fit the time budget, over a window of n consecutive sequences of it
    (the windows rotate through the batch); n is set from the time of one
    warm-up pass of the whole batch.  The metric is the same bytes per second
    as our arm's: every visible key's K and V once per KV head, q, out, the
    tables and the scattered rows of the sequences processed."""
    if rank != 0:
        return None
    import oracle
    oracle.build()
    case = oracle_decode_sample(64)
    step = OracleDecodeStep(case)
    t_full = min(step.run() for _ in range(max(1, min(args.warmup, 3))))
    n = max(1, min(case.num_seqs, int(case.num_seqs * budget_s / (args.steps * t_full))))
    times, nbytes = [], 0
    for i in range(args.steps):
        s0 = (i * n) % case.num_seqs
        m = min(n, case.num_seqs - s0)
        times.append(step.run(s0, m))
        nbytes += step.bytes(s0, m)
    total = sum(times)
    gbs = nbytes / total / 1e9
    sample = (f"each step: the oracle's literal cache write + fp64 attention over "
              + ("the whole 64-sequence decode batch (seed 1002)" if n == case.num_seqs else
                 f"a window of {n} consecutive sequences of the 64-sequence decode batch "
                 f"(seed 1002), windows rotating through the batch")
              + f"; {args.steps} steps, {total:.1f} s")
    return {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": headline_config(world, args.graph),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": oracle.num_threads(),
                         "cpu": cpu_model(), "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-components", action="store_true")
    ap.add_argument("--e2e-serial", action="store_true",
                    help="end-to-end leg: copy in, kernels, copy out serially on one stream")
    ap.add_argument("--graph", action="store_true",
                    help="time the step (and the end-to-end leg) as replays of a CUDA graph")
    ap.add_argument("--workload", default="decode_batch",
                    choices=sorted(list(workloads.NAMED) + ["spans_prefill", "smallseq_bwd",
                                                           "scatter_varlen"]),
                    help="decode_batch is the headline; the others time one workload alone")
    ap.add_argument("--timeline", action="store_true",
                    help="with --workload: also list one step's kernels with start / end times")
    ap.add_argument("--traffic", type=float, default=None,
                    help="dram bytes per dominant-kernel launch from an ncu capture, if current")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if args.workload != "decode_batch":
        print(json.dumps(run_single_workload(args)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        result, case = run_ours(args, rank, world, local_rank)
        if rank == 0:
            hbm_peak, tc_peak, tc_sust, peak_kind = measured_peaks()
            if world == 1 and not args.no_components:
                del case
                torch.cuda.empty_cache()
                import paged_kv_gqa_reshape_b200 as pa
                result["components"] = components(pa, hbm_peak, tc_peak, peak_kind)
            if world == 1 and not args.no_cpu_baseline:
                result["cpu_baseline"] = cpu_baseline()
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
