"""Benchmark of one absorbed-MLA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload v3] [--impl ours|reference]

A step is the whole hot path for one layer: this step's cache rows and
absorbed queries (mla_append_absorb: mla_append_latent and mla_absorb_q in one
launch; the two calls in turn above 16 tokens), then mla_decode_attn (split-KV
attention, LSE combine, W_UV) over a batch of synthetic sequences whose latent
cache is resident in HBM.  The default workload is DeepSeek-V3-shaped decode: 16
sequences, 128 heads, context 32768, 64-token pages, shuffled page table.

Timing: W untimed warm-up steps, then K steps bracketed by a barrier and a
device synchronise, timed with two CUDA events on the launching stream and
none in between (an event between two kernels ends the overlap of their
launches).  When the latent cache is larger than L2 (604 MB at the default
workload) no flush is inserted; when it fits in L2 (the V2-shaped workload)
every step is timed alone with a 256 MB buffer rewritten before it, and the
back-to-back (hot-L2) figure is reported beside it.  The roofline's kernel
time is mla_decode_attn alone, timed the same way in a loop of its own after
the steps; append, absorb and decode are also reported one by one ("phases").
Multi-GPU (torchrun): every rank runs its own replica on its own batch (data
parallel over sequences, no collective on the data path) and the slowest
rank's time is reported.  Rank 0 prints one JSON line.

e2e: the same K steps through the public C ABI with every step's inputs (h, q,
positions, lengths) copied from pinned host memory and its output copied back,
inside the timed region, double-buffered on a second stream the way a serving
loop overlaps transfers with the neighbouring steps' compute.

next_rows: the layer output projection y = W_O concat_h(o_h) (mla_out_proj, on
the step's output) and the q-LoRA query path c_Q = W_DQ h, q = W_UQ c_Q
(mla_query_proj, q_lora_rank 1536), each timed alone after the step (neither is
part of the step); W_O (235 MB at the V3 shape) is larger than L2, W_DQ + W_UQ
(97.5 MB) are not, so an L2-sized buffer is rewritten before each timed call of
the query path (query_proj.layers_back_to_back: the same calls back to back, each
with another layer's copy of the weights, the copies together over twice the
L2).  next_rows.prefill: mla_decode_attn on a chunk of 128 new tokens
per sequence (2 sequences of 32768, V3 heads), compute-bound, against the bf16
tensor peak.

--impl reference times the CPU oracle (float64 numpy, absorbed form) on a
bounded sample of the same workload on the host cores, as the comparison arm.

--prefill-forms prints one JSON line comparing, on chunks of 128 to 1024 new
tokens per sequence (2 sequences of 32768, V3 heads), this library's absorbed
prefill with the decompressing form built from library kernels (cuBLAS GEMMs
and fused attention through torch), to place their crossover.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workload as W  # noqa: E402

METRIC = "MLA latent decode tokens/s; HBM GB/s and TFLOPS as fraction of B200 roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


L2_BYTES = 126 * 2 ** 20
FLUSH_BYTES = 256 * 2 ** 20


def cache_fits_l2(w: W.Workload, lens) -> bool:
    return int(np.sum(lens)) * w.row * 2 < L2_BYTES


def describe(w: W.Workload, lens=None) -> dict:
    d = {"workload": f"{w.name}: batch {w.batch}, {w.nq} query token(s)/seq, {w.n_heads} heads, "
                     + (f"context {w.context}" if w.context else f"context U[{w.ragged[0]},{w.ragged[1]}]")
                     + f", d_c {w.d_c}, d_rope {w.d_rope}, page {w.page_size}",
         "batch": w.batch, "nq": w.nq, "n_heads": w.n_heads, "d_c": w.d_c, "d_rope": w.d_rope,
         "qk_nope": w.qk_nope, "v_head": w.v_head, "d_model": w.d_model, "page_size": w.page_size,
         "context": w.context if w.context else list(w.ragged), "page_table": "shuffled"}
    if lens is not None and cache_fits_l2(w, lens):
        d["l2"] = ("L2 flushed: the latent cache fits in the 126 MB L2, so a 256 MB buffer is rewritten "
                   "before each timed step (each step timed alone)")
    else:
        d["l2"] = "inputs larger than L2: the latent cache streamed each step exceeds the 126 MB L2"
    return d


def algorithmic_counts(w: W.Workload, lens: np.ndarray) -> dict:
    """Bytes and flops mla_decode_attn must move / compute (cache read once per
    sequence, W_UV once, q_lat in, out written), per launch."""
    R = w.row
    T = w.tokens
    cache = int(lens.sum()) * R * 2
    nbytes = cache + w.n_heads * w.v_head * w.d_c * 2 + T * w.n_heads * R * 2 + T * w.n_heads * w.v_head * 2
    # visible keys per query token: N_b - nq + 1 + i
    keys = sum(int(n) - w.nq + 1 + i for n in lens for i in range(w.nq))
    flops = keys * w.n_heads * 2 * (R + w.d_c) + T * w.n_heads * 2 * w.d_c * w.v_head
    return {"bytes": nbytes, "flops": flops, "cache_bytes": cache}


PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "decode_pair_kernel_v3.md")
KERNEL_SOURCES = ["decode_pair.cu", "decode_combine.cu", "plan.cuh", "sm100.cuh", "common.cuh", "mma_frag.cuh",
                  "decode.h", "tma_map.cu", "api.cu"]   # the kernels, their tensor maps and launch shapes


def kernel_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in sorted(KERNEL_SOURCES):
        h.update(f.encode())
        with open(os.path.join(ROOT, "head_latent_attention_07_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(workload_name: str):
    """DRAM bytes (read + write) of one mla_decode_attn call from the committed
    ncu summary, or None when the summary is for another workload or the
    kernel sources changed since it was taken."""
    if workload_name != "v3" or not os.path.exists(PROFILE_SUMMARY):
        return None, "no ncu capture for this workload"
    fields = {}
    for line in open(PROFILE_SUMMARY):
        if ":" in line:
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    if fields.get("sources_sha256") != kernel_sources_sha256():
        return None, "kernel sources changed since the ncu capture"
    return int(fields["traffic_bytes_per_call"]), "ncu dram__bytes_read.sum + dram__bytes_write.sum, split + combine"


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (all ranks get the result); the
    identity when no process group is running."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, tokens_per_rank: int, steps: int, ms: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch of tokens_per_rank
    query tokens per step (weak scaling), timed by the slowest rank."""
    return world * tokens_per_rank * steps / (ms / 1000.0)


def layer_copies(nbytes_per_layer: int) -> int:
    """How many copies of one layer's weights a back-to-back loop cycles through
    so that a copy is evicted from L2 before its next use: their total exceeds
    twice the L2, with at least two copies."""
    return max(2, -(-2 * L2_BYTES // nbytes_per_layer) + 1)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i in range(4) if r[i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ our arm

def run_ours(args, w: W.Workload, rank: int, world: int, local_rank: int):
    import torch
    import head_latent_attention_07_b200 as M

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    x = W.make_decode_inputs(w, seed=args.seed + rank)
    to_bf16 = lambda b: torch.from_numpy(np.ascontiguousarray(b)).view(torch.bfloat16).to(dev)
    to_i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    dims = M.MlaDims(n_heads=w.n_heads, d_c=w.d_c, d_rope=w.d_rope, qk_nope=w.qk_nope, v_head=w.v_head,
                     d_model=w.d_model, page_size=w.page_size)
    T = w.tokens
    h, q = to_bf16(x.bits["h"]), to_bf16(x.bits["q"])
    w_dkv, w_uk, w_uv = to_bf16(x.bits["w_dkv"]), to_bf16(x.bits["w_uk"]), to_bf16(x.bits["w_uv"])
    pool = to_bf16(x.bits["pool"])
    del x.bits["pool"]
    page_table = to_i32(x.page_table)
    seq_lens, seq_idx, pos = to_i32(x.lens), to_i32(x.h_seq_idx), to_i32(x.pos)
    q_lat = torch.empty((w.batch, w.nq, w.n_heads, w.row), dtype=torch.bfloat16, device=dev)
    out = torch.empty((w.batch, w.nq, w.n_heads, w.v_head), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.batch, w.nq, w.n_heads), dtype=torch.float32, device=dev)
    ws = torch.empty(M.mla_decode_workspace_bytes(dims, w.batch, w.nq), dtype=torch.uint8, device=dev)
    status = torch.zeros(4, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flushed = cache_fits_l2(w, x.lens)
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if flushed else None

    def append_(h_, seq_idx_, pos_):
        M.mla_append_latent(dims, h_, w_dkv, seq_idx_, pos_, page_table, pool, dev_status=status, stream=stream)

    def absorb_(q_, pos_):
        M.mla_absorb_q(dims, q_, pos_, w_uk, q_lat.view(T, w.n_heads, w.row), stream=stream)

    def decode_(seq_lens_):
        M.mla_decode_attn(dims, q_lat, pool, page_table, seq_lens_, w_uv, ws, out, lse, dev_status=status,
                          stream=stream)

    # the step's append and absorb (the same tokens and positions) in one call
    fused = T <= 16 and np.array_equal(x.h_pos, x.pos) and np.array_equal(x.h_seq_idx, x.seq_idx)

    def prologue_(h_, q_, seq_idx_, pos_):
        if fused:
            M.mla_append_absorb(dims, h_, w_dkv, seq_idx_, pos_, page_table, pool, q_, w_uk,
                                q_lat.view(T, w.n_heads, w.row), dev_status=status, stream=stream)
        else:
            append_(h_, seq_idx_, pos_)
            absorb_(q_, pos_)

    def step(h_, q_, seq_idx_, pos_, seq_lens_):
        prologue_(h_, q_, seq_idx_, pos_)
        decode_(seq_lens_)

    # append + absorb (one launch when fused), decode split, decode combine
    launches_per_step = 3 if fused else 4

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(dev)

    def timed(fn, n):
        """Device time (ms) of n calls of fn: two events around the whole loop, or,
        when the cache fits in L2, each call alone after an L2 flush (summed)."""
        if not flushed:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                fn()
            e1.record(stream)
            barrier()
            return e0.elapsed_time(e1)
        pairs = []
        for _ in range(n):
            flush_buf.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            pairs.append((e0, e1))
        barrier()
        return float(sum(a.elapsed_time(b) for a, b in pairs))

    # ---- device-resident timing: the whole step
    for _ in range(args.warmup):
        step(h, q, seq_idx, pos, seq_lens)
    barrier()
    assert M.mla_status_read(status, stream) == 0, "device status after warm-up"
    sampler = ClockSampler(local_rank)
    sampler.start()
    barrier()
    ms_total = timed(lambda: step(h, q, seq_idx, pos, seq_lens), args.steps)
    clocks = sampler.stop()
    # the same calls one by one: mla_decode_attn (the roofline's kernel time), then append and absorb
    n_phase = min(args.steps, 200)
    decode_ms = timed(lambda: decode_(seq_lens), n_phase) / n_phase
    append_ms = timed(lambda: append_(h, seq_idx, pos), n_phase) / n_phase
    absorb_ms = timed(lambda: absorb_(q, pos), n_phase) / n_phase
    prologue_ms = timed(lambda: prologue_(h, q, seq_idx, pos), n_phase) / n_phase
    hot_ms = None
    if flushed:   # the same steps back to back with the cache hot in L2
        flushed = False
        hot_ms = timed(lambda: step(h, q, seq_idx, pos, seq_lens), args.steps)
        flushed = True
    # ---- end to end through the C ABI with host buffers (pinned), copies inside the timed region.
    # A serving loop's double buffering: step i's inputs go host -> device and
    # step i's output device -> host on a copy stream, overlapped with the
    # compute of the neighbouring steps; every step's copies are still done
    # inside the timed region (the clock stops after the last output copy).
    host = {k: v.cpu().pin_memory() for k, v in (("h", h), ("q", q), ("seq_idx", seq_idx), ("pos", pos),
                                                  ("seq_lens", seq_lens))}
    dbuf = [{k: torch.empty_like(v, device=dev) for k, v in host.items()} for _ in range(2)]
    outs = [torch.empty_like(out) for _ in range(2)]
    out_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    copy_stream = torch.cuda.Stream(dev)

    def e2e_run(n, start=None):
        in_ready = [torch.cuda.Event() for _ in range(n)]
        done = [torch.cuda.Event() for _ in range(n)]
        out_read = [torch.cuda.Event() for _ in range(n)]

        def h2d_copy(i):
            with torch.cuda.stream(copy_stream):
                if i >= 2:
                    copy_stream.wait_event(done[i - 2])      # buffer i % 2 no longer read by step i - 2
                for k in host:
                    dbuf[i % 2][k].copy_(host[k], non_blocking=True)
                in_ready[i].record(copy_stream)

        if start is not None:
            copy_stream.wait_event(start)                    # the first input copy is inside the timed region
        h2d_copy(0)
        for i in range(n):
            if i + 1 < n:
                h2d_copy(i + 1)
            stream.wait_event(in_ready[i])
            if i >= 2:
                stream.wait_event(out_read[i - 2])           # outs[i % 2] has been copied out
            b = dbuf[i % 2]
            prologue_(b["h"], b["q"], b["seq_idx"], b["pos"])
            M.mla_decode_attn(dims, q_lat, pool, page_table, b["seq_lens"], w_uv, ws, outs[i % 2], lse,
                              dev_status=status, stream=stream)
            done[i].record(stream)
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(done[i])
                out_host[i % 2].copy_(outs[i % 2], non_blocking=True)
                out_read[i].record(copy_stream)
        return out_read[n - 1]

    e2e_run(args.warmup)
    barrier()
    if not flushed:
        e0 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        last = e2e_run(args.steps, start=e0)
        e1 = torch.cuda.Event(enable_timing=True)
        stream.wait_event(last)
        e1.record(stream)
        barrier()
        e2e_ms = e0.elapsed_time(e1)
    else:
        # cache in L2: each step alone after an L2 flush, its copies in and out
        # serialised with it on one stream, timed from the first input copy to
        # the last output copy
        pairs = []
        for i in range(args.steps):
            flush_buf.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            b = dbuf[i % 2]
            for k in host:
                b[k].copy_(host[k], non_blocking=True)
            prologue_(b["h"], b["q"], b["seq_idx"], b["pos"])
            M.mla_decode_attn(dims, q_lat, pool, page_table, b["seq_lens"], w_uv, ws, outs[i % 2], lse,
                              dev_status=status, stream=stream)
            out_host[i % 2].copy_(outs[i % 2], non_blocking=True)
            e1.record(stream)
            pairs.append((e0, e1))
        barrier()
        e2e_ms = float(sum(a.elapsed_time(b) for a, b in pairs))
    assert M.mla_status_read(status, stream) == 0, "device status after timing"
    # the copies really happened: the last output read back equals the device result
    assert torch.equal(out_host[(args.steps - 1) % 2], outs[(args.steps - 1) % 2].cpu()), "e2e output copy"

    extra = {}
    if w.name == "v3":   # the next rows of the hot-path table, at the V3 shape
        extra = {"out_proj": measure_out_proj(M, w, dims, out, dev, stream, args.seed + rank),
                 "query_proj": measure_query_proj(M, w, dims, dev, stream, args.seed + rank),
                 "prefill": measure_prefill(M, w, dims, dev, stream, args.seed + rank)}
    keys = sorted(extra)
    vals = max_over_ranks([ms_total, e2e_ms, decode_ms, append_ms, absorb_ms, prologue_ms, hot_ms or 0.0]
                          + [extra[k]["time_us"] for k in keys], dev)
    ms_total, e2e_ms, decode_ms, append_ms, absorb_ms, prologue_ms, hot_ms2 = vals[:7]
    for k, v in zip(keys, vals[7:]):
        extra[k]["time_us"] = v
    return {"ms_total": ms_total, "e2e_ms": e2e_ms, "decode_ms": decode_ms, "decode_loop_ms": decode_ms * n_phase,
            "phases_ms": {"append": append_ms, "absorb": absorb_ms,
                          ("append_absorb" if fused else "append_then_absorb"): prologue_ms, "decode": decode_ms},
            "hot_ms": hot_ms2 if hot_ms is not None else None, "clocks": clocks,
            "h2d": h2d, "d2h": d2h, "launches": launches_per_step * args.steps, "lens": x.lens, **extra}


def measure_prefill(M, w: W.Workload, dims, dev, stream, seed: int, chunk: int = 128, batch: int = 2,
                    context: int = 32768, iters: int = 5) -> dict:
    """Average device time of mla_decode_attn on a prefill chunk: `chunk` new tokens
    per sequence (already appended), each attending causally over its sequence."""
    import torch
    wp = dataclasses.replace(w, name="prefill", batch=batch, nq=chunk, context=context)
    x = W.make_decode_inputs(wp, seed=seed)
    to_bf16 = lambda b: torch.from_numpy(np.ascontiguousarray(b)).view(torch.bfloat16).to(dev)
    to_i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)
    pool, page_table, lens, pos = to_bf16(x.bits["pool"]), to_i32(x.page_table), to_i32(x.lens), to_i32(x.pos)
    T = wp.tokens
    q_lat = torch.empty((batch, chunk, wp.n_heads, wp.row), dtype=torch.bfloat16, device=dev)
    M.mla_absorb_q(dims, to_bf16(x.bits["q"]), pos, to_bf16(x.bits["w_uk"]), q_lat.view(T, wp.n_heads, wp.row),
                   stream=stream)
    w_uv = to_bf16(x.bits["w_uv"])
    out = torch.empty((batch, chunk, wp.n_heads, wp.v_head), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((batch, chunk, wp.n_heads), dtype=torch.float32, device=dev)
    ws = torch.empty(M.mla_decode_workspace_bytes(dims, batch, chunk), dtype=torch.uint8, device=dev)
    call = lambda: M.mla_decode_attn(dims, q_lat, pool, page_table, lens, w_uv, ws, out, lse, stream=stream)
    for _ in range(2):
        call()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(iters):
        call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    keys = int(sum(int(n) - chunk + i + 1 for n in x.lens for i in range(chunk)))   # visible keys, all queries
    flops = keys * wp.n_heads * 2 * (wp.row + wp.d_c) + T * wp.n_heads * 2 * wp.d_c * wp.v_head
    return {"time_us": e0.elapsed_time(e1) * 1000.0 / iters, "flops": flops, "launches": 2 * iters,
            "shape": f"{batch} sequences x {chunk} new tokens, context {context}, {wp.n_heads} heads"}


def measure_prefill_naive(w: W.Workload, dev, stream, seed: int, chunk: int, batch: int = 2,
                          context: int = 32768, iters: int = 3) -> dict:
    """The decompressing (naive) form of the same prefill chunk, for comparison with
    the absorbed form this library implements: K_nope = c W_UK^T and V = c W_UV^T for
    every cached token and head (cuBLAS bf16 GEMMs through torch), then attention of
    the chunk's queries over [K_nope || k_R] and V with torch's fused attention
    (cuDNN, else the memory-efficient kernel).  Library kernels, timed only to place
    the crossover; the gather of the paged cache into contiguous rows is not timed,
    and the causal mask inside the chunk is left out (it covers chunk^2 / 2 of the
    chunk x context scores)."""
    import torch
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel
    wp = dataclasses.replace(w, name="prefill", batch=batch, nq=chunk, context=context)
    x = W.make_decode_inputs(wp, seed=seed)
    to_bf16 = lambda b: torch.from_numpy(np.ascontiguousarray(b)).view(torch.bfloat16).to(dev)
    pool = to_bf16(x.bits["pool"])
    pt = torch.from_numpy(np.ascontiguousarray(x.page_table, dtype=np.int64)).to(dev)
    H, dn, dr, dv, dc = wp.n_heads, wp.qk_nope, wp.d_rope, wp.v_head, wp.d_c
    rows = pool[pt].reshape(batch, -1, wp.row)[:, :context]          # [B, N, d_c + d_rope], untimed gather
    c = rows[..., :dc].reshape(-1, dc).contiguous()
    k_r = rows[..., dc:].contiguous()
    w_uk = to_bf16(x.bits["w_uk"]).reshape(H * dn, dc)             # [H, d_h, d_c] rows
    w_uv = to_bf16(x.bits["w_uv"]).reshape(H * dv, dc)             # [H, d_v, d_c] rows
    q = to_bf16(x.bits["q"]).reshape(batch, chunk, H, dn + dr).transpose(1, 2)
    N = context

    def decompress():
        k_n = (c @ w_uk.t()).view(batch, N, H, dn)
        v = (c @ w_uv.t()).view(batch, N, H, dv)
        k = torch.cat([k_n, k_r.view(batch, N, 1, dr).expand(batch, N, H, dr)], dim=-1)
        return k.transpose(1, 2), v.transpose(1, 2)

    backend = None
    for b in (SDPBackend.CUDNN_ATTENTION, SDPBackend.EFFICIENT_ATTENTION):
        try:
            with sdpa_kernel([b]):
                k, v = decompress()
                F.scaled_dot_product_attention(q, k, v)
            backend = b
            break
        except RuntimeError:
            continue
    if backend is None:
        return {"chunk": chunk, "unavailable": "no fused attention backend takes d_qk 192, d_v 128 here"}
    torch.cuda.synchronize(dev)
    t_dec, t_att = [], []
    with torch.cuda.stream(stream), sdpa_kernel([backend]):
        for _ in range(iters + 1):
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record(stream)
            k, v = decompress()
            e1.record(stream)
            F.scaled_dot_product_attention(q, k, v)
            e2.record(stream)
            t_dec.append((e0, e1))
            t_att.append((e1, e2))
            del k, v
    torch.cuda.synchronize(dev)
    dec = float(np.mean([a.elapsed_time(b) for a, b in t_dec[1:]])) * 1000.0
    att = float(np.mean([a.elapsed_time(b) for a, b in t_att[1:]])) * 1000.0
    flops = batch * (2 * N * dc * H * (dn + dv) + 2 * chunk * N * H * (dn + dr + dv))
    return {"chunk": chunk, "time_us": dec + att, "decompress_us": dec, "attention_us": att, "flops": flops,
            "attention_backend": str(backend).split(".")[-1]}


def prefill_forms(args, w: W.Workload) -> None:
    """One JSON line: the absorbed form (this library's mla_decode_attn) against the
    decompressing form (library kernels) on prefill chunks of V3 heads over 32K keys."""
    import torch
    import head_latent_attention_07_b200 as M
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    dims = M.MlaDims(n_heads=w.n_heads, d_c=w.d_c, d_rope=w.d_rope, qk_nope=w.qk_nope, v_head=w.v_head,
                     d_model=w.d_model, page_size=w.page_size)
    rows = []
    for chunk in (128, 256, 512, 1024):
        ab = measure_prefill(M, w, dims, dev, stream, args.seed, chunk=chunk, iters=3)
        nv = measure_prefill_naive(w, dev, stream, args.seed, chunk)
        rows.append({"chunk": chunk, "absorbed_us": ab["time_us"], "absorbed_flops": ab["flops"],
                     "naive": nv})
        torch.cuda.empty_cache()
    print(json.dumps({"prefill_forms": rows, "batch": 2, "context": 32768, "heads": w.n_heads}), flush=True)


def measure_query_proj(M, w: W.Workload, dims, dev, stream, seed: int, iters: int = 50) -> dict:
    """Average device time of mla_query_proj (its two launches) with a 256 MB
    buffer rewritten between calls, so that the weights come from HBM each time;
    each call is bracketed by its own CUDA events on the launching stream.  Also
    the average over back-to-back calls that take, in turn, the weights of as many
    layers (copies) as exceed twice the L2: the weights again come from HBM, and
    each call overlaps its neighbours as a model's layers would."""
    import torch
    r = W.Q_LORA_RANK
    x = W.make_query_proj_inputs(w, seed, w.tokens, r)
    h, w_dq, w_uq = (torch.from_numpy(x[k]).view(torch.bfloat16).to(dev) for k in ("h", "w_dq", "w_uq"))
    c_q = torch.empty((w.tokens, r), dtype=torch.bfloat16, device=dev)
    q = torch.empty((w.tokens, w.n_heads, w.qk_nope + w.d_rope), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(3):
        M.mla_query_proj(dims, h, w_dq, w_uq, c_q, q, stream=stream)
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(iters):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        M.mla_query_proj(dims, h, w_dq, w_uq, c_q, q, stream=stream)
        e1.record(stream)
        times.append((e0, e1))
    torch.cuda.synchronize(dev)
    us = float(np.mean([a.elapsed_time(b) for a, b in times])) * 1000.0
    nbytes = (w_dq.numel() + w_uq.numel() + h.numel() + 2 * c_q.numel() + q.numel()) * 2
    # as a model's layers run it: back-to-back calls, each with another layer's
    # weights (copies whose total exceeds twice the L2), no flush in between
    layers = layer_copies((w_dq.numel() + w_uq.numel()) * 2)
    mats = [(w_dq, w_uq)] + [(w_dq.clone(), w_uq.clone()) for _ in range(layers - 1)]
    for i in range(2 * layers):
        M.mla_query_proj(dims, h, *mats[i % layers], c_q, q, stream=stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(iters):
        M.mla_query_proj(dims, h, *mats[i % layers], c_q, q, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    b2b_us = e0.elapsed_time(e1) * 1000.0 / iters
    del mats
    return {"time_us": us, "bytes_per_launch": nbytes, "launches": 2 * iters, "tokens": w.tokens,
            "layers_us": b2b_us, "layers": layers,
            "layers_bytes": layers * (w_dq.numel() + w_uq.numel()) * 2,
            "shape": f"c_Q[{w.tokens}, {r}] = h[{w.tokens}, {w.d_model}] . W_DQ^T; "
                     f"q[{w.tokens}, {w.n_heads}, {w.qk_nope + w.d_rope}] = c_Q . W_UQ^T"}


def measure_out_proj(M, w: W.Workload, dims, out, dev, stream, seed: int, iters: int = 50) -> dict:
    """Average device time of mla_out_proj over `iters` back-to-back launches on
    the decode output `out` (CUDA events on the launching stream, 3 warm-up launches)."""
    import torch
    x = W.make_out_proj_inputs(w, seed, w.tokens)
    w_o = torch.from_numpy(x["w_o"]).view(torch.bfloat16).to(dev)
    y = torch.empty((w.tokens, w.d_model), dtype=torch.bfloat16, device=dev)
    for _ in range(3):
        M.mla_out_proj(dims, out, w_o, y, stream=stream)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(iters):
        M.mla_out_proj(dims, out, w_o, y, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    nbytes = (w_o.numel() + out.numel() + y.numel()) * 2
    return {"time_us": e0.elapsed_time(e1) * 1000.0 / iters, "bytes_per_launch": nbytes, "launches": iters,
            "tokens": w.tokens, "shape": f"y[{w.tokens}, {w.d_model}] = o[{w.tokens}, {w.n_heads * w.v_head}]"
                                         f" . W_O[{w.d_model}, {w.n_heads * w.v_head}]^T"}


# ------------------------------------------------------------------ CPU oracle timing

class OracleArm:
    """The CPU oracle's absorbed form (float64 numpy), as it stands, on query
    tokens of this workload.  Inputs are drawn once; each measure() call runs
    whole query tokens (all heads) until ~budget_s of host time is spent."""

    def __init__(self, w: W.Workload, seed: int):
        from oracle import mla as O
        self.O, self.w = O, w
        try:
            from threadpoolctl import threadpool_info
            self.cores = max((int(i.get("num_threads", 1)) for i in threadpool_info()), default=1)
        except Exception:  # noqa: BLE001
            self.cores = 1
        # a uniform workload: one sequence's cache stands for all (same work per query token)
        x = W.make_decode_inputs(dataclasses.replace(w, batch=1) if w.context else w, seed=seed)
        self.args = dict(h=x.f64("h"), h_seq_idx=x.h_seq_idx, h_pos=x.h_pos, q=x.f64("q"), q_pos=x.pos,
                         pool=_Widen(x.bits["pool"]), page_table=x.page_table, lens=x.lens,
                         nq=x.workload.nq, w_dkv=x.f64("w_dkv"), w_uk=x.f64("w_uk"), w_uv=x.f64("w_uv"),
                         d_c=w.d_c)
        self.tokens = x.workload.tokens
        self.done = 0

    def measure(self, budget_s: float):
        n, t0 = 0, time.perf_counter()
        while n == 0 or time.perf_counter() - t0 < budget_s:
            self.O.decode_step(**self.args, form="absorbed", queries=[self.done % self.tokens])
            self.done += 1
            n += 1
        el = time.perf_counter() - t0
        ctx = f"context {self.w.context}" if self.w.context else "ragged contexts"
        return n / el, (f"oracle absorbed form (float64 numpy): {n} query token(s) x {self.w.n_heads} heads "
                        f"over {ctx} in {el:.1f} s, scaled to tokens/s")


class _Widen:
    """bf16 pool bits read as float32 rows on demand."""

    def __init__(self, bits):
        self.b, self.shape = bits, bits.shape

    def __getitem__(self, i):
        return W.bf16_to_f32(self.b[i])


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="v3", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prefill-forms", action="store_true",
                    help="only compare the absorbed and the decompressing prefill forms (one JSON line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    w = W.WORKLOADS[args.workload]
    if args.prefill_forms:
        if rank == 0:
            prefill_forms(args, w)
        return

    if args.impl == "reference":
        if rank != 0:
            return
        # each step: the oracle on a bounded sample (one query token at least)
        arm = OracleArm(w, args.seed)
        per_step = []
        budget = max(0.2, min(8.0, 120.0 / (args.steps + args.warmup)))
        for i in range(args.warmup + args.steps):
            v, sample = arm.measure(budget)
            if i >= args.warmup:
                per_step.append(v)
        value = float(np.mean(per_step))
        cores = arm.cores
        ms = 1000.0 * w.tokens / value
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": describe(w),
                "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                 "sample": sample},
                "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    r = run_ours(args, w, rank, world, local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, src = load_peaks()
    cnt = algorithmic_counts(w, r["lens"])
    T = w.tokens
    value = job_throughput(world, T, args.steps, r["ms_total"])
    dec_s = r["decode_ms"] / 1000.0
    gbs = cnt["bytes"] / dec_s / 1e9
    tfs = cnt["flops"] / dec_s / 1e12
    # the decode loop runs for seconds only on the larger workloads: the tensor peak
    # is the sustained (power-capped) figure there, the burst figure otherwise
    tc_key = "bf16_tflops_sustained" if r["decode_loop_ms"] >= 500.0 and "bf16_tflops_sustained" in peaks \
        else "bf16_tflops"
    t_hbm = cnt["bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_tc = cnt["flops"] / (peaks[tc_key] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    roof = ({"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s"} if bound == "hbm" else
            {"bound": "tensor", "achieved": tfs, "peak": peaks[tc_key], "unit": "TFLOP/s"})
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"], roof["traffic_source"] = profiled_traffic(w.name)
    roof["kernel"] = "mla_decode_attn (split + combine launches), timed in a loop of its own after the steps"
    roof["peak_source"] = (f"{src} (MEASURED_PEAKS.json: hbm_gbs, {tc_key})" if src == "measured" else "fallback")
    roof["hbm_frac"] = gbs / peaks["hbm_gbs"]
    roof["tensor_frac"] = tfs / peaks[tc_key]
    roof["time_us"] = r["decode_ms"] * 1000.0
    roof["bytes_per_launch"] = cnt["bytes"]
    roof["flops_per_launch"] = cnt["flops"]

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": r["ms_total"] / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {**describe(w, r["lens"]), "parallelism": f"dp{world} (independent replicas)"},
            "roofline": roof,
            "e2e": {"value": job_throughput(world, T, args.steps, r["e2e_ms"]), "unit": "tokens/s",
                    "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                    "copies": ("pinned host buffers, double-buffered on a second stream, inside the timed region"
                               if r["hot_ms"] is None else
                               "pinned host buffers, each step's copies serialised with it, L2 flushed before")},
            "gpu_launches": r["launches"], "clocks": r["clocks"],
            "phases_us": {k: v * 1000.0 for k, v in r["phases_ms"].items()}}
    if r["hot_ms"] is not None:
        line["hot_l2"] = {"value": job_throughput(world, T, args.steps, r["hot_ms"]), "unit": "tokens/s",
                          "ms_per_step": r["hot_ms"] / args.steps, "note": "the same steps back to back, cache hot in L2"}
    if "out_proj" in r:
        op = r["out_proj"]
        op_gbs = op["bytes_per_launch"] / (op["time_us"] * 1e-6) / 1e9
        line["next_rows"] = {"out_proj": {
            "kernel": "token_linear_kernel (mla_out_proj), timed alone after the step, not part of it",
            "shape": op["shape"], "bound": "hbm", "achieved": op_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": op_gbs / peaks["hbm_gbs"], "time_us": op["time_us"], "bytes_per_launch": op["bytes_per_launch"],
            "launches_timed": op["launches"], "l2": "W_O is larger than L2"}}
        qp = r["query_proj"]
        qp_gbs = qp["bytes_per_launch"] / (qp["time_us"] * 1e-6) / 1e9
        line["next_rows"]["query_proj"] = {
            "kernel": "token_linear_kernel x 2 (mla_query_proj), timed alone after the step, not part of it",
            "shape": qp["shape"], "bound": "hbm", "achieved": qp_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": qp_gbs / peaks["hbm_gbs"], "time_us": qp["time_us"], "bytes_per_call": qp["bytes_per_launch"],
            "launches_timed": qp["launches"], "l2": "256 MB buffer rewritten before each call",
            "layers_back_to_back": {
                "time_us": qp["layers_us"],
                "frac": qp["bytes_per_launch"] / (qp["layers_us"] * 1e-6) / 1e9 / peaks["hbm_gbs"],
                "l2": f"{qp['layers']} layers' W_DQ and W_UQ ({qp['layers_bytes'] / 1e6:.0f} MB) in turn, "
                      "back to back, no flush"}}
        pf = r["prefill"]
        pf_tfs = pf["flops"] / (pf["time_us"] * 1e-6) / 1e12
        line["next_rows"]["prefill"] = {
            "kernel": "mla_decode_attn (split + combine) on a prefill chunk, timed alone after the step",
            "shape": pf["shape"], "bound": "tensor", "achieved": pf_tfs, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": pf_tfs / peaks["bf16_tflops"], "time_us": pf["time_us"],
            "flops_per_call": pf["flops"], "launches_timed": pf["launches"]}
    if world == 1 and not args.no_cpu_baseline:
        arm = OracleArm(w, args.seed)
        v, sample = arm.measure(args.cpu_budget)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": arm.cores, "kind": "oracle",
                                "sample": sample}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
