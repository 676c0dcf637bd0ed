#!/usr/bin/env python3
"""Benchmark: chunked cache attention + summed weights + H2O eviction.

One step = one sequence pushed through the whole hot path, chunk by chunk
(h2o_evict_insert, then attn_chunk_with_scoresum), plus the final fold of the
last chunk's weights.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--only]
  python bench.py --impl reference ...   # the CPU oracle on the host cores

The printed line is the headline workload (default: the Qwen3-4B-shaped layer at
128K tokens, batch 1, 32 query / 8 KV heads, head_dim 128, bf16, a 32768-slot
cache, chunks of 1024); unless --only is given it also carries, under "configs",
the same measurements for every other workload: the tiny fp32 layer, the 64K
layer, the int8-cache layer and the 36-layer int4 stack at batch 4.  The stack
runs as one model: per chunk, every layer's eviction in one batched call
(h2o_evict_insert_many) and then every layer's attention, its inputs made per
chunk outside the timed region (the whole sequence would be ~216 GB).

Under torchrun: single layers run one independent layer per rank (seed + rank;
"weak" scaling); the stack's 36 layers are split round-robin over the ranks, so
the job processes the same tokens faster ("strong").  No collective runs on the
data path.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from h2o_kv_cache_attn_b200.configs import SHORT  # noqa: E402

METRIC = "chunked cache-attention+scoresum tokens/s; % BF16 tensor peak; evict µs/chunk"
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NESTED = ("tiny", "64k", "int8", "int4stack")  # measured beside the headline


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- #
def strip_comments(code: str) -> str:
    """C/C++ source without comments and blank lines, each line stripped (string
    literals are kept as they are; none of the kernels' contains a comment marker)."""
    code = re.sub(r"/\*.*?\*/", "", code, flags=re.S)
    code = re.sub(r"//[^\n]*", "", code)
    return "\n".join(line.strip() for line in code.splitlines() if line.strip())


def kernel_source_hash(files=None):
    """Hash of the code (comments excluded) of the CUDA sources a kernel is built from
    (all of csrc/ when files is None); paths are relative to csrc/."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "h2o_kv_cache_attn_b200", "csrc")
    if files is None:
        files = sorted(f for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))
    for f in files:
        with open(os.path.normpath(os.path.join(csrc, f)), encoding="utf-8") as fh:
            h.update(os.path.basename(f).encode() + strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_name, config):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current sources of that kernel and on this workload (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel_name)
    if not e or e.get("config") != config or e.get("source_hash") != kernel_source_hash(e.get("sources")):
        return None
    return e.get("bytes_per_launch")


def alg_flops_chunk(wl, n_valid, S):
    """Algorithmic attention FLOPs of one chunk of one layer: QK^T and PV over the
    valid slots, 4 * B * H_q * S * n_valid * d."""
    return 4.0 * wl.B * wl.Hq * S * n_valid * wl.d


def exec_flops_chunk(wl, n_valid, S):
    """Executed tensor FLOPs: the score-sum pass recomputes QK^T once more."""
    return 6.0 * wl.B * wl.Hq * S * n_valid * wl.d


def evict_bytes_chunk(wl, S):
    """Algorithmic HBM bytes of one layer's evict/insert call: scores read+write and
    w_prev read (3 * 4 * N_C), new K/V read (2 * S * d * 2), stored K/V rows and
    scales written, token_pos and slot list written, per (b, h_k)."""
    row = {"f32": wl.d * 4, "bf16": wl.d * 2, "i8": wl.d, "i4": wl.d // 2}[wl.kv_dtype]
    sc = 2 if wl.kv_dtype in ("i8", "i4") else 0
    per = 3 * 4 * wl.capacity + 2 * S * wl.d * 2 + 2 * S * (row + sc) + 2 * S * 4
    return per * wl.B * wl.Hk


def split_schedule(wl, S, sms):
    """Whether the library runs a chunk of S tokens of a quantized cache with the split
    (persistent) tensor-core schedule: the same rule as the library's (an even number
    of query tiles per KV group, the one-CTA-per-pair grid filling less than 75 % of
    its last wave, at least 4 units per SM and 4 K/V tiles)."""
    if wl.kv_dtype not in ("i8", "i4") or wl.d != 128 or wl.q_dtype != "bf16":
        return False
    tiles = -(-S // 128)
    n_qt = wl.q_g * tiles
    if n_qt % 2:
        return False
    pairs = wl.B * wl.Hk * n_qt // 2
    n_kt = -(-wl.capacity // 128)
    waves = -(-pairs // sms)
    return pairs / (waves * sms) < 0.75 and pairs * n_kt >= 4 * sms and n_kt >= 4


def tc_used(wl):
    """The tensor-core path serves head_dim 128 with a bf16, int8 or int4 cache and
    bf16 queries (the same rule as the library)."""
    return wl.d == 128 and wl.kv_dtype in ("bf16", "i8", "i4") and wl.q_dtype == "bf16"


def attention_launches(wl, S, n_valid, sms):
    """Kernels one attention call launches (the library's dispatch rules)."""
    if not tc_used(wl):
        return 2  # CUDA-core path: two passes
    if wl.kv_dtype == "bf16" and os.environ.get("H2OKV_TC_FUSED") != "1":
        pairs = wl.B * wl.Hk * ((wl.q_g * (-(-S // 128)) + 1) // 2)
        fill = pairs / (-(-pairs // sms) * sms)
        combine = fill < 0.75 and -(-n_valid // 128) >= 32
        return 3 + (1 if combine else 0)  # attention pass, [combine], score sums, reduction
    return 4 if split_schedule(wl, S, sms) else 2


def evict_launches(n_filled, S, capacity):
    """Kernels of one h2o_evict_insert call: fold (+ choose when evicting) + rows."""
    if S == 0:
        return 1
    return 2 if n_filled + S <= capacity else 3


def roofline(wl, at_ms, flops_alg, flops_exec, config_key, kernel):
    pk, pk_kind = peaks()
    at_s = sum(at_ms) / 1e3
    tf_alg = flops_alg / at_s / 1e12
    tf_exec = flops_exec / at_s / 1e12
    per_launch_alg = flops_alg / len(at_ms)
    per_launch_ms = sum(at_ms) / len(at_ms)
    if tc_used(wl):
        sus = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
        two_pass = wl.kv_dtype == "bf16" and os.environ.get("H2OKV_TC_FUSED") != "1"
        return {"bound": "tensor", "achieved": round(tf_alg, 2), "peak": sus, "unit": "TFLOP/s",
                "frac": round(tf_alg / sus, 4),
                "frac_of_burst_peak": round(tf_alg / pk["bf16_tflops"], 4),
                "burst_peak": pk["bf16_tflops"],
                "traffic": recorded_traffic("attn_fwd_kernel" if two_pass else "attn_tc_kernel",
                                            config_key),
                "kernel": kernel, "alg_flops_per_launch": per_launch_alg,
                "avg_launch_ms": round(per_launch_ms, 4),
                "pct_peak_exec": round(100 * tf_exec / sus, 2),
                "peak_kind": f"{pk_kind} bf16 dense, sustained (kernel timed inside a long step); "
                             "frac_of_burst_peak against the burst figure"}
    fma_peak = 148 * 128 * 2 * 1.965e9 / 1e12
    return {"bound": "alu", "achieved": round(tf_alg, 3), "peak": round(fma_peak, 1),
            "unit": "TFLOP/s", "frac": round(tf_alg / fma_peak, 4),
            "traffic": recorded_traffic("simt_attn_kernel", config_key),
            "kernel": kernel, "alg_flops_per_launch": per_launch_alg,
            "avg_launch_ms": round(per_launch_ms, 4),
            "peak_kind": "derived: 148 SMs x 128 FP32 FMA/clk x 2 x 1965 MHz"}


class EventClock:
    """Device time between points of the work on one stream (CUDA events)."""

    def __init__(self, stream):
        self.stream = stream

    def mark(self):
        import torch
        e = torch.cuda.Event(enable_timing=True)
        e.record(self.stream)
        return e

    def sync(self):
        import torch
        torch.cuda.synchronize()

    @staticmethod
    def ms(a, b):
        return a.elapsed_time(b)


# --------------------------------------------------------------------------- #
def run_layer(wl, config_key, steps, warmup, ws, rank, local, with_bwd, with_e2e):
    """One attention layer, the whole sequence per step (seed + rank under torchrun)."""
    import torch

    from h2o_kv_cache_attn_b200 import binding as hb
    from h2o_kv_cache_attn_b200 import dist as hdist
    from h2o_kv_cache_attn_b200.runner import LayerRunner
    from h2o_kv_cache_attn_b200.synth import ChunkSource

    hb.load()  # raises if the CUDA library is missing
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    src = ChunkSource(wl, layer=rank, device=dev)
    chunks = [src.chunk(c) for c in range(wl.n_chunks)]
    runner = LayerRunner(wl, dev, with_wq=False, with_lse=False)
    n_valid = [min(wl.capacity, sum(wl.chunk_len(i) for i in range(c + 1))) for c in range(wl.n_chunks)]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    def one_step(events=None):
        runner.reset()
        for c, (q, k, v) in enumerate(chunks):
            S = q.shape[2]
            if events is not None:
                e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
                e0.record(stream)
            runner.cache.evict_insert(runner.w_prev(), k, v, S, runner.P, None)
            if events is not None:
                e1.record(stream)
            runner.cache.attend(q, S, runner.P, runner.y if S == wl.chunk else torch.empty_like(q),
                                None, runner.w_cur(), None)
            if events is not None:
                e2.record(stream)
                events.append((c, e0, e1, e2))
            runner.chunk_index += 1
            runner.P += S
        runner.finish()

    for _ in range(warmup):
        one_step()
    torch.cuda.synchronize()
    hdist.barrier()
    torch.cuda.synchronize()
    events = []
    with ClockSampler(local) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            one_step(events)
        t1.record(stream)
        torch.cuda.synchronize()
    hdist.barrier()
    torch.cuda.synchronize()
    ms_total = hdist.max_over_ranks(t0.elapsed_time(t1))
    ms_step = ms_total / steps
    tokens_step = wl.B * wl.seq_len
    value = tokens_step * ws * steps / (ms_total / 1e3)

    # per-call durations inside the timed region
    ev_ms, at_ms, fl_exec, fl_alg, evict_full_ms = [], [], 0.0, 0.0, []
    for (c, e0, e1, e2) in events:
        ev = e0.elapsed_time(e1)
        ev_ms.append(ev)
        at_ms.append(e1.elapsed_time(e2))
        S = wl.chunk_len(c)
        fl_exec += exec_flops_chunk(wl, n_valid[c], S)
        fl_alg += alg_flops_chunk(wl, n_valid[c], S)
        if c * wl.chunk >= wl.capacity:  # a full cache: the choice runs
            evict_full_ms.append(ev)
    pk, _ = peaks()
    evict_us = statistics.median(evict_full_ms) * 1e3 if evict_full_ms else None
    evict_gbs = evict_bytes_chunk(wl, wl.chunk) / (evict_us * 1e-6) / 1e9 if evict_us else None
    launches_step = 2  # reset + final fold
    filled = 0
    for c in range(wl.n_chunks):
        S = wl.chunk_len(c)
        launches_step += evict_launches(filled, S, wl.capacity)
        filled = min(wl.capacity, filled + S)
        launches_step += attention_launches(wl, S, n_valid[c], sms)
    if tc_used(wl):
        kernel = ("attention call per chunk (attn_fwd_kernel + [combine_fwd_kernel] + scoresum_kernel"
                  " + reduce_w_kernel)" if wl.kv_dtype == "bf16" else
                  "attention call per chunk (attn_tc_kernel or split phases + reduce_w_kernel)")
    else:
        kernel = "attention call per chunk, CUDA-core path (2 passes)"
    res = {"value": value, "ms_per_step": ms_step, "steps": steps, "warmup": warmup,
           "roofline": roofline(wl, at_ms, fl_alg, fl_exec, config_key, kernel),
           "evict_us_per_chunk": round(evict_us, 2) if evict_us else None,
           "evict_gbs": round(evict_gbs, 1) if evict_gbs else None,
           "evict_frac_hbm": round(evict_gbs / pk["hbm_gbs"], 4) if evict_gbs else None,
           "attn_ms_per_step": round(sum(at_ms) / steps, 3),
           "evict_ms_per_step": round(sum(ev_ms) / steps, 3),
           "gpu_launches": launches_step * steps, "clocks": clk.summary(), "scaling": "weak",
           "layers_per_rank": 1}

    if with_bwd:
        # gradients of the last chunk's SDPA, outside the step; algorithmic FLOPs QK^T,
        # dy V^T, dS K, dS^T Q, P^T dy = 10 * B * H_q * S * n_valid * d
        q_l = chunks[-1][0]
        S_l = q_l.shape[2]
        lse_l = torch.empty(q_l.shape[:3], dtype=torch.float32, device=dev)
        y_l = torch.empty_like(q_l)
        runner.cache.attend(q_l, S_l, runner.P - S_l, y_l, lse_l, runner.w[0], None)
        g = torch.Generator(device=dev)
        g.manual_seed(7)
        dy_l = torch.randn(q_l.shape, generator=g, device=dev).to(q_l.dtype)
        dq_l = torch.empty(q_l.shape, dtype=torch.float32, device=dev)
        dk_l = torch.empty((wl.B, wl.Hk, wl.capacity, wl.d), dtype=torch.float32, device=dev)
        dv_l = torch.empty_like(dk_l)
        bwd_ms = []
        for it in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            runner.cache.attend_backward(q_l, dy_l, lse_l, S_l, runner.P - S_l, dq_l, dk_l, dv_l)
            e1.record(stream)
            torch.cuda.synchronize()
            if it:
                bwd_ms.append(e0.elapsed_time(e1))
        bwd = statistics.median(bwd_ms)
        res["bwd_ms_per_chunk"] = round(bwd, 3)
        res["bwd_tflops_alg"] = round(10.0 * wl.B * wl.Hq * S_l * n_valid[-1] * wl.d / (bwd * 1e-3) / 1e12, 2)

    if with_e2e:
        res["e2e"] = _layer_e2e(wl, runner, chunks, steps, ws, dev, stream)
    del chunks
    return res


def _layer_e2e(wl, runner, chunks, steps, ws, dev, stream):
    """The same metric through the public API with HOST buffers: pinned host inputs
    in, y and w out, every chunk.  One copy stream moves chunk c + 1's inputs in and
    another chunk c - 1's outputs out while chunk c computes (two device buffer sets;
    events order every reuse).  The timed region ends when the last output copy has
    landed."""
    import torch

    from h2o_kv_cache_attn_b200 import dist as hdist

    host = [(q.cpu().pin_memory(), k.cpu().pin_memory(), v.cpu().pin_memory()) for (q, k, v) in chunks]
    qdb = [torch.empty_like(host[0][0], device=dev) for _ in range(2)]
    kdb = [torch.empty_like(host[0][1], device=dev) for _ in range(2)]
    vdb = [torch.empty_like(host[0][2], device=dev) for _ in range(2)]
    ydb = [torch.empty_like(host[0][0], device=dev) for _ in range(2)]
    y_h = [torch.empty(host[0][0].shape, dtype=host[0][0].dtype).pin_memory() for _ in range(2)]
    w_h = [torch.empty((wl.B, wl.Hk, wl.capacity), dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for ch in host for t in ch)
    d2h = sum(t.numel() * t.element_size() for (t, _, _) in host) + \
        wl.n_chunks * (w_h[0].numel() * w_h[0].element_size())
    cs_in, cs_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ready = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]

    def e2e_step():
        runner.reset()
        stream.wait_stream(cs_out)  # the previous step's outputs have been copied out
        cs_in.wait_stream(stream)  # the previous step is done with both input sets
        last = None
        for c, (qh, kh, vh) in enumerate(host):
            S = qh.shape[2]
            b = c % 2
            same = S == wl.chunk
            qd, kd, vd, yd = (qdb[b], kdb[b], vdb[b], ydb[b]) if same else tuple(
                torch.empty_like(t, device=dev) for t in (qh, kh, vh, qh))
            with torch.cuda.stream(cs_in):
                if c >= 2:
                    cs_in.wait_event(consumed[b])  # chunk c - 2 no longer reads this input set
                qd.copy_(qh, non_blocking=True)
                kd.copy_(kh, non_blocking=True)
                vd.copy_(vh, non_blocking=True)
                ready[b].record(cs_in)
            stream.wait_event(ready[b])
            if c >= 2:
                stream.wait_event(out_done[b])  # chunk c - 2's y and w have been copied out
            runner.cache.evict_insert(runner.w_prev(), kd, vd, S, runner.P, None)
            w = runner.w_cur()
            runner.cache.attend(qd, S, runner.P, yd, None, w, None)
            consumed[b].record(stream)
            with torch.cuda.stream(cs_out):
                cs_out.wait_event(consumed[b])
                (y_h[b] if same else torch.empty(qh.shape, dtype=qh.dtype).pin_memory()).copy_(
                    yd, non_blocking=True)
                w_h[b].copy_(w, non_blocking=True)
                out_done[b].record(cs_out)
            last = out_done[b]
            runner.chunk_index += 1
            runner.P += S
        runner.finish()
        if last is not None:
            stream.wait_event(last)

    e2e_step()
    torch.cuda.synchronize()
    hdist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        e2e_step()
    t1.record(stream)
    torch.cuda.synchronize()
    hdist.barrier()
    ms_e2e = hdist.max_over_ranks(t0.elapsed_time(t1))
    return {"value": wl.B * wl.seq_len * ws * steps / (ms_e2e / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


# --------------------------------------------------------------------------- #
def run_stack_cfg(wl, config_key, ws, rank, local, warmup_chunks, with_e2e):
    """The stack: this rank's layers (round-robin), every chunk's eviction batched
    over them, inputs made per chunk outside the timed region.  One timed pass over
    the sequence after `warmup_chunks` chunks of warm-up."""
    import torch

    from h2o_kv_cache_attn_b200 import binding as hb
    from h2o_kv_cache_attn_b200 import dist as hdist
    from h2o_kv_cache_attn_b200.runner import LayerRunner
    from h2o_kv_cache_attn_b200.stack import run_stack
    from h2o_kv_cache_attn_b200.synth import ChunkSource

    hb.load()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    layers = hdist.layers_for_rank(wl.layers, ws, rank)
    one = wl.with_(layers=1)
    runners = {L: LayerRunner(one, dev, with_wq=False, with_lse=False) for L in layers}
    sources = {L: ChunkSource(wl, layer=L, device=dev) for L in layers}
    n_valid = [min(wl.capacity, sum(wl.chunk_len(i) for i in range(c + 1))) for c in range(wl.n_chunks)]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    clock = EventClock(stream)

    def evict(c, inputs):
        w = None if c == 0 else [runners[L].w_prev() for L in layers]
        S = wl.chunk_len(c)
        hb.h2o_evict_insert_many([runners[L].cache.handle for L in layers], w,
                                 [inputs[L][1] for L in layers], [inputs[L][2] for L in layers],
                                 S, runners[layers[0]].P, None)

    def attend(L, c, inp):
        r = runners[L]
        q = inp[0]
        S = q.shape[2]
        r.cache.attend(q, S, r.P, r.y if S == wl.chunk else torch.empty_like(q), None, r.w_cur(), None)
        r.chunk_index += 1
        r.P += S

    def finish():
        hb.h2o_evict_insert_many([runners[L].cache.handle for L in layers],
                                 [runners[L].w_prev() for L in layers], None, None, 0,
                                 runners[layers[0]].P, None)

    def reset():
        for r in runners.values():
            r.reset()

    # warm-up: the first chunks of the sequence, then back to an empty cache
    reset()
    run_stack(layers, min(warmup_chunks, wl.n_chunks), wl.chunk_len,
              lambda L, c: sources[L].chunk(c), evict, attend, lambda: None, clock)
    reset()
    torch.cuda.synchronize()
    hdist.barrier()
    with ClockSampler(local) as clk:
        times = run_stack(layers, wl.n_chunks, wl.chunk_len, lambda L, c: sources[L].chunk(c),
                          evict, attend, finish, clock)
    hdist.barrier()
    ms_step = hdist.max_over_ranks(times.total_ms)
    tokens = wl.B * wl.seq_len  # every layer of the stack sees these tokens
    value = tokens / (ms_step / 1e3)
    fl_alg = sum(alg_flops_chunk(wl, n_valid[c], wl.chunk_len(c)) for c in range(wl.n_chunks)) * len(layers)
    fl_exec = sum(exec_flops_chunk(wl, n_valid[c], wl.chunk_len(c)) for c in range(wl.n_chunks)) * len(layers)
    # per-layer attention launches: the time per chunk covers all of this rank's layers
    at_ms = [a / len(layers) for a in times.attn_ms for _ in layers]
    pk, _ = peaks()
    full = [e for c, e in enumerate(times.evict_ms) if c * wl.chunk >= wl.capacity]
    evict_us = statistics.median(full) * 1e3 if full else None
    ev_bytes = evict_bytes_chunk(wl, wl.chunk) * len(layers)
    evict_gbs = ev_bytes / (evict_us * 1e-6) / 1e9 if evict_us else None
    launches = 2 * len(layers) + 1  # resets + the batched final fold
    filled = 0
    for c in range(wl.n_chunks):
        S = wl.chunk_len(c)
        launches += evict_launches(filled, S, wl.capacity)
        filled = min(wl.capacity, filled + S)
        launches += attention_launches(wl, S, n_valid[c], sms) * len(layers)
    res = {"value": value, "ms_per_step": ms_step, "steps": 1,
           "warmup": f"{warmup_chunks} chunks of the stack",
           "roofline": roofline(wl, at_ms, fl_alg, fl_exec, config_key,
                                "attention call per chunk and layer (int4 cache)"),
           "evict_us_per_chunk": round(evict_us, 2) if evict_us else None,
           "evict_scope": f"one h2o_evict_insert_many call over {len(layers)} layers x batch "
                          f"{wl.B} x {wl.Hk} KV heads",
           "evict_gbs": round(evict_gbs, 1) if evict_gbs else None,
           "evict_frac_hbm": round(evict_gbs / pk["hbm_gbs"], 4) if evict_gbs else None,
           "attn_ms_per_step": round(sum(times.attn_ms), 3),
           "evict_ms_per_step": round(sum(times.evict_ms), 3),
           "gpu_launches": launches, "clocks": clk.summary(), "scaling": "strong",
           "layers_per_rank": len(layers),
           "timed_region": "sum over chunks of the device time of the batched eviction and the "
                           "layers' attention (inputs made between chunks, outside it)"}

    if with_e2e:
        # host inputs: two pinned chunk buffers per layer, copied in every chunk (the
        # sequence itself does not fit host memory); y and w of every layer copied out
        host = {L: [tuple(t.cpu().pin_memory() for t in sources[L].chunk(i)) for i in range(2)]
                for L in layers}
        dev_in = {L: [tuple(torch.empty_like(t, device=dev) for t in host[L][0]) for _ in range(2)]
                  for L in layers}
        y_h = {L: torch.empty(host[L][0][0].shape, dtype=host[L][0][0].dtype).pin_memory() for L in layers}
        w_h = {L: torch.empty((wl.B, wl.Hk, wl.capacity), dtype=torch.float32).pin_memory() for L in layers}
        cs_in, cs_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        h2d = d2h = 0

        def make_dev(L, c):
            nonlocal h2d
            src_h = host[L][c % 2]
            dst = dev_in[L][c % 2]
            with torch.cuda.stream(cs_in):
                cs_in.wait_stream(stream)  # chunk c - 2 has finished with this buffer set
                for d_, h_ in zip(dst, src_h):
                    d_.copy_(h_, non_blocking=True)
                    h2d += h_.numel() * h_.element_size()
            stream.wait_stream(cs_in)
            return dst

        def attend_out(L, c, inp):
            nonlocal d2h
            attend(L, c, inp)
            r = runners[L]
            with torch.cuda.stream(cs_out):
                cs_out.wait_stream(stream)
                y_h[L].copy_(r.y, non_blocking=True)
                w_h[L].copy_(r.w[(r.chunk_index - 1) % 2], non_blocking=True)
                d2h += y_h[L].numel() * y_h[L].element_size() + w_h[L].numel() * 4

        reset()
        torch.cuda.synchronize()
        hdist.barrier()
        # the timed region spans the whole pass, copies included
        t0 = clock.mark()
        run_stack(layers, wl.n_chunks, wl.chunk_len, make_dev, evict, attend_out, finish, clock)
        stream.wait_stream(cs_out)
        t1 = clock.mark()
        clock.sync()
        hdist.barrier()
        ms = hdist.max_over_ranks(EventClock.ms(t0, t1))
        res["e2e"] = {"value": tokens / (ms / 1e3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h,
                      "note": "host inputs cycle through two pinned chunk buffers per layer"}
    del runners
    torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------------------- #
def _limit_blas_threads(n=1):
    try:
        import threadpoolctl
        threadpoolctl.threadpool_limits(n)
    except Exception:
        pass


def _start_worker(n):
    _limit_blas_threads(n)
    return os.getpid()


def _oracle_group(task):
    """One (batch row, KV head) group of one steady-state eviction chunk in the oracle:
    a full cache of earlier tokens with random scores, then the chunk's evict/insert and
    the attention with summed weights of its first R query rows.  Returns the seconds
    of those two steps."""
    import oracle
    (q_g, d, capacity, kv, S, R, P, q, k, v, seed) = task
    rng = np.random.default_rng(seed)
    oc = oracle.OracleCache(1, q_g, 1, d, capacity, kv)
    kk = rng.standard_normal((1, 1, capacity, d)).astype(np.float32)
    vv = rng.standard_normal((1, 1, capacity, d)).astype(np.float32)
    oc.evict_insert(None, kk, vv, capacity, P - capacity)
    oc.scores[:] = rng.random(oc.scores.shape).astype(np.float32)
    w_prev = rng.random((1, 1, capacity)).astype(np.float32)
    t0 = time.perf_counter()
    oc.evict_insert(w_prev, k, v, S, P)
    oc.attend(q[:, :, :R], R, P)
    return time.perf_counter() - t0


def oracle_sample(wl, rows=256, layer=0):
    """Time the CPU oracle on a bounded sample of one steady-state eviction chunk:
    every (batch row, KV head) group inserts the chunk and attends with its first
    `rows` query rows, one spawned process per group, the host cores shared out
    among them as BLAS threads.  The sample's time is the slowest group's;
    tokens/s = B * rows over that time (divided by the layers of a stack)."""
    import concurrent.futures as cf
    import multiprocessing as mp

    from h2o_kv_cache_attn_b200.synth import ChunkSource

    groups = wl.B * wl.Hk
    chunk = -(-wl.capacity // wl.chunk) + 1  # the second eviction chunk
    src = ChunkSource(wl, layer, "cpu")
    q, k, v = (t.float().numpy() for t in src.chunk(chunk))
    S = q.shape[2]
    R = min(rows, S)
    P = chunk * wl.chunk
    tasks = []
    for gi in range(groups):
        b, g = divmod(gi, wl.Hk)
        tasks.append((wl.q_g, wl.d, wl.capacity, wl.kv_dtype, S, R, P,
                      np.ascontiguousarray(q[b:b + 1, g * wl.q_g:(g + 1) * wl.q_g]),
                      np.ascontiguousarray(k[b:b + 1, g:g + 1]),
                      np.ascontiguousarray(v[b:b + 1, g:g + 1]), 1 + gi))
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    workers = max(1, min(cores, groups))
    threads = max(1, cores // workers)
    with cf.ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn"),
                                initializer=_limit_blas_threads, initargs=(threads,)) as ex:
        list(ex.map(_start_worker, [threads] * workers))  # every worker up before timing
        t0 = time.perf_counter()
        secs = list(ex.map(_oracle_group, tasks))
        wall = time.perf_counter() - t0
    rounds = -(-groups // workers)
    sample_s = max(secs) * rounds * wl.layers
    return {"value": wl.B * R / sample_s, "unit": UNIT, "cores": workers * threads, "kind": "oracle",
            "sample": (f"one steady-state eviction chunk (S={S}, P={P}): every one of the {groups} "
                       f"(batch, KV-head) groups inserts it and attends with its first {R} query "
                       f"rows; float64 numpy oracle, {workers} spawned processes x {threads} BLAS "
                       f"threads on {cores} host cores; slowest group {max(secs):.2f} s "
                       f"(wall {wall:.2f} s)" + (f", x{rounds} rounds" if rounds > 1 else "")
                       + (f", x{wl.layers} layers" if wl.layers > 1 else "")),
            "seconds": wall}


# --------------------------------------------------------------------------- #
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="128k", choices=sorted(SHORT))
    ap.add_argument("--only", action="store_true", help="measure the named workload only")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--stack-warmup-chunks", type=int, default=3)
    args = ap.parse_args()
    wl = SHORT[args.config]
    if args.warmup < 3:
        print("warning: --warmup < 3; using 3", file=sys.stderr)
        args.warmup = 3
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))

    def config_of(w):
        return {"workload": w.name, "batch": w.B, "q_heads": w.Hq, "kv_heads": w.Hk,
                "head_dim": w.d, "cache_slots": w.capacity, "seq_len": w.seq_len,
                "chunk": w.chunk, "kv_dtype": w.kv_dtype, "layers": w.layers,
                "parallelism": (f"stack layers round-robin over {ws} rank(s) (no collective)"
                                if w.layers > 1 else f"independent layers x{ws} (no collective)"),
                "l2": "inputs larger than L2 (cache buffers + chunk inputs > 126 MB per step)"
                      if w.name != SHORT["tiny"].name else "tiny workload: resident in L2"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        vals = []
        for s in range(args.warmup + args.steps):
            r = oracle_sample(wl, rows=32)
            if s >= args.warmup:
                vals.append(r)
        value = statistics.median(v["value"] for v in vals)
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": wl.B * wl.seq_len / value * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded, recipe of the workload)", "config": config_of(wl),
                "cpu_baseline": {k: vals[-1][k] for k in ("kind", "cores", "sample")} | {"value": value},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    from h2o_kv_cache_attn_b200 import dist as hdist

    ws, rank, local = hdist.init("nccl")

    def measure(w, key, headline):
        if w.layers > 1:
            return run_stack_cfg(w, key, ws, rank, local, args.stack_warmup_chunks, with_e2e=True)
        return run_layer(w, key, args.steps, args.warmup, ws, rank, local, with_bwd=headline,
                         with_e2e=True)

    res = measure(wl, args.config, True)
    nested = {}
    if not args.only:
        for key in NESTED:
            if key == args.config:
                continue
            w = SHORT[key]
            r = measure(w, key, False)
            r["config"] = config_of(w)
            r["metric"] = METRIC
            r["unit"] = UNIT
            r["dtype"] = "f32" if w.q_dtype == "f32" else "bf16"
            nested[w.name] = r
    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(wl)
        cpu.pop("seconds", None)
    if rank == 0:
        extra = {k: v for k, v in res.items()
                 if k not in ("value", "ms_per_step", "steps", "warmup", "roofline", "e2e",
                              "gpu_launches", "clocks", "scaling")}
        line = {"metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": ws,
                "steps": res["steps"], "warmup": res["warmup"], "ms_per_step": res["ms_per_step"],
                "higher_is_better": True, "scaling": res["scaling"], "vs_baseline": None,
                "dtype": "f32" if wl.q_dtype == "f32" else "bf16",
                "data": "synthetic (seeded N(0,1), 1% heavy-hitter keys x4 where the workload has "
                        "them, bf16 or f32)",
                "config": config_of(wl), "roofline": res["roofline"], "cpu_baseline": cpu,
                "e2e": res["e2e"],
                "gpu_launches": res["gpu_launches"],
                "clocks": res["clocks"], **extra}
        if nested:
            line["configs"] = nested
        print(json.dumps(line))
    hdist.shutdown()
    return 0


if __name__ == "__main__":
    sys.exit(main())
