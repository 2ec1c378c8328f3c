"""Benchmark of the InfLLM block-memory attention layer on B200.

One step = one pass of the whole hot path over one batch: the Mistral-7B-shaped 128K-token
stream (256 chunks of 512 tokens: append + unit lookup + attention per chunk), inputs
resident in HBM.  Prints ONE JSON line (rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload mistral_128k] [--no-decode] [--no-e2e]

Multi-GPU: one process per GPU (torchrun); the layer does not shard, so every rank runs an
independent replica of the workload (weak scaling) and the device time is the max over ranks.
`--impl reference` times the fp64 CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "prefill tok/s and decode \u00b5s/step at 128K\u20131M ctx; % of HBM / TC roofline"


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sust=d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                    sm_max=d.get("sm_max_mhz", 1965.0), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sust=1400.0, sm_max=1965.0, src="fallback")


# ------------------------------------------------------------------------------------------------
# distributed plumbing (replicas only)


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def dist_init(backend):
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=600))
    return rank, world


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        t = torch.tensor([x], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return x


# ------------------------------------------------------------------------------------------------
# clocks during the timed region


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.skip = 0
        self.proc = None
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            # nvidia-smi takes a while to start: wait (bounded) for its first sample, so that sampling is
            # live when the timed region begins; only the samples after this one are summarised
            t0 = time.time()
            while not self.rows and time.time() - t0 < 5.0 and self.proc.poll() is None:
                time.sleep(0.01)
            self.skip = len(self.rows)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def __exit__(self, *a):
        if self.proc:
            # a region shorter than the sampling period still gets the sample that ends it
            t0 = time.time()
            while len(self.rows) <= self.skip and time.time() - t0 < 0.5 and self.proc.poll() is None:
                time.sleep(0.01)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)

    def summary(self):
        rows = self.rows[self.skip:] or self.rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 5 + i and r[5 + i] == "Active"})
        load = [s for s in sm if s > 0.5 * (max(sm) if sm else 1)]
        return {"sm_mhz": float(np.median(load)) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------------------------------------
# algorithmic work


def chunk_flops(w, c0, n):
    """4*d*sum_t sum_h |K_t| for a chunk: QK^T and PV multiply-adds (2 flops each) per key and dim."""
    S, W, U, k, d = w.n_sink, w.window, w.unit_size, w.top_k, w.head_dim
    x = c0 - W - S
    nm = x // U if x > 0 else 0
    kk = min(k, nm)
    B = S + U * nm
    t = c0 + np.arange(n, dtype=np.int64)
    keys = np.minimum(S, t + 1) + kk * U + np.maximum(0, t - B + 1)
    return 4.0 * d * float(keys.sum()) * w.n_q_heads


def decode_bytes(w, t, score_mode):
    """Algorithmic HBM bytes of one decode step: unit scoring operand + attended K/V."""
    S, W, U, k, d, Hkv = w.n_sink, w.window, w.unit_size, w.top_k, w.head_dim, w.n_kv_heads
    x = t - W - S
    nm = x // U if x > 0 else 0
    kk = min(k, nm)
    B = S + U * nm
    keys = min(S, t + 1) + kk * U + (t - B + 1)
    elt = 2 if w.dtype == "bf16" else 4
    per_unit = {"reps": w.n_reps * d * elt, "repsum": d * 4, "meankey": d * elt}[score_mode]
    return nm * Hkv * per_unit + keys * Hkv * d * elt * 2


# ------------------------------------------------------------------------------------------------
# our implementation


def to_dev(a, torch, device):
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


def gen_full(w, torch, device):
    q = np.empty((w.n_tokens, w.n_q_heads, w.head_dim), dtype=np.uint16 if w.dtype == "bf16" else np.float32)
    k = np.empty((w.n_tokens, w.n_kv_heads, w.head_dim), dtype=q.dtype)
    v = np.empty_like(k)
    step = 16384
    for t0 in range(0, w.n_tokens, step):
        n = min(step, w.n_tokens - t0)
        q[t0:t0 + n], k[t0:t0 + n], v[t0:t0 + n] = synth.gen_chunk(w, t0, n)
    return q, k, v


ATTN_PROFILE = os.path.join(ROOT, "profiles", "k_attn_tc_mistral_128k.md")
ATTN_SOURCE = os.path.join(ROOT, "block_memory_sparse_b200", "csrc", "attend_tc.cu")


def attn_device_hash(src=None):
    """sha256 of the attention kernel's device code: attend_tc.cu up to its host-side part (the
    tensor-map encoding and the launcher), which does not change what the kernel moves, with
    comments, trailing blanks and empty lines removed (editing a comment does not change the kernel)."""
    import hashlib
    import re
    src = open(ATTN_SOURCE).read() if src is None else src
    cut = src.find("typedef CUresult (*EncodeTiledFn)")
    code = src if cut < 0 else src[:cut]
    code = re.sub(r"/\*.*?\*/", "", code, flags=re.S)
    code = "\n".join(x for x in (line.split("//", 1)[0].rstrip() for line in code.splitlines()) if x)
    return hashlib.sha256(code.encode()).hexdigest()


def attn_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, or None when the kernel's
    device code has changed since the counters were taken (its sha256 is recorded there)."""
    import re
    try:
        txt = open(ATTN_PROFILE).read()
        want = re.search(r"attend_tc\.cu device-code sha256: ([0-9a-f]{64})", txt).group(1)
        traffic = float(re.search(r"dram bytes per launch: ([0-9.eE+]+)", txt).group(1))
    except (OSError, AttributeError, ValueError):
        return None
    return traffic if attn_device_hash() == want else None


def workload_config(w, world, big=True, in_bytes=None):
    """The `config` object of the JSON line (the same for both arms)."""
    if in_bytes is None:
        elt = 2 if w.dtype == "bf16" else 4
        in_bytes = w.n_tokens * (w.n_q_heads + 2 * w.n_kv_heads) * w.head_dim * elt
    l2 = (f"inputs larger than L2 ({in_bytes / 1e9:.2f} GB of Q/K/V per step)" if big else
          f"inputs ({in_bytes / 1e6:.1f} MB) smaller than L2: L2 flushed (256 MB read) before every step, "
          "steps timed one by one, median")
    return {"workload": f"{w.name}: {w.n_q_heads}q/{w.n_kv_heads}kv heads, d={w.head_dim}, "
                        f"{w.n_tokens} tokens in {w.chunk}-token chunks, W={w.window}, S={w.n_sink}, "
                        f"U={w.unit_size}, r={w.n_reps}, k={w.top_k}, base={w.rope_base:g}, {w.dtype}",
            "global_batch": 1 * world, "seq_len": w.n_tokens, "parallelism": f"replicas x{world}", "l2": l2}


L2_BYTES = 126 * 1024 * 1024


def attn_roofline(w, st, flops, P, clk):
    """Roofline object of the chunk-attention kernel from its event-timed launches.  The tcgen05 kernel
    is a bf16 contraction: its peak is the measured bf16 GEMM rate, burst when the clocks sampled over
    the attention-only pass sat at their maximum with no power cap (the kernel then runs as a short
    burst), else sustained; both fractions are reported.  The fp32 CUDA-core kernel is bound by FP32
    FMA issue: 148 SMs x 128 lanes x 2 flops x the maximum SM clock."""
    att_ms, n_att = st["ms_attend"], st["n_attend"]
    achieved = flops / (att_ms / 1e3) / 1e12 if att_ms > 0 else None
    if st["attend_path"] == 1:
        c = clk.summary()
        capped = "sw_power_cap" in c["reasons"]
        at_max = c["sm_mhz"] is not None and c["sm_max_mhz"] and c["sm_mhz"] >= 0.95 * c["sm_max_mhz"]
        burst = bool(at_max and not capped)
        peak = P["bf16"] if burst else P["bf16_sust"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": (achieved / peak) if achieved else None,
                "frac_of_burst": (achieved / P["bf16"]) if achieved else None,
                "frac_of_sustained": (achieved / P["bf16_sust"]) if achieved else None,
                "traffic": attn_traffic() if w.name == "mistral_128k" else None,
                "kernel": "attention (tcgen05)",
                "peak_source": f"{P['src']} bf16 {'burst' if burst else 'sustained'} (clocks over the attention pass: "
                               f"median {c['sm_mhz']} of {c['sm_max_mhz']} MHz, reasons {c['reasons']})",
                "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one steady-chunk launch "
                                  "(profiles/k_attn_tc_mistral_128k.md); null if the kernel changed since, or for "
                                  "another workload"}
    else:
        peak = 148 * 128 * 2 * P["sm_max"] * 1e6 / 1e12
        roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": (achieved / peak) if achieved else None, "traffic": None,
                "kernel": "attention (CUDA cores, fp32)", "peak_source": "148 SMs x 128 FP32 lanes x 2 x max SM clock"}
    roof["avg_launch_ms"] = att_ms / n_att if n_att else None
    roof["launches"] = n_att
    roof["timing"] = "CUDA events around each attention launch, over a repeat of the timed steps"
    return roof


def time_prefill(args, w, torch, device, stream, local, world, P, plan=None):
    """The whole-prompt prefill of workload w (reset + infllm_prefill per step).  Inputs larger than L2 are
    timed as K back-to-back steps; smaller ones step by step, each after an L2 flush (median reported).
    With a KV-head shard plan, this rank runs its heads' slice of the layer (strong scaling: all ranks
    together process the prompt once; the output gather is the model's tensor-parallel step, outside).
    Returns (fields of the JSON line, layer, host inputs)."""
    from block_memory_sparse_b200 import InfLLMLayer
    chunks = synth.chunk_bounds(w)
    q_h, k_h, v_h = gen_full(w, torch, device)
    if plan is not None:
        q_h = np.ascontiguousarray(q_h[:, plan.q0:plan.q1])
        k_h = np.ascontiguousarray(k_h[:, plan.kv0:plan.kv1])
        v_h = np.ascontiguousarray(v_h[:, plan.kv0:plan.kv1])
        w = w.replace(n_q_heads=plan.q1 - plan.q0, n_kv_heads=plan.kv1 - plan.kv0)
    Q, K, V = (to_dev(a, torch, device) for a in (q_h, k_h, v_h))
    OUT = torch.empty_like(Q)
    in_bytes = q_h.nbytes + k_h.nbytes + v_h.nbytes
    big = in_bytes > L2_BYTES
    layer = InfLLMLayer.from_workload(w, max_tokens=w.n_tokens, max_chunk=w.chunk)

    def one_step():  # the whole prompt, chunk by chunk, in one call of the public API
        layer.reset()
        layer.prefill(Q, K, V, w.chunk, out=OUT)

    flush = None if big else torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    fsum = torch.empty((), dtype=torch.float32, device=device)
    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    layer.set_profiling(False)  # no events in the timed steps: they would break launch chaining
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        if big:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(args.steps):
                one_step()
            e1.record(stream)
            torch.cuda.synchronize()
            ms_step = e0.elapsed_time(e1) / args.steps
        else:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
            for a, b2 in evs:
                torch.sum(flush, dim=0, out=fsum)  # read 256 MB (> L2) before every step
                a.record(stream)
                one_step()
                b2.record(stream)
            torch.cuda.synchronize()
            ms_step = float(np.median([a.elapsed_time(b2) for a, b2 in evs]))
    barrier()
    ms_step = max_over_ranks(ms_step, device)
    launches = layer.stats()["kernel_launches"]
    # the attention kernel's own duration: the same steps again with CUDA events around each
    # attention launch on the layer's stream (outside the timed region: events serialise it)
    layer.set_profiling(["attend"])
    with ClockSampler(local) as clk_att:
        for _ in range(args.steps):
            if not big:
                torch.sum(flush, dim=0, out=fsum)
            one_step()
        torch.cuda.synchronize()
    st = layer.stats()
    # where a step's time goes: one more step with events around every launch (diagnostic only;
    # the events break launch overlap, so these sum to more than the timed step)
    layer.set_profiling(True)
    one_step()
    torch.cuda.synchronize()
    split = layer.stats()
    layer.set_profiling(False)
    flops = sum(chunk_flops(w, c0, n) for c0, n in chunks) * args.steps
    tokens_all = w.n_tokens * (1 if plan is not None else world)  # shards split one prompt; replicas run one each
    fields = {"value": tokens_all / (ms_step / 1e3), "unit": "tok/s", "ms_per_step": ms_step,
              "dtype": w.dtype, "config": workload_config(w, world, big, in_bytes),
              "roofline": attn_roofline(w, st, flops, P, clk_att), "gpu_launches": launches * (1 if big else 1),
              "clocks": clk.summary(),
              "time_split_ms_per_step": {k: split[f"ms_{k}"] for k in ("append", "reps", "prep", "select", "attend")}}
    del Q, K, V, OUT, flush
    return fields, layer, (q_h, k_h, v_h)


def run_ours(args, rank, world):
    import torch

    _, _, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    w = synth.WORKLOADS[args.workload]
    if args.tokens:
        w = w.replace(n_tokens=min(args.tokens, w.n_tokens))
    P = peaks()
    stream = torch.cuda.current_stream(device)
    plan = None
    if args.parallel == "kv" and world > 1:
        from block_memory_sparse_b200.sharding import ShardPlan
        plan = ShardPlan(w.n_q_heads, w.n_kv_heads, world, rank)
    fields, layer, (q_h, k_h, v_h) = time_prefill(args, w, torch, device, stream, local, world, P, plan)
    if plan is not None:
        fields["config"]["parallelism"] = f"KV heads split over {world} ranks ({plan.kv_per_rank} per rank)"
    res = {"metric": METRIC, "value": fields["value"], "unit": "tok/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": fields["ms_per_step"], "higher_is_better": True,
           "scaling": "strong" if plan is not None else "weak", "vs_baseline": None, "dtype": w.dtype,
           "data": "synthetic (seeded Philox normals, K channel bias N(0,4))", "config": fields["config"],
           "roofline": fields["roofline"], "gpu_launches": fields["gpu_launches"], "clocks": fields["clocks"],
           "time_split_ms_per_step": fields["time_split_ms_per_step"]}
    if not args.no_e2e and plan is None:
        res["e2e"] = run_e2e(args, w, layer, q_h, k_h, v_h, torch, device, stream, world, args.e2e_group)
    layer.close()
    del q_h, k_h, v_h
    torch.cuda.empty_cache()
    if rank == 0 and not args.no_cpu:
        res["cpu_baseline"] = cpu_baseline(w.name)
    # the other prefill workloads: same metric, their own roofline and oracle baseline
    if not args.no_others:
        others = {}
        for name in ("llama3_128k", "needle_256k", "tiny_f32"):
            if name == w.name:
                continue
            wo = synth.WORKLOADS[name]
            f, lo, _ = time_prefill(args, wo, torch, device, stream, local, world, P)
            lo.close()
            torch.cuda.empty_cache()
            if rank == 0 and not args.no_cpu:
                f["cpu_baseline"] = cpu_baseline(name)
            others[name] = f
        res["other_workloads"] = others
    if not args.no_decode:
        res["decode"] = run_decode(args, torch, device, stream, local)
    return res


def run_e2e(args, w, layer, q_h, k_h, v_h, torch, device, stream, world, group_chunks=32):
    """Same prompt through the public API with inputs in pinned host memory and the output read
    back to host: host<->device copies are inside the timed region.  The prompt goes in groups
    of `group_chunks` chunks (one infllm_prefill call each); the copies run on two side streams
    (host->device of group i+1 and device->host of group i-1 overlap the layer's work on group
    i), with double-buffered device staging and events for the order."""
    gt = group_chunks * w.chunk
    groups = [(g0, min(gt, w.n_tokens - g0)) for g0 in range(0, w.n_tokens, gt)]
    pin = lambda a: (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if a.dtype == np.uint16
                     else torch.from_numpy(a)).pin_memory()
    qp, kp, vp = pin(q_h), pin(k_h), pin(v_h)
    outp = torch.empty_like(qp).pin_memory()
    mk = lambda h: torch.empty((gt, h, w.head_dim), dtype=qp.dtype, device=device)
    bufs = [(mk(w.n_q_heads), mk(w.n_kv_heads), mk(w.n_kv_heads), mk(w.n_q_heads)) for _ in range(2)]
    h2d_s, d2h_s = torch.cuda.Stream(device), torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

    def one_step():
        layer.reset()
        for i, (g0, n) in enumerate(groups):
            b = i & 1
            qd, kd, vd, od = bufs[b]
            with torch.cuda.stream(h2d_s):
                if i >= 2:
                    h2d_s.wait_event(comp_done[b])  # group i-2 no longer reads this buffer
                qd[:n].copy_(qp[g0:g0 + n], non_blocking=True)
                kd[:n].copy_(kp[g0:g0 + n], non_blocking=True)
                vd[:n].copy_(vp[g0:g0 + n], non_blocking=True)
                h2d_done[b].record(h2d_s)
            stream.wait_event(h2d_done[b])
            if i >= 2:
                stream.wait_event(d2h_done[b])  # group i-2's output has left this buffer
            layer.prefill(qd[:n], kd[:n], vd[:n], w.chunk, out=od[:n])
            comp_done[b].record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(comp_done[b])
                outp[g0:g0 + n].copy_(od[:n], non_blocking=True)
                d2h_done[b].record(d2h_s)
        stream.wait_event(d2h_done[(len(groups) - 1) & 1])

    one_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        one_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), device)
    elt = qp.element_size()
    h2d = w.n_tokens * (w.n_q_heads + 2 * w.n_kv_heads) * w.head_dim * elt
    d2h = w.n_tokens * w.n_q_heads * w.head_dim * elt
    return {"value": w.n_tokens * args.steps * world / (ms / 1e3), "unit": "tok/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms / args.steps,
            "copies": f"pinned host buffers; {group_chunks}-chunk groups, host->device and device->host on side "
                      f"streams overlapping compute"}


def run_decode(args, torch, device, stream, local):
    """Decode workload: 8192-unit (1M-token) memory built with append_chunk (untimed), then
    single-token steps, each timed with CUDA events after an L2 flush."""
    from block_memory_sparse_b200 import InfLLMLayer
    w = synth.WORKLOADS["decode_1m"]
    if args.decode_units:  # a smaller memory (profiling captures)
        w = w.replace(n_tokens=w.n_sink + args.decode_units * w.unit_size + w.window)
    steps = min(w.decode_steps, args.decode_steps)
    P = peaks()
    out = {}
    # memory of 1,052,800 tokens built once (untimed); both scoring pools are kept by the library
    layer = InfLLMLayer.from_workload(w, max_tokens=w.n_tokens + 3 * steps + 48, max_chunk=w.build_chunk)
    t0 = time.time()
    for c0 in range(0, w.n_tokens, w.build_chunk):
        n = min(w.build_chunk, w.n_tokens - c0)
        q, k, v = synth.gen_chunk(w, c0, n)
        layer.append_chunk(to_dev(q, torch, device), to_dev(k, torch, device), to_dev(v, torch, device))
    torch.cuda.synchronize()
    build_s = time.time() - t0
    modes = ("reps", "repsum", "meankey")
    nmodes = len(modes)
    qkv = [tuple(to_dev(a, torch, device) for a in synth.gen_chunk(w, w.n_tokens + s, 1))
           for s in range(nmodes * steps)]
    qkv_extra = [tuple(to_dev(a, torch, device) for a in synth.gen_chunk(w, w.n_tokens + nmodes * steps + s, 1))
                 for s in range(16 * nmodes)]
    o = torch.empty((1, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device=device)
    flush = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    fsum = torch.empty((), dtype=torch.float32, device=device)

    def flush_l2():  # read 256 MB (> 126 MB L2): leaves clean lines, so no write-back lands in the step
        torch.sum(flush, dim=0, out=fsum)
    for mi, mode in enumerate(modes):
        layer.set_score_mode(mode)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        n_launch0 = layer.stats()["kernel_launches"]
        with ClockSampler(local) as clk:
            for s in range(steps):
                flush_l2()  # evict the rep pool and window from L2 between steps
                a, b = evs[s]
                a.record(stream)
                layer.decode_step(*qkv[mi * steps + s], out=o)
                b.record(stream)
            torch.cuda.synchronize()
        us = np.array([a.elapsed_time(b) * 1e3 for a, b in evs])
        launches = layer.stats()["kernel_launches"] - n_launch0
        # per-kernel-class device time (events around each launch; breaks launch overlap, so the
        # sum exceeds the step time above): where a step's time goes
        layer.set_profiling(True)
        for s in range(16):  # extra tokens after both timed passes' tokens
            flush_l2()
            layer.decode_step(*qkv_extra[16 * mi + s], out=o)
        torch.cuda.synchronize()
        st_prof = layer.stats()
        layer.set_profiling(False)
        byts = np.array([decode_bytes(w, w.n_tokens + mi * steps + s, mode) for s in range(steps)])
        med = float(np.median(us))
        gbs = float(np.median(byts / (us * 1e-6) / 1e9))
        out[mode] = {"us_per_step_median": med, "us_per_step_p90": float(np.percentile(us, 90)),
                     "algorithmic_bytes_per_step": float(np.median(byts)),
                     "hbm_gbs": gbs, "hbm_frac_of_measured": gbs / P["hbm"], "hbm_frac_of_8tbs_nominal": gbs / 8000.0,
                     "launches_per_step": launches / steps, "steps": steps, "clocks": clk.summary()}
        if st_prof["n_decode"]:
            out[mode]["profiled_us_per_step"] = {k: 1e3 * st_prof[f"ms_{k}"] / 16 for k in
                                                 ("append", "reps", "select", "decode")}
    layer.close()
    del qkv, flush
    torch.cuda.empty_cache()
    out["build_s"] = build_s
    units = (w.n_tokens - w.n_sink - w.window) // w.unit_size
    out["workload"] = (f"{w.name}: {units} units x 128 + 128 sinks + 4096 window = {w.n_tokens} tokens built, then "
                       f"{steps} single-token steps per scoring mode (tokens continue across modes); L2 flushed "
                       f"(256 MB read) before each timed step")
    return out


# ------------------------------------------------------------------------------------------------
# CPU oracle


def oracle_sample(workload):
    """A bounded sample of the workload through the fp64 oracle.  128K-token streams: one steady chunk
    (chunk 64) recomputed statelessly -- representatives of every eligible unit, unit lookup, attention
    for the chunk's tokens; the needle stream: its final chunk (the one that must find the needle); the
    tiny fp32 stream: the whole stream, chunk by chunk (streaming oracle)."""
    from oracle import infllm_oracle as O
    from tests._source import Source
    w = synth.WORKLOADS[workload]
    src = Source(w)
    chunks = synth.chunk_bounds(w)
    if len(chunks) <= 64:
        t = time.time()
        layer = O.OracleLayer(w.as_config(), rep_method="linear")
        for c0, n in chunks:
            layer.append_chunk(src.q(c0, n), src.k(c0, n), src.v(c0, n))
            layer.attend_chunk()
        return w.n_tokens, time.time() - t, f"the whole {w.name} stream ({len(chunks)} chunks), streaming oracle"
    ci = len(chunks) - 1 if w.needle else 64
    c0, n = chunks[ci]
    t = time.time()
    O.chunk_stateless(src.q, src.k, src.v, c0, n, w.as_config())
    return n, time.time() - t, f"chunk {ci} (tokens [{c0}, {c0 + n})) of {w.name}, stateless recomputation"


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count()


def cpu_baseline(workload):
    n, s, what = oracle_sample(workload)
    return {"value": n / s, "unit": "tok/s", "cores": cpu_threads(), "kind": "oracle", "sample": what,
            "seconds": s}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    times = []
    for i in range(args.warmup + max(1, args.steps)):
        n, s, what = oracle_sample(args.workload)
        if i >= args.warmup:
            times.append(s)
    tot = sum(times)
    w = synth.WORKLOADS[args.workload]
    v = n * len(times) / tot
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "tok/s", "n_gpus": 1, "steps": len(times),
            "warmup": args.warmup, "ms_per_step": tot / len(times) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded Philox normals)",
            "config": workload_config(w, 1),
            "cpu_baseline": {"value": v, "unit": "tok/s", "cores": cpu_threads(), "kind": "oracle", "sample": what},
            "e2e": {"value": v, "unit": "tok/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="mistral_128k", choices=["mistral_128k", "llama3_128k", "needle_256k",
                                                                    "tiny_f32"])
    ap.add_argument("--decode-steps", type=int, default=256)
    ap.add_argument("--decode-units", type=int, default=0, help="memory units of the decode workload (0: 8192)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-group", type=int, default=32,
                    help="chunks per host<->device copy group of the e2e arm (32 measured best of 4-64)")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-others", action="store_true", help="skip the other prefill workloads")
    ap.add_argument("--parallel", choices=["replicas", "kv"], default="replicas",
                    help="N > 1: independent replicas (default, weak scaling) or one prompt's KV heads split over "
                         "the ranks (strong scaling)")
    ap.add_argument("--tokens", type=int, default=0, help="truncate the prefill stream (small profiling cases)")
    ap.add_argument("--only", choices=["prefill", "decode"], default=None,
                    help="run only one part (profiling); the JSON line then carries that part alone")
    args = ap.parse_args()
    assert args.warmup >= 3 or args.impl == "reference", "at least 3 warm-up steps"
    rank, world, _ = dist_env()
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    dist_init("nccl")
    if args.only == "decode":
        import torch
        _, _, local = dist_env()
        torch.cuda.set_device(local)
        res = {"impl": "ours", "decode": run_decode(args, torch, torch.device("cuda", local),
                                                    torch.cuda.current_stream(), local)}
    else:
        res = run_ours(args, rank, world)
    if rank == 0:
        print(json.dumps(res), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
