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
        self.proc = None
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if len(r) > 5 + i and r[5 + i] == "Active"})
        load = [s for s in sm if s > 0.5 * (max(sm) if sm else 1)]
        return {"sm_mhz": float(np.median(load)) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


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
    score = nm * Hkv * (w.n_reps * d * elt if score_mode == "reps" else d * 4)
    return score + keys * Hkv * d * elt * 2


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


def attn_device_hash():
    """sha256 of the attention kernel's device code: attend_tc.cu up to its host-side part (the
    tensor-map encoding and the launcher), which does not change what the kernel moves."""
    import hashlib
    src = open(ATTN_SOURCE, "rb").read()
    cut = src.find(b"typedef CUresult (*EncodeTiledFn)")
    return hashlib.sha256(src if cut < 0 else src[:cut]).hexdigest()


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


def workload_config(w, world):
    """The `config` object of the JSON line (the same for both arms)."""
    return {"workload": f"{w.name}: {w.n_q_heads}q/{w.n_kv_heads}kv heads, d={w.head_dim}, "
                        f"{w.n_tokens} tokens in {w.chunk}-token chunks, W={w.window}, S={w.n_sink}, "
                        f"U={w.unit_size}, r={w.n_reps}, k={w.top_k}, base={w.rope_base:g}",
            "global_batch": 1 * world, "seq_len": w.n_tokens, "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2 (1.6 GB of Q/K/V per step)"}


def run_ours(args, rank, world):
    import torch
    from block_memory_sparse_b200 import InfLLMLayer

    _, _, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    w = synth.WORKLOADS[args.workload]
    if args.tokens:
        w = w.replace(n_tokens=min(args.tokens, w.n_tokens))
    P = peaks()
    chunks = synth.chunk_bounds(w)
    q_h, k_h, v_h = gen_full(w, torch, device)
    Q, K, V = (to_dev(a, torch, device) for a in (q_h, k_h, v_h))
    OUT = torch.empty_like(Q)
    stream = torch.cuda.current_stream(device)
    layer = InfLLMLayer.from_workload(w, max_tokens=w.n_tokens, max_chunk=w.chunk)

    def one_step():  # the whole prompt, chunk by chunk, in one call of the public API
        layer.reset()
        layer.prefill(Q, K, V, w.chunk, out=OUT)

    for _ in range(args.warmup):
        one_step()
    torch.cuda.synchronize()
    layer.set_profiling(False)  # no events in the timed steps: they would break launch chaining
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(args.steps):
            one_step()
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = e0.elapsed_time(e1)
    ms = max_over_ranks(ms, device)
    launches = layer.stats()["kernel_launches"]
    # the attention kernel's own duration: the same steps again with CUDA events around each
    # attention launch on the layer's stream (outside the timed region: events serialise it)
    layer.set_profiling(["attend"])
    for _ in range(args.steps):
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
    tokens_all = w.n_tokens * args.steps * world
    value = tokens_all / (ms / 1e3)

    # dominant kernel: the attention kernel (tensor-bound on the tcgen05 path)
    flops = sum(chunk_flops(w, c0, n) for c0, n in chunks) * args.steps
    att_ms = st["ms_attend"]
    n_att = st["n_attend"]
    achieved_tf = flops / (att_ms / 1e3) / 1e12 if att_ms > 0 else None
    tc = st["attend_path"] == 1
    if tc:
        peak = P["bf16_sust"]
        roof = {"bound": "tensor", "achieved": achieved_tf, "peak": peak, "unit": "TFLOP/s",
                "frac": (achieved_tf / peak) if achieved_tf else None, "traffic": attn_traffic(),
                "kernel": "attention (tcgen05)", "peak_source": f"{P['src']} bf16 sustained",
                "traffic_source": "ncu dram__bytes_read.sum + dram__bytes_write.sum of one steady-chunk launch "
                                  "(profiles/k_attn_tc_mistral_128k.md); null if the kernel changed since"}
    else:
        # CUDA-core fp32 FMA path: 148 SMs x 128 FP32 lanes x 2 flop x max SM clock
        peak = 148 * 128 * 2 * P["sm_max"] * 1e6 / 1e12
        roof = {"bound": "alu", "achieved": achieved_tf, "peak": peak, "unit": "TFLOP/s",
                "frac": (achieved_tf / peak) if achieved_tf else None, "traffic": None,
                "kernel": "attention (SIMT fp32)", "peak_source": "148 SMs x 128 FP32 x 2 x max clock"}
    roof["avg_launch_ms"] = att_ms / n_att if n_att else None
    roof["launches"] = n_att
    roof["timing"] = "CUDA events around each attention launch, over a repeat of the timed steps"
    res = {"metric": METRIC, "value": value, "unit": "tok/s", "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded Philox normals, K channel bias N(0,4))",
           "config": workload_config(w, world),
           "roofline": roof, "gpu_launches": launches,
           "clocks": clk.summary(),
           "time_split_ms_per_step": {k: split[f"ms_{k}"]
                                      for k in ("append", "reps", "prep", "select", "attend")}}

    if not args.no_e2e:
        res["e2e"] = run_e2e(args, w, layer, q_h, k_h, v_h, torch, device, stream, world)
    if not args.no_decode:
        del Q, K, V, OUT
        layer.close()
        torch.cuda.empty_cache()
        res["decode"] = run_decode(args, torch, device, stream, local)
    else:
        layer.close()
    if rank == 0 and not args.no_cpu:
        res["cpu_baseline"] = cpu_baseline(args.workload)
    return res


def run_e2e(args, w, layer, q_h, k_h, v_h, torch, device, stream, world, group_chunks=8):
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
    layer = InfLLMLayer.from_workload(w, max_tokens=w.n_tokens + 2 * steps + 32, max_chunk=w.build_chunk)
    t0 = time.time()
    for c0 in range(0, w.n_tokens, w.build_chunk):
        n = min(w.build_chunk, w.n_tokens - c0)
        q, k, v = synth.gen_chunk(w, c0, n)
        layer.append_chunk(to_dev(q, torch, device), to_dev(k, torch, device), to_dev(v, torch, device))
    torch.cuda.synchronize()
    build_s = time.time() - t0
    qkv = [tuple(to_dev(a, torch, device) for a in synth.gen_chunk(w, w.n_tokens + s, 1)) for s in range(2 * steps)]
    qkv_extra = [tuple(to_dev(a, torch, device) for a in synth.gen_chunk(w, w.n_tokens + 2 * steps + s, 1))
                 for s in range(32)]
    o = torch.empty((1, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device=device)
    flush = torch.ones(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    fsum = torch.empty((), dtype=torch.float32, device=device)

    def flush_l2():  # read 256 MB (> 126 MB L2): leaves clean lines, so no write-back lands in the step
        torch.sum(flush, dim=0, out=fsum)
    for mi, mode in enumerate(("reps", "repsum")):
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
    """One steady chunk of the workload recomputed statelessly by the fp64 oracle: representatives
    of every eligible unit, unit lookup, attention for the chunk's tokens."""
    from oracle import infllm_oracle as O
    from tests._source import Source
    w = synth.WORKLOADS[workload]
    c0, n = synth.chunk_bounds(w)[64]
    src = Source(w)
    t = time.time()
    O.chunk_stateless(src.q, src.k, src.v, c0, n, w.as_config())
    return n, time.time() - t, f"chunk 64 (tokens [{c0}, {c0 + n})) of {w.name}, stateless recomputation"


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
    ap.add_argument("--workload", default="mistral_128k", choices=["mistral_128k", "llama3_128k", "needle_256k"])
    ap.add_argument("--decode-steps", type=int, default=256)
    ap.add_argument("--decode-units", type=int, default=0, help="memory units of the decode workload (0: 8192)")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
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
