"""Helpers that run a workload through the CUDA library and compare with the fp64 oracle."""
from __future__ import annotations

import numpy as np

import synth
from oracle import infllm_oracle as O
from tests._source import Source

TOL = {"bf16": 2e-2, "f32": 1e-4}


def to_torch(a: np.ndarray, device="cuda"):
    import torch
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def to_np64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def make_layer(w: synth.Workload, score_mode="reps", max_tokens=None, max_chunk=None):
    from block_memory_sparse_b200 import InfLLMLayer
    return InfLLMLayer.from_workload(w, max_tokens=max_tokens, max_chunk=max_chunk, score_mode=score_mode)


def run_prefill(w: synth.Workload, layer=None, record=None, score_mode="reps", n_tokens=None):
    """Stream the workload through append_chunk + attend_chunk.

    record: set of chunk indices whose outputs/selection/scores are kept (None = all).
    Returns (layer, {chunk index: dict(c0, n, out, sel, scores, stats)}).
    """
    import torch
    if layer is None:
        layer = make_layer(w, score_mode=score_mode)
    res = {}
    for ci, (c0, n) in enumerate(synth.chunk_bounds(w)):
        if n_tokens is not None and c0 >= n_tokens:
            break
        q, k, v = synth.gen_chunk(w, c0, n)
        qd, kd, vd = to_torch(q), to_torch(k), to_torch(v)
        layer.append_chunk(qd, kd, vd)
        out = layer.attend_chunk(qd)
        if record is None or ci in record:
            torch.cuda.synchronize()
            res[ci] = dict(c0=c0, n=n, out=to_np64(out), sel=layer.selection().copy(),
                           scores=layer.unit_scores().copy(), stats=layer.stats())
    return layer, res


def compare_reps(gpu_reps: np.ndarray, rho: np.ndarray, r: int):
    """gpu_reps [Hkv][n_units][r] ascending ids; rho [n_units, Hkv, U] oracle scores.

    Returns (n_decisive, n_total, mismatches on decisive cases, mismatches overall)."""
    n_units, Hkv = rho.shape[0], rho.shape[1]
    dec = tot = bad_dec = bad_all = 0
    for j in range(n_units):
        for h in range(Hkv):
            want = sorted(O.select_reps(rho[j, h], r))
            got = sorted(int(x) for x in gpu_reps[h, j])
            d = O.decisive(rho[j, h], r)
            tot += 1
            dec += d
            if got != want:
                bad_all += 1
                if d:
                    bad_dec += 1
                else:  # must still be a valid choice inside the near-tie band
                    assert _valid_near_tie(rho[j, h], got, r), (j, h, got, want)
    return dec, tot, bad_dec, bad_all


def _valid_near_tie(scores, got, k, rel=1e-3):
    """`got` differs from the exact top-k only by swaps among scores within the near-tie band."""
    s = np.asarray(scores, dtype=np.float64)
    order = sorted(range(len(s)), key=lambda i: (-s[i], i))
    kth = s[order[k - 1]]
    band = rel * max(abs(kth), 1e-30) * 4
    for i in got:
        if s[i] < kth - band:
            return False
    return True


def compare_selection(gpu_sel: np.ndarray, sigma_list, k: int):
    """gpu_sel [Hkv][top_k] ascending ids (-1 pad); sigma_list[h] oracle unit scores."""
    dec = bad = 0
    for h, sig in enumerate(sigma_list):
        nm = len(sig)
        kk = min(k, nm)
        want = sorted(O.topk_stable(sig, kk))
        got = sorted(int(x) for x in gpu_sel[h][:kk])
        assert all(int(x) == -1 for x in gpu_sel[h][kk:])
        d = O.decisive(sig, kk)
        dec += d
        if got != want:
            assert not d, (h, got, want)
            assert _valid_near_tie(sig, got, kk), (h, got, want)
            bad += 1
    return dec, bad


def oracle_chunk_on_gpu_state(w: synth.Workload, src: Source, c0: int, n: int, gpu_reps: np.ndarray,
                              gpu_sel: np.ndarray):
    """Oracle lookup + attention for one chunk, given the GPU's representatives (for the scores)
    and the GPU's selection (for the attention).  Returns (out, info) with oracle sigma."""
    cfg = w.as_config()
    nm = O.n_mem(c0, w.n_sink, w.window, w.unit_size)
    reps = [[list(gpu_reps[h, j]) for h in range(w.n_kv_heads)] for j in range(nm)]
    sel = [[int(x) for x in gpu_sel[h] if x >= 0] for h in range(w.n_kv_heads)]
    return O.chunk_stateless(src.q, src.k, src.v, c0, n, cfg, reps=reps, sel_override=sel)
