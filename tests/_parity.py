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

    Returns (n_decisive, n_total, mismatches on decisive cases, mismatches overall).  Where the
    oracle's cut is not decisive, a different choice must still be a valid top-r set inside the
    near-tie band (valid_near_tie)."""
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
                else:
                    assert valid_near_tie(rho[j, h], got, r), (j, h, got, want)
    return dec, tot, bad_dec, bad_all


def valid_near_tie(scores, got, k, rel=1e-3) -> bool:
    """Whether `got` is one of the correct top-k choices when the oracle's cut is a near-tie.

    The band is the decisive rule's own: rel * max(|s_(k)|, |s_(k+1)|), s sorted descending (the
    scores within it are the ones whose order fp32 and fp64 may legitimately disagree on).  A
    valid choice
      * holds min(k, n) distinct ids, each in range;
      * contains every id whose score exceeds s_(k) + band (clearly inside the top k);
      * contains no id whose score is below s_(k) - band (clearly outside it).
    """
    s = np.asarray(scores, dtype=np.float64)
    n = len(s)
    kk = min(k, n)
    got = [int(i) for i in got]
    if len(got) != kk or len(set(got)) != kk or any(i < 0 or i >= n for i in got):
        return False
    if kk == 0 or kk == n:
        return True
    srt = np.sort(s)[::-1]
    a, b = srt[kk - 1], srt[kk]
    band = rel * max(abs(a), abs(b))
    chosen = set(got)
    if any(s[i] > a + band and i not in chosen for i in range(n)):
        return False
    return all(s[i] >= a - band for i in got)


def compare_selection(gpu_sel: np.ndarray, sigma_list, k: int):
    """gpu_sel [Hkv][top_k] ascending ids (-1 pad); sigma_list[h] oracle unit scores."""
    dec = bad = 0
    for h, sig in enumerate(sigma_list):
        nm = len(sig)
        kk = min(k, nm)
        want = sorted(O.topk_stable(sig, kk))
        got = [int(x) for x in gpu_sel[h][:kk]]
        assert got == sorted(got), (h, got)  # ascending ids
        assert all(int(x) == -1 for x in gpu_sel[h][kk:])
        d = O.decisive(sig, kk)
        dec += d
        if sorted(got) != want:
            assert not d, (h, got, want)
            bad += 1
        assert valid_near_tie(sig, got, kk), (h, got, want)
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
