"""Parity at the full sizes of the four large workloads.

Prefill workloads run twice through the C ABI: once through infllm_prefill, the whole prompt in
one call -- the entry point and launch configuration the benchmark times (one-chunk lookahead,
three query slots, two selection buffers) -- and once through append_chunk + attend_chunk per
chunk.  The two outputs must be equal bit for bit over the whole stream, as must the final
selection, unit scores and representatives.  The per-chunk run records the selection and unit
scores of sampled chunks, and the fp64 oracle recomputes those chunks statelessly from the full
prefix with its OWN representatives and selection.  Decode runs through infllm_decode_step, one
call per token, as the benchmark times it.

Indices must be bit-exact wherever the oracle's fp64 score gap exceeds 1e-3 relative; where a
near-tie makes several choices correct, the GPU's choice must be a valid one inside the band
and the outputs are checked on the GPU's selection.  Outputs within 2e-2 max-abs (bf16).
"""
from __future__ import annotations

import numpy as np
import pytest

import synth
from oracle import infllm_oracle as O
from tests._parity import TOL, compare_reps, compare_selection, make_layer, to_np64, to_torch
from tests._source import Source

pytestmark = pytest.mark.gpu


def _check_chunk(w, src, cfg, oreps, rep_keys, c0, n, g_out, g_sel, g_scores, g_reps):
    """Oracle chain on one chunk against the GPU's results for it."""
    nm = O.n_mem(c0, w.n_sink, w.window, w.unit_size)
    ref, info = O.chunk_stateless(src.q, src.k, src.v, c0, n, cfg, reps=oreps[:nm], rep_keys=rep_keys)
    tol = TOL[w.dtype]
    n_dec, bad = compare_selection(g_sel, info["sigma"], w.top_k)
    # unit scores: where the GPU chose the same representatives, the scores must agree
    if cfg.get("unit_repr") == "meankey":  # mean keys do not depend on the representatives
        same = np.ones((w.n_kv_heads, nm), dtype=bool)
    else:
        same = np.array([[sorted(oreps[j][h]) == sorted(int(x) for x in g_reps[h, j]) for j in range(nm)]
                         for h in range(w.n_kv_heads)])
    for h in range(w.n_kv_heads):
        scale = max(1e-6, float(np.max(np.abs(info["sigma"][h]))))
        diff = np.abs(g_scores[h][:nm] - info["sigma"][h])[same[h]]
        assert diff.size == 0 or float(diff.max()) <= 2e-5 * scale + 1e-5
    own = [sorted(s) for s in info["sel"]]
    gpu = [sorted(int(x) for x in r if x >= 0) for r in g_sel]
    if own != gpu:  # a near-tie: outputs on the GPU's (valid) selection
        ref, _ = O.chunk_stateless(src.q, src.k, src.v, c0, n, cfg, reps=oreps[:nm], rep_keys=rep_keys,
                                   sel_override=gpu)
    err = float(np.max(np.abs(g_out - ref)))
    assert err <= tol, (c0, err)
    return info, n_dec


def _prefill_both_paths(w, sample):
    """The whole stream through infllm_prefill and through per-chunk calls (bit-equal outputs and
    final state).  Returns (per-chunk layer, prefill output as float64 numpy, {chunk: record})."""
    import torch
    q, k, v = synth.gen_chunk(w, 0, w.n_tokens)
    qd, kd, vd = to_torch(q), to_torch(k), to_torch(v)
    del q, k, v
    glayer = make_layer(w)
    outs = torch.empty_like(qd)
    rec = {}
    for ci, (c0, n) in enumerate(synth.chunk_bounds(w)):
        glayer.append_chunk(qd[c0:c0 + n], kd[c0:c0 + n], vd[c0:c0 + n])
        glayer.attend_chunk(qd[c0:c0 + n], out=outs[c0:c0 + n])
        if ci in sample:
            torch.cuda.synchronize()
            rec[ci] = dict(c0=c0, n=n, sel=glayer.selection().copy(), scores=glayer.unit_scores().copy())
    player = make_layer(w)
    outp = player.prefill(qd, kd, vd, w.chunk)
    torch.cuda.synchronize()
    assert torch.equal(outp, outs), "infllm_prefill differs from the per-chunk calls"
    assert player.selection().tolist() == glayer.selection().tolist()
    assert np.array_equal(player.unit_scores(), glayer.unit_scores())
    nu = glayer.stats()["units_with_reps"]
    assert player.stats()["units_with_reps"] == nu
    assert np.array_equal(player.reps(0, nu), glayer.reps(0, nu))
    player.close()
    for ci, r in rec.items():
        r["out"] = to_np64(outp[r["c0"]:r["c0"] + r["n"]])
    del outs, outp, qd, kd, vd
    torch.cuda.empty_cache()
    return glayer, rec


@pytest.mark.parametrize("name", ["mistral_128k", "llama3_128k"])
def test_prefill_stream_fullsize(cuda_ok, name):
    w = synth.WORKLOADS[name]
    cfg, src = w.as_config(), Source(w)
    chunks = synth.chunk_bounds(w)
    sample = {64, 160, len(chunks) - 1}
    glayer, res = _prefill_both_paths(w, sample)
    last_c0 = chunks[-1][0]
    nu = O.n_mem(last_c0, w.n_sink, w.window, w.unit_size)
    g_reps = glayer.reps(0, nu)
    oreps, rho = O.all_reps_linear(src.q, src.k, last_c0, cfg)
    dec, tot, bad_dec, _ = compare_reps(g_reps, rho, w.n_reps)
    assert bad_dec == 0 and dec >= 0.5 * tot
    rep_keys = O.rep_key_table(src.k, oreps, nu, cfg)
    for ci in sorted(sample):
        g = res[ci]
        _check_chunk(w, src, cfg, oreps, rep_keys, g["c0"], g["n"], g["out"], g["sel"], g["scores"], g_reps)
    glayer.close()


def test_needle_256k_fullsize(cuda_ok):
    w = synth.WORKLOADS["needle_256k"]
    cfg, src = w.as_config(), Source(w)
    chunks = synth.chunk_bounds(w)
    last = len(chunks) - 1
    j_star = synth.needle_info(w)[0]
    glayer, res = _prefill_both_paths(w, {last})
    g = res[last]
    nu = O.n_mem(g["c0"], w.n_sink, w.window, w.unit_size)
    g_reps = glayer.reps(0, nu)
    oreps, rho = O.all_reps_linear(src.q, src.k, g["c0"], cfg)
    assert compare_reps(g_reps, rho, w.n_reps)[2] == 0
    rep_keys = O.rep_key_table(src.k, oreps, nu, cfg)
    info, _ = _check_chunk(w, src, cfg, oreps, rep_keys, g["c0"], g["n"], g["out"], g["sel"], g["scores"], g_reps)
    for h in range(w.n_kv_heads):  # the planted unit is found, by the GPU and by the oracle
        assert j_star in g["sel"][h].tolist() and j_star in info["sel"][h]
        assert int(np.argmax(g["scores"][h])) == j_star
    glayer.close()


def test_decode_1m_fullsize(cuda_ok):
    import torch
    w = synth.WORKLOADS["decode_1m"]
    cfg, src = w.as_config(), Source(w)
    layer = make_layer(w, max_tokens=w.total_tokens + 2)
    for c0 in range(0, w.n_tokens, w.build_chunk):
        n = min(w.build_chunk, w.n_tokens - c0)
        q, k, v = synth.gen_chunk(w, c0, n)
        layer.append_chunk(to_torch(q), to_torch(k), to_torch(v))
    sample = {0, 127, 128, w.decode_steps - 1}  # a unit is evicted at step 128
    rec = {}
    for s in range(w.decode_steps):
        t = w.n_tokens + s
        q, k, v = synth.gen_chunk(w, t, 1)
        out = layer.decode_step(to_torch(q), to_torch(k), to_torch(v))
        if s in sample:
            torch.cuda.synchronize()
            rec[s] = dict(out=to_np64(out), sel=layer.selection().copy(), scores=layer.unit_scores().copy())
    t_last = w.n_tokens + w.decode_steps - 1
    nu = O.n_mem(t_last, w.n_sink, w.window, w.unit_size)
    assert nu == 8193
    g_reps = layer.reps(0, nu)
    oreps, rho = O.all_reps_linear(src.q, src.k, t_last, cfg)
    dec, tot, bad_dec, _ = compare_reps(g_reps, rho, w.n_reps)
    assert bad_dec == 0 and dec >= 0.5 * tot
    rep_keys = O.rep_key_table(src.k, oreps, nu, cfg)
    for s in sorted(sample):
        t = w.n_tokens + s
        nm = O.n_mem(t, w.n_sink, w.window, w.unit_size)
        _check_chunk(w, src, cfg, oreps, rep_keys[:, :nm], t, 1, rec[s]["out"], rec[s]["sel"], rec[s]["scores"],
                     g_reps)
    # two more steps scoring units by their mean keys, against the oracle's mean-key table
    layer.set_score_mode("meankey")
    mcfg = dict(cfg, unit_repr="meankey")
    nu2 = O.n_mem(w.n_tokens + w.decode_steps + 1, w.n_sink, w.window, w.unit_size)  # a unit is evicted at step 256
    means = O.mean_key_table(src.k, nu2, mcfg)[:, :, None, :]
    for s in range(w.decode_steps, w.decode_steps + 2):
        t = w.n_tokens + s
        q, k, v = synth.gen_chunk(w, t, 1)
        out = layer.decode_step(to_torch(q), to_torch(k), to_torch(v))
        torch.cuda.synchronize()
        _check_chunk(w, src, mcfg, oreps, means, t, 1, to_np64(out), layer.selection().copy(),
                     layer.unit_scores().copy(), g_reps)
    layer.close()
