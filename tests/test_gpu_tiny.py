"""The tiny fp32 workload end to end on the GPU: one q head and one KV head, d = 64, 4096
tokens streamed in 128-token chunks, RoPE base 1e4, units of 128 with 4 representatives,
top-k 4, window 512, 16 sinks, seed 0 ("InfLLM Guide: Training-Free Long-Context Memory
Units", "Core Innovation 1: Structured Context Partitioning" for the partition; "Core
Innovation 2", item 2 for the top-k lookup).

Every one of the 32 chunks is compared with the streaming fp64 oracle, whose representatives
come from the plain double loop: outputs within 1e-4 max-abs (fp32), representatives and unit
selections bit-exact where the oracle's gap is decisive and otherwise a valid choice inside the
near-tie band.  The whole-prompt entry point (the path the benchmark times) must equal the
per-chunk calls bit for bit.  A decode leg of 64 single-token steps follows the prompt and is
checked against the oracle the same way.
"""
from __future__ import annotations

import numpy as np
import pytest

import synth
from oracle import infllm_oracle as O
from tests._parity import TOL, compare_reps, compare_selection, make_layer, to_np64, to_torch
from tests._source import Source

pytestmark = pytest.mark.gpu

DECODE_STEPS = 64


def _oracle_on_gpu_state(olayer, glayer, w, gsel):
    """Oracle attention for the chunk just appended, with the GPU's representatives for the unit
    scores and the GPU's selection for the attention (equal to the oracle's where decisive)."""
    nm = O.n_mem(olayer._chunk[0], w.n_sink, w.window, w.unit_size)
    saved = olayer.reps
    if nm > 0:
        greps = glayer.reps(0, nm)
        olayer.reps = [[list(greps[h, j]) for h in range(w.n_kv_heads)] for j in range(nm)]
    ref = olayer.attend_chunk(sel_override=[[int(x) for x in gsel[h] if x >= 0] for h in range(w.n_kv_heads)])
    sig = olayer.last["sigma"]
    olayer.reps = saved
    return ref, sig, nm


def test_tiny_f32_stream_and_decode(cuda_ok):
    import torch
    w = synth.WORKLOADS["tiny_f32"]
    assert (w.n_q_heads, w.n_kv_heads, w.head_dim, w.chunk, w.n_tokens, w.seed) == (1, 1, 64, 128, 4096, 0)
    T = w.n_tokens
    total = T + DECODE_STEPS
    q, k, v = synth.gen_chunk(w, 0, total)
    qd, kd, vd = to_torch(q), to_torch(k), to_torch(v)
    src = Source(w)
    q64, k64, v64 = src.q(0, total), src.k(0, total), src.v(0, total)
    tol = TOL[w.dtype]
    assert tol == 1e-4

    glayer = make_layer(w, max_tokens=total)
    olayer = O.OracleLayer(w.as_config(), rep_method="plain")
    chunks = synth.chunk_bounds(w)
    assert len(chunks) == 32
    outs = torch.empty_like(qd[:T])
    n_dec = n_sel = 0
    for ci, (c0, n) in enumerate(chunks):
        glayer.append_chunk(qd[c0:c0 + n], kd[c0:c0 + n], vd[c0:c0 + n])
        glayer.attend_chunk(qd[c0:c0 + n], out=outs[c0:c0 + n])
        torch.cuda.synchronize()
        st = glayer.stats()
        assert st["attend_path"] == 0  # fp32 runs on the CUDA cores
        gsel = glayer.selection()
        olayer.append_chunk(q64[c0:c0 + n], k64[c0:c0 + n], v64[c0:c0 + n])
        ref, sig, nm = _oracle_on_gpu_state(olayer, glayer, w, gsel)
        assert st["n_mem"] == nm
        if nm > 0:
            gs = glayer.unit_scores()
            scale = max(1e-6, float(np.max(np.abs(sig[0]))))
            assert np.max(np.abs(gs[0][:nm] - sig[0])) <= 2e-5 * scale + 1e-5
            d, _ = compare_selection(gsel, sig, w.top_k)
            n_dec += d
            n_sel += 1
        err = float(np.max(np.abs(to_np64(outs[c0:c0 + n]) - ref)))
        assert err <= tol, (ci, err)
    assert O.n_mem(chunks[-1][0], w.n_sink, w.window, w.unit_size) == 26
    # representatives of every evicted unit against the oracle's plain double loop
    nu = len(olayer.reps)
    dec, tot, bad_dec, _ = compare_reps(glayer.reps(0, nu), np.stack(olayer.rep_scores), w.n_reps)
    assert bad_dec == 0 and dec >= 0.5 * tot
    assert n_sel > 0 and n_dec >= 0.5 * n_sel

    # the whole-prompt entry point equals the per-chunk calls
    player = make_layer(w, max_tokens=total)
    outp = player.prefill(qd[:T], kd[:T], vd[:T], w.chunk)
    torch.cuda.synchronize()
    assert torch.equal(outp, outs)
    assert player.selection().tolist() == glayer.selection().tolist()
    assert np.array_equal(player.reps(0, nu), glayer.reps(0, nu))

    # decode leg: one token at a time after the prompt, on both contexts
    for s in range(DECODE_STEPS):
        t = T + s
        o = glayer.decode_step(qd[t:t + 1], kd[t:t + 1], vd[t:t + 1])
        op = player.decode_step(qd[t:t + 1], kd[t:t + 1], vd[t:t + 1])
        torch.cuda.synchronize()
        assert torch.equal(o, op)
        gsel = glayer.selection()
        olayer.append_chunk(q64[t:t + 1], k64[t:t + 1], v64[t:t + 1])
        ref, sig, nm = _oracle_on_gpu_state(olayer, glayer, w, gsel)
        compare_selection(gsel, sig, w.top_k)
        err = float(np.max(np.abs(to_np64(o) - ref)))
        assert err <= tol, (s, err)
    glayer.close()
    player.close()
