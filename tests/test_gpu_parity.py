"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Bar: representative and unit indices bit-exact wherever the oracle's fp64 score gap at the
cut exceeds 1e-3 relative (elsewhere a valid choice inside the near-tie band); outputs
within 2e-2 max-abs (bf16) or 1e-4 (fp32) of the oracle evaluated on the GPU's selection.
"""
from __future__ import annotations

import numpy as np
import pytest

import synth
from oracle import infllm_oracle as O
from tests._parity import (TOL, compare_reps, compare_selection, make_layer, oracle_chunk_on_gpu_state, run_prefill,
                           to_np64, to_torch)
from tests._source import Source

pytestmark = pytest.mark.gpu

SMALL_PREFILL = ["small_gqa", "small_g4", "small_d64", "small_u256", "small_nosink", "small_streaming",
                 "small_allunits", "small_f32", "small_needle", "small_g8",
                 "small_g2"]


def _stream_oracle(w, score_mode="reps"):
    src = Source(w)
    T = w.n_tokens
    layer = O.OracleLayer(_oracle_cfg(w, score_mode), rep_method="linear")
    q, k, v = src.q(0, T), src.k(0, T), src.v(0, T)
    return layer, q, k, v


# every shape with the representative keys; the fp32 sum of them (REPSUM) and the units' mean keys
# (MEANKEY) on four shapes each
PREFILL_CASES = ([(n, "reps") for n in SMALL_PREFILL] +
                 [(n, "repsum") for n in ("small_gqa", "small_g4", "small_f32", "small_g8")] +
                 [(n, "meankey") for n in ("small_gqa", "small_g4", "small_f32", "small_d64")])


def _oracle_cfg(w, score_mode):
    cfg = w.as_config()
    if score_mode == "meankey":
        cfg["unit_repr"] = "meankey"
    return cfg


@pytest.mark.parametrize("name,score_mode", PREFILL_CASES)
def test_prefill_stream_matches_oracle(cuda_ok, name, score_mode):
    w = synth.SMALL[name]
    glayer, res = run_prefill(w, score_mode=score_mode)
    olayer, q, k, v = _stream_oracle(w, score_mode)
    tol = TOL[w.dtype]
    worst = 0.0
    n_dec = n_sel = 0
    for ci, (c0, n) in enumerate(synth.chunk_bounds(w)):
        olayer.append_chunk(q[c0:c0 + n], k[c0:c0 + n], v[c0:c0 + n])
        g = res[ci]
        nm = O.n_mem(c0, w.n_sink, w.window, w.unit_size)
        assert g["stats"]["n_mem"] == nm
        # bf16 runs on the tcgen05 kernel (d = 64 and 128); fp32 on the CUDA-core kernel
        assert g["stats"]["attend_path"] == (1 if w.dtype == "bf16" else 0)
        # unit scores: oracle on the GPU's representatives
        if nm > 0 and w.top_k > 0:
            greps = glayer.reps(0, nm) if nm else None
            saved = olayer.reps
            olayer.reps = [[list(greps[h, j]) for h in range(w.n_kv_heads)] for j in range(nm)]
            ref = olayer.attend_chunk(sel_override=[[int(x) for x in g["sel"][h] if x >= 0]
                                                    for h in range(w.n_kv_heads)])
            sig = olayer.last["sigma"]
            olayer.reps = saved
            for h in range(w.n_kv_heads):
                scale = max(1e-6, float(np.max(np.abs(sig[h]))))
                assert np.max(np.abs(g["scores"][h][:nm] - sig[h])) <= 2e-5 * scale + 1e-5
            d, bad = compare_selection(g["sel"], sig, w.top_k)
            n_dec += d
            n_sel += w.n_kv_heads
        else:
            ref = olayer.attend_chunk()
        err = float(np.max(np.abs(g["out"] - ref)))
        worst = max(worst, err)
        assert err <= tol, (ci, err)
    # representatives of every evicted unit against the oracle's plain double loop
    nu = len(olayer.reps)
    if nu:
        greps = glayer.reps(0, nu)
        rho = np.stack(olayer.rep_scores)
        dec, tot, bad_dec, bad_all = compare_reps(greps, rho, w.n_reps)
        assert bad_dec == 0
        assert dec >= 0.5 * tot  # near-ties are rare; the bar is exactness where decisive
    glayer.close()


def test_chunked_equals_stateless_on_gpu_reps(cuda_ok):
    """Streaming GPU results at sampled chunks equal the stateless oracle recomputation."""
    w = synth.SMALL["small_g4"]
    src = Source(w)
    glayer, res = run_prefill(w, record={5, 10, 17})
    for ci, g in res.items():
        nm = O.n_mem(g["c0"], w.n_sink, w.window, w.unit_size)
        greps = glayer.reps(0, nm)
        ref, info = oracle_chunk_on_gpu_state(w, src, g["c0"], g["n"], greps, g["sel"])
        compare_selection(g["sel"], info["sigma"], w.top_k)
        assert np.max(np.abs(g["out"] - ref)) <= TOL[w.dtype]
        # full oracle chain (own representatives, own selection) agrees where decisive
        own, oinfo = O.chunk_stateless(src.q, src.k, src.v, g["c0"], g["n"], w.as_config())
        if all(O.decisive(s, min(w.top_k, len(s))) for s in oinfo["sigma"]):
            assert [sorted(s) for s in oinfo["sel"]] == [sorted(int(x) for x in r if x >= 0) for r in g["sel"]]
            assert np.max(np.abs(g["out"] - own)) <= TOL[w.dtype]
    glayer.close()


@pytest.mark.parametrize("name,score_mode", [("small_decode", "reps"), ("small_decode_g8", "reps"),
                                             ("small_decode", "meankey"), ("small_decode", "repsum")])
def test_decode_matches_oracle(cuda_ok, name, score_mode):
    import torch
    w = synth.SMALL[name]
    glayer = make_layer(w, score_mode=score_mode)
    src = Source(w)
    olayer = O.OracleLayer(_oracle_cfg(w, score_mode), rep_method="linear")
    T0 = w.n_tokens
    for c0 in range(0, T0, w.build_chunk):
        n = min(w.build_chunk, T0 - c0)
        q, k, v = synth.gen_chunk(w, c0, n)
        glayer.append_chunk(to_torch(q), to_torch(k), to_torch(v))
        olayer.append_chunk(src.q(c0, n), src.k(c0, n), src.v(c0, n))
    tol = TOL[w.dtype]
    for s in range(w.decode_steps):
        t = T0 + s
        q, k, v = synth.gen_chunk(w, t, 1)
        out = glayer.decode_step(to_torch(q), to_torch(k), to_torch(v))
        olayer.append_chunk(src.q(t, 1), src.k(t, 1), src.v(t, 1))
        gsel = glayer.selection()
        nm = O.n_mem(t, w.n_sink, w.window, w.unit_size)
        greps = glayer.reps(0, nm)
        saved = olayer.reps
        olayer.reps = [[list(greps[h, j]) for h in range(w.n_kv_heads)] for j in range(nm)]
        ref = olayer.attend_chunk(sel_override=[[int(x) for x in gsel[h] if x >= 0] for h in range(w.n_kv_heads)])
        compare_selection(gsel, olayer.last["sigma"], w.top_k)
        olayer.reps = saved
        torch.cuda.synchronize()
        err = float(np.max(np.abs(to_np64(out) - ref)))
        assert err <= tol, (s, err)
    glayer.close()


def test_lookup_while_decoding_only(cuda_ok):
    """Ablation of lookup during pre-filling (research-map summary, "Measured effects"): chunks attend
    to sinks + window only, the representatives are still built, decode steps look up as usual."""
    import torch
    w = synth.SMALL["small_decode"]
    cfg = w.as_config()
    glayer = make_layer(w)
    glayer.set_prefill_lookup(False)
    src = Source(w)
    olayer = O.OracleLayer(dict(cfg, top_k=0), rep_method="linear")  # representatives do not depend on k
    tol = TOL[w.dtype]
    T0 = w.n_tokens
    for c0 in range(0, T0, w.build_chunk):
        n = min(w.build_chunk, T0 - c0)
        q, k, v = (to_torch(x) for x in synth.gen_chunk(w, c0, n))
        glayer.append_chunk(q, k, v)
        out = glayer.attend_chunk(q)
        olayer.append_chunk(src.q(c0, n), src.k(c0, n), src.v(c0, n))
        ref = olayer.attend_chunk()
        torch.cuda.synchronize()
        assert float(np.max(np.abs(to_np64(out) - ref))) <= tol, c0
        assert glayer.stats()["n_selected"] == 0 and bool((glayer.selection() < 0).all())
    assert glayer.stats()["units_with_reps"] == O.n_mem(T0 - n, w.n_sink, w.window, w.unit_size)
    olayer.cfg = dict(cfg)  # decoding looks up with the configured k
    for s in range(6):
        t = T0 + s
        q, k, v = synth.gen_chunk(w, t, 1)
        out = glayer.decode_step(to_torch(q), to_torch(k), to_torch(v))
        olayer.append_chunk(src.q(t, 1), src.k(t, 1), src.v(t, 1))
        gsel = glayer.selection()
        nm = O.n_mem(t, w.n_sink, w.window, w.unit_size)
        assert glayer.stats()["n_selected"] == min(w.top_k, nm) > 0
        greps = glayer.reps(0, nm)
        saved = olayer.reps
        olayer.reps = [[list(greps[h, j]) for h in range(w.n_kv_heads)] for j in range(nm)]
        ref = olayer.attend_chunk(sel_override=[[int(x) for x in gsel[h] if x >= 0] for h in range(w.n_kv_heads)])
        compare_selection(gsel, olayer.last["sigma"], w.top_k)
        olayer.reps = saved
        torch.cuda.synchronize()
        assert float(np.max(np.abs(to_np64(out) - ref))) <= tol, s
    # the whole-prompt entry point obeys the switch too
    layer2 = make_layer(w)
    layer2.set_prefill_lookup(False)
    q, k, v = (to_torch(x) for x in synth.gen_chunk(w, 0, T0))
    o2 = layer2.prefill(q, k, v, w.build_chunk)
    torch.cuda.synchronize()
    olayer2 = O.OracleLayer(dict(cfg, top_k=0), rep_method="linear")
    for c0 in range(0, T0, w.build_chunk):
        n = min(w.build_chunk, T0 - c0)
        olayer2.append_chunk(src.q(c0, n), src.k(c0, n), src.v(c0, n))
        ref = olayer2.attend_chunk()
        assert float(np.max(np.abs(to_np64(o2[c0:c0 + n]) - ref))) <= tol, c0
    glayer.close()
    layer2.close()


def test_needle_selected_on_gpu(cuda_ok):
    w = synth.SMALL["small_needle"]
    j_star = synth.needle_info(w)[0]
    last = len(synth.chunk_bounds(w)) - 1
    glayer, res = run_prefill(w, record={last})
    sel = res[last]["sel"]
    for h in range(w.n_kv_heads):
        assert j_star in sel[h].tolist()
        assert int(np.argmax(res[last]["scores"][h])) == j_star
    glayer.close()


def test_state_errors(cuda_ok):
    import torch
    from block_memory_sparse_b200 import InfLLMError
    w = synth.SMALL["small_gqa"]
    layer = make_layer(w, max_tokens=600, max_chunk=200)
    q, k, v = (to_torch(x) for x in synth.gen_chunk(w, 0, 200))
    with pytest.raises(InfLLMError) as e:
        layer.attend_chunk(q)
    assert e.value.status == 3  # ESTATE: nothing appended
    layer.append_chunk(q, k, v)
    with pytest.raises(InfLLMError) as e:
        layer.attend_chunk(q[:100].contiguous())
    assert e.value.status == 3  # n mismatch
    layer.attend_chunk(q)
    q2, k2, v2 = (to_torch(x) for x in synth.gen_chunk(w, 0, 201))
    with pytest.raises(InfLLMError) as e:
        layer.append_chunk(q2, k2, v2)
    assert e.value.status == 1  # n > max_chunk
    layer.append_chunk(q, k, v)
    layer.append_chunk(q, k, v)
    with pytest.raises(InfLLMError) as e:
        layer.append_chunk(q, k, v)
    assert e.value.status == 2  # capacity
    st = layer.stats()
    assert st["tokens"] == 600
    layer.reset()
    assert layer.stats()["tokens"] == 0
    layer.close()


def test_bf16_runs_on_the_tensor_cores_or_is_refused(cuda_ok):
    """bf16 attention has one path, the tcgen05 kernel (head dim 64 or 128); a bf16 shape that it cannot
    take is refused at create with EINVAL rather than run elsewhere.  fp32 runs on the CUDA cores."""
    from block_memory_sparse_b200 import InfLLMError, InfLLMLayer
    for name in ("small_d64", "small_g4"):
        layer = make_layer(synth.SMALL[name], max_tokens=64)
        assert layer.stats()["attend_path"] == 1, name
        layer.close()
    base = dict(n_q_heads=12, n_kv_heads=4, head_dim=64, n_sink=4, window=64, unit_size=16, n_reps=2, top_k=2,
                max_chunk=64, max_tokens=256, rope_base=1e4)
    for bad in (dict(), dict(n_q_heads=8, top_k=5000)):  # 3 q heads per KV head; too many selected units
        with pytest.raises(InfLLMError) as e:
            InfLLMLayer(**dict(base, **bad), dtype="bf16")
        assert e.value.status == 1  # EINVAL
    layer = InfLLMLayer(**base, dtype="f32")
    assert layer.stats()["attend_path"] == 0
    layer.close()
