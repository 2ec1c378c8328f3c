"""The whole-prompt entry point and launch chaining, through the C ABI on the GPU.

infllm_prefill runs the same kernels as append_chunk + attend_chunk per chunk, chained across
chunks; launch chaining only changes when a kernel may start, never what it computes.  So
every comparison here is bit-exact (the per-chunk path itself is checked against the oracle
in test_gpu_parity.py).
"""
from __future__ import annotations

import numpy as np
import pytest

import synth
from tests._parity import make_layer, to_torch

pytestmark = pytest.mark.gpu

CASES = {
    "small_g4": synth.SMALL["small_g4"],                      # tcgen05 attention, 4 q heads per kv head
    "small_gqa": synth.SMALL["small_gqa"],                    # tcgen05, ragged chunks of 200
    # one q head per kv head: 128 queries per packed tile (largest prep tile)
    "small_g1": synth.SMALL["small_g4"].replace(n_q_heads=4, n_kv_heads=4, n_tokens=3000),
    "small_f32": synth.SMALL["small_f32"],                    # CUDA-core attention, fp32
    "small_d64": synth.SMALL["small_d64"],                    # CUDA-core attention, d = 64
}


def _inputs(w, T):
    q, k, v = synth.gen_chunk(w, 0, T)
    return to_torch(q), to_torch(k), to_torch(v)


def _per_chunk(w, q, k, v, chaining=True):
    import torch
    layer = make_layer(w)
    layer.set_launch_chaining(chaining)
    outs = []
    for c0, n in synth.chunk_bounds(w):
        layer.append_chunk(q[c0:c0 + n].contiguous(), k[c0:c0 + n].contiguous(), v[c0:c0 + n].contiguous())
        outs.append(layer.attend_chunk(q[c0:c0 + n].contiguous()))
    torch.cuda.synchronize()
    return layer, torch.cat(outs)


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_equals_chunk_calls(cuda_ok, name):
    import torch
    w = CASES[name]
    q, k, v = _inputs(w, w.n_tokens)
    ref_layer, ref = _per_chunk(w, q, k, v)
    layer = make_layer(w)
    out = layer.prefill(q, k, v, w.chunk)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert layer.selection().tolist() == ref_layer.selection().tolist()
    assert np.array_equal(layer.unit_scores(), ref_layer.unit_scores())
    s, r = layer.stats(), ref_layer.stats()
    for key in ("tokens", "units_with_reps", "n_mem", "n_selected", "window_base", "active_tokens"):
        assert s[key] == r[key], key
    nu = s["units_with_reps"]
    if nu:
        assert np.array_equal(layer.reps(0, nu), ref_layer.reps(0, nu))
    layer.close()
    ref_layer.close()


@pytest.mark.parametrize("name", ["small_g4", "small_g1", "small_f32"])
def test_chaining_does_not_change_results(cuda_ok, name):
    import torch
    w = CASES[name]
    q, k, v = _inputs(w, w.n_tokens)
    a = make_layer(w, max_tokens=w.n_tokens + 8)
    b = make_layer(w, max_tokens=w.n_tokens + 8)
    b.set_launch_chaining(False)
    oa = a.prefill(q, k, v, w.chunk)
    ob = b.prefill(q, k, v, w.chunk)
    torch.cuda.synchronize()
    assert torch.equal(oa, ob)
    # decode steps after the prompt, with and without chaining
    T = w.n_tokens
    for s in range(6):
        qs, ks, vs = (to_torch(x) for x in synth.gen_chunk(w, T + s, 1))
        da = a.decode_step(qs, ks, vs)
        db = b.decode_step(qs, ks, vs)
        torch.cuda.synchronize()
        assert torch.equal(da, db), s
    a.close()
    b.close()


def test_prefill_in_pieces_and_mixed_with_decode(cuda_ok):
    """prefill(part 1) + prefill(part 2) == one prefill when part 1 ends on a chunk boundary;
    the decode steps that follow agree as well."""
    import torch
    w = CASES["small_g4"].replace(n_tokens=3000, chunk=256)
    q, k, v = _inputs(w, w.n_tokens + 4)
    one = make_layer(w, max_tokens=w.n_tokens + 4)
    two = make_layer(w, max_tokens=w.n_tokens + 4)
    T, cut = w.n_tokens, 1024
    o1 = one.prefill(q[:T].contiguous(), k[:T].contiguous(), v[:T].contiguous(), w.chunk)
    a = two.prefill(q[:cut].contiguous(), k[:cut].contiguous(), v[:cut].contiguous(), w.chunk)
    b = two.prefill(q[cut:T].contiguous(), k[cut:T].contiguous(), v[cut:T].contiguous(), w.chunk)
    torch.cuda.synchronize()
    assert torch.equal(o1, torch.cat([a, b]))
    for s in range(4):
        t = T + s
        x = one.decode_step(q[t:t + 1].contiguous(), k[t:t + 1].contiguous(), v[t:t + 1].contiguous())
        y = two.decode_step(q[t:t + 1].contiguous(), k[t:t + 1].contiguous(), v[t:t + 1].contiguous())
        torch.cuda.synchronize()
        assert torch.equal(x, y)
    one.close()
    two.close()


def test_prefill_errors(cuda_ok):
    import torch
    from block_memory_sparse_b200 import InfLLMError
    w = CASES["small_gqa"]
    layer = make_layer(w, max_tokens=600, max_chunk=200)
    q, k, v = _inputs(w, 700)
    for chunk, status in ((0, 1), (201, 1)):
        with pytest.raises(InfLLMError) as e:
            layer.prefill(q[:400].contiguous(), k[:400].contiguous(), v[:400].contiguous(), chunk)
        assert e.value.status == status
    with pytest.raises(InfLLMError) as e:  # capacity: nothing is launched
        layer.prefill(q, k, v, 200)
    assert e.value.status == 2
    assert layer.stats()["tokens"] == 0
    # a chunk appended without its attend joins the context with no outputs of its own (how a memory
    # is built from a prompt whose outputs are not needed); a later attend no longer refers to it
    layer.append_chunk(q[:100].contiguous(), k[:100].contiguous(), v[:100].contiguous())
    out = layer.prefill(q[100:600].contiguous(), k[100:600].contiguous(), v[100:600].contiguous(), 200)
    torch.cuda.synchronize()
    assert out.shape == (500, w.n_q_heads, w.head_dim)
    assert layer.stats()["tokens"] == 600
    with pytest.raises(InfLLMError) as e:
        layer.attend_chunk(q[:100].contiguous())
    assert e.value.status == 3
    # the same context as appending the first 100 tokens and prefilling the rest from scratch
    ref = make_layer(w, max_tokens=600, max_chunk=200)
    ref.append_chunk(q[:100].contiguous(), k[:100].contiguous(), v[:100].contiguous())
    ref.attend_chunk(q[:100].contiguous())
    ref_out = ref.prefill(q[100:600].contiguous(), k[100:600].contiguous(), v[100:600].contiguous(), 200)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out)
    ref.close()
    layer.close()
