"""The allocation-free lookup entry point against the library's own decode lookup and the oracle.

infllm_select_units_noalloc serves callers that cannot allocate device memory (stream
capture under frameworks that forbid it, engines that plan every device byte, real-time
loops).  It keeps its scratch in a static device array, so it is checked here on two calls
in a row, each against the unit scores that infllm_decode_step produced for the same token and
against the fp64 oracle's scores on the same representatives, within the tolerances the parity
tests use; its selection is the oracle's where the oracle's cut is decisive, and otherwise a
valid choice inside the near-tie band.  This file is collected last on purpose and must pass
alone in a fresh process as well.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest

import synth
from oracle import infllm_oracle as O
from tests._parity import make_layer, to_torch, valid_near_tie

pytestmark = pytest.mark.gpu


def test_noalloc_selection_matches_decode_lookup(cuda_ok):
    import torch

    import block_memory_sparse_b200 as bms
    w = synth.SMALL["small_decode"]
    L = bms.load_library()
    layer = make_layer(w)
    T0 = w.n_tokens
    k_host = np.empty((T0 + 2, w.n_kv_heads, w.head_dim), dtype=np.uint16)
    for c0 in range(0, T0, w.build_chunk):
        n = min(w.build_chunk, T0 - c0)
        q, k, v = synth.gen_chunk(w, c0, n)
        k_host[c0:c0 + n] = k
        layer.append_chunk(to_torch(q), to_torch(k), to_torch(v))
    stream = torch.cuda.current_stream()
    for s in range(2):  # two calls in a row share the static scratch area
        t = T0 + s
        q, k, v = synth.gen_chunk(w, t, 1)
        k_host[t] = k[0]
        qd = to_torch(q)
        layer.decode_step(qd, to_torch(k), to_torch(v))
        ref_sel = layer.selection()
        ref_scores = layer.unit_scores()
        nm = ref_scores.shape[1]
        assert nm == O.n_mem(t, w.n_sink, w.window, w.unit_size) > w.top_k
        ids = layer.reps(0, nm)  # [Hkv][nm][r] unit-local offsets
        pool = np.empty((w.n_kv_heads, nm, w.n_reps, w.head_dim), dtype=np.uint16)
        for h in range(w.n_kv_heads):
            for j in range(nm):
                pool[h, j] = k_host[w.n_sink + j * w.unit_size + ids[h, j], h]
        pool_d = to_torch(pool)
        sel_d = torch.full((w.n_kv_heads, w.top_k), 7, dtype=torch.int32, device="cuda")
        sc_d = torch.zeros((w.n_kv_heads, nm), dtype=torch.float32, device="cuda")
        st = L.infllm_select_units_noalloc(
            ctypes.c_void_p(pool_d.data_ptr()), ctypes.c_void_p(qd.data_ptr()), w.n_q_heads, w.n_kv_heads,
            w.head_dim, nm, w.n_reps, w.window, w.rope_base, 1, w.top_k, ctypes.c_void_p(sel_d.data_ptr()),
            ctypes.c_void_p(sc_d.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
        assert st == 0
        torch.cuda.synchronize()
        got_scores = sc_d.cpu().numpy()
        got_sel = sel_d.cpu().numpy()
        q64 = synth.to_f64(q)[0]  # [Hq, d]
        G = w.n_q_heads // w.n_kv_heads
        for h in range(w.n_kv_heads):
            # oracle: the token's group queries against the same representative keys, in fp64
            sig = O.unit_scores(q64[None, h * G:(h + 1) * G], synth.to_f64(pool[h]), w.window, w.rope_base)
            scale = max(1e-6, float(np.max(np.abs(sig))))
            assert np.max(np.abs(got_scores[h] - sig)) <= 2e-5 * scale + 1e-5
            assert np.max(np.abs(got_scores[h] - ref_scores[h])) <= 2e-5 * scale + 1e-5
            got = got_sel[h].tolist()
            assert got == sorted(got)
            if O.decisive(sig, w.top_k):
                assert got == sorted(O.topk_stable(sig, w.top_k))
                assert got == ref_sel[h].tolist()
            else:
                assert valid_near_tie(sig, got, w.top_k), (h, got)
    # sizes beyond the scratch area are refused before any work is enqueued
    st = L.infllm_select_units_noalloc(ctypes.c_void_p(pool_d.data_ptr()), ctypes.c_void_p(qd.data_ptr()), 65 * 4,
                                       65, w.head_dim, 10, w.n_reps, w.window, w.rope_base, 1, w.top_k,
                                       ctypes.c_void_p(sel_d.data_ptr()), None, ctypes.c_void_p(stream.cuda_stream))
    assert st == 2
    st = L.infllm_select_units_noalloc(ctypes.c_void_p(pool_d.data_ptr()), ctypes.c_void_p(qd.data_ptr()),
                                       w.n_q_heads, w.n_kv_heads, w.head_dim, 16385, w.n_reps, w.window, w.rope_base,
                                       1, w.top_k, ctypes.c_void_p(sel_d.data_ptr()), None,
                                       ctypes.c_void_p(stream.cuda_stream))
    assert st == 2
    layer.close()
