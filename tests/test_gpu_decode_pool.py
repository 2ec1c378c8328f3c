"""Decode lookup over a large pool (2101 units: the scoring grid's last CTA ends on a ragged
32-unit block), against the fp64 oracle with its own representatives; both scoring modes."""
from __future__ import annotations

import numpy as np
import pytest

import synth
from oracle import infllm_oracle as O
from tests._parity import compare_reps, make_layer, to_np64, to_torch
from tests._source import Source
from tests.test_gpu_fullsize import _check_chunk

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("score_mode", ["reps", "repsum"])
def test_decode_lookup_over_2101_units(cuda_ok, score_mode):
    import torch
    base = synth.SMALL["small_decode"]  # 8 q / 2 KV heads, d = 128, S = 16, W = 512, U = 64, k = 4
    units = 2101
    T0 = base.n_sink + units * base.unit_size + base.window
    w = base.replace(n_tokens=T0, decode_steps=3, build_chunk=2048)
    cfg, src = w.as_config(), Source(w)
    layer = make_layer(w, score_mode=score_mode)
    for c0 in range(0, T0, w.build_chunk):
        n = min(w.build_chunk, T0 - c0)
        layer.append_chunk(*(to_torch(x) for x in synth.gen_chunk(w, c0, n)))
    rec = {}
    for s in range(w.decode_steps):
        q, k, v = synth.gen_chunk(w, T0 + s, 1)
        out = layer.decode_step(to_torch(q), to_torch(k), to_torch(v))
        torch.cuda.synchronize()
        rec[s] = dict(out=to_np64(out), sel=layer.selection().copy(), scores=layer.unit_scores().copy())
    t_last = T0 + w.decode_steps - 1
    nu = O.n_mem(t_last, w.n_sink, w.window, w.unit_size)
    assert nu >= units
    g_reps = layer.reps(0, nu)
    oreps, rho = O.all_reps_linear(src.q, src.k, t_last, cfg)
    dec, tot, bad_dec, _ = compare_reps(g_reps, rho, w.n_reps)
    assert bad_dec == 0 and dec >= 0.5 * tot
    rep_keys = O.rep_key_table(src.k, oreps, nu, cfg)
    for s in range(w.decode_steps):
        t = T0 + s
        nm = O.n_mem(t, w.n_sink, w.window, w.unit_size)
        assert nm >= 2048
        _check_chunk(w, src, cfg, oreps, rep_keys[:, :nm], t, 1, rec[s]["out"], rec[s]["sel"], rec[s]["scores"],
                     g_reps)
    layer.close()
