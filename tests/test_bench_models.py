"""The bench's algorithmic work models against the oracle's own key sets (no GPU needed).

`chunk_flops` (the attention kernel's roofline numerator) must equal 4 d Hq times the number of
(query, key) pairs the oracle attends; `decode_bytes` must count the keys one decode token attends
plus the scoring operand of every eligible unit."""
from __future__ import annotations

import numpy as np
import pytest

import bench
import synth
from oracle import infllm_oracle as O
from tests._source import Source


@pytest.mark.parametrize("name", ["small_gqa", "small_g4", "small_nosink", "small_allunits"])
def test_chunk_flops_counts_the_attended_pairs(name):
    w = synth.SMALL[name]
    src = Source(w)
    cfg = w.as_config()
    layer = O.OracleLayer(cfg, rep_method="linear")
    for c0, n in synth.chunk_bounds(w):
        layer.append_chunk(src.q(c0, n), src.k(c0, n), src.v(c0, n))
        layer.attend_chunk()
        pairs = layer.last["key_counts"]  # [Hkv, n] keys attended by each query of each group
        assert np.all(pairs == pairs[0])  # the same key set for every KV group
        want = 4.0 * w.head_dim * w.n_q_heads * float(pairs[0].sum())
        assert bench.chunk_flops(w, c0, n) == want, (c0, n)


@pytest.mark.parametrize("mode", ["reps", "repsum"])
def test_decode_bytes_counts_keys_and_the_scoring_operand(mode):
    w = synth.SMALL["small_decode"]
    src = Source(w)
    layer = O.OracleLayer(w.as_config(), rep_method="linear")
    T0 = w.n_tokens
    elt = 2 if w.dtype == "bf16" else 4
    for t in (T0, T0 + 37, T0 + 64):
        t_have = layer.t
        if t > t_have:  # tokens before t, then t alone as a one-token chunk (a decode step)
            layer.append_chunk(src.q(t_have, t - t_have), src.k(t_have, t - t_have), src.v(t_have, t - t_have))
        layer.append_chunk(src.q(t, 1), src.k(t, 1), src.v(t, 1))
        layer.attend_chunk()
        keys = int(layer.last["key_counts"][0, 0])
        nm = layer.last["n_mem"]
        per_unit = w.n_reps * w.head_dim * elt if mode == "reps" else w.head_dim * 4
        want = nm * w.n_kv_heads * per_unit + keys * w.n_kv_heads * w.head_dim * elt * 2
        assert bench.decode_bytes(w, t, mode) == want, t


def test_attention_traffic_key_ignores_comments_only():
    """The captured DRAM traffic is keyed to the attention kernel's device code: editing a comment
    keeps the key, changing a statement or anything before the host-side part changes it, and the
    host-side part (tensor maps, launcher) does not enter it."""
    src = open(bench.ATTN_SOURCE).read()
    cut = src.index("typedef CUresult (*EncodeTiledFn)")
    base = bench.attn_device_hash(src)
    line = "constexpr int BN = 128;  // keys per tile"
    assert line in src
    assert bench.attn_device_hash(src.replace(line, "constexpr int BN = 128;  // keys in one tile")) == base
    assert bench.attn_device_hash(src.replace("// Exact attention", "/* a block comment */\n// Exact attention", 1)) == base
    assert bench.attn_device_hash(src.replace(line, "constexpr int BN = 64;  // keys per tile")) != base
    assert bench.attn_device_hash(src[:cut] + src[cut:].replace("return", "return ", 1)) == base
    # the committed profile's key matches the committed kernel, so the bench reports its traffic
    assert bench.attn_traffic() is not None
