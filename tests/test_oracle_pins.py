"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test checks an oracle function against a closed form, a textbook/library routine
(torch's scaled_dot_product_attention in float64 on CPU), brute force on tiny inputs, an
invariant, or a value the InfLLM pages print (tests/golden).  The inputs are chosen so that
a dropped term, a wrong sign or offset, or a transposed operand changes the result.
"""
from __future__ import annotations

import itertools
import math
import os

import numpy as np
import pytest
import torch

import synth
from oracle import infllm_oracle as O
from tests._source import Source

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


# ------------------------------------------------------------------------------------------
# independent helpers (not the oracle's code): complex-number RoPE and SDPA formulations


def rope_complex(x: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate-half RoPE as complex multiplication: (x1 + i x2) * exp(i pos theta)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    inv_freq = 1.0 / (base ** (np.arange(0, d, 2, dtype=np.float64) / d))
    z = x[..., : d // 2] + 1j * x[..., d // 2:]
    z = z * np.exp(1j * np.asarray(pos, dtype=np.float64)[..., None] * inv_freq)
    return np.concatenate([z.real, z.imag], axis=-1)


def sdpa_layer(q, K, V, c0, sels, cfg):
    """Method output for chunk [c0, c0+n) written as ONE torch SDPA call per q head.

    Keys are every token < c0+n; a boolean mask keeps sinks (n < S, n <= t), tokens of the
    selected units and the window [B, t].  The two position frames are folded into one dot
    product by augmenting to 2d dims: query [R(W) q, R(t) q], far key [k, 0], window key
    [0, R(n) k] (absolute positions: <R(t)q, R(n)k> equals the relative form).
    """
    S, W, U, base = cfg["n_sink"], cfg["window"], cfg["unit_size"], cfg["rope_base"]
    n, Hq, d = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    T = c0 + n
    B = S + U * (max(0, (c0 - W - S) // U) if c0 - W - S > 0 else 0)
    t = c0 + np.arange(n)
    idx = np.arange(T)
    out = np.zeros_like(q)
    for h in range(Hq):
        hk = h // G
        sel_tok = np.zeros(T, dtype=bool)
        for j in sels[hk]:
            sel_tok[S + j * U:S + (j + 1) * U] = True
        far = (idx < S) | sel_tok
        win = (idx >= B) & ~far
        qa = np.concatenate([rope_complex(q[:, h], np.full(n, float(W)), base),
                             rope_complex(q[:, h], t.astype(np.float64), base)], axis=-1)
        ka = np.zeros((T, 2 * d))
        ka[far, :d] = K[:T, hk][far]
        ka[win, d:] = rope_complex(K[:T, hk][win], idx[win].astype(np.float64), base)
        mask = ((idx[None] < S) & (idx[None] <= t[:, None])) | sel_tok[None] | \
               ((idx[None] >= B) & (idx[None] <= t[:, None]))
        o = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qa)[None, None], torch.from_numpy(ka)[None, None],
            torch.from_numpy(V[:T, hk])[None, None], attn_mask=torch.from_numpy(mask)[None, None],
            scale=1.0 / math.sqrt(d))
        out[:, h] = o[0, 0].numpy()
    return out


def run_stream(cfg, q, k, v, chunk, rep_method="plain", sel_fn=None):
    layer = O.OracleLayer(cfg, rep_method=rep_method)
    outs, infos = [], []
    for c0 in range(0, q.shape[0], chunk):
        n = min(chunk, q.shape[0] - c0)
        layer.append_chunk(q[c0:c0 + n], k[c0:c0 + n], v[c0:c0 + n])
        outs.append(layer.attend_chunk(None if sel_fn is None else sel_fn(layer)))
        infos.append(dict(layer.last, c0=c0, n=n))
    return layer, outs, infos


def small_cfg(**kw):
    c = dict(n_q_heads=4, n_kv_heads=2, head_dim=16, n_sink=3, window=40, unit_size=8, n_reps=2, top_k=3,
             rope_base=1e4, dtype="f32")
    c.update(kw)
    return c


def rand_stream(cfg, T, seed=0, kbias=0.0):
    r = np.random.default_rng(seed)
    q = r.standard_normal((T, cfg["n_q_heads"], cfg["head_dim"]))
    k = r.standard_normal((T, cfg["n_kv_heads"], cfg["head_dim"])) + kbias * r.standard_normal(
        (1, cfg["n_kv_heads"], cfg["head_dim"]))
    v = r.standard_normal((T, cfg["n_kv_heads"], cfg["head_dim"]))
    return q, k, v


# ------------------------------------------------------------------------------------------
# 1. RoPE


def test_rope_matches_complex_rotation():
    x = np.array([1.0, 2.0, 3.0, 4.0])
    # d=4, base 1e4: theta = (1, 0.01); closed form at position 1
    want = np.array([1 * math.cos(1) - 3 * math.sin(1), 2 * math.cos(0.01) - 4 * math.sin(0.01),
                     3 * math.cos(1) + 1 * math.sin(1), 4 * math.cos(0.01) + 2 * math.sin(0.01)])
    np.testing.assert_allclose(O.rope(x, 1.0, 1e4), want, rtol=0, atol=1e-15)
    xs = rng.standard_normal((7, 128))
    pos = np.array([0, 1, 5, 4095, 131071, 1048575, 1052799], dtype=np.float64)
    for base in (1e4, 5e5, 1e6):
        # the two theta formulas round differently: angle error ~ pos * 1e-16 rad
        err = np.abs(O.rope(xs, pos, base) - rope_complex(xs, pos, base))
        assert np.all(err <= 1e-14 + 2e-15 * pos[:, None] * np.abs(xs).max())


def test_rope_relative_identity_and_norm():
    for base in (1e4, 1e6):
        x, y = rng.standard_normal((2, 64))
        for a, b in [(0, 0), (3, 17), (1_000_000, 1_004_096), (4096, 0)]:
            lhs = O.rope(x, a, base) @ O.rope(y, b, base)
            rhs = x @ O.rope(y, b - a, base)
            assert abs(lhs - rhs) <= 1e-9 * (1 + abs(rhs))
            assert abs(np.linalg.norm(O.rope(x, a, base)) - np.linalg.norm(x)) < 1e-12
        np.testing.assert_allclose(O.rope(O.rope(x, 7, base), 11, base), O.rope(x, 18, base), atol=1e-13)
        np.testing.assert_array_equal(O.rope(x, 0, base), x)


# ------------------------------------------------------------------------------------------
# 2. selection: brute force on tiny inputs with forced ties


def _brute_topk_sets(scores, k):
    """All k-subsets T such that every member beats every non-member under (score desc, index asc)."""
    n = len(scores)
    good = []
    for T in itertools.combinations(range(n), k):
        ok = all((scores[i] > scores[j]) or (scores[i] == scores[j] and i < j)
                 for i in T for j in range(n) if j not in T)
        if ok:
            good.append(set(T))
    return good


def test_topk_stable_brute_force_with_ties():
    r = np.random.default_rng(7)
    for trial in range(300):
        n = int(r.integers(1, 9))
        s = r.integers(-2, 3, size=n).astype(float)  # integer values: many exact ties
        k = int(r.integers(0, n + 1))
        got = O.topk_stable(s, k)
        sets = _brute_topk_sets(list(s), k)
        assert len(sets) == 1 and set(got) == sets[0], (s, k, got)
        # rank order: non-increasing score, ties by increasing index
        for a, b in zip(got, got[1:]):
            assert s[a] > s[b] or (s[a] == s[b] and a < b)


def test_decisive_rule():
    assert O.decisive([3.0, 2.0, 1.0], 1)
    assert not O.decisive([1.0, 1.0, 0.0], 1)
    assert not O.decisive([1000.0, 999.5, 0.0], 1)  # gap 0.5 <= 1e-3 * 1000
    assert O.decisive([1000.0, 998.9, 0.0], 1)
    assert O.decisive([1.0, 1.0], 2) and O.decisive([1.0], 0)


# ------------------------------------------------------------------------------------------
# 3. representative scores: closed form for d = 2, linear form, brute-force selection


def test_rep_scores_closed_form_d2():
    # d = 2: theta_0 = 1 for any base.  q = (1, 0), k = (1, 0) everywhere:
    # <R(i) q, R(m) k> = cos(i - m); rho_m = G/sqrt(2) * sum_{i=e}^{e+W-1} cos(i - m)
    W, G, U, e, m0 = 37, 3, 5, 105, 100
    q = np.zeros((W, G, 2)); q[..., 0] = 1.0
    k = np.zeros((U, 2)); k[:, 0] = 1.0
    rho = O.rep_scores_plain(q, e, k, m0, 1e4)
    for m in range(U):
        a, b = e - (m0 + m), e + W - 1 - (m0 + m)  # sum_{n=a}^{b} cos n (Dirichlet closed form)
        closed = (math.sin(b + 0.5) - math.sin(a - 0.5)) / (2 * math.sin(0.5))
        assert abs(rho[m] - G * closed / math.sqrt(2)) < 1e-12
    # k = (0, 1): <R(i) q, R(m) k> = <(cos i, sin i), (-sin m, cos m)> = sin(i - m)
    k2 = np.zeros((U, 2)); k2[:, 1] = 1.0
    rho2 = O.rep_scores_plain(q, e, k2, m0, 1e4)
    for m in range(U):
        a, b = e - (m0 + m), e + W - 1 - (m0 + m)
        closed = (math.cos(a - 0.5) - math.cos(b + 0.5)) / (2 * math.sin(0.5))  # sum sin n
        assert abs(rho2[m] - G * closed / math.sqrt(2)) < 1e-12


def test_rep_scores_linear_equals_plain():
    # pin 5: sum_i <a_i, b> = <sum_i a_i, b>, at large absolute positions
    W, G, U, d = 64, 4, 16, 32
    for e in (100, 1_000_000):
        q = rng.standard_normal((W, G, d)); k = rng.standard_normal((U, d))
        plain = O.rep_scores_plain(q, e, k, e - U, 1e6)
        qs = O.rope(q, (e + np.arange(W))[:, None], 1e6).sum(axis=(0, 1))
        lin = O.rep_scores_linear(qs, k, e - U, 1e6)
        assert np.max(np.abs(plain - lin)) <= 1e-12 * np.max(np.abs(plain))


def test_rep_scores_relative_form():
    # independent formulation: rho_m = sum_i sum_h <q_{i,h}, R(m - i) k_m> / sqrt(d), complex RoPE
    W, G, U, d, e, m0 = 20, 2, 6, 8, 50, 44
    q = rng.standard_normal((W, G, d)); k = rng.standard_normal((U, d))
    rho = O.rep_scores_plain(q, e, k, m0, 1e4)
    for m in range(U):
        s = sum(q[i, h] @ rope_complex(k[m], float(m0 + m - (e + i)), 1e4) for i in range(W) for h in range(G))
        assert abs(rho[m] - s / math.sqrt(d)) < 1e-12


# ------------------------------------------------------------------------------------------
# 4. unit scores


def test_unit_scores_closed_form_d2():
    C, G, n_units, r, W = 9, 2, 4, 3, 4096
    q = np.zeros((C, G, 2)); q[..., 0] = 1.0
    keys = np.zeros((n_units, r, 2)); keys[..., 1] = 1.0
    keys[2] *= 2.0
    sig = O.unit_scores(q, keys, W, 1e6)
    # <R(W)(1,0), (0,1)> = sin(W)
    want = C * G * r * math.sin(W) / math.sqrt(2) * np.array([1, 1, 2, 1])
    np.testing.assert_allclose(sig, want, rtol=0, atol=1e-12)


def test_unit_scores_linearity():
    C, G, n_units, r, d, W = 7, 4, 11, 4, 16, 100
    q = rng.standard_normal((C, G, d)); keys = rng.standard_normal((n_units, r, d))
    sig = O.unit_scores(q, keys, W, 1e4)
    alt = (rope_complex(q.sum(axis=(0, 1)), float(W), 1e4) @ keys.sum(axis=1).T) / math.sqrt(d)
    np.testing.assert_allclose(sig, alt, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------------------------------
# 5. attention: special cases that reduce to textbook attention, and the general SDPA form


def test_vanilla_causal_rope_when_no_sinks_and_window_covers_all():
    cfg = small_cfg(n_sink=0, window=10_000, top_k=3)
    T = 150
    q, k, v = rand_stream(cfg, T, seed=1)
    _, outs, infos = run_stream(cfg, q, k, v, chunk=40)
    out = np.concatenate(outs)
    G = cfg["n_q_heads"] // cfg["n_kv_heads"]
    pos = np.arange(T, dtype=np.float64)
    for h in range(cfg["n_q_heads"]):
        qr = torch.from_numpy(rope_complex(q[:, h], pos, 1e4))[None, None]
        kr = torch.from_numpy(rope_complex(k[:, h // G], pos, 1e4))[None, None]
        ref = torch.nn.functional.scaled_dot_product_attention(qr, kr, torch.from_numpy(v[:, h // G])[None, None],
                                                               is_causal=True)[0, 0].numpy()
        np.testing.assert_allclose(out[:, h], ref, rtol=0, atol=1e-12)
    assert all(i["n_mem"] == 0 for i in infos)


@pytest.mark.parametrize("top_k", [0, 2, 1000])
def test_layer_matches_sdpa_formulation(top_k):
    # top_k = 0: StreamingLLM (sinks + window); 1000 >= n_mem: every unit (dense over n <= t)
    cfg = small_cfg(top_k=top_k)
    T = 230
    q, k, v = rand_stream(cfg, T, seed=2, kbias=2.0)
    layer, outs, infos = run_stream(cfg, q, k, v, chunk=33)
    for o, inf in zip(outs, infos):
        c0, n = inf["c0"], inf["n"]
        ref = sdpa_layer(q[c0:c0 + n], k, v, c0, inf["sel"], cfg)
        np.testing.assert_allclose(o, ref, rtol=0, atol=1e-11)
        if top_k >= 1000:
            assert all(sorted(s) == list(range(inf["n_mem"])) for s in inf["sel"])
        if top_k == 0:
            assert all(s == [] for s in inf["sel"])
    assert infos[-1]["n_mem"] > 10


def test_dense_when_all_units_selected():
    # with every unit selected the key set of query t is every n <= t
    cfg = small_cfg(top_k=1000)
    T = 200
    q, k, v = rand_stream(cfg, T, seed=3)
    layer, outs, infos = run_stream(cfg, q, k, v, chunk=50)
    for inf in infos:
        t_last = inf["c0"] + inf["n"] - 1
        counts = inf["key_counts"]  # [Hkv, n]
        np.testing.assert_array_equal(counts, np.broadcast_to(inf["c0"] + np.arange(inf["n"]) + 1, counts.shape))
        assert counts.max() == t_last + 1


def test_softmax_rows_and_convex_hull():
    cfg = small_cfg()
    q, k, v = rand_stream(cfg, 180, seed=4)
    layer = O.OracleLayer(cfg)
    G = 2
    for c0 in range(0, 180, 45):
        layer.append_chunk(q[c0:c0 + 45], k[c0:c0 + 45], v[c0:c0 + 45])
        for hk in range(2):
            sel = [0] if c0 >= 120 else []
            o, rows, keys, valid = O.attend_group(q[c0:c0 + 45, hk * G:(hk + 1) * G], c0, sel,
                                                  lambda i: k[i, hk], lambda i: v[i, hk], cfg)
            assert np.max(np.abs(rows - 1.0)) < 1e-12
            for ti in range(45):
                vv = v[keys[valid[ti]], hk]
                assert np.all(o[ti] >= vv.min(axis=0) - 1e-12) and np.all(o[ti] <= vv.max(axis=0) + 1e-12)


def test_active_token_count_golden():
    # the page's count: sinks + k * unit + local window.  Under the window reading [B, t], the
    # first query of a chunk whose start c0 has c0 - B = W sees W + 1 window tokens, so the
    # page's local window of L tokens is the window parameter W = L - 1 at that query.
    rows = [l.split() for l in open(os.path.join(GOLDEN, "active_tokens.txt")) if l.strip() and l[0] != "#"]
    for S, k, U, L, want in ([int(x) for x in r] for r in rows):
        cfg = small_cfg(n_q_heads=1, n_kv_heads=1, head_dim=8, n_sink=S, top_k=k, unit_size=U, window=L - 1)
        c0 = S + (L - 1) + k * U  # n_mem(c0) = k, B = c0 - (L - 1)
        q, kk, v = rand_stream(cfg, c0 + 1, seed=5)
        layer = O.OracleLayer(cfg, rep_method="linear")
        layer.append_chunk(q[:c0], kk[:c0], v[:c0])
        layer.append_chunk(q[c0:], kk[c0:], v[c0:])
        layer.attend_chunk()
        assert layer.last["n_mem"] == k and layer.last["B"] == c0 - (L - 1)
        assert int(layer.last["key_counts"][0, 0]) == want == S + k * U + L


# ------------------------------------------------------------------------------------------
# 6. chunked (stateful) results equal the stateless recomputation from the full prefix


def test_streaming_equals_stateless_recomputation():
    w = synth.SMALL["small_gqa"].replace(n_tokens=1500, window=256, chunk=170)
    cfg = w.as_config()
    src = Source(w)
    T = w.n_tokens
    q, k, v = src.q(0, T), src.k(0, T), src.v(0, T)
    layer, outs, infos = run_stream(cfg, q, k, v, chunk=w.chunk, rep_method="plain")
    for o, inf in zip(outs, infos):
        ref, rinfo = O.chunk_stateless(src.q, src.k, src.v, inf["c0"], inf["n"], cfg)
        assert rinfo["sel"] == inf["sel"]
        np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    # representatives: plain double loop (stateful) vs summed-query form (stateless)
    reps, rho = O.all_reps_linear(src.q, src.k, T, cfg)
    for j in range(len(layer.reps)):
        assert np.max(np.abs(layer.rep_scores[j] - rho[j])) <= 1e-12 * np.max(np.abs(rho[j]))
        assert layer.reps[j] == reps[j]
    assert infos[-1]["n_mem"] >= 15


def test_batched_linear_reps_and_key_table_past_256_units():
    # the summed-query form fetches keys 256 units at a time: more than 256 units here, against
    # the plain double loop of the streaming layer and a direct gather of the representative keys
    cfg = small_cfg(n_q_heads=2, n_kv_heads=1, head_dim=8, n_sink=2, window=8, unit_size=4, n_reps=2)
    T = 2 + 4 * 300 + 8 + 4
    q, k, v = rand_stream(cfg, T, seed=7)
    layer = O.OracleLayer(cfg, rep_method="plain")
    for c0 in range(0, T, 128):
        n = min(128, T - c0)
        layer.append_chunk(q[c0:c0 + n], k[c0:c0 + n], v[c0:c0 + n])
    layer._evict_to(T)
    nu = len(layer.reps)
    assert nu > 256
    reps, rho = O.all_reps_linear(lambda t0, n: q[t0:t0 + n], lambda t0, n: k[t0:t0 + n], T, cfg)
    assert len(reps) == nu
    for j in range(nu):
        assert reps[j] == layer.reps[j]
        assert np.max(np.abs(rho[j] - layer.rep_scores[j])) <= 1e-12 * np.max(np.abs(rho[j]))
    table = O.rep_key_table(lambda t0, n: k[t0:t0 + n], reps, nu, cfg)
    for j in (0, 255, 256, nu - 1):
        assert np.array_equal(table[0, j], k[[2 + 4 * j + m for m in reps[j][0]], 0])


def test_representatives_brute_force_ties():
    # integer-valued q/k with d=2 at positions multiple of 2*pi are not available, so force ties by
    # duplicated keys: equal keys at different positions differ only by rotation; use W so that the
    # score is position independent: q = 0 except one token -> ties broken to the lower index.
    cfg = small_cfg(n_q_heads=1, n_kv_heads=1, head_dim=4, n_sink=0, window=8, unit_size=8, n_reps=3)
    T = 24
    q = np.zeros((T, 1, 4)); k = np.zeros((T, 1, 4)); v = np.ones((T, 1, 4))
    layer = O.OracleLayer(cfg)
    layer.append_chunk(q[:16], k[:16], v[:16])
    layer.append_chunk(q[16:], k[16:], v[16:])  # unit 0 evicted at c0 = 16; all rho = 0
    assert layer.reps[0] == [[0, 1, 2]]


# ------------------------------------------------------------------------------------------
# 7. planted needle


def test_needle_unit_is_selected():
    w = synth.SMALL["small_needle"]
    cfg = w.as_config()
    src = Source(w)
    j_star = synth.needle_info(w)[0]
    c0, n = synth.chunk_bounds(w)[-1]
    out, info = O.chunk_stateless(src.q, src.k, src.v, c0, n, cfg)
    for hk in range(w.n_kv_heads):
        assert info["sel"][hk][0] == j_star
        sig = np.sort(info["sigma"][hk])[::-1]
        assert sig[0] > 3 * abs(sig[1])


# ------------------------------------------------------------------------------------------
# generator (shared input module): published Philox known answers, statistics


def test_philox_known_answers():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) if l.strip() and l[0] != "#"]
    for r in rows:
        vals = [int(x, 16) for x in r]
        got = synth.philox4x32_10(vals[0:4], vals[4:6])
        assert [int(x) for x in got] == vals[6:10]


def test_generator_is_counter_based_and_normal():
    a = synth.normal(9, 1, 0, 300, 4, 64, dtype="f32")
    b = synth.normal(9, 1, 100, 100, 4, 64, dtype="f32")
    np.testing.assert_array_equal(a[100:200], b)
    bf = synth.normal(9, 1, 0, 300, 4, 64, dtype="bf16")
    np.testing.assert_array_equal(bf, synth.round_bf16(a))
    big = synth.normal(3, 2, 0, 4096, 8, 128, dtype="f32").ravel()
    assert abs(big.mean()) < 0.01 and abs(big.std() - 1) < 0.01


# ------------------------------------------------------------------------------------------
# 8. the mean-of-keys unit representation ("InfLLM: Training-Free Long-Context Extrapolation
#    ...", research-map summary, "Measured effects", row "Use selected representative tokens
#    instead of mean key-vector representations")


def test_bf16_rounding_hand_values():
    # bf16 keeps 8 significant bits: the grid next to 1 is 1 + k 2^-7; halfway cases go to even k
    x = [1.0 + 2 ** -9, 1.0 + 3 * 2 ** -9, 1.0 + 3 * 2 ** -8, -(1.0 + 3 * 2 ** -8), 3.0, 0.1, 1.0 + 2 ** -8]
    want = [1.0, 1.0 + 2 ** -7, 1.0 + 2 ** -6, -(1.0 + 2 ** -6), 3.0, 0.10009765625, 1.0]
    assert O.round_to_dtype(x, "bf16").tolist() == want
    assert O.round_to_dtype([0.1], "f32")[0] == float(np.float32(0.1))


def test_mean_key_of_constant_and_hand_units():
    c = O.round_to_dtype(rng.standard_normal(16), "bf16")
    for U in (1, 3, 128):
        np.testing.assert_array_equal(O.unit_mean_key(np.tile(c, (U, 1)), "bf16"), c)
    np.testing.assert_array_equal(O.unit_mean_key(np.array([[1.0, 2.0], [3.0, 4.0]]), "f64"), [2.0, 3.0])
    # (0.5 + 1.0 + 2.0) / 3 = 7/6 -> bf16 1.1640625 (7/6 = 1.00101010..b: 8 bits 1.0010101 then 0 1 0...)
    assert O.unit_mean_key(np.array([[0.5], [1.0], [2.0]]), "bf16")[0] == 1.1640625


def test_mean_key_score_is_the_all_token_score_over_u():
    """Scored with its mean key (unrounded), a unit's score is the score it gets with all of its U tokens
    as representatives, divided by U -- the sum over representatives is linear in the keys."""
    C, G, U, n_units, d, W = 5, 4, 16, 6, 32, 300
    q = rng.standard_normal((C, G, d))
    keys = rng.standard_normal((n_units, U, d)) + 2.0
    all_tok = O.unit_scores(q, keys, W, 1e4)
    means = np.stack([O.unit_mean_key(keys[j], "f64") for j in range(n_units)])[:, None, :]
    np.testing.assert_allclose(O.unit_scores(q, means, W, 1e4), all_tok / U, rtol=1e-12, atol=1e-12)


def test_mean_key_layer_streaming_equals_stateless():
    w = synth.SMALL["small_gqa"].replace(n_tokens=1300, window=256, chunk=170)
    cfg = dict(w.as_config(), unit_repr="meankey")
    src = Source(w)
    T = w.n_tokens
    q, k, v = src.q(0, T), src.k(0, T), src.v(0, T)
    layer, outs, infos = run_stream(cfg, q, k, v, chunk=w.chunk, rep_method="linear")
    table = O.mean_key_table(src.k, O.n_mem(T, w.n_sink, w.window, w.unit_size), cfg)
    for hk in range(w.n_kv_heads):
        for j in range(table.shape[1]):
            u = k[w.n_sink + j * w.unit_size:w.n_sink + (j + 1) * w.unit_size, hk]
            np.testing.assert_array_equal(table[hk, j], O.round_to_dtype(u.mean(axis=0), "bf16"))
    n_cmp = 0
    for o, inf in zip(outs, infos):
        ref, rinfo = O.chunk_stateless(src.q, src.k, src.v, inf["c0"], inf["n"], cfg)
        assert rinfo["sel"] == inf["sel"]
        np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
        n_cmp += inf["n_mem"] > w.top_k
    assert n_cmp >= 3
    # the mean-key selection is a different one than the representatives' on this stream
    rep_layer, _, rep_infos = run_stream(w.as_config(), q, k, v, chunk=w.chunk, rep_method="linear")
    assert any(a["sel"] != b["sel"] for a, b in zip(infos, rep_infos))
