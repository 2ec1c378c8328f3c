"""Plain fp64 CPU oracle for InfLLM block-memory sparse attention (one layer).

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import
this module.  It shares no code with the CUDA path: it reads the same
generated input values (widened exactly to float64) and recomputes every
step of the method with numpy in float64, in the order the method states.

Sources (the method as described on the InfLLM pages):
  [G1] "InfLLM Guide: Training-Free Long-Context Memory Units", section
       "Core Innovation 1: Structured Context Partitioning" -- sinks, memory
       units of fixed size, local window.
  [G2] same page, "Core Innovation 2 ... Dynamic Top-K Selection", item 2
       "Query-Aware Top-K Scoring and Loading" -- Score(M_j) = q . r / sqrt(d),
       keep the top-k units; item 3 "Exact Attention Evaluation" -- one
       exact softmax over Sinks U selected units U local window.
  [G3] same page, "Operational Checklist" -- native RoPE base, relative
       offsets inside memory.
  [S1] "InfLLM: Training-Free Long-Context Extrapolation for LLMs with an
       Efficient Context Memory" (atlas.scime.ai summary), "Approach" --
       units are represented by their top-scoring representative tokens
       chosen by attention scores; lookup at every step.
  [S2] same page, "Measured effects" table, ablation rows -- lookup in both
       encoding (chunked prefill) and decoding.
  [R1] OpenReview rebuttal (paperhub.cn), Q2 "Comparison to Well-trained Long
       LLM" -- lookup during pre-filling is done per block (chunk).
  [S3] same summary page as [S1], "Measured effects" row "Use selected
       representative tokens instead of mean key-vector representations" and
       "Surprising findings" -- the mean of a unit's keys as the alternative unit
       representation; [G2]'s listing ("Step-by-Step Implementation",
       append_context_block) builds it by mean pooling the unit's keys.

Readings taken where the pages leave a step open (each is listed with its
reason in the design notes of the repository):
  * q head h uses kv head h // G (contiguous grouped-query attention).
  * R(p) is rotate-half RoPE: pairs (i, i + d/2), angle p * base^(-2i/d).
  * A representative score is the raw scaled logit summed over the W
    queries that follow the unit ([e_j, e_j + W)) and over the G q heads of
    the kv group, at true positions; the top n_reps tokens are kept, ties
    to the lower token index.
  * The unit score of a chunk is the scaled logit summed over the chunk's
    queries, the group's q heads and the unit's representatives, with the
    query at relative distance W from the (unrotated) key; the top
    min(top_k, n_mem) units are kept per kv head, ties to the lower unit.
  * n_mem(c0) = max(0, floor((c0 - W - S) / U)); the window of query t is
    [B, t] with B = S + U * n_mem(c0); sinks are tokens n < S with n <= t.
  * Sinks and memory tokens sit at relative distance W (query rotated by
    R(W), key raw); window pairs use true relative distance t - n.
  * The mean-of-keys representation of a unit is the mean of its U raw keys,
    stored in the layer's dtype (rounded to nearest, ties to even), like the
    listing's mean of a key block in the model's dtype; a unit's score is then
    the same scaled logit with that one vector as the unit's only key.

Parity pins for every function live in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math
from typing import Callable, Sequence

import numpy as np

# --------------------------------------------------------------------------------------------
# positions  [G3]


def theta(d: int, base: float) -> np.ndarray:
    """RoPE frequencies theta_i = base^(-2i/d), i < d/2 (float64)."""
    return base ** (-2.0 * np.arange(d // 2, dtype=np.float64) / d)


def rope(x: np.ndarray, pos, base: float) -> np.ndarray:
    """R(pos) x for rotate-half RoPE.  x [..., d]; pos broadcasts against x.shape[:-1]."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    half = d // 2
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta(d, base)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# --------------------------------------------------------------------------------------------
# context partition  [G1]


def n_mem(c0: int, n_sink: int, window: int, unit: int) -> int:
    """Units whose last token is at least `window` tokens before c0 (eligible for lookup)."""
    x = c0 - window - n_sink
    return x // unit if x > 0 else 0


def window_base(c0: int, n_sink: int, window: int, unit: int) -> int:
    """First token of the local window for a chunk starting at c0."""
    return n_sink + unit * n_mem(c0, n_sink, window, unit)


def unit_tokens(j: int, n_sink: int, unit: int) -> range:
    return range(n_sink + j * unit, n_sink + (j + 1) * unit)


# --------------------------------------------------------------------------------------------
# selection helpers


def topk_stable(scores: Sequence[float], k: int) -> list[int]:
    """Indices of the k largest scores, ties broken to the lower index (full stable sort)."""
    order = sorted(range(len(scores)), key=lambda i: (-float(scores[i]), i))
    return order[:k]


def decisive(scores: Sequence[float], k: int, rel: float = 1e-3) -> bool:
    """True iff the k-th and (k+1)-th largest scores differ by more than rel * max(|s_k|, |s_k+1|)."""
    n = len(scores)
    if k <= 0 or k >= n:
        return True
    s = sorted((float(x) for x in scores), reverse=True)
    a, b = s[k - 1], s[k]
    return (a - b) > rel * max(abs(a), abs(b))


# --------------------------------------------------------------------------------------------
# representative tokens  [S1]


def rep_scores_plain(q_win: np.ndarray, e: int, k_unit: np.ndarray, m0: int, base: float) -> np.ndarray:
    """rho_m = sum_{i=e}^{e+W-1} sum_{h in group} <R(i) q_{i,h}, R(m) k_m> / sqrt(d).

    q_win [W, G, d]: the group's queries at tokens e..e+W-1; k_unit [U, d]: the unit's raw keys
    at tokens m0..m0+U-1.  Explicit loop over query tokens and heads.
    """
    W, G, d = q_win.shape
    U = k_unit.shape[0]
    k_rot = rope(k_unit, m0 + np.arange(U), base)  # [U, d]
    rho = np.zeros(U, dtype=np.float64)
    for i in range(W):
        for h in range(G):
            qi = rope(q_win[i, h], e + i, base)
            rho += k_rot @ qi
    return rho / math.sqrt(d)


def rep_scores_linear(q_rot_sum: np.ndarray, k_unit: np.ndarray, m0: int, base: float) -> np.ndarray:
    """Same scores through sum_i <a_i, b> = <sum_i a_i, b>: q_rot_sum = sum_i sum_h R(i) q_{i,h} [d]."""
    d = k_unit.shape[-1]
    k_rot = rope(k_unit, m0 + np.arange(k_unit.shape[0]), base)
    return (k_rot @ q_rot_sum) / math.sqrt(d)


def select_reps(rho: np.ndarray, n_reps: int) -> list[int]:
    """The n_reps highest-scoring tokens of a unit (unit-local indices, rank order)."""
    return topk_stable(rho, n_reps)


# --------------------------------------------------------------------------------------------
# mean-of-keys unit representation  [S3]


def round_to_dtype(x, dtype: str) -> np.ndarray:
    """Round float64 values to the nearest value of `dtype` ("f64": unchanged; "f32": float32;
    "bf16": 8 significant bits), ties to even, returned as float64.  Normal numbers only for bf16."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f64":
        return x.copy()
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    assert dtype == "bf16", dtype
    m, e = np.frexp(x)  # x = m * 2^e, 0.5 <= |m| < 1: 8 significant bits keep m * 2^8 integral
    return np.ldexp(np.rint(m * 256.0) / 256.0, e)


def unit_mean_key(k_unit: np.ndarray, dtype: str) -> np.ndarray:
    """The unit's representation as the mean of its raw keys: k_unit [U, d] -> [d] in `dtype`."""
    return round_to_dtype(k_unit.sum(axis=0) / k_unit.shape[0], dtype)


def mean_key_table(ksrc: Callable, n_units: int, cfg: dict) -> np.ndarray:
    """Mean key of every unit < n_units: [Hkv, n_units, d] (keys fetched 256 units at a time)."""
    S, U, Hkv, d = cfg["n_sink"], cfg["unit_size"], cfg["n_kv_heads"], cfg["head_dim"]
    out = np.zeros((Hkv, n_units, d))
    for j0 in range(0, n_units, 256):
        nb = min(256, n_units - j0)
        kb = ksrc(S + j0 * U, nb * U)
        for j in range(j0, j0 + nb):
            for hk in range(Hkv):
                out[hk, j] = unit_mean_key(kb[(j - j0) * U:(j - j0 + 1) * U, hk], cfg["dtype"])
    return out


# --------------------------------------------------------------------------------------------
# unit lookup  [G2] item 2, [R1]


def unit_scores(q_chunk: np.ndarray, rep_keys: np.ndarray, window: int, base: float) -> np.ndarray:
    """sigma_j = sum_t sum_h sum_m <R(W) q_{t,h}, k_m> / sqrt(d).

    q_chunk [C, G, d] the chunk's queries of one kv group; rep_keys [n_units, r, d] raw keys.
    """
    d = q_chunk.shape[-1]
    qr = rope(q_chunk, float(window), base)  # every memory token sits at distance W
    return np.einsum("thd,jmd->j", qr, rep_keys, optimize=True) / math.sqrt(d)


# --------------------------------------------------------------------------------------------
# exact attention over sinks U selected units U window  [G2] item 3


def attend_group(q: np.ndarray, c0: int, sel: Sequence[int], K: Callable, V: Callable, cfg: dict):
    """Outputs of one kv group for the chunk's queries.

    q [n, G, d] queries of tokens c0..c0+n-1 (the group's heads); sel: selected unit ids;
    K(idx), V(idx) return float64 [len(idx), d] raw keys / values of that kv head.
    Returns out [n, G, d], row sums of the softmax weights [n, G], key indices [n_keys] and the
    validity mask [n, n_keys] (key attended by query row).
    """
    S, W, U, base = cfg["n_sink"], cfg["window"], cfg["unit_size"], cfg["rope_base"]
    n, G, d = q.shape
    B = window_base(c0, S, W, U)
    t = c0 + np.arange(n)
    sink_idx = np.arange(min(S, c0 + n))
    mem_idx = np.array([m for j in sorted(sel) for m in unit_tokens(j, S, U)], dtype=np.int64)
    win_idx = np.arange(B, c0 + n)
    keys = np.concatenate([sink_idx, mem_idx, win_idx]).astype(np.int64)
    n_far = len(sink_idx) + len(mem_idx)

    kk = K(keys)  # [n_keys, d]
    vv = V(keys)
    # logits: far keys at distance W (query R(W), key raw); window keys at true relative distance
    q_far = rope(q, float(W), base)  # [n, G, d]
    q_win = rope(q, (t - B)[:, None], base)  # [n, G, d]
    k_win = rope(kk[n_far:], keys[n_far:] - B, base)
    logits = np.empty((n, G, len(keys)), dtype=np.float64)
    logits[:, :, :n_far] = q_far @ kk[:n_far].T
    logits[:, :, n_far:] = q_win @ k_win.T
    logits /= math.sqrt(d)

    valid = np.ones((n, len(keys)), dtype=bool)
    valid[:, :len(sink_idx)] = sink_idx[None, :] <= t[:, None]
    valid[:, n_far:] = keys[None, n_far:] <= t[:, None]
    logits = np.where(valid[:, None, :], logits, -np.inf)

    mx = logits.max(axis=-1, keepdims=True)
    p = np.exp(logits - mx)
    p /= p.sum(axis=-1, keepdims=True)
    out = p @ vv
    return out, p.sum(axis=-1), keys, valid


# --------------------------------------------------------------------------------------------
# streaming layer: the method step by step over a token stream


class OracleLayer:
    """Stateful oracle: append_chunk / attend_chunk over a token stream, like the library's calls.

    Keeps every token's q/k/v in float64 (small streams only).  Representatives of a unit are
    computed when the unit becomes eligible, from the W queries that follow it.
    `rep_method` "plain" uses the explicit double loop, "linear" the summed-query form.
    cfg["unit_repr"] = "meankey" scores units by the mean of their keys instead of their
    representatives (default "reps").
    """

    def __init__(self, cfg: dict, rep_method: str = "plain"):
        self.cfg = dict(cfg)
        self.G = cfg["n_q_heads"] // cfg["n_kv_heads"]
        self.rep_method = rep_method
        self.q = np.zeros((0, cfg["n_q_heads"], cfg["head_dim"]))
        self.k = np.zeros((0, cfg["n_kv_heads"], cfg["head_dim"]))
        self.v = np.zeros((0, cfg["n_kv_heads"], cfg["head_dim"]))
        self.reps: list[list[list[int]]] = []  # [unit][kv head] -> rank-ordered unit-local ids
        self.rep_scores: list[np.ndarray] = []  # [unit] -> rho [Hkv, U]
        self.last = None

    @property
    def t(self) -> int:
        return self.q.shape[0]

    def _evict_to(self, c0: int):
        c = self.cfg
        S, W, U, r = c["n_sink"], c["window"], c["unit_size"], c["n_reps"]
        G, base = self.G, c["rope_base"]
        for j in range(len(self.reps), n_mem(c0, S, W, U)):
            e = S + (j + 1) * U
            per_head, rhos = [], []
            for hk in range(c["n_kv_heads"]):
                qw = self.q[e:e + W, hk * G:(hk + 1) * G]
                ku = self.k[S + j * U:e, hk]
                if self.rep_method == "plain":
                    rho = rep_scores_plain(qw, e, ku, S + j * U, base)
                else:
                    qs = rope(qw, (e + np.arange(W))[:, None], base).sum(axis=(0, 1))
                    rho = rep_scores_linear(qs, ku, S + j * U, base)
                rhos.append(rho)
                per_head.append(select_reps(rho, r))
            self.reps.append(per_head)
            self.rep_scores.append(np.stack(rhos))

    def append_chunk(self, q: np.ndarray, k: np.ndarray, v: np.ndarray):
        c0 = self.t
        self._evict_to(c0)  # uses only queries < c0
        self.q = np.concatenate([self.q, q])
        self.k = np.concatenate([self.k, k])
        self.v = np.concatenate([self.v, v])
        self._chunk = (c0, q.shape[0])

    def attend_chunk(self, sel_override=None):
        """Unit lookup + exact attention for the chunk just appended.

        sel_override: optional [Hkv] list of unit-id lists to attend with instead of the oracle's
        own selection (to check outputs on another correct selection near ties).
        """
        c = self.cfg
        c0, n = self._chunk
        S, W, U, k = c["n_sink"], c["window"], c["unit_size"], c["top_k"]
        G = self.G
        nm = n_mem(c0, S, W, U)
        out = np.zeros((n, c["n_q_heads"], c["head_dim"]))
        rows = np.zeros((n, c["n_q_heads"]))
        sels, sigmas, counts = [], [], []
        for hk in range(c["n_kv_heads"]):
            qg = self.q[c0:c0 + n, hk * G:(hk + 1) * G]
            if nm > 0 and k > 0:
                if c.get("unit_repr", "reps") == "meankey":
                    rk = np.stack([unit_mean_key(self.k[S + j * U:S + (j + 1) * U, hk], c["dtype"])[None]
                                   for j in range(nm)])
                else:
                    rk = np.stack([self.k[[S + j * U + m for m in self.reps[j][hk]], hk] for j in range(nm)])
                sigma = unit_scores(qg, rk, W, c["rope_base"])
                sel = topk_stable(sigma, min(k, nm))
            else:
                sigma, sel = np.zeros(nm), []
            sels.append(sel)
            sigmas.append(sigma)
            use = sel if sel_override is None else sel_override[hk]
            o, rs, keys, valid = attend_group(qg, c0, use, lambda idx, h=hk: self.k[idx, h],
                                              lambda idx, h=hk: self.v[idx, h], c)
            out[:, hk * G:(hk + 1) * G] = o
            rows[:, hk * G:(hk + 1) * G] = rs
            counts.append(valid.sum(axis=1))
        self.last = dict(sel=sels, sigma=sigmas, row_sums=rows, key_counts=np.stack(counts), n_mem=nm,
                         B=window_base(c0, S, W, U))
        return out


# --------------------------------------------------------------------------------------------
# stateless recomputation of one chunk from the full prefix (large streams)


def query_prefix_sums(qsrc: Callable, c0: int, positions: Sequence[int], cfg: dict, block: int = 4096):
    """P(p) = sum_{i<p} sum_{h in group} R(i) q_{i,h} for each requested p <= c0, per kv head.

    qsrc(t0, n) -> float64 [n, Hq, d].  Returns dict p -> [Hkv, d].
    """
    Hq, Hkv, d, base = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"], cfg["rope_base"]
    G = Hq // Hkv
    want = sorted(set(int(p) for p in positions))
    out = {}
    acc = np.zeros((Hkv, d))
    wi = 0
    while wi < len(want) and want[wi] == 0:
        out[0] = acc.copy()
        wi += 1
    t0 = 0
    stop = max(want) if want else 0
    while t0 < stop:
        n = min(block, stop - t0)
        q = qsrc(t0, n).reshape(n, Hkv, G, d)
        # sum_h R(i) q_{i,h} = R(i) sum_h q_{i,h}: every head of token i has the same angle
        qr = rope(q.sum(axis=2), (t0 + np.arange(n))[:, None], base)  # [n, Hkv, d]
        cs = np.cumsum(qr, axis=0) + acc[None]
        while wi < len(want) and want[wi] <= t0 + n:
            out[want[wi]] = cs[want[wi] - t0 - 1].copy()
            wi += 1
        acc = cs[-1].copy()
        t0 += n
    return out


def all_reps_linear(qsrc: Callable, ksrc: Callable, c0: int, cfg: dict):
    """Representatives of every unit eligible at c0, by the summed-query form.

    ksrc(t0, n) -> float64 [n, Hkv, d].  Returns (reps [n_units][Hkv] rank-ordered lists,
    rho [n_units, Hkv, U]).
    """
    S, W, U, r, base = cfg["n_sink"], cfg["window"], cfg["unit_size"], cfg["n_reps"], cfg["rope_base"]
    nm = n_mem(c0, S, W, U)
    ends = [S + (j + 1) * U for j in range(nm)]
    P = query_prefix_sums(qsrc, c0, ends + [e + W for e in ends], cfg)
    reps, rhos = [], []
    kbatch, kb0 = None, 0
    for j, e in enumerate(ends):
        if kbatch is None or j >= kb0 + kbatch.shape[0] // U:  # fetch keys 256 units at a time
            kb0 = j
            kbatch = ksrc(S + j * U, min(256, nm - j) * U)
        ku = kbatch[(j - kb0) * U:(j - kb0 + 1) * U]  # [U, Hkv, d]
        per, rr = [], []
        for hk in range(cfg["n_kv_heads"]):
            rho = rep_scores_linear(P[e + W][hk] - P[e][hk], ku[:, hk], S + j * U, base)
            rr.append(rho)
            per.append(select_reps(rho, r))
        reps.append(per)
        rhos.append(np.stack(rr))
    return reps, (np.stack(rhos) if rhos else np.zeros((0, cfg["n_kv_heads"], U)))


def rep_key_table(ksrc: Callable, reps, n_units: int, cfg: dict) -> np.ndarray:
    """Raw keys of every unit's representatives: [Hkv, n_units, n_reps, d] (keys fetched 256 units at a time)."""
    S, U, Hkv, d = cfg["n_sink"], cfg["unit_size"], cfg["n_kv_heads"], cfg["head_dim"]
    out = np.zeros((Hkv, n_units, cfg["n_reps"], d))
    for j0 in range(0, n_units, 256):
        nb = min(256, n_units - j0)
        kb = ksrc(S + j0 * U, nb * U)
        for j in range(j0, j0 + nb):
            ku = kb[(j - j0) * U:(j - j0 + 1) * U]
            for hk in range(Hkv):
                out[hk, j] = ku[reps[j][hk], hk]
    return out


def chunk_stateless(qsrc: Callable, ksrc: Callable, vsrc: Callable, c0: int, n: int, cfg: dict,
                    reps=None, sel_override=None, rep_keys=None):
    """Recompute chunk [c0, c0+n) from scratch: reps of all eligible units, lookup, attention.

    `reps` may be passed in (e.g. the GPU's own representatives, to check the later steps on
    them); `sel_override` likewise for the selection; `rep_keys` [Hkv, n_units, r, d] the units'
    scoring vectors.  cfg["unit_repr"] = "meankey" scores by mean keys.  Returns (out [n, Hq, d],
    info dict).
    """
    S, W, U, k, base = cfg["n_sink"], cfg["window"], cfg["unit_size"], cfg["top_k"], cfg["rope_base"]
    Hq, Hkv, d = cfg["n_q_heads"], cfg["n_kv_heads"], cfg["head_dim"]
    G = Hq // Hkv
    nm = n_mem(c0, S, W, U)
    rhos = None
    if reps is None:
        reps, rhos = all_reps_linear(qsrc, ksrc, c0, cfg)
    q = qsrc(c0, n)
    out = np.zeros((n, Hq, d))
    rows = np.zeros((n, Hq))
    sels, sigmas = [], []
    cache = {}

    def kv_rows(idx, hk, which):
        idx = np.asarray(idx, dtype=np.int64)
        res = np.empty((len(idx), d))
        # fetch contiguous runs
        if len(idx):
            brk = np.flatnonzero(np.diff(idx) != 1) + 1
            for seg in np.split(np.arange(len(idx)), brk):
                a = int(idx[seg[0]])
                key = (which, a, len(seg))
                if key not in cache:
                    cache[key] = (ksrc if which == "k" else vsrc)(a, len(seg))
                res[seg] = cache[key][:, hk]
        return res

    if k > 0 and rep_keys is None:
        if cfg.get("unit_repr", "reps") == "meankey":
            rep_keys = mean_key_table(ksrc, nm, cfg)[:, :, None, :]  # one vector per unit
        else:
            rep_keys = rep_key_table(ksrc, reps, nm, cfg)  # raw keys of every unit's representatives
    elif rep_keys is not None:
        rep_keys = rep_keys[:, :nm]
    for hk in range(Hkv):
        qg = q[:, hk * G:(hk + 1) * G]
        if nm > 0 and k > 0:
            sigma = unit_scores(qg, rep_keys[hk], W, base)
            sel = topk_stable(sigma, min(k, nm))
        else:
            sigma, sel = np.zeros(nm), []
        sels.append(sel)
        sigmas.append(sigma)
        use = sel if sel_override is None else sel_override[hk]
        o, rs, _, _ = attend_group(qg, c0, use, lambda idx, h=hk: kv_rows(idx, h, "k"),
                                   lambda idx, h=hk: kv_rows(idx, h, "v"), cfg)
        out[:, hk * G:(hk + 1) * G] = o
        rows[:, hk * G:(hk + 1) * G] = rs
    return out, dict(sel=sels, sigma=sigmas, reps=reps, rho=rhos, row_sums=rows, n_mem=nm,
                     B=window_base(c0, S, W, U))
