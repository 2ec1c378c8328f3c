"""Workload definitions and per-chunk input recipes.

Each workload is one attention layer's token stream, shaped like the
layers the InfLLM pages evaluate (Mistral-7B: 32 q / 8 kv heads, d=128,
RoPE base 1e6; Llama-3-8B: same heads, base 5e5), with seeded synthetic
values in place of the pages' datasets (no dataset or trained weight is
used anywhere).

Recipe (all values are float32 normals from the counter-based generator,
rounded to the workload dtype):
  q[t,h,:] = z(seed, Q, ...)                       ~ N(0, 1)
  k[t,h,:] = z(seed, K, ...) + b[h,:]              b = sqrt(k_bias_var) * z(seed, KBIAS, h*d + i)
  v[t,h,:] = z(seed, V, ...)                       ~ N(0, 1)
Planted needle (``needle=True``): one unit j* (seeded) gets, on every KV
head h, keys at cosine 0.9 to a seeded unit direction u_h, scaled to norm
sqrt(d); the last ``needle_queries`` queries of every q head of group h are
sqrt(d) * R(-window) u_h, so that in the frame in which memory units are
scored (query rotated by the window length, key unrotated) they point along
u_h.  The rotation here is input construction only (a plain rotate-half
rotation by -window * theta_i), written independently of the oracle.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

T_Q, T_K, T_V, T_KBIAS, T_NEEDLE_U, T_NEEDLE_W, T_NEEDLE_POS = 1, 2, 3, 4, 5, 6, 7


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    n_sink: int
    window: int
    unit_size: int
    n_reps: int
    top_k: int
    chunk: int
    n_tokens: int
    rope_base: float
    dtype: str  # "f32" | "bf16"
    seed: int
    k_bias_var: float = 0.0
    needle: bool = False
    needle_queries: int = 64
    decode_steps: int = 0  # >0: tokens [n_tokens, n_tokens+decode_steps) are decoded one at a time
    build_chunk: int = 0  # chunk size used to build the memory before decoding

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def total_tokens(self) -> int:
        return self.n_tokens + self.decode_steps

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def as_config(self) -> dict:
        return dict(n_q_heads=self.n_q_heads, n_kv_heads=self.n_kv_heads, head_dim=self.head_dim,
                    n_sink=self.n_sink, window=self.window, unit_size=self.unit_size, n_reps=self.n_reps,
                    top_k=self.top_k, rope_base=self.rope_base, dtype=self.dtype)


# The five configurations the layer is specified on.
WORKLOADS = {
    # tiny fp32 stream, seed 0
    "tiny_f32": Workload("tiny_f32", 1, 1, 64, 16, 512, 128, 4, 4, 128, 4096, 1e4, "f32", seed=0),
    # Mistral-7B-shaped layer, 128K tokens in 512-token chunks, K channel bias N(0, 4)
    "mistral_128k": Workload("mistral_128k", 32, 8, 128, 128, 4096, 128, 4, 16, 512, 131072, 1e6, "bf16",
                             seed=1, k_bias_var=4.0),
    # Llama-3-8B-shaped layer, 128K tokens, window 8192, top-k 32
    "llama3_128k": Workload("llama3_128k", 32, 8, 128, 128, 8192, 128, 4, 32, 512, 131072, 5e5, "bf16",
                            seed=2, k_bias_var=4.0),
    # decode: 8192 memory units (1M tokens) + 128 sinks + 4096 window built first, then 256 single-token steps
    "decode_1m": Workload("decode_1m", 32, 8, 128, 128, 4096, 128, 4, 16, 1, 128 + 8192 * 128 + 4096, 1e6,
                          "bf16", seed=3, decode_steps=256, build_chunk=4096),
    # planted needle, 256K tokens
    "needle_256k": Workload("needle_256k", 32, 8, 128, 128, 4096, 128, 4, 16, 512, 262144, 1e6, "bf16",
                            seed=4, needle=True),
}

# Smaller cases the oracle runs end to end in seconds (several tiles, ragged tails, edge cases).
SMALL = {
    "small_gqa": Workload("small_gqa", 8, 2, 128, 20, 512, 64, 4, 4, 200, 2900, 1e4, "bf16", seed=11,
                          k_bias_var=4.0),
    "small_g4": Workload("small_g4", 16, 4, 128, 128, 1024, 128, 4, 8, 256, 4500, 1e6, "bf16", seed=12,
                         k_bias_var=4.0),
    "small_d64": Workload("small_d64", 4, 2, 64, 16, 256, 128, 4, 3, 160, 2000, 1e4, "bf16", seed=13),
    "small_u256": Workload("small_u256", 8, 2, 128, 8, 512, 256, 8, 2, 300, 3300, 1e4, "bf16", seed=14),
    "small_nosink": Workload("small_nosink", 4, 1, 128, 0, 256, 128, 4, 2, 128, 1800, 1e4, "bf16", seed=15),
    "small_streaming": Workload("small_streaming", 4, 4, 64, 4, 256, 64, 4, 0, 100, 1500, 1e4, "bf16", seed=16),
    "small_allunits": Workload("small_allunits", 4, 2, 64, 4, 256, 64, 4, 64, 128, 1600, 1e4, "bf16", seed=17),
    "small_f32": Workload("small_f32", 4, 2, 64, 16, 256, 64, 4, 4, 96, 1400, 1e4, "f32", seed=18),
    "small_needle": Workload("small_needle", 8, 2, 128, 16, 512, 128, 4, 4, 256, 8192, 1e6, "bf16", seed=19,
                             needle=True),
    "small_decode": Workload("small_decode", 8, 2, 128, 16, 512, 64, 4, 4, 1, 2048, 1e4, "bf16", seed=20,
                             decode_steps=200, build_chunk=512),
    # eight q heads per KV head: 16 queries per packed 128-row tile (smallest tensor-core tile)
    "small_g8": Workload("small_g8", 16, 2, 128, 32, 512, 128, 4, 4, 256, 2600, 1e6, "bf16", seed=21,
                         k_bias_var=4.0),
    # two q heads per KV head: 64 queries per packed tile; chunks of 2.5 tiles
    "small_g2": Workload("small_g2", 4, 2, 128, 64, 256, 64, 4, 3, 160, 2000, 1e4, "bf16", seed=23,
                         k_bias_var=4.0),
    "small_decode_g8": Workload("small_decode_g8", 16, 2, 128, 16, 512, 64, 4, 4, 1, 2048, 1e6, "bf16", seed=22,
                                decode_steps=64, build_chunk=512),
}

ALL = {**WORKLOADS, **SMALL}


def chunk_bounds(w: Workload):
    """Chunk start/length pairs for the prefill stream (the last chunk may be ragged)."""
    out = []
    t = 0
    while t < w.n_tokens:
        n = min(w.chunk, w.n_tokens - t)
        out.append((t, n))
        t += n
    return out


def _n_mem(c0: int, w: Workload) -> int:
    x = c0 - w.window - w.n_sink
    return max(0, x // w.unit_size) if x > 0 else 0


def _k_bias(w: Workload) -> np.ndarray | None:
    from . import normal_flat
    if w.k_bias_var <= 0:
        return None
    z = normal_flat(w.seed, T_KBIAS, 0, w.n_kv_heads * w.head_dim).reshape(w.n_kv_heads, w.head_dim)
    return (np.float32(math.sqrt(w.k_bias_var)) * z).astype(np.float32)


def needle_info(w: Workload):
    """(j_star, unit token range, directions u [Hkv, d] float64) for a needle workload, else None."""
    from . import normal_flat, philox4x32_10
    if not w.needle:
        return None
    last_c0 = chunk_bounds(w)[-1][0]
    n_units = _n_mem(last_c0, w)
    assert n_units > 0
    r = philox4x32_10([0, 0, T_NEEDLE_POS, 0], [w.seed & 0xFFFFFFFF, w.seed >> 32])
    j_star = int(r[0]) % n_units
    t_lo = w.n_sink + j_star * w.unit_size
    u = normal_flat(w.seed, T_NEEDLE_U, 0, w.n_kv_heads * w.head_dim).astype(np.float64)
    u = u.reshape(w.n_kv_heads, w.head_dim)
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    return j_star, (t_lo, t_lo + w.unit_size), u


def _rotate_half_by(x: np.ndarray, p: float, base: float) -> np.ndarray:
    d = x.shape[-1]
    half = d // 2
    theta = base ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    c, s = np.cos(p * theta), np.sin(p * theta)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def _store(x64: np.ndarray, dtype: str) -> np.ndarray:
    from . import round_bf16
    x32 = x64.astype(np.float32)
    return x32 if dtype == "f32" else round_bf16(x32)


def gen_chunk(w: Workload, t0: int, n: int, parts: str = "qkv"):
    """(q, k, v) for tokens [t0, t0+n): q [n,Hq,d], k/v [n,Hkv,d] (float32 or bf16 bits).

    `parts` selects which tensors to generate; the others are returned as None.
    """
    from . import normal
    d, Hq, Hkv = w.head_dim, w.n_q_heads, w.n_kv_heads
    q = normal(w.seed, T_Q, t0, n, Hq, d, dtype=w.dtype) if "q" in parts else None
    k = normal(w.seed, T_K, t0, n, Hkv, d, dtype=w.dtype, bias=_k_bias(w)) if "k" in parts else None
    v = normal(w.seed, T_V, t0, n, Hkv, d, dtype=w.dtype) if "v" in parts else None
    info = needle_info(w)
    if info is not None:
        _, (a, b), u = info
        sd = math.sqrt(d)
        lo, hi = max(a, t0), min(b, t0 + n)
        if lo < hi and k is not None:  # needle keys
            wz = normal(w.seed, T_NEEDLE_W, lo, hi - lo, Hkv, d, dtype="f32").astype(np.float64)
            wz -= np.sum(wz * u[None], axis=-1, keepdims=True) * u[None]
            wz /= np.linalg.norm(wz, axis=-1, keepdims=True)
            kn = sd * (0.9 * u[None] + math.sqrt(0.19) * wz)
            k[lo - t0:hi - t0] = _store(kn, w.dtype)
        qa = w.n_tokens - w.needle_queries
        lo, hi = max(qa, t0), min(w.n_tokens, t0 + n)
        if lo < hi and q is not None:  # needle queries
            qv = sd * _rotate_half_by(u, -float(w.window), w.rope_base)  # [Hkv, d]
            qv = np.repeat(qv, w.group, axis=0)  # q head h uses kv head h // group
            q[lo - t0:hi - t0] = _store(np.broadcast_to(qv, (hi - lo, Hq, d)), w.dtype)
    return q, k, v
