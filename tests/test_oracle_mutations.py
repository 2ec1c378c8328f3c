"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a COPY of the oracle (a dropped term, a wrong sign, an
off-by-one position or index, a reversed tie rule, a transposed operand...), then runs the pin
suite against the copy in a subprocess and expects it to fail.  The repository's oracle is never
modified.  CPU only.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# name -> (text in oracle/infllm_oracle.py, replacement)
MUTATIONS = {
    "rope_sign": ("x2 * c + x1 * s], axis=-1)", "x2 * c - x1 * s], axis=-1)"),
    "rep_scale_dropped": ("return rho / math.sqrt(d)", "return rho"),
    "rep_query_position": ("qi = rope(q_win[i, h], e + i, base)", "qi = rope(q_win[i, h], e + i + 1, base)"),
    "unit_distance": ("qr = rope(q_chunk, float(window), base)", "qr = rope(q_chunk, float(window) + 1, base)"),
    "unit_scale_dropped": ('"thd,jmd->j", qr, rep_keys, optimize=True) / math.sqrt(d)',
                           '"thd,jmd->j", qr, rep_keys, optimize=True)'),
    "window_frame": ("q_win = rope(q, (t - B)[:, None], base)", "q_win = rope(q, (t - B + 1)[:, None], base)"),
    "window_drops_first_key": ("win_idx = np.arange(B, c0 + n)", "win_idx = np.arange(B + 1, c0 + n)"),
    "tie_to_higher_index": ("key=lambda i: (-float(scores[i]), i))", "key=lambda i: (-float(scores[i]), -i))"),
    "n_mem_off_by_one": ("return x // unit if x > 0 else 0", "return (x + 1) // unit if x > 0 else 0"),
    "sinks_not_causal": ("valid[:, :len(sink_idx)] = sink_idx[None, :] <= t[:, None]",
                         "valid[:, :len(sink_idx)] = True"),
    "softmax_not_normalised": ("p /= p.sum(axis=-1, keepdims=True)", "p /= 1.0"),
    "prefix_sum_position": ("qr = rope(q.sum(axis=2), (t0 + np.arange(n))[:, None], base)",
                            "qr = rope(q.sum(axis=2), (t0 + np.arange(n) + 1)[:, None], base)"),
    "key_batch_not_refetched": ("if kbatch is None or j >= kb0 + kbatch.shape[0] // U:", "if kbatch is None:"),
    "gqa_groups_transposed": ("qg = self.q[c0:c0 + n, hk * G:(hk + 1) * G]",
                              "qg = self.q[c0:c0 + n, hk::self.cfg['n_kv_heads']]"),
    "mean_key_is_sum": ("return round_to_dtype(k_unit.sum(axis=0) / k_unit.shape[0], dtype)",
                        "return round_to_dtype(k_unit.sum(axis=0), dtype)"),
    "bf16_keeps_nine_bits": ("np.rint(m * 256.0) / 256.0", "np.rint(m * 512.0) / 512.0"),
}


def _stage(tmp):
    for d in ("oracle", "synth", "tests"):
        shutil.copytree(os.path.join(ROOT, d), os.path.join(tmp, d),
                        ignore=shutil.ignore_patterns("__pycache__", "test_oracle_mutations.py"))


def _run_pins(tmp):
    env = dict(os.environ, PYTHONPATH=tmp, PYTHONDONTWRITEBYTECODE="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-x", "-q", "-p",
                        "no:cacheprovider"], cwd=tmp, env=env, capture_output=True, text=True, timeout=600)
    return r.returncode, (r.stdout.strip().splitlines() or [""])[-1]


def test_unmutated_copy_passes(tmp_path):
    _stage(str(tmp_path))
    rc, last = _run_pins(str(tmp_path))
    assert rc == 0, last


def test_every_planted_mistake_fails_a_pin(tmp_path):
    src = open(os.path.join(ROOT, "oracle", "infllm_oracle.py")).read()
    dirs = {}
    for name, (a, b) in MUTATIONS.items():
        assert src.count(a) == 1, f"{name}: anchor text not found once in the oracle"
        d = str(tmp_path / name)
        _stage(d)
        with open(os.path.join(d, "oracle", "infllm_oracle.py"), "w") as f:
            f.write(src.replace(a, b))
        dirs[name] = d
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = dict(zip(dirs, ex.map(_run_pins, dirs.values())))
    missed = {n: last for n, (rc, last) in results.items() if rc == 0}
    assert not missed, f"mistakes no pin caught: {missed}"
