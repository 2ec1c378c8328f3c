"""The C-ABI library loads and exports every entry point include/infllm.h declares; host-side
argument checks (no GPU needed: nothing here launches or allocates on a device)."""
from __future__ import annotations

import ctypes
import os
import re
import subprocess

import pytest

import block_memory_sparse_b200 as bms

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include")) if f.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    from block_memory_sparse_b200 import build
    build.build()
    return bms.load_library()


def declared_functions():
    names = set()
    for h in HEADERS:
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(infllm_\w+)\s*\(", src))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 13
    out = subprocess.run(["nm", "-D", "--defined-only", bms.library_path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)", out))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(lib, n)
    assert set(bms.SIGNATURES) >= set(names)


def test_struct_layouts_match_header(tmp_path):
    prog = tmp_path / "layout.c"
    prog.write_text("""
#include <stdio.h>
#include <stddef.h>
#include "infllm.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu\\n", sizeof(infllm_config), offsetof(infllm_config, max_tokens),
         offsetof(infllm_config, rope_base), offsetof(infllm_config, score_mode), sizeof(infllm_stats),
         offsetof(infllm_stats, n_decode));
  return 0;
}
""")
    exe = tmp_path / "layout"
    subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), str(prog), "-o", str(exe)])
    got = [int(x) for x in subprocess.check_output([str(exe)]).split()]
    want = [ctypes.sizeof(bms.Config), bms.Config.max_tokens.offset, bms.Config.rope_base.offset,
            bms.Config.score_mode.offset, ctypes.sizeof(bms.Stats), bms.Stats.n_decode.offset]
    assert got == want


def _cfg(**kw):
    c = dict(n_q_heads=32, n_kv_heads=8, head_dim=128, n_sink=128, window=4096, unit_size=128, n_reps=4, top_k=16,
             max_chunk=512, max_tokens=131072, rope_base=1e6, dtype=1, score_mode=0)
    c.update(kw)
    return bms.Config(**c)


@pytest.mark.parametrize("bad", [
    dict(n_q_heads=0), dict(n_q_heads=30), dict(head_dim=96), dict(n_sink=-1), dict(window=0),
    dict(unit_size=0), dict(unit_size=2048), dict(n_reps=0), dict(n_reps=33), dict(n_reps=200, unit_size=128),
    dict(top_k=-1), dict(max_chunk=0), dict(max_tokens=0), dict(rope_base=1.0), dict(dtype=7), dict(score_mode=3),
    dict(top_k=64, max_tokens=1 << 22), dict(max_tokens=(1 << 21) + 128 * 16384),
])
def test_invalid_configs_are_rejected_before_any_device_work(lib, bad):
    h = ctypes.c_void_p(123)
    st = lib.infllm_create(ctypes.byref(_cfg(**bad)), None, ctypes.byref(h))
    assert st == 1  # INFLLM_EINVAL
    assert h.value is None


def test_null_arguments(lib):
    assert lib.infllm_create(None, None, None) == 1
    assert lib.infllm_destroy(None) == 0
    assert lib.infllm_append_chunk(None, None, None, None, 1) == 1
    assert lib.infllm_attend_chunk(None, None, 1, None) == 1
    assert lib.infllm_decode_step(None, None, None, None, None) == 1
    assert lib.infllm_prefill(None, None, None, None, 0, 1, None) == 1
    assert lib.infllm_set_launch_chaining(None, 1) == 1
    assert lib.infllm_set_prefill_lookup(None, 0) == 1
    assert lib.infllm_get_selection(None, None) == 1
    assert lib.infllm_get_stats(None, None) == 1
    assert lib.infllm_last_error(None) == b"null context"
    assert lib.infllm_version().startswith(b"infllm-b200")


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(ImportError):
        bms.load_library(str(tmp_path / "nope.so"))
