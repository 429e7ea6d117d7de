"""The decode benchmark's launch count per call (its `gpu_launches` claim),
on CPU: the library's rules are one decode kernel; a merge kernel unless the
splits are merged inside the decode (tensor-core engine, at most 4
partitions) or there is one partition; and, with the step's cache write on
the CUDA-core engine, a write launch before it.  The calls themselves are
stubbed; only the count is checked."""
import os
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def fake_session(dtype, engine, P, max_len):
    s = bench.Session.__new__(bench.Session)
    s.pa = types.SimpleNamespace(pa_decode=lambda *a, **k: None)
    s.w = types.SimpleNamespace(dtype=dtype, scale=1.0)
    s.engine = engine
    s.P = P
    s.max_len = max_len
    s.kc = s.vc = s.ws = s.err = None
    return s


ST = {"q": None, "tab": None, "lens": None, "k": None, "v": None, "slots": None}


@pytest.mark.parametrize("dtype,engine,P,max_len,write,want", [
    ("f16", None, 1024, 2080, False, 1),     # 3 partitions: merged inside
    ("f16", None, 1024, 2080, True, 1),      # ... and the write inside
    ("bf16", None, 1024, 8200, True, 2),     # 9 partitions: merge kernel
    ("bf16", None, 0, 8200, True, 1),        # one partition per sequence
    ("f16", "core", 1024, 2080, False, 2),   # CUDA cores: merge kernel
    ("f16", "core", 1024, 2080, True, 3),    # ... and a write launch
    ("f32", None, 16, 40, True, 3),          # fp32 runs on CUDA cores
    ("f32", None, 0, 40, True, 2),
])
def test_decode_launch_count(dtype, engine, P, max_len, write, want):
    s = fake_session(dtype, engine, P, max_len)
    assert s.decode(ST, None, write=write) == want
