"""pa_decode_static: decode for callers that cannot allocate device memory.

Some callers of this library may not call cudaMalloc: a plugin inside a host
that owns every device allocation, code with a memory budget fixed up front,
or a latency-critical path where an allocation (which may synchronise the
device) is not acceptable.  pa_decode_static runs the same decode with the
workspace in a fixed array the library keeps in device memory.  These tests
call it through the C ABI and compare it with pa_decode (caller workspace) on
the same inputs, two calls in a row, and check that a request larger than the
fixed array is refused before anything is launched.

This file is collected last on purpose (pytest orders files by name), so a
failure here never hides the results of the other tests.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.harness import CudaPathRun, check_close, out_f64

pytestmark = pytest.mark.gpu
pa = pytest.importorskip("paged_kv_cache_426_b200")


def _static_call(out, q, kc, vc, tab, lens, max_len, scale, P, err):
    """Straight through the C ABI (no Python wrapper logic)."""
    S, hq, d = q.shape
    NB, hkv, bs, _ = kc.shape
    return pa.lib.pa_decode_static(
        C.c_void_p(out.data_ptr()), C.c_void_p(q.data_ptr()), C.c_void_p(kc.data_ptr()),
        C.c_void_p(vc.data_ptr()), C.c_void_p(tab.data_ptr()), tab.shape[1],
        C.c_void_p(lens.data_ptr()), max_len, S, hq, hkv, d, bs, NB, C.c_float(scale), P,
        pa.pa_dtype(q), C.c_void_p(err.data_ptr()),
        C.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("name,P", [("mha", 512), ("gqa", 64)])
def test_static_matches_workspace_two_calls(name, P):
    if name == "mha":
        w = workloads.mha7b_f16(steps=2, num_seqs=8)
    else:
        w = workloads.gqa8b_bf16(num_seqs=12, steps=2)
    rec = oracle.run(w, keep_prefill_cache=True)
    g = CudaPathRun(w, rec, partition_size=P)
    g.replay_prefill()
    for k in range(2):                       # two calls in a row, on successive steps
        ref_out = g.step(k)                  # pa_decode with a caller workspace
        st = rec.steps[k]
        q = w.step_q[k].cuda()
        out = torch.full_like(q, float("nan"))
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        status = _static_call(out, q, g.kc, g.vc, torch.from_numpy(st.block_tables).cuda(),
                              torch.from_numpy(st.context_lens).cuda(), g.max_len, w.scale, P,
                              err)
        torch.cuda.synchronize()
        assert status == pa.PA_OK, pa.lib.pa_status_string(status)
        assert err.item() == 0
        check_close(out_f64(out, w.dtype), out_f64(ref_out, w.dtype), w.dtype,
                    f"{w.name} step {k}: static vs caller workspace")
        check_close(out_f64(out, w.dtype), st.out, w.dtype, f"{w.name} step {k}: static vs oracle")


def test_static_rejects_oversize_workspace():
    need = pa.pa_decode_workspace_size(256, 32, 8, 128, 131072, 512)
    assert need > pa.PA_DECODE_STATIC_WORKSPACE_BYTES
    q = torch.zeros(256, 32, 128, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(4, 8, 16, 128, dtype=torch.bfloat16, device="cuda")
    tab = torch.zeros(256, 8192, dtype=torch.int32, device="cuda")
    lens = torch.zeros(256, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros_like(q)
    status = _static_call(out, q, kc, kc, tab, lens, 131072, 0.1, 512, err)
    assert status == pa.PA_ERR_INVALID
    torch.cuda.synchronize()
    assert not out.any() and err.item() == 0
