"""The C ABI without a GPU: the library loads, exports every function that
include/pa.h declares, rejects bad arguments before launching anything, and
its host block manager reproduces the oracle's block tables, slot mappings and
copy-on-write pairs bit for bit on every workload script."""
import ctypes as C
import os
import re

import numpy as np
import pytest
import torch

import oracle
import workloads

pa = pytest.importorskip("paged_kv_cache_426_b200")

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "pa.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) >= 20
    lib = C.CDLL(pa.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing
    assert set(names) == set(pa.SIGNATURES), "binding and header disagree"


def test_status_strings_and_version():
    assert pa.lib.pa_status_string(pa.PA_ERR_OOM) == b"PA_ERR_OOM"
    assert pa.lib.pa_version() >= 200


def test_bad_arguments_rejected_before_launch():
    L = pa.lib
    # null pointers
    assert L.pa_reshape_and_cache(None, None, None, None, None, 4, 2, 128, 16, 8, 1, None, None) == pa.PA_ERR_INVALID
    assert L.pa_decode(None, None, None, None, None, 4, None, 64, 2, 4, 2, 128, 16, 8, 1.0, 0,
                       None, 0, 1, None, None) == pa.PA_ERR_INVALID
    assert L.pa_copy_blocks(None, None, None, 3, 2, 128, 16, 8, 1, None, None) == pa.PA_ERR_INVALID
    # unsupported shapes
    assert L.pa_reshape_and_cache(None, None, None, None, None, 4, 2, 96, 16, 8, 1, None, None) == pa.PA_ERR_UNSUPPORTED
    assert L.pa_copy_blocks(None, None, None, 3, 2, 128, 12, 8, 1, None, None) == pa.PA_ERR_UNSUPPORTED
    fake = 1 << 20   # never dereferenced: validation fails first
    assert L.pa_decode(fake, fake, fake, fake, fake, 4, fake, 64, 2, 4, 2, 96, 16, 8, 1.0, 0,
                       fake, 1 << 20, 1, None, None) == pa.PA_ERR_UNSUPPORTED
    # group not dividing, partition not a multiple of 16, bad dtype, short workspace
    assert L.pa_decode(fake, fake, fake, fake, fake, 4, fake, 64, 2, 6, 4, 128, 16, 8, 1.0, 0,
                       fake, 1 << 20, 1, None, None) == pa.PA_ERR_INVALID
    assert L.pa_decode(fake, fake, fake, fake, fake, 4, fake, 64, 2, 4, 2, 128, 16, 8, 1.0, 24,
                       fake, 1 << 20, 1, None, None) == pa.PA_ERR_INVALID
    assert L.pa_decode(fake, fake, fake, fake, fake, 4, fake, 64, 2, 4, 2, 128, 16, 8, 1.0, 0,
                       fake, 1 << 20, 7, None, None) == pa.PA_ERR_INVALID
    assert L.pa_decode(fake, fake, fake, fake, fake, 4, fake, 4096, 2, 4, 2, 128, 16, 8, 1.0, 16,
                       fake, 300, 1, None, None) == pa.PA_ERR_INVALID
    # empty work is a no-op
    assert L.pa_reshape_and_cache(None, None, None, None, None, 0, 2, 128, 16, 8, 1, None, None) == pa.PA_OK
    assert L.pa_copy_blocks(None, None, None, 0, 2, 128, 16, 8, 1, None, None) == pa.PA_OK


def test_decode_options_are_per_call():
    """Engine choice and the failure-detection aid are per-call options of
    pa_decode_ex; the library keeps no process-wide switch for either."""
    lib = C.CDLL(pa.LIB_PATH)
    assert not hasattr(lib, "pa_set_decode_engine")
    assert not hasattr(lib, "pa_test_withhold_stage")
    L = pa.lib
    f = 1 << 20                          # aligned, never dereferenced: validation fails first

    def call(opts):
        return L.pa_decode_ex(f, f, f, f, f, 4, f, 64, 2, 4, 2, 96, 16, 8, 1.0, 0, f, 1 << 20, 1,
                              None, None, C.byref(opts) if opts is not None else None)

    size = C.sizeof(pa.pa_decode_options)
    # valid options: the call proceeds to the argument checks (head_dim 96 unsupported)
    assert call(None) == pa.PA_ERR_UNSUPPORTED
    assert call(pa.pa_decode_options(size, pa.PA_ENGINE_TENSOR, -1)) == pa.PA_ERR_UNSUPPORTED
    assert call(pa.pa_decode_options(size, pa.PA_ENGINE_CUDA_CORE, 3)) == pa.PA_ERR_UNSUPPORTED
    # a caller built against the first three fields only: the rest read as unset
    assert call(pa.pa_decode_options(12, 0, -1, 1, 2, 3)) == pa.PA_ERR_UNSUPPORTED
    # the step's cache write: all three pointers, 16-B aligned rows, 8-B aligned slots
    g = 1 << 21
    assert call(pa.pa_decode_options(size, 0, -1, f, g, f)) == pa.PA_ERR_UNSUPPORTED
    # bad options are rejected first
    assert call(pa.pa_decode_options(8, 0, -1)) == pa.PA_ERR_INVALID
    assert call(pa.pa_decode_options(size, 3, -1)) == pa.PA_ERR_INVALID
    assert call(pa.pa_decode_options(size, -1, -1)) == pa.PA_ERR_INVALID
    assert call(pa.pa_decode_options(size, 0, -2)) == pa.PA_ERR_INVALID
    assert call(pa.pa_decode_options(size, 0, -1, f, None, f)) == pa.PA_ERR_INVALID
    assert call(pa.pa_decode_options(size, 0, -1, None, None, f)) == pa.PA_ERR_INVALID
    assert call(pa.pa_decode_options(size, 0, -1, f + 8, g, f)) == pa.PA_ERR_INVALID
    assert call(pa.pa_decode_options(size, 0, -1, f, g, f + 4)) == pa.PA_ERR_INVALID


def test_static_decode_checks_arguments_before_the_device():
    """pa_decode_static runs every host check of pa_decode before it looks up
    or clears its fixed array, so a rejected call touches no device state."""
    L = pa.lib
    f = 1 << 20

    def call(hq=4, hkv=2, d=128, bs=16, P=0, dt=1, ptr=f, max_len=64, S=2):
        return L.pa_decode_static(ptr, f, f, f, f, 4, f, max_len, S, hq, hkv, d, bs, 8, 1.0, P,
                                  dt, None, None)

    assert call(S=0) == pa.PA_OK
    assert call(d=96) == pa.PA_ERR_UNSUPPORTED
    assert call(bs=24) == pa.PA_ERR_UNSUPPORTED
    assert call(hq=6, hkv=2) == pa.PA_ERR_UNSUPPORTED          # G = 3
    assert call(hq=7, hkv=2) == pa.PA_ERR_INVALID
    assert call(P=24) == pa.PA_ERR_INVALID
    assert call(dt=7) == pa.PA_ERR_INVALID
    assert call(ptr=None) == pa.PA_ERR_INVALID
    assert call(ptr=f + 8) == pa.PA_ERR_INVALID
    # larger than the fixed array
    assert L.pa_decode_static(f, f, f, f, f, 8192, f, 131072, 256, 32, 8, 128, 16, 8, 1.0, 512,
                              2, None, None) == pa.PA_ERR_INVALID


def test_prefill_bad_arguments_rejected_before_launch():
    """pa_prefill validates everything on the host before touching the
    device: arguments (args order: out, query, key_cache, value_cache,
    block_tables, max_blocks_per_seq, context_lens, cu_seqlens_q, num_seqs,
    total_q, max_query_len, Hq, Hkv, head_dim, block_size, num_blocks, scale,
    workspace, workspace_bytes, dtype, err_flag, stream)."""
    L = pa.lib
    f = 1 << 20                          # aligned, never dereferenced: validation fails first
    ok = dict(mbps=4, S=2, T=8, maxq=8, hq=8, hkv=2, d=128, bs=16, nb=8, scale=0.125, dt=2,
              ws=f, wsb=pa.PREFILL_WORKSPACE_BYTES)

    def call(ptr=f, **kw):
        a = dict(ok, **kw)
        return L.pa_prefill(ptr, f, f, f, f, a["mbps"], f, f, a["S"], a["T"], a["maxq"], a["hq"],
                            a["hkv"], a["d"], a["bs"], a["nb"], a["scale"], a["ws"], a["wsb"], a["dt"],
                            None, None)

    assert call(S=0) == pa.PA_OK and call(T=0) == pa.PA_OK         # nothing to do
    assert call(ptr=None) == pa.PA_ERR_INVALID
    assert call(ptr=f + 8) == pa.PA_ERR_INVALID                    # not 16-byte aligned
    assert call(dt=0) == pa.PA_ERR_UNSUPPORTED                     # fp32: no tensor-core path
    assert call(dt=7) == pa.PA_ERR_INVALID
    assert call(d=96) == pa.PA_ERR_UNSUPPORTED
    assert call(hq=6) == pa.PA_ERR_UNSUPPORTED                     # G = 3
    assert call(hq=7) == pa.PA_ERR_INVALID                         # not a multiple of Hkv
    assert call(bs=24) == pa.PA_ERR_UNSUPPORTED
    assert call(maxq=0) == pa.PA_ERR_INVALID
    assert call(scale=0.0) == pa.PA_ERR_INVALID and call(scale=-1.0) == pa.PA_ERR_INVALID
    assert call(scale=float("inf")) == pa.PA_ERR_INVALID
    assert call(nb=0) == pa.PA_ERR_INVALID and call(mbps=0) == pa.PA_ERR_INVALID
    assert call(ws=None) == pa.PA_ERR_INVALID                       # the item counter
    assert call(wsb=pa.PREFILL_WORKSPACE_BYTES - 4) == pa.PA_ERR_INVALID
    assert call(ws=f + 4) == pa.PA_ERR_INVALID                      # not 16-byte aligned


def test_workspace_size_formula():
    # the scheduler header only when nothing is split
    n0 = pa.pa_decode_workspace_size(64, 32, 32, 128, 2080, 0)
    assert n0 == 256
    # + a split counter per (sequence, KV head), (m, l) and the unnormalised
    # output of every partition of every head, each part rounded up to 256 bytes
    n1 = pa.pa_decode_workspace_size(64, 32, 32, 128, 2080, 512)
    n_p = 5
    assert n1 == 256 + 64 * 32 * 4 + 64 * 32 * n_p * 2 * 4 + 64 * 32 * n_p * 128 * 4
    n2 = pa.pa_decode_workspace_size(3, 8, 2, 64, 100, 16)
    r = lambda b: -(-b // 256) * 256
    assert n2 == 256 + r(3 * 2 * 4) + r(3 * 8 * 7 * 2 * 4) + 3 * 8 * 7 * 64 * 4


def test_allocator_errors():
    a = pa.BlockAllocator(3, [2, 0])
    assert a.refcount(1) == 1
    assert a.allocate_block() == 2 and a.allocate_block() == 0
    with pytest.raises(pa.PAError) as e:
        a.allocate_block()
    assert e.value.status == pa.PA_ERR_OOM
    a.free_block(2)
    with pytest.raises(pa.PAError) as e:
        a.free_block(2)
    assert e.value.status == pa.PA_ERR_STATE
    with pytest.raises(pa.PAError):
        pa.BlockAllocator(3, [1, 1])


def test_append_is_all_or_nothing():
    a = pa.BlockAllocator(3)
    m = pa.BlockManager(a, 4)
    m.add_seq(0)
    m.append(0, 10)                       # 3 blocks
    before = (m.seq_len(0), a.num_free())
    with pytest.raises(pa.PAError) as e:
        m.append(0, 3)                    # needs a 4th block at the 13th token
    assert e.value.status == pa.PA_ERR_OOM
    assert (m.seq_len(0), a.num_free()) == before
    m.add_seq(1)
    m.fork(0, 2)
    with pytest.raises(pa.PAError):
        m.append_step([0, 2, 1])          # 0 copies its shared last block: no free block
    assert m.seq_len(0) == 10 and m.seq_len(2) == 10 and m.seq_len(1) == 0
    assert [a.refcount(b) for b in range(3)] == [2, 2, 2]


def test_append_step_rejects_a_sequence_named_twice():
    """One token per sequence per step: a batch naming a sequence twice is
    rejected before anything is appended, and the next step still works."""
    a = pa.BlockAllocator(16)
    m = pa.BlockManager(a, 4)
    for s in range(3):
        m.add_seq(s)
    m.append_step([0, 1, 2])
    with pytest.raises(pa.PAError) as e:
        m.append_step([2, 0, 1, 0])
    assert e.value.status == pa.PA_ERR_INVALID
    assert [m.seq_len(s) for s in range(3)] == [1, 1, 1] and a.num_free() == 13
    slots, cow = m.append_step([1, 0, 2])
    assert [m.seq_len(s) for s in range(3)] == [2, 2, 2] and cow.shape[0] == 0
    assert slots.tolist() == [5, 1, 9]


def test_beam_sharing_example_matches_page():
    """velog 메모리 공유 example, through the C++ manager."""
    from tests.conftest import golden
    fx = golden("velog_beam_sharing.json")
    a = pa.BlockAllocator(fx["num_blocks"], fx["free_order"])
    m = pa.BlockManager(a, fx["block_size"])
    m.add_seq(0)
    m.append(0, fx["prompt_tokens"])
    m.fork(0, 1)
    _, c0 = m.append(0)
    _, c1 = m.append(1)
    tab, _ = m.block_tables([0, 1], 4)
    assert tab[0, :3].tolist() == fx["expect_tables"]["A"]
    assert tab[1, :3].tolist() == fx["expect_tables"]["B"]
    for b, rc in fx["expect_refcounts"].items():
        assert a.refcount(int(b)) == rc
    assert c0 == [] and c1 == []
    m.free_seq(0)
    m.free_seq(1)
    assert a.num_free() == fx["num_blocks"]


def _replay(w, steps=None):
    """C++ manager through the workload script; compare with the oracle's record."""
    rec = oracle.run(w, decode=False, steps=steps)
    a = pa.BlockAllocator(w.num_blocks, w.free_order)
    m = pa.BlockManager(a, w.block_size)
    mb = oracle.max_blocks_needed(w)
    k = 0
    for op in w.ops:
        if op[0] == "add":
            m.add_seq(op[1])
        elif op[0] == "fork":
            m.fork(op[1], op[2])
        elif op[0] == "write":
            slots, cow = m.append(op[1], w.kv["k" + op[2]].shape[0])
            assert np.array_equal(slots.numpy(), rec.prefill_slots[(op[1], op[2])])
        elif op[0] == "step":
            if k >= len(rec.steps):
                break
            st = rec.steps[k]
            slots, cow = m.append_step(op[1])
            assert np.array_equal(slots.numpy(), st.slot_mapping)
            assert [tuple(c) for c in cow.tolist()] == [tuple(c) for c in st.cow_pairs]
            tab, lens = m.block_tables(op[1], mb)
            assert np.array_equal(tab.numpy(), st.block_tables)
            assert np.array_equal(lens.numpy(), st.context_lens)
            k += 1
    for b in range(w.num_blocks):
        assert a.refcount(b) == rec.manager.alloc.refcount[b]
    assert a.num_free() == rec.manager.alloc.num_free()
    return m, a, rec


@pytest.mark.parametrize("name,kw", [
    ("tiny_f32", {}),
    ("mha7b_f16", dict(steps=32)),
    ("gqa8b_bf16_bs16", {}),
    ("gqa8b_bf16_bs32", {}),
    ("prefix_f16", {}),
    ("prefix_f16", dict(duplicate_prefix=True)),
])
def test_manager_matches_oracle(name, kw):
    w = workloads.make(name, **kw)
    m, a, rec = _replay(w)
    # every sequence freed -> all references back to the outside holders only
    for s in list(rec.manager.tables):
        m.free_seq(s)
    held = w.num_blocks - len(w.free_order)
    assert a.num_free() == w.num_blocks - held
