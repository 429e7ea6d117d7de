"""Paged prefill attention (pa_prefill, tcgen05) against the oracle.

Each batch is replayed twice from the same seeded inputs: through the oracle
(its own manager, cache writes and float64 causal attention) and through the
CUDA path (the library's manager, pa_reshape_and_cache, pa_prefill).  The
block tables must be identical; the outputs must agree within the 16-bit
tolerance (the kernel rounds P to the input type, accumulates in fp32 and
rounds the output).

Chunk shapes cover: a whole short prompt, a chunk inside a long context, a
multi-tile prompt with a ragged last query tile, a one-row chunk (a decode
step), an empty chunk, and a chunk whose key range ends inside a block.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.harness import TOL, GpuPrefill, check_close, out_f64

pa = pytest.importorskip("paged_kv_cache_426_b200")

pytestmark = pytest.mark.gpu

LENS = [5, 40, 150, 300, 129, 64, 1000, 77]
QLENS = [5, 17, 150, 1, 64, 0, 333, 77]

SHAPES = [   # dtype, hq, hkv, d, bs
    ("bf16", 8, 2, 128, 16),
    ("f16", 4, 4, 64, 8),
    ("bf16", 16, 2, 128, 32),
    ("f16", 4, 2, 128, 64),
    ("bf16", 8, 8, 128, 128),
    ("f16", 8, 1, 64, 16),
]


def _run(b, fill=0.0):
    ref = oracle.run_prefill(b)
    g = GpuPrefill(b, fill=fill)
    assert np.array_equal(g.tab_h.numpy(), ref.block_tables)
    assert np.array_equal(g.lens_h.numpy(), ref.context_lens)
    out = g.step()
    assert int(g.err.item()) == 0
    return out_f64(out, b.dtype), ref.out, g


@pytest.mark.parametrize("dtype,hq,hkv,d,bs", SHAPES)
def test_prefill_matches_oracle(dtype, hq, hkv, d, bs):
    b = workloads.prefill_custom(dtype, LENS, QLENS, hq, hkv, d, bs, seed=hq * 131 + d + bs)
    got, ref, _ = _run(b)
    check_close(got, ref, dtype, f"prefill {dtype} {hq}/{hkv} d{d} bs{bs}")


MANY_LENS = [900, 700, 1200, 333, 1024, 65, 1500, 257]
MANY_QLENS = [900, 300, 600, 333, 512, 65, 700, 257]


@pytest.mark.parametrize("dtype,hq,hkv,d,bs", [("f16", 8, 8, 64, 8), ("bf16", 16, 8, 128, 32),
                                               ("bf16", 64, 8, 64, 16)])
def test_several_items_per_cta(dtype, hq, hkv, d, bs):
    """More pairs of query tiles than SMs (256, 512 and 1856 items), so the
    persistent CTAs take several items each, across item boundaries of every
    kind (one-tile items, short and long ones), at block sizes 8-32 and both
    head dims."""
    b = workloads.prefill_custom(dtype, MANY_LENS, MANY_QLENS, hq, hkv, d, bs, seed=hq + 7 * bs + d)
    got, ref, _ = _run(b)
    check_close(got, ref, dtype, f"prefill items {dtype} {hq}/{hkv} d{d} bs{bs}")


def test_unwritten_slots_never_leak():
    """Every cache element no token wrote is NaN; keys past a chunk's range
    and the tail of its last block must still get weight 0 and a finite V."""
    b = workloads.prefill_custom("bf16", [17, 65, 200, 31], [17, 3, 129, 31], 8, 2, 128, 16,
                                 seed=5, extra_blocks=4)
    got, ref, _ = _run(b, fill=float("nan"))
    assert np.isfinite(got).all()
    check_close(got, ref, "bf16", "NaN-filled pool")


def test_one_row_chunks_equal_decode():
    """n = 1 per sequence: pa_prefill and pa_decode read the same cache and
    must agree with the oracle (and hence with each other)."""
    lens = [1, 16, 17, 300, 1025]
    b = workloads.prefill_custom("bf16", lens, [1] * len(lens), 32, 8, 128, 16, seed=9)
    got, ref, g = _run(b)
    check_close(got, ref, "bf16", "one-row chunks")
    ws = pa.alloc_workspace(len(lens), 32, 8, 128, max(lens), 0, "cuda")
    dec = torch.empty_like(g.q)
    pa.pa_decode(dec, g.q, g.kc, g.vc, g.tab, g.lens, max(lens), b.scale, workspace=ws,
                 err_flag=g.err)
    torch.cuda.synchronize()
    check_close(out_f64(dec, "bf16"), ref, "bf16", "decode on the same cache")


@pytest.mark.parametrize("name", ["prefill_gqa8b_bf16", "prefill_mha7b_f16"])
def test_full_size_sampled_rows(name):
    """The benchmark's batches at full size: every output row is finite, and
    sampled rows (first, last and random rows of random chunks, all heads)
    match the oracle computed row by row."""
    b = workloads.PREFILL_BUILDERS[name]()
    g = GpuPrefill(b)
    out = g.step()
    assert int(g.err.item()) == 0
    got = out_f64(out, b.dtype)
    assert np.isfinite(got).all()
    rng = np.random.default_rng(17)
    S = len(b.context_lens)
    rows = {}
    for s in rng.choice(S, size=min(S, 6), replace=False):
        n = b.query_lens[s]
        rows[int(s)] = sorted({0, n - 1, *rng.integers(0, n, size=3).tolist()})
    ref = oracle.run_prefill(b, rows=rows)
    assert np.array_equal(g.tab_h.numpy(), ref.block_tables)
    cu = b.query_offsets
    for s, rs in rows.items():
        idx = [cu[s] + r for r in rs]
        check_close(got[idx], ref.out[idx], b.dtype, f"{name} seq {s} rows {rs}")


def test_bad_block_and_bad_len_are_reported():
    b = workloads.prefill_custom("f16", [100, 50], [30, 50], 4, 2, 64, 16, seed=3)
    g = GpuPrefill(b)
    g.write_chunks()
    tab = g.tab.clone()
    tab[0, 2] = b.num_blocks + 7             # a block the chunk reads
    pa.pa_prefill(g.out, g.q, g.kc, g.vc, tab, g.lens, g.cu, g.max_q, b.scale, err_flag=g.err)
    torch.cuda.synchronize()
    assert int(g.err.item()) == pa.PA_DEV_BAD_BLOCK
    g.err.zero_()
    lens = g.lens.clone()
    lens[1] = 20                              # shorter than its 50-row chunk
    pa.pa_prefill(g.out, g.q, g.kc, g.vc, g.tab, lens, g.cu, g.max_q, b.scale, err_flag=g.err)
    torch.cuda.synchronize()
    assert int(g.err.item()) == pa.PA_DEV_BAD_LEN
    g.err.zero_()
    g.attend()                                # the context is still usable
    torch.cuda.synchronize()
    assert int(g.err.item()) == 0
    check_close(out_f64(g.out, "f16"), oracle.run_prefill(b).out, "f16", "after bad calls")


def test_rejected_shapes_and_empty_batch():
    b = workloads.prefill_custom("bf16", [20], [20], 4, 2, 128, 16, seed=1)
    g = GpuPrefill(b)
    with pytest.raises(pa.PAError) as e:     # fp32 has no tensor-core path
        pa.pa_prefill(g.out.float(), g.q.float(), g.kc.float(), g.vc.float(), g.tab, g.lens,
                      g.cu, g.max_q, b.scale)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
    q3 = torch.zeros((20, 6, 128), dtype=torch.bfloat16, device="cuda")   # G = 3
    with pytest.raises(pa.PAError) as e:
        pa.pa_prefill(torch.empty_like(q3), q3, g.kc, g.vc, g.tab, g.lens, g.cu, g.max_q, b.scale)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
    empty = torch.zeros((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    cu0 = torch.zeros(2, dtype=torch.int32, device="cuda")
    pa.pa_prefill(empty, empty, g.kc, g.vc, g.tab, g.lens, cu0, 1, b.scale)   # nothing to do


def test_repeat_is_bit_identical():
    b = workloads.prefill_custom("bf16", LENS, QLENS, 8, 2, 128, 16, seed=21)
    g = GpuPrefill(b)
    a = g.step().clone()
    g.attend()
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), g.out.view(torch.int16))
    assert TOL["bf16"]["atol"] > 0


def test_prefix_cache_prefills_only_the_suffix():
    """Prefix caching + paged prefill: request B's prompt starts with request
    A's first 64 tokens (four full blocks), so the manager serves those from
    A's cached blocks and B's prefill chunk is only its own suffix, attending
    over the shared blocks through its table.  Both managers (the library's
    and the oracle's) give the same tables; B's and A's outputs match the
    oracle's causal attention over the same tokens."""
    hq, hkv, d, bs = 8, 2, 128, 16
    LA, LB, shared = 100, 150, 64
    b = workloads.prefill_custom("bf16", [LA, LB], [LA, LB - shared], hq, hkv, d, bs, seed=31,
                                 extra_blocks=8)
    rng = np.random.default_rng(31)
    tok_a = rng.integers(1, 1000, LA).tolist()
    tok_b = tok_a[:shared] + rng.integers(1000, 2000, LB - shared).tolist()
    kB, vB = b.k[1].clone(), b.v[1].clone()
    kB[:shared], vB[:shared] = b.k[0][:shared], b.v[0][:shared]   # same tokens, same K/V

    # oracle: its own prefix-caching manager, cache writes and causal attention
    om = oracle.BlockManager(oracle.BlockAllocator(b.num_blocks, b.free_order), bs)
    om.enable_prefix_cache()
    osa, ca = om.add_seq_prompt(0, tok_a)
    osb, cb = om.add_seq_prompt(1, tok_b)
    assert (ca, cb) == (0, shared)
    okc = oracle.empty_cache(b.num_blocks, hkv, bs, d, "bf16")
    ovc = oracle.empty_cache(b.num_blocks, hkv, bs, d, "bf16")
    oracle.reshape_and_cache(okc, ovc, oracle.as_storage(b.k[0], "bf16"),
                             oracle.as_storage(b.v[0], "bf16"), osa)
    oracle.reshape_and_cache(okc, ovc, oracle.as_storage(kB, "bf16")[shared:],
                             oracle.as_storage(vB, "bf16")[shared:], osb[shared:])
    mb = -(-LB // bs)
    otab, olens = om.table_rows([0, 1], mb)
    otab = np.asarray(otab, dtype=np.int32)
    cu = np.array([0, LA, LA + LB - shared], dtype=np.int32)
    ref = oracle.paged_prefill(oracle.as_storage(b.q, "bf16"), okc, ovc, otab, olens, cu, b.scale,
                               "bf16")

    # CUDA path: the library's manager, cache writes of what is not cached, prefill
    m = pa.BlockManager(pa.BlockAllocator(b.num_blocks, b.free_order), bs)
    m.enable_prefix_cache()
    sa, _ = m.add_seq_prompt(0, tok_a)
    sb, cached = m.add_seq_prompt(1, tok_b)
    assert cached == shared and sb[:shared].tolist() == [-1] * shared
    kc = torch.zeros((b.num_blocks, hkv, bs, d), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    keys = torch.cat([b.k[0], kB[shared:]]).cuda()
    vals = torch.cat([b.v[0], vB[shared:]]).cuda()
    slots = torch.cat([sa, sb[shared:]]).cuda()
    pa.pa_reshape_and_cache(keys, vals, kc, vc, slots, err_flag=err)
    tab, lens = m.block_tables([0, 1], mb)
    assert np.array_equal(tab.numpy(), otab) and lens.tolist() == [LA, LB]
    q = b.q.cuda()
    out = torch.full_like(q, float("nan"))
    pa.pa_prefill(out, q, kc, vc, tab.cuda(), lens.cuda(), torch.from_numpy(cu).cuda(),
                  max(LA, LB - shared), b.scale, err_flag=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    check_close(out_f64(out, "bf16"), ref, "bf16", "prefix-cached prompt, suffix prefill")


def test_workspace_left_zeroed_and_reused():
    """The persistent launch takes work items from a counter in the caller's
    workspace; every call leaves it zeroed (after a bad table entry too), so
    back-to-back calls on one workspace give the same output.  More items
    than SMs (about 300 pairs of tiles), so CTAs take several each."""
    b = workloads.prefill_custom("bf16", [1200, 700, 900, 333, 1024, 65],
                                 [1200, 300, 900, 333, 512, 65], 32, 8, 128, 16, seed=11)
    g = GpuPrefill(b)
    g.write_chunks()
    ws = pa.prefill_workspace(g.out.device)
    outs = []
    for _ in range(3):
        g.out.zero_()
        pa.pa_prefill(g.out, g.q, g.kc, g.vc, g.tab, g.lens, g.cu, g.max_q, b.scale, workspace=ws,
                      err_flag=g.err)
        torch.cuda.synchronize()
        assert int(g.err.item()) == 0
        assert int(ws.abs().sum().item()) == 0
        outs.append(g.out.clone())
    assert all(torch.equal(outs[0], o) for o in outs[1:])
    check_close(out_f64(outs[0], "bf16"), oracle.run_prefill(b).out, "bf16", "persistent items")
    tab = g.tab.clone()
    tab[0, 3] = -5                            # a bad entry: the call reports it, ws still zero
    pa.pa_prefill(g.out, g.q, g.kc, g.vc, tab, g.lens, g.cu, g.max_q, b.scale, workspace=ws,
                  err_flag=g.err)
    torch.cuda.synchronize()
    assert int(g.err.item()) == pa.PA_DEV_BAD_BLOCK
    assert int(ws.abs().sum().item()) == 0


def test_output_only_16_byte_aligned():
    """The output rows are written 32 bytes a store when `out` is 32-byte
    aligned; an output starting 16 bytes into an allocation takes the 16-byte
    stores and must match the same way."""
    b = workloads.prefill_custom("f16", [300, 129], [300, 64], 8, 2, 128, 16, seed=5)
    g = GpuPrefill(b)
    g.write_chunks()
    T, hq, d = g.q.shape
    big = torch.zeros(T * hq * d + 8, dtype=g.out.dtype, device=g.out.device)
    out = big[8:].view(T, hq, d)                 # 16 bytes past a 256-byte boundary
    assert out.data_ptr() % 32 == 16
    pa.pa_prefill(out, g.q, g.kc, g.vc, g.tab, g.lens, g.cu, g.max_q, b.scale, err_flag=g.err)
    torch.cuda.synchronize()
    assert int(g.err.item()) == 0
    check_close(out_f64(out, "f16"), oracle.run_prefill(b).out, "f16", "16-byte aligned output")
