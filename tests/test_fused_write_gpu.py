"""The step's cache write done by the decode call (pa_decode_ex's key_new /
value_new / slot_mapping).  "Paged Attention" (velog), 작동 예시, and "09.
PagedAttention" (119-ai-studio), 해법: the new token's K/V goes into the slot
its table assigns, then attention reads it.  Each engine is compared with the
oracle (outputs element by element, caches bit for bit), the fused write with
the separate cache write bit for bit, and the slot checks on crafted tables.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.harness import CudaPathRun, check_close, out_f64
from tests.test_gpu_parity import run_full_compare

pytestmark = pytest.mark.gpu
pa = pytest.importorskip("paged_kv_cache_426_b200")

ENGINES = ["auto", "core", "tensor"]


@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("P", [0, 64])
def test_fused_mha_f16_small(engine, P):
    run_full_compare(workloads.mha7b_f16(steps=3, num_seqs=5), partition_size=P, engine=engine,
                     fused=True)


@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("bs", [16, 32])
def test_fused_gqa_bf16_small(engine, bs):
    run_full_compare(workloads.gqa8b_bf16(block_size=bs, num_seqs=10), partition_size=512,
                     engine=engine, fused=True)


@pytest.mark.parametrize("engine", ENGINES)
def test_fused_prefix_f16_small(engine):
    """Shared prefix blocks and forked beams: the copy-on-write copies run
    before the decode call, whose write then lands in the private copy."""
    w = workloads.prefix_f16(n_req=6, plen=64, suffix_max=40, n_fork=2, heads=4)
    run_full_compare(w, partition_size=32, engine=engine, fused=True)


@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("bs", [8, 16, 32, 64, 128])
def test_fused_block_sizes(engine, bs):
    w = workloads.custom("f16", [3, 8, 9, 129, 300], 8, 2, 128, bs, seed=bs, partition_size=128)
    run_full_compare(w, engine=engine, fused=True)


@pytest.mark.parametrize("engine", ENGINES)
@pytest.mark.parametrize("bs", [64, 128])
def test_fused_partitions_inside_blocks(engine, bs):
    """Partitions of 16 tokens inside 64- and 128-token blocks: the block that
    receives the new token is also read by the sequence's earlier partitions
    (other work units, other CTAs), which never read the written row."""
    w = workloads.custom("bf16", [15, 16, 17, 130, 300, 511], 16, 4, 128, bs, seed=bs + 3,
                         partition_size=16, steps=3)
    run_full_compare(w, engine=engine, fused=True)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_fused_shapes_and_groups(dtype, d, G):
    hkv = 2
    w = workloads.custom(dtype, [1, 15, 16, 17, 100, 257], hkv * G, hkv, d, 16, seed=G * d + 1,
                         partition_size=64)
    run_full_compare(w, engine="tensor", fused=True)


@pytest.mark.parametrize("P", [0, 16])
def test_fused_tiny_f32(P):
    run_full_compare(workloads.tiny_f32(), partition_size=P, engine="auto", fused=True)


@pytest.mark.parametrize("engine", ["auto", "tensor"])
def test_fused_many_units_per_cta(engine):
    """Every CTA takes several units, so writes happen in units taken from the
    ticket counter, not only in a CTA's first one."""
    rng = np.random.default_rng(8)
    lens = [int(x) for x in rng.integers(200, 420, size=40)]
    w = workloads.custom("bf16", lens, 32, 8, 128, 16, seed=42, partition_size=32, steps=2)
    run_full_compare(w, engine=engine, fused=True)


@pytest.mark.parametrize("engine", ["core", "tensor"])
def test_fused_bit_identical_to_separate_write(engine):
    """Same steps with the cache write as its own launch and inside the decode
    call: identical outputs and caches, bit for bit."""
    w = workloads.gqa8b_bf16(block_size=16, num_seqs=12)
    rec = oracle.run(w, keep_prefill_cache=True, decode=False)
    runs = []
    for fused in (False, True):
        g = CudaPathRun(w, rec, partition_size=64, engine=engine, fused=fused)
        g.replay_prefill()
        runs.append((g, [g.step(k).cpu() for k in range(len(rec.steps))]))
    (g0, o0), (g1, o1) = runs
    for k, (a, b) in enumerate(zip(o0, o1)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"step {k}"
    assert torch.equal(g0.kc.view(torch.int16), g1.kc.view(torch.int16))
    assert torch.equal(g0.vc.view(torch.int16), g1.vc.view(torch.int16))


@pytest.mark.parametrize("engine", ["core", "tensor"])
@pytest.mark.parametrize("P", [0, 16])
def test_fused_write_slot_checks(engine, P):
    """slot_mapping[s] must be the slot of position L - 1 through the table:
    a wrong slot sets PA_DEV_BAD_SLOT and writes nothing, a negative one skips
    the write, a sequence with no tokens has no slot; the other sequences'
    writes and outputs are unaffected."""
    d, hkv, G, bs, NB = 128, 2, 2, 16, 8
    gen = torch.Generator().manual_seed(5 + P)
    kc = torch.randn(NB, hkv, bs, d, generator=gen).bfloat16().cuda()
    vc = torch.randn(NB, hkv, bs, d, generator=gen).bfloat16().cuda()
    q = torch.randn(5, hkv * G, d, generator=gen).bfloat16().cuda()
    kn = torch.randn(5, hkv, d, generator=gen).bfloat16().cuda()
    vn = torch.randn(5, hkv, d, generator=gen).bfloat16().cuda()
    tab = torch.tensor([[0, 1], [2, -1], [3, -1], [4, 5], [-1, -1]], dtype=torch.int32,
                       device="cuda")
    lens = torch.tensor([20, 5, 9, 32, 0], dtype=torch.int32, device="cuda")
    # positions L - 1: 19 -> block 1 row 3 (slot 19); 4 -> block 2 row 4 (36);
    # 8 -> block 3 row 8 (56); 31 -> block 5 row 15 (95); none for L = 0
    good = torch.tensor([19, 36, 56, 95, -1], dtype=torch.int64, device="cuda")
    bad = torch.tensor([19, 37, -1, 95, 7], dtype=torch.int64, device="cuda")
    kref, vref = kc.clone(), vc.clone()
    for s, (b, r) in {0: (1, 3), 3: (5, 15)}.items():       # the writes that happen
        kref[b, :, r] = kn[s]
        vref[b, :, r] = vn[s]
    ws = pa.alloc_workspace(5, hkv * G, hkv, d, 32, P)
    out = torch.full_like(q, float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode(out, q, kc, vc, tab, lens, 32, 0.1, partition_size=P, workspace=ws,
                 err_flag=err, engine=engine, write=(kn, vn, bad))
    torch.cuda.synchronize()
    assert err.item() == pa.PA_DEV_BAD_SLOT
    assert torch.equal(kc.view(torch.int16), kref.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), vref.view(torch.int16))
    ref = oracle.paged_decode(oracle.as_storage(q.cpu(), "bf16"),
                              oracle.as_storage(kref.cpu(), "bf16"),
                              oracle.as_storage(vref.cpu(), "bf16"), tab.cpu().numpy(),
                              lens.cpu().numpy(), 0.1, "bf16")
    check_close(out_f64(out, "bf16"), ref, "bf16", "outputs over the cache as written")
    # valid slots for every sequence: no error, every token written
    err.zero_()
    for s, (b, r) in {1: (2, 4), 2: (3, 8)}.items():
        kref[b, :, r] = kn[s]
        vref[b, :, r] = vn[s]
    pa.pa_decode(out, q, kc, vc, tab, lens, 32, 0.1, partition_size=P, workspace=ws,
                 err_flag=err, engine=engine, write=(kn, vn, good))
    torch.cuda.synchronize()
    assert err.item() == 0
    assert torch.equal(kc.view(torch.int16), kref.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), vref.view(torch.int16))


@pytest.mark.parametrize("engine", ["core", "tensor"])
def test_fused_write_zero_length_sequence(engine):
    """A sequence with no tokens has no position for a new one: a
    non-negative slot for it sets PA_DEV_BAD_SLOT (and nothing is written);
    -1 is a skipped write, no error."""
    d, hkv, G, bs, NB = 64, 1, 4, 16, 4
    gen = torch.Generator().manual_seed(9)
    kc = torch.randn(NB, hkv, bs, d, generator=gen).half().cuda()
    vc = torch.randn(NB, hkv, bs, d, generator=gen).half().cuda()
    q = torch.randn(2, hkv * G, d, generator=gen).half().cuda()
    kn = torch.randn(2, hkv, d, generator=gen).half().cuda()
    vn = torch.randn(2, hkv, d, generator=gen).half().cuda()
    tab = torch.tensor([[0, 1], [-1, -1]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([17, 0], dtype=torch.int32, device="cuda")
    ws = pa.alloc_workspace(2, hkv * G, hkv, d, 32, 16)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    kref, vref = kc.clone(), vc.clone()
    kref[1, :, 0] = kn[0]
    vref[1, :, 0] = vn[0]
    for slot1, want in ((-1, 0), (40, pa.PA_DEV_BAD_SLOT)):
        kc.copy_(kref); vc.copy_(vref)
        kc[1, :, 0] = 0
        vc[1, :, 0] = 0
        err.zero_()
        slots = torch.tensor([16, slot1], dtype=torch.int64, device="cuda")
        pa.pa_decode(out, q, kc, vc, tab, lens, 32, 0.125, partition_size=16, workspace=ws,
                     err_flag=err, engine=engine, write=(kn, vn, slots))
        torch.cuda.synchronize()
        assert err.item() == want
        assert torch.equal(kc.view(torch.int16), kref.view(torch.int16))
        assert torch.equal(vc.view(torch.int16), vref.view(torch.int16))
        assert not out[1].any()
