"""GPU parity: the CUDA path against the float64 oracle on the same seeded inputs.

* cache writes and copy-on-write copies: bit-exact over the whole caches
  (untouched slots keep their previous bits);
* host metadata (slot mappings, copy pairs, block tables): equal to the
  oracle's;
* decode outputs: fp32 max-abs 1e-5; fp16/bf16 |gpu - ref| <= 3e-3 + 1e-2 |ref|
  element-wise, plus a per-(sequence, head) normalised L2 error <= 5e-3 (fp16)
  / 1e-2 (bf16).

Small variants of the five workloads are compared element by element (they
span several stages, partitions and a ragged tail; one set has more work units
than three per resident CTA).  The full-size workloads, in the launch
configuration the benchmark times, are compared element by element at step 0,
every 8th step and the last step, and on sampled (sequence, head) outputs
that the oracle computes one by one at the steps between.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from tests.harness import (CudaPathRun, check_close, oracle_sampled, out_f64, sample_pairs,
                           to_torch_storage)

pytestmark = pytest.mark.gpu
pa = pytest.importorskip("paged_kv_cache_426_b200")

# auto: tensor cores for 16-bit types, CUDA cores for fp32; each call passes
# the engine as a per-call option (pa_decode_ex)
ENGINES = {"auto": 0, "core": 1, "tensor": 2}


@pytest.fixture(params=list(ENGINES))
def engine(request):
    return request.param


def run_full_compare(w, partition_size=None, steps=None, engine="auto", fused=False):
    if engine == "tensor" and w.dtype == "f32":
        pytest.skip("the tensor-core engine takes 16-bit types")
    rec = oracle.run(w, keep_prefill_cache=True, steps=steps)
    g = CudaPathRun(w, rec, partition_size=partition_size, engine=engine, fused=fused)
    g.replay_prefill()
    errs = []
    for k in range(len(rec.steps)):
        out = g.step(k)
        errs.append(check_close(out_f64(out, w.dtype), rec.steps[k].out, w.dtype,
                                f"{w.name} step {k} P={g.P}"))
    assert g.caches_equal_oracle(), "caches differ from the oracle after the steps"
    return errs


# ---------------------------------------------------------------- element by element

@pytest.mark.parametrize("P", [0, 16, 32])
def test_tiny_f32(engine, P):
    run_full_compare(workloads.tiny_f32(), partition_size=P, engine=engine)


@pytest.mark.parametrize("P", [0, 64, 512])
def test_mha_f16_small(engine, P):
    run_full_compare(workloads.mha7b_f16(steps=3, num_seqs=5), partition_size=P, engine=engine)


@pytest.mark.parametrize("bs", [16, 32])
def test_gqa_bf16_small(engine, bs):
    run_full_compare(workloads.gqa8b_bf16(block_size=bs, num_seqs=10), partition_size=512, engine=engine)


def test_prefix_f16_small(engine):
    w = workloads.prefix_f16(n_req=6, plen=64, suffix_max=40, n_fork=2, heads=4)
    run_full_compare(w, partition_size=32, engine=engine)


def test_long_bf16_small(engine):
    w = workloads.custom("bf16", [3001, 4096, 1500], 32, 8, 128, 64, seed=77,
                         partition_size=512)
    run_full_compare(w, engine=engine)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_shapes_and_groups(engine, dtype, d, G):
    hkv = 2
    w = workloads.custom(dtype, [1, 15, 16, 17, 100, 257], hkv * G, hkv, d, 16, seed=G * d,
                         partition_size=64)
    run_full_compare(w, engine=engine)


@pytest.mark.parametrize("L", [511, 512, 513, 1000])
def test_split_merge_boundary(engine, L):
    """Up to 32 partitions the merge kernel takes one CTA per (sequence, KV
    head), from 33 one CTA per (sequence, query head) with sliced partitions:
    both sides of the boundary, with a short sequence in the same batch."""
    w = workloads.custom("bf16", [L, 40], 16, 4, 128, 16, seed=L, partition_size=16)
    run_full_compare(w, engine=engine)


@pytest.mark.parametrize("bs", [8, 16, 32, 64, 128])
def test_block_sizes(engine, bs):
    w = workloads.custom("f16", [3, 8, 9, 129, 300], 8, 2, 128, bs, seed=bs, partition_size=128)
    run_full_compare(w, engine=engine)


# ---------------------------------------------------------------- invariances

def _decode_outputs(w, P, engine_id=0):
    rec = oracle.run(w, keep_prefill_cache=True, decode=False)
    g = CudaPathRun(w, rec, partition_size=P, engine=engine_id)
    g.replay_prefill()
    return [g.step(k).cpu() for k in range(len(rec.steps))], rec


def test_block_size_invariance_bit_identical():
    """Same logical K/V, block 16 vs 32, different fragmented pools."""
    a, _ = _decode_outputs(workloads.gqa8b_bf16(block_size=16, num_seqs=12), 512)
    b, _ = _decode_outputs(workloads.gqa8b_bf16(block_size=32, num_seqs=12), 512)
    assert torch.equal(a[0], b[0])


def test_physical_permutation_invariance_bit_identical():
    w1 = workloads.mha7b_f16(steps=2, num_seqs=4)
    w2 = workloads.mha7b_f16(steps=2, num_seqs=4)
    w2.free_order = list(reversed(w2.free_order))
    a, _ = _decode_outputs(w1, 64)
    b, _ = _decode_outputs(w2, 64)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_shared_vs_duplicated_prefix_bit_identical():
    kw = dict(n_req=6, plen=64, suffix_max=40, n_fork=2, heads=4)
    a, ra = _decode_outputs(workloads.prefix_f16(**kw), 32)
    b, rb = _decode_outputs(workloads.prefix_f16(duplicate_prefix=True, **kw), 32)
    assert torch.equal(a[0], b[0])
    # the shared layout really holds fewer blocks
    used = lambda r: r.manager.alloc.num_blocks - r.manager.alloc.num_free()
    assert used(ra) < used(rb)


@pytest.mark.parametrize("P", [16, 512, 1024, 2048])
def test_partition_sizes_agree(P):
    w = workloads.custom("bf16", [5000, 2049, 77], 16, 4, 128, 32, seed=3)
    ref, _ = _decode_outputs(w, 0)
    got, _ = _decode_outputs(w, P)
    check_close(got[0].double().numpy(), ref[0].double().numpy(), "bf16", f"P={P} vs unsplit")


@pytest.mark.parametrize("engine_id", [1, 2])
def test_physical_permutation_invariance_each_engine(engine_id):
    w1 = workloads.gqa8b_bf16(num_seqs=6)
    w2 = workloads.gqa8b_bf16(num_seqs=6)
    w2.free_order = list(reversed(w2.free_order))
    a, _ = _decode_outputs(w1, 64, engine_id)
    b, _ = _decode_outputs(w2, 64, engine_id)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_tensor_engine_rejects_f32():
    w = workloads.tiny_f32()
    with pytest.raises(pa.PAError) as e:
        _decode_outputs(w, 16, pa.PA_ENGINE_TENSOR)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED


@pytest.mark.parametrize("engine_id", [1, 2])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_growing_logits(engine_id, dtype):
    """Logits that rise by far more than 2^8 (log2 units) along the sequence and
    then fall: the running max moves many times within a unit, so the tensor
    engine's deferred rescale of O in tensor memory is exercised."""
    g = torch.Generator().manual_seed(5)
    d, hkv, G, bs, L = 128, 2, 4, 16, 700
    nb = (L + bs - 1) // bs
    q = torch.randn(1, hkv * G, d, generator=g)
    ramp = torch.cat([torch.linspace(0, 6, 400), torch.linspace(6, -3, L - 400)])
    k = torch.randn(L, hkv, d, generator=g) * 0.3 + ramp[:, None, None] * q.view(hkv, G, d).mean(1)[None]
    v = torch.randn(L, hkv, d, generator=g)
    kc = torch.zeros(nb, hkv, bs, d)
    vc = torch.zeros(nb, hkv, bs, d)
    perm = torch.randperm(nb, generator=g)
    for t in range(L):
        kc[perm[t // bs], :, t % bs] = k[t]
        vc[perm[t // bs], :, t % bs] = v[t]
    q, kc, vc = q.to(dtype), kc.to(dtype), vc.to(dtype)
    tab = perm.view(1, -1).to(torch.int32)
    lens = torch.tensor([L], dtype=torch.int32)
    name = "f16" if dtype == torch.float16 else "bf16"
    ref = oracle.paged_decode(oracle.as_storage(q, name), oracle.as_storage(kc, name),
                              oracle.as_storage(vc, name), tab.numpy(), lens.numpy(), 1.0, name)
    for P in (0, 256):
        ws = pa.alloc_workspace(1, hkv * G, hkv, d, L, P)
        out = torch.full_like(q, float("nan")).cuda()
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        pa.pa_decode(out, q.cuda(), kc.cuda(), vc.cuda(), tab.cuda(), lens.cuda(), L, 1.0,
                     partition_size=P, workspace=ws, err_flag=err, engine=engine_id)
        torch.cuda.synchronize()
        assert err.item() == 0
        check_close(out_f64(out, name), ref, name, f"growing logits P={P}")


# ---------------------------------------------------------------- edge cases

def _cache(NB, hkv, bs, d, dt, fill=0):
    return torch.full((NB, hkv, bs, d), fill, dtype=dt, device="cuda")


def test_zero_and_one_token():
    d, hkv, G, bs = 128, 2, 4, 16
    kc = torch.randn(4, hkv, bs, d, device="cuda").to(torch.bfloat16)
    vc = torch.randn(4, hkv, bs, d, device="cuda").to(torch.bfloat16)
    q = torch.randn(3, hkv * G, d, device="cuda").to(torch.bfloat16)
    tab = torch.tensor([[2, -1], [-1, -1], [1, 3]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([1, 0, 17], dtype=torch.int32, device="cuda")
    ws = pa.alloc_workspace(3, hkv * G, hkv, d, 32, 16)
    out = torch.full_like(q, float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode(out, q, kc, vc, tab, lens, 32, 0.1, partition_size=16, workspace=ws, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    for h in range(hkv * G):                       # one token: exactly its V row
        assert torch.equal(out[0, h], vc[2, h // G, 0])
    assert not out[1].any()                        # no token: zeros
    ref = oracle.paged_decode(oracle.as_storage(q.cpu(), "bf16"), oracle.as_storage(kc.cpu(), "bf16"),
                              oracle.as_storage(vc.cpu(), "bf16"), tab.cpu().numpy(),
                              lens.cpu().numpy(), 0.1, "bf16")
    check_close(out_f64(out[2:], "bf16"), ref[2:], "bf16", "17 tokens over two blocks")


def test_max_context_fills_table_exactly():
    w = workloads.custom("f16", [256, 255], 8, 8, 128, 16, seed=11, partition_size=64)
    rec = oracle.run(w, keep_prefill_cache=True)
    g = CudaPathRun(w, rec, max_blocks=16)            # 256 tokens = 16 blocks exactly
    g.replay_prefill()
    out = g.step(0)
    check_close(out_f64(out, "f16"), rec.steps[0].out, "f16", "full table")


def test_bad_block_id_sets_flag_without_fault():
    d, bs = 128, 16
    kc = torch.randn(4, 1, bs, d, device="cuda").half()
    vc = torch.randn(4, 1, bs, d, device="cuda").half()
    q = torch.randn(2, 1, d, device="cuda").half()
    tab = torch.tensor([[0, 9], [1, 2]], dtype=torch.int32, device="cuda")   # 9 >= num_blocks
    lens = torch.tensor([20, 20], dtype=torch.int32, device="cuda")
    ws = pa.alloc_workspace(2, 1, 1, d, 32, 0)
    out = torch.zeros_like(q)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode(out, q, kc, vc, tab, lens, 32, 0.1, workspace=ws, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == pa.PA_DEV_BAD_BLOCK
    ref = oracle.paged_decode(oracle.as_storage(q.cpu()[1:], "f16"), oracle.as_storage(kc.cpu(), "f16"),
                              oracle.as_storage(vc.cpu(), "f16"), tab.cpu().numpy()[1:],
                              lens.cpu().numpy()[1:], 0.1, "f16")
    check_close(out_f64(out[1:], "f16"), ref, "f16", "the valid sequence is unaffected")
    # the workspace is still usable: a clean call succeeds
    err.zero_()
    tab[0, 1] = 3
    pa.pa_decode(out, q, kc, vc, tab, lens, 32, 0.1, workspace=ws, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0


def test_bad_block_id_tensor_engine():
    d, bs, hkv, G = 128, 16, 2, 4
    kc = torch.randn(4, hkv, bs, d, device="cuda").bfloat16()
    vc = torch.randn(4, hkv, bs, d, device="cuda").bfloat16()
    q = torch.randn(2, hkv * G, d, device="cuda").bfloat16()
    tab = torch.tensor([[0, 9], [1, 2]], dtype=torch.int32, device="cuda")   # 9 >= num_blocks
    lens = torch.tensor([20, 20], dtype=torch.int32, device="cuda")
    ws = pa.alloc_workspace(2, hkv * G, hkv, d, 32, 16)
    out = torch.zeros_like(q)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode(out, q, kc, vc, tab, lens, 32, 0.1, partition_size=16, workspace=ws,
                 err_flag=err, engine="tensor")
    torch.cuda.synchronize()
    assert err.item() == pa.PA_DEV_BAD_BLOCK
    ref = oracle.paged_decode(oracle.as_storage(q.cpu()[1:], "bf16"),
                              oracle.as_storage(kc.cpu(), "bf16"),
                              oracle.as_storage(vc.cpu(), "bf16"), tab.cpu().numpy()[1:],
                              lens.cpu().numpy()[1:], 0.1, "bf16")
    check_close(out_f64(out[1:], "bf16"), ref, "bf16", "the valid sequence is unaffected")
    assert torch.isfinite(out[0].float()).all()
    err.zero_()
    tab[0, 1] = 3
    pa.pa_decode(out, q, kc, vc, tab, lens, 32, 0.1, partition_size=16, workspace=ws,
                 err_flag=err, engine="tensor")
    torch.cuda.synchronize()
    assert err.item() == 0


def test_bad_length_is_clamped_and_flagged():
    d = 64
    kc = torch.randn(4, 1, 16, d, device="cuda")
    vc = torch.randn(4, 1, 16, d, device="cuda")
    q = torch.randn(1, 1, d, device="cuda")
    tab = torch.tensor([[0, 1]], dtype=torch.int32, device="cuda")
    lens = torch.tensor([40], dtype=torch.int32, device="cuda")      # > 2 blocks * 16
    ws = pa.alloc_workspace(1, 1, 1, d, 64, 0)
    out = torch.zeros_like(q)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode(out, q, kc, vc, tab, lens, 64, 0.125, workspace=ws, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == pa.PA_DEV_BAD_LEN
    ref = oracle.paged_decode(q.cpu().numpy(), kc.cpu().numpy(), vc.cpu().numpy(),
                              tab.cpu().numpy(), np.array([32]), 0.125, "f32")
    check_close(out.double().cpu().numpy(), ref, "f32", "clamped to the table")


# ---------------------------------------------------------------- cache ops

@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("bs", [8, 16, 64])
def test_reshape_and_cache_bit_exact(dtype, bs):
    g = torch.Generator().manual_seed(bs)
    NB, hkv, d, T = 9, 3, 128, 40
    k = torch.randn(T, hkv, d, generator=g).to(dtype)
    v = torch.randn(T, hkv, d, generator=g).to(dtype)
    slots = torch.randperm(NB * bs, generator=g)[:T].to(torch.int64)
    slots[5] = -1
    name = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}[dtype]
    kc0 = oracle.empty_cache(NB, hkv, bs, d, name, fill=0x5A5A)
    vc0 = oracle.empty_cache(NB, hkv, bs, d, name, fill=0x3C3C)
    kc_gpu = to_torch_storage(kc0.copy(), name).cuda()
    vc_gpu = to_torch_storage(vc0.copy(), name).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_reshape_and_cache(k.cuda(), v.cuda(), kc_gpu, vc_gpu, slots.cuda(), err_flag=err)
    oracle.reshape_and_cache(kc0, vc0, oracle.as_storage(k, name), oracle.as_storage(v, name),
                             slots.numpy())
    torch.cuda.synchronize()
    assert err.item() == 0
    assert np.array_equal(oracle.as_storage(kc_gpu.cpu(), name).view(np.uint8), kc0.view(np.uint8))
    assert np.array_equal(oracle.as_storage(vc_gpu.cpu(), name).view(np.uint8), vc0.view(np.uint8))


def test_reshape_and_cache_bad_slot():
    kc = torch.zeros(2, 1, 16, 64, device="cuda")
    vc = torch.zeros_like(kc)
    k = torch.ones(2, 1, 64, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_reshape_and_cache(k, k, kc, vc, torch.tensor([3, 32], device="cuda"), err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == pa.PA_DEV_BAD_SLOT
    assert kc[0, 0, 3].eq(1).all() and kc.sum().item() == 64


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
def test_copy_blocks_bit_exact(dtype):
    name = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}[dtype]
    g = torch.Generator().manual_seed(1)
    kc = torch.randn(12, 4, 16, 128, generator=g).to(dtype)
    vc = torch.randn(12, 4, 16, 128, generator=g).to(dtype)
    pairs = [(1, 7), (3, 0), (3, 11), (10, 2)]
    kg, vg = kc.cuda(), vc.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks(kg, vg, torch.tensor(pairs, dtype=torch.int64, device="cuda"), err_flag=err)
    ko, vo = oracle.as_storage(kc, name).copy(), oracle.as_storage(vc, name).copy()
    oracle.copy_blocks(ko, vo, pairs)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert np.array_equal(oracle.as_storage(kg.cpu(), name).view(np.uint8), ko.view(np.uint8))
    assert np.array_equal(oracle.as_storage(vg.cpu(), name).view(np.uint8), vo.view(np.uint8))
    err.zero_()
    pa.pa_copy_blocks(kg, vg, torch.tensor([[0, 12]], device="cuda"), err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == pa.PA_DEV_BAD_PAIR


# ---------------------------------------------------------------- full-size workloads

FULL = [
    ("mha7b_f16", dict(steps=32)),
    ("gqa8b_bf16_bs16", {}),
    ("gqa8b_bf16_bs32", {}),
    ("prefix_f16", {}),
    ("long_bf16", {}),
]


@pytest.mark.slow
@pytest.mark.parametrize("name,kw", FULL, ids=[f[0] for f in FULL])
def test_full_size(name, kw):
    """Full-size workload in the benchmark's launch configuration (its
    partition size, the step's cache write done by the decode call), every
    decode step.  Step 0, every 8th step and the last
    step are compared element by element (every sequence, query head and
    column) with the oracle's output computed from the cache as it stands at
    that step; the other steps on sampled (sequence, head) rows the oracle
    computes one by one; the whole caches bit-exact after the last step."""
    w = workloads.make(name, **kw)
    n = w.num_steps
    full = {0, n - 1} | set(range(0, n, 8))
    rec = oracle.run(w, keep_prefill_cache=True, decode_steps=full)
    g = CudaPathRun(w, rec, fused=True)
    g.replay_prefill()
    S, Hq = rec.steps[0].context_lens.shape[0], w.num_q_heads
    for k in range(len(rec.steps)):
        out = g.step(k)
        got = out_f64(out, w.dtype)
        if k in full:
            check_close(got, rec.steps[k].out, w.dtype, f"{name} step {k}, every row")
        elif k % 4 == 0:
            pairs = sample_pairs(S, Hq, 48, seed=k)
            for (s, h), r in oracle_sampled(w, rec, k, pairs).items():
                check_close(got[s, h][None, None], r[None, None], w.dtype,
                            f"{name} step {k} ({s},{h})")
    assert g.caches_equal_oracle()


@pytest.mark.parametrize("engine_id", ["auto", "core", "tensor"])
@pytest.mark.parametrize("dtype,hq,hkv,P", [("bf16", 32, 8, 32), ("f16", 32, 32, 64)])
def test_many_units_per_cta(engine_id, dtype, hq, hkv, P):
    """More work units than three per resident CTA (2 x 148 for the tensor-core
    engine, 148 x pipelines for the CUDA-core one), so every CTA takes several
    units: the unit ring, the alternating output buffers and the ticket
    prefetch run through many units.  Element by element against the oracle."""
    rng = np.random.default_rng(hq + hkv)
    lens = [int(x) for x in rng.integers(200, 420, size=40)]
    w = workloads.custom(dtype, lens, hq, hkv, 128, 16, seed=41, partition_size=P, steps=2)
    units = sum(-(-(L + 1) // P) for L in lens) * hkv
    assert units > 3 * 296
    run_full_compare(w, engine=engine_id)


# ---------------------------------------------------------------- prefix caching

def test_prefix_cache_decode_bit_identical():
    """Prompts sharing leading tokens, K/V a function of the token id: with the
    prefix cache, later prompts map the cached blocks (written once, their own
    slots come back as -1 and are skipped by the cache write); the decode equals
    the same prompts stored privately bit for bit, and the oracle's within
    tolerance."""
    g = torch.Generator().manual_seed(7)
    bs, hkv, G, d, V = 16, 2, 4, 128, 40
    emb_k = torch.randn(V, hkv, d, generator=g).bfloat16()
    emb_v = torch.randn(V, hkv, d, generator=g).bfloat16()
    base = torch.randint(0, V, (96,), generator=g).tolist()
    prompts = [base[:L] + torch.randint(0, V, (t,), generator=g).tolist()
               for L, t in [(96, 5), (64, 20), (96, 0), (33, 40), (80, 17), (0, 50)]]
    S = len(prompts)
    nb = sum(-(-len(p) // bs) for p in prompts) + 4
    max_len = max(len(p) for p in prompts)
    mb = -(-max_len // bs)
    q = torch.randn(S, hkv * G, d, generator=g).bfloat16().cuda()

    def run(cached):
        alloc = pa.BlockAllocator(nb)
        mgr = pa.BlockManager(alloc, bs)
        if cached:
            mgr.enable_prefix_cache()
        kc = torch.zeros(nb, hkv, bs, d, dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        hits = 0
        for s, p in enumerate(prompts):
            if cached:
                slots, n = mgr.add_seq_prompt(s, p)
                hits += n
            else:
                mgr.add_seq(s)
                slots, _ = mgr.append(s, len(p))
            ids = torch.tensor(p, dtype=torch.long)
            pa.pa_reshape_and_cache(emb_k[ids].cuda(), emb_v[ids].cuda(), kc, vc, slots.cuda())
        tab, lens = mgr.block_tables(range(S), mb)
        out = torch.empty_like(q)
        ws = pa.alloc_workspace(S, hkv * G, hkv, d, max_len, 32)
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        pa.pa_decode(out, q, kc, vc, tab.cuda(), lens.cuda(), max_len, d ** -0.5,
                     partition_size=32, workspace=ws, err_flag=err)
        torch.cuda.synchronize()
        assert err.item() == 0
        blocks_used = alloc.num_blocks - alloc.num_free()
        return out.cpu(), kc.cpu(), vc.cpu(), tab, lens, hits, blocks_used

    a_out, a_k, a_v, a_tab, a_lens, hits, a_used = run(True)
    b_out, b_k, b_v, b_tab, b_lens, _, b_used = run(False)
    assert hits >= 3 * bs and a_used < b_used      # the cache really served blocks
    assert torch.equal(a_out, b_out)
    ref = oracle.paged_decode(oracle.as_storage(q.cpu(), "bf16"), oracle.as_storage(a_k, "bf16"),
                              oracle.as_storage(a_v, "bf16"), a_tab.numpy(), a_lens.numpy(),
                              d ** -0.5, "bf16")
    check_close(out_f64(a_out, "bf16"), ref, "bf16", "prefix-cached prompts vs oracle")


# ---------------------------------------------------------------- failure detection

@pytest.mark.parametrize("engine_id,P", [(1, 512), (2, 512), (2, 2048)])
def test_bounded_wait_reports_timeout(engine_id, P):
    """Failure detection without a fault: a stage whose barrier nothing will
    arrive on (per-call option test_withhold_stage of pa_decode_ex) makes the
    waiting warps give up after the 2 s limit; the call returns, err_flag says
    PA_DEV_TIMEOUT, and the next call on the same workspace and context is
    correct.  With P = 2048 the tensor-core engine merges the sequences' 3
    partitions itself: the timed-out call leaves split counters partly
    counted, and the kernel's last CTA must zero them again."""
    import time
    w = workloads.gqa8b_bf16(num_seqs=6)
    rec = oracle.run(w, keep_prefill_cache=True)
    g = CudaPathRun(w, rec, partition_size=P)
    g.replay_prefill()
    st = rec.steps[0]
    slots, _ = g.mgr.append_step(st.seqs)
    tab, lens = g.mgr.block_tables(st.seqs, g.mb)
    pa.pa_reshape_and_cache(w.step_k[0].cuda(), w.step_v[0].cuda(), g.kc, g.vc, slots.cuda(),
                            err_flag=g.err)
    q = w.step_q[0].cuda()
    out = torch.empty_like(q)
    tab_d, lens_d = tab.cuda(), lens.cuda()
    S = q.shape[0]

    def decode(hold):
        pa.pa_decode(out, q, g.kc, g.vc, tab_d, lens_d, g.max_len, w.scale, partition_size=P,
                     workspace=g.ws, err_flag=g.err, engine=engine_id, test_withhold_stage=hold)
        torch.cuda.synchronize()

    def scheduler_words_clear():
        # header (ticket, CTA count, dirty flag), then one split counter per
        # (sequence, KV head)
        hdr = g.ws[:256].view(torch.int32)
        cnt = g.ws[256:256 + 4 * S * w.num_kv_heads].view(torch.int32)
        return int(hdr[:3].abs().sum()) == 0 and int(cnt.abs().sum()) == 0

    t0 = time.time()
    decode(0)
    dt = time.time() - t0
    assert int(g.err.item()) == pa.PA_DEV_TIMEOUT
    assert 1.0 < dt < 30.0
    assert scheduler_words_clear()
    for _ in range(2):
        g.err.zero_()
        out.fill_(float("nan"))
        decode(-1)
        assert int(g.err.item()) == 0
        check_close(out_f64(out, w.dtype), st.out, w.dtype, "the call after a timed-out one")
        assert scheduler_words_clear()
