"""Pins for the oracle: each check ties it to something other than itself.

* the pages' worked examples (block tables of the velog trace, the vLLM study
  note's diagram, the 119-ai-studio flowchart, the velog beam-sharing example),
  stored under tests/golden with their citations;
* hand-derived closed forms of softmax attention (tests/golden);
* brute force on tiny inputs: a pure-Python attention over the logical
  (never paged) K/V, without max subtraction, with exactly rounded sums;
* special cases and invariants (one token, zero query, constant V, dominant
  logit, GQA = MHA with repeated KV heads, physical-permutation and block-size
  invariance, refcounts back to zero, only the last block partly filled).
"""
import math
import random

import numpy as np
import pytest
import torch

import oracle
from oracle import BlockAllocator, BlockManager, BlockStateError, OutOfBlocks
from tests.conftest import golden

# --------------------------------------------------------------------------
# block tables against the pages' examples


def _manager(fx):
    return BlockManager(BlockAllocator(fx["num_blocks"], fx["free_order"]), fx["block_size"])


def test_velog_growth_trace():
    fx = golden("velog_growth_trace.json")
    m = _manager(fx)
    m.add_seq(0)
    want = {e["tokens"]: e["table"] for e in fx["expect"]}
    growth = []
    for n in range(1, 49):
        before = len(m.tables[0])
        m.append(0)
        if len(m.tables[0]) != before:
            growth.append(n)
        if n in want:
            assert m.tables[0] == want[n], n
    assert growth == fx["growth_at_tokens"]


def test_velog_beam_sharing():
    fx = golden("velog_beam_sharing.json")
    m = _manager(fx)
    m.add_seq("A")
    cows = []
    for _ in range(fx["prompt_tokens"]):
        _, c = m.append("A")
        assert c is None
    m.fork("A", "B")
    for s in ("A", "B"):
        _, c = m.append(s)
        if c:
            cows.append(list(c))
    assert m.tables["A"] == fx["expect_tables"]["A"]
    assert m.tables["B"] == fx["expect_tables"]["B"]
    for b, rc in fx["expect_refcounts"].items():
        assert m.alloc.refcount[int(b)] == rc
    assert cows == fx["expect_cow_pairs"]
    m.free_seq("A")
    m.free_seq("B")
    assert all(rc == 0 for rc in m.alloc.refcount)
    assert m.alloc.num_free() == fx["num_blocks"]


def test_vllm_diagram_tables():
    fx = golden("vllm_diagram_tables.json")
    m = _manager(fx)
    m.add_seq("A")
    m.add_seq("B")
    a, b = fx["tokens"]["A"], fx["tokens"]["B"]
    for i in range(max(a, b)):
        if i < a:
            m.append("A")
        if i < b:
            m.append("B")
    assert m.tables["A"] == fx["expect_tables"]["A"]
    assert m.tables["B"] == fx["expect_tables"]["B"]


def test_ai119_table_and_gather_roundtrip():
    fx = golden("ai119_block_table.json")
    m = _manager(fx)
    m.add_seq(0)
    bs, n, hkv, d = fx["block_size"], fx["tokens"], 2, 8
    slots = np.array([m.append(0)[0] for _ in range(n)])
    assert m.tables[0] == fx["expect_table"]
    rng = np.random.default_rng(5)
    K = rng.standard_normal((n, hkv, d)).astype(np.float32)
    V = rng.standard_normal((n, hkv, d)).astype(np.float32)
    kc = oracle.empty_cache(fx["num_blocks"], hkv, bs, d, "f32")
    vc = oracle.empty_cache(fx["num_blocks"], hkv, bs, d, "f32")
    oracle.reshape_and_cache(kc, vc, K, V, slots)
    for j in range(hkv):
        assert np.array_equal(oracle.gather_kv(kc, m.tables[0], n, j), K[:, j])
        assert np.array_equal(oracle.gather_kv(vc, m.tables[0], n, j), V[:, j])
    # the table order is not the physical order: a gather through a sorted
    # table must differ (the indirection is really used)
    assert not np.array_equal(oracle.gather_kv(kc, sorted(m.tables[0]), n, 0), K[:, 0])


# --------------------------------------------------------------------------
# allocator behaviour


def test_allocator_fifo_errors_and_outside_holders():
    a = BlockAllocator(4, [2, 0])
    assert a.refcount == [0, 1, 0, 1]          # 1 and 3 held by an outside owner
    assert a.allocate_block() == 2
    assert a.allocate_block() == 0
    with pytest.raises(OutOfBlocks):
        a.allocate_block()
    a.free_block(3)                             # the outside owner lets go
    a.free_block(2)
    assert list(a.free) == [3, 2]               # freed blocks join at the back
    with pytest.raises(BlockStateError):
        a.free_block(2)                         # double free
    with pytest.raises(BlockStateError):
        a.incref(2)                             # sharing a free block
    with pytest.raises(ValueError):
        BlockAllocator(4, [1, 1])


def test_cow_on_shared_partial_block():
    """Reading: writing into a shared, partly filled last block copies it first;
    the last remaining holder writes in place."""
    m = BlockManager(BlockAllocator(8), 16)
    m.add_seq(0)
    for _ in range(20):                         # blocks 0 (full), 1 (4 of 16)
        m.append(0)
    m.fork(0, 1)
    m.fork(0, 2)
    assert m.alloc.refcount[:2] == [3, 3]
    slot0, c0 = m.append(0)
    assert c0 == (1, 2) and m.tables[0] == [0, 2] and slot0 == 2 * 16 + 4
    slot1, c1 = m.append(1)
    assert c1 == (1, 3) and m.tables[1] == [0, 3] and slot1 == 3 * 16 + 4
    slot2, c2 = m.append(2)
    assert c2 is None and m.tables[2] == [0, 1] and slot2 == 1 * 16 + 4
    assert m.alloc.refcount[:4] == [3, 1, 1, 1]


def _check_invariants(m):
    bs = m.bs
    holders = {}
    for s, t in m.tables.items():
        assert len(t) == -(-m.lens[s] // bs)    # only the last block may be partial
        for b in t:
            holders[b] = holders.get(b, 0) + 1
    for b, n in holders.items():
        assert m.alloc.refcount[b] == n         # shared only with refcount >= 2
    allocated = sum(1 for rc in m.alloc.refcount if rc > 0)
    assert allocated + m.alloc.num_free() == m.alloc.num_blocks


def test_random_script_invariants_and_refcounts_return_to_zero():
    rnd = random.Random(7)
    m = BlockManager(BlockAllocator(400, rnd.sample(range(400), 400)), 8)
    live, nxt = [], 0
    for _ in range(3000):
        r = rnd.random()
        if r < 0.05 or not live:
            m.add_seq(nxt)
            live.append(nxt)
            nxt += 1
        elif r < 0.10:
            p = rnd.choice(live)
            m.fork(p, nxt)
            live.append(nxt)
            nxt += 1
        elif r < 0.14:
            s = rnd.choice(live)
            m.free_seq(s)
            live.remove(s)
        else:
            s = rnd.choice(live)
            try:
                m.append(s)
            except OutOfBlocks:
                s = rnd.choice(live)
                m.free_seq(s)
                live.remove(s)
        _check_invariants(m)
    for s in list(live):
        m.free_seq(s)
    assert all(rc == 0 for rc in m.alloc.refcount)
    assert m.alloc.num_free() == 400


# --------------------------------------------------------------------------
# cache write / copy against the hand-written example


def test_cache_write_and_copy_tiny():
    fx = golden("cache_write_tiny.json")
    shape = (fx["num_blocks"], fx["num_kv_heads"], fx["block_size"], fx["head_dim"])
    kc = oracle.empty_cache(*shape, "f32")
    vc = oracle.empty_cache(*shape, "f32")
    k = np.array(fx["k"], np.float32)
    v = np.array(fx["v"], np.float32)
    oracle.reshape_and_cache(kc, vc, k, v, fx["slot_mapping"])
    assert np.array_equal(kc, np.array(fx["expect_key_cache"], np.float32))
    assert np.array_equal(vc, np.array(fx["expect_value_cache"], np.float32))
    oracle.copy_blocks(kc, vc, fx["copy_pairs"])
    assert np.array_equal(kc, np.array(fx["expect_key_cache_after_copy"], np.float32))


def test_cache_write_keeps_bits_and_canary():
    """bf16 values travel as raw bits; untouched slots keep the canary."""
    kc = oracle.empty_cache(4, 1, 4, 8, "bf16", fill=0xDEAD)
    vc = oracle.empty_cache(4, 1, 4, 8, "bf16", fill=0xBEEF)
    k = np.arange(16, dtype=np.uint16).reshape(2, 1, 8) + 0x7F80 - 8   # incl. inf/NaN bits
    oracle.reshape_and_cache(kc, vc, k, k, [13, -1])
    assert np.array_equal(kc[3, 0, 1], k[0, 0])
    mask = np.ones(kc.shape, bool)
    mask[3, 0, 1] = False
    assert (kc[mask] == 0xDEAD).all() and (vc[mask] == 0xBEEF).all()


def test_to_f64_exact():
    bits = np.array([0x3F80, 0xC000, 0x0001, 0x7F7F], np.uint16)   # 1, -2, min subnormal, max
    want = [1.0, -2.0, 2.0 ** -133, (2 - 2 ** -7) * 2.0 ** 127]
    assert oracle.to_f64(bits, "bf16").tolist() == want
    h = np.array([1.0, 65504.0, 2 ** -24], np.float16)
    assert oracle.to_f64(h, "f16").tolist() == [1.0, 65504.0, 2.0 ** -24]
    t = torch.tensor([1.0, -3.5, 2.0 ** -126], dtype=torch.bfloat16)
    assert oracle.to_f64(oracle.as_storage(t, "bf16"), "bf16").tolist() == [1.0, -3.5, 2.0 ** -126]


# --------------------------------------------------------------------------
# attention: closed forms


@pytest.mark.parametrize("case", golden("attention_closed_forms.json")["cases"],
                         ids=lambda c: c["name"])
def test_attention_closed_forms(case):
    q = np.array(case["q"])
    K, V = np.array(case["K"]), np.array(case["V"])
    out = oracle.attend(q, K, V, case["scale"])
    assert np.allclose(out, case["out"], rtol=0, atol=1e-12)


def _paged_from_logical(K, V, bs, rnd, extra_blocks=3, dtype="f32"):
    """Place logical per-sequence K/V [L, Hkv, D] into a shuffled pool through
    the oracle's own manager.  Returns caches, tables, lens."""
    L = [k.shape[0] for k in K]
    need = sum(-(-x // bs) for x in L) + extra_blocks
    order = list(range(need))
    rnd.shuffle(order)
    m = BlockManager(BlockAllocator(need, order), bs)
    hkv, d = K[0].shape[1], K[0].shape[2]
    kc = oracle.empty_cache(need, hkv, bs, d, dtype)
    vc = oracle.empty_cache(need, hkv, bs, d, dtype)
    for s in range(len(K)):
        m.add_seq(s)
        slots = [m.append(s)[0] for _ in range(L[s])]
        oracle.reshape_and_cache(kc, vc, K[s], V[s], slots)
    mb = max(1, max(-(-x // bs) for x in L))
    rows, lens = m.table_rows(range(len(K)), mb)
    return kc, vc, np.array(rows, np.int32), np.array(lens, np.int32)


def test_gqa_grouping_golden():
    fx = golden("attention_closed_forms.json")["gqa_grouping"]
    rnd = random.Random(1)
    hkv, T = fx["num_kv_heads"], fx["tokens"]
    Vc = np.array(fx["V_per_kv_head"], np.float32)
    K = [np.random.default_rng(3).standard_normal((T, hkv, 2)).astype(np.float32)]
    V = [np.broadcast_to(Vc, (T, hkv, 2)).copy()]
    kc, vc, tab, lens = _paged_from_logical(K, V, 2, rnd)
    q = np.random.default_rng(4).standard_normal((1, fx["num_q_heads"], 2)).astype(np.float32)
    out = oracle.paged_decode(q, kc, vc, tab, lens, 0.7, "f32")
    assert np.allclose(out[0], fx["out"], rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# attention: brute force on tiny inputs


def _brute(qv, keys, vals, scale):
    """Pure Python, no max subtraction, exactly rounded sums (math.fsum)."""
    e = [math.exp(scale * math.fsum(a * b for a, b in zip(qv, k))) for k in keys]
    z = math.fsum(e)
    return [math.fsum(et * v[dd] for et, v in zip(e, vals)) / z for dd in range(len(vals[0]))]


@pytest.mark.parametrize("seed", range(6))
def test_paged_decode_vs_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    rnd = random.Random(seed)
    S, hkv, G, D = 3, 2, 2 + seed % 2, 8
    bs = [2, 4, 8][seed % 3]
    L = [int(x) for x in rng.integers(1, 40, S)]
    K = [rng.standard_normal((n, hkv, D)).astype(np.float32) for n in L]
    V = [rng.standard_normal((n, hkv, D)).astype(np.float32) for n in L]
    q = rng.standard_normal((S, hkv * G, D)).astype(np.float32)
    scale = 1 / math.sqrt(D)
    kc, vc, tab, lens = _paged_from_logical(K, V, bs, rnd)
    out = oracle.paged_decode(q, kc, vc, tab, lens, scale, "f32")
    for s in range(S):
        for h in range(hkv * G):
            j = h // G
            want = _brute(q[s, h].astype(float).tolist(), K[s][:, j].astype(float).tolist(),
                          V[s][:, j].astype(float).tolist(), scale)
            assert np.allclose(out[s, h], want, rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# attention: special cases and invariants


def _rand_case(seed, L, hkv=2, G=2, D=16, bs=4, dtype="f32"):
    rng = np.random.default_rng(seed)
    K = [rng.standard_normal((n, hkv, D)).astype(np.float32) for n in L]
    V = [rng.standard_normal((n, hkv, D)).astype(np.float32) for n in L]
    q = rng.standard_normal((len(L), hkv * G, D)).astype(np.float32)
    return q, K, V


def test_single_token_returns_its_value_exactly():
    q, K, V = _rand_case(1, [1, 1])
    kc, vc, tab, lens = _paged_from_logical(K, V, 4, random.Random(0))
    out = oracle.paged_decode(q, kc, vc, tab, lens, 0.3, "f32")
    for s in range(2):
        for h in range(4):
            assert np.array_equal(out[s, h], V[s][0, h // 2].astype(np.float64))


def test_zero_query_and_equal_keys_give_mean_value():
    q, K, V = _rand_case(2, [7, 30])
    kc, vc, tab, lens = _paged_from_logical(K, V, 4, random.Random(0))
    out0 = oracle.paged_decode(np.zeros_like(q), kc, vc, tab, lens, 0.3, "f32")
    Keq = [np.broadcast_to(k[:1], k.shape).copy() for k in K]
    kc2, vc2, tab2, lens2 = _paged_from_logical(Keq, V, 4, random.Random(0))
    out1 = oracle.paged_decode(q, kc2, vc2, tab2, lens2, 0.3, "f32")
    for s in range(2):
        for h in range(4):
            mean = V[s][:, h // 2].astype(np.float64).mean(axis=0)
            assert np.allclose(out0[s, h], mean, rtol=1e-13, atol=1e-14)
            assert np.allclose(out1[s, h], mean, rtol=1e-13, atol=1e-14)


def test_constant_value_is_returned():
    q, K, V = _rand_case(3, [9, 33])
    V = [np.full_like(v, -2.5) for v in V]
    kc, vc, tab, lens = _paged_from_logical(K, V, 8, random.Random(0))
    out = oracle.paged_decode(q * 4, kc, vc, tab, lens, 1.0, "f32")
    assert np.allclose(out, -2.5, rtol=0, atol=1e-14)


def test_dominant_logit_selects_its_value():
    D, L, t_star = 4, 20, 13
    rng = np.random.default_rng(9)
    K = rng.standard_normal((L, 1, D)).astype(np.float32) * 0.01
    K[t_star, 0] = [50.0, 0, 0, 0]
    V = rng.standard_normal((L, 1, D)).astype(np.float32)
    q = np.array([[[1.0, 0, 0, 0]]], np.float32)
    kc, vc, tab, lens = _paged_from_logical([K], [V], 4, random.Random(0))
    out = oracle.paged_decode(q, kc, vc, tab, lens, 1.0, "f32")
    assert np.allclose(out[0, 0], V[t_star, 0], rtol=0, atol=1e-18 + 25 * math.exp(-49))


def test_gqa_equals_mha_with_repeated_kv():
    G = 4
    q, K, V = _rand_case(4, [5, 22, 17], hkv=2, G=G)
    kc, vc, tab, lens = _paged_from_logical(K, V, 4, random.Random(0))
    out_gqa = oracle.paged_decode(q, kc, vc, tab, lens, 0.25, "f32")
    Kr = [np.repeat(k, G, axis=1) for k in K]
    Vr = [np.repeat(v, G, axis=1) for v in V]
    kc2, vc2, tab2, lens2 = _paged_from_logical(Kr, Vr, 4, random.Random(1))
    out_mha = oracle.paged_decode(q, kc2, vc2, tab2, lens2, 0.25, "f32")
    assert np.allclose(out_gqa, out_mha, rtol=1e-14, atol=1e-15)


def test_invariant_under_physical_permutation_and_block_size():
    q, K, V = _rand_case(5, [1, 16, 17, 31, 64])
    ref = None
    for bs, seed in [(4, 0), (4, 1), (8, 2), (16, 3), (2, 4)]:
        kc, vc, tab, lens = _paged_from_logical(K, V, bs, random.Random(seed))
        out = oracle.paged_decode(q, kc, vc, tab, lens, 0.25, "f32")
        if ref is None:
            ref = out
        assert np.array_equal(out, ref)      # same gathered arrays, same arithmetic


def test_zero_length_gives_zeros():
    q, K, V = _rand_case(6, [3])
    kc, vc, tab, lens = _paged_from_logical(K, V, 4, random.Random(0))
    lens = np.array([0], np.int32)
    assert not oracle.paged_decode(q, kc, vc, tab, lens, 1.0, "f32").any()


def test_planted_mistakes_are_caught():
    """A wrong KV-head map, a dropped max shift overflow, a transposed operand
    and a dropped token each change the output of a tiny case."""
    q, K, V = _rand_case(8, [6], hkv=2, G=2, D=4)
    kc, vc, tab, lens = _paged_from_logical(K, V, 2, random.Random(0))
    good = oracle.paged_decode(q, kc, vc, tab, lens, 0.5, "f32")
    qh = q[0].astype(np.float64)
    Kf, Vf = K[0].astype(np.float64), V[0].astype(np.float64)
    wrong_map = np.stack([oracle.attend(qh[h:h + 1], Kf[:, h % 2], Vf[:, h % 2], 0.5)[0]
                          for h in range(4)])
    dropped = np.stack([oracle.attend(qh[h:h + 1], Kf[:-1, h // 2], Vf[:-1, h // 2], 0.5)[0]
                        for h in range(4)])
    swapped = np.stack([oracle.attend(qh[h:h + 1], Vf[:, h // 2], Kf[:, h // 2], 0.5)[0]
                        for h in range(4)])
    for bad in (wrong_map, dropped, swapped):
        assert not np.allclose(bad, good[0], atol=1e-6)


# --------------------------------------------------------------------------
# the oracle's workload runner


def test_runner_prefix_scenario_cow_count_and_sharing():
    import workloads
    w = workloads.prefix_f16()
    r = oracle.run(w, decode=False)
    st = r.steps[0]
    suffix, forkers = w.meta["suffix"], w.meta["forkers"]
    partial = [f for f in forkers if suffix[f] % 16]
    assert len(st.cow_pairs) == 3 * len(partial)
    # the 64 prefix blocks are shared by all 112 sequences and stored once
    pre = st.block_tables[:, :64]
    assert (pre == pre[0]).all()
    assert all(r.manager.alloc.refcount[b] == 112 for b in pre[0])
    assert list(st.context_lens) == w.meta["lens"]


def test_runner_tiny_matches_recipe():
    import workloads
    w = workloads.tiny_f32()
    r = oracle.run(w)
    st = r.steps[0]
    assert list(st.context_lens) == [5, 17, 33, 48]
    # only the last block partly filled; the positions 16 and 32 open new blocks
    assert [int((row >= 0).sum()) for row in st.block_tables] == [1, 2, 3, 3]
    # the step's slots point at the last token of each sequence
    for b, s in enumerate(st.seqs):
        L = st.context_lens[b]
        assert st.slot_mapping[b] == st.block_tables[b][(L - 1) // 16] * 16 + (L - 1) % 16
