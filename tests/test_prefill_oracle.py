"""Pins for the prefill oracle (no GPU): each ties it to something other than
itself.

* A whole prompt (chunk = the sequence) is causal self-attention: it must
  equal torch's scaled_dot_product_attention(is_causal=True) in float64 over
  the contiguous (never paged) K/V, with the query heads of a group reading
  the same KV head.
* A chunk of the last n tokens is the last n rows of that full causal
  product (the mask is aligned at the end of the sequence).
* n = 1 is a decode step: bit-identical to the decode oracle.
* Closed forms: the first prompt position sees only token 0 (output = V_0
  exactly); keys that are all equal give uniform weights (output = running
  mean of V); a KV head whose V rows are all c gives exactly c to every query
  head of its group.
* Invariance: the physical block ids are irrelevant (two different free
  orders give bit-identical outputs).

A plausible slip in the oracle (K[:p] for K[:p+1], the chunk aligned at the
start of the sequence, h % Hkv for h // G, a missing scale, a transposed
product) fails at least one of these.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import BlockAllocator, BlockManager
from workloads import DTYPES


def _paged(Ks, Vs, bs, dtype, seed, extra_blocks=3):
    """Write each sequence's K/V rows [L, Hkv, D] (storage dtype) into a
    fresh paged cache through the oracle's manager; returns caches, tables."""
    hkv, d = Ks[0].shape[1], Ks[0].shape[2]
    need = sum(-(-k.shape[0] // bs) for k in Ks)
    nb = need + extra_blocks
    order = np.random.default_rng(seed).permutation(nb).tolist()
    mgr = BlockManager(BlockAllocator(nb, order), bs)
    kc = oracle.empty_cache(nb, hkv, bs, d, dtype)
    vc = oracle.empty_cache(nb, hkv, bs, d, dtype)
    for s, (K, V) in enumerate(zip(Ks, Vs)):
        mgr.add_seq(s)
        slots = [mgr.append(s)[0] for _ in range(K.shape[0])]
        oracle.reshape_and_cache(kc, vc, K, V, slots)
    rows, lens = mgr.table_rows(list(range(len(Ks))), max(1, need))
    return kc, vc, np.asarray(rows, dtype=np.int32), lens


def _rand(rng, shape, dtype="f32"):
    x = torch.from_numpy(rng.standard_normal(shape).astype(np.float32))
    return oracle.as_storage(x.to(DTYPES[dtype]), dtype)


def _sdpa_full(q, K, V, scale, G):
    """Causal attention of all L rows by torch (float64): q [L, Hq, D],
    K, V [L, Hkv, D] -> [L, Hq, D]."""
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]                       # [1, Hq, L, D]
    kt = torch.from_numpy(K).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    vt = torch.from_numpy(V).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


def _cu(ns):
    return np.concatenate([[0], np.cumsum(ns)]).astype(np.int32)


@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 2)])
def test_whole_prompt_and_chunks_match_torch_causal_sdpa(hq, hkv):
    rng = np.random.default_rng(1)
    D, bs, G = 16, 8, hq // hkv
    Ls, ns = [37, 70, 1, 24], [37, 23, 1, 5]
    fullq = [_rand(rng, (L, hq, D)) for L in Ls]
    Ks = [_rand(rng, (L, hkv, D)) for L in Ls]
    Vs = [_rand(rng, (L, hkv, D)) for L in Ls]
    kc, vc, tab, lens = _paged(Ks, Vs, bs, "f32", 7)
    q = np.concatenate([fq[L - n:] for fq, L, n in zip(fullq, Ls, ns)])
    scale = 0.3
    out = oracle.paged_prefill(q, kc, vc, tab, lens, _cu(ns), scale, "f32")
    a = 0
    for fq, K, V, L, n in zip(fullq, Ks, Vs, Ls, ns):
        ref = _sdpa_full(fq.astype(np.float64), K.astype(np.float64), V.astype(np.float64), scale, G)
        np.testing.assert_allclose(out[a:a + n], ref[L - n:], rtol=0, atol=1e-12)
        a += n


def test_single_row_is_the_decode_oracle():
    rng = np.random.default_rng(2)
    hq, hkv, D, bs = 8, 2, 32, 16
    Ls = [1, 16, 17, 90]
    Ks = [_rand(rng, (L, hkv, D), "bf16") for L in Ls]
    Vs = [_rand(rng, (L, hkv, D), "bf16") for L in Ls]
    kc, vc, tab, lens = _paged(Ks, Vs, bs, "bf16", 3)
    q = _rand(rng, (len(Ls), hq, D), "bf16")
    pre = oracle.paged_prefill(q, kc, vc, tab, lens, _cu([1] * len(Ls)), 0.125, "bf16")
    dec = oracle.paged_decode(q, kc, vc, tab, lens, 0.125, "bf16")
    assert np.array_equal(pre, dec)


def test_first_position_is_v0_and_equal_keys_give_running_mean():
    rng = np.random.default_rng(3)
    hq = hkv = 2
    D, bs, L = 8, 4, 19
    K1 = _rand(rng, (1, hkv, D))
    K = np.repeat(K1, L, axis=0)                                # every key equal
    V = _rand(rng, (L, hkv, D))
    kc, vc, tab, lens = _paged([K], [V], bs, "f32", 5)
    q = _rand(rng, (L, hq, D))
    out = oracle.paged_prefill(q, kc, vc, tab, lens, _cu([L]), 1.0, "f32")
    V64 = V.astype(np.float64)
    assert np.array_equal(out[0], V64[0])                       # one key: weight exactly 1
    running = np.cumsum(V64, axis=0) / np.arange(1, L + 1)[:, None, None]
    np.testing.assert_allclose(out, running, rtol=0, atol=1e-12)


def test_group_reads_its_own_kv_head():
    rng = np.random.default_rng(4)
    hq, hkv, D, bs, L, n = 8, 4, 8, 8, 21, 9
    G = hq // hkv
    K = _rand(rng, (L, hkv, D))
    V = np.empty((L, hkv, D), np.float32)
    for j in range(hkv):
        V[:, j, :] = 0.5 * (j + 1)                              # exact in every dtype
    kc, vc, tab, lens = _paged([K], [V], bs, "f32", 9)
    q = _rand(rng, (n, hq, D))
    out = oracle.paged_prefill(q, kc, vc, tab, lens, _cu([n]), 0.5, "f32")
    for h in range(hq):
        np.testing.assert_allclose(out[:, h, :], 0.5 * (h // G + 1), rtol=0, atol=1e-15)


def test_physical_block_ids_do_not_matter():
    rng = np.random.default_rng(5)
    hq, hkv, D, bs = 4, 2, 16, 8
    Ls, ns = [29, 50], [11, 50]
    Ks = [_rand(rng, (L, hkv, D), "f16") for L in Ls]
    Vs = [_rand(rng, (L, hkv, D), "f16") for L in Ls]
    q = _rand(rng, (sum(ns), hq, D), "f16")
    outs = []
    for seed in (11, 12):
        kc, vc, tab, lens = _paged(Ks, Vs, bs, "f16", seed, extra_blocks=6)
        outs.append(oracle.paged_prefill(q, kc, vc, tab, lens, _cu(ns), 0.25, "f16"))
    assert np.array_equal(outs[0], outs[1])


def test_empty_chunk_and_bad_chunk():
    rng = np.random.default_rng(6)
    K = _rand(rng, (10, 1, 8))
    V = _rand(rng, (10, 1, 8))
    kc, vc, tab, lens = _paged([K, K], [V, V], 4, "f32", 1)
    q = _rand(rng, (3, 1, 8))
    out = oracle.paged_prefill(q, kc, vc, tab, lens, np.array([0, 0, 3], np.int32), 1.0, "f32")
    assert out.shape == (3, 1, 8)
    with pytest.raises(ValueError):
        oracle.prefill_rows(_rand(rng, (11, 1, 8)), kc, vc, tab[0], 10, 11, 1.0, 0, "f32")
