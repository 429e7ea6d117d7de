"""The seeded input recipes: deterministic, and shaped as stated."""
import math

import torch

import workloads


def test_deterministic():
    a, b = workloads.tiny_f32(), workloads.tiny_f32()
    assert a.free_order == b.free_order
    for k in a.kv:
        assert torch.equal(a.kv[k], b.kv[k])
    assert torch.equal(a.step_q[0], b.step_q[0])


def test_tiny_recipe():
    w = workloads.tiny_f32()
    assert w.meta["lens"] == [5, 17, 33, 48]
    assert sorted(w.free_order) == list(range(32)) and w.free_order != list(range(32))
    assert w.kv["k3"].shape == (47, 4, 64) and w.kv["k3"].dtype == torch.float32
    assert w.scale == 1 / 8


def test_mha_recipe():
    w = workloads.mha7b_f16(steps=32)
    L = w.meta["lens"]
    assert len(L) == 64 and min(L) >= 128 and max(L) <= 2048
    assert w.num_blocks == math.ceil(1.1 * sum(-(-(x - 1 + 32) // 16) for x in L))
    assert w.step_q[0].shape == (64, 32, 128) and w.step_q[0].dtype == torch.float16
    std = w.kv["k0"].float().std().item()
    assert 0.45 < std < 0.55


def test_gqa_recipe_same_values_both_block_sizes():
    a = workloads.gqa8b_bf16(block_size=16)
    b = workloads.gqa8b_bf16(block_size=32)
    assert a.meta["lens"] == b.meta["lens"]
    assert torch.equal(a.kv["k5"], b.kv["k5"]) and torch.equal(a.step_q[0], b.step_q[0])
    L = sorted(a.meta["lens"])
    assert L[0] >= 16 and L[-1] <= 8192 and 300 < L[len(L) // 2] < 800
    for w in (a, b):
        assert len(w.free_order) == math.ceil(0.4 * w.num_blocks)
        assert len(w.free_order) >= w.meta["blocks_needed"]
        assert len(set(w.free_order)) == len(w.free_order)


def test_prefix_recipe():
    w = workloads.prefix_f16()
    assert len(w.meta["lens"]) == 112 and w.step_q[0].shape[0] == 112
    assert len(w.meta["forkers"]) == 16
    assert all(0 <= s <= 256 for s in w.meta["suffix"])


def test_long_recipe_shapes_only():
    g = workloads._gen(workloads.BASE_SEED + 5)
    L = workloads._uniform_int(g, 32768, 131072, 8)
    assert all(32768 <= x <= 131072 for x in L)
