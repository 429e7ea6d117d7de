"""Memory accounting (host only): the blocks the library's allocator actually
hands out for a batch, against closed forms and against the oracle's own
block manager replaying the same script.

* Paged storage of a sequence of L tokens holds exactly ceil(L / bs) blocks:
  the waste is only the unfilled tail of the last block (the pages' "only the
  last block may be partially filled").
* A contiguous reservation of max_len slots per sequence wastes
  1 - sum(L) / (n * max_len).
* With a shared prefix and forked beams, shared blocks are held once: the
  block count equals the oracle manager's for the same script, and is far
  below the count with every prefix duplicated.
"""
import math
import os
import sys

import pytest

import oracle
import workloads

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
pa = pytest.importorskip("paged_kv_cache_426_b200")


def test_paged_blocks_are_the_minimum():
    import bench
    lens = [1, 16, 17, 33, 0, 200]
    rows = bench.waste_report("t", lens, (8, 16, 64), max_len=256)
    for r in rows:
        bs = r["block_size"]
        assert r["paged_blocks"] == sum(math.ceil(L / bs) for L in lens)
        assert r["paged_slots"] - r["tokens"] == sum((-L) % bs for L in lens)
        assert r["paged_waste"] == pytest.approx(1 - sum(lens) / r["paged_slots"], abs=1e-4)
        assert r["contiguous_waste"] == pytest.approx(1 - sum(lens) / (len(lens) * 256), abs=1e-4)


def _oracle_blocks(w, duplicate):
    """Blocks held after the script's prefill, by the oracle's manager."""
    alloc = oracle.BlockAllocator(1 << 16)
    mgr = oracle.BlockManager(alloc, w.block_size)
    lengths = {}
    for op in w.ops:
        if op[0] == "add":
            mgr.add_seq(op[1])
            lengths[op[1]] = 0
        elif op[0] == "fork":
            if duplicate:
                mgr.add_seq(op[2])
                for _ in range(lengths[op[1]]):
                    mgr.append(op[2])
            else:
                mgr.fork(op[1], op[2])
            lengths[op[2]] = lengths[op[1]]
        elif op[0] == "write":
            for _ in range(w.kv["k" + op[2]].shape[0]):
                mgr.append(op[1])
            lengths[op[1]] += w.kv["k" + op[2]].shape[0]
        elif op[0] == "step":
            break
    return alloc.num_blocks - alloc.num_free()


def test_sharing_matches_oracle_manager():
    import bench
    w = workloads.prefix_f16(n_req=6, plen=64, suffix_max=40, n_fork=2, heads=4)
    r = bench.sharing_report(w)
    assert r["blocks_shared"] == _oracle_blocks(w, duplicate=False)
    assert r["blocks_duplicated"] == _oracle_blocks(w, duplicate=True)
    assert r["blocks_shared"] < r["blocks_duplicated"]
    assert r["memory_saved"] == pytest.approx(1 - r["blocks_shared"] / r["blocks_duplicated"], abs=1e-4)
