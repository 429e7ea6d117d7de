"""Oracle: run a workload's host script with the oracle's own manager.

TEST INFRASTRUCTURE ONLY.  Nothing in the product imports this module.

Interprets ``workloads.Workload.ops`` (add / write / fork / step) with
``oracle.blocks.BlockManager`` and the cache operations of ``oracle.cache``,
and records, per decode step, the slot mapping, the copy-on-write pairs, the
block tables and lengths handed to attention, and (optionally) the float64
attention output.  Within a step the copies happen before the writes, and
both before attention, as in the CUDA path.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from .attention import paged_decode
from .blocks import BlockAllocator, BlockManager
from .cache import as_storage, copy_blocks, empty_cache, reshape_and_cache
from .prefill import paged_prefill, prefill_rows


@dataclass
class StepRecord:
    seqs: list
    slot_mapping: np.ndarray          # int64 [S]
    cow_pairs: list                   # [(src, dst)]
    block_tables: np.ndarray          # int32 [S, max_blocks], -1 padded
    context_lens: np.ndarray          # int32 [S]
    out: np.ndarray | None = None     # float64 [S, Hq, D]


@dataclass
class OracleRun:
    key_cache: np.ndarray
    value_cache: np.ndarray
    manager: BlockManager
    prefill_slots: dict = field(default_factory=dict)   # (seq, key) -> int64 slots
    prefill_cows: list = field(default_factory=list)
    steps: list = field(default_factory=list)
    prefill_key_cache: np.ndarray | None = None
    prefill_value_cache: np.ndarray | None = None


def max_blocks_needed(w) -> int:
    return max(1, -(-(max(w.meta["lens"]) - 1 + w.num_steps) // w.block_size))


def run(w, *, decode=True, steps=None, max_blocks=None, canary=0,
        keep_prefill_cache=False, decode_steps=None) -> OracleRun:
    """Execute the script.  ``steps``: how many decode steps to run (default all);
    ``decode``: compute the float64 outputs of each step; ``decode_steps``
    (optional set of step indices): compute them for those steps only, each
    from the cache as it stands at that step."""
    alloc = BlockAllocator(w.num_blocks, w.free_order)
    mgr = BlockManager(alloc, w.block_size)
    kc = empty_cache(w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim, w.dtype, canary)
    vc = empty_cache(w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim, w.dtype, canary)
    rec = OracleRun(kc, vc, mgr)
    mb = max_blocks if max_blocks is not None else max_blocks_needed(w)
    n_steps = w.num_steps if steps is None else steps
    first_step = True
    for op in w.ops:
        if op[0] == "add":
            mgr.add_seq(op[1])
        elif op[0] == "fork":
            mgr.fork(op[1], op[2])
        elif op[0] == "write":
            seq, key = op[1], op[2]
            K = as_storage(w.kv["k" + key], w.dtype)
            V = as_storage(w.kv["v" + key], w.dtype)
            slots = np.empty(K.shape[0], dtype=np.int64)
            for i in range(K.shape[0]):
                slots[i], cow = mgr.append(seq)
                if cow is not None:
                    copy_blocks(kc, vc, [cow])
                    rec.prefill_cows.append(cow)
            reshape_and_cache(kc, vc, K, V, slots)
            rec.prefill_slots[(seq, key)] = slots
        elif op[0] == "step":
            seqs, k = op[1], op[2]
            if k >= n_steps:
                continue
            if first_step and keep_prefill_cache:
                rec.prefill_key_cache = kc.copy()
                rec.prefill_value_cache = vc.copy()
            first_step = False
            slots = np.empty(len(seqs), dtype=np.int64)
            cows = []
            for b, s in enumerate(seqs):
                slots[b], cow = mgr.append(s)
                if cow is not None:
                    cows.append(cow)
            copy_blocks(kc, vc, cows)
            reshape_and_cache(kc, vc, as_storage(w.step_k[k], w.dtype),
                              as_storage(w.step_v[k], w.dtype), slots)
            rows, lens = mgr.table_rows(seqs, mb)
            st = StepRecord(list(seqs), slots, cows, np.asarray(rows, np.int32),
                            np.asarray(lens, np.int32))
            if decode and (decode_steps is None or k in decode_steps):
                st.out = paged_decode(as_storage(w.step_q[k], w.dtype), kc, vc,
                                      st.block_tables, st.context_lens, w.scale, w.dtype)
            rec.steps.append(st)
        else:
            raise ValueError(f"unknown op {op[0]}")
    return rec


@dataclass
class PrefillRecord:
    key_cache: np.ndarray
    value_cache: np.ndarray
    context_slots: list               # per sequence: int64 slots of the tokens before the chunk
    chunk_slots: np.ndarray           # int64 [sum(query_lens)], the chunk's slots packed
    block_tables: np.ndarray          # int32 [S, max_blocks], -1 padded
    context_lens: np.ndarray          # int32 [S]
    cu_seqlens_q: np.ndarray          # int32 [S + 1]
    out: np.ndarray | None = None     # float64 [sum(query_lens), Hq, D] (rows asked for)


def run_prefill(b, *, rows=None, compute=True, canary=0) -> PrefillRecord:
    """Replay a ``workloads.PrefillBatch``: every sequence takes its
    context_lens[s] slots from a fresh manager (FIFO pool), the tokens before
    the chunk are written, then the chunk's, then causal attention.  ``rows``
    (optional): {seq: [chunk rows]} to compute only those rows (others zero)."""
    alloc = BlockAllocator(b.num_blocks, b.free_order)
    mgr = BlockManager(alloc, b.block_size)
    kc = empty_cache(b.num_blocks, b.num_kv_heads, b.block_size, b.head_dim, b.dtype, canary)
    vc = empty_cache(b.num_blocks, b.num_kv_heads, b.block_size, b.head_dim, b.dtype, canary)
    ctx_slots, chunk_slots = [], []
    for s, (L, n) in enumerate(zip(b.context_lens, b.query_lens)):
        mgr.add_seq(s)
        slots = np.array([mgr.append(s)[0] for _ in range(L)], dtype=np.int64)
        k, v = as_storage(b.k[s], b.dtype), as_storage(b.v[s], b.dtype)
        reshape_and_cache(kc, vc, k[:L - n], v[:L - n], slots[:L - n])
        ctx_slots.append(slots[:L - n])
        chunk_slots.append(slots[L - n:])
    for s, (L, n) in enumerate(zip(b.context_lens, b.query_lens)):
        k, v = as_storage(b.k[s], b.dtype), as_storage(b.v[s], b.dtype)
        reshape_and_cache(kc, vc, k[L - n:], v[L - n:], chunk_slots[s])
    S = len(b.context_lens)
    mb = max(1, max(-(-L // b.block_size) for L in b.context_lens))
    tab, lens = mgr.table_rows(list(range(S)), mb)
    cu = np.asarray(b.query_offsets, dtype=np.int32)
    rec = PrefillRecord(kc, vc, ctx_slots,
                        np.concatenate(chunk_slots) if chunk_slots else np.zeros(0, np.int64),
                        np.asarray(tab, dtype=np.int32), np.asarray(lens, dtype=np.int32), cu)
    if compute:
        q = as_storage(b.q, b.dtype)
        if rows is None:
            rec.out = paged_prefill(q, kc, vc, rec.block_tables, rec.context_lens, cu, b.scale,
                                    b.dtype)
        else:
            hkv, G = b.num_kv_heads, b.num_q_heads // b.num_kv_heads
            rec.out = np.zeros((int(cu[-1]), b.num_q_heads, b.head_dim))
            for s, rs in rows.items():
                a, e = int(cu[s]), int(cu[s + 1])
                for j in range(hkv):
                    o = prefill_rows(q[a:e], kc, vc, rec.block_tables[s], int(rec.context_lens[s]),
                                     e - a, b.scale, j, b.dtype, rows=rs)
                    rec.out[a:e, j * G:(j + 1) * G] = o
    return rec
