"""Oracle: the paged KV cache's contents (write, copy, gather).

TEST INFRASTRUCTURE ONLY.  Nothing in the product imports this module.

The cache holds, per physical block b, KV head h and in-block offset o, one
token row of ``head_dim`` values: ``cache[b, h, o, :]`` (a layout choice of
this library: one (block, head) tile is ``block_size * head_dim`` contiguous
elements).  Values are kept in their storage type at bit level:
float32 -> np.float32, float16 -> np.float16, bfloat16 -> np.uint16 (bits).

Sources (page title, section):
* "09. PagedAttention" (119-ai-studio), 해법: 페이지처럼 나눠 담기: the KV cache
  is cut into fixed-size blocks; a request's tokens are spread over them and
  the block table maps logical block -> physical block.
* "Paged Attention" (velog @junegood), 주요 구성 요소 (블록 테이블): the table is
  the page table of this scheme; physical blocks need not be contiguous.
* "KV Cache & PagedAttention" studynote (agnusdei1207), Ⅱ 핵심 원리: a shared
  block is copied to a new block before a sharer writes into it.
"""
from __future__ import annotations

import numpy as np
import torch

STORAGE = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16}


def as_storage(t, dtype: str) -> np.ndarray:
    """torch CPU tensor in the storage dtype -> numpy array holding the same bits."""
    t = t.contiguous()
    if dtype == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact conversion of stored values to float64 (every f32/f16/bf16 value is
    a float64 value)."""
    if dtype == "bf16":
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def empty_cache(num_blocks, num_kv_heads, block_size, head_dim, dtype, fill=0):
    """A cache tensor [num_blocks, num_kv_heads, block_size, head_dim] whose
    every element has the bit pattern ``fill`` (a canary for untouched slots)."""
    bits = np.uint32 if dtype == "f32" else np.uint16
    a = np.full((num_blocks, num_kv_heads, block_size, head_dim), fill, dtype=bits)
    return a.view(STORAGE[dtype])


def reshape_and_cache(key_cache, value_cache, k, v, slot_mapping):
    """Write token t's K/V rows of every KV head into physical slot
    ``slot_mapping[t]`` = block * block_size + offset.  Negative slots are
    padding and skipped.  ``k``, ``v``: [T, num_kv_heads, head_dim]."""
    bs = key_cache.shape[2]
    slots = np.asarray(slot_mapping, dtype=np.int64)
    keep = slots >= 0
    slots = slots[keep]
    if slots.size != np.unique(slots).size:
        raise ValueError("a slot is written twice")
    if slots.size and slots.max() >= key_cache.shape[0] * bs:
        raise ValueError("slot out of range")
    blk, off = slots // bs, slots % bs
    # cache[blk[i], :, off[i], :] = k[i] for every kept token i
    key_cache[blk, :, off, :] = np.asarray(k)[keep]
    value_cache[blk, :, off, :] = np.asarray(v)[keep]


def copy_blocks(key_cache, value_cache, pairs):
    """Copy-on-write: for each (src, dst), block dst becomes a bit copy of
    block src (all KV heads, all offsets), in K and in V."""
    for src, dst in pairs:
        key_cache[dst] = key_cache[src]
        value_cache[dst] = value_cache[src]


def gather_kv(cache, table_row, context_len: int, kv_head: int) -> np.ndarray:
    """The sequence's rows for one KV head in logical order: row t is
    ``cache[table_row[t // bs], kv_head, t % bs, :]`` for t < context_len."""
    bs = cache.shape[2]
    t = np.arange(context_len)
    blocks = np.asarray(table_row, dtype=np.int64)[t // bs]
    if context_len and (blocks.min() < 0 or blocks.max() >= cache.shape[0]):
        raise ValueError("block table entry out of range")
    return cache[blocks, kv_head, t % bs, :]
