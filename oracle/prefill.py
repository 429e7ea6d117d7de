"""Oracle: prefill (multi-query, causal) attention over the paged KV cache, in
float64.

TEST INFRASTRUCTURE ONLY.  Nothing in the product imports this module.

Sources (page title, section):
* "KV Cache & PagedAttention" studynote (agnusdei1207), Ⅲ 비교 및 연결: the
  serving stack pairs FlashAttention (attention computed in tiles so that data
  crosses between HBM and on-chip memory fewer times) with PagedAttention
  (where the K/V live); the related-concept map repeats the pairing.
* "09. PagedAttention" (119-ai-studio), the closing section on what the block
  design enables: requests with the same prompt start can share the prefilled
  K/V blocks, so the prompt's K/V are computed into the paged cache.

The pages give no prefill formula.  Reading taken here (the plainest one the
rest supports): a prefill chunk of sequence s is its last n_s tokens, whose
K/V are already written into the cache; the chunk's query row i sits at
position p = L_s - n_s + i (L_s = context length, counting the chunk) and
attends, exactly like a decode query at that position, to the sequence's
tokens 0..p (causal mask, aligned at the end of the sequence).  A chunk with
n_s = L_s is a whole prompt; n_s = 1 is a decode step.

Each row is therefore the decode oracle's attention over the first p + 1
gathered tokens: no tiling, no online softmax.
"""
from __future__ import annotations

import numpy as np

from .attention import attend
from .cache import gather_kv, to_f64


def prefill_rows(q_rows, key_cache, value_cache, table_row, context_len, query_len,
                 scale, kv_head, dtype, rows=None) -> np.ndarray:
    """Outputs [n, G, D] (float64) of one sequence's chunk for the G query
    heads that read ``kv_head``.  ``q_rows`` is the chunk's query
    [n, num_q_heads, D] in the storage dtype; ``rows`` (optional) picks which
    chunk rows to compute (the others stay zero)."""
    hkv = key_cache.shape[1]
    n, Hq, D = q_rows.shape
    G = Hq // hkv
    if query_len != n or query_len > context_len:
        raise ValueError("a chunk holds query_len <= context_len rows")
    K = to_f64(gather_kv(key_cache, table_row, context_len, kv_head), dtype)
    V = to_f64(gather_kv(value_cache, table_row, context_len, kv_head), dtype)
    out = np.zeros((n, G, D))
    for i in (range(n) if rows is None else rows):
        p = context_len - query_len + i
        qh = to_f64(q_rows[i, kv_head * G:(kv_head + 1) * G], dtype)
        out[i] = attend(qh, K[:p + 1], V[:p + 1], scale)
    return out


def paged_prefill(q, key_cache, value_cache, block_tables, context_lens, cu_seqlens_q,
                  scale, dtype) -> np.ndarray:
    """out [T, Hq, D] float64 for the packed chunk queries q [T, Hq, D]
    (storage dtype); sequence s owns rows cu_seqlens_q[s] .. cu_seqlens_q[s+1]-1."""
    T, Hq, D = q.shape
    hkv = key_cache.shape[1]
    if Hq % hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    G = Hq // hkv
    out = np.zeros((T, Hq, D))
    for s in range(len(context_lens)):
        a, b = int(cu_seqlens_q[s]), int(cu_seqlens_q[s + 1])
        for j in range(hkv):
            out[a:b, j * G:(j + 1) * G] = prefill_rows(
                q[a:b], key_cache, value_cache, block_tables[s], int(context_lens[s]),
                b - a, scale, j, dtype)
    return out
