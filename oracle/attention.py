"""Oracle: decode attention over the paged KV cache, in float64.

TEST INFRASTRUCTURE ONLY.  Nothing in the product imports this module.

Sources (page title, section):
* "KV Cache & PagedAttention" studynote (agnusdei1207), Ⅱ 아키텍처 and Ⅲ 비교:
  attention itself is changed so that it reads K/V spread over scattered
  blocks through the block table.
* "09. PagedAttention" (119-ai-studio), 해법: the request sees its blocks as
  logically contiguous; the table supplies the physical location.

The pages give no attention formula.  Reading taken here (the plainest one):
one query token per sequence (decode), scaled dot-product softmax attention
over the sequence's first ``context_len`` tokens, no other mask.  Query head
h reads KV head h // G with G = num_q_heads // num_kv_heads (consecutive query
heads share a KV head).  Each (sequence, KV head) is first gathered through
the block table into a contiguous float64 array, then

    x_t = scale * <q_h, K_t>,   w_t = exp(x_t - max_u x_u) / sum_u exp(x_u - max_u x_u),
    out_h = sum_t w_t V_t.

No partitioning, no blocking.  A sequence with context_len 0 gives zeros.
"""
from __future__ import annotations

import numpy as np

from .cache import gather_kv, to_f64


def attend(q64: np.ndarray, K64: np.ndarray, V64: np.ndarray, scale: float) -> np.ndarray:
    """Softmax attention of query rows q64 [H, D] over K64, V64 [L, D]."""
    if K64.shape[0] == 0:
        return np.zeros((q64.shape[0], V64.shape[1]))
    x = scale * (q64 @ K64.T)                    # [H, L]
    e = np.exp(x - x.max(axis=1, keepdims=True))
    w = e / e.sum(axis=1, keepdims=True)
    return w @ V64                               # [H, D]


def decode_one(q, key_cache, value_cache, table_row, context_len, scale, kv_head,
               dtype) -> np.ndarray:
    """Outputs [G, D] of the G query heads of one sequence that read ``kv_head``.
    ``q`` is that sequence's [num_q_heads, D] query in the storage dtype."""
    hkv = key_cache.shape[1]
    G = q.shape[0] // hkv
    K = to_f64(gather_kv(key_cache, table_row, context_len, kv_head), dtype)
    V = to_f64(gather_kv(value_cache, table_row, context_len, kv_head), dtype)
    qh = to_f64(q[kv_head * G:(kv_head + 1) * G], dtype)
    return attend(qh, K, V, scale)


def paged_decode(q, key_cache, value_cache, block_tables, context_lens, scale,
                 dtype) -> np.ndarray:
    """out [S, Hq, D] float64 for queries q [S, Hq, D] (storage dtype)."""
    S, Hq, D = q.shape
    hkv = key_cache.shape[1]
    if Hq % hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    G = Hq // hkv
    out = np.zeros((S, Hq, D))
    for s in range(S):
        for j in range(hkv):
            out[s, j * G:(j + 1) * G] = decode_one(
                q[s], key_cache, value_cache, block_tables[s],
                int(context_lens[s]), scale, j, dtype)
    return out
