"""Seeded synthetic decode workloads for paged KV-cache attention.

This module is shared by the tests, the benchmark and the oracle's callers.  It
holds random numbers, sizes and a scenario script, and nothing of the method
itself: no block allocation, no slot arithmetic, no attention.  Whoever runs a
workload (the CUDA path's host manager, or the oracle's) interprets the script
with its own implementation.

A workload is:

* shapes: ``num_q_heads``, ``num_kv_heads``, ``head_dim``, ``block_size``,
  ``dtype`` ("f32" | "f16" | "bf16") and the pool size ``num_blocks``;
* ``free_order``: the ids handed out first-in-first-out by a fresh block
  allocator.  Ids of the pool that are not listed start out held by an outside
  owner (this models a pool that other requests have already fragmented);
* ``kv``: named K/V token tensors ``[n, num_kv_heads, head_dim]`` in the storage
  dtype, in logical (token) order;
* ``ops``: the host script, a list of tuples
    - ``("add", seq)``             new empty sequence,
    - ``("write", seq, key)``      append the tokens of ``kv[key]`` to ``seq``,
    - ``("fork", parent, child)``  child shares all of parent's blocks,
    - ``("step", seqs, k)``        one decode step: every sequence in ``seqs``
      (batch order) appends one token, ``step_k[k]``/``step_v[k]`` row ``b`` for
      ``seqs[b]``, then attends with query ``step_q[k]`` row ``b``;
* ``partition_size``: the split-K partition length (tokens) the workload's
  long-context decode uses (0 = no split).

All draws come from one ``torch.Generator`` seeded per workload, in a fixed
order, so the same name and step count always give the same bytes.  Values are
drawn in fp32 and rounded once to the storage dtype (round to nearest even).

The five workloads follow the five decode batches the PagedAttention pages'
serving scenario is measured on (tiny correctness batch, 7B-shaped MHA batch,
8B-shaped GQA batch at two block sizes, shared-prefix/beam batch, long-context
split-K batch).  The input recipe of each is spelled out in its builder below.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
BASE_SEED = 426


@dataclass
class Workload:
    name: str
    dtype: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    free_order: list
    partition_size: int
    kv: dict
    ops: list
    step_q: list
    step_k: list
    step_v: list
    meta: dict = field(default_factory=dict)

    @property
    def torch_dtype(self):
        return DTYPES[self.dtype]

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(head_dim) (the tiny batch states 1/sqrt(64);
        the others are silent and take the same textbook value)."""
        return 1.0 / math.sqrt(self.head_dim)

    def step_seqs(self, k: int) -> list:
        for op in self.ops:
            if op[0] == "step" and op[2] == k:
                return list(op[1])
        raise KeyError(k)

    @property
    def num_steps(self) -> int:
        return len(self.step_q)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _normal(g, shape, dtype, std=1.0, chunk_elems=1 << 26):
    """N(0, std^2) drawn in fp32 (chunked to bound host memory), rounded to dtype."""
    n = 1
    for s in shape:
        n *= s
    out = torch.empty(n, dtype=DTYPES[dtype])
    for lo in range(0, n, chunk_elems):
        hi = min(n, lo + chunk_elems)
        x = torch.randn(hi - lo, generator=g, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        out[lo:hi] = x.to(DTYPES[dtype])
    return out.view(*shape)


def _uniform_int(g, lo, hi, n):
    """n integers uniform on [lo, hi] inclusive."""
    return torch.randint(lo, hi + 1, (n,), generator=g).tolist()


def _perm(g, n):
    return torch.randperm(n, generator=g).tolist()


def _decode_batch(name, dtype, seed, lens, hq, hkv, d, bs, steps, kv_std,
                  pool, partition_size, meta):
    """Common builder: every sequence s is prefilled with lens[s]-1 tokens,
    then ``steps`` decode steps each append one token per sequence, so at the
    first step the attended length is lens[s] (it counts the token written in
    that step).  ``pool(g, blocks_needed)`` returns (num_blocks, free_order)."""
    g = _gen(seed)
    S = len(lens)
    kv = {}
    ops = []
    for s in range(S):
        n = lens[s] - 1
        kv[f"k{s}"] = _normal(g, (n, hkv, d), dtype, kv_std)
        kv[f"v{s}"] = _normal(g, (n, hkv, d), dtype, kv_std)
    step_q, step_k, step_v = [], [], []
    for k in range(steps):
        step_q.append(_normal(g, (S, hq, d), dtype))
        step_k.append(_normal(g, (S, hkv, d), dtype, kv_std))
        step_v.append(_normal(g, (S, hkv, d), dtype, kv_std))
    for s in range(S):
        ops.append(("add", s))
        ops.append(("write", s, f"{s}"))
    for k in range(steps):
        ops.append(("step", list(range(S)), k))
    needed = sum(-(-(L - 1 + steps) // bs) for L in lens)
    num_blocks, free_order = pool(g, needed)
    meta = dict(meta)
    meta.update(lens=list(lens), blocks_needed=needed)
    return Workload(name=name, dtype=dtype, num_q_heads=hq, num_kv_heads=hkv,
                    head_dim=d, block_size=bs, num_blocks=num_blocks,
                    free_order=free_order, partition_size=partition_size,
                    kv=kv, ops=ops, step_q=step_q, step_k=step_k,
                    step_v=step_v, meta=meta)


def tiny_f32(steps: int = 1) -> Workload:
    """Tiny fp32 batch: 4 sequences, context lengths {5,17,33,48}, block 16,
    4 query = 4 KV heads, head dim 64, a pool of 32 blocks whose ids come from
    a seeded permutation, q/K/V ~ N(0,1)."""
    def pool(g, needed):
        return 32, _perm(g, 32)
    return _decode_batch("tiny_f32", "f32", BASE_SEED + 1, [5, 17, 33, 48],
                         4, 4, 64, 16, steps, 1.0, pool, 0,
                         dict(recipe="q,K,V~N(0,1); ids = seeded permutation of 32"))


def mha7b_f16(steps: int = 32, num_seqs: int = 64) -> Workload:
    """7B-shaped MHA layer, fp16: 64 sequences, 32 = 32 heads, head dim 128,
    block 16, context lengths uniform on [128, 2048], K/V ~ 0.5*N(0,1),
    q ~ N(0,1), pool = total blocks the run needs + 10%, shuffled ids,
    ``steps`` consecutive decode steps with cache writes.  The batch fixes no
    split-K partition; 1024 tokens balances the decode's dynamic schedule
    against merge work on one B200 (512 and 2048 are both slower)."""
    g = _gen(BASE_SEED + 2)
    lens = _uniform_int(g, 128, 2048, num_seqs)

    def pool(g, needed):
        nb = math.ceil(1.1 * needed)
        return nb, _perm(g, nb)
    return _decode_batch("mha7b_f16", "f16", BASE_SEED + 2 + 1000, lens,
                         32, 32, 128, 16, steps, 0.5, pool, 1024,
                         dict(recipe="L~U{128..2048}; K,V~0.5N(0,1); q~N(0,1); "
                                     "pool=ceil(1.1*needed), shuffled ids"))


def _lognormal_lens(g, n, median, sigma, lo, hi):
    z = torch.randn(n, generator=g, dtype=torch.float64)
    x = torch.exp(math.log(median) + sigma * z)
    return [int(min(hi, max(lo, round(float(v))))) for v in x]


def gqa8b_bf16(block_size: int = 16, steps: int = 1, num_seqs: int = 256,
               sigma: float = 1.0) -> Workload:
    """8B-shaped GQA batch, bf16: 256 sequences, 32 query heads over 8 KV
    heads (4 query heads share each KV head), head dim 128, block 16 or 32,
    context lengths log-normal (median 512, ln-space sigma 1.0) clipped to
    [16, 8192], q/K/V ~ N(0,1).  Fragmented pool: the pool is sized so that
    exactly 40% of it is free; those 40% are a random subset handed out in a
    random order, the other 60% stay held.  The same seed gives the same
    lengths and values for both block sizes; only the pool differs.  The batch
    fixes no split-K partition; 1024 tokens balances the decode's dynamic
    schedule against merge work on one B200 (512 and 2048 are both slower)."""
    g = _gen(BASE_SEED + 3)
    lens = _lognormal_lens(g, num_seqs, 512, sigma, 16, 8192)

    def pool(g2, needed):
        nb = math.ceil(needed / 0.4) + 1
        n_free = math.ceil(0.4 * nb)
        gp = _gen(BASE_SEED + 3 + 7 * block_size)
        order = _perm(gp, nb)[:n_free]
        return nb, order
    return _decode_batch(f"gqa8b_bf16_bs{block_size}", "bf16", BASE_SEED + 3 + 1000,
                         lens, 32, 8, 128, block_size, steps, 1.0, pool, 1024,
                         dict(recipe=f"L=clip(round(exp(ln512+{sigma}N(0,1))),16,8192); "
                                     "q,K,V~N(0,1); 40% of pool free, random subset "
                                     "in random order", sigma=sigma))


def prefix_f16(steps: int = 1, duplicate_prefix: bool = False, n_req: int = 64,
               plen: int = 1024, suffix_max: int = 256, n_fork: int = 16,
               heads: int = 32) -> Workload:
    """Shared-prefix / parallel-sampling batch, fp16: 64 requests share one
    1024-token prefix; each then appends its own suffix of U{0..256} tokens;
    16 of them (a seeded choice) fork into beam width 4 (3 children each, so
    112 sequences); then decode steps in which every sequence appends one
    token.  32 = 32 heads, head dim 128, block 16, q/K/V ~ N(0,1), shuffled
    ids.  With ``duplicate_prefix`` every request writes its own copy of the
    same prefix instead of sharing it (same logical K/V, other layout).  The
    keyword sizes shrink the batch for element-by-element tests."""
    hq = hkv = heads
    d, bs = 128, 16
    g = _gen(BASE_SEED + 4)
    suffix = _uniform_int(g, 0, suffix_max, n_req)
    forkers = sorted(_perm(g, n_req)[:n_fork])
    kv = {"kprefix": _normal(g, (plen, hkv, d), "f16"),
          "vprefix": _normal(g, (plen, hkv, d), "f16")}
    for r in range(n_req):
        kv[f"ksuf{r}"] = _normal(g, (suffix[r], hkv, d), "f16")
        kv[f"vsuf{r}"] = _normal(g, (suffix[r], hkv, d), "f16")
    children = {}
    nxt = n_req
    for f in forkers:
        children[f] = [nxt, nxt + 1, nxt + 2]
        nxt += 3
    S = nxt
    step_q, step_k, step_v = [], [], []
    for k in range(steps):
        step_q.append(_normal(g, (S, hq, d), "f16"))
        step_k.append(_normal(g, (S, hkv, d), "f16"))
        step_v.append(_normal(g, (S, hkv, d), "f16"))
    ops = []
    if duplicate_prefix:
        for r in range(n_req):
            ops += [("add", r), ("write", r, "prefix"), ("write", r, f"suf{r}")]
    else:
        ops += [("add", 0), ("write", 0, "prefix")]
        for r in range(1, n_req):
            ops.append(("fork", 0, r))
        for r in range(n_req):
            ops.append(("write", r, f"suf{r}"))
    for f in forkers:
        for c in children[f]:
            ops.append(("fork", f, c))
    for k in range(steps):
        ops.append(("step", list(range(S)), k))
    unique = (plen // bs) * (n_req if duplicate_prefix else 1) + \
        sum(-(-s // bs) for s in suffix)
    needed = unique + S * (steps + 1) + 3 * len(forkers)
    nb = math.ceil(1.1 * needed)
    free_order = _perm(g, nb)
    lens = []
    for r in range(n_req):
        lens.append(plen + suffix[r] + 1)
    for f in forkers:
        lens += [plen + suffix[f] + 1] * 3
    return Workload(name="prefix_f16" + ("_dup" if duplicate_prefix else ""),
                    dtype="f16", num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                    block_size=bs, num_blocks=nb, free_order=free_order,
                    partition_size=512, kv=kv, ops=ops, step_q=step_q,
                    step_k=step_k, step_v=step_v,
                    meta=dict(lens=lens, suffix=suffix, forkers=forkers,
                              children=children, prefix_len=plen,
                              recipe="prefix 1024 tok; suffix~U{0..256}; 16 of 64 "
                                     "fork to beam 4; q,K,V~N(0,1); shuffled ids"))


def long_bf16(steps: int = 1, num_seqs: int = 8) -> Workload:
    """Long-context split-K batch, bf16: 8 sequences, 32 query heads over 8
    KV heads, head dim 128, block 64, context lengths uniform on
    [32768, 131072], partition 512 tokens, q/K/V ~ N(0,1), fully shuffled
    pool (exactly the blocks needed)."""
    g = _gen(BASE_SEED + 5)
    lens = _uniform_int(g, 32768, 131072, num_seqs)

    def pool(g, needed):
        return needed, _perm(g, needed)
    return _decode_batch("long_bf16", "bf16", BASE_SEED + 5 + 1000, lens,
                         32, 8, 128, 64, steps, 1.0, pool, 512,
                         dict(recipe="L~U{32768..131072}; q,K,V~N(0,1); "
                                     "fully shuffled pool"))


@dataclass
class PrefillBatch:
    """A chunked-prefill batch.  Sequence s holds ``context_lens[s]`` tokens
    once its chunk is written; the chunk is its last ``query_lens[s]`` tokens.
    ``k[s]``/``v[s]`` are all of its K/V rows [context_lens[s], Hkv, D] in
    logical order (the runner writes the first context_lens[s] -
    query_lens[s] before the step and the chunk's rows in the step), ``q``
    the chunk queries of every sequence packed in order [sum(query_lens), Hq,
    D].  Block pool as in ``Workload``."""
    name: str
    dtype: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    free_order: list
    context_lens: list
    query_lens: list
    k: list
    v: list
    q: torch.Tensor
    meta: dict = field(default_factory=dict)

    @property
    def torch_dtype(self):
        return DTYPES[self.dtype]

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(head_dim), as for the decode batches."""
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def query_offsets(self) -> list:
        """Row of ``q`` where each sequence's chunk starts, and the total."""
        out = [0]
        for n in self.query_lens:
            out.append(out[-1] + n)
        return out


def _prefill_batch(name, dtype, seed, lens, qlens, hq, hkv, d, bs, pool, meta):
    g = _gen(seed)
    k = [_normal(g, (L, hkv, d), dtype) for L in lens]
    v = [_normal(g, (L, hkv, d), dtype) for L in lens]
    q = _normal(g, (sum(qlens), hq, d), dtype)
    needed = sum(-(-L // bs) for L in lens)
    num_blocks, free_order = pool(g, needed)
    meta = dict(meta)
    meta.update(blocks_needed=needed)
    return PrefillBatch(name=name, dtype=dtype, num_q_heads=hq, num_kv_heads=hkv, head_dim=d,
                        block_size=bs, num_blocks=num_blocks, free_order=free_order,
                        context_lens=list(lens), query_lens=list(qlens), k=k, v=v, q=q,
                        meta=meta)


def _shuffled_pool(extra=0.1):
    def pool(g, needed):
        nb = math.ceil((1 + extra) * needed) + 1
        return nb, _perm(g, nb)
    return pool


def prefill_gqa8b_bf16(num_seqs: int = 32, chunk: int = 512) -> PrefillBatch:
    """Chunked prefill on the 8B-shaped GQA layer, bf16: 32 sequences, 32
    query heads over 8 KV heads, head dim 128, block 16; context lengths
    uniform on [512, 4096] and each sequence's chunk its last 512 tokens (the
    latest chunk of a long prompt; a 512-token prompt is a whole prompt);
    q/K/V ~ N(0,1); pool = blocks needed + 10%, shuffled ids."""
    g = _gen(BASE_SEED + 20)
    lens = _uniform_int(g, chunk, 4096, num_seqs)
    return _prefill_batch("prefill_gqa8b_bf16", "bf16", BASE_SEED + 20 + 1000, lens,
                          [chunk] * num_seqs, 32, 8, 128, 16, _shuffled_pool(),
                          dict(recipe=f"L~U{{{chunk}..4096}}, chunk = last {chunk} tokens; "
                                      "q,K,V~N(0,1); pool=needed+10%, shuffled ids"))


def prefill_mha7b_f16(num_seqs: int = 16) -> PrefillBatch:
    """Whole-prompt prefill on the 7B-shaped MHA layer, fp16: 16 prompts of
    lengths uniform on [128, 2048], 32 = 32 heads, head dim 128, block 16,
    q/K/V ~ N(0,1), pool = blocks needed + 10%, shuffled ids."""
    g = _gen(BASE_SEED + 21)
    lens = _uniform_int(g, 128, 2048, num_seqs)
    return _prefill_batch("prefill_mha7b_f16", "f16", BASE_SEED + 21 + 1000, lens, lens,
                          32, 32, 128, 16, _shuffled_pool(),
                          dict(recipe="L~U{128..2048}, whole prompts; q,K,V~N(0,1); "
                                      "pool=needed+10%, shuffled ids"))


def prefill_custom(dtype, lens, qlens, hq, hkv, d, bs, seed, extra_blocks=3) -> PrefillBatch:
    """Small ad-hoc prefill batch for edge cases (same recipe: q/K/V ~ N(0,1),
    pool = blocks needed + extra_blocks, shuffled ids)."""
    def pool(g, needed):
        nb = needed + extra_blocks
        return nb, _perm(g, nb)
    return _prefill_batch(f"prefill_custom_{dtype}_{seed}", dtype, seed, list(lens), list(qlens),
                          hq, hkv, d, bs, pool, {})


PREFILL_BUILDERS = {
    "prefill_gqa8b_bf16": prefill_gqa8b_bf16,
    "prefill_mha7b_f16": prefill_mha7b_f16,
}


BUILDERS = {
    "tiny_f32": tiny_f32,
    "mha7b_f16": mha7b_f16,
    "gqa8b_bf16_bs16": lambda **kw: gqa8b_bf16(block_size=16, **kw),
    "gqa8b_bf16_bs32": lambda **kw: gqa8b_bf16(block_size=32, **kw),
    "prefix_f16": prefix_f16,
    "long_bf16": long_bf16,
}


def make(name: str, **kw) -> Workload:
    return BUILDERS[name](**kw)


def custom(dtype, lens, hq, hkv, d, bs, seed, steps=1, num_blocks=None,
           kv_std=1.0, partition_size=0, shuffle=True) -> Workload:
    """Small ad-hoc batch for edge cases and sweeps (same recipe as the named
    ones: prefill lens[s]-1 tokens, then ``steps`` one-token steps)."""
    def pool(g, needed):
        nb = num_blocks if num_blocks is not None else needed
        return nb, (_perm(g, nb) if shuffle else list(range(nb)))
    return _decode_batch(f"custom_{dtype}_{seed}", dtype, seed, list(lens), hq,
                         hkv, d, bs, steps, kv_std, pool, partition_size, {})
