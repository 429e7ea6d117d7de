"""Test glue: run one seeded workload through the oracle and through the CUDA
path, and compare.

The oracle executes the workload's host script with its own manager and
builds its own caches (``oracle.run``).  The CUDA path runs the same script
with the library's C++ manager; its slot mappings, copy-on-write pairs and
block tables must equal the oracle's bit for bit.  The GPU caches start from
the oracle's prefill cache (uploaded), then every decode step runs on the GPU
(copy-on-write copies, cache write, decode) with the library's own metadata.
Nothing the oracle consumes comes from the GPU.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import paged_kv_cache_426_b200 as pa

TOL = {"f32": dict(atol=1e-5, rtol=0.0, nrm=1e-6),
       "f16": dict(atol=3e-3, rtol=1e-2, nrm=5e-3),
       "bf16": dict(atol=3e-3, rtol=1e-2, nrm=1e-2)}


def to_torch_storage(a: np.ndarray, dtype: str) -> torch.Tensor:
    """numpy storage array (bits) -> torch tensor of the storage dtype (CPU)."""
    if dtype == "bf16":
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(a)


def to_numpy_storage(t: torch.Tensor, dtype: str) -> np.ndarray:
    return oracle.as_storage(t.detach().cpu(), dtype)


def check_close(gpu: np.ndarray, ref: np.ndarray, dtype: str, what: str = ""):
    """gpu: float64 view of the GPU output [S, H, D]; ref: oracle float64."""
    t = TOL[dtype]
    err = np.abs(gpu - ref)
    bound = t["atol"] + t["rtol"] * np.abs(ref)
    bad = err > bound
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} elements out of tolerance; worst {float(err.max()):.3e} "
        f"at {np.unravel_index(int(np.argmax(err - bound)), err.shape)}")
    num = np.sqrt((err ** 2).sum(axis=-1))
    den = np.sqrt((ref ** 2).sum(axis=-1))
    rel = num / np.maximum(den, 1e-30)
    rel = np.where(den > 0, rel, num)
    assert rel.max() <= t["nrm"], f"{what}: normalised error {rel.max():.3e} > {t['nrm']}"
    return float(err.max()), float(rel.max())


class CudaPathRun:
    """The CUDA path driven through a workload's script."""

    def __init__(self, w, rec: oracle.OracleRun, *, partition_size=None, device="cuda",
                 max_blocks=None, engine=None, fused=False):
        self.w = w
        self.engine = engine          # None: plain pa_decode; else a per-call engine option
        self.fused = fused            # the step's cache write done by the pa_decode call
        self.dev = device
        self.P = w.partition_size if partition_size is None else partition_size
        self.mb = max_blocks if max_blocks is not None else oracle.max_blocks_needed(w)
        self.alloc = pa.BlockAllocator(w.num_blocks, w.free_order)
        self.mgr = pa.BlockManager(self.alloc, w.block_size)
        src_k = rec.prefill_key_cache if rec.prefill_key_cache is not None else rec.key_cache
        src_v = rec.prefill_value_cache if rec.prefill_value_cache is not None else rec.value_cache
        self.kc = to_torch_storage(src_k, w.dtype).to(device)
        self.vc = to_torch_storage(src_v, w.dtype).to(device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.rec = rec
        self.max_len = max(w.meta["lens"]) - 1 + w.num_steps
        S_max = max(len(op[1]) for op in w.ops if op[0] == "step")
        self.ws = pa.alloc_workspace(S_max, w.num_q_heads, w.num_kv_heads, w.head_dim,
                                     self.max_len, self.P, device)

    def replay_prefill(self):
        """Run the non-step ops with the C++ manager; check slots and copies
        against the oracle's record (the caches themselves came from it)."""
        w, rec = self.w, self.rec
        for op in w.ops:
            if op[0] == "add":
                self.mgr.add_seq(op[1])
            elif op[0] == "fork":
                self.mgr.fork(op[1], op[2])
            elif op[0] == "write":
                n = w.kv["k" + op[2]].shape[0]
                slots, cow = self.mgr.append(op[1], n)
                want = rec.prefill_slots[(op[1], op[2])]
                assert np.array_equal(slots.numpy(), want), f"slots of {op}"
                for c in cow:
                    assert c in [tuple(x) for x in rec.prefill_cows]
            elif op[0] == "step":
                break

    def step(self, k, out_dtype_check=True):
        """One decode step on the GPU with the library's own metadata."""
        w = self.w
        st = self.rec.steps[k]
        seqs = st.seqs
        slots, cow = self.mgr.append_step(seqs)
        assert np.array_equal(slots.numpy(), st.slot_mapping), "step slot mapping"
        assert [tuple(map(int, c)) for c in cow.tolist()] == [tuple(c) for c in st.cow_pairs], \
            "copy-on-write pairs"
        tab, lens = self.mgr.block_tables(seqs, self.mb)
        assert np.array_equal(tab.numpy(), st.block_tables), "block tables"
        assert np.array_equal(lens.numpy(), st.context_lens), "context lens"
        dev = self.dev
        if cow.shape[0]:
            pa.pa_copy_blocks(self.kc, self.vc, cow.to(dev), err_flag=self.err)
        new = (w.step_k[k].to(dev), w.step_v[k].to(dev), slots.to(dev))
        if not self.fused:
            pa.pa_reshape_and_cache(*new[:2], self.kc, self.vc, new[2], err_flag=self.err)
        q = w.step_q[k].to(dev)
        out = torch.empty_like(q)
        pa.pa_decode(out, q, self.kc, self.vc, tab.to(dev), lens.to(dev), self.max_len, w.scale,
                     partition_size=self.P, workspace=self.ws, err_flag=self.err,
                     engine=self.engine, write=new if self.fused else None)
        torch.cuda.synchronize()
        assert int(self.err.item()) == 0, f"err_flag {int(self.err.item())}"
        return out

    def caches_equal_oracle(self):
        kc = to_numpy_storage(self.kc, self.w.dtype)
        vc = to_numpy_storage(self.vc, self.w.dtype)
        return (np.array_equal(kc.view(np.uint8), self.rec.key_cache.view(np.uint8)) and
                np.array_equal(vc.view(np.uint8), self.rec.value_cache.view(np.uint8)))


def out_f64(t: torch.Tensor, dtype: str) -> np.ndarray:
    return oracle.to_f64(to_numpy_storage(t, dtype), dtype)


def sample_pairs(S, Hq, n, seed):
    rng = np.random.default_rng(seed)
    pairs = {(int(s), int(h)) for s, h in zip(rng.integers(0, S, n), rng.integers(0, Hq, n))}
    pairs |= {(0, 0), (S - 1, Hq - 1)}
    return sorted(pairs)


def oracle_sampled(w, rec, k, pairs):
    """Oracle outputs for sampled (seq, q head) pairs of step k, one by one."""
    st = rec.steps[k]
    q = oracle.as_storage(w.step_q[k], w.dtype)
    G = w.num_q_heads // w.num_kv_heads
    res = {}
    by_group = {}
    for s, h in pairs:
        by_group.setdefault((s, h // G), []).append(h)
    for (s, j), hs in by_group.items():
        o = oracle.decode_one(q[s], rec.key_cache, rec.value_cache, st.block_tables[s],
                              int(st.context_lens[s]), w.scale, j, w.dtype)
        for h in hs:
            res[(s, h)] = o[h - j * G]
    return res


def scale_of(d):
    return 1.0 / math.sqrt(d)


class GpuPrefill:
    """A ``workloads.PrefillBatch`` through the CUDA path: the library's
    manager hands out the slots (same FIFO pool as the oracle's), the tokens
    before each chunk are written with pa_reshape_and_cache, then the chunks'
    (the step), then pa_prefill attends.  ``fill``: value of every cache
    element no token writes (NaN checks that unwritten slots never leak)."""

    def __init__(self, b, device="cuda", fill=0.0):
        self.b = b
        td = b.torch_dtype
        self.alloc = pa.BlockAllocator(b.num_blocks, b.free_order)
        self.mgr = pa.BlockManager(self.alloc, b.block_size)
        shape = (b.num_blocks, b.num_kv_heads, b.block_size, b.head_dim)
        self.kc = torch.full(shape, fill, dtype=td, device=device)
        self.vc = torch.full(shape, fill, dtype=td, device=device)
        self.err = torch.zeros(1, dtype=torch.int32, device=device)
        self.ws = pa.prefill_workspace(device)
        S = len(b.context_lens)
        ctx_s, chunk_s, ctx_k, ctx_v, ch_k, ch_v = [], [], [], [], [], []
        for s, (L, n) in enumerate(zip(b.context_lens, b.query_lens)):
            self.mgr.add_seq(s)
            slots = self.mgr.append(s, L)[0] if L else torch.zeros(0, dtype=torch.int64)
            ctx_s.append(slots[:L - n])
            chunk_s.append(slots[L - n:])
            ctx_k.append(b.k[s][:L - n])
            ctx_v.append(b.v[s][:L - n])
            ch_k.append(b.k[s][L - n:])
            ch_v.append(b.v[s][L - n:])
        self.ctx_slots = torch.cat(ctx_s)
        self.chunk_slots = torch.cat(chunk_s)
        if self.ctx_slots.numel():
            pa.pa_reshape_and_cache(torch.cat(ctx_k).to(device), torch.cat(ctx_v).to(device),
                                    self.kc, self.vc, self.ctx_slots.to(device), err_flag=self.err)
        self.chunk_k = torch.cat(ch_k).to(device)
        self.chunk_v = torch.cat(ch_v).to(device)
        self.chunk_slots_d = self.chunk_slots.to(device)
        self.mb = max(1, max(-(-L // b.block_size) for L in b.context_lens))
        tab, lens = self.mgr.block_tables(list(range(S)), self.mb)
        self.tab_h, self.lens_h = tab, lens
        self.tab, self.lens = tab.to(device), lens.to(device)
        self.cu = torch.tensor(b.query_offsets, dtype=torch.int32, device=device)
        self.q = b.q.to(device)
        self.out = torch.full_like(self.q, float("nan"))
        self.max_q = max(1, max(b.query_lens))

    def write_chunks(self):
        if self.chunk_slots.numel():
            pa.pa_reshape_and_cache(self.chunk_k, self.chunk_v, self.kc, self.vc,
                                    self.chunk_slots_d, err_flag=self.err)

    def attend(self):
        pa.pa_prefill(self.out, self.q, self.kc, self.vc, self.tab, self.lens, self.cu, self.max_q,
                      self.b.scale, workspace=self.ws, err_flag=self.err)

    def step(self):
        self.write_chunks()
        self.attend()
        torch.cuda.synchronize()
        return self.out
