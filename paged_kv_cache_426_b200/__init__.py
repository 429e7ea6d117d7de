"""Python binding of libpa_b200.so: paged KV-cache decode attention on B200.

Argument marshalling only.  Every step of the hot path runs in the library's
CUDA kernels (cache write, copy-on-write block copy, decode attention) or its
C++ host code (block allocator, block tables); PyTorch supplies device memory
and streams.  There is no fallback: importing this package fails if the
library has not been built (``python paged_kv_cache_426_b200/build.py``).

The functions keep the C names (``pa_reshape_and_cache``, ``pa_decode``,
``pa_copy_blocks``, ...).  Tensor arguments give the pointers and the sizes;
the C ABI and its error codes are documented in ``include/pa.h``.
"""
from __future__ import annotations

import ctypes as C
import os
import weakref

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python paged_kv_cache_426_b200/build.py` "
        "(nvcc, sm_100a).  There is no CPU or PyTorch fallback.")
lib = C.CDLL(LIB_PATH)

PA_OK, PA_ERR_INVALID, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_OOM, PA_ERR_STATE = 0, -1, -2, -3, -4, -5
PA_F32, PA_F16, PA_BF16 = 0, 1, 2
PA_DEV_BAD_SLOT, PA_DEV_BAD_BLOCK, PA_DEV_BAD_LEN, PA_DEV_BAD_PAIR, PA_DEV_TIMEOUT = 1, 2, 3, 4, 5
PA_ENGINE_AUTO, PA_ENGINE_CUDA_CORE, PA_ENGINE_TENSOR = 0, 1, 2

_vp, _i, _i64, _sz, _f = C.c_void_p, C.c_int, C.c_int64, C.c_size_t, C.c_float
_pi32, _pi64 = C.POINTER(C.c_int32), C.POINTER(C.c_int64)

SIGNATURES = {
    "pa_status_string": ([_i], C.c_char_p),
    "pa_version": ([], _i),
    "pa_reshape_and_cache": ([_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp], _i),
    "pa_decode_workspace_size": ([_i, _i, _i, _i, _i, _i, C.POINTER(_sz)], _i),
    "pa_decode_workspace_init": ([_vp, _sz, _vp], _i),
    "pa_decode": ([_vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i, _vp,
                   _sz, _i, _vp, _vp], _i),
    "pa_decode_static": ([_vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i,
                          _i, _vp, _vp], _i),
    "pa_decode_ex": ([_vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _i, _i, _i, _i, _f, _i, _vp,
                      _sz, _i, _vp, _vp, _vp], _i),
    "pa_prefill": ([_vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _f,
                    _vp, _sz, _i, _vp, _vp], _i),
    "pa_copy_blocks": ([_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp], _i),
    "pa_allocator_create": ([_i, _pi32, _i, C.POINTER(_vp)], _i),
    "pa_allocator_destroy": ([_vp], None),
    "pa_allocator_allocate": ([_vp, _pi32], _i),
    "pa_allocator_incref": ([_vp, C.c_int32], _i),
    "pa_allocator_free": ([_vp, C.c_int32], _i),
    "pa_allocator_refcount": ([_vp, C.c_int32, _pi32], _i),
    "pa_allocator_num_free": ([_vp, _pi32], _i),
    "pa_manager_create": ([_vp, _i, C.POINTER(_vp)], _i),
    "pa_manager_destroy": ([_vp], None),
    "pa_manager_add_seq": ([_vp, _i64], _i),
    "pa_manager_fork": ([_vp, _i64, _i64], _i),
    "pa_manager_free_seq": ([_vp, _i64], _i),
    "pa_manager_append": ([_vp, _i64, _i, _pi64, _pi64, C.POINTER(_i)], _i),
    "pa_manager_append_step": ([_vp, _vp, _i, _vp, _vp, C.POINTER(_i)], _i),
    "pa_manager_seq_len": ([_vp, _i64, _pi32], _i),
    "pa_manager_block_tables": ([_vp, _vp, _i, _vp, _i, _vp], _i),
    "pa_manager_enable_prefix_cache": ([_vp], _i),
    "pa_manager_add_seq_prompt": ([_vp, _i64, _pi32, _i, _pi64, C.POINTER(_i)], _i),
    "pa_manager_prefix_cache_stats": ([_vp, _pi64], _i),
}
for _name, (_args, _ret) in SIGNATURES.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = _ret


class PAError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {lib.pa_status_string(status).decode()} ({status})")


def check(status: int, what: str) -> None:
    if status != PA_OK:
        raise PAError(status, what)


_DT = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}


def pa_dtype(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise PAError(PA_ERR_UNSUPPORTED, f"dtype {t.dtype}") from None


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _cuda(*ts):
    for t in ts:
        if t is not None and not (t.is_cuda and t.is_contiguous()):
            raise PAError(PA_ERR_INVALID, "tensors must be contiguous CUDA tensors")


# ------------------------------------------------------------------ kernels

def pa_reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, *, err_flag=None,
                         stream=None):
    """key/value [T, Hkv, D]; caches [NB, Hkv, bs, D]; slot_mapping int64 [T]."""
    _cuda(key, value, key_cache, value_cache, slot_mapping, err_flag)
    NB, hkv, bs, d = key_cache.shape
    check(lib.pa_reshape_and_cache(_ptr(key), _ptr(value), _ptr(key_cache), _ptr(value_cache),
                                   _ptr(slot_mapping), key.shape[0], hkv, d, bs, NB,
                                   pa_dtype(key_cache), _ptr(err_flag), _stream(stream)),
          "pa_reshape_and_cache")


def pa_copy_blocks(key_cache, value_cache, block_pairs, *, err_flag=None, stream=None):
    """block_pairs int64 [n, 2] (src, dst) on the device."""
    _cuda(key_cache, value_cache, block_pairs, err_flag)
    NB, hkv, bs, d = key_cache.shape
    check(lib.pa_copy_blocks(_ptr(key_cache), _ptr(value_cache), _ptr(block_pairs),
                             block_pairs.shape[0], hkv, d, bs, NB, pa_dtype(key_cache),
                             _ptr(err_flag), _stream(stream)), "pa_copy_blocks")


def pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                             partition_size) -> int:
    n = C.c_size_t(0)
    check(lib.pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                       max_context_len, partition_size, C.byref(n)),
          "pa_decode_workspace_size")
    return n.value


def pa_decode_workspace_init(workspace, stream=None):
    check(lib.pa_decode_workspace_init(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream(stream)), "pa_decode_workspace_init")


def alloc_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, max_context_len,
                    partition_size, device="cuda"):
    """A zero-filled workspace of the size pa_decode needs (uint8 tensor)."""
    n = pa_decode_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                 max_context_len, partition_size)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device)


class pa_decode_options(C.Structure):
    """Per-call options of pa_decode_ex (include/pa.h)."""
    _fields_ = [("struct_size", C.c_int), ("engine", C.c_int), ("test_withhold_stage", C.c_int),
                ("key_new", C.c_void_p), ("value_new", C.c_void_p), ("slot_mapping", C.c_void_p)]


ENGINES = {"auto": PA_ENGINE_AUTO, "core": PA_ENGINE_CUDA_CORE, "tensor": PA_ENGINE_TENSOR}


def pa_decode(out, query, key_cache, value_cache, block_tables, context_lens, max_context_len,
              scale, *, partition_size=0, workspace=None, err_flag=None, stream=None,
              engine=None, test_withhold_stage=-1, write=None):
    """out/query [S, Hq, D]; caches [NB, Hkv, bs, D]; block_tables int32 [S, max_blocks];
    context_lens int32 [S].  ``engine`` ("auto", "core", "tensor" or a PA_ENGINE_*
    value), ``test_withhold_stage`` and ``write`` = (key_new, value_new,
    slot_mapping) - the step's cache write, [S, Hkv, D] twice and int64 [S],
    done by this call - are per-call options (pa_decode_ex); with none given
    this is the plain pa_decode call."""
    _cuda(out, query, key_cache, value_cache, block_tables, context_lens, workspace, err_flag)
    if write is not None:
        _cuda(*write)
    S, hq, d = query.shape
    NB, hkv, bs, _ = key_cache.shape
    if workspace is None:
        raise PAError(PA_ERR_INVALID, "pa_decode needs a workspace (alloc_workspace)")
    args = (_ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache), _ptr(block_tables),
            block_tables.shape[1], _ptr(context_lens), int(max_context_len), S, hq, hkv, d, bs,
            NB, float(scale), int(partition_size), _ptr(workspace),
            workspace.numel() * workspace.element_size(), pa_dtype(query), _ptr(err_flag),
            _stream(stream))
    if engine is None and test_withhold_stage == -1 and write is None:
        check(lib.pa_decode(*args), "pa_decode")
        return
    eng = ENGINES[engine] if isinstance(engine, str) else (PA_ENGINE_AUTO if engine is None
                                                            else int(engine))
    kn, vn, sm = write if write is not None else (None, None, None)
    opts = pa_decode_options(C.sizeof(pa_decode_options), eng, int(test_withhold_stage),
                             _ptr(kn), _ptr(vn), _ptr(sm))
    check(lib.pa_decode_ex(*args, C.byref(opts)), "pa_decode_ex")


PA_DECODE_STATIC_WORKSPACE_BYTES = 16 << 20


def pa_decode_static(out, query, key_cache, value_cache, block_tables, context_lens,
                     max_context_len, scale, *, partition_size=0, err_flag=None, stream=None):
    """pa_decode with the library's fixed device workspace (no allocation by
    anyone); same arguments as pa_decode minus the workspace."""
    _cuda(out, query, key_cache, value_cache, block_tables, context_lens, err_flag)
    S, hq, d = query.shape
    NB, hkv, bs, _ = key_cache.shape
    check(lib.pa_decode_static(_ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache),
                               _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                               int(max_context_len), S, hq, hkv, d, bs, NB, float(scale),
                               int(partition_size), pa_dtype(query), _ptr(err_flag),
                               _stream(stream)), "pa_decode_static")


PREFILL_WORKSPACE_BYTES = 64


def prefill_workspace(device):
    """A zero-filled pa_prefill workspace (every call leaves it zeroed, so one
    serves all calls ordered on a stream)."""
    return torch.zeros(PREFILL_WORKSPACE_BYTES // 4, dtype=torch.int32, device=device)


def pa_prefill(out, query, key_cache, value_cache, block_tables, context_lens, cu_seqlens_q,
               max_query_len, scale, *, workspace=None, err_flag=None, stream=None):
    """Causal attention of packed prefill chunks: out/query [T, Hq, D]; caches
    [NB, Hkv, bs, D]; block_tables int32 [S, max_blocks]; context_lens int32
    [S] (counting the chunk); cu_seqlens_q int32 [S + 1] (row offsets of the
    chunks in query).  ``workspace``: from prefill_workspace (a fresh one per
    call when None)."""
    if workspace is None:
        workspace = prefill_workspace(query.device)
    _cuda(out, query, key_cache, value_cache, block_tables, context_lens, cu_seqlens_q, workspace,
          err_flag)
    T, hq, d = query.shape
    NB, hkv, bs, _ = key_cache.shape
    S = context_lens.shape[0]
    if cu_seqlens_q.shape[0] != S + 1:
        raise PAError(PA_ERR_INVALID, "cu_seqlens_q needs num_seqs + 1 entries")
    check(lib.pa_prefill(_ptr(out), _ptr(query), _ptr(key_cache), _ptr(value_cache),
                         _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                         _ptr(cu_seqlens_q), S, T, int(max_query_len), hq, hkv, d, bs, NB,
                         float(scale), _ptr(workspace), workspace.numel() * workspace.element_size(),
                         pa_dtype(query), _ptr(err_flag), _stream(stream)),
          "pa_prefill")


# ------------------------------------------------------------------ host objects

class BlockAllocator:
    """FIFO pool of physical block ids with reference counts (C++ pa_allocator)."""

    def __init__(self, num_blocks: int, free_order=None):
        self._h = C.c_void_p()
        if free_order is None:
            check(lib.pa_allocator_create(num_blocks, None, 0, C.byref(self._h)), "allocator")
        else:
            arr = (C.c_int32 * len(free_order))(*free_order)
            check(lib.pa_allocator_create(num_blocks, arr, len(free_order), C.byref(self._h)),
                  "allocator")
        self.num_blocks = num_blocks
        weakref.finalize(self, lib.pa_allocator_destroy, self._h.value)

    def allocate_block(self) -> int:
        b = C.c_int32()
        check(lib.pa_allocator_allocate(self._h, C.byref(b)), "allocate_block")
        return b.value

    def incref(self, b: int) -> None:
        check(lib.pa_allocator_incref(self._h, b), "incref")

    def free_block(self, b: int) -> None:
        check(lib.pa_allocator_free(self._h, b), "free_block")

    def refcount(self, b: int) -> int:
        r = C.c_int32()
        check(lib.pa_allocator_refcount(self._h, b, C.byref(r)), "refcount")
        return r.value

    def num_free(self) -> int:
        r = C.c_int32()
        check(lib.pa_allocator_num_free(self._h, C.byref(r)), "num_free")
        return r.value


class BlockManager:
    """Per-sequence block tables over a BlockAllocator (C++ pa_manager)."""

    def __init__(self, allocator: BlockAllocator, block_size: int):
        self.alloc = allocator          # keeps the allocator alive
        self.block_size = block_size
        self._h = C.c_void_p()
        check(lib.pa_manager_create(allocator._h, block_size, C.byref(self._h)), "manager")
        weakref.finalize(self, lib.pa_manager_destroy, self._h.value)

    def add_seq(self, seq: int) -> None:
        check(lib.pa_manager_add_seq(self._h, seq), "add_seq")

    def fork(self, parent: int, child: int) -> None:
        check(lib.pa_manager_fork(self._h, parent, child), "fork")

    def free_seq(self, seq: int) -> None:
        check(lib.pa_manager_free_seq(self._h, seq), "free_seq")

    def append(self, seq: int, num_tokens: int = 1):
        """Returns (slots int64 tensor [num_tokens], cow list of (src, dst))."""
        slots = torch.empty(max(num_tokens, 1), dtype=torch.int64)
        cow = (C.c_int64 * 2)()
        n = C.c_int(0)
        check(lib.pa_manager_append(self._h, seq, num_tokens,
                                    C.cast(slots.data_ptr(), _pi64), cow, C.byref(n)), "append")
        return slots[:num_tokens], ([(cow[0], cow[1])] if n.value else [])

    def append_step(self, seqs, slots_out=None, cow_out=None):
        """One token for each sequence.  Returns (slots int64 [n], cow int64 [k, 2])."""
        ids = torch.as_tensor(list(seqs) if not torch.is_tensor(seqs) else seqs, dtype=torch.int64)
        n = ids.numel()
        slots = slots_out if slots_out is not None else torch.empty(n, dtype=torch.int64)
        cow = cow_out if cow_out is not None else torch.empty((max(n, 1), 2), dtype=torch.int64)
        k = C.c_int(0)
        # per-step call: raw addresses, no ctypes casts (the arrays are contiguous int64)
        check(lib.pa_manager_append_step(self._h, ids.data_ptr(), n, slots.data_ptr(),
                                         cow.data_ptr(), C.byref(k)), "append_step")
        return (slots if slots.numel() == n else slots[:n]), cow[:k.value]

    def seq_len(self, seq: int) -> int:
        r = C.c_int32()
        check(lib.pa_manager_seq_len(self._h, seq, C.byref(r)), "seq_len")
        return r.value

    def block_tables(self, seqs, max_blocks: int, tables_out=None, lens_out=None):
        """(block_tables int32 [n, max_blocks] padded with -1, context_lens int32 [n])."""
        ids = torch.as_tensor(list(seqs) if not torch.is_tensor(seqs) else seqs, dtype=torch.int64)
        n = ids.numel()
        tab = tables_out if tables_out is not None else torch.empty((n, max_blocks), dtype=torch.int32)
        lens = lens_out if lens_out is not None else torch.empty(n, dtype=torch.int32)
        check(lib.pa_manager_block_tables(self._h, ids.data_ptr(), n, tab.data_ptr(), max_blocks,
                                          lens.data_ptr()), "block_tables")
        return tab, lens

    # ---- prefix caching
    def enable_prefix_cache(self) -> None:
        check(lib.pa_manager_enable_prefix_cache(self._h), "enable_prefix_cache")

    def add_seq_prompt(self, seq: int, tokens):
        """New sequence holding the prompt `tokens` (ids).  Returns (slots int64
        [n], -1 for the leading tokens served from the cache; num_cached)."""
        ids = torch.as_tensor(list(tokens) if not torch.is_tensor(tokens) else tokens,
                              dtype=torch.int32).contiguous()
        n = ids.numel()
        slots = torch.empty(max(n, 1), dtype=torch.int64)
        k = C.c_int(0)
        check(lib.pa_manager_add_seq_prompt(self._h, seq, C.cast(ids.data_ptr(), _pi32), n,
                                            C.cast(slots.data_ptr(), _pi64), C.byref(k)),
              "add_seq_prompt")
        return slots[:n], k.value

    def prefix_cache_stats(self) -> dict:
        st = (C.c_int64 * 4)()
        check(lib.pa_manager_prefix_cache_stats(self._h, st), "prefix_cache_stats")
        return dict(cached_blocks=st[0], hits=st[1], misses=st[2], evictions=st[3])
