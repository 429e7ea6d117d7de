"""Oracle for paged decode attention: plain, slow, float64, CPU only.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference legs may import it.  It shares no code
with the CUDA path (``paged_kv_cache_426_b200``) and imports nothing from it;
the only common dependency is the seeded input module ``workloads``.

Modules:
* ``blocks``    - BlockAllocator (FIFO free pool + reference counts) and the
                  per-sequence block tables with on-demand growth and
                  copy-on-write;
* ``cache``     - cache write / block copy / gather through the block table,
                  at bit level in the storage dtype;
* ``attention`` - gather, then textbook softmax attention in float64;
* ``prefill``   - the causal multi-query (prefill chunk) form of the same;
* ``run``       - executes a workload's host script with the above (and
                  replays a prefill batch).

Every function is pinned by ``tests/test_oracle_pins.py`` against the pages'
worked examples (``tests/golden``), closed forms, brute force on tiny inputs
and invariants.
"""
from .attention import attend, decode_one, paged_decode
from .blocks import BlockAllocator, BlockManager, BlockStateError, OutOfBlocks
from .prefill import paged_prefill, prefill_rows
from .cache import (STORAGE, as_storage, copy_blocks, empty_cache, gather_kv,
                    reshape_and_cache, to_f64)
from .run import OracleRun, PrefillRecord, StepRecord, max_blocks_needed, run, run_prefill

__all__ = [
    "attend", "decode_one", "paged_decode", "paged_prefill", "prefill_rows",
    "BlockAllocator", "BlockManager",
    "BlockStateError", "OutOfBlocks", "STORAGE", "as_storage", "copy_blocks",
    "empty_cache", "gather_kv", "reshape_and_cache", "to_f64", "OracleRun",
    "StepRecord", "max_blocks_needed", "run", "PrefillRecord", "run_prefill",
]
