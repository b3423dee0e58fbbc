"""Oracle: plain, slow, CPU definitions of what the paged-KV path computes.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only ``tests/``, the package smoke check (``__graft_entry__.smoke``) and the
bench's CPU-baseline leg call it.  It shares no code with the CUDA path.

Contents
--------
``attention.c`` (float64 C, built here into ``liboracle.so``)
    paged attention with causal chunks and GQA, the plain definition.
``kv_ops.py``
    slot-mapped KV append, whole-block copy (copy-on-write) and whole-block
    swaps between the device pool and a host pool.
``allocator.py``
    host block manager: free list, block tables, reference counts, fork,
    copy-on-write, tail-waste accounting, swapping to a host pool.
``capacity.py``
    the capacity arithmetic the pages print (token-slot toy, KV bytes per
    token, sessions per pool).

Every pin that ties these to the pages lives in ``tests/test_oracle_*.py``.
"""

from .attention import paged_attention, paged_attention_rows, num_threads, set_num_threads  # noqa: F401
from .kv_ops import kv_append, block_copy, swap_blocks  # noqa: F401
from .allocator import OracleBlockManager, OracleOOM  # noqa: F401
from . import capacity  # noqa: F401
