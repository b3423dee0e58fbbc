"""Python API over the C ABI of libpagedkv.so.

Only argument marshalling happens here; every step of the data path runs in
the library's CUDA kernels.  PyTorch supplies device memory and streams.

    pool = kv_pool_create(num_blocks, block_size, n_kv_heads, head_dim, torch.bfloat16)
    paged_kv_append(k, v, slot_mapping, pool=pool)
    out = paged_attention(q, pool.k_pool, pool.v_pool, block_tables, context_lens,
                          query_start_lens, scale)
    block_copy(src_dst_pairs, pool=pool)
    host = host_pool_create(num_host_blocks, pool)        # pinned, for swapping
    swap_blocks(pairs, to_host=True, host_pool=host, pool=pool)
"""

import ctypes
import weakref

import torch

from ._lib import (PK_BF16, PK_ERR_TIMEOUT, PK_F32, PK_PATH_CHUNK_TCGEN05,  # noqa: F401
                   PK_PATH_DECODE_BLOCKS, PK_PATH_TENSOR_CORE, BmStats, OutOfBlocks, PagedKVError,
                   check, lib)

_DTYPES = {torch.float32: PK_F32, torch.bfloat16: PK_BF16}
_WINDOW_SEQS = 512   # sequences per kernel launch window (the attention scratch stops growing there)
_pools = weakref.WeakValueDictionary()  # k_pool data_ptr -> KVPool


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _need(t, name, dtype, device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


class KVPool:
    """A pool of physical KV blocks on one GPU.

    k_pool / v_pool: [num_blocks, n_kv_heads, block_size, head_dim] tensors
    (owned here, through torch); the library holds a small descriptor.
    """

    def __init__(self, num_blocks, block_size, n_kv_heads, head_dim, dtype=torch.bfloat16,
                 device=None, k_pool=None, v_pool=None):
        if dtype not in _DTYPES:
            raise TypeError("pool dtype must be torch.float32 or torch.bfloat16")
        device = torch.device(device or "cuda")
        if device.type != "cuda":
            raise ValueError("the pool lives on a CUDA device")
        if device.index is None:
            device = torch.device("cuda", torch.cuda.current_device())
        shape = (num_blocks, n_kv_heads, block_size, head_dim)
        self.k_pool = k_pool if k_pool is not None else torch.zeros(shape, dtype=dtype, device=device)
        self.v_pool = v_pool if v_pool is not None else torch.zeros(shape, dtype=dtype, device=device)
        for name, t in (("k_pool", self.k_pool), ("v_pool", self.v_pool)):
            _need(t, name, dtype, device)
            if tuple(t.shape) != shape:
                raise ValueError(f"{name} must have shape {shape}")
        self.num_blocks, self.block_size = num_blocks, block_size
        self.n_kv_heads, self.head_dim, self.dtype, self.device = n_kv_heads, head_dim, dtype, device
        self._handle = ctypes.c_void_p()
        with torch.cuda.device(device):
            check(lib().pk_pool_create(num_blocks, block_size, n_kv_heads, head_dim, _DTYPES[dtype],
                                       _ptr(self.k_pool), _ptr(self.v_pool),
                                       ctypes.byref(self._handle)))
        self._workspaces = {}     # CUDA stream handle -> its workspace
        _pools[self.k_pool.data_ptr()] = self

    @property
    def handle(self):
        if not self._handle:
            raise RuntimeError("pool is closed")
        return self._handle

    def close(self):
        if self._handle:
            with torch.cuda.device(self.device):
                check(lib().pk_pool_destroy(self._handle))
            self._handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace(self, num_seqs, num_tokens, n_q_heads, max_blocks, stream=None):
        """Device scratch for one attention call of this shape on `stream`
        (default: the current stream), kept and grown.  Calls in flight at the
        same time must not share scratch, so each stream has its own."""
        n = ctypes.c_size_t()
        check(lib().pk_attention_workspace_size(self.handle, num_seqs, num_tokens, n_q_heads,
                                                max_blocks, ctypes.byref(n)))
        if stream is None:
            stream = torch.cuda.current_stream(self.device)
        ws = self._workspaces.get(stream.cuda_stream)
        if ws is None or ws.numel() < n.value:
            # sized at once for a full launch window of sequences (the size stops
            # growing there; a few tens of MiB at most), so that a serving loop
            # whose batches grow does not allocate, and wait on the allocator, in
            # the middle of its steps
            full = ctypes.c_size_t()
            check(lib().pk_attention_workspace_size(self.handle, max(num_seqs, _WINDOW_SEQS), num_tokens,
                                                    n_q_heads, max_blocks, ctypes.byref(full)))
            # zero-filled once, on the stream that uses it; every completed call
            # leaves its counters zeroed again
            with torch.cuda.stream(stream):
                ws = torch.zeros(max(n.value, full.value, 256), dtype=torch.uint8, device=self.device)
            self._workspaces[stream.cuda_stream] = ws
        return ws

    def paths(self):
        """The PK_PATH_* bit set of the kernels that serve this pool."""
        f = ctypes.c_int()
        check(lib().pk_pool_paths(self.handle, ctypes.byref(f)))
        return f.value

    def check_device_errors(self):
        """PK_OK or the first device-side error code recorded since the last check.
        After PK_ERR_TIMEOUT every workspace of the pool is zeroed again: a call
        that gave up on a bounded wait may have left split-K counters set."""
        code = ctypes.c_int()
        check(lib().pk_check_device_errors(self.handle, _stream(self.device), ctypes.byref(code)))
        if code.value == PK_ERR_TIMEOUT:
            for ws in self._workspaces.values():
                ws.zero_()
            torch.cuda.synchronize(self.device)
        return code.value


def kv_pool_create(num_blocks, block_size, n_kv_heads, head_dim, dtype=torch.bfloat16, device=None):
    return KVPool(num_blocks, block_size, n_kv_heads, head_dim, dtype, device)


def _pool_of(k_pool, v_pool):
    pool = _pools.get(k_pool.data_ptr())
    if pool is None or pool.v_pool.data_ptr() != v_pool.data_ptr():
        raise ValueError("k_pool / v_pool were not created by kv_pool_create")
    return pool


def paged_kv_append(k, v, slot_mapping, *, pool):
    """Store k, v ([T, Hkv, d]) at slot_mapping ([T] int64, -1 = skip)."""
    d = pool.device
    _need(k, "k", pool.dtype, d)
    _need(v, "v", pool.dtype, d)
    _need(slot_mapping, "slot_mapping", torch.int64, d)
    T = k.shape[0]
    if tuple(k.shape) != (T, pool.n_kv_heads, pool.head_dim) or v.shape != k.shape or \
            slot_mapping.shape != (T,):
        raise ValueError("k, v must be [T, n_kv_heads, head_dim] and slot_mapping [T]")
    check(lib().pk_paged_kv_append(pool.handle, _ptr(k), _ptr(v), _ptr(slot_mapping), T, _stream(d)))


def block_copy(src_dst_pairs, *, pool):
    """Copy whole blocks src -> dst (int32 [n, 2] on the pool's device)."""
    d = pool.device
    _need(src_dst_pairs, "src_dst_pairs", torch.int32, d)
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [n, 2]")
    check(lib().pk_block_copy(pool.handle, _ptr(src_dst_pairs), src_dst_pairs.shape[0], _stream(d)))


class HostPool:
    """Page-locked host blocks with a device pool's block geometry, the target
    of swapped-out blocks: k / v [num_host_blocks, n_kv_heads, block_size,
    head_dim] pinned CPU tensors."""

    def __init__(self, num_host_blocks, pool):
        shape = (num_host_blocks, pool.n_kv_heads, pool.block_size, pool.head_dim)
        self.k = torch.zeros(shape, dtype=pool.dtype, pin_memory=True)
        self.v = torch.zeros(shape, dtype=pool.dtype, pin_memory=True)
        self.num_blocks = num_host_blocks


def host_pool_create(num_host_blocks, pool):
    return HostPool(num_host_blocks, pool)


def swap_blocks(pairs, *, to_host, host_pool, pool):
    """Move whole blocks between the device pool and a host pool (int32
    [n, 2] pairs on the pool's device): to_host, (device, host) pairs;
    otherwise (host, device) pairs.  Asynchronous on the current stream."""
    d = pool.device
    _need(pairs, "pairs", torch.int32, d)
    if pairs.dim() != 2 or pairs.shape[1] != 2:
        raise ValueError("pairs must be [n, 2]")
    check(lib().pk_swap_blocks(pool.handle, _ptr(host_pool.k), _ptr(host_pool.v), host_pool.num_blocks,
                               _ptr(pairs), pairs.shape[0], 1 if to_host else 0, _stream(d)))


def paged_attention(q, k_pool, v_pool, block_tables, context_lens, query_start_lens, scale,
                    out=None):
    """Attention of q ([T, Hq, d]) over each sequence's paged K/V.

    block_tables int32 [B, W]; context_lens int32 [B] (tokens stored, this
    step's included); query_start_lens int32 [B + 1]; returns [T, Hq, d].
    """
    pool = _pool_of(k_pool, v_pool)
    d = pool.device
    _need(q, "q", pool.dtype, d)
    _need(block_tables, "block_tables", torch.int32, d)
    _need(context_lens, "context_lens", torch.int32, d)
    _need(query_start_lens, "query_start_lens", torch.int32, d)
    T, Hq, hd = q.shape
    B = context_lens.shape[0]
    if hd != pool.head_dim or block_tables.dim() != 2 or block_tables.shape[0] != B or \
            query_start_lens.shape != (B + 1,):
        raise ValueError("inconsistent shapes")
    if out is None:
        out = torch.empty_like(q)
    else:
        _need(out, "out", pool.dtype, d)
    W = block_tables.shape[1]
    ws = pool.workspace(B, T, Hq, W)
    check(lib().pk_paged_attention(pool.handle, _ptr(q), _ptr(out), _ptr(block_tables), W,
                                   _ptr(context_lens), _ptr(query_start_lens), B, T, Hq,
                                   float(scale), _ptr(ws), ws.numel(), _stream(d)))
    return out


def paged_attention_append(q, k, v, k_pool, v_pool, block_tables, context_lens, query_start_lens, scale,
                           out=None):
    """Store the query rows' own K/V (k, v: [T, Hkv, d]) at their positions
    (position c_b - q_b + i of sequence b, slot from its block table), then
    attend: the same as paged_kv_append with the slots the tables give,
    followed by paged_attention, in one call."""
    pool = _pool_of(k_pool, v_pool)
    d = pool.device
    _need(q, "q", pool.dtype, d)
    _need(k, "k", pool.dtype, d)
    _need(v, "v", pool.dtype, d)
    _need(block_tables, "block_tables", torch.int32, d)
    _need(context_lens, "context_lens", torch.int32, d)
    _need(query_start_lens, "query_start_lens", torch.int32, d)
    T, Hq, hd = q.shape
    B = context_lens.shape[0]
    if hd != pool.head_dim or block_tables.dim() != 2 or block_tables.shape[0] != B or \
            query_start_lens.shape != (B + 1,) or tuple(k.shape) != (T, pool.n_kv_heads, hd) or \
            k.shape != v.shape:
        raise ValueError("inconsistent shapes")
    if out is None:
        out = torch.empty_like(q)
    else:
        _need(out, "out", pool.dtype, d)
    W = block_tables.shape[1]
    ws = pool.workspace(B, T, Hq, W)
    check(lib().pk_paged_attention_append(pool.handle, _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                          _ptr(block_tables), W, _ptr(context_lens),
                                          _ptr(query_start_lens), B, T, Hq, float(scale), _ptr(ws),
                                          ws.numel(), _stream(d)))
    return out


class BlockManager:
    """Host block manager (free list, tables, reference counts, fork, copy-on-write)."""

    def __init__(self, num_blocks, block_size):
        self.num_blocks, self.block_size = num_blocks, block_size
        self._h = ctypes.c_void_p()
        check(lib().pk_bm_create(num_blocks, block_size, ctypes.byref(self._h)))

    def __del__(self):
        if getattr(self, "_h", None):
            lib().pk_bm_destroy(self._h)
            self._h = None

    def add_seq(self):
        s = ctypes.c_int64()
        check(lib().pk_bm_add_seq(self._h, ctypes.byref(s)))
        return s.value

    def blocks_needed(self, seq, n):
        r = ctypes.c_int()
        check(lib().pk_bm_blocks_needed(self._h, seq, n, ctypes.byref(r)))
        return r.value

    def append_slots(self, seq, n):
        """Returns (slots, pairs); raises OutOfBlocks with nothing changed."""
        slots = (ctypes.c_int64 * max(n, 1))()
        pairs = (ctypes.c_int32 * 2)()
        npairs = ctypes.c_int()
        check(lib().pk_bm_append_slots(self._h, seq, n, slots, pairs, 1, ctypes.byref(npairs)))
        return list(slots[:n]), [(pairs[0], pairs[1])] if npairs.value else []

    def append_one_each(self, seqs):
        """One token for each seq in order, stopping at the first that needs a
        block when none is free.  Returns (number served, their slots, the
        copy-on-write pairs in order)."""
        n = len(seqs)
        ids = (ctypes.c_int64 * max(n, 1))(*seqs)
        slots = (ctypes.c_int64 * max(n, 1))()
        pairs = (ctypes.c_int32 * max(2 * n, 2))()
        npairs, done = ctypes.c_int(), ctypes.c_int()
        check(lib().pk_bm_append_one_each(self._h, ids, n, slots, pairs, ctypes.byref(npairs),
                                          ctypes.byref(done)))
        return done.value, list(slots[:done.value]), [(pairs[2 * i], pairs[2 * i + 1])
                                                      for i in range(npairs.value)]

    def fork(self, parent):
        c = ctypes.c_int64()
        check(lib().pk_bm_fork(self._h, parent, ctypes.byref(c)))
        return c.value

    def free(self, seq):
        check(lib().pk_bm_free(self._h, seq))

    def set_host_blocks(self, num_host_blocks):
        check(lib().pk_bm_set_host_blocks(self._h, num_host_blocks))

    def _swap(self, fn, seq):
        cap = self.length(seq) // self.block_size + 2
        buf = (ctypes.c_int32 * (2 * cap))()
        n = ctypes.c_int()
        check(fn(self._h, seq, buf, cap, ctypes.byref(n)))
        return [(buf[2 * i], buf[2 * i + 1]) for i in range(n.value)]

    def swap_out(self, seq):
        """Move all of seq's blocks to the host pool; returns the (device, host)
        pairs to copy.  Raises OutOfBlocks (host pool short) or PagedKVError
        (shared blocks), with nothing changed."""
        return self._swap(lib().pk_bm_swap_out, seq)

    def swap_in(self, seq):
        """Bring a swapped seq back; returns the (host, device) pairs to copy.
        Raises OutOfBlocks with nothing changed."""
        return self._swap(lib().pk_bm_swap_in, seq)

    @staticmethod
    def _keys(keys):
        return (ctypes.c_uint64 * max(len(keys), 1))(*[k & 0xFFFFFFFFFFFFFFFF for k in keys])

    def cache_blocks(self, seq, keys):
        """Register seq's first len(keys) (full) blocks in the prefix cache."""
        check(lib().pk_bm_cache_blocks(self._h, seq, self._keys(keys), len(keys)))

    def cached_prefix(self, keys):
        n = ctypes.c_int()
        check(lib().pk_bm_cached_prefix(self._h, self._keys(keys), len(keys), ctypes.byref(n)))
        return n.value

    def add_seq_cached(self, keys):
        """New sequence on the cached blocks of keys' longest cached prefix;
        returns (seq id, blocks hit)."""
        s, n = ctypes.c_int64(), ctypes.c_int()
        check(lib().pk_bm_add_seq_cached(self._h, self._keys(keys), len(keys), ctypes.byref(s),
                                         ctypes.byref(n)))
        return s.value, n.value

    def set_state_slots(self, num_slots):
        """Add a pool of fixed-size per-sequence state slots (two-pool manager)."""
        check(lib().pk_bm_set_state_slots(self._h, num_slots))

    def state_slot(self, seq):
        r = ctypes.c_int()
        check(lib().pk_bm_state_slot(self._h, seq, ctypes.byref(r)))
        return r.value

    def is_swapped(self, seq):
        r = ctypes.c_int()
        check(lib().pk_bm_is_swapped(self._h, seq, ctypes.byref(r)))
        return bool(r.value)

    def block_table(self, seq):
        n = ctypes.c_int()
        cap = self.length(seq) // self.block_size + 2
        buf = (ctypes.c_int32 * cap)()
        check(lib().pk_bm_block_table(self._h, seq, buf, cap, ctypes.byref(n)))
        return list(buf[:n.value])

    def fill_tables(self, seqs, width):
        """int32 tensor [len(seqs), width] of block tables, -1 padded (host memory)."""
        out = torch.empty((len(seqs), width), dtype=torch.int32)
        ids = (ctypes.c_int64 * max(len(seqs), 1))(*seqs)
        check(lib().pk_bm_fill_tables(self._h, ids, len(seqs), _ptr(out), width))
        return out

    def length(self, seq):
        n = ctypes.c_int64()
        check(lib().pk_bm_seq_len(self._h, seq, ctypes.byref(n)))
        return n.value

    def refcount(self, block):
        n = ctypes.c_int()
        check(lib().pk_bm_refcount(self._h, block, ctypes.byref(n)))
        return n.value

    def stats(self):
        s = BmStats()
        check(lib().pk_bm_get_stats(self._h, ctypes.byref(s)))
        return {name: getattr(s, name) for name, _ in BmStats._fields_}

    def num_free(self):
        n = ctypes.c_int()
        check(lib().pk_bm_num_free(self._h, ctypes.byref(n)))
        return n.value

    def num_used(self):
        return self.stats()["used_blocks"]

    def tail_waste(self):
        return self.stats()["tail_waste_slots"]
