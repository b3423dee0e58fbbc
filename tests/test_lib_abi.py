"""The C-ABI library loads without a GPU, exports every function the public
header declares, and rejects bad host-side arguments before touching CUDA."""

import ctypes

import pytest

from paged_kv_cache_chunked_b200 import _lib


def test_every_declared_symbol_is_exported():
    L = _lib.lib()
    declared = _lib.header_symbols()
    assert len(declared) >= 20
    missing = [s for s in declared if not hasattr(L, s)]
    assert missing == []
    # the binding wraps exactly what the header declares
    assert sorted(_lib.SIGNATURES) == declared


def test_version_and_error_strings():
    L = _lib.lib()
    assert b"sm_100a" in L.pk_version()
    out = ctypes.c_void_p()
    rc = L.pk_pool_create(0, 16, 8, 128, _lib.PK_BF16, None, None, ctypes.byref(out))
    assert rc == 1 and not out
    assert b"positive" in L.pk_last_error()


@pytest.mark.parametrize("args", [
    (16, 16, 8, 512, _lib.PK_BF16),   # head_dim above the limit
    (16, 16, 8, 128, 7),              # unknown dtype
])
def test_pool_create_rejects_unsupported(args):
    L = _lib.lib()
    out = ctypes.c_void_p()
    fake = ctypes.c_void_p(1 << 20)   # never dereferenced: rejected first
    assert L.pk_pool_create(*args, fake, fake, ctypes.byref(out)) == 3


def test_null_pool_is_rejected():
    L = _lib.lib()
    assert L.pk_paged_attention(None, None, None, None, 1, None, None, 1, 1, 1, 1.0, None, 0, None) == 1
    assert L.pk_paged_attention_append(None, None, None, None, None, None, 1, None, None, 1, 1, 1, 1.0,
                                       None, 0, None) == 1
    assert L.pk_paged_kv_append(None, None, None, None, 1, None) == 1
    assert L.pk_block_copy(None, None, 1, None) == 1
    assert L.pk_swap_blocks(None, None, None, 4, None, 1, 1, None) == 1


def test_block_manager_extensions_reject_bad_arguments():
    # swap pool, prefix cache and state slots: argument checks on the host,
    # each failure leaving the manager as it was
    L = _lib.lib()
    bm = ctypes.c_void_p()
    assert L.pk_bm_create(8, 4, ctypes.byref(bm)) == 0
    try:
        assert L.pk_bm_set_host_blocks(bm, -1) == 1
        assert L.pk_bm_set_host_blocks(bm, 4) == 0
        assert L.pk_bm_set_host_blocks(bm, 4) == 1            # only once
        seq = ctypes.c_int64()
        assert L.pk_bm_add_seq(bm, ctypes.byref(seq)) == 0
        assert L.pk_bm_set_state_slots(bm, 2) == 1            # sequences exist already
        slots = (ctypes.c_int64 * 6)()
        pairs = (ctypes.c_int32 * 2)()
        n = ctypes.c_int()
        assert L.pk_bm_append_slots(bm, seq.value, 6, slots, pairs, 1, ctypes.byref(n)) == 0
        keys = (ctypes.c_uint64 * 2)(11, 12)
        assert L.pk_bm_cache_blocks(bm, seq.value, keys, 2) == 1   # block 1 holds 2 of 4 slots
        assert L.pk_bm_cache_blocks(bm, seq.value, keys, 1) == 0
        hit = ctypes.c_int()
        assert L.pk_bm_cached_prefix(bm, keys, 2, ctypes.byref(hit)) == 0 and hit.value == 1
        out = (ctypes.c_int32 * 2)()
        assert L.pk_bm_swap_out(bm, seq.value, out, 1, ctypes.byref(n)) == 1   # 2 pairs, room for 1
        assert L.pk_bm_swap_in(bm, seq.value, out, 1, ctypes.byref(n)) == 1    # not swapped
        sw = ctypes.c_int()
        assert L.pk_bm_is_swapped(bm, seq.value, ctypes.byref(sw)) == 0 and sw.value == 0
        assert L.pk_bm_is_swapped(bm, 99, ctypes.byref(sw)) == 1
        st = _lib.BmStats()
        assert L.pk_bm_get_stats(bm, ctypes.byref(st)) == 0
        assert (st.host_blocks, st.host_free_blocks, st.cached_blocks, st.state_slots) == (4, 4, 1, 0)
    finally:
        L.pk_bm_destroy(bm)
