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
    assert L.pk_paged_kv_append(None, None, None, None, 1, None) == 1
    assert L.pk_block_copy(None, None, 1, None) == 1
