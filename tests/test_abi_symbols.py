"""libpa.so loads on a machine without a GPU and exports every function pa.h declares."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b(pa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from paged_kv_cache_374_b200 import build
    path = build.build()
    return ctypes.CDLL(path)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("pa_reshape_and_cache", "pa_decode", "pa_decode_workspace_size", "pa_allocator_create",
                     "pa_alloc", "pa_alloc_n", "pa_free", "pa_add_ref", "pa_fork", "pa_append_slots"):
        assert required in names
    assert len(names) >= 19


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_exposes_the_same_names():
    from paged_kv_cache_374_b200 import binding
    missing = [n for n in declared_functions() if not hasattr(binding, n)]
    assert not missing, missing


def test_host_checks_reject_bad_arguments_without_a_gpu():
    """Argument checks run before any CUDA call, so they work without a device."""
    from paged_kv_cache_374_b200 import binding as pa
    lib = pa._lib
    # unsupported head_dim / block size / dtype; num_heads not a multiple of num_kv_heads
    args = dict(q=None, k=None, v=None, t=None, l=None)
    call = lambda **kw: lib.pa_decode(None, None, None, None, None, 0.125, kw.get("hk", 4), None, kw.get("s", 2),
                                      kw.get("h", 4), kw.get("d", 128), kw.get("bs", 16), 10, 4, kw.get("dt", 0),
                                      kw.get("pt", 0), None, 0, None, None)
    assert call(d=96) == pa.PA_ERR_UNSUPPORTED
    assert call(bs=8) == pa.PA_ERR_UNSUPPORTED
    assert call(dt=7) == pa.PA_ERR_UNSUPPORTED
    assert call(h=6, hk=4) == pa.PA_ERR_INVALID_ARG
    assert call(pt=100) == pa.PA_ERR_INVALID_ARG
    assert call() == pa.PA_ERR_INVALID_ARG          # null pointers
    assert call(s=0) == pa.PA_OK                    # empty batch: nothing to do
    assert lib.pa_reshape_and_cache(None, None, None, None, None, 0, 4, 64, 16, 4, 0, None, None) == pa.PA_OK
    assert lib.pa_reshape_and_cache(None, None, None, None, None, 3, 4, 64, 16, 4, 0, None, None) == \
        pa.PA_ERR_INVALID_ARG
    assert lib.pa_reshape_and_cache(None, None, None, None, None, 3, 4, 60, 16, 4, 0, None, None) == \
        pa.PA_ERR_UNSUPPORTED
    # misaligned pointers are refused before anything is launched
    odd = ctypes.c_void_p(0x1008)
    al = ctypes.c_void_p(0x1000)
    assert lib.pa_decode(odd, al, al, al, al, 0.1, 4, al, 2, 4, 128, 16, 10, 4, 0, 0, None, 0, None, None) == \
        pa.PA_ERR_INVALID_ARG


def test_workspace_size_arithmetic():
    from paged_kv_cache_374_b200 import binding as pa
    # one partition: only the 256 bytes of scheduling counters
    assert pa.pa_decode_workspace_size(8, 32, 32, 128, 16, 4, 512) == 256
    # 4096 tokens at 512 per partition: a merge counter and a merge-queue entry per (s, h), then
    # 8 partitions of (m, l, o[128]) per (s, h), in 256-byte aligned pieces
    n = pa.pa_decode_workspace_size(64, 32, 32, 128, 16, 256, 512)
    sh, p = 64 * 32, 8
    up = lambda x: (x + 255) // 256 * 256
    assert n == 256 + 2 * up(sh * 4) + 2 * up(sh * p * 4) + up(sh * p * 128 * 4)
    assert pa.pa_decode_workspace_size(8, 32, 32, 128, 16, 4, 100) == 0   # bad partition size
    assert pa.pa_decode_partition_tokens(64, 32, 32, 128, 16, 256) % 64 == 0
