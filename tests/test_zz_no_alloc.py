"""pa_decode_noalloc: attention for callers that cannot allocate device memory.

Such callers (code inside a device memory allocator or pool, plug-in hosts that
pass in only the tensors they own, launch sequences that must keep the memory
footprint fixed) cannot hand pa_decode a workspace of their own.  The entry
point takes the workspace from a fixed array inside the library instead.  These
tests call it through the C ABI and compare it with pa_decode on the same inputs,
two calls in a row (the second reuses the array the first one left behind),
within the decode tolerance the other tests use.  This file is collected last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from gpu_cases import assert_close
from pins import F16, PagedCase
from paged_kv_cache_374_b200 import binding as pa


def _dev(bits, dtype=torch.float16):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(dtype).cuda()


def _c_noalloc(q, kc, vc, tables, lens, scale, hk, out, partition_tokens=0, err=None):
    """Direct C-ABI call (no Python-side allocation on this path)."""
    s, h, d = q.shape
    nb, bs = kc.shape[:2]
    return pa._lib.pa_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(vc.data_ptr()),
        ctypes.c_void_p(tables.data_ptr()), ctypes.c_void_p(lens.data_ptr()), ctypes.c_float(scale), hk,
        ctypes.c_void_p(out.data_ptr()), s, h, d, bs, nb, tables.shape[1], pa.PA_F16, partition_tokens,
        ctypes.c_void_p(err.data_ptr()) if err is not None else None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _case(seed, lens, heads, kv_heads):
    rng = np.random.default_rng(seed)
    c = PagedCase(rng, lens, heads, kv_heads, 128, 16, F16, 1 / math.sqrt(128), extra_blocks=3)
    return c, _dev(c.q), _dev(c.k_cache), _dev(c.v_cache), torch.from_numpy(c.tables).cuda(), \
        torch.from_numpy(c.lens).cuda()


@pytest.mark.gpu
def test_noalloc_matches_pa_decode_two_calls_in_a_row():
    cases = [_case(41, [1800, 700, 33, 2500], 8, 8),    # split sequences: partials and merge in the array
             _case(42, [5, 17, 48, 300, 0], 4, 2)]      # one partition, GQA, an empty context
    free_after = []
    for c, q, kc, vc, tb, ln in cases:
        ref = torch.empty_like(q)
        pa.pa_decode(q, kc, vc, tb, ln, c.scale, c.Hk, ref)
        out = torch.full_like(q, float("nan"))
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        st = _c_noalloc(q, kc, vc, tb, ln, c.scale, c.Hk, out, err=err)
        torch.cuda.synchronize()
        free_after.append((free_before, torch.cuda.mem_get_info()[0]))
        assert st == pa.PA_OK, pa.pa_status_string(st)
        assert err.item() == 0
        assert_close(out, ref.double().cpu().numpy(), "f16", "noalloc vs pa_decode")
    # the second call (set-up already done) leaves the device's free memory as it was
    assert free_after[1][0] == free_after[1][1]


def test_noalloc_refuses_sizes_beyond_its_array():
    """Needs no GPU: the size check comes before any CUDA call."""
    need = pa.pa_decode_workspace_size(1024, 64, 8, 128, 16, 2048, 0)
    assert need > 64 << 20
    st = pa._lib.pa_decode_noalloc(None, None, None, None, None, ctypes.c_float(0.1), 8, None, 1024, 64, 128, 16,
                                   10, 2048, pa.PA_F16, 0, None, None)
    assert st == pa.PA_ERR_UNSUPPORTED
