"""pa_decode_noalloc: attention for callers that cannot allocate device memory.

Such callers (code inside a device memory allocator or pool, plug-in hosts that
pass in only the tensors they own, launch sequences that must keep the memory
footprint fixed) cannot hand pa_decode a workspace of their own.  The entry
point takes the workspace from a fixed array inside the library instead.

The GPU test calls it through the C ABI several times in a row on problems of
different lengths and head counts, all with split contexts, so that each call
reads partials from an array the previous call left full of its own.  Every call
must equal pa_decode on the same inputs bit for bit (the same kernels run; a unit
is computed by one warp and the merge is deterministic, so any difference is a
scratch-layout fault) and match the fp64 oracle within the decode tolerance.
This file is collected last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle as oracle_pkg
from gpu_cases import assert_close
from pins import BF16, F16, PagedCase
from paged_kv_cache_374_b200 import binding as pa

TDT = {F16: torch.float16, BF16: torch.bfloat16}
CODE = {F16: pa.PA_F16, BF16: pa.PA_BF16}
WK = {F16: "f16", BF16: "bf16"}


def _dev(bits, dtype):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(TDT[dtype]).cuda()


def _c_noalloc(c, q, kc, vc, tables, lens, out, err=None, partition_tokens=0):
    """Direct C-ABI call: nothing on this path allocates."""
    s, h, d = q.shape
    nb, bs = kc.shape[:2]
    return pa._lib.pa_decode_noalloc(
        ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kc.data_ptr()), ctypes.c_void_p(vc.data_ptr()),
        ctypes.c_void_p(tables.data_ptr()), ctypes.c_void_p(lens.data_ptr()), ctypes.c_float(c.scale), c.Hk,
        ctypes.c_void_p(out.data_ptr()), s, h, d, bs, nb, tables.shape[1], CODE[c.dtype], partition_tokens,
        ctypes.c_void_p(err.data_ptr()) if err is not None else None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _case(seed, lens, heads, kv_heads, dtype):
    rng = np.random.default_rng(seed)
    c = PagedCase(rng, lens, heads, kv_heads, 128, 16, dtype, 1 / math.sqrt(128), extra_blocks=3)
    return dict(c=c, q=_dev(c.q, dtype), kc=_dev(c.k_cache, dtype), vc=_dev(c.v_cache, dtype),
                tb=torch.from_numpy(c.tables).cuda(), ln=torch.from_numpy(c.lens).cuda())


@pytest.mark.gpu
def test_noalloc_equals_pa_decode_and_oracle_on_calls_in_a_row():
    cases = [_case(41, [1800, 700, 33, 2500], 8, 8, F16),              # MHA, split sequences
             _case(43, [3100, 260, 4999, 90, 1300], 16, 4, BF16),      # GQA group 4, other lengths
             _case(42, [5, 17, 48, 300, 0], 4, 2, F16)]                # one partition, an empty context
    order = [0, 1, 0, 2]              # case 0 again after case 1 filled the array with its own partials
    refs = []
    for k in cases:                   # pa_decode with its own workspace (allocated through torch)
        ref = torch.empty_like(k["q"])
        pa.pa_decode(k["q"], k["kc"], k["vc"], k["tb"], k["ln"], k["c"].scale, k["c"].Hk, ref)
        refs.append(ref)
    outs = [torch.full_like(cases[i]["q"], float("nan")) for i in order]
    errs = torch.zeros(len(order), dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    reserved = torch.cuda.memory_reserved()
    free_after_first = None
    for n, i in enumerate(order):
        k = cases[i]
        st = _c_noalloc(k["c"], k["q"], k["kc"], k["vc"], k["tb"], k["ln"], outs[n], err=errs[n:n + 1])
        assert st == pa.PA_OK, pa.pa_status_string(st)
        torch.cuda.synchronize()
        if n == 0:                    # the first call on the device looks the array up (one-time set-up)
            free_after_first = torch.cuda.mem_get_info()[0]
    assert errs.tolist() == [0] * len(order)
    # no call allocated through torch, and the calls after the set-up took no device memory
    assert torch.cuda.memory_reserved() == reserved
    assert torch.cuda.mem_get_info()[0] >= free_after_first - (1 << 20)
    o = oracle_pkg.get()
    for n, i in enumerate(order):
        c = cases[i]["c"]
        assert torch.equal(outs[n], refs[i]), f"call {n}: differs from pa_decode"
        assert_close(outs[n], c.run(o, nthreads=8), WK[c.dtype], f"call {n} (case {i}) vs oracle")


def test_noalloc_refuses_sizes_beyond_its_array():
    """Needs no GPU: every check below comes before any CUDA call (a CUDA call
    without a GPU would return PA_ERR_CUDA)."""
    fake = ctypes.c_void_p(4096)      # aligned stand-ins: checked, never dereferenced
    need = pa.pa_decode_workspace_size(1024, 64, 8, 128, 16, 2048, 0)
    assert need > 64 << 20

    def call(num_seqs, heads, kv_heads):
        return pa._lib.pa_decode_noalloc(fake, fake, fake, fake, fake, ctypes.c_float(0.1), kv_heads, fake,
                                         num_seqs, heads, 128, 16, 10, 2048, pa.PA_F16, 0, None, None)
    assert call(1024, 64, 8) == pa.PA_ERR_UNSUPPORTED
    # pa_decode's own argument errors come first, whatever the size
    assert call(1024, 64, 7) == pa.PA_ERR_INVALID_ARG
    # an empty batch is done before the array is touched
    assert call(0, 64, 8) == pa.PA_OK
    st = pa._lib.pa_decode_noalloc(None, fake, fake, fake, fake, ctypes.c_float(0.1), 8, fake, 4, 64, 128, 16, 10,
                                   64, pa.PA_F16, 0, None, None)
    assert st == pa.PA_ERR_INVALID_ARG
