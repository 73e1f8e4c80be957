"""Thin Python binding over libpa.so's C ABI (include/pa.h), same names.

Argument marshalling only: torch tensors become device pointers and sizes, numpy
arrays become host pointers, status codes become ``PAError``.  Every step of the
path runs in the library's kernels; there is no fallback, and importing this
module fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY = os.path.join(_PKG, "libpa.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_OUT_OF_BLOCKS, PA_ERR_REFCOUNT, PA_ERR_CUDA = range(6)
PA_F16, PA_BF16 = 0, 1
PA_DEVERR_SLOT_RANGE, PA_DEVERR_TABLE_RANGE, PA_DEVERR_LEN_RANGE, PA_DEVERR_TIMEOUT = 1, 2, 4, 8
PA_DEVERR_GROUP_RANGE, PA_DEVERR_PAIR_CONFLICT = 16, 32

if not os.path.exists(LIBRARY):
    raise ImportError(f"{LIBRARY} is missing: build it with `python -m paged_kv_cache_374_b200.build` "
                      "(the library has no CPU fallback)")

_lib = ctypes.CDLL(LIBRARY)

_vp = ctypes.c_void_p
_i32 = ctypes.c_int
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)


def _sig(name, restype, *argtypes):
    f = getattr(_lib, name)
    f.restype = restype
    f.argtypes = list(argtypes)
    return f


_sig("pa_status_string", ctypes.c_char_p, _i32)
_sig("pa_reshape_and_cache", _i32, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp)
_sig("pa_decode_partition_tokens", _i32, _i32, _i32, _i32, _i32, _i32, _i32)
_sig("pa_decode_workspace_size", ctypes.c_size_t, _i32, _i32, _i32, _i32, _i32, _i32, _i32)
_sig("pa_decode", _i32, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
     _i32, _i32, _vp, ctypes.c_size_t, _vp, _vp)
_sig("pa_decode_step", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _i32, _vp, _i32, _i32, _i32,
     _i32, _i32, _i32, _i32, _i32, _vp, ctypes.c_size_t, _vp, _vp)
_sig("pa_decode_step_fp8", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, ctypes.c_float,
     ctypes.c_float, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, ctypes.c_size_t, _vp, _vp)
_sig("pa_decode_noalloc", _i32, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _i32, _vp, _i32, _i32, _i32, _i32, _i32,
     _i32, _i32, _i32, _vp, _vp)
_sig("pa_reshape_and_cache_fp8", _i32, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, ctypes.c_float,
     ctypes.c_float, _vp, _vp)
_sig("pa_decode_fp8", _i32, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, ctypes.c_float, ctypes.c_float, _i32, _vp, _i32,
     _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, ctypes.c_size_t, _vp, _vp)
_sig("pa_prefill", _i32, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
     _i32, _i32, _vp, _vp)
_sig("pa_decode_shared_prefix", _i32, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _i32, _vp, _i32, _i32, _i32, _i32, _i32,
     _i32, _i32, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _vp, ctypes.c_size_t, _vp, _vp)
_sig("pa_decode_step_shared_prefix", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float, _i32, _vp, _i32,
     _i32, _i32, _i32, _i32, _i32, _i32, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _vp, ctypes.c_size_t, _vp, _vp)
_sig("pa_find_shared_prefixes", _i32, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp,
     ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int))
_sig("pa_selftest_bounded_wait", _i32, _vp, _vp, _vp)
_sig("pa_allocator_create", _vp, _i32, _i32p)
_sig("pa_allocator_destroy", None, _vp)
_sig("pa_num_required_blocks", _i32, _i32, _i32)
_sig("pa_alloc", _i32, _vp, _i32p)
_sig("pa_alloc_n", _i32, _vp, _i32, _i32p)
_sig("pa_free", _i32, _vp, ctypes.c_int32)
_sig("pa_free_n", _i32, _vp, _i32, _i32p)
_sig("pa_add_ref", _i32, _vp, ctypes.c_int32)
_sig("pa_fork", _i32, _vp, _i32p, _i32, _i32p)
_sig("pa_refcount", _i32, _vp, ctypes.c_int32)
_sig("pa_num_free", _i32, _vp)
_sig("pa_num_blocks", _i32, _vp)
_sig("pa_usage", ctypes.c_double, _vp)
_sig("pa_append_slots", _i32, _vp, _i32p, _i32, _i32p, _i32, _i32, _i64p)
_sig("pa_prefill_slots", _i32, _vp, _i32p, _i32, _i32p, _i32p, _i32, _i32, _i64p)
_sig("pa_cow_prepare", _i32, _vp, _i32p, _i32, _i32p, _i32, _i32, _i32p, ctypes.POINTER(ctypes.c_int))
_sig("pa_copy_blocks", _i32, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp)
_sig("pa_swap_plan", _i32, _vp, _vp, _i32p, _i32, _i32p)
_sig("pa_swap_blocks", _i32, _vp, _vp, _i32, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _vp, _vp)


class PAError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        name = _lib.pa_status_string(status).decode()
        super().__init__(f"{what}: {name}" if what else name)


def _check(status: int, what: str):
    if status != PA_OK:
        raise PAError(status, what)


def pa_status_string(status: int) -> str:
    return _lib.pa_status_string(status).decode()


# ----------------------------------------------------------------- tensors

def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return PA_F16
    if t.dtype == torch.bfloat16:
        return PA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: float16 or bfloat16")


def _dev(t, name, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _h32(a: np.ndarray):
    """Host pointer of a C-contiguous int32 numpy array."""
    assert a.dtype == np.int32 and a.flags.c_contiguous
    return a.ctypes.data_as(_i32p)


def _h32_addr(a: np.ndarray) -> int:
    """Address of a C-contiguous int32 numpy array, for a void* argument (cheaper per
    call than building a typed pointer: the grouping runs every decode step)."""
    assert a.dtype == np.int32 and a.flags.c_contiguous
    return a.ctypes.data


def _stream(stream, like):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(like.device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def pa_reshape_and_cache(k, v, slot_mapping, k_cache, v_cache, err_word=None, stream=None) -> None:
    """K1.  k, v [N, Hk, d]; slot_mapping int64 [N]; caches [NB, B, Hk, d] (CUDA)."""
    import torch
    n, hk, d = k.shape
    nb, bs, hk2, d2 = k_cache.shape
    if v.shape != k.shape or v_cache.shape != k_cache.shape or (hk2, d2) != (hk, d):
        raise ValueError("shape mismatch")
    if slot_mapping.shape != (n,):
        raise ValueError("slot_mapping must be [num_tokens]")
    dt = _dtype_code(k)
    for t in (v, k_cache, v_cache):
        if t.dtype != k.dtype:
            raise TypeError("k, v and the caches must share one dtype")
    st = _lib.pa_reshape_and_cache(_dev(k, "k"), _dev(v, "v"), _dev(slot_mapping, "slot_mapping", torch.int64),
                                   _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), n, hk, d, bs, nb, dt,
                                   _dev(err_word, "err_word", torch.int32), _stream(stream, k))
    _check(st, "pa_reshape_and_cache")


def pa_decode_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq) -> int:
    return _lib.pa_decode_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                           max_blocks_per_seq)


def pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq,
                             partition_tokens=0) -> int:
    return _lib.pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                         max_blocks_per_seq, partition_tokens)


def pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, out, workspace=None,
              partition_tokens=0, err_word=None, stream=None):
    """K2 + K3.  q/out [S, H, d]; caches [NB, B, Hk, d]; block_tables int32 [S, MB];
    context_lens int32 [S]; workspace: a CUDA uint8 tensor of at least
    pa_decode_workspace_size(...) bytes, or None to have one made here (torch).
    Returns ``out``."""
    import torch
    s, h, d = q.shape
    nb, bs, hk, d2 = k_cache.shape
    if hk != num_kv_heads or d2 != d or v_cache.shape != k_cache.shape or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, MB] and context_lens [S]")
    mb = block_tables.shape[1]
    dt = _dtype_code(q)
    for t in (k_cache, v_cache, out):
        if t.dtype != q.dtype:
            raise TypeError("q, the caches and out must share one dtype")
    if workspace is None:
        need = pa_decode_workspace_size(s, h, hk, d, bs, mb, partition_tokens)
        workspace = torch.zeros(max(need, 1), dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = _lib.pa_decode(_dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                        _dev(block_tables, "block_tables", torch.int32),
                        _dev(context_lens, "context_lens", torch.int32), float(scale), hk, _dev(out, "out"),
                        s, h, d, bs, nb, mb, dt, int(partition_tokens), ws_ptr, ws_bytes,
                        _dev(err_word, "err_word", torch.int32), _stream(stream, q))
    _check(st, "pa_decode")
    return out


def pa_decode_step(k, v, slot_mapping, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, out,
                   workspace=None, partition_tokens=0, err_word=None, stream=None):
    """K1 then K2 + K3 in one call: each sequence's new k/v [S, Hk, d] into its slot
    (slot_mapping int64 [S]), then attention as pa_decode.  Returns ``out``."""
    import torch
    s, h, d = q.shape
    nb, bs, hk, d2 = k_cache.shape
    if hk != num_kv_heads or d2 != d or v_cache.shape != k_cache.shape or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if k.shape != (s, hk, d) or v.shape != k.shape or slot_mapping.shape != (s,):
        raise ValueError("k, v must be [S, Hk, d] and slot_mapping [S]")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, MB] and context_lens [S]")
    mb = block_tables.shape[1]
    dt = _dtype_code(q)
    for t in (k, v, k_cache, v_cache, out):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, the caches and out must share one dtype")
    if workspace is None:
        need = pa_decode_workspace_size(s, h, hk, d, bs, mb, partition_tokens)
        workspace = torch.zeros(max(need, 1), dtype=torch.uint8, device=q.device)
    st = _lib.pa_decode_step(_dev(k, "k"), _dev(v, "v"), _dev(slot_mapping, "slot_mapping", torch.int64),
                             _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                             _dev(block_tables, "block_tables", torch.int32),
                             _dev(context_lens, "context_lens", torch.int32), float(scale), hk, _dev(out, "out"),
                             s, h, d, bs, nb, mb, dt, int(partition_tokens), _dev(workspace, "workspace"),
                             workspace.numel() * workspace.element_size(), _dev(err_word, "err_word", torch.int32),
                             _stream(stream, q))
    _check(st, "pa_decode_step")
    return out


def pa_decode_step_fp8(k, v, slot_mapping, q, k_cache, v_cache, block_tables, context_lens, scale, k_scale,
                       v_scale, num_kv_heads, out, workspace=None, partition_tokens=0, err_word=None, stream=None):
    """pa_decode_step over uint8 E4M3 caches: the fp8 cache write then pa_decode_fp8,
    in one call.  Returns ``out``."""
    import torch
    s, h, d = q.shape
    nb, bs, hk, d2 = k_cache.shape
    if hk != num_kv_heads or d2 != d or v_cache.shape != k_cache.shape or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if k.shape != (s, hk, d) or v.shape != k.shape or slot_mapping.shape != (s,):
        raise ValueError("k, v must be [S, Hk, d] and slot_mapping [S]")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, MB] and context_lens [S]")
    if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise TypeError("fp8 caches are uint8 E4M3 codes")
    for t in (k, v, out):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v and out must share one dtype")
    mb = block_tables.shape[1]
    if workspace is None:
        need = pa_decode_workspace_size(s, h, hk, d, bs, mb, partition_tokens)
        workspace = torch.zeros(max(need, 1), dtype=torch.uint8, device=q.device)
    st = _lib.pa_decode_step_fp8(_dev(k, "k"), _dev(v, "v"), _dev(slot_mapping, "slot_mapping", torch.int64),
                                 _dev(q, "q"), _dev(k_cache, "k_cache", torch.uint8),
                                 _dev(v_cache, "v_cache", torch.uint8),
                                 _dev(block_tables, "block_tables", torch.int32),
                                 _dev(context_lens, "context_lens", torch.int32), float(scale), float(k_scale),
                                 float(v_scale), hk, _dev(out, "out"), s, h, d, bs, nb, mb, _dtype_code(q),
                                 int(partition_tokens), _dev(workspace, "workspace"),
                                 workspace.numel() * workspace.element_size(), _dev(err_word, "err_word", torch.int32),
                                 _stream(stream, q))
    _check(st, "pa_decode_step_fp8")
    return out


class SharedPrefixes:
    """Result of pa_find_shared_prefixes (host numpy arrays)."""

    def __init__(self, seq_start, group_offsets, group_members, num_groups, max_group_size, max_shared_tokens):
        self.seq_start = seq_start
        self.group_offsets = group_offsets
        self.group_members = group_members
        self.num_groups = num_groups
        self.max_group_size = max_group_size
        self.max_shared_tokens = max_shared_tokens

    def to(self, device):
        """The three arrays as int32 tensors on ``device`` (a tuple)."""
        import torch
        return tuple(torch.from_numpy(np.ascontiguousarray(x)).to(device)
                     for x in (self.seq_start, self.group_offsets, self.group_members))


def pa_find_shared_prefixes(block_tables: np.ndarray, context_lens: np.ndarray, block_size: int,
                            partition_tokens: int) -> SharedPrefixes:
    """Host grouping of sequences that share whole partitions through the same blocks."""
    tb = np.ascontiguousarray(block_tables, dtype=np.int32)
    ln = np.ascontiguousarray(context_lens, dtype=np.int32)
    s, mb = tb.shape
    start = np.zeros(s, dtype=np.int32)
    offs = np.zeros(s + 1, dtype=np.int32)
    members = np.zeros(max(s, 1), dtype=np.int32)
    ng, mg, mt = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    st = _lib.pa_find_shared_prefixes(_h32_addr(tb), _h32_addr(ln), s, mb, block_size, partition_tokens,
                                      _h32_addr(start), _h32_addr(offs), _h32_addr(members), ctypes.byref(ng),
                                      ctypes.byref(mg), ctypes.byref(mt))
    _check(st, "pa_find_shared_prefixes")
    n = int(ng.value)
    return SharedPrefixes(start, offs[: n + 1].copy(), members[: int(offs[n])].copy(), n, int(mg.value),
                          int(mt.value))


def pa_decode_shared_prefix(q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, out, seq_start,
                            group_offsets, group_members, num_groups, max_group_size, max_shared_tokens,
                            workspace=None, partition_tokens=0, err_word=None, stream=None):
    """pa_decode with the shared prefixes of groups attended once per group
    (seq_start / group_offsets / group_members: int32 device tensors, e.g. from
    ``pa_find_shared_prefixes(...).to(device)``).  Returns ``out``."""
    import torch
    s, h, d = q.shape
    nb, bs, hk, d2 = k_cache.shape
    if hk != num_kv_heads or d2 != d or v_cache.shape != k_cache.shape or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, MB] and context_lens [S]")
    mb = block_tables.shape[1]
    dt = _dtype_code(q)
    for t in (k_cache, v_cache, out):
        if t.dtype != q.dtype:
            raise TypeError("q, the caches and out must share one dtype")
    if workspace is None:
        need = pa_decode_workspace_size(s, h, hk, d, bs, mb, partition_tokens)
        workspace = torch.zeros(max(need, 1), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _lib.pa_decode_shared_prefix(
        _dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32), _dev(context_lens, "context_lens", torch.int32),
        float(scale), hk, _dev(out, "out"), s, h, d, bs, nb, mb, dt, _dev(seq_start, "seq_start", torch.int32),
        int(num_groups), _dev(group_offsets, "group_offsets", torch.int32),
        _dev(group_members, "group_members", torch.int32), int(max_group_size), int(max_shared_tokens),
        int(partition_tokens), _dev(workspace, "workspace"), ws_bytes, _dev(err_word, "err_word", torch.int32),
        _stream(stream, q))
    _check(st, "pa_decode_shared_prefix")
    return out


def pa_decode_step_shared_prefix(k, v, slot_mapping, q, k_cache, v_cache, block_tables, context_lens, scale,
                                 num_kv_heads, out, seq_start, group_offsets, group_members, num_groups,
                                 max_group_size, max_shared_tokens, workspace=None, partition_tokens=0, err_word=None,
                                 stream=None):
    """K1 then pa_decode_shared_prefix in one call: each sequence's new k/v [S, Hk, d]
    into its slot (slot_mapping int64 [S]), then attention with the groups' shared
    prefixes attended once per group.  Returns ``out``."""
    import torch
    s, h, d = q.shape
    nb, bs, hk, d2 = k_cache.shape
    if hk != num_kv_heads or d2 != d or v_cache.shape != k_cache.shape or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if k.shape != (s, hk, d) or v.shape != k.shape or slot_mapping.shape != (s,):
        raise ValueError("k, v must be [S, Hk, d] and slot_mapping [S]")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, MB] and context_lens [S]")
    mb = block_tables.shape[1]
    dt = _dtype_code(q)
    for t in (k, v, k_cache, v_cache, out):
        if t.dtype != q.dtype:
            raise TypeError("q, k, v, the caches and out must share one dtype")
    if workspace is None:
        need = pa_decode_workspace_size(s, h, hk, d, bs, mb, partition_tokens)
        workspace = torch.zeros(max(need, 1), dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = _lib.pa_decode_step_shared_prefix(
        _dev(k, "k"), _dev(v, "v"), _dev(slot_mapping, "slot_mapping", torch.int64), _dev(q, "q"),
        _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32), float(scale), hk, _dev(out, "out"), s, h, d, bs, nb, mb, dt,
        _dev(seq_start, "seq_start", torch.int32), int(num_groups), _dev(group_offsets, "group_offsets", torch.int32),
        _dev(group_members, "group_members", torch.int32), int(max_group_size), int(max_shared_tokens),
        int(partition_tokens), _dev(workspace, "workspace"), ws_bytes, _dev(err_word, "err_word", torch.int32),
        _stream(stream, q))
    _check(st, "pa_decode_step_shared_prefix")
    return out


def pa_selftest_bounded_wait(err_word, outcome=None, stream=None) -> None:
    """Run the bounded-wait check (a wait nothing completes must time out and report)."""
    import torch
    st = _lib.pa_selftest_bounded_wait(_dev(err_word, "err_word", torch.int32), _dev(outcome, "outcome", torch.int32),
                                       _stream(stream, err_word))
    _check(st, "pa_selftest_bounded_wait")


def pa_decode_noalloc(q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, out,
                      partition_tokens=0, err_word=None, stream=None):
    """pa_decode with its workspace taken from the library's fixed device array
    (for callers that cannot allocate device memory).  Returns ``out``."""
    import torch
    s, h, d = q.shape
    nb, bs, hk, d2 = k_cache.shape
    if hk != num_kv_heads or d2 != d or v_cache.shape != k_cache.shape or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if block_tables.dim() != 2 or block_tables.shape[0] != s or context_lens.shape != (s,):
        raise ValueError("block_tables must be [S, MB] and context_lens [S]")
    dt = _dtype_code(q)
    for t in (k_cache, v_cache, out):
        if t.dtype != q.dtype:
            raise TypeError("q, the caches and out must share one dtype")
    st = _lib.pa_decode_noalloc(_dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                                _dev(block_tables, "block_tables", torch.int32),
                                _dev(context_lens, "context_lens", torch.int32), float(scale), hk,
                                _dev(out, "out"), s, h, d, bs, nb, block_tables.shape[1], dt,
                                int(partition_tokens), _dev(err_word, "err_word", torch.int32), _stream(stream, q))
    _check(st, "pa_decode_noalloc")
    return out


def pa_reshape_and_cache_fp8(k, v, slot_mapping, k_cache, v_cache, k_scale, v_scale, err_word=None, stream=None):
    """K1 into fp8 caches.  k, v fp16/bf16 [N, Hk, d]; caches uint8 (E4M3 codes) [NB, B, Hk, d]."""
    import torch
    n, hk, d = k.shape
    nb, bs, hk2, d2 = k_cache.shape
    if v.shape != k.shape or v_cache.shape != k_cache.shape or (hk2, d2) != (hk, d):
        raise ValueError("shape mismatch")
    if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise TypeError("fp8 caches are uint8 tensors of E4M3 codes")
    dt = _dtype_code(k)
    st = _lib.pa_reshape_and_cache_fp8(_dev(k, "k", k.dtype), _dev(v, "v", k.dtype),
                                       _dev(slot_mapping, "slot_mapping", torch.int64), _dev(k_cache, "k_cache"),
                                       _dev(v_cache, "v_cache"), n, hk, d, bs, nb, dt, float(k_scale), float(v_scale),
                                       _dev(err_word, "err_word", torch.int32), _stream(stream, k))
    _check(st, "pa_reshape_and_cache_fp8")


def pa_decode_fp8(q, k_cache, v_cache, block_tables, context_lens, scale, k_scale, v_scale, num_kv_heads, out,
                  workspace=None, partition_tokens=0, err_word=None, stream=None):
    """K2 + K3 over fp8 caches (uint8 E4M3 codes [NB, B, Hk, d]); q / out fp16 or bf16."""
    import torch
    s, h, d = q.shape
    nb, bs, hk, d2 = k_cache.shape
    if hk != num_kv_heads or d2 != d or v_cache.shape != k_cache.shape or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise TypeError("fp8 caches are uint8 tensors of E4M3 codes")
    if out.dtype != q.dtype:
        raise TypeError("q and out must share one dtype")
    mb = block_tables.shape[1]
    dt = _dtype_code(q)
    if workspace is None:
        need = pa_decode_workspace_size(s, h, hk, d, bs, mb, partition_tokens)
        workspace = torch.zeros(max(need, 1), dtype=torch.uint8, device=q.device)
    st = _lib.pa_decode_fp8(_dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                            _dev(block_tables, "block_tables", torch.int32),
                            _dev(context_lens, "context_lens", torch.int32), float(scale), float(k_scale),
                            float(v_scale), hk, _dev(out, "out"), s, h, d, bs, nb, mb, dt, int(partition_tokens),
                            _dev(workspace, "workspace"), workspace.numel(), _dev(err_word, "err_word", torch.int32),
                            _stream(stream, q))
    _check(st, "pa_decode_fp8")
    return out


def pa_prefill(q, k_cache, v_cache, block_tables, context_lens, query_start, scale, num_kv_heads, out,
               max_query_len, err_word=None, stream=None):
    """Causal chunk attention.  q / out [T, H, d] packed by sequence; query_start int32 [S+1] (CUDA)."""
    import torch
    total, h, d = q.shape
    nb, bs, hk, d2 = k_cache.shape
    s = context_lens.shape[0]
    if hk != num_kv_heads or d2 != d or v_cache.shape != k_cache.shape or out.shape != q.shape:
        raise ValueError("shape mismatch")
    if query_start.shape != (s + 1,) or block_tables.shape[0] != s:
        raise ValueError("query_start must be [S+1] and block_tables [S, MB]")
    dt = _dtype_code(q)
    for t in (k_cache, v_cache, out):
        if t.dtype != q.dtype:
            raise TypeError("q, the caches and out must share one dtype")
    st = _lib.pa_prefill(_dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                         _dev(block_tables, "block_tables", torch.int32),
                         _dev(context_lens, "context_lens", torch.int32),
                         _dev(query_start, "query_start", torch.int32), float(scale), hk, _dev(out, "out"), s, h, d,
                         bs, nb, block_tables.shape[1], int(max_query_len), dt, _dev(err_word, "err_word", torch.int32),
                         _stream(stream, q))
    _check(st, "pa_prefill")
    return out


# --------------------------------------------------------------- allocator

def _np_i32(a, name):
    a = np.asarray(a)
    if a.dtype != np.int32 or not a.flags.c_contiguous:
        raise TypeError(f"{name} must be a C-contiguous int32 array")
    return a


def pa_allocator_create(num_blocks: int, initial_order=None) -> int:
    order = None
    if initial_order is not None:
        order = np.ascontiguousarray(initial_order, dtype=np.int32)
        if order.shape != (num_blocks,):
            raise ValueError("initial_order must have num_blocks entries")
    h = _lib.pa_allocator_create(num_blocks, order.ctypes.data_as(_i32p) if order is not None else None)
    if not h:
        raise PAError(PA_ERR_INVALID_ARG, "pa_allocator_create")
    return h


def pa_allocator_destroy(handle) -> None:
    _lib.pa_allocator_destroy(handle)


def pa_num_required_blocks(num_tokens: int, block_size: int) -> int:
    return _lib.pa_num_required_blocks(num_tokens, block_size)


def pa_alloc(handle) -> int:
    out = ctypes.c_int32()
    _check(_lib.pa_alloc(handle, ctypes.byref(out)), "pa_alloc")
    return out.value


def pa_alloc_n(handle, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    _check(_lib.pa_alloc_n(handle, n, out.ctypes.data_as(_i32p)), "pa_alloc_n")
    return out


def pa_free(handle, block_id: int) -> None:
    _check(_lib.pa_free(handle, int(block_id)), "pa_free")


def pa_free_n(handle, ids) -> None:
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    _check(_lib.pa_free_n(handle, ids.size, ids.ctypes.data_as(_i32p)), "pa_free_n")


def pa_add_ref(handle, block_id: int) -> None:
    _check(_lib.pa_add_ref(handle, int(block_id)), "pa_add_ref")


def pa_fork(handle, src) -> np.ndarray:
    src = np.ascontiguousarray(src, dtype=np.int32)
    dst = np.empty_like(src)
    _check(_lib.pa_fork(handle, src.ctypes.data_as(_i32p), src.size, dst.ctypes.data_as(_i32p)), "pa_fork")
    return dst


def pa_refcount(handle, block_id: int) -> int:
    return _lib.pa_refcount(handle, int(block_id))


def pa_num_free(handle) -> int:
    return _lib.pa_num_free(handle)


def pa_num_blocks(handle) -> int:
    return _lib.pa_num_blocks(handle)


def pa_usage(handle) -> float:
    return _lib.pa_usage(handle)


def pa_append_slots(handle, block_tables: np.ndarray, context_lens: np.ndarray, block_size: int) -> np.ndarray:
    """In place on block_tables (int32 [S, MB]) and context_lens (int32 [S]); returns slot_mapping int64 [S]."""
    tables = _np_i32(block_tables, "block_tables")
    lens = _np_i32(context_lens, "context_lens")
    s, mb = tables.shape
    slots = np.empty(s, dtype=np.int64)
    _check(_lib.pa_append_slots(handle, tables.ctypes.data_as(_i32p), mb, lens.ctypes.data_as(_i32p), s,
                                block_size, slots.ctypes.data_as(_i64p)), "pa_append_slots")
    return slots


def pa_prefill_slots(handle, block_tables: np.ndarray, context_lens: np.ndarray, new_tokens,
                     block_size: int) -> np.ndarray:
    """In place on block_tables and context_lens (int32); returns the new tokens' slots, int64 [sum(new)]."""
    tables = _np_i32(block_tables, "block_tables")
    lens = _np_i32(context_lens, "context_lens")
    new = np.ascontiguousarray(new_tokens, dtype=np.int32)
    s, mb = tables.shape
    slots = np.empty(max(int(new.sum()), 1), dtype=np.int64)
    _check(_lib.pa_prefill_slots(handle, tables.ctypes.data_as(_i32p), mb, lens.ctypes.data_as(_i32p),
                                 new.ctypes.data_as(_i32p), s, block_size, slots.ctypes.data_as(_i64p)),
           "pa_prefill_slots")
    return slots[:int(new.sum())]


def pa_cow_prepare(handle, block_tables: np.ndarray, context_lens: np.ndarray, block_size: int) -> np.ndarray:
    """In place on block_tables (int32 [S, MB]); returns the (src, dst) copy pairs, int32 [k, 2]."""
    tables = _np_i32(block_tables, "block_tables")
    lens = _np_i32(np.ascontiguousarray(context_lens, dtype=np.int32), "context_lens")
    s, mb = tables.shape
    pairs = np.empty(2 * max(s, 1), dtype=np.int32)
    k = ctypes.c_int(0)
    _check(_lib.pa_cow_prepare(handle, tables.ctypes.data_as(_i32p), mb, lens.ctypes.data_as(_i32p), s, block_size,
                               pairs.ctypes.data_as(_i32p), ctypes.byref(k)), "pa_cow_prepare")
    return pairs[:2 * k.value].reshape(-1, 2).copy()


def pa_copy_blocks(k_cache, v_cache, copy_pairs, err_word=None, stream=None) -> None:
    """Device block copies; copy_pairs: int32 CUDA tensor [n, 2] of (src, dst)."""
    import torch
    nb, bs, hk, d = k_cache.shape
    if v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype:
        raise ValueError("k_cache and v_cache must match")
    if copy_pairs.dim() != 2 or copy_pairs.shape[1] != 2:
        raise ValueError("copy_pairs must be [n, 2]")
    st = _lib.pa_copy_blocks(_dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                             _dev(copy_pairs, "copy_pairs", torch.int32), copy_pairs.shape[0], hk, d, bs, nb,
                             k_cache.element_size(), _dev(err_word, "err_word", torch.int32), _stream(stream, k_cache))
    _check(st, "pa_copy_blocks")


def pa_swap_plan(from_handle, to_handle, table_row: np.ndarray, num_blocks: int) -> np.ndarray:
    """Move num_blocks ids of table_row (int32, in place) from one pool to another;
    returns the (old, new) pairs, int32 [num_blocks, 2]."""
    row = _np_i32(table_row, "table_row")
    pairs = np.empty(2 * max(num_blocks, 1), dtype=np.int32)
    _check(_lib.pa_swap_plan(from_handle, to_handle, row.ctypes.data_as(_i32p), num_blocks,
                             pairs.ctypes.data_as(_i32p)), "pa_swap_plan")
    return pairs[:2 * num_blocks].reshape(-1, 2).copy()


def pa_swap_blocks(src_k, src_v, dst_k, dst_v, pairs, err_word=None, stream=None) -> None:
    """Copy blocks between two pools (torch tensors [NB, B, Hk, d]; either may be pinned
    host memory); pairs: int32 tensor [n, 2] of (src, dst) in device-readable memory."""
    import torch
    snb, bs, hk, d = src_k.shape
    dnb = dst_k.shape[0]
    if dst_k.shape[1:] != src_k.shape[1:] or src_v.shape != src_k.shape or dst_v.shape != dst_k.shape:
        raise ValueError("pools must share block geometry")
    if src_k.dtype != dst_k.dtype:
        raise TypeError("pools must share one dtype")
    for name, t in (("src_k", src_k), ("src_v", src_v), ("dst_k", dst_k), ("dst_v", dst_v), ("pairs", pairs)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if not t.is_cuda and not t.is_pinned():
            raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")
    if pairs.dtype != torch.int32 or pairs.dim() != 2 or pairs.shape[1] != 2:
        raise ValueError("pairs must be int32 [n, 2]")
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    st = _lib.pa_swap_blocks(ptr(src_k), ptr(src_v), snb, ptr(dst_k), ptr(dst_v), dnb, ptr(pairs), pairs.shape[0],
                             hk, d, bs, src_k.element_size(), _dev(err_word, "err_word", torch.int32),
                             _stream(stream, src_k if src_k.is_cuda else dst_k))
    _check(st, "pa_swap_blocks")


class BlockAllocator:
    """Owning wrapper over a pa_allocator handle."""

    def __init__(self, num_blocks: int, initial_order=None):
        # the C function is held here: at interpreter exit the module's globals
        # may already be gone when __del__ runs
        self._destroy = _lib.pa_allocator_destroy
        self.handle = pa_allocator_create(num_blocks, initial_order)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h:
            self._destroy(h)
            self.handle = None

    def alloc(self) -> int:
        return pa_alloc(self.handle)

    def alloc_n(self, n: int) -> np.ndarray:
        return pa_alloc_n(self.handle, n)

    def free(self, block_id: int) -> None:
        pa_free(self.handle, block_id)

    def free_n(self, ids) -> None:
        pa_free_n(self.handle, ids)

    def add_ref(self, block_id: int) -> None:
        pa_add_ref(self.handle, block_id)

    def fork(self, src) -> np.ndarray:
        return pa_fork(self.handle, src)

    def refcount(self, block_id: int) -> int:
        return pa_refcount(self.handle, block_id)

    def num_free(self) -> int:
        return pa_num_free(self.handle)

    def num_blocks(self) -> int:
        return pa_num_blocks(self.handle)

    def usage(self) -> float:
        return pa_usage(self.handle)

    def append_slots(self, block_tables: np.ndarray, context_lens: np.ndarray, block_size: int) -> np.ndarray:
        return pa_append_slots(self.handle, block_tables, context_lens, block_size)

    def prefill_slots(self, block_tables: np.ndarray, context_lens: np.ndarray, new_tokens, block_size: int):
        return pa_prefill_slots(self.handle, block_tables, context_lens, new_tokens, block_size)

    def cow_prepare(self, block_tables: np.ndarray, context_lens: np.ndarray, block_size: int) -> np.ndarray:
        return pa_cow_prepare(self.handle, block_tables, context_lens, block_size)
