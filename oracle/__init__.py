"""fp64 CPU oracle for the paged decode path -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
import this package.  It shares no code with the CUDA library and never imports
it.  The arithmetic lives in ``pa_oracle.c`` (plain C, double precision); this
module is argument marshalling over numpy arrays of raw 16-bit patterns.

Pages cited: P1 "大模型部署中的PagedAttention：KV Cache显存管理突破"; P2 "大模型推理优化：KV
Cache与PagedAttention技术详解"; P3 "LLM 推理中的 PageAttention 实现原理：虚拟内存管理在 KV
Cache 中的创新应用".

Functions and what they follow:
  decode               softmax(q K^T * scale) V, one softmax over all tokens (P1 §1)
  reshape_and_cache    new K/V rows copied into their slots, bit for bit (P2 §2.1)
  copy_blocks          whole-block copies for copy-on-write after a fork (P3 §四)
  reshape_and_cache_fp8 / decode_fp8 / e4m3_*   the fp8 (E4M3) cache variant
  prefill              causal attention of a chunk of new query tokens over the paged
                       cache (the step before decode, P2 §2.1 steps 1-2)
  slot_mapping         slot of the newest token through the table (P3 §三)
  physical_location    token -> (table[idx // B], idx % B)  (P3 §三)
  num_required_blocks  ceil(n / B)  (P3 §三)
  kv_bytes             2 * seq * layers * heads * head_dim * dtype_size  (P2 §2.2)
  half_to_double / bf16_to_double   exact widening of the 16-bit formats
The host block allocator's oracle is the pure-Python model in ``block_pool.py``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

F16 = 0
BF16 = 1

_c_i32p = ctypes.POINTER(ctypes.c_int32)
_c_i64p = ctypes.POINTER(ctypes.c_int64)
_c_u16p = ctypes.POINTER(ctypes.c_uint16)
_c_u8p = ctypes.POINTER(ctypes.c_uint8)
_c_f64p = ctypes.POINTER(ctypes.c_double)


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(ctype)


class Oracle:
    """One loaded copy of the C oracle (the default build or a planted mutant)."""

    def __init__(self, path: str):
        self.path = path
        lib = ctypes.CDLL(path)
        lib.pa_oracle_half_to_double.restype = ctypes.c_double
        lib.pa_oracle_half_to_double.argtypes = [ctypes.c_uint16]
        lib.pa_oracle_bf16_to_double.restype = ctypes.c_double
        lib.pa_oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.pa_oracle_num_required_blocks.restype = ctypes.c_int64
        lib.pa_oracle_num_required_blocks.argtypes = [ctypes.c_int64, ctypes.c_int64]
        lib.pa_oracle_physical_location.restype = ctypes.c_int
        lib.pa_oracle_physical_location.argtypes = [_c_i32p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                                    _c_i64p, _c_i64p]
        lib.pa_oracle_kv_bytes.restype = ctypes.c_int64
        lib.pa_oracle_kv_bytes.argtypes = [ctypes.c_int64] * 5
        lib.pa_oracle_slot_mapping.restype = ctypes.c_int
        lib.pa_oracle_slot_mapping.argtypes = [_c_i32p, ctypes.c_int, _c_i32p, ctypes.c_int, ctypes.c_int, _c_i64p]
        lib.pa_oracle_reshape_and_cache.restype = ctypes.c_int
        lib.pa_oracle_reshape_and_cache.argtypes = [_c_u16p, _c_u16p, _c_i64p, _c_u16p, _c_u16p] + [ctypes.c_int] * 5
        lib.pa_oracle_decode.restype = ctypes.c_int
        lib.pa_oracle_decode.argtypes = ([_c_u16p, _c_u16p, _c_u16p, _c_i32p, _c_i32p, ctypes.c_double]
                                         + [ctypes.c_int] * 8 + [_c_i32p, ctypes.c_int, _c_f64p, ctypes.c_int])
        lib.pa_oracle_copy_blocks.restype = ctypes.c_int
        lib.pa_oracle_copy_blocks.argtypes = [_c_u16p, _c_u16p, _c_i32p] + [ctypes.c_int] * 5
        lib.pa_oracle_e4m3_to_double.restype = ctypes.c_double
        lib.pa_oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
        lib.pa_oracle_e4m3_from_float.restype = ctypes.c_uint8
        lib.pa_oracle_e4m3_from_float.argtypes = [ctypes.c_float]
        lib.pa_oracle_reshape_and_cache_fp8.restype = ctypes.c_int
        lib.pa_oracle_reshape_and_cache_fp8.argtypes = ([_c_u16p, _c_u16p, _c_i64p, _c_u8p, _c_u8p]
                                                        + [ctypes.c_int] * 6 + [ctypes.c_float] * 2)
        lib.pa_oracle_decode_fp8.restype = ctypes.c_int
        lib.pa_oracle_decode_fp8.argtypes = ([_c_u16p, _c_u8p, _c_u8p, _c_i32p, _c_i32p] + [ctypes.c_double] * 3
                                             + [ctypes.c_int] * 8 + [_c_i32p, ctypes.c_int, _c_f64p, ctypes.c_int])
        lib.pa_oracle_prefill.restype = ctypes.c_int
        lib.pa_oracle_prefill.argtypes = ([_c_u16p, _c_u16p, _c_u16p, _c_i32p, _c_i32p, _c_i32p, ctypes.c_double]
                                          + [ctypes.c_int] * 8 + [_c_f64p, ctypes.c_int])
        lib.pa_oracle_mutant_id.restype = ctypes.c_int
        lib.pa_oracle_mutant_id.argtypes = []
        self._lib = lib
        self.mutant = lib.pa_oracle_mutant_id()

    # -- formats -------------------------------------------------------------
    def half_to_double(self, bits: int) -> float:
        return self._lib.pa_oracle_half_to_double(int(bits))

    def bf16_to_double(self, bits: int) -> float:
        return self._lib.pa_oracle_bf16_to_double(int(bits))

    def e4m3_to_double(self, code: int) -> float:
        return self._lib.pa_oracle_e4m3_to_double(int(code))

    def e4m3_from_float(self, x: float) -> int:
        return self._lib.pa_oracle_e4m3_from_float(float(x))

    # -- slot arithmetic -----------------------------------------------------
    def num_required_blocks(self, num_tokens: int, block_size: int) -> int:
        return self._lib.pa_oracle_num_required_blocks(num_tokens, block_size)

    def physical_location(self, table, token_idx: int, block_size: int):
        """(phys, offset), or None when the table has no entry (P3 §三)."""
        t = np.ascontiguousarray(np.asarray(table, dtype=np.int32).reshape(-1))
        phys = ctypes.c_int64()
        off = ctypes.c_int64()
        rc = self._lib.pa_oracle_physical_location(_ptr(t, _c_i32p), t.size, token_idx, block_size,
                                                   ctypes.byref(phys), ctypes.byref(off))
        return None if rc != 0 else (phys.value, off.value)

    def kv_bytes(self, seq_len, num_layers, num_heads, head_dim, dtype_size) -> int:
        return self._lib.pa_oracle_kv_bytes(seq_len, num_layers, num_heads, head_dim, dtype_size)

    def slot_mapping(self, block_tables: np.ndarray, context_lens: np.ndarray, block_size: int) -> np.ndarray:
        tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        num_seqs, mb = tables.shape
        slots = np.empty(num_seqs, dtype=np.int64)
        rc = self._lib.pa_oracle_slot_mapping(_ptr(tables, _c_i32p), mb, _ptr(lens, _c_i32p), num_seqs,
                                              block_size, _ptr(slots, _c_i64p))
        if rc != 0:
            raise ValueError("slot_mapping: a table has no entry for the newest token")
        return slots

    # -- K1 ------------------------------------------------------------------
    def reshape_and_cache(self, k: np.ndarray, v: np.ndarray, slot_mapping: np.ndarray,
                          k_cache: np.ndarray, v_cache: np.ndarray) -> int:
        """In place on k_cache / v_cache (uint16 [NB, B, Hk, d]); returns skipped count."""
        for a in (k, v, k_cache, v_cache):
            assert a.dtype == np.uint16 and a.flags.c_contiguous
        num_tokens, hk, d = k.shape
        nb, bs = k_cache.shape[:2]
        slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        return self._lib.pa_oracle_reshape_and_cache(_ptr(k, _c_u16p), _ptr(v, _c_u16p), _ptr(slots, _c_i64p),
                                                     _ptr(k_cache, _c_u16p), _ptr(v_cache, _c_u16p),
                                                     num_tokens, hk, d, bs, nb)

    def copy_blocks(self, k_cache: np.ndarray, v_cache: np.ndarray, pairs) -> int:
        """In place: block dst of both caches := block src, for each (src, dst)."""
        for a in (k_cache, v_cache):
            assert a.dtype == np.uint16 and a.flags.c_contiguous
        nb, bs, hk, d = k_cache.shape
        pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
        return self._lib.pa_oracle_copy_blocks(_ptr(k_cache, _c_u16p), _ptr(v_cache, _c_u16p), _ptr(pr, _c_i32p),
                                               pr.shape[0], nb, bs, hk, d)

    def reshape_and_cache_fp8(self, k: np.ndarray, v: np.ndarray, slot_mapping: np.ndarray, k_cache: np.ndarray,
                              v_cache: np.ndarray, dtype: int, k_scale: float, v_scale: float) -> int:
        """Quantising cache write into uint8 E4M3 caches [NB, B, Hk, d]; returns skipped count."""
        for a in (k, v):
            assert a.dtype == np.uint16 and a.flags.c_contiguous
        for a in (k_cache, v_cache):
            assert a.dtype == np.uint8 and a.flags.c_contiguous
        num_tokens, hk, d = k.shape
        nb, bs = k_cache.shape[:2]
        slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
        return self._lib.pa_oracle_reshape_and_cache_fp8(_ptr(k, _c_u16p), _ptr(v, _c_u16p), _ptr(slots, _c_i64p),
                                                         _ptr(k_cache, _c_u8p), _ptr(v_cache, _c_u8p), num_tokens,
                                                         hk, d, bs, nb, dtype, float(k_scale), float(v_scale))

    def prefill(self, q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, block_tables: np.ndarray,
                context_lens: np.ndarray, query_start: np.ndarray, scale: float, dtype: int,
                nthreads: int = 1) -> np.ndarray:
        """fp64 causal prefill.  q uint16 [T, H, d] packed by sequence (query_start [S+1]);
        query row i of sequence s sits at position context_lens[s] - n_s + i.  Returns [T, H, d]."""
        for a in (q, k_cache, v_cache):
            assert a.dtype == np.uint16 and a.flags.c_contiguous
        total, num_heads, d = q.shape
        nb, bs, hk, d2 = k_cache.shape
        assert d2 == d and v_cache.shape == k_cache.shape
        tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        qs = np.ascontiguousarray(query_start, dtype=np.int32)
        num_seqs, mb = tables.shape
        assert qs.shape == (num_seqs + 1,) and qs[-1] == total
        out = np.zeros((total, num_heads, d), dtype=np.float64)
        rc = self._lib.pa_oracle_prefill(_ptr(q, _c_u16p), _ptr(k_cache, _c_u16p), _ptr(v_cache, _c_u16p),
                                         _ptr(tables, _c_i32p), _ptr(lens, _c_i32p), _ptr(qs, _c_i32p), float(scale),
                                         num_seqs, num_heads, hk, d, bs, nb, mb, dtype, _ptr(out, _c_f64p),
                                         int(nthreads))
        if rc != 0:
            raise ValueError(f"oracle prefill rejected its input (code {rc})")
        return out

    def decode_fp8(self, q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, block_tables: np.ndarray,
                   context_lens: np.ndarray, scale: float, k_scale: float, v_scale: float, dtype: int, pairs=None,
                   nthreads: int = 1) -> np.ndarray:
        """fp64 decode over uint8 E4M3 caches (K = code * k_scale, V = code * v_scale)."""
        assert q.dtype == np.uint16 and q.flags.c_contiguous
        for a in (k_cache, v_cache):
            assert a.dtype == np.uint8 and a.flags.c_contiguous
        num_seqs, num_heads, d = q.shape
        nb, bs, hk, d2 = k_cache.shape
        assert d2 == d and v_cache.shape == k_cache.shape
        tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        mb = tables.shape[1] if tables.ndim == 2 else 0
        if pairs is None:
            out = np.zeros((num_seqs, num_heads, d), dtype=np.float64)
            pp, npairs = None, 0
        else:
            pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
            npairs = pr.shape[0]
            out = np.zeros((npairs, d), dtype=np.float64)
            pp = _ptr(pr, _c_i32p)
        rc = self._lib.pa_oracle_decode_fp8(_ptr(q, _c_u16p), _ptr(k_cache, _c_u8p), _ptr(v_cache, _c_u8p),
                                            _ptr(tables, _c_i32p), _ptr(lens, _c_i32p), float(scale), float(k_scale),
                                            float(v_scale), num_seqs, num_heads, hk, d, bs, nb, mb, dtype, pp,
                                            npairs, _ptr(out, _c_f64p), int(nthreads))
        if rc != 0:
            raise ValueError(f"oracle decode_fp8 rejected its input (code {rc})")
        return out

    # -- K2 + K3 -------------------------------------------------------------
    def decode(self, q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, block_tables: np.ndarray,
               context_lens: np.ndarray, scale: float, dtype: int, pairs=None, nthreads: int = 1) -> np.ndarray:
        """fp64 decode attention.  q uint16 [S, H, d]; caches uint16 [NB, B, Hk, d].

        Returns [S, H, d] float64, or [len(pairs), d] when ``pairs`` lists (s, h).
        """
        for a in (q, k_cache, v_cache):
            assert a.dtype == np.uint16 and a.flags.c_contiguous
        num_seqs, num_heads, d = q.shape
        nb, bs, hk, d2 = k_cache.shape
        assert d2 == d and v_cache.shape == k_cache.shape
        tables = np.ascontiguousarray(block_tables, dtype=np.int32)
        lens = np.ascontiguousarray(context_lens, dtype=np.int32)
        mb = tables.shape[1] if tables.ndim == 2 else 0
        if pairs is None:
            out = np.zeros((num_seqs, num_heads, d), dtype=np.float64)
            pp, npairs = None, 0
        else:
            pr = np.ascontiguousarray(np.asarray(pairs, dtype=np.int32).reshape(-1, 2))
            npairs = pr.shape[0]
            out = np.zeros((npairs, d), dtype=np.float64)
            pp = _ptr(pr, _c_i32p)
        rc = self._lib.pa_oracle_decode(_ptr(q, _c_u16p), _ptr(k_cache, _c_u16p), _ptr(v_cache, _c_u16p),
                                        _ptr(tables, _c_i32p), _ptr(lens, _c_i32p), float(scale), num_seqs,
                                        num_heads, hk, d, bs, nb, mb, dtype, pp, npairs, _ptr(out, _c_f64p),
                                        int(nthreads))
        if rc != 0:
            raise ValueError(f"oracle decode rejected its input (code {rc})")
        return out


_default: Oracle | None = None


def get() -> Oracle:
    """The default oracle, compiled on first use if needed."""
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def load_mutant(mutant: int, out_dir: str) -> Oracle:
    return Oracle(_build.build_mutant(mutant, out_dir))


def __getattr__(name):  # module-level convenience: oracle.decode(...) etc.
    if name.startswith("_"):
        raise AttributeError(name)
    return getattr(get(), name)
