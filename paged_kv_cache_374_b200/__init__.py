"""B200 paged decode attention: a C-ABI CUDA library (libpa.so) and its binding.

    from paged_kv_cache_374_b200 import binding as pa
    pa.pa_reshape_and_cache(k, v, slot_mapping, k_cache, v_cache)
    pa.pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, out)

The binding is imported lazily, so ``paged_kv_cache_374_b200.workloads`` (the
seeded input generator) can be used without the CUDA library; any use of the
binding's names loads ``libpa.so`` and fails loudly if it is missing.
"""
import importlib

__all__ = ["binding", "workloads", "build"]


def __getattr__(name):
    if name in ("binding", "workloads", "build"):
        return importlib.import_module(f"{__name__}.{name}")
    binding = importlib.import_module(f"{__name__}.binding")
    try:
        return getattr(binding, name)
    except AttributeError:
        raise AttributeError(f"module {__name__!r} has no attribute {name!r}") from None
