"""Set-up shared by the GPU parity tests: one decode step of a workload, built
twice -- through the library (C++ allocator, CUDA kernels) and through the oracle
side (Python allocator model, fp64 C oracle) -- from the same seeded inputs.

Tolerances (stated on the decode output against the fp64 oracle):
  fp16: max |err| <= 2e-3 and relative L2 <= 1e-3.
  bf16: max |err| <= 1e-2; relative L2 <= 1e-3 measured against the oracle rounded
        once to bf16.  Rounding the exact result to bf16 alone has a relative L2
        of about 1.5e-3 (half an ulp of 2^-7, uniform), so the 1e-3 bound can only
        apply to the error beyond that unavoidable final rounding.
  The max |err| bounds apply to the computation before that one final rounding:
  element i may differ from the unrounded oracle by the bound plus half an ulp of
  the output type at ref_i.  Rounding alone reaches half an ulp, which is above
  1e-2 in bf16 from |out| = 4 on (and above 2e-3 in fp16 from 8 on), where a
  peaked softmax puts outputs with N(0, 1) values.
  cache writes: bit-exact.
"""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle as oracle_pkg
from oracle.block_pool import BlockPoolModel
from paged_kv_cache_374_b200 import binding as pa
from paged_kv_cache_374_b200 import workloads as wk

NTHREADS = os.cpu_count() or 1
TOL = {wk.F16: (2e-3, 1e-3), wk.BF16: (1e-2, 1e-3)}
DT = {wk.F16: 0, wk.BF16: 1}


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw uint16 patterns of a 16-bit tensor, on the host."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def half_ulp(ref: np.ndarray, dtype: str) -> np.ndarray:
    """Half the spacing of the output type's numbers at |ref| (normal range)."""
    mant = 10 if dtype == wk.F16 else 7
    e = np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -14)))
    return 0.5 * np.exp2(e - mant)


def errors(got: torch.Tensor, ref: np.ndarray, dtype: str):
    """(max |err| beyond half an ulp of the output type, relative L2)."""
    g = got.detach().double().cpu().numpy()
    r_target = ref
    if dtype == wk.BF16:
        r_target = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    max_abs = float(np.max(np.abs(g - ref) - half_ulp(ref, dtype))) if g.size else 0.0
    den = float(np.linalg.norm(r_target))
    rel = float(np.linalg.norm(g - r_target) / den) if den > 0 else float(np.linalg.norm(g - r_target))
    return max_abs, rel


def assert_close(got: torch.Tensor, ref: np.ndarray, dtype: str, what=""):
    assert not torch.isnan(got).any(), f"{what}: NaN in output"
    max_abs, rel = errors(got, ref, dtype)
    tol_abs, tol_rel = TOL[dtype]
    assert max_abs <= tol_abs and rel <= tol_rel, (
        f"{what}: max_abs beyond the final rounding {max_abs:.3g} rel_l2 {rel:.3g}")
    return max_abs, rel


class Step:
    """A workload with its tables built by both allocators and its step-1 slots resolved."""

    def __init__(self, name, device="cuda", num_seqs=None, seed=None):
        self.wl = wl = wk.make_workload(name, seed=seed, num_seqs=num_seqs)
        self.spec = spec = wl.spec
        self.bs = bs = spec.block_size
        self.dtype = spec.dtype
        s = spec.num_seqs
        self.alloc = pa.BlockAllocator(wl.num_blocks, wl.pool_order)
        self.model = BlockPoolModel(wl.num_blocks, wl.pool_order)
        stored = (wl.context_lens - 1).astype(np.int32)   # tokens in the cache before step 1
        mb = wl.max_blocks_per_seq
        self.tables = np.full((s, mb), -1, dtype=np.int32)
        model_tables = [[] for _ in range(s)]
        if spec.prefix_tokens:
            npre = pa.pa_num_required_blocks(spec.prefix_tokens, bs)
            prefix = self.alloc.alloc_n(npre)                 # the prompt owner's blocks
            assert list(prefix) == self.model.allocate_n(npre)
            for i in range(s):
                self.tables[i, :npre] = self.alloc.fork(prefix)   # every beam holds the prefix
                model_tables[i] = self.model.fork(list(prefix))
        for i in range(s):
            have = len(model_tables[i])
            n = pa.pa_num_required_blocks(int(stored[i]), bs) - have
            got = self.alloc.alloc_n(n)
            want = self.model.allocate_n(n)
            assert list(got) == want, "allocator differs from the model"
            self.tables[i, have:have + n] = got
            model_tables[i] += want
        self.model_tables = model_tables
        self.stored = stored
        self.lens = stored.copy()
        self.slots = self.append()                            # a1 for step 1

    def append(self):
        """a1: resolve this step's slots with the library and check them against
        the model and the oracle's slot arithmetic."""
        before = self.lens.copy()
        slots = self.alloc.append_slots(self.tables, self.lens, self.bs)
        for i in range(len(before)):
            if before[i] % self.bs == 0:
                model_tables_i = self.model_tables[i]
                model_tables_i.append(self.model.allocate())
            assert list(self.tables[i, :len(self.model_tables[i])]) == self.model_tables[i]
        want = oracle_pkg.get().slot_mapping(self.tables, self.lens, self.bs)
        assert np.array_equal(slots, want), "slot mapping differs from the oracle"
        return slots

    def tensors(self, device="cuda", seed_offset=0):
        t = wk.make_tensors(self.wl, device=device, seed_offset=seed_offset)
        wk.poison_unused(t["k_cache"], t["v_cache"], self.tables, self.stored, self.bs)
        return t


def device_inputs(step: Step, t, device="cuda"):
    return (torch.from_numpy(step.tables).to(device), torch.from_numpy(step.lens).to(device),
            torch.from_numpy(step.slots).to(device))


def run_library(step: Step, t, partition_tokens=0, err=None):
    tables, lens, slots = device_inputs(step, t)
    pa.pa_reshape_and_cache(t["k"], t["v"], slots, t["k_cache"], t["v_cache"], err_word=err)
    out = torch.empty_like(t["q"])
    pa.pa_decode(t["q"], t["k_cache"], t["v_cache"], tables, lens, step.spec.scale, step.spec.num_kv_heads, out,
                 partition_tokens=partition_tokens, err_word=err)
    return out


def oracle_decode(step: Step, q_bits, kc_bits, vc_bits, pairs=None):
    o = oracle_pkg.get()
    return o.decode(q_bits, kc_bits, vc_bits, step.tables, step.lens, step.spec.scale, DT[step.dtype],
                    pairs=pairs, nthreads=NTHREADS)
