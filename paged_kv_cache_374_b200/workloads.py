"""Seeded synthetic workloads for the paged decode path.

This module serves both the CUDA library's tests/benchmark and the fp64 oracle,
so it holds none of the method's arithmetic: it draws sequence lengths, the
shuffled physical-id order of the block pool, and the q / K / V values, and it can
NaN-fill cache rows that hold no token.  Building block tables and slot mappings
is left to the allocators (the C++ one in the library, the Python model beside the
oracle), which the tests compare id for id.

Shapes follow the decode workloads the paged-attention pages discuss: a 7B
(32 heads, head_dim 128) and a 13B (40 heads) layer, a GQA long-context case, and
prefix sharing across beams.  Lengths count this step's new token.

Randomness: numpy ``Generator(PCG64(seed))`` for the integer structure, a
``torch.Generator`` seeded with the same number for the values (on the device for
the large workloads, so that generating 3 GB of values takes milliseconds).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

F16 = "f16"
BF16 = "bf16"


@dataclasses.dataclass
class WorkloadSpec:
    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    dtype: str                  # "f16" | "bf16"
    scale: float
    value_dist: str             # "uniform" (U[-1, 1]) | "normal" (N(0, 1))
    seed: int
    steps: int = 1              # decode steps, each appending one token per sequence
    headroom: float = 1.2       # pool size over the blocks the workload needs
    prefix_tokens: int = 0      # tokens of one prefix shared by every sequence
    beam_width: int = 1
    description: str = ""


SPECS: dict[str, WorkloadSpec] = {
    "tiny": WorkloadSpec("tiny", 4, 4, 4, 64, 16, F16, 1.0 / 8.0, "uniform", 0, headroom=0.0,
                         description="4 seqs, context_lens {5,17,33,50}, 4 heads MHA, head_dim 64, block_size 16, "
                                     "pool of 16 blocks in seeded random order, fp16 U[-1,1], scale 1/8"),
    "llama7b": WorkloadSpec("llama7b", 64, 32, 32, 128, 16, F16, 1.0 / math.sqrt(128), "normal", 1,
                            description="Llama-2-7B layer: batch 64, 32 heads MHA, head_dim 128, block_size 16, "
                                        "context_lens U[512,4096], fp16 N(0,1), pool +20% shuffled"),
    "llama13b": WorkloadSpec("llama13b", 32, 40, 40, 128, 16, BF16, 1.0 / math.sqrt(128), "normal", 2, steps=32,
                             description="Llama-2-13B layer: batch 32, 40 heads MHA, head_dim 128, block_size 16, "
                                         "initial lengths N(2000,400) clipped [64,4096], bf16 N(0,1), 32 decode "
                                         "steps"),
    "gqa70b": WorkloadSpec("gqa70b", 16, 64, 8, 128, 32, BF16, 1.0 / math.sqrt(128), "normal", 3,
                           description="70B-style GQA: batch 16, 64 q heads / 8 kv heads, head_dim 128, "
                                       "block_size 32, context_lens log-uniform [4096,32768], bf16 N(0,1)"),
    "beam": WorkloadSpec("beam", 128, 32, 32, 128, 64, F16, 1.0 / math.sqrt(128), "normal", 4,
                         prefix_tokens=512, beam_width=4,
                         description="32 prompts x beam 4, one 512-token prefix shared by all, suffixes "
                                     "geometric mean 256 (max 2048), block_size 64, 32 heads MHA, head_dim 128, "
                                     "fp16 N(0,1)"),
}


@dataclasses.dataclass
class Workload:
    spec: WorkloadSpec
    context_lens: np.ndarray     # int32 [S]: lengths after the first step's new token
    num_blocks: int              # physical blocks in the pool
    pool_order: np.ndarray       # int32 [num_blocks]: seeded order of the free queue
    max_blocks_per_seq: int      # table width

    @property
    def num_seqs(self) -> int:
        return self.spec.num_seqs


def _ceil_div(a, b):
    return -(-a // b)


def draw_lengths(spec: WorkloadSpec, rng: np.random.Generator) -> np.ndarray:
    """Context lengths (new token included) for the first decode step."""
    s = spec.num_seqs
    if spec.name == "tiny":
        return np.array([5, 17, 33, 50], dtype=np.int32)
    if spec.name == "llama7b":
        return rng.integers(512, 4096, size=s, endpoint=True).astype(np.int32)
    if spec.name == "llama13b":
        initial = np.clip(np.rint(rng.normal(2000.0, 400.0, size=s)), 64, 4096).astype(np.int32)
        return initial + 1  # the first step appends one token to the initial length
    if spec.name == "gqa70b":
        return np.floor(np.exp(rng.uniform(math.log(4096), math.log(32768), size=s))).astype(np.int32)
    if spec.name == "beam":
        suffix = np.minimum(rng.geometric(1.0 / 256.0, size=s), 2048).astype(np.int32)
        return spec.prefix_tokens + suffix
    raise KeyError(spec.name)


def make_workload(name: str, seed: int | None = None, num_seqs: int | None = None) -> Workload:
    """Host-side structure of a workload: lengths, pool size and pool order.

    ``num_seqs`` truncates the batch (a smaller case with the same distributions).
    """
    spec = dataclasses.replace(SPECS[name])
    if seed is not None:
        spec.seed = seed
    rng = np.random.Generator(np.random.PCG64(spec.seed))
    lens = draw_lengths(spec, rng)
    if num_seqs is not None:
        lens = lens[:num_seqs]
        spec.num_seqs = int(num_seqs)
    bs = spec.block_size
    final = lens.astype(np.int64) + (spec.steps - 1)  # lengths after the last step
    if spec.prefix_tokens:
        # the prefix is held once; every sequence owns blocks for its suffix only
        pref = _ceil_div(spec.prefix_tokens, bs)
        need = pref + int(np.sum(_ceil_div(final, bs) - pref))
    else:
        need = int(np.sum(_ceil_div(final, bs)))
    if name == "tiny":
        num_blocks = 16
    else:
        num_blocks = int(math.ceil(spec.headroom * need))
    mb = int(np.max(_ceil_div(final, bs))) if len(final) else 0
    order = rng.permutation(num_blocks).astype(np.int32)
    return Workload(spec, lens.astype(np.int32), num_blocks, order, mb)


def torch_dtype(dtype: str):
    import torch
    return {F16: torch.float16, BF16: torch.bfloat16}[dtype]


def draw_values(spec: WorkloadSpec, shape, device, generator):
    """Values of the spec's distribution, rounded once to the spec's dtype."""
    import torch
    if spec.value_dist == "uniform":
        x = torch.rand(shape, generator=generator, device=device, dtype=torch.float32) * 2.0 - 1.0
    else:
        x = torch.randn(shape, generator=generator, device=device, dtype=torch.float32)
    return x.to(torch_dtype(spec.dtype))


def make_tensors(wl: Workload, device="cpu", seed_offset: int = 0):
    """q [S,H,d], new k/v [S,Hk,d] and the two caches [NB,B,Hk,d], all random.

    Every cache row starts random; ``poison_unused`` turns the rows that hold no
    token into NaN.
    """
    import torch
    spec = wl.spec
    g = torch.Generator(device=device)
    g.manual_seed(spec.seed * 1000003 + seed_offset)
    s, h, hk, d, bs = spec.num_seqs, spec.num_heads, spec.num_kv_heads, spec.head_dim, spec.block_size
    out = {
        "q": draw_values(spec, (s, h, d), device, g),
        "k": draw_values(spec, (s, hk, d), device, g),
        "v": draw_values(spec, (s, hk, d), device, g),
        "k_cache": draw_values(spec, (wl.num_blocks, bs, hk, d), device, g),
        "v_cache": draw_values(spec, (wl.num_blocks, bs, hk, d), device, g),
    }
    return out


def poison_unused(k_cache, v_cache, block_tables: np.ndarray, stored_lens: np.ndarray, block_size: int):
    """NaN-fill every cache row that holds no stored token.

    ``stored_lens[s]`` tokens of sequence ``s`` are held in the blocks listed in
    ``block_tables[s]`` (in logical order, ``block_size`` tokens per block); rows
    past them in the sequence's last block, and every block no table lists, become
    NaN, so reading any of them shows up in the output.
    """
    import torch
    nb = k_cache.shape[0]
    dev = k_cache.device
    used = np.zeros(nb, dtype=bool)
    rows_keep = np.zeros((nb, block_size), dtype=bool)
    for s in range(block_tables.shape[0]):
        n = int(stored_lens[s])
        full, rem = divmod(n, block_size)
        ids = block_tables[s, :_ceil_div(n, block_size)]
        used[ids] = True
        rows_keep[block_tables[s, :full]] = True
        if rem:
            rows_keep[block_tables[s, full], :rem] = True
    mask = torch.from_numpy(~rows_keep).to(dev)
    nan = float("nan")
    k_cache[mask] = nan
    v_cache[mask] = nan
    return used
