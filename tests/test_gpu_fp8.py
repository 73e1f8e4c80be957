"""fp8 (E4M3) KV cache on the GPU against the oracle.

The cache write must produce the oracle's codes bit for bit (both sides divide in
fp32 and round to nearest even with saturation).  Decode works on exactly
dequantised values in fp32, so it is held to the same tolerance as the 16-bit
path, against the oracle's fp64 decode over the same codes.  Padding rows hold the
NaN code, so reading one would show in the output.
"""
import math

import numpy as np
import pytest
import torch

from gpu_cases import Step, assert_close, bits
from pins import BF16, F16, PagedCase, from_bits, to_bits
import oracle as oracle_pkg
from paged_kv_cache_374_b200 import binding as pa

pytestmark = pytest.mark.gpu

TDT = {F16: torch.float16, BF16: torch.bfloat16}
WK = {F16: "f16", BF16: "bf16"}


def to_codes(x64: np.ndarray, scale: float) -> np.ndarray:
    """E4M3 codes of x / scale (NaN stays NaN), as uint8 -- input preparation only."""
    t = torch.from_numpy((x64 / scale).astype(np.float32)).clamp(-448, 448)
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()


def test_cache_write_codes_are_bit_exact():
    rng = np.random.default_rng(50)
    nb, bs, hk, d, n = 10, 16, 8, 128, 24
    o = oracle_pkg.get()
    for dtype in (F16, BF16):
        # normal values, tiny ones (subnormal codes), values past the saturation point
        vals = np.concatenate([rng.normal(0, 3, n * hk * d // 2), rng.normal(0, 0.01, n * hk * d // 4),
                               rng.normal(0, 400, n * hk * d // 4)])
        k = torch.from_numpy(rng.permutation(vals).reshape(n, hk, d).astype(np.float32)).to(TDT[dtype]).cuda()
        v = torch.from_numpy(rng.permutation(vals).reshape(n, hk, d).astype(np.float32)).to(TDT[dtype]).cuda()
        kc = torch.zeros(nb, bs, hk, d, dtype=torch.uint8, device="cuda")
        vc = torch.zeros_like(kc)
        slots = rng.choice(nb * bs, size=n, replace=False).astype(np.int64)
        slots[3] = -1
        ks, vs = 0.37, 1.9
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        pa.pa_reshape_and_cache_fp8(k, v, torch.from_numpy(slots).cuda(), kc, vc, ks, vs, err_word=err)
        torch.cuda.synchronize()
        kh = np.zeros((nb, bs, hk, d), dtype=np.uint8)
        vh = np.zeros_like(kh)
        assert o.reshape_and_cache_fp8(bits(k), bits(v), slots, kh, vh, dtype, ks, vs) == 1
        assert err.item() == 0
        assert np.array_equal(kc.cpu().numpy(), kh) and np.array_equal(vc.cpu().numpy(), vh)


# groups 1 (CUDA cores), 2-8 and 16 (tensor cores, one or two head tiles), 32 (CUDA cores again)
SHAPES = [(16, 1, F16), (32, 1, BF16), (64, 1, F16), (16, 8, BF16), (32, 4, F16), (64, 2, BF16), (16, 16, F16),
          (32, 16, BF16), (16, 32, F16)]


@pytest.mark.parametrize("bs,g,dtype", SHAPES)
def test_decode_fp8_matches_oracle(bs, g, dtype):
    rng = np.random.default_rng(51 + bs + g)
    hk, d = 2, 128
    lens = [0, 1, bs - 1, bs + 1, 256, 257, 700, 1500]
    c = PagedCase(rng, lens, hk * g, hk, d, bs, dtype, 1 / math.sqrt(d), extra_blocks=4)
    ks, vs = 0.08, 0.05
    k8 = to_codes(from_bits(c.k_cache, dtype), ks)   # NaN padding rows become the NaN code
    v8 = to_codes(from_bits(c.v_cache, dtype), vs)
    assert ((k8 & 0x7f) == 0x7f).any()
    ref = oracle_pkg.get().decode_fp8(c.q, k8, v8, c.tables, c.lens, c.scale, ks, vs, dtype, nthreads=8)
    q = torch.from_numpy(c.q.view(np.int16)).view(TDT[dtype]).cuda()
    tb, ln = torch.from_numpy(c.tables).cuda(), torch.from_numpy(c.lens).cuda()
    for pt in (0, 64, 320, 512):
        out = torch.empty_like(q)
        pa.pa_decode_fp8(q, torch.from_numpy(k8).cuda(), torch.from_numpy(v8).cuda(), tb, ln, c.scale, ks, vs, hk,
                         out, partition_tokens=pt)
        torch.cuda.synchronize()
        assert_close(out, ref, WK[dtype], f"fp8 bs{bs} g{g} pt{pt}")
        assert torch.count_nonzero(out[0]) == 0


def test_llama7b_fp8_full_size():
    """The 7B workload with its cache stored as fp8: one step of K1 (quantising) and
    K2 + K3, compared with the oracle on a sample of (sequence, head) pairs."""
    step = Step("llama7b")
    t = step.tensors()
    ks, vs = 1 / 32, 1 / 32
    k8 = (t["k_cache"].float() / ks).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    v8 = (t["v_cache"].float() / vs).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    kh, vh = k8.cpu().numpy(), v8.cpu().numpy()
    slots = torch.from_numpy(step.slots).cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_reshape_and_cache_fp8(t["k"], t["v"], slots, k8, v8, ks, vs, err_word=err)
    out = torch.empty_like(t["q"])
    pa.pa_decode_fp8(t["q"], k8, v8, torch.from_numpy(step.tables).cuda(), torch.from_numpy(step.lens).cuda(),
                     step.spec.scale, ks, vs, step.spec.num_kv_heads, out, err_word=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    o = oracle_pkg.get()
    o.reshape_and_cache_fp8(bits(t["k"]), bits(t["v"]), step.slots, kh, vh, F16, ks, vs)
    assert np.array_equal(k8.cpu().numpy(), kh) and np.array_equal(v8.cpu().numpy(), vh)
    rng = np.random.default_rng(52)
    pairs = np.array([(int(np.argmax(step.lens)), 0), (int(np.argmin(step.lens)), 31)]
                     + [(int(rng.integers(0, 64)), int(rng.integers(0, 32))) for _ in range(62)], dtype=np.int32)
    ref = o.decode_fp8(bits(t["q"]), kh, vh, step.tables, step.lens, step.spec.scale, ks, vs, F16, pairs=pairs,
                       nthreads=8)
    got = out[torch.from_numpy(pairs[:, 0]).long(), torch.from_numpy(pairs[:, 1]).long()]
    assert_close(got, ref, "f16", "llama7b fp8")


@pytest.mark.parametrize("g", [1, 8])
@pytest.mark.parametrize("exp2", [40, -40])
def test_decode_fp8_bf16_q_outside_f16_range(g, exp2):
    """bf16 q enters the f16 arithmetic of both fp8 policies as q * 2^k, k chosen per
    unit: q scaled by 2^40 (past f16's largest finite value) or 2^-40 (below its
    smallest subnormal), with the softmax scale compensating so that the scores stay
    in the usual range, must give the oracle's result.  One head also holds elements
    about 2^30 below its largest: the unit's scale keeps them (the few under 2^-31 of
    the largest round to f16's subnormal grid, a negligible change of the score)."""
    rng = np.random.default_rng(53 + g + exp2)
    hk, d, bs = 2, 128, 16
    lens = [1, 17, 300, 777]
    c = PagedCase(rng, lens, hk * g, hk, d, bs, BF16, 1 / math.sqrt(d), extra_blocks=2)
    q64 = from_bits(c.q, BF16) * 2.0 ** exp2
    q64[1, 0, 64:] *= 2.0 ** -30                      # one head: dims 64.. far below the head's largest
    q_bits = to_bits(q64, BF16)
    assert np.array_equal(from_bits(q_bits, BF16), q64)   # the scaling is exact in bf16
    scale = c.scale * 2.0 ** -exp2
    ks, vs = 0.08, 0.05
    k8 = to_codes(from_bits(c.k_cache, BF16), ks)
    v8 = to_codes(from_bits(c.v_cache, BF16), vs)
    ref = oracle_pkg.get().decode_fp8(q_bits, k8, v8, c.tables, c.lens, scale, ks, vs, BF16, nthreads=8)
    q = torch.from_numpy(q_bits.view(np.int16)).view(torch.bfloat16).cuda()
    out = torch.empty_like(q)
    pa.pa_decode_fp8(q, torch.from_numpy(k8).cuda(), torch.from_numpy(v8).cuda(), torch.from_numpy(c.tables).cuda(),
                     torch.from_numpy(c.lens).cuda(), scale, ks, vs, hk, out)
    torch.cuda.synchronize()
    assert_close(out, ref, "bf16", f"fp8 bf16 q x 2^{exp2} g{g}")
