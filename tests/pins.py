"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix.

Each ``pin_*`` takes a loaded oracle (the default build or a planted mutant) and
raises AssertionError when the oracle disagrees with
  - a worked example printed on the pages (tests/golden/*.json),
  - a library routine the operation reduces to (numpy's float16 widening, torch's
    bfloat16 widening, torch's scaled_dot_product_attention on a contiguous
    cache, in float64),
  - a closed form (one token, equal scores, two tokens, a dominant token),
  - brute force on tiny inputs, or an invariant (relabelled physical blocks,
    shared prefixes).
Paged inputs here are built the other way round from the oracle: each sequence's
K/V is drawn contiguously first and then copied block by block into the pool, so
a mistake in the oracle's token -> slot arithmetic cannot cancel out.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
F16, BF16 = 0, 1


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def to_bits(x: np.ndarray, dtype: int) -> np.ndarray:
    """Round float values to fp16/bf16 and return the raw uint16 patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    t = t.to(torch.float16 if dtype == F16 else torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def from_bits(bits: np.ndarray, dtype: int) -> np.ndarray:
    """Widen raw fp16/bf16 patterns to float64 with torch (a library routine)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    t = t.view(torch.float16 if dtype == F16 else torch.bfloat16)
    return t.to(torch.float64).numpy()


class PagedCase:
    """A random paged decode problem, assembled block by block.

    seq_k[s] / seq_v[s]: [L_s, Hk, d] uint16, the sequence's K/V in logical order.
    The pool gets each sequence's j-th chunk of ``bs`` tokens copied whole into
    physical block ``tables[s][j]``; rows no sequence uses hold NaN.
    """

    def __init__(self, rng, lens, num_heads, num_kv_heads, head_dim, block_size, dtype, scale,
                 extra_blocks=3, dist="normal"):
        self.lens = np.asarray(lens, dtype=np.int32)
        self.S, self.H, self.Hk, self.d, self.bs = len(lens), num_heads, num_kv_heads, head_dim, block_size
        self.dtype, self.scale = dtype, scale
        nblk = [(-(-int(n) // block_size)) for n in lens]
        self.NB = sum(nblk) + extra_blocks
        self.MB = max(max(nblk), 1)
        ids = rng.permutation(self.NB).astype(np.int32)
        self.tables = np.full((self.S, self.MB), -7, dtype=np.int32)  # padding is never read
        pos = 0
        for s, n in enumerate(nblk):
            self.tables[s, :n] = ids[pos:pos + n]
            pos += n
        draw = (lambda shape: rng.uniform(-1, 1, shape)) if dist == "uniform" else (lambda shape: rng.normal(0, 1, shape))
        self.q = to_bits(draw((self.S, self.H, self.d)), dtype)
        self.seq_k = [to_bits(draw((int(n), self.Hk, self.d)), dtype) for n in lens]
        self.seq_v = [to_bits(draw((int(n), self.Hk, self.d)), dtype) for n in lens]
        self._assemble()

    def _assemble(self):
        nan = to_bits(np.full(1, np.nan), self.dtype)[0]
        shape = (self.NB, self.bs, self.Hk, self.d)
        self.k_cache = np.full(shape, nan, dtype=np.uint16)
        self.v_cache = np.full(shape, nan, dtype=np.uint16)
        for s in range(self.S):
            n = int(self.lens[s])
            for j in range(-(-n // self.bs)):
                chunk = slice(j * self.bs, min(n, (j + 1) * self.bs))
                rows = chunk.stop - chunk.start
                self.k_cache[self.tables[s, j], :rows] = self.seq_k[s][chunk]
                self.v_cache[self.tables[s, j], :rows] = self.seq_v[s][chunk]

    def relabel(self, perm: np.ndarray):
        """Move physical block b to perm[b] (data and tables alike)."""
        self.tables = np.where(self.tables >= 0, perm[np.clip(self.tables, 0, None)], self.tables).astype(np.int32)
        self._assemble()

    def run(self, oracle, **kw):
        return oracle.decode(self.q, self.k_cache, self.v_cache, self.tables, self.lens, self.scale,
                             self.dtype, **kw)

    def sdpa(self):
        """torch scaled_dot_product_attention, float64, on the contiguous K/V."""
        out = np.zeros((self.S, self.H, self.d))
        for s in range(self.S):
            n = int(self.lens[s])
            if n == 0:
                continue
            q = torch.from_numpy(from_bits(self.q[s], self.dtype))[None, :, None, :]          # [1,H,1,d]
            k = torch.from_numpy(from_bits(self.seq_k[s], self.dtype)).permute(1, 0, 2)[None]  # [1,Hk,L,d]
            v = torch.from_numpy(from_bits(self.seq_v[s], self.dtype)).permute(1, 0, 2)[None]
            o = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=self.scale,
                                                                 enable_gqa=self.H != self.Hk)
            out[s] = o[0, :, 0, :].numpy()
        return out


# ---------------------------------------------------------------- formats

def pin_half_widening(o):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([o.half_to_double(int(b)) for b in bits])
    assert np.array_equal(np.isnan(got), np.isnan(ref)), "fp16 NaN patterns differ"
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m]), "fp16 widening differs from numpy"


def pin_bf16_widening(o):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = from_bits(bits, BF16)
    got = np.array([o.bf16_to_double(int(b)) for b in bits])
    assert np.array_equal(np.isnan(got), np.isnan(ref)), "bf16 NaN patterns differ"
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m]), "bf16 widening differs from torch"


# ---------------------------------------------------------- slot arithmetic

def pin_num_required_blocks(o):
    for ex in _golden("pages_worked_examples.json")["num_required_blocks"]:
        assert o.num_required_blocks(ex["tokens"], ex["block_size"]) == ex["blocks"], ex["cite"]
    for bs in (4, 16, 32, 64):
        for n in range(0, 300):
            k = 0
            while k * bs < n:  # brute force: fewest blocks that hold n tokens
                k += 1
            assert o.num_required_blocks(n, bs) == k, (n, bs)


def pin_block_mapping(o):
    ex = _golden("pages_worked_examples.json")["block_mapping"]
    names = {"A": 17, "B": 3, "C": 9}  # arbitrary physical ids for blocks A, B, C
    table = [names["A"], names["B"], names["C"]]
    for lo, hi, blk in ex["ranges"]:
        for i, t in enumerate(range(lo, hi + 1)):
            assert o.physical_location(table, t, ex["block_size"]) == (names[blk], i), (t, ex["cite"])
    assert o.physical_location(table, 12, ex["block_size"]) is None


def pin_kv_bytes(o):
    ex = _golden("pages_worked_examples.json")["kv_bytes"]
    got = o.kv_bytes(ex["seq_len"], ex["num_layers"], ex["num_heads"], ex["head_dim"], ex["dtype_size"])
    assert got == ex["bytes"] == 2 ** 30, ex["cite"]


def pin_slot_mapping(o):
    rng = np.random.default_rng(11)
    for bs in (4, 16, 64):
        lens = rng.integers(0, 5 * bs, size=9).astype(np.int32)
        mb = max(1, int(max(-(-int(n) // bs) for n in lens)))
        tables = rng.permutation(9 * mb).astype(np.int32).reshape(9, mb)
        got = o.slot_mapping(tables, lens, bs)
        for s in range(9):
            # brute force: walk the blocks slot by slot and keep the last token's slot
            last, count = -1, 0
            for phys in tables[s]:
                for off in range(bs):
                    if count < lens[s]:
                        last = int(phys) * bs + off
                        count += 1
            assert got[s] == last, (bs, s, lens[s])


# ---------------------------------------------------------------- cache write

def pin_reshape_and_cache(o):
    rng = np.random.default_rng(12)
    nb, bs, hk, d, n = 6, 16, 3, 64, 10
    kc = rng.integers(0, 65535, size=(nb, bs, hk, d), dtype=np.uint16)
    vc = rng.integers(0, 65535, size=(nb, bs, hk, d), dtype=np.uint16)
    k = rng.integers(0, 65535, size=(n, hk, d), dtype=np.uint16)
    v = rng.integers(0, 65535, size=(n, hk, d), dtype=np.uint16)
    slots = rng.choice(nb * bs, size=n, replace=False).astype(np.int64)
    slots[3] = -1                 # padding token: skipped
    slots[7] = nb * bs + 5        # out of range: skipped
    ek, ev = kc.copy(), vc.copy()
    for i in range(n):
        if 0 <= slots[i] < nb * bs:
            blk, off = divmod(int(slots[i]), bs)
            ek[blk, off] = k[i]
            ev[blk, off] = v[i]
    skipped = o.reshape_and_cache(k, v, slots, kc, vc)
    assert skipped == 2
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev), "cache write differs from the slot rule"


def pin_copy_blocks(o):
    """Whole-block copies against numpy assignment on the 4-D view; bad ids skipped."""
    rng = np.random.default_rng(23)
    nb, bs, hk, d = 9, 16, 2, 64
    kc = rng.integers(0, 65535, size=(nb, bs, hk, d), dtype=np.uint16)
    vc = rng.integers(0, 65535, size=(nb, bs, hk, d), dtype=np.uint16)
    pairs = np.array([[3, 7], [0, 5], [8, 1], [2, 99]], dtype=np.int32)
    ek, ev = kc.copy(), vc.copy()
    for src, dst in pairs[:3]:
        ek[dst] = kc[src]
        ev[dst] = vc[src]
    assert o.copy_blocks(kc, vc, pairs) == 1
    assert np.array_equal(kc, ek) and np.array_equal(vc, ev)


# ------------------------------------------------------------ fp8 (E4M3) cache

def pin_e4m3_decoding(o):
    """All 256 codes against torch's float8_e4m3fn widening."""
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([o.e4m3_to_double(int(c)) for c in range(256)])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    m = ~np.isnan(ref)
    assert np.array_equal(got[m], ref[m])


def pin_e4m3_rounding(o):
    """Round to nearest even against torch inside the finite range (ties included);
    saturation to +-448 beyond it (closed form: the largest finite code)."""
    rng = np.random.default_rng(24)
    vals = np.concatenate([
        rng.uniform(-464, 464, 4000), rng.normal(0, 1, 4000), rng.normal(0, 1e-2, 2000),
        np.ldexp(rng.integers(-60, 60, 2000).astype(np.float64), -12),       # ties and exact values
        np.array([0.0, -0.0, 448.0, -448.0, 464.0, 2.0 ** -10, 3 * 2.0 ** -11, 2.0 ** -6, 15.0 * 2.0 ** -10]),
    ]).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([o.e4m3_from_float(float(x)) for x in vals], dtype=np.uint8)
    assert np.array_equal(got, ref), vals[got != ref][:5]
    for x, code in ((465.0, 0x7e), (1e30, 0x7e), (float("inf"), 0x7e), (-1e9, 0xfe), (-float("inf"), 0xfe)):
        assert o.e4m3_from_float(x) == code, x
    assert o.e4m3_from_float(float("nan")) & 0x7f == 0x7f


def pin_reshape_and_cache_fp8(o):
    """Codes land in their slots: the fp32 quotient rounded by torch, compared per slot."""
    rng = np.random.default_rng(25)
    nb, bs, hk, d, n = 5, 16, 2, 64, 7
    k = to_bits(rng.normal(0, 2, (n, hk, d)), BF16)
    v = to_bits(rng.normal(0, 2, (n, hk, d)), BF16)
    kc = np.zeros((nb, bs, hk, d), dtype=np.uint8)
    vc = np.zeros_like(kc)
    slots = rng.choice(nb * bs, size=n, replace=False).astype(np.int64)
    slots[1] = -1
    ks, vs = np.float32(0.5), np.float32(0.125)
    assert o.reshape_and_cache_fp8(k, v, slots, kc, vc, BF16, ks, vs) == 1
    q = lambda x, sc: torch.from_numpy((from_bits(x, BF16).astype(np.float32) / sc).astype(np.float32)) \
        .to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for i in range(n):
        if slots[i] < 0:
            continue
        blk, off = divmod(int(slots[i]), bs)
        assert np.array_equal(kc[blk, off], q(k[i], ks)) and np.array_equal(vc[blk, off], q(v[i], vs))
    assert np.count_nonzero(kc) <= (n - 1) * hk * d


def pin_decode_fp8_matches_16bit_decode(o):
    """With power-of-two scales every dequantised value is exact in fp16, so decode
    over the codes equals decode over the dequantised fp16 cache, bit for bit."""
    rng = np.random.default_rng(26)
    c = PagedCase(rng, [7, 40, 100], 4, 2, 64, 16, F16, 0.125)
    k8 = rng.integers(0, 256, size=c.k_cache.shape, dtype=np.uint8)
    v8 = rng.integers(0, 256, size=c.v_cache.shape, dtype=np.uint8)
    for arr in (k8, v8):            # keep clear of the NaN codes and of fp16 subnormals after scaling
        arr[(arr & 0x7f) == 0x7f] = 0x38
        arr[(arr & 0x78) == 0] = 0x38
    ks, vs = 0.25, 2.0
    deq = lambda a, sc: torch.from_numpy(a).view(torch.float8_e4m3fn).to(torch.float64).numpy() * sc
    kc16 = to_bits(deq(k8, ks), F16)
    vc16 = to_bits(deq(v8, vs), F16)
    assert np.array_equal(from_bits(kc16, F16), deq(k8, ks)) and np.array_equal(from_bits(vc16, F16), deq(v8, vs))
    got = o.decode_fp8(c.q, k8, v8, c.tables, c.lens, c.scale, ks, vs, F16)
    ref = o.decode(c.q, kc16, vc16, c.tables, c.lens, c.scale, F16)
    assert np.array_equal(got, ref)


# -------------------------------------------------------------------- decode

def pin_decode_one_token(o):
    """L = 1: the softmax weight is exactly 1, so out = V[0] exactly."""
    rng = np.random.default_rng(13)
    c = PagedCase(rng, [1, 1, 1], 4, 2, 64, 16, F16, 0.125)
    out = c.run(o)
    for s in range(3):
        for h in range(4):
            assert np.array_equal(out[s, h], from_bits(c.seq_v[s][0, h // 2], F16)), (s, h)


def pin_decode_equal_scores(o):
    """q = 0 makes every score equal: out = mean of V over the sequence."""
    rng = np.random.default_rng(14)
    c = PagedCase(rng, [7, 40, 129], 2, 2, 128, 16, BF16, 0.3)
    c.q[:] = 0
    out = c.run(o)
    for s in range(3):
        ref = from_bits(c.seq_v[s], BF16).mean(axis=0)   # [Hk, d]
        assert np.allclose(out[s], ref, rtol=0, atol=1e-13), s


def pin_decode_two_tokens(o):
    """Two tokens: out = sigma(x0 - x1) v0 + sigma(x1 - x0) v1."""
    rng = np.random.default_rng(15)
    c = PagedCase(rng, [2], 1, 1, 64, 16, F16, 0.2)
    qd = from_bits(c.q[0, 0], F16)
    k = from_bits(c.seq_k[0][:, 0], F16)
    v = from_bits(c.seq_v[0][:, 0], F16)
    x0, x1 = 0.2 * np.dot(qd, k[0]), 0.2 * np.dot(qd, k[1])
    sig = 1.0 / (1.0 + math.exp(-(x0 - x1)))
    ref = sig * v[0] + (1.0 - sig) * v[1]
    assert np.allclose(c.run(o)[0, 0], ref, rtol=0, atol=1e-14)


def pin_decode_dominant_token(o):
    """A one-hot q with a large scale picks the token with the largest key entry."""
    rng = np.random.default_rng(16)
    c = PagedCase(rng, [45], 1, 1, 64, 16, F16, 1.0e3, dist="uniform")
    c.q[:] = to_bits(np.eye(64)[5][None, None, :], F16)
    t_star = 29
    c.seq_k[0][:, 0, 5] = to_bits(rng.uniform(-1.0, 0.5, 45), F16)
    c.seq_k[0][t_star, 0, 5] = to_bits(np.array([0.9]), F16)[0]   # winner by >= 0.4 * 1e3 in score
    c._assemble()
    out = c.run(o)[0, 0]
    assert np.allclose(out, from_bits(c.seq_v[0][t_star, 0], F16), rtol=0, atol=1e-12)


def _sdpa_cases():
    rng = np.random.default_rng(17)
    return [
        PagedCase(rng, [5, 17, 33, 50], 4, 4, 64, 16, F16, 1 / 8, dist="uniform"),   # the tiny workload's shape
        PagedCase(rng, [1, 31, 64, 100], 8, 2, 128, 16, BF16, 0.09),               # GQA, group 4
        PagedCase(rng, [3, 70, 129], 6, 3, 64, 4, F16, 0.5),                        # block size 4
        PagedCase(rng, [65, 200], 4, 1, 128, 64, BF16, 1 / math.sqrt(128)),          # block size 64, MQA
    ]


def pin_decode_matches_sdpa(o):
    """Paged attention equals dense attention over the contiguous cache."""
    for c in _sdpa_cases():
        got = c.run(o)
        ref = c.sdpa()
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12), "oracle differs from contiguous attention"


def pin_decode_relabel_invariance(o):
    """Relabelling physical blocks (moving their data along) changes nothing, bit for bit."""
    rng = np.random.default_rng(18)
    c = PagedCase(rng, [9, 48, 77], 4, 2, 64, 16, F16, 0.125, extra_blocks=5)
    a = c.run(o)
    c.relabel(rng.permutation(c.NB).astype(np.int32))
    b = c.run(o)
    assert np.array_equal(a, b)


def pin_decode_shared_prefix(o):
    """Sequences whose tables share prefix blocks and whose suffixes hold the same
    data give the same output as unshared copies, bit for bit."""
    rng = np.random.default_rng(19)
    c = PagedCase(rng, [48 + 10, 48 + 10], 2, 2, 64, 16, F16, 0.125, extra_blocks=4)
    c.q[1] = c.q[0]
    c.seq_k[1] = c.seq_k[0].copy()
    c.seq_v[1] = c.seq_v[0].copy()
    c._assemble()
    unshared = c.run(o)
    c.tables[1, :3] = c.tables[0, :3]       # share the 3 full prefix blocks
    c._assemble()
    shared = c.run(o)
    assert np.array_equal(unshared[0], unshared[1]) and np.array_equal(shared, unshared)


def pin_decode_empty(o):
    rng = np.random.default_rng(20)
    c = PagedCase(rng, [0, 3], 2, 2, 64, 16, F16, 0.125)
    out = c.run(o)
    assert np.array_equal(out[0], np.zeros((2, 64)))


def pin_decode_split_merge(o):
    """Partials (m_p, l_p, o_p) over any split of the tokens merge to the unsplit
    result: M = max m_p, l = sum l_p e^(m_p - M), out = sum o_p e^(m_p - M) / l."""
    rng = np.random.default_rng(21)
    c = PagedCase(rng, [300], 2, 2, 64, 16, BF16, 0.11)
    full = c.run(o)
    k = from_bits(c.seq_k[0], BF16)
    v = from_bits(c.seq_v[0], BF16)
    for h in range(2):
        qd = from_bits(c.q[0, h], BF16)
        x = c.scale * (k[:, h] @ qd)
        cuts = np.sort(rng.choice(np.arange(1, 300), size=6, replace=False))
        parts = np.split(np.arange(300), cuts)
        ms = np.array([x[p].max() for p in parts])
        ls = np.array([np.exp(x[p] - x[p].max()).sum() for p in parts])
        os_ = np.array([(np.exp(x[p] - x[p].max())[:, None] * v[p, h]).sum(0) for p in parts])
        mm = ms.max()
        w = np.exp(ms - mm)
        merged = (w[:, None] * os_).sum(0) / (w * ls).sum()
        assert np.allclose(merged, full[0, h], rtol=1e-12, atol=1e-12)


def pin_decode_not_per_block_sum(o):
    """The per-block sum of softmaxes printed as the 'blocked' formula is not
    normalised: for more than one block it differs from the oracle."""
    rng = np.random.default_rng(22)
    c = PagedCase(rng, [64], 1, 1, 64, 16, F16, 0.125)
    qd = from_bits(c.q[0, 0], F16)
    k = from_bits(c.seq_k[0][:, 0], F16)
    v = from_bits(c.seq_v[0][:, 0], F16)
    blocked = np.zeros(64)
    for b in range(4):
        xb = 0.125 * (k[16 * b:16 * b + 16] @ qd)
        pb = np.exp(xb - xb.max())
        blocked += (pb / pb.sum()) @ v[16 * b:16 * b + 16]
    got = c.run(o)[0, 0]
    assert np.abs(got - blocked).max() > 0.1


# ------------------------------------------------------------------- prefill

def _packed_queries(c, n_new, rng):
    """Query rows of the last n_new[s] tokens of each sequence, packed by sequence."""
    qs = np.concatenate([[0], np.cumsum(n_new)]).astype(np.int32)
    q = to_bits(rng.normal(0, 1, (int(qs[-1]), c.H, c.d)), c.dtype)
    return q, qs


def pin_prefill_single_query_is_decode(o):
    """A chunk of one query token per sequence is exactly a decode step."""
    rng = np.random.default_rng(27)
    c = PagedCase(rng, [9, 40, 130], 4, 2, 64, 16, F16, 0.125)
    got = o.prefill(c.q.reshape(3, 4, 64).copy(), c.k_cache, c.v_cache, c.tables, c.lens,
                    np.arange(4, dtype=np.int32), c.scale, F16)
    assert np.array_equal(got, c.run(o))


def pin_prefill_matches_masked_sdpa(o):
    """Against torch's scaled_dot_product_attention on the contiguous K/V with the
    causal mask of the chunk: query i of a chunk of n over L tokens sees t <= L-n+i
    (a whole-prompt chunk, n = L, is the plain causal case)."""
    rng = np.random.default_rng(28)
    for lens, n_new, h, hk, bs in (([37, 80], [37, 80], 4, 4, 16), ([50, 129, 64], [5, 33, 64], 6, 2, 16),
                                   ([70], [19], 2, 1, 64)):
        c = PagedCase(rng, lens, h, hk, 64, bs, BF16, 0.13)
        q, qs = _packed_queries(c, n_new, rng)
        got = o.prefill(q, c.k_cache, c.v_cache, c.tables, c.lens, qs, c.scale, BF16)
        for s, (L, n) in enumerate(zip(lens, n_new)):
            qq = torch.from_numpy(from_bits(q[qs[s]:qs[s + 1]], BF16)).permute(1, 0, 2)[None]   # [1,H,n,d]
            k = torch.from_numpy(from_bits(c.seq_k[s], BF16)).permute(1, 0, 2)[None]           # [1,Hk,L,d]
            v = torch.from_numpy(from_bits(c.seq_v[s], BF16)).permute(1, 0, 2)[None]
            mask = torch.arange(L)[None, :] <= (L - n + torch.arange(n))[:, None]
            ref = torch.nn.functional.scaled_dot_product_attention(qq, k, v, attn_mask=mask, scale=c.scale,
                                                                   enable_gqa=h != hk)
            assert np.allclose(got[qs[s]:qs[s + 1]], ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
