// Tensor-core compute policy for fp8 (E4M3) caches: one unit = one kv head with
// its whole group of query heads, as on the 16-bit GQA path, so one fetch of a
// token's K/V codes serves every query head of the group.
//
// The codes go from the landed (128-byte-swizzled) stage straight into mma.sync
// fragments, with no 16-bit copy of the tile: E4M3 -> f16 is exact, and one
// cvt turns two codes into one 16-bit pair of a fragment.  Both products run in
// f16 with fp32 accumulation whatever q's type:
//   S^T[16 tok x 8 heads] = K[16 tok x 128] . Q^T[128 x 8 heads]
//   O^T[128 x 8 heads]   += V^T[128 x 16 tok] . P^T[16 tok x 8 heads]
// Each product permutes one index whose order is free, so that its fragments come
// from 16-byte shared loads that hit every bank once per quarter warp:
//   q K^T: the reduction index (a contraction may visit it in any order).  Lane
//          (g, t) takes code bytes 32t .. 32t+31 of token rows g and g+8;
//          k-step ks covers dims 32t' + 4ks + {0,1} as k = 2t', 2t'+1 and
//          32t' + 4ks + {2,3} as k = 2t'+8, 2t'+9 (t' = 0..3), and q^T's B
//          fragment is loaded in the same order.
//   V^T P^T: the M index (the output dims, put back in order when written).
//          m-tile mt holds dims 16g + 2mt (row g) and 16g + 2mt + 1 (row g+8),
//          so lane (g, t) reads 16-byte chunk g of token rows 2t, 2t+1, 2t+8,
//          2t+9 and transposes bytes in registers (prmt) into the (dim, token
//          pair) fragments.
// q of a bf16 model enters as f16 scaled by a power of two 2^k that brings the
// group's largest |q| to [2^14, 2^15); the scale is undone on the scores.  This
// is exact except for elements below 2^-31 of that largest one, which round to
// f16's subnormal grid (a relative error under 2^-31 in the dot product).  The K
// scale multiplies the scores and the V scale the output, as on the CUDA-core
// fp8 path.
#pragma once

#include "decode_gqa.cuh"

namespace pa {

__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t pair16) { return E4M3Tag::to_f16x2(pair16); }

__device__ __forceinline__ uint32_t byte_perm(uint32_t lo, uint32_t hi, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(lo), "r"(hi), "r"(sel));
    return d;
}

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

// Tag: q's (and the output's) type.  TOK: tokens per landed stage of codes, a
// multiple of 16, computed 16 at a time.  NT: 8-head tiles of the group.
template <class Tag, int TOK, int NT>
struct Fp8TcPolicy {
    static constexpr int D = 128;       // one 128-byte code row per token
    static constexpr int KS = D / 16;   // k-steps of q K^T
    static constexpr int MT = D / 16;   // m-tiles of V^T P^T
    static constexpr int NTT = TOK / 16;
    static_assert(TOK % 16 == 0, "stage shape");
    static constexpr int kScratchBytes = 0;
    using Ops = MmaOps<F16Tag>;

    int lane, g, t;
    uint32_t qb[NT][KS][2];  // f16 Q^T B fragments of the current unit (permuted dims)
    uint32_t qn[NT][16];     // q words of the next unit: dims 32t + 2j, +1 of head nt*8 + g
    float qinv;              // 2^-k of the current unit's q scale
    float m[NT][2], lsum[NT][2];
    float o[NT][MT][4];      // O^T: rows g -> dim 16g + 2mt, g+8 -> 16g + 2mt + 1; heads 2t, 2t+1
    bool poisoned;

    __device__ __forceinline__ void setup(int lane_, uint8_t* /*scratch*/) {
        lane = lane_;
        g = lane >> 2;
        t = lane & 3;
    }

    __device__ __forceinline__ void fetch_q(const DecodeArgs& a, const Unit& U) {
        if (U.kind != kUnitNormal) return;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int head = nt * 8 + g;
            const bool real = head < a.heads_per_unit;
            const uint4* row = reinterpret_cast<const uint4*>(
                a.q + ((int64_t)U.s * a.num_heads + U.h * a.heads_per_unit + (real ? head : 0)) * D);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 w = real ? __ldg(row + 4 * t + i) : make_uint4(0u, 0u, 0u, 0u);
                qn[nt][4 * i] = w.x;
                qn[nt][4 * i + 1] = w.y;
                qn[nt][4 * i + 2] = w.z;
                qn[nt][4 * i + 3] = w.w;
            }
        }
    }

    __device__ __forceinline__ void take_q(const DecodeArgs& a) {
        (void)a;
        if constexpr (Tag::kIsBF16) {
            float mx = 0.f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float2 v = BF16Tag::widen2(qn[nt][j]);
                    mx = fmaxf(mx, fmaxf(fabsf(v.x), fabsf(v.y)));
                }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, off));
            float s;
            f16_entry_scale(mx, s, qinv);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int ks = 0; ks < KS; ++ks)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float2 v = BF16Tag::widen2(qn[nt][2 * ks + h]);
                        qb[nt][ks][h] = pack_f16x2(v.x * s, v.y * s);
                    }
        } else {
            qinv = 1.f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    qb[nt][ks][0] = qn[nt][2 * ks];      // dims 32t + 4ks, +1
                    qb[nt][ks][1] = qn[nt][2 * ks + 1];  // dims 32t + 4ks + 2, +3
                }
        }
    }

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m[nt][0] = m[nt][1] = -INFINITY;
            lsum[nt][0] = lsum[nt][1] = 0.f;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) o[nt][mt][0] = o[nt][mt][1] = o[nt][mt][2] = o[nt][mt][3] = 0.f;
        }
        poisoned = false;
    }

    __device__ __forceinline__ void poison() { poisoned = true; }

    // q K^T of one 16-token tile (rows g and g+8 of the codes at kr) into x, two
    // accumulators (even and odd k-steps) halving the chain of dependent MMAs
    __device__ __forceinline__ void scores(const uint8_t* kr, float (&x)[NT][4]) const {
        const uint4 k0a = lds128(kr + g * 128 + (((2 * t) ^ g) << 4));
        const uint4 k0b = lds128(kr + g * 128 + (((2 * t + 1) ^ g) << 4));
        const uint4 k1a = lds128(kr + (g + 8) * 128 + (((2 * t) ^ g) << 4));
        const uint4 k1b = lds128(kr + (g + 8) * 128 + (((2 * t + 1) ^ g) << 4));
        const uint32_t kw0[8] = {k0a.x, k0a.y, k0a.z, k0a.w, k0b.x, k0b.y, k0b.z, k0b.w};  // token g
        const uint32_t kw1[8] = {k1a.x, k1a.y, k1a.z, k1a.w, k1b.x, k1b.y, k1b.z, k1b.w};  // token g+8
        float y[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) x[nt][j] = y[nt][j] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            uint32_t af[4];
            af[0] = e4m3x2_to_f16x2(kw0[ks] & 0xffffu);
            af[1] = e4m3x2_to_f16x2(kw1[ks] & 0xffffu);
            af[2] = e4m3x2_to_f16x2(kw0[ks] >> 16);
            af[3] = e4m3x2_to_f16x2(kw1[ks] >> 16);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) Ops::mma((ks & 1) ? y[nt] : x[nt], af, qb[nt][ks][0], qb[nt][ks][1]);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) x[nt][j] += y[nt][j];
    }

    // O^T += V^T P^T for one 16-token tile (codes at vr, nv valid tokens)
    __device__ __forceinline__ void values(const uint8_t* vr, int nv, const uint32_t (&bhi)[NT][2],
                                           const uint32_t (&blo)[NT][2]) {
        const uint4 r0 = lds128(vr + (2 * t) * 128 + ((g ^ (2 * t)) << 4));
        const uint4 r1 = lds128(vr + (2 * t + 1) * 128 + ((g ^ (2 * t + 1)) << 4));
        const uint4 r8 = lds128(vr + (2 * t + 8) * 128 + ((g ^ (2 * t)) << 4));
        const uint4 r9 = lds128(vr + (2 * t + 9) * 128 + ((g ^ (2 * t + 1)) << 4));
        const uint32_t w0[4] = {r0.x, r0.y, r0.z, r0.w}, w1[4] = {r1.x, r1.y, r1.z, r1.w};
        const uint32_t w8[4] = {r8.x, r8.y, r8.z, r8.w}, w9[4] = {r9.x, r9.y, r9.z, r9.w};
        const uint32_t mask01 = gqa_pair_mask(2 * t, nv), mask89 = gqa_pair_mask(2 * t + 8, nv);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
            const uint32_t p01 = byte_perm(w0[mt >> 1], w1[mt >> 1], sel);
            const uint32_t p89 = byte_perm(w8[mt >> 1], w9[mt >> 1], sel);
            uint32_t af[4];
            af[0] = e4m3x2_to_f16x2(p01 & 0xffffu);
            af[1] = e4m3x2_to_f16x2(p01 >> 16);
            af[2] = e4m3x2_to_f16x2(p89 & 0xffffu);
            af[3] = e4m3x2_to_f16x2(p89 >> 16);
            if (nv < 16) {
                af[0] &= mask01;
                af[1] &= mask01;
                af[2] &= mask89;
                af[3] &= mask89;
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                Ops::mma(o[nt][mt], af, bhi[nt][0], bhi[nt][1]);
                Ops::mma(o[nt][mt], af, blo[nt][0], blo[nt][1]);
            }
        }
    }

    __device__ __forceinline__ void stage(const DecodeArgs& a, const uint8_t* kt, const uint8_t* vt, int ntok) {
        const float sc = a.scale_log2 * a.k_scale * qinv;
        if (NTT == 2 && ntok > 16) {
            // both 16-token tiles of the stage together: two independent score chains,
            // one softmax step over the 32 tokens, then both P.V products
            float xa[NT][4], xb[NT][4];
            scores(kt, xa);
            scores(kt + 2048, xb);
            uint32_t bhi[2][NT][2], blo[2][NT][2];
            gqa_softmax_2tiles<F16Tag>(xa, xb, g, 16, ntok - 16, sc, m, lsum, o, bhi, blo);
            values(vt, 16, bhi[0], blo[0]);
            values(vt + 2048, ntok - 16, bhi[1], blo[1]);
            return;
        }
#pragma unroll
        for (int tt = 0; tt < NTT; ++tt) {
            const int nv = ntok - tt * 16;  // valid tokens in this tile (warp-uniform)
            if (nv <= 0) break;
            // Code chunk c (bytes 16c .. 16c+15) of tile row r sits at r*128 + ((c ^ r%8) << 4); tiles
            // start at multiples of 16 rows, so the phase r % 8 is the row's index within the tile mod 8.
            const uint8_t* kr = kt + tt * 2048;
            const uint4 k0a = lds128(kr + g * 128 + (((2 * t) ^ g) << 4));
            const uint4 k0b = lds128(kr + g * 128 + (((2 * t + 1) ^ g) << 4));
            const uint4 k1a = lds128(kr + (g + 8) * 128 + (((2 * t) ^ g) << 4));
            const uint4 k1b = lds128(kr + (g + 8) * 128 + (((2 * t + 1) ^ g) << 4));
            const uint32_t kw0[8] = {k0a.x, k0a.y, k0a.z, k0a.w, k0b.x, k0b.y, k0b.z, k0b.w};  // token g
            const uint32_t kw1[8] = {k1a.x, k1a.y, k1a.z, k1a.w, k1b.x, k1b.y, k1b.z, k1b.w};  // token g+8
            // two accumulators (even and odd k-steps) halve the chain of dependent MMAs
            float x[NT][4], y[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 4; ++j) x[nt][j] = y[nt][j] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t af[4];
                af[0] = e4m3x2_to_f16x2(kw0[ks] & 0xffffu);  // token g,   dims 32t + 4ks, +1
                af[1] = e4m3x2_to_f16x2(kw1[ks] & 0xffffu);  // token g+8
                af[2] = e4m3x2_to_f16x2(kw0[ks] >> 16);      // token g,   dims 32t + 4ks + 2, +3
                af[3] = e4m3x2_to_f16x2(kw1[ks] >> 16);      // token g+8
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) Ops::mma((ks & 1) ? y[nt] : x[nt], af, qb[nt][ks][0], qb[nt][ks][1]);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 4; ++j) x[nt][j] += y[nt][j];
            uint32_t bhi[NT][2], blo[NT][2];
            gqa_softmax_tile<F16Tag>(x, g, nv, sc, m, lsum, o, bhi, blo);

            // V: chunk g of token rows 2t, 2t+1, 2t+8, 2t+9 (phases 2t, 2t+1, 2t, 2t+1)
            const uint8_t* vr = vt + tt * 2048;
            const uint4 r0 = lds128(vr + (2 * t) * 128 + ((g ^ (2 * t)) << 4));
            const uint4 r1 = lds128(vr + (2 * t + 1) * 128 + ((g ^ (2 * t + 1)) << 4));
            const uint4 r8 = lds128(vr + (2 * t + 8) * 128 + ((g ^ (2 * t)) << 4));
            const uint4 r9 = lds128(vr + (2 * t + 9) * 128 + ((g ^ (2 * t + 1)) << 4));
            const uint32_t w0[4] = {r0.x, r0.y, r0.z, r0.w}, w1[4] = {r1.x, r1.y, r1.z, r1.w};
            const uint32_t w8[4] = {r8.x, r8.y, r8.z, r8.w}, w9[4] = {r9.x, r9.y, r9.z, r9.w};
            const uint32_t mask01 = gqa_pair_mask(2 * t, nv), mask89 = gqa_pair_mask(2 * t + 8, nv);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                // bytes 2mt, 2mt+1 of the chunk (dims 16g + 2mt, +1) of a token pair, interleaved:
                // [v(tok, d0), v(tok+1, d0), v(tok, d1), v(tok+1, d1)]
                const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
                const uint32_t p01 = byte_perm(w0[mt >> 1], w1[mt >> 1], sel);
                const uint32_t p89 = byte_perm(w8[mt >> 1], w9[mt >> 1], sel);
                uint32_t af[4];
                af[0] = e4m3x2_to_f16x2(p01 & 0xffffu);  // dim 16g + 2mt,     tokens 2t, 2t+1
                af[1] = e4m3x2_to_f16x2(p01 >> 16);      // dim 16g + 2mt + 1, tokens 2t, 2t+1
                af[2] = e4m3x2_to_f16x2(p89 & 0xffffu);  // dim 16g + 2mt,     tokens 2t+8, 2t+9
                af[3] = e4m3x2_to_f16x2(p89 >> 16);      // dim 16g + 2mt + 1, tokens 2t+8, 2t+9
                if (nv < 16) {
                    af[0] &= mask01;
                    af[1] &= mask01;
                    af[2] &= mask89;
                    af[3] &= mask89;
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    Ops::mma(o[nt][mt], af, bhi[nt][0], bhi[nt][1]);
                    Ops::mma(o[nt][mt], af, blo[nt][0], blo[nt][1]);
                }
            }
        }
    }

    __device__ __forceinline__ void finish(const DecodeArgs& a, const Unit& U) {
        const bool bad = __any_sync(kFullMask, poisoned);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float l = lsum[nt][j];
                l += __shfl_xor_sync(kFullMask, l, 4);
                l += __shfl_xor_sync(kFullMask, l, 8);
                l += __shfl_xor_sync(kFullMask, l, 16);
                if (bad) l = __int_as_float(0x7fc00000);
                const int head = nt * 8 + 2 * t + j;
                if (head >= a.heads_per_unit) continue;
                const int64_t sh = (int64_t)U.s * a.num_heads + U.h * a.heads_per_unit + head;
                // this lane's 16 output dims are 16g .. 16g+15: (row g, row g+8) of m-tile mt are 16g + 2mt, +1
                if (U.np == 1) {
                    const float inv = a.v_scale / l;
                    uint32_t h[8];
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)
                        h[mt] = (uint32_t)Tag::round1(o[nt][mt][j] * inv) |
                                ((uint32_t)Tag::round1(o[nt][mt][j + 2] * inv) << 16);
                    uint4* dst = reinterpret_cast<uint4*>(a.out + sh * D + 16 * g);
                    dst[0] = make_uint4(h[0], h[1], h[2], h[3]);
                    dst[1] = make_uint4(h[4], h[5], h[6], h[7]);
                } else {
                    const int64_t pi = sh * a.num_partitions + U.p;
                    float4* dst = reinterpret_cast<float4*>(a.ws_o + pi * D + 16 * g);
                    const float vs = a.v_scale;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        dst[q4] = make_float4(o[nt][2 * q4][j] * vs, o[nt][2 * q4][j + 2] * vs,
                                              o[nt][2 * q4 + 1][j] * vs, o[nt][2 * q4 + 1][j + 2] * vs);
                    if (g == 0) {
                        a.ws_m[pi] = m[nt][j];
                        a.ws_l[pi] = l;
                    }
                }
            }
    }
};

}  // namespace pa
