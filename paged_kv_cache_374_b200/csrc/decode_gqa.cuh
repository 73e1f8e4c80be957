// Tensor-core compute policy of the decode engine for grouped-query attention:
// one unit = one kv head with its group of up to 8 * NT query heads, which share
// every K/V tile the unit streams.
//
// The group makes q K^T a small dense contraction, run with mma.sync m16n8k16
// (16-bit inputs, fp32 accumulation) with the tokens of a 16-token tile on M and
// the group's query heads on N:
//   S^T[16 tok x 8 heads] = K[16 tok x D] . Q^T[D x 8 heads]      (KS = D/16 MMAs)
//   O^T[D x 8 heads]     += V^T[D x 16 tok] . P^T[16 tok x 8 heads] (D/16 MMAs, twice)
// K comes from the swizzled shared tile with ldmatrix, V^T with ldmatrix.trans.
// Products of two 16-bit inputs are exact in fp32, so the logits are the fp32
// dot products.  P^T (the B operand of the second product) is the accumulator
// fragment of S^T transposed in registers with movmatrix; to keep p at about 16
// significant bits it enters as two 16-bit terms, p = hi + lo, and the second
// product is issued once for each.  The online softmax runs per query head in
// base 2 on the fp32 accumulator values; the per-head max over the tile's tokens
// and the rescale of O^T run only when some score exceeds its head's running max.
// Padding heads (group < 8 * NT) get q = 0 and are never written.
#pragma once

#include "decode_engine.cuh"

namespace pa {

template <class Tag>
struct MmaOps;

template <>
struct MmaOps<F16Tag> {
    static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    // (lo, hi) -> packed pair, lo in the low half
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        uint32_t d;
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
        return d;
    }
};

template <>
struct MmaOps<BF16Tag> {
    static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        uint32_t d;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
        return d;
    }
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(p)));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// One online-softmax step over a 16-token tile of S^T, shared by the tensor-core
// policies.  This lane holds tokens g and g+8 x query heads 2t, 2t+1 of each of the
// NT head tiles (the m16n8 accumulator layout).  The raw dot products are scaled
// by sc into base-2 units, tokens at or past nv are masked, the per-head running
// max (and with it the rescale of lsum and of O^T) moves only when some score
// exceeds it, and P^T is returned as the B fragments of V^T P^T: p = hi + lo in
// 16-bit pairs of the MMA type P, transposed to (head row, tokens 2t/2t+1).
template <class P, int NT, int MT>
__device__ __forceinline__ void gqa_softmax_tile(float (&x)[NT][4], int g, int nv, float sc, float (&m)[NT][2],
                                                 float (&lsum)[NT][2], float (&o)[NT][MT][4],
                                                 uint32_t (&bhi)[NT][2], uint32_t (&blo)[NT][2]) {
    const bool v0 = g < nv, v1 = g + 8 < nv;
    bool up = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int j = 0; j < 4; ++j) x[nt][j] *= sc;
        if (!v0) x[nt][0] = x[nt][1] = -INFINITY;
        if (!v1) x[nt][2] = x[nt][3] = -INFINITY;
        up |= x[nt][0] > m[nt][0] || x[nt][2] > m[nt][0] || x[nt][1] > m[nt][1] || x[nt][3] > m[nt][1];
    }
    if (__any_sync(kFullMask, up)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float mx = fmaxf(x[nt][j], x[nt][j + 2]);
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 16));
                const float m_new = fmaxf(m[nt][j], mx);
                const float alpha = fast_exp2(m[nt][j] - m_new);
                lsum[nt][j] *= alpha;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    o[nt][mt][j] *= alpha;
                    o[nt][mt][j + 2] *= alpha;
                }
                m[nt][j] = m_new;
            }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        float p[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) p[j] = fast_exp2(x[nt][j] - m[nt][j & 1]);
        lsum[nt][0] += p[0] + p[2];
        lsum[nt][1] += p[1] + p[3];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const uint32_t hi = MmaOps<P>::pack(p[2 * half], p[2 * half + 1]);
            const float2 hv = P::widen2(hi);
            const uint32_t lo = MmaOps<P>::pack(p[2 * half] - hv.x, p[2 * half + 1] - hv.y);
            bhi[nt][half] = movmatrix_trans(hi);
            blo[nt][half] = movmatrix_trans(lo);
        }
    }
}

// The same step over two 16-token tiles at once (tokens g, g+8 of tile A in xa,
// of tile B in xb; nva, nvb valid tokens): one max update and one rescale for the
// 32 tokens, then P^T fragments for both tiles.  The result is the online
// softmax of the two tiles taken in one step (the same softmax up to rounding).
template <class P, int NT, int MT>
__device__ __forceinline__ void gqa_softmax_2tiles(float (&xa)[NT][4], float (&xb)[NT][4], int g, int nva, int nvb,
                                                   float sc, float (&m)[NT][2], float (&lsum)[NT][2],
                                                   float (&o)[NT][MT][4], uint32_t (&bhi)[2][NT][2],
                                                   uint32_t (&blo)[2][NT][2]) {
    bool up = false;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            xa[nt][j] *= sc;
            xb[nt][j] *= sc;
        }
        if (!(g < nva)) xa[nt][0] = xa[nt][1] = -INFINITY;
        if (!(g + 8 < nva)) xa[nt][2] = xa[nt][3] = -INFINITY;
        if (!(g < nvb)) xb[nt][0] = xb[nt][1] = -INFINITY;
        if (!(g + 8 < nvb)) xb[nt][2] = xb[nt][3] = -INFINITY;
#pragma unroll
        for (int j = 0; j < 2; ++j)
            up |= fmaxf(fmaxf(xa[nt][j], xa[nt][j + 2]), fmaxf(xb[nt][j], xb[nt][j + 2])) > m[nt][j];
    }
    if (__any_sync(kFullMask, up)) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float mx = fmaxf(fmaxf(xa[nt][j], xa[nt][j + 2]), fmaxf(xb[nt][j], xb[nt][j + 2]));
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 16));
                const float m_new = fmaxf(m[nt][j], mx);
                const float alpha = fast_exp2(m[nt][j] - m_new);
                lsum[nt][j] *= alpha;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    o[nt][mt][j] *= alpha;
                    o[nt][mt][j + 2] *= alpha;
                }
                m[nt][j] = m_new;
            }
    }
#pragma unroll
    for (int tile = 0; tile < 2; ++tile)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float p[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) p[j] = fast_exp2((tile ? xb : xa)[nt][j] - m[nt][j & 1]);
            lsum[nt][0] += p[0] + p[2];
            lsum[nt][1] += p[1] + p[3];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const uint32_t hi = MmaOps<P>::pack(p[2 * half], p[2 * half + 1]);
                const float2 hv = P::widen2(hi);
                const uint32_t lo = MmaOps<P>::pack(p[2 * half] - hv.x, p[2 * half + 1] - hv.y);
                bhi[tile][nt][half] = movmatrix_trans(hi);
                blo[tile][nt][half] = movmatrix_trans(lo);
            }
        }
}

// Keep-mask of a 16-bit pair holding tokens k and k+1 of a tile with nv valid
// tokens.  Rows past the sequence end may hold anything (NaN included): their p
// is 0, but 0 * NaN is NaN inside the MMA, so their V entries are zeroed.
__device__ __forceinline__ uint32_t gqa_pair_mask(int k, int nv) {
    return (k < nv ? 0x0000ffffu : 0u) | (k + 1 < nv ? 0xffff0000u : 0u);
}

template <class Tag, int D, int TOK, int NT>
struct GqaPolicy {
    static constexpr int KS = D / 16;     // k-steps of q K^T over the head dims
    static constexpr int MT = D / 16;     // m-tiles of V^T P^T over the head dims
    static constexpr int NTT = TOK / 16;  // 16-token tiles per stage
    static_assert(TOK % 16 == 0, "stage shape");
    static constexpr int HALF_BYTES = TOK * 128;
    using Ops = MmaOps<Tag>;

    int lane, g, t;                 // mma groupID (lane / 4) and thread-in-group (lane % 4)
    int kbase, vbase;               // ldmatrix row offsets of this lane in a tile
    uint32_t qb[NT][KS][2];         // Q^T B fragments of the current unit
    uint32_t qn[NT][KS][2];         // ... of the next unit
    float m[NT][2], lsum[NT][2];    // per query head 2t, 2t+1 of each head tile
    float o[NT][MT][4];             // O^T fragments: dims mt*16 + g (+8), heads 2t, 2t+1
    bool poisoned;

    static constexpr int kScratchBytes = 0;

    __device__ __forceinline__ void setup(int lane_, uint8_t* /*scratch*/) {
        lane = lane_;
        g = lane >> 2;
        t = lane & 3;
        // K (A of q K^T, row-major): matrices (rows 0-7 | 8-15) x (k 0-7 | 8-15)
        kbase = ((lane & 7) + ((lane >> 3) & 1) * 8) * 128;
        // V^T (A of V^T P^T, from token-major rows with .trans): (dims 0-7 | 8-15) x (tokens 0-7 | 8-15)
        vbase = ((lane & 7) + ((lane >> 4) & 1) * 8) * 128;
    }

    // shared offset of 16-byte chunk kc (0..D/8-1) of the row this lane addresses
    __device__ __forceinline__ int koff(int ks) const {
        const int kc = ks * 2 + (lane >> 4);
        return (kc >> 3) * HALF_BYTES + kbase + (((kc & 7) ^ (lane & 7)) << 4);
    }
    __device__ __forceinline__ int voff(int mt) const {
        const int kc = mt * 2 + ((lane >> 3) & 1);
        return (kc >> 3) * HALF_BYTES + vbase + (((kc & 7) ^ (lane & 7)) << 4);
    }

    __device__ __forceinline__ void fetch_q(const DecodeArgs& a, const Unit& U) {
        if (U.kind != kUnitNormal) return;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int head = nt * 8 + g;
            const bool real = head < a.heads_per_unit;
            const uint32_t* row = reinterpret_cast<const uint32_t*>(
                a.q + ((int64_t)U.s * a.num_heads + U.h * a.heads_per_unit + (real ? head : 0)) * D);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                qn[nt][ks][0] = real ? __ldg(row + ks * 8 + t) : 0u;      // dims ks*16 + 2t, +1
                qn[nt][ks][1] = real ? __ldg(row + ks * 8 + 4 + t) : 0u;  // dims ks*16 + 8 + 2t, +1
            }
        }
    }

    __device__ __forceinline__ void take_q(const DecodeArgs& a) {
        (void)a;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                qb[nt][ks][0] = qn[nt][ks][0];
                qb[nt][ks][1] = qn[nt][ks][1];
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

    __device__ __forceinline__ void stage(const DecodeArgs& a, const uint8_t* kt, const uint8_t* vt, int ntok) {
#pragma unroll
        for (int tt = 0; tt < NTT; ++tt) {
            const int nv = ntok - tt * 16;  // valid tokens in this tile (warp-uniform)
            if (nv <= 0) break;
            // S^T for this 16-token tile: lane holds tokens g, g+8 x heads 2t, 2t+1
            float x[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) x[nt][0] = x[nt][1] = x[nt][2] = x[nt][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t af[4];
                ldsm_x4(af, kt + tt * 2048 + koff(ks));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) Ops::mma(x[nt], af, qb[nt][ks][0], qb[nt][ks][1]);
            }
            const float sc = a.scale_log2 * a.k_scale;  // k_scale: 1, or the fp8 cache's K scale
            uint32_t bhi[NT][2], blo[NT][2];
            gqa_softmax_tile<Tag>(x, g, nv, sc, m, lsum, o, bhi, blo);
            // V^T entries of tokens past the end are zeroed (lane: tokens 2t, 2t+1 and 2t+8, 2t+9)
            const uint32_t mask01 = gqa_pair_mask(2 * t, nv), mask89 = gqa_pair_mask(2 * t + 8, nv);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t af[4];
                ldsm_x4_trans(af, vt + tt * 2048 + voff(mt));
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
                if (a.v_scale != 1.f) {  // fp8 cache: V = code * v_scale
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        o[nt][mt][j] *= a.v_scale;
                        o[nt][mt][j + 2] *= a.v_scale;
                    }
                }
                const int head = nt * 8 + 2 * t + j;
                if (head >= a.heads_per_unit) continue;
                const int64_t sh = (int64_t)U.s * a.num_heads + U.h * a.heads_per_unit + head;
                if (U.np == 1) {
                    const float inv = 1.f / l;
                    uint16_t* row = a.out + sh * D;
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        row[mt * 16 + g] = Tag::round1(o[nt][mt][j] * inv);
                        row[mt * 16 + g + 8] = Tag::round1(o[nt][mt][j + 2] * inv);
                    }
                } else {
                    const int64_t pi = sh * a.num_partitions + U.p;
                    float* row = a.ws_o + pi * D;
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        row[mt * 16 + g] = o[nt][mt][j];
                        row[mt * 16 + g + 8] = o[nt][mt][j + 2];
                    }
                    if (g == 0) {
                        a.ws_m[pi] = m[nt][j];
                        a.ws_l[pi] = l;
                    }
                }
            }
    }
};

}  // namespace pa
