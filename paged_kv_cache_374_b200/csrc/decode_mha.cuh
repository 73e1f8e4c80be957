// CUDA-core compute policy of the decode engine: one unit = one query head.
//
// Per stage of TOK tokens (fp32 arithmetic), for softmax(scale * q K^T) V with one
// softmax over all of a sequence's tokens (P1 "大模型部署中的PagedAttention：KV
// Cache显存管理突破", §1, first formula):
//   - lane = c * 8 + r owns dims [c*DL, (c+1)*DL) and token rows r, r+8, ... of the
//     stage, so a row's dot product is split over the 4 lanes with the same r;
//     the tiles are 128-byte swizzled half rows, so the 16-byte shared loads of 8
//     consecutive rows hit all 32 banks once;
//   - partial dot products (packed fp32x2 FMAs) are reduced over those 4 lanes
//     with a reduce-scatter of warp shuffles;
//   - online softmax in base 2 (log2(e) folded into the pre-scaled q): the
//     warp-wide max and the rescale of o run only when some score exceeds the
//     running max, which one warp vote decides;
//   - o += p * V with packed fp32x2 FMAs.
// Rows past the sequence end get score -inf and their V rows are skipped (not
// multiplied by 0: they may hold NaN).
#pragma once

#include "decode_engine.cuh"

namespace pa {

// Tag: q / out element type; CTag: cache element type (16-bit, or E4M3 codes whose
// scales are folded into q (k_scale) and into the result (v_scale)).
template <class Tag, class CTag, int D, int TOK>
struct MhaPolicy {
    static constexpr int DL = D / 4;       // dims per lane
    static constexpr int EPC = 16 / CTag::kBytes;  // cache elements per 16-byte chunk
    static constexpr int NCH = DL / EPC;   // 16-byte chunks per lane per row
    static constexpr int NROW = TOK / 8;   // rows per lane per stage
    static_assert(NROW == 1 || NROW == 2 || NROW == 4, "stage shape");
    static constexpr int DUP = 4 / NROW;   // lanes that end up holding one token's score
    static constexpr int HALF_BYTES = TOK * 128;

    // fp8 codes: q K^T as f32 += f16 * f16 (sm_100 mixed-precision fma) on f16 q pairs and
    // the exactly widened codes; the scale is applied to the sum.  fp16 q enters as it is;
    // bf16 q as f16 q * 2^k, with 2^k chosen per unit from its largest |q| (exact for every
    // element above 2^-31 of that one) and 2^-k applied to the sum with the scale.
    static constexpr bool kMixed = CTag::kBytes == 1;

    int lane, r, c;
    int swz[NCH];       // offset of this lane's chunk j of row r in a tile
    uint4 qn[DL / 8];   // raw q of the next unit
    float2 qc[DL / 2];  // q of the current unit, pre-scaled by scale * log2(e)
    uint32_t qh[DL / 2];  // kMixed: q of the current unit as f16 pairs (times 2^k for bf16 q)
    float qinv;           // kMixed: 2^-k
    float m, lsum;
    float2 o[DL / 2];
    bool poisoned;

    static constexpr int kScratchBytes = 0;

    __device__ __forceinline__ void setup(int lane_, uint8_t* /*scratch*/) {
        lane = lane_;
        r = lane & 7;
        c = lane >> 3;
        const int lane_byte = c * DL * CTag::kBytes;  // this lane's first byte in a row
        const int lane_half = lane_byte / 128;
        const int chunk0 = (lane_byte % 128) / 16;
#pragma unroll
        for (int j = 0; j < NCH; ++j) swz[j] = lane_half * HALF_BYTES + r * 128 + (((chunk0 + j) ^ r) << 4);
    }

    __device__ __forceinline__ void fetch_q(const DecodeArgs& a, const Unit& U) {
        if (U.kind != kUnitNormal) return;
        const uint4* src = reinterpret_cast<const uint4*>(a.q + ((int64_t)U.s * a.num_heads + U.h) * D + c * DL);
#pragma unroll
        for (int j = 0; j < DL / 8; ++j) qn[j] = __ldg(src + j);
    }

    __device__ __forceinline__ void take_q(const DecodeArgs& a) {
        if constexpr (kMixed) {
            if constexpr (Tag::kIsBF16) {
                // lanes with the same c hold the same dims: the max over lane bits 3 and 4 covers the head
                float mx = 0.f;
#pragma unroll
                for (int j = 0; j < DL / 8; ++j) {
                    const uint32_t w[4] = {qn[j].x, qn[j].y, qn[j].z, qn[j].w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 v = BF16Tag::widen2(w[k]);
                        mx = fmaxf(mx, fmaxf(fabsf(v.x), fabsf(v.y)));
                    }
                }
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 16));
                float s;
                f16_entry_scale(mx, s, qinv);
#pragma unroll
                for (int j = 0; j < DL / 8; ++j) {
                    const uint32_t w[4] = {qn[j].x, qn[j].y, qn[j].z, qn[j].w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const float2 v = BF16Tag::widen2(w[k]);
                        qh[4 * j + k] = pack_f16x2(v.x * s, v.y * s);
                    }
                }
            } else {
                qinv = 1.f;
#pragma unroll
                for (int j = 0; j < DL / 8; ++j) {
                    qh[4 * j] = qn[j].x;
                    qh[4 * j + 1] = qn[j].y;
                    qh[4 * j + 2] = qn[j].z;
                    qh[4 * j + 3] = qn[j].w;
                }
            }
            return;
        }
        const float sc = a.scale_log2 * a.k_scale;
#pragma unroll
        for (int j = 0; j < DL / 8; ++j) {
            float2 f[4];
            widen8<Tag>(qn[j], f);
#pragma unroll
            for (int k = 0; k < 4; ++k) qc[j * 4 + k] = make_float2(f[k].x * sc, f[k].y * sc);
        }
    }

    // the EPC cache values of a 16-byte chunk as EPC/2 float pairs
    static __device__ __forceinline__ void widen_chunk(const uint4& w, float2 (&f)[EPC / 2]) {
        if constexpr (CTag::kBytes == 2) {
            widen8<CTag>(w, f);
        } else {
            const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                f[2 * k] = CTag::widen2(words[k] & 0xffffu);
                f[2 * k + 1] = CTag::widen2(words[k] >> 16);
            }
        }
    }

    __device__ __forceinline__ void reset() {
        m = -INFINITY;
        lsum = 0.f;
#pragma unroll
        for (int k = 0; k < DL / 2; ++k) o[k] = make_float2(0.f, 0.f);
        poisoned = false;
    }

    __device__ __forceinline__ void poison() { poisoned = true; }

    // acc + lo(a) lo(b) + hi(a) hi(b) for two f16 pairs, accumulated in f32
    static __device__ __forceinline__ float2 fma_f16x2(uint32_t a2, uint32_t b2, float2 acc) {
        float2 d;
        asm("{\n\t.reg .f16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %2;\n\tmov.b32 {bl, bh}, %3;\n\t"
            "fma.rn.f32.f16 %0, al, bl, %4;\n\tfma.rn.f32.f16 %1, ah, bh, %5;\n\t}"
            : "=f"(d.x), "=f"(d.y)
            : "r"(a2), "r"(b2), "f"(acc.x), "f"(acc.y));
        return d;
    }

    __device__ __forceinline__ void stage(const DecodeArgs& a, const uint8_t* kt, const uint8_t* vt, int ntok) {
        // partial dot products of rows i*8 + r over this lane's dims
        float acc[NROW];
        float sum_scale = 1.f;
        if constexpr (kMixed) sum_scale = a.scale_log2 * a.k_scale * qinv;
#pragma unroll
        for (int i = 0; i < NROW; ++i) {
            float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int j = 0; j < NCH; ++j) {
                const uint4 w = *reinterpret_cast<const uint4*>(kt + i * 1024 + swz[j]);
                if constexpr (kMixed) {
                    const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        d2 = fma_f16x2(qh[j * 8 + 2 * k], E4M3Tag::to_f16x2(words[k] & 0xffffu), d2);
                        d2 = fma_f16x2(qh[j * 8 + 2 * k + 1], E4M3Tag::to_f16x2(words[k] >> 16), d2);
                    }
                } else {
                    float2 kf[EPC / 2];
                    widen_chunk(w, kf);
#pragma unroll
                    for (int k = 0; k < EPC / 2; ++k) d2 = __ffma2_rn(qc[j * (EPC / 2) + k], kf[k], d2);
                }
            }
            acc[i] = d2.x + d2.y;
            if constexpr (kMixed) acc[i] *= sum_scale;
        }
        // reduce over the 4 lanes of a row (lane bits 4 and 3), scattering the
        // NROW rows so that lane c keeps row group g(c)
#pragma unroll
        for (int width = NROW, mask = 16; width > 1; width >>= 1, mask >>= 1) {
            const int half = width >> 1;
            const bool upper = (lane & mask) != 0;
#pragma unroll
            for (int j = 0; j < half; ++j) {
                const float keep = upper ? acc[j + half] : acc[j];
                const float send = upper ? acc[j] : acc[j + half];
                acc[j] = keep + __shfl_xor_sync(kFullMask, send, mask);
            }
        }
        float x = acc[0];
        if (NROW == 1) {
            x += __shfl_xor_sync(kFullMask, x, 16);
            x += __shfl_xor_sync(kFullMask, x, 8);
        } else if (NROW == 2) {
            x += __shfl_xor_sync(kFullMask, x, 8);
        }
        const int g = NROW == 4 ? c : (NROW == 2 ? (c >> 1) : 0);
        if (g * 8 + r >= ntok) x = -INFINITY;
        // the warp-wide max and the rescale of o are needed only when some score
        // exceeds the running max
        if (__any_sync(kFullMask, x > m)) {
            const float m_new = fmaxf(m, warp_max(x));
            const float alpha = fast_exp2(m - m_new);
            lsum *= alpha;
            const float2 al2 = make_float2(alpha, alpha);
#pragma unroll
            for (int k = 0; k < DL / 2; ++k) o[k] = __fmul2_rn(o[k], al2);
            m = m_new;
        }
        const float p = fast_exp2(x - m);
        lsum += p;
        // o += p_row * V_row for the rows this lane covers
#pragma unroll
        for (int i = 0; i < NROW; ++i) {
            const float pr = __shfl_sync(kFullMask, p, (i * DUP) * 8 + r);
            if (i * 8 + r < ntok) {
                const float2 p2 = make_float2(pr, pr);
#pragma unroll
                for (int j = 0; j < NCH; ++j) {
                    const uint4 w = *reinterpret_cast<const uint4*>(vt + i * 1024 + swz[j]);
                    float2 vf[EPC / 2];
                    widen_chunk(w, vf);
#pragma unroll
                    for (int k = 0; k < EPC / 2; ++k) o[j * (EPC / 2) + k] = __ffma2_rn(p2, vf[k], o[j * (EPC / 2) + k]);
                }
            }
        }
    }

    __device__ __forceinline__ void finish(const DecodeArgs& a, const Unit& U) {
        const int64_t sh = (int64_t)U.s * a.num_heads + U.h;
        // fold the 8 row classes r; each token's p sits on DUP lanes
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
#pragma unroll
            for (int k = 0; k < DL / 2; ++k) {
                o[k].x += __shfl_xor_sync(kFullMask, o[k].x, off);
                o[k].y += __shfl_xor_sync(kFullMask, o[k].y, off);
            }
        }
        float l = warp_sum(lsum) * (1.f / DUP);
        if (__any_sync(kFullMask, poisoned)) l = __int_as_float(0x7fc00000);
        if (CTag::kBytes == 1) {
#pragma unroll
            for (int k = 0; k < DL / 2; ++k) o[k] = make_float2(o[k].x * a.v_scale, o[k].y * a.v_scale);
        }
        if (U.np == 1) {
            if (r == 0) {
                const float inv = 1.f / l;
                uint4* dst = reinterpret_cast<uint4*>(a.out + sh * D + c * DL);
#pragma unroll
                for (int j = 0; j < DL / 8; ++j) {
                    uint4 w;
                    w.x = pack2<Tag>(o[j * 4 + 0].x * inv, o[j * 4 + 0].y * inv);
                    w.y = pack2<Tag>(o[j * 4 + 1].x * inv, o[j * 4 + 1].y * inv);
                    w.z = pack2<Tag>(o[j * 4 + 2].x * inv, o[j * 4 + 2].y * inv);
                    w.w = pack2<Tag>(o[j * 4 + 3].x * inv, o[j * 4 + 3].y * inv);
                    dst[j] = w;
                }
            }
        } else {
            const int64_t pi = sh * a.num_partitions + U.p;
            if (r == 0) {
                float4* dst = reinterpret_cast<float4*>(a.ws_o + pi * D + c * DL);
#pragma unroll
                for (int k = 0; k < DL / 4; ++k)
                    dst[k] = make_float4(o[2 * k].x, o[2 * k].y, o[2 * k + 1].x, o[2 * k + 1].y);
            }
            if (lane == 0) {
                a.ws_m[pi] = m;
                a.ws_l[pi] = l;
            }
        }
    }
};

}  // namespace pa
