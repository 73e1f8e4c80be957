// Tensor-core compute policy for fp8 (E4M3) caches: one unit = one kv head with
// its whole group of query heads, as on the 16-bit GQA path.  Each landed stage of
// codes is widened, 16 tokens at a time, in the warp's own
// shared scratch, into the 16-bit 128-byte-swizzled tiles the GQA policy reads
// (E4M3 -> f16 is exact, and so is f16 -> bf16 for these values); then q K^T and
// V^T P^T run as mma.sync on them.  The K scale multiplies the scores and the V
// scale the output, as on the CUDA-core fp8 path.  One fetch of a token's K/V
// rows serves every query head of the group, and the conversion plus a few MMAs
// replace the per-element widening and FMAs of the CUDA-core path.
#pragma once

#include "decode_gqa.cuh"

namespace pa {

// TOK: tokens per landed stage of codes (16 or 32); they are widened and computed
// 16 at a time, through one 16-token scratch tile pair.
template <class Tag, int TOK, int NT>
struct Fp8TcPolicy {
    static constexpr int D = 128;                      // one 128-byte code row per token
    static constexpr int TI = 16;                      // tokens per widened tile
    static_assert(TOK % TI == 0, "stage shape");
    static constexpr int kTile16 = 2 * TI * 128;       // a 16-bit tile: two 64-dim halves
    static constexpr int kScratchBytes = 2 * kTile16;  // K then V
    static_assert(kScratchBytes % 1024 == 0, "scratch tiles keep the 1 KiB swizzle alignment");
    using Inner = GqaPolicy<Tag, D, TI, NT>;

    Inner in;
    uint8_t* scr;
    int lane;

    __device__ __forceinline__ void setup(int lane_, uint8_t* scratch) {
        lane = lane_;
        scr = scratch;
        in.setup(lane_, nullptr);
    }
    __device__ __forceinline__ void fetch_q(const DecodeArgs& a, const Unit& U) { in.fetch_q(a, U); }
    __device__ __forceinline__ void take_q(const DecodeArgs& a) { in.take_q(a); }
    __device__ __forceinline__ void reset() { in.reset(); }
    __device__ __forceinline__ void poison() { in.poison(); }
    __device__ __forceinline__ void finish(const DecodeArgs& a, const Unit& U) { in.finish(a, U); }

    // two codes (low byte first) -> two Tag values, low half first
    static __device__ __forceinline__ uint32_t widen_pair(uint32_t pair16) {
        const uint32_t h = E4M3Tag::to_f16x2(pair16);
        if constexpr (Tag::kIsBF16) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
            return MmaOps<Tag>::pack(f.x, f.y);  // exact: the codes are representable in bf16
        } else {
            return h;
        }
    }

    __device__ __forceinline__ void stage(const DecodeArgs& a, const uint8_t* kt, const uint8_t* vt, int ntok) {
#pragma unroll 1
        for (int t0 = 0; t0 < TOK && t0 < ntok; t0 += TI) {
            // 16-byte code chunk c (dims 16c .. 16c+15) of row r sits at r*128 + ((c ^ r%8) << 4); its two
            // 8-dim halves go to chunks 2c, 2c+1 (mod 8) of 16-bit half c/4, same swizzle (t0 is a
            // multiple of 8, so the phase r % 8 is unchanged).  The previous tile's ldmatrix reads of the
            // scratch completed before this warp got here.
            __syncwarp();
#pragma unroll
            for (int i = 0; i < (2 * TI * 8) / 32; ++i) {
                const int idx = i * 32 + lane;
                const int tile = idx / (TI * 8), rem = idx % (TI * 8), r = rem >> 3, c = rem & 7;
                const uint4 w =
                    *reinterpret_cast<const uint4*>((tile ? vt : kt) + (t0 + r) * 128 + ((c ^ (r & 7)) << 4));
                const uint32_t words[4] = {w.x, w.y, w.z, w.w};
                uint32_t h[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    h[2 * k] = widen_pair(words[k] & 0xffffu);
                    h[2 * k + 1] = widen_pair(words[k] >> 16);
                }
                uint8_t* row = scr + tile * kTile16 + (c >> 2) * (TI * 128) + r * 128;
                const int j = (2 * c) & 7;
                *reinterpret_cast<uint4*>(row + ((j ^ (r & 7)) << 4)) = make_uint4(h[0], h[1], h[2], h[3]);
                *reinterpret_cast<uint4*>(row + (((j + 1) ^ (r & 7)) << 4)) = make_uint4(h[4], h[5], h[6], h[7]);
            }
            __syncwarp();
            in.stage(a, scr, scr + kTile16, ntok - t0);
        }
    }
};

}  // namespace pa
