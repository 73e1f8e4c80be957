// K2 + K3: single-query (decode) attention over the paged KV cache.
//
// What is computed (P1 "大模型部署中的PagedAttention：KV Cache显存管理突破", §1, first
// formula; P3 "LLM 推理中的 PageAttention 实现原理", §二 and §三): for sequence s and
// query head h, out = softmax(scale * q K^T) V over the sequence's L tokens taken
// in logical order, token t living in physical block block_tables[s][t / B] at
// offset t % B -- one softmax over all L tokens.
//
// Units of work.  A sequence is cut into partitions of P tokens; a unit is one
// (sequence, partition, query head).  A sequence of one partition gets its output
// row directly; a longer one leaves a partial result per partition (running max m,
// running sum l, unnormalised o) in the workspace, merged by K3.
//
// K2 is persistent: one CTA per SM, NW warps per CTA, and every warp is a
// self-contained streaming engine -- it claims units from a global counter, loads
// the unit's block-table entries with one coalesced warp load per 32 entries
// (each entry is read once, by one warp), and keeps its own ring of R
// shared-memory slots filled with TMA tensor copies (cp.async.bulk.tensor; one
// slot = K and V of TOK tokens of one kv head), completion tracked by one
// mbarrier per slot.  Issue runs R stages ahead of compute and crosses into the
// next claimed unit before the current one ends, so the warp's copies never drain
// at unit boundaries.  No warp ever waits for another.
//
// Claim order: every full partition first (sequence-major, query heads fastest, so
// warps running together read the same physical blocks), then each sequence's
// last partition, longest first, so that the units left at the end are the
// shortest.  Every CTA derives the same order from context_lens in its prologue.
//
// Per stage (fp32 arithmetic): a token row is split over CH lanes (one 16-byte
// chunk each); partial dot products are reduced by a reduce-scatter over warp
// shuffles, then the online softmax update (running max / sum, base-2 exponentials
// with log2(e) folded into the pre-scaled q) and p * V accumulate with packed
// fp32x2 FMAs.  Rows past the sequence end inside the last block are never used:
// their scores become -inf and their V rows are skipped (not multiplied by 0, as
// they may hold NaN).  Table entries outside [0, num_blocks) are never
// dereferenced: the stage is dropped, the output row becomes NaN and
// PA_DEVERR_TABLE_RANGE is set.
#include <cmath>

#include "pa_device.cuh"
#include "pa_host.h"

// Tile configuration (compile-time; the defaults are the tuned ones).
#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 12       // warps (streaming engines) per CTA, one CTA per SM
#endif
#ifndef PA_DECODE_SLOTS
#define PA_DECODE_SLOTS 2        // shared-memory slots per warp
#endif
#ifndef PA_DECODE_TOK128
#define PA_DECODE_TOK128 16      // tokens per slot at head_dim 128
#endif
#ifndef PA_DECODE_TOK64
#define PA_DECODE_TOK64 32       // tokens per slot at head_dim 64
#endif
#ifndef PA_DECODE_PARTITION
#define PA_DECODE_PARTITION 256  // default context partition, tokens
#endif

namespace pa {

constexpr int kMaxSeqsPerLaunch = 1024;   // sequences scheduled by one K2 launch
constexpr int kMaxPartitionTokens = 65536;

struct DecodeArgs {
    const uint16_t* q;
    uint16_t* out;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* ws_m;      // [S*H][Pmax], base-2 units
    float* ws_l;      // [S*H][Pmax]
    float* ws_o;      // [S*H][Pmax][D]
    int32_t* sched;   // [0] claim counter, [1] finished-warp counter; zero between launches
    int32_t* err_word;
    float scale_log2; // scale * log2(e)
    int num_seqs;     // sequences in this launch (<= kMaxSeqsPerLaunch)
    int num_heads;
    int group;        // num_heads / num_kv_heads
    int block_size;
    int box_rows;     // token rows per TMA box (min(TOK, block_size))
    int num_blocks;
    int max_blocks_per_seq;
    int partition_tokens;
    int num_partitions;  // Pmax: partitions allotted per (s, h) in the workspace
};

enum UnitKind { kUnitNone = 0, kUnitNormal = 1, kUnitZero = 2, kUnitNaN = 3 };

struct Unit {
    int kind;
    int s, h, p, np;
    int t_begin, t_end, nst, kv_head, blk0, nblk;
};

template <int D, int TOK, int NW, int R>
struct Layout {
    static constexpr int kTileBytes = TOK * D * 2;
    static constexpr int kSlotBytes = 2 * kTileBytes;          // K tile then V tile
    static constexpr int kOffSlots = 0;
    static constexpr int kOffBars = NW * R * kSlotBytes;
    static constexpr int kOffCum = kOffBars + NW * R * 8;         // int[S + 1]
    static constexpr int kOffKey = kOffCum + (kMaxSeqsPerLaunch + 1) * 4 + 12;  // uint32[S_pow2]
    static constexpr int kOffLen = kOffKey + kMaxSeqsPerLaunch * 4;            // int[S]
    static constexpr int kBytes = kOffLen + kMaxSeqsPerLaunch * 4;
    static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1 KiB
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <class Tag>
__device__ __forceinline__ void widen8(const uint4& w, float2 (&f)[4]) {
    f[0] = Tag::widen2(w.x);
    f[1] = Tag::widen2(w.y);
    f[2] = Tag::widen2(w.z);
    f[3] = Tag::widen2(w.w);
}

template <class Tag>
__device__ __forceinline__ uint32_t pack2(float a, float b) {
    return (uint32_t)Tag::round1(a) | ((uint32_t)Tag::round1(b) << 16);
}

// Decode claim index u into a unit (warp-uniform; reads the schedule in smem).
__device__ __forceinline__ Unit decode_unit(int u, const DecodeArgs& a, const int* s_cum, const uint32_t* s_key,
                                            const int* s_len, int TOK) {
    Unit U;
    const int S = a.num_seqs, H = a.num_heads;
    const int A = s_cum[S];
    if (u < 0 || u >= H * (A + S)) {
        U.kind = kUnitNone;
        U.s = U.h = U.p = U.np = U.t_begin = U.t_end = U.nst = U.kv_head = U.blk0 = U.nblk = 0;
        return U;
    }
    int s, p, h;
    if (u < H * A) {
        const int idx = u / H;
        h = u - idx * H;
        int lo = 0, hi = S - 1;  // largest s with s_cum[s] <= idx
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s_cum[mid] <= idx) lo = mid; else hi = mid - 1;
        }
        s = lo;
        p = idx - s_cum[s];
    } else {
        const int v = u - H * A;
        const int idx = v / H;
        h = v - idx * H;
        s = (int)(s_key[idx] & 0xfffu);
        p = s_cum[s + 1] - s_cum[s];
    }
    U.s = s;
    U.h = h;
    U.p = p;
    U.np = s_cum[s + 1] - s_cum[s] + 1;
    const int L = s_len[s];
    const int maxlen = a.max_blocks_per_seq * a.block_size;
    U.kind = (L < 0 || L > maxlen) ? kUnitNaN : (L == 0 ? kUnitZero : kUnitNormal);
    const int P = a.partition_tokens;
    U.t_begin = p * P;
    U.t_end = U.kind == kUnitNormal ? min(L, U.t_begin + P) : U.t_begin;
    U.nst = (U.t_end - U.t_begin + TOK - 1) / TOK;
    U.kv_head = h / a.group;
    U.blk0 = U.t_begin / a.block_size;
    U.nblk = U.kind == kUnitNormal ? (U.t_end + a.block_size - 1) / a.block_size - U.blk0 : 0;
    return U;
}

template <class Tag, int D, int TOK, int NW, int R>
__global__ void __launch_bounds__(NW * 32, 1) paged_decode_kernel(const DecodeArgs a,
                                                                  const __grid_constant__ CUtensorMap kmap,
                                                                  const __grid_constant__ CUtensorMap vmap) {
    using Lay = Layout<D, TOK, NW, R>;
    // Lane layout for a stage of TOK tokens held as swizzled 128-byte half rows:
    // lane = c * 8 + r.  Lane (c, r) owns dims [c*DL, (c+1)*DL) and token rows
    // r, r + 8, ... of the stage, so a row's dot product is split over the 4 lanes
    // with the same r (lanes r, r+8, r+16, r+24).
    constexpr int DL = D / 4;          // dims per lane
    constexpr int NCH = DL / 8;        // 16-byte chunks per lane per row
    constexpr int NROW = TOK / 8;      // rows per lane per stage
    static_assert(NROW == 1 || NROW == 2 || NROW == 4, "stage shape");
    constexpr int DUP = 4 / NROW;      // lanes that end up holding one token's score
    constexpr int HALF_BYTES = TOK * 128;   // one 64-dim half tile
    constexpr int MAXSUB = TOK / 8 > 2 ? 2 : 1;  // TMA boxes per half tile (box_rows >= TOK/2)
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    int* s_cum = reinterpret_cast<int*>(smem + Lay::kOffCum);
    uint32_t* s_key = reinterpret_cast<uint32_t*>(smem + Lay::kOffKey);
    int* s_len = reinterpret_cast<int*>(smem + Lay::kOffLen);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = a.num_seqs;
    const int H = a.num_heads;
    const int P = a.partition_tokens;
    const int bs = a.block_size;
    const int maxlen = a.max_blocks_per_seq * bs;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kOffBars) + warp * R;
    uint8_t* slots = smem + Lay::kOffSlots + warp * R * Lay::kSlotBytes;

    // ------------------------------------------------------------- prologue
    int spow = 1;
    while (spow < S) spow <<= 1;
    for (int s = threadIdx.x; s < spow; s += blockDim.x) {
        if (s < S) {
            const int L = a.context_lens[s];
            s_len[s] = L;
            const bool normal = L > 0 && L <= maxlen;
            const int np = normal ? (L + P - 1) / P : 1;
            const int last = normal ? L - (np - 1) * P : 0;
            s_cum[s] = np - 1;  // full partitions, scanned below
            s_key[s] = ((uint32_t)(P - last) << 12) | (uint32_t)s;
        } else {
            s_key[s] = 0xffffffffu;
        }
    }
    if (lane == 0) {
        for (int i = 0; i < R; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scan of the full-partition counts; s_cum[S] = total
        const int per = (S + 31) / 32;
        const int b = min(S, lane * per), e = min(S, b + per);
        int local = 0;
        for (int i = b; i < e; ++i) local += s_cum[i];
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(FULL, incl, o);
            if (lane >= o) incl += y;
        }
        int run = incl - local;
        for (int i = b; i < e; ++i) {
            const int v = s_cum[i];
            s_cum[i] = run;
            run += v;
        }
        if (lane == 31) s_cum[S] = incl;
    }
    // bitonic sort of the last-partition keys: (P - size) ascending, then s
    for (int k = 2; k <= spow; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < spow; i += blockDim.x) {
                const int ixj = i ^ j;
                if (ixj > i) {
                    const uint32_t x = s_key[i], y = s_key[ixj];
                    if ((x > y) == ((i & k) == 0)) {
                        s_key[i] = y;
                        s_key[ixj] = x;
                    }
                }
            }
            __syncthreads();
        }
    }
    __syncthreads();

    // ------------------------------------------------------------ warp engine
    const int r = lane & 7;
    const int c = lane >> 3;
    // shared-memory offset of this lane's chunk j of row (i*8 + r) in a K or V tile:
    // half tile of the lane's dims, the row, and the swizzled 16-byte chunk
    const int lane_half = (D == 128) ? (c >> 1) : 0;
    const int chunk0 = (D == 128) ? (c & 1) * 4 : c * 2;
    int swz[NCH];
#pragma unroll
    for (int j = 0; j < NCH; ++j) swz[j] = lane_half * HALF_BYTES + r * 128 + (((chunk0 + j) ^ r) << 4);
    int32_t* claim_ctr = a.sched;

    auto claim = [&]() -> int { return lane == 0 ? atomicAdd(claim_ctr, 1) : 0; };
    // q of a unit: fetched as raw 16-bit values, widened and pre-scaled on use
    auto fetch_q = [&](const Unit& U, uint4 (&raw)[NCH]) {
        if (U.kind != kUnitNormal) return;
        const uint4* src = reinterpret_cast<const uint4*>(a.q + ((int64_t)U.s * H + U.h) * D + c * DL);
#pragma unroll
        for (int j = 0; j < NCH; ++j) raw[j] = __ldg(src + j);
    };
    auto widen_q = [&](const uint4 (&raw)[NCH], float2 (&qv)[DL / 2]) {
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
            float2 f[4];
            widen8<Tag>(raw[j], f);
#pragma unroll
            for (int k = 0; k < 4; ++k) qv[j * 4 + k] = make_float2(f[k].x * a.scale_log2, f[k].y * a.scale_log2);
        }
    };
    auto load_tab = [&](const Unit& U, int chunk) -> int {
        const int idx = chunk * 32 + lane;
        return (U.kind == kUnitNormal && idx < U.nblk)
                   ? __ldg(a.block_tables + (int64_t)U.s * a.max_blocks_per_seq + U.blk0 + idx)
                   : -1;
    };

    // current unit C (being consumed), next unit N, and a pending raw claim
    Unit C = decode_unit(__shfl_sync(FULL, claim(), 0), a, s_cum, s_key, s_len, TOK);
    Unit N = decode_unit(__shfl_sync(FULL, claim(), 0), a, s_cum, s_key, s_len, TOK);
    int pend = claim();
    float2 qc[DL / 2];
    uint4 qn[NCH];
    {
        uint4 q0[NCH];
        fetch_q(C, q0);
        widen_q(q0, qc);
    }
    fetch_q(N, qn);
    int ntab0 = load_tab(N, 0), ntab1 = load_tab(N, 1);
    // issue cursor: in C (in_next = false) or N; its rolling table chunk pair
    bool in_next = false;
    int ist = 0;
    int ichunk = 0, itab_cur = load_tab(C, 0), itab_nxt = load_tab(C, 1);
    uint32_t issued = 0, consumed = 0;
    uint32_t badmask = 0;  // slots whose stage was dropped for a bad table entry
    bool aborted = false;

    // softmax state of C (m is warp-uniform, base-2 units)
    float m = -INFINITY, lsum = 0.f;
    float2 o[DL / 2];
#pragma unroll
    for (int k = 0; k < DL / 2; ++k) o[k] = make_float2(0.f, 0.f);
    bool poisoned = false;
    int cst = 0;

    auto issue_stage = [&](const Unit& I, int st) {
        const int slot = issued % R;
        const int t0 = I.t_begin + st * TOK;
        const int br = a.box_rows;
        const int first_e = t0 / bs - I.blk0;
        while ((first_e >> 5) > ichunk) {  // roll the table window forward
            ++ichunk;
            itab_cur = itab_nxt;
            itab_nxt = load_tab(I, ichunk + 1);
        }
        int phys[MAXSUB];
        bool bad = false;
        uint32_t tx = 0;
#pragma unroll
        for (int j = 0; j < MAXSUB; ++j) {
            const int tj = t0 + j * br;
            const bool use = j * br < TOK && tj < I.t_end;
            const int e = tj / bs - I.blk0;
            const int v = (e >> 5) == ichunk ? itab_cur : itab_nxt;
            phys[j] = __shfl_sync(FULL, v, e & 31);
            if (use) {
                bad |= phys[j] < 0 || phys[j] >= a.num_blocks;
                tx += 2u * br * D * 2;
            }
        }
        uint8_t* dst = slots + slot * Lay::kSlotBytes;
        if (bad) badmask |= 1u << slot;
        if (lane == 0) {
            if (bad) {
                report(a.err_word, PA_DEVERR_TABLE_RANGE);
                mbar_arrive(&bars[slot]);
            } else {
                fence_proxy_async_shared();  // our earlier reads of this slot come first
                mbar_arrive_expect_tx(&bars[slot], tx);
#pragma unroll
                for (int j = 0; j < MAXSUB; ++j) {
                    const int tj = t0 + j * br;
                    if (j * br < TOK && tj < I.t_end) {
                        const int row = phys[j] * bs + (tj % bs);
#pragma unroll
                        for (int hh = 0; hh < D / 64; ++hh) {
                            uint8_t* kd = dst + hh * HALF_BYTES + j * br * 128;
                            tma_load_3d(kd, &kmap, hh * 64, I.kv_head, row, &bars[slot]);
                            tma_load_3d(kd + Lay::kTileBytes, &vmap, hh * 64, I.kv_head, row, &bars[slot]);
                        }
                    }
                }
            }
        }
        ++issued;
    };

    auto finish_unit = [&](const Unit& U) {
        const int64_t sh = (int64_t)U.s * H + U.h;
        if (U.kind == kUnitZero || U.kind == kUnitNaN) {
            if (lane < D / 8) {
                const uint32_t w = U.kind == kUnitZero ? 0u : pack2<Tag>(__int_as_float(0x7fc00000),
                                                                          __int_as_float(0x7fc00000));
                reinterpret_cast<uint4*>(a.out + sh * D)[lane] = make_uint4(w, w, w, w);
            }
            if (U.kind == kUnitNaN && lane == 0) report(a.err_word, PA_DEVERR_LEN_RANGE);
            return;
        }
        // fold the 8 row classes r; each token's p sits on DUP lanes
#pragma unroll
        for (int off = 1; off < 8; off <<= 1) {
#pragma unroll
            for (int k = 0; k < DL / 2; ++k) {
                o[k].x += __shfl_xor_sync(FULL, o[k].x, off);
                o[k].y += __shfl_xor_sync(FULL, o[k].y, off);
            }
        }
        float l = warp_sum(lsum) * (1.f / DUP);
        if (__any_sync(FULL, poisoned)) l = __int_as_float(0x7fc00000);
        if (U.np == 1) {
            if (r == 0) {
                const float inv = 1.f / l;
                uint4* dst = reinterpret_cast<uint4*>(a.out + sh * D + c * DL);
#pragma unroll
                for (int j = 0; j < NCH; ++j) {
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
    };

    while (C.kind != kUnitNone && !aborted) {
        if (C.kind != kUnitNormal || C.nst == 0) {
            finish_unit(C);
        } else {
            // keep R stages in flight: C's remaining stages, then N's
            while (issued - consumed < (uint32_t)R) {
                if (!in_next) {
                    if (ist < C.nst) {
                        issue_stage(C, ist++);
                        continue;
                    }
                    if (N.kind != kUnitNormal) break;
                    in_next = true;
                    ist = 0;
                    ichunk = 0;
                    itab_cur = ntab0;
                    itab_nxt = ntab1;
                }
                if (ist < N.nst) issue_stage(N, ist++);
                else break;
            }
            // consume one stage of C
            const int slot = consumed % R;
            const bool ok = __all_sync(FULL, mbar_wait(&bars[slot], (consumed / R) & 1));
            if (!ok) {
                if (lane == 0) report(a.err_word, PA_DEVERR_TIMEOUT);
                aborted = true;
                break;
            }
            if ((badmask >> slot) & 1u) {
                poisoned = true;
                badmask &= ~(1u << slot);
            } else {
                const int ntok = min(TOK, C.t_end - (C.t_begin + cst * TOK));
                const uint8_t* kt = slots + slot * Lay::kSlotBytes;
                const uint8_t* vt = kt + Lay::kTileBytes;
                // partial dot products of rows i*8 + r over this lane's dims
                float acc[NROW];
#pragma unroll
                for (int i = 0; i < NROW; ++i) {
                    float2 d2 = make_float2(0.f, 0.f);
#pragma unroll
                    for (int j = 0; j < NCH; ++j) {
                        const uint4 w = *reinterpret_cast<const uint4*>(kt + i * 1024 + swz[j]);
                        float2 kf[4];
                        widen8<Tag>(w, kf);
#pragma unroll
                        for (int k = 0; k < 4; ++k) d2 = __ffma2_rn(qc[j * 4 + k], kf[k], d2);
                    }
                    acc[i] = d2.x + d2.y;
                }
                // reduce over the 4 lanes of a row (lane bits 4 and 3), scattering
                // the NROW rows so that lane c keeps row group g(c)
#pragma unroll
                for (int width = NROW, mask = 16; width > 1; width >>= 1, mask >>= 1) {
                    const int half = width >> 1;
                    const bool upper = (lane & mask) != 0;
#pragma unroll
                    for (int j = 0; j < half; ++j) {
                        const float keep = upper ? acc[j + half] : acc[j];
                        const float send = upper ? acc[j] : acc[j + half];
                        acc[j] = keep + __shfl_xor_sync(FULL, send, mask);
                    }
                }
                float x = acc[0];
                if (NROW == 1) {
                    x += __shfl_xor_sync(FULL, x, 16);
                    x += __shfl_xor_sync(FULL, x, 8);
                } else if (NROW == 2) {
                    x += __shfl_xor_sync(FULL, x, 8);
                }
                const int g = NROW == 4 ? c : (NROW == 2 ? (c >> 1) : 0);
                if (g * 8 + r >= ntok) x = -INFINITY;
                // online softmax: the warp-wide max and the rescale of o are needed
                // only when some score exceeds the running max
                if (__any_sync(FULL, x > m)) {
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
                    const float pr = __shfl_sync(FULL, p, (i * DUP) * 8 + r);
                    if (i * 8 + r < ntok) {
                        const float2 p2 = make_float2(pr, pr);
#pragma unroll
                        for (int j = 0; j < NCH; ++j) {
                            const uint4 w = *reinterpret_cast<const uint4*>(vt + i * 1024 + swz[j]);
                            float2 vf[4];
                            widen8<Tag>(w, vf);
#pragma unroll
                            for (int k = 0; k < 4; ++k) o[j * 4 + k] = __ffma2_rn(p2, vf[k], o[j * 4 + k]);
                        }
                    }
                }
            }
            __syncwarp();
            ++consumed;
            if (++cst < C.nst) continue;
            finish_unit(C);
        }
        // rotate: N becomes current; decode the pending claim as the new N
        const bool issue_was_in_next = in_next;
        C = N;
        if (C.kind == kUnitNormal) widen_q(qn, qc);
        N = decode_unit(__shfl_sync(FULL, pend, 0), a, s_cum, s_key, s_len, TOK);
        fetch_q(N, qn);
        ntab0 = load_tab(N, 0);
        ntab1 = load_tab(N, 1);
        if (N.kind != kUnitNone) pend = claim();
        if (issue_was_in_next) {
            in_next = false;  // the issue cursor already runs inside the new C
        } else {
            in_next = false;
            ist = 0;
            ichunk = 0;
            itab_cur = load_tab(C, 0);
            itab_nxt = load_tab(C, 1);
        }
        m = -INFINITY;
        lsum = 0.f;
#pragma unroll
        for (int k = 0; k < DL / 2; ++k) o[k] = make_float2(0.f, 0.f);
        poisoned = false;
        cst = 0;
    }

    // never leave with copies into shared memory in flight
    for (uint32_t k = consumed; k < issued; ++k)
        if (!__all_sync(FULL, mbar_wait(&bars[k % R], (k / R) & 1)) && lane == 0)
            report(a.err_word, PA_DEVERR_TIMEOUT);
    // the last warp of the launch to finish puts the claim counters back to zero
    if (lane == 0) {
        __threadfence();
        const int total = (int)(gridDim.x * NW);
        if (atomicAdd(a.sched + 1, 1) == total - 1) {
            atomicExch(a.sched, 0);
            atomicExch(a.sched + 1, 0);
            __threadfence();
        }
    }
}

// K3: merge the partitions of each (s, h): M = max_p m_p,
// out = sum_p o_p 2^(m_p - M) / sum_p l_p 2^(m_p - M)  (scores are in base-2 units).
template <class Tag, int D>
__global__ void __launch_bounds__(D) paged_decode_merge_kernel(const DecodeArgs a) {
    const int64_t sh = blockIdx.x;
    const int s = (int)(sh / a.num_heads);
    const int L = a.context_lens[s];
    if (L <= 0 || L > a.max_blocks_per_seq * a.block_size) return;  // rows written by K2
    const int nparts = (L + a.partition_tokens - 1) / a.partition_tokens;
    if (nparts <= 1) return;
    const float* pm = a.ws_m + sh * a.num_partitions;
    const float* pl = a.ws_l + sh * a.num_partitions;
    const float* po = a.ws_o + sh * a.num_partitions * D;
    float M = -INFINITY;
    for (int p = 0; p < nparts; ++p) M = fmaxf(M, pm[p]);
    float den = 0.f, acc = 0.f;
    const int i = threadIdx.x;
    for (int p = 0; p < nparts; ++p) {
        const float w = pm[p] == -INFINITY ? 0.f : exp2f(pm[p] - M);
        den = fmaf(pl[p], w, den);
        acc = fmaf(po[(int64_t)p * D + i], w, acc);
    }
    a.out[sh * D + i] = Tag::round1(acc / den);
}

// ------------------------------------------------------------------------ host

namespace {

constexpr int kDefaultPartition = PA_DECODE_PARTITION;
constexpr size_t kSchedBytes = 256;

int64_t num_partitions(int max_blocks_per_seq, int block_size, int ptok) {
    const int64_t max_len = (int64_t)max_blocks_per_seq * block_size;
    return max_len <= 0 ? 1 : (max_len + ptok - 1) / ptok;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

size_t workspace_bytes_for(int64_t sh, int64_t P, int D) {
    if (P <= 1) return kSchedBytes;
    return kSchedBytes + up256(sh * P * 4) * 2 + up256(sh * P * D * 4);
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

template <class Tag, int D>
int launch_decode(DecodeArgs args, const void* k_cache, const void* v_cache, int num_kv_heads,
                  cudaStream_t stream) {
    constexpr int TOK = D == 128 ? PA_DECODE_TOK128 : PA_DECODE_TOK64;
    constexpr int NW = PA_DECODE_WARPS;
    constexpr int R = PA_DECODE_SLOTS;
    using Lay = Layout<D, TOK, NW, R>;
    static std::atomic<uint64_t> smem_done{0};
    auto kernel = paged_decode_kernel<Tag, D, TOK, NW, R>;
    if (ensure_smem_limit(kernel, Lay::kAlloc, smem_done) != cudaSuccess) return PA_ERR_CUDA;
    args.box_rows = TOK < args.block_size ? TOK : args.block_size;
    const int64_t total_tokens = (int64_t)args.num_blocks * args.block_size;
    CUtensorMap kmap, vmap;
    if (!encode_cache_map_swizzled(&kmap, k_cache, D, num_kv_heads, total_tokens, args.box_rows) ||
        !encode_cache_map_swizzled(&vmap, v_cache, D, num_kv_heads, total_tokens, args.box_rows))
        return PA_ERR_CUDA;
    const int sms = sm_count();
    if (sms <= 0) return PA_ERR_CUDA;
    const int total_seqs = args.num_seqs;
    for (int s0 = 0; s0 < total_seqs; s0 += kMaxSeqsPerLaunch) {
        DecodeArgs c = args;
        c.num_seqs = total_seqs - s0 < kMaxSeqsPerLaunch ? total_seqs - s0 : kMaxSeqsPerLaunch;
        const int64_t shoff = (int64_t)s0 * args.num_heads;
        c.q += shoff * D;
        c.out += shoff * D;
        c.block_tables += (int64_t)s0 * args.max_blocks_per_seq;
        c.context_lens += s0;
        if (args.num_partitions > 1) {
            c.ws_m += shoff * args.num_partitions;
            c.ws_l += shoff * args.num_partitions;
            c.ws_o += shoff * args.num_partitions * D;
        }
        kernel<<<sms, NW * 32, Lay::kAlloc, stream>>>(c, kmap, vmap);
        if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
        if (args.num_partitions > 1) {
            paged_decode_merge_kernel<Tag, D><<<(unsigned)((int64_t)c.num_seqs * args.num_heads), D, 0, stream>>>(c);
            if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
        }
    }
    return PA_OK;
}

}  // namespace
}  // namespace pa

extern "C" int pa_decode_partition_tokens(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                          int block_size, int max_blocks_per_seq) {
    (void)num_seqs; (void)num_heads; (void)num_kv_heads; (void)head_dim; (void)block_size;
    (void)max_blocks_per_seq;
    return pa::kDefaultPartition;
}

extern "C" size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                           int block_size, int max_blocks_per_seq, int partition_tokens) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        max_blocks_per_seq < 0 || partition_tokens < 0 || partition_tokens % 64 != 0 ||
        partition_tokens > pa::kMaxPartitionTokens)
        return 0;
    const int ptok = partition_tokens > 0
                         ? partition_tokens
                         : pa_decode_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                      max_blocks_per_seq);
    const int64_t P = pa::num_partitions(max_blocks_per_seq, block_size, ptok);
    return pa::workspace_bytes_for((int64_t)num_seqs * num_heads, P, head_dim);
}

extern "C" int pa_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                         const int32_t* context_lens, float scale, int num_kv_heads, void* out, int num_seqs,
                         int num_heads, int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                         int dtype, int partition_tokens, void* workspace, size_t workspace_bytes,
                         int32_t* err_word, void* stream) {
    using namespace pa;
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
        num_blocks <= 0 || max_blocks_per_seq <= 0 || partition_tokens < 0 || partition_tokens % 64 != 0 ||
        partition_tokens > kMaxPartitionTokens)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (block_size != 16 && block_size != 32 && block_size != 64) return PA_ERR_UNSUPPORTED;
    if ((int64_t)num_blocks * block_size > INT32_MAX || (int64_t)max_blocks_per_seq * block_size > INT32_MAX)
        return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PA_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out || !workspace)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        !aligned16(workspace) || !aligned4(block_tables) || !aligned4(context_lens) ||
        (err_word && !aligned4(err_word)))
        return PA_ERR_INVALID_ARG;
    const int ptok = partition_tokens > 0
                         ? partition_tokens
                         : pa_decode_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                      max_blocks_per_seq);
    const int64_t P = num_partitions(max_blocks_per_seq, block_size, ptok);
    // claim indices of one launch must fit in int32
    const int64_t chunk = num_seqs < kMaxSeqsPerLaunch ? num_seqs : kMaxSeqsPerLaunch;
    if ((int64_t)num_heads * chunk * (P + 1) > INT32_MAX) return PA_ERR_UNSUPPORTED;
    const int64_t SH = (int64_t)num_seqs * num_heads;
    const size_t need = workspace_bytes_for(SH, P, head_dim);
    if (workspace_bytes < need) return PA_ERR_INVALID_ARG;

    DecodeArgs args{};
    args.q = static_cast<const uint16_t*>(q);
    args.out = static_cast<uint16_t*>(out);
    args.block_tables = block_tables;
    args.context_lens = context_lens;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    args.sched = reinterpret_cast<int32_t*>(w);
    if (P > 1) {
        args.ws_m = reinterpret_cast<float*>(w + kSchedBytes);
        args.ws_l = reinterpret_cast<float*>(w + kSchedBytes + up256(SH * P * 4));
        args.ws_o = reinterpret_cast<float*>(w + kSchedBytes + 2 * up256(SH * P * 4));
    }
    args.err_word = err_word;
    args.scale_log2 = scale * 1.4426950408889634f;
    args.num_seqs = num_seqs;
    args.num_heads = num_heads;
    args.group = num_heads / num_kv_heads;
    args.block_size = block_size;
    args.num_blocks = num_blocks;
    args.max_blocks_per_seq = max_blocks_per_seq;
    args.partition_tokens = ptok;
    args.num_partitions = (int)P;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (head_dim == 128)
        return dtype == PA_F16 ? launch_decode<F16Tag, 128>(args, k_cache, v_cache, num_kv_heads, st)
                               : launch_decode<BF16Tag, 128>(args, k_cache, v_cache, num_kv_heads, st);
    return dtype == PA_F16 ? launch_decode<F16Tag, 64>(args, k_cache, v_cache, num_kv_heads, st)
                           : launch_decode<BF16Tag, 64>(args, k_cache, v_cache, num_kv_heads, st);
}
