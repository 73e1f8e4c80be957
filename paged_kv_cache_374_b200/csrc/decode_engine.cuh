// The persistent K2 engine shared by both decode compute paths.
//
// Units of work.  A sequence is cut into partitions of P tokens; a unit is one
// (sequence, partition, head slot) where a head slot is one query head (CUDA-core
// path) or one kv head with its whole group of query heads (tensor-core GQA
// path).  A sequence of one partition gets its output rows directly; a longer one
// leaves a partial result per partition and query head (running max m, running
// sum l, unnormalised o) in the workspace, merged by K3.
//
// One CTA per SM, NW warps per CTA, and every warp is a self-contained streaming
// engine: it claims units from a global counter, loads the unit's block-table
// entries with one coalesced warp load per 32 entries (each entry is read once,
// by one warp), and keeps its own ring of R shared-memory slots filled with TMA
// tensor copies (cp.async.bulk.tensor; a slot holds K and V of TOK tokens of one
// kv head as 64-dim half rows of 128 bytes under the 128-byte swizzle),
// completion tracked by one mbarrier per slot.  Issue runs R stages ahead of
// compute and crosses into the next claimed unit before the current one ends, so
// the warp's copies never drain at unit boundaries; no warp waits for another.
//
// Claim order: every full partition first (sequence-major, head slots fastest, so
// warps running together read the same physical blocks), then each sequence's
// last partition, longest first, so that the units left at the end are the
// shortest.  Every CTA derives the same order from context_lens in its prologue.
//
// The compute policy (decode_mha.cuh, decode_gqa.cuh) owns the per-unit state:
// q, the online-softmax statistics and the output accumulator.
#pragma once

#include <cmath>

#include "pa_device.cuh"

namespace pa {

constexpr int kMaxSeqsPerLaunch = 1024;   // sequences scheduled by one K2 launch
constexpr int kMaxPartitionTokens = 65536;
constexpr unsigned kFullMask = 0xffffffffu;

struct DecodeArgs {
    const uint16_t* q;
    uint16_t* out;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* ws_m;      // [S*H][Pmax], base-2 units
    float* ws_l;      // [S*H][Pmax]
    float* ws_o;      // [S*H][Pmax][D]
    int32_t* sched;   // [0] claim counter, [1] finished-warp counter, [2] merge-queue length,
                      // [3] engine-done flag, [4] finished merge CTAs; zero between launches
    int32_t* err_word;
    float scale_log2; // scale * log2(e)
    float k_scale;    // fp8 caches: K = code * k_scale (1 for 16-bit caches)
    float v_scale;    // fp8 caches: V = code * v_scale (1 for 16-bit caches)
    int num_seqs;     // sequences in this launch (<= kMaxSeqsPerLaunch)
    int num_heads;    // query heads
    int group;        // num_heads / num_kv_heads
    int unit_heads;   // head slots per sequence: num_heads (CUDA-core path) or num_kv_heads (GQA path)
    int heads_per_unit;  // query heads one unit computes: 1 or group
    int block_size;
    int box_rows;     // token rows per TMA box (min(TOK, block_size))
    int num_blocks;
    int max_blocks_per_seq;
    int partition_tokens;
    int num_partitions;  // Pmax: partitions allotted per (s, h) in the workspace
    // Nullable.  seq_start[s] > 0: the partitions of sequence s below token
    // seq_start[s] (a multiple of partition_tokens below context_lens[s]) are
    // already in the workspace (a shared prefix); this launch runs the rest.
    const int32_t* seq_start;
    // Nonzero: launched as a programmatic dependent of the cache write of the same
    // decode step, which may still be running.  The prologue and the first claims
    // read only the lengths, tables and q, which that write does not touch; every
    // warp waits for the write to complete before its first cache load.
    int wait_prior;
    // Nonzero (split partitions, no shared prefix): the merge kernel is launched
    // right after this launch's prologue and merges each (s, h) as soon as its last
    // partition lands.  merge_cnt[s*H + h] counts the partitions written;
    // merge_queue lists the (s*H + h) + 1 of completed pairs in completion order.
    // Both are left zero by the merge kernel.
    int early_merge;
    int32_t* merge_cnt;
    int32_t* merge_queue;
};

enum UnitKind { kUnitNone = 0, kUnitNormal = 1, kUnitZero = 2, kUnitNaN = 3 };

struct Unit {
    int kind;
    int s, h, p, np;  // h: head slot (a query head, or a kv head on the GQA path)
    int t_begin, t_end, nst, kv_head, blk0, nblk;
};

// ROWB: bytes of one token's row of one kv head (head_dim * element size);
// SCR: shared scratch bytes a compute policy keeps per warp (a multiple of 1 KiB)
template <int ROWB, int TOK, int NW, int R, int SCR = 0>
struct Layout {
    static constexpr int kTileBytes = TOK * ROWB;
    static constexpr int kHalfBytes = TOK * 128;               // one 128-byte-wide box column of a tile
    static constexpr int kSlotBytes = 2 * kTileBytes;          // K tile then V tile
    static constexpr int kOffSlots = 0;
    static constexpr int kOffScratch = NW * R * kSlotBytes;
    static constexpr int kOffBars = kOffScratch + NW * SCR;
    static constexpr int kOffCum = kOffBars + NW * R * 8;         // int[S + 1]
    static constexpr int kOffKey = kOffCum + (kMaxSeqsPerLaunch + 1) * 4 + 12;  // uint32[S_pow2]
    static constexpr int kOffLen = kOffKey + kMaxSeqsPerLaunch * 4;            // int[S]
    static constexpr int kBytes = kOffLen + kMaxSeqsPerLaunch * 4;
    static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1 KiB
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(kFullMask, x, o));
    return x;
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(kFullMask, x, o);
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
// First partition this launch runs for sequence s (0 unless a valid seq_start).
__device__ __forceinline__ int first_partition(const DecodeArgs& a, int s, int L) {
    if (!a.seq_start) return 0;
    const int st = __ldg(a.seq_start + s);
    const int P = a.partition_tokens;
    return (st > 0 && st < L && L <= a.max_blocks_per_seq * a.block_size && st % P == 0) ? st / P : 0;
}

__device__ __forceinline__ Unit decode_unit(int u, const DecodeArgs& a, const int* s_cum, const uint32_t* s_key,
                                            const int* s_len, int TOK) {
    Unit U;
    const int S = a.num_seqs, H = a.unit_heads;
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
    const int L = s_len[s];
    const int p0 = first_partition(a, s, L);
    U.s = s;
    U.h = h;
    U.p = p0 + p;
    U.np = p0 + s_cum[s + 1] - s_cum[s] + 1;
    const int maxlen = a.max_blocks_per_seq * a.block_size;
    U.kind = (L < 0 || L > maxlen) ? kUnitNaN : (L == 0 ? kUnitZero : kUnitNormal);
    const int P = a.partition_tokens;
    U.t_begin = U.p * P;
    U.t_end = U.kind == kUnitNormal ? min(L, U.t_begin + P) : U.t_begin;
    U.nst = (U.t_end - U.t_begin + TOK - 1) / TOK;
    U.kv_head = (h * a.heads_per_unit) / a.group;
    U.blk0 = U.t_begin / a.block_size;
    U.nblk = U.kind == kUnitNormal ? (U.t_end + a.block_size - 1) / a.block_size - U.blk0 : 0;
    return U;
}

// Output rows of a unit whose sequence has no tokens (zeros) or a bad length (NaN).
template <class Tag, int D>
__device__ __forceinline__ void write_special_rows(const DecodeArgs& a, const Unit& U, int lane) {
    const uint32_t w = U.kind == kUnitZero ? 0u : pack2<Tag>(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
    for (int i = lane; i < a.heads_per_unit * (D / 8); i += 32) {
        const int hq = U.h * a.heads_per_unit + i / (D / 8);
        reinterpret_cast<uint4*>(a.out + ((int64_t)U.s * a.num_heads + hq) * D)[i % (D / 8)] = make_uint4(w, w, w, w);
    }
    if (U.kind == kUnitNaN && lane == 0) report(a.err_word, PA_DEVERR_LEN_RANGE);
}

template <class Tag, class CTag, int D, int TOK, int NW, int R, class Policy>
__global__ void __launch_bounds__(NW * 32, 1) paged_decode_kernel(const DecodeArgs a,
                                                                  const __grid_constant__ CUtensorMap kmap,
                                                                  const __grid_constant__ CUtensorMap vmap) {
    constexpr int ROWB = D * CTag::kBytes;      // bytes per token row of one kv head
    static_assert(ROWB % 128 == 0, "rows are loaded as 128-byte swizzled boxes");
    using Lay = Layout<ROWB, TOK, NW, R, Policy::kScratchBytes>;
    constexpr int MAXSUB = TOK / 8 > 2 ? 2 : 1;  // TMA boxes per half tile (box_rows >= TOK/2)

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    int* s_cum = reinterpret_cast<int*>(smem + Lay::kOffCum);
    uint32_t* s_key = reinterpret_cast<uint32_t*>(smem + Lay::kOffKey);
    int* s_len = reinterpret_cast<int*>(smem + Lay::kOffLen);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = a.num_seqs;
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
            const int p0 = first_partition(a, s, L);
            if (a.seq_start && blockIdx.x == 0 && p0 == 0 && a.seq_start[s] != 0)
                report(a.err_word, PA_DEVERR_LEN_RANGE);  // unusable start: every partition runs here
            s_cum[s] = np - 1 - p0;  // full partitions this launch runs, scanned below
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
            const int y = __shfl_up_sync(kFullMask, incl, o);
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
    Policy pol;
    pol.setup(lane, smem + Lay::kOffScratch + warp * Policy::kScratchBytes);
    // The first two units of warp w are w and w + (all warps): no claim for them,
    // so that the launch does not start with every warp's atomics queued on one
    // counter.  The counter hands out the rest, from unit 2 x (all warps) on.
    // Behind the shared-prefix kernel the CTAs start over several microseconds,
    // as that kernel's CTAs leave the SMs: there every unit is claimed, so that
    // the first CTAs to start take the first units.
    int32_t* claim_ctr = a.sched;
    const bool static_first = a.seq_start == nullptr;
    const int all_warps = (int)gridDim.x * NW, gw = (int)blockIdx.x * NW + warp;
    const int claim_base = static_first ? 2 * all_warps : 0;
    auto claim = [&]() -> int { return lane == 0 ? atomicAdd(claim_ctr, 1) + claim_base : 0; };
    auto load_tab = [&](const Unit& U, int chunk) -> int {
        const int idx = chunk * 32 + lane;
        return (U.kind == kUnitNormal && idx < U.nblk)
                   ? __ldg(a.block_tables + (int64_t)U.s * a.max_blocks_per_seq + U.blk0 + idx)
                   : -1;
    };

    // current unit C (being consumed), next unit N, and a pending raw claim
    Unit C = decode_unit(static_first ? gw : __shfl_sync(kFullMask, claim(), 0), a, s_cum, s_key, s_len, TOK);
    Unit N = decode_unit(static_first ? gw + all_warps : __shfl_sync(kFullMask, claim(), 0), a, s_cum, s_key,
                         s_len, TOK);
    int pend = claim();
    pol.fetch_q(a, C);  // taken once C's first copies are issued (q_first below)
    bool q_first = true;
    pol.reset();
    int ntab0 = load_tab(N, 0), ntab1 = load_tab(N, 1);
    // issue cursor: in C (in_next = false) or N; its rolling table chunk pair
    bool in_next = false;
    int ist = 0;
    int ichunk = 0, itab_cur = load_tab(C, 0), itab_nxt = load_tab(C, 1);
    uint32_t issued = 0, consumed = 0;
    uint32_t badmask = 0;  // slots whose stage was dropped for a bad table entry
    bool aborted = false;
    int cst = 0;
    // Every K/V row is read once per launch: its lines are the first the L2 gives
    // up, so that the partials (written here, read back by the merge, rewritten at
    // the next step), q, the tables and the output stay resident.
    const uint64_t kv_policy = policy_evict_first();

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
            phys[j] = __shfl_sync(kFullMask, v, e & 31);
            if (use) {
                bad |= phys[j] < 0 || phys[j] >= a.num_blocks;
                tx += 2u * br * ROWB;
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
                        for (int hh = 0; hh < ROWB / 128; ++hh) {
                            uint8_t* kd = dst + hh * Lay::kHalfBytes + j * br * 128;
                            const int x = hh * (128 / CTag::kBytes);
                            tma_load_3d_hint(kd, &kmap, x, I.kv_head, row, &bars[slot], kv_policy);
                            tma_load_3d_hint(kd + Lay::kTileBytes, &vmap, x, I.kv_head, row, &bars[slot],
                                             kv_policy);
                        }
                    }
                }
            }
        }
        ++issued;
    };

    // The merge kernel may launch now: its CTAs take the SMs this grid's CTAs leave
    // and merge each (s, h) when its partitions are complete.
    if (a.early_merge) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (a.wait_prior) asm volatile("griddepcontrol.wait;" ::: "memory");  // the step's K/V are in the cache

    // Early merge: the split units this warp finished (lane i holds the i-th, as
    // s * unit_heads + head slot) are counted in batches, one fence per batch: all
    // of the warp's partial stores, then one count per query head; the count that
    // completes a head's partitions queues (s, h) for the merge.  A fence per unit
    // would stall the warp's stream once per unit.
    int fin = 0, nfin = 0;  // finished split units not yet counted
    auto publish = [&]() {
        __threadfence();
        __syncwarp();
        // the (unit, query head) counts spread over the lanes, so that their
        // round trips overlap: item i is head i % heads_per_unit of unit i / heads_per_unit
        const int hpu = a.heads_per_unit, items = nfin * hpu;
        for (int i0 = 0; i0 < items; i0 += 32) {
            const int i = i0 + lane;
            const int e = i < items ? i / hpu : 0;
            const int u = __shfl_sync(kFullMask, fin, e);
            if (i < items) {
                const int s = u / a.unit_heads, hs = u - s * a.unit_heads;
                const int np = (s_len[s] + P - 1) / P;
                const int sh = s * a.num_heads + hs * hpu + (i - e * hpu);
                if (atomicAdd(a.merge_cnt + sh, 1) == np - 1) {
                    const int slot = atomicAdd(a.sched + 2, 1);
                    asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(a.merge_queue + slot), "r"(sh + 1)
                                 : "memory");
                }
            }
        }
        __syncwarp();
        nfin = 0;
    };

    while (C.kind != kUnitNone && !aborted) {
        if (C.kind != kUnitNormal || C.nst == 0) {
            if (q_first) {
                pol.fetch_q(a, N);
                q_first = false;
            }
            write_special_rows<Tag, D>(a, C, lane);
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
            if (q_first) {  // the first unit's q, loaded while its first copies were issued
                pol.take_q(a);
                pol.fetch_q(a, N);
                q_first = false;
            }
            // consume one stage of C
            const int slot = consumed % R;
            const bool ok = __all_sync(kFullMask, mbar_wait(&bars[slot], (consumed / R) & 1));
            if (!ok) {
                if (lane == 0) report(a.err_word, PA_DEVERR_TIMEOUT);
                aborted = true;
                break;
            }
            if ((badmask >> slot) & 1u) {
                pol.poison();
                badmask &= ~(1u << slot);
            } else {
                const int ntok = min(TOK, C.t_end - (C.t_begin + cst * TOK));
                const uint8_t* kt = slots + slot * Lay::kSlotBytes;
                pol.stage(a, kt, kt + Lay::kTileBytes, ntok);
            }
            __syncwarp();
            ++consumed;
            if (++cst < C.nst) continue;
            pol.finish(a, C);
            if (a.early_merge && C.np > 1) {  // counted later, with one fence for many units
                if (nfin == 32) publish();
                if (lane == nfin) fin = C.s * a.unit_heads + C.h;
                ++nfin;
            }
        }
        // rotate: N becomes current; decode the pending claim as the new N
        const bool issue_was_in_next = in_next;
        C = N;
        if (C.kind == kUnitNormal) pol.take_q(a);
        N = decode_unit(__shfl_sync(kFullMask, pend, 0), a, s_cum, s_key, s_len, TOK);
        pol.fetch_q(a, N);
        ntab0 = load_tab(N, 0);
        ntab1 = load_tab(N, 1);
        if (N.kind != kUnitNone) pend = claim();
        in_next = false;
        if (!issue_was_in_next) {  // else the issue cursor already runs inside the new C
            ist = 0;
            ichunk = 0;
            itab_cur = load_tab(C, 0);
            itab_nxt = load_tab(C, 1);
        }
        pol.reset();
        cst = 0;
    }

    if (nfin > 0) publish();
    // never leave with copies into shared memory in flight
    for (uint32_t k = consumed; k < issued; ++k)
        if (!__all_sync(kFullMask, mbar_wait(&bars[k % R], (k / R) & 1)) && lane == 0)
            report(a.err_word, PA_DEVERR_TIMEOUT);
    // this warp writes nothing more: the merge kernel may be scheduled
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // the last warp of the launch to finish puts the claim counters back to zero
    // and, with an early merge, tells the merge kernel that the queue is complete
    if (lane == 0) {
        __threadfence();
        const int total = (int)(gridDim.x * NW);
        if (atomicAdd(a.sched + 1, 1) == total - 1) {
            atomicExch(a.sched, 0);
            atomicExch(a.sched + 1, 0);
            __threadfence();
            if (a.early_merge) {
                // behind the shared-prefix kernel: its counts and queue entries are
                // complete and visible once that grid is
                if (a.seq_start) asm volatile("griddepcontrol.wait;" ::: "memory");
                asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(a.sched + 3), "r"(1) : "memory");
            }
        }
    }
    // Launched behind the shared-prefix kernel (programmatic dependent launch),
    // this launch may run beside it but must not complete before it: the merge
    // kernel, which waits for this one, reads its partials too.  (A no-op for a
    // plain launch.)
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace pa
