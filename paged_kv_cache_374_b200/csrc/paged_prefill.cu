// Paged prefill: causal attention of a chunk of new query tokens over the paged
// cache -- the step before decode (P2 "大模型推理优化：KV Cache与PagedAttention技术详解",
// §2.1: the prompt's K/V enter the cache, then every position attends to the ones
// before it; prefix reuse across requests, P3 "LLM 推理中的 PageAttention 实现原理：虚拟内存管理在 KV Cache
// 中的创新应用" §三, makes the chunk start after
// cached tokens).  Query row i of sequence s (chunk of n rows over L tokens) sits
// at position L - n + i and attends to tokens 0 .. L - n + i through the table.
//
// A real dense contraction, run on the 5th-generation tensor cores (tcgen05, fp32
// accumulators in tensor memory).  One CTA per SM runs two query tiles A and B of
// 128 rows each (the MMAs' M) against the same K/V tiles of 128 tokens:
//   - warp 8 streams the kv head's K and V tiles through two-stage TMA rings (the
//     128-byte-swizzled tensor maps of the decode path; a tile's table entries
//     are read as it is issued, after one up-front range check); both query tiles
//     read every K and V tile the ring holds;
//   - warp 9 owns the tensor memory (O_A, O_B, and one S/P buffer per query tile)
//     and issues every MMA from one thread:
//       S_X = Q_X K_j^T  (A = Q_X, B = K_j, both K-major in shared memory; M 128 x N 128)
//       O_X += P_X V_j   (A = P_X in tensor memory, B = V_j MN-major; M 128 x N d)
//     in the order S_A0, S_B0, PV_A0, S_A1, PV_B0, S_B1, PV_A1, ...: while one
//     tile's softmax runs, the tensor core works on the other tile's MMAs;
//   - warps 0-3 (tile A) and 4-7 (tile B) own one query row per thread
//     (tensor-memory lane = row): read S_X, apply the causal mask and the online
//     softmax in base 2, write P_X over S_X (one f16 term for f16 inputs; for
//     bf16, two terms hi + lo, about 16 significant bits, so the result keeps the
//     decode path's accuracy), and at the end normalise O_X and store it.
// S_X(j+1) is issued after PV_X(j) and the tensor core runs one thread's MMAs in
// order, so the arrival that says S_X(j+1) landed also says PV_X(j) has: the
// softmax may rescale O_X then without another wait.  The running max used for
// the exponentials only moves when a row's max grows by more than 2^8 (then O_X
// and the row sum are rescaled in tensor memory); the result is the same
// softmax, p stays <= 256.  V rows past the sequence end are zeroed in shared
// memory before PV (0 * NaN is NaN in an MMA).  Every wait is bounded; a timeout
// reports PA_DEVERR_TIMEOUT and the CTA drains its copies and MMAs before freeing
// tensor memory.
#include <cmath>

#include "decode_gqa.cuh"
#include "pa_host.h"
#include "tcgen05.cuh"

namespace pa {

constexpr int kPfRows = 128;          // query rows of one tile (the MMAs' M)
constexpr int kPfCtaRows = 2 * kPfRows; // tiles A and B
constexpr int kPfTok = 128;           // tokens per K/V tile (the S MMAs' N)
constexpr int kPfLoadWarp = 8, kPfMmaWarp = 9;
constexpr int kPfThreads = 320;       // softmax warps 0-3 (A) and 4-7 (B), load warp, MMA warp
constexpr uint32_t kPfTmemCols = 512;   // O_X at column X d, S/P of tile X at 256 + 128 X
constexpr float kPfRescaleLog2 = 8.f;
constexpr int kPfWindow = 16;         // (sequence, head) pairs ordered together (launch order)

#ifndef PA_PF_SPIN
#define PA_PF_SPIN 1
#endif


// Bounded wait on an mbarrier phase: the suspending try_wait of the library, or
// (PA_PF_SPIN) a poll of test_wait bounded by 2 s of the global timer.
__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity) {
#if PA_PF_SPIN
    uint64_t t0;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    for (uint32_t i = 0;; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (done) return true;
        if ((i & 255u) == 255u) {
            uint64_t t1;
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
            if (t1 - t0 > 2000000000ull) return false;
        }
    }
#else
    return mbar_wait(bar, parity);
#endif
}

// A row's tile is read from tensor memory 64 tokens at a time (two passes: the
// max, then the weights), so that no thread holds more than 64 scores.
constexpr int kPfHalf = 64;

// The largest visible raw score of 64 tokens of a row (8 independent max chains);
// tokens past `vis` are left out when kDiag.
template <bool kDiag>
__device__ __forceinline__ float half_row_max(const float (&x)[kPfHalf], int vis) {
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = (!kDiag || i <= vis) ? x[i] : -INFINITY;
#pragma unroll
    for (int t = 8; t < kPfHalf; ++t)
        if (!kDiag || t <= vis) m[t & 7] = fmaxf(m[t & 7], x[t]);
#pragma unroll
    for (int w = 4; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) m[i] = fmaxf(m[i], m[i + w]);
    return m[0];
}

// p_t = 2^(x_t c - m) for 64 tokens of a row (0 past `vis` when kDiag), written to
// tensor memory two tokens per column: P_hi at tHi (32 columns) and, when kHiLo,
// P_lo = p - P_hi at tLo.  Returns the sum of the weights the MMA sees (P_hi + P_lo
// = p, or the rounded P_hi alone), so that the row's weights always sum to its
// denominator.  Packed fp32x2 arithmetic.  p <= 256, so an f16 P_hi alone is
// within 2^-11 of p (the f16 path); a bf16 P_hi (2^-8) needs the lo term to keep
// that accuracy.
template <class Tag, bool kDiag, bool kHiLo>
__device__ __forceinline__ float half_row_p(const float (&x)[kPfHalf], int vis, float c, float m, uint32_t tHi,
                                            uint32_t tLo) {
    const float2 c2 = make_float2(c, c), nm2 = make_float2(-m, -m), neg1 = make_float2(-1.f, -1.f);
    float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int part = 0; part < 2; ++part) {  // 32 tokens -> 16 hi and 16 lo columns
        uint32_t ph[16], pl[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int t = 32 * part + 2 * k;
            const float2 e = __ffma2_rn(make_float2(x[t], x[t + 1]), c2, nm2);
            float2 p = make_float2(fast_exp2(e.x), fast_exp2(e.y));
            if (kDiag) {
                p.x = t <= vis ? p.x : 0.f;
                p.y = t + 1 <= vis ? p.y : 0.f;
            }
            ph[k] = MmaOps<Tag>::pack(p.x, p.y);
            if (kHiLo) {
                acc[k & 3] = __fadd2_rn(acc[k & 3], p);
                const float2 lo = __ffma2_rn(Tag::widen2(ph[k]), neg1, p);  // p - hi, exact
                pl[k] = MmaOps<Tag>::pack(lo.x, lo.y);
            } else {
                acc[k & 3] = __fadd2_rn(acc[k & 3], Tag::widen2(ph[k]));  // the rounded weights
            }
        }
        umma::st16(tHi + 16 * part, ph);
        if (kHiLo) umma::st16(tLo + 16 * part, pl);
    }
    acc[0] = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
    return acc[0].x + acc[0].y;
}

// 64 scores of a row from tensor memory (two 32-column loads, one wait).
__device__ __forceinline__ void load_half(uint32_t taddr, float (&x)[kPfHalf]) {
    uint32_t a[32], b[32];
    umma::ld32(taddr, a);
    umma::ld32(taddr + 32, b);
    umma::wait_ld();
#pragma unroll
    for (int t = 0; t < 32; ++t) {
        x[t] = __uint_as_float(a[t]);
        x[32 + t] = __uint_as_float(b[t]);
    }
}

struct PrefillArgs {
    const uint16_t* q;    // [T][H][D]
    uint16_t* out;        // [T][H][D]
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* query_start;  // [S + 1]
    int32_t* err_word;
    float scale_log2;
    int num_heads, group, block_size, box_rows, num_blocks, max_blocks_per_seq;
    // shared-prefix mode (the prefix half of a two-level decode): group g's member
    // sequences group_members[group_offsets[g] .. group_offsets[g+1]) share the
    // partitions below seq_start[member]; each CTA computes one partition of one
    // kv head for up to 128 (member, query head) rows and leaves partials
    const int32_t* group_offsets;
    const int32_t* group_members;
    const int32_t* seq_start;
    float* ws_m;
    float* ws_l;
    float* ws_o;
    int partition_tokens, num_partitions, max_shared_partitions;
    int num_seqs;  // shared-prefix mode: group offsets lie in [0, num_seqs], members in [0, num_seqs)
    // shared-prefix mode with an early merge: count each partial written per (s, h)
    // and queue the (s, h) whose partitions it completes (the decode engine counts
    // the rest; the merge kernel reads the queue)
    int early_merge;
    int32_t* sched;
    int32_t* merge_cnt;
    int32_t* merge_queue;
};

// n partition slots of (seq, head) are in the workspace (this thread's stores
// fenced first); the write that completes the sequence's partitions queues it.
__device__ __forceinline__ void count_partial(const PrefillArgs& a, int seq, int head, int n) {
    __threadfence();
    const int sh = seq * a.num_heads + head;
    const int np = (a.context_lens[seq] + a.partition_tokens - 1) / a.partition_tokens;
    if (atomicAdd(a.merge_cnt + sh, n) + n == np) {
        const int slot = atomicAdd(a.sched + 2, 1);
        asm volatile("st.release.gpu.global.s32 [%0], %1;" ::"l"(a.merge_queue + slot), "r"(sh + 1) : "memory");
    }
}

template <int D>
struct PfLayout {
    static constexpr int kQHalf = kPfRows * 128;  // 64 dims of every row of a query tile
    static constexpr int kQTile = (D / 64) * kQHalf;
    static constexpr int kTHalf = kPfTok * 128;   // 64 dims of every token of a K/V tile
    static constexpr int kTile = (D / 64) * kTHalf;
    static constexpr int kOffK = 2 * kQTile;      // Q tiles A and B first
    static constexpr int kOffV = kOffK + 2 * kTile;
    static constexpr int kOffBars = kOffV + 2 * kTile;
    static constexpr int kNumBars = 16;
    static constexpr int kBytes = kOffBars + kNumBars * 8 + 16;
    // each CTA takes all 512 tensor-memory columns, so at most one may be resident
    // per SM: at least 116 KiB of shared memory (the head_dim 64 layout needs less)
    static constexpr int kAlloc = kBytes + 1024 > 116 * 1024 ? kBytes + 1024 : 116 * 1024;
};

// mbarrier slots
enum : int {
    kBarKFull = 0,   // [2] TMA landed a K tile
    kBarKEmpty = 2,  // [2] the S MMAs reading a K stage are done
    kBarVFull = 4,   // [2]
    kBarVEmpty = 6,  // [2] the PV MMAs reading a V stage are done
    kBarSFull = 8,   // [A, B] S_X(j) is in tile X's buffer (and PV_X(j-1) in O_X)
    kBarPFull = 10,  // [A, B] tile X's 4 row warps wrote P_X(j)
    kBarOLast = 12,  // [A, B] tile X's last PV has landed
    kBarDrain = 14,  // every MMA issued has completed
    kBarQ = 15,      // (prefill) the query tiles copied by TMA have landed
};

template <class Tag, int D, bool kShared>
__global__ void __launch_bounds__(kPfThreads, 1) paged_prefill_kernel(const PrefillArgs a,
                                                                      const __grid_constant__ CUtensorMap kmap,
                                                                      const __grid_constant__ CUtensorMap vmap,
                                                                      const __grid_constant__ CUtensorMap qmap) {
    using Lay = PfLayout<D>;
    constexpr bool kBF16 = Tag::kIsBF16;
    constexpr bool kHiLo = kBF16;  // P as hi + lo 16-bit terms (bf16), or one f16 term
    constexpr uint32_t kIdS = umma::idesc_f16(kBF16, false, kPfRows, kPfTok);
    constexpr uint32_t kIdO = umma::idesc_f16(kBF16, true, kPfRows, D);
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kOffBars);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + Lay::kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
    volatile int* bad_flag = reinterpret_cast<volatile int*>(tslot + 2);  // a table entry out of range
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bs = a.block_size;

    // The job of this CTA: nrows query rows (row r at position base_pos + r sees
    // tokens 0 .. base_pos + r) over the tokens [tok0, tok_end) of the table row
    // `tab`, of a sequence of L tokens; rows 0-127 are tile A, 128-255 tile B.
    int nrows, L, base_pos, tok0, tok_end, kv_head;
    const int32_t* tab;
    // prefill: rows q_first .. of sequence s, head h
    int s = 0, h = 0, q0 = 0, q_first = 0;
    // shared prefix: rows q_first .. of the group's (member, query head) list
    int m0 = 0;
    // prefill: the load warp's table entries for its boxes of tiles 0 and 1, read
    // before the lengths arrive (entries past the sequence are ignored later)
    int pre0 = -1, pre1 = -1;
    if constexpr (!kShared) {
        // CTA b (in launch order) -> (sequence, head, row tile): the (s, h) pairs go
        // in windows of kPfWindow; inside a window every pair's heaviest row tile
        // comes first, then every pair's next one, so that the launch ends on the
        // lightest CTAs while a window's K/V (at most kPfWindow heads' worth) is in L2
        const int64_t gx = gridDim.x, npairs = (int64_t)gridDim.y * gridDim.z;
        const int64_t b = blockIdx.x + gx * (blockIdx.y + (int64_t)gridDim.y * blockIdx.z);
        const int64_t w0 = b / (kPfWindow * gx) * kPfWindow;  // first pair of the window
        const int64_t wn = min((int64_t)kPfWindow, npairs - w0);  // pairs in the window
        const int64_t ib = b - w0 * gx;
        const int64_t pair_id = w0 + ib % wn;
        s = (int)(pair_id / gridDim.y);
        h = (int)(pair_id % gridDim.y);
        if (warp == kPfLoadWarp && lane < kPfTok / a.box_rows) {
            const int32_t* row = a.block_tables + (int64_t)s * a.max_blocks_per_seq;
            const int e0 = lane * a.box_rows / bs, e1 = (kPfTok + lane * a.box_rows) / bs;
            if (e0 < a.max_blocks_per_seq) pre0 = __ldg(row + e0);
            if (e1 < a.max_blocks_per_seq) pre1 = __ldg(row + e1);
        }
        const int qt = (int)(gx - 1 - ib / wn);  // the most context first
        q0 = a.query_start[s];
        const int n = a.query_start[s + 1] - q0;
        if (qt * kPfCtaRows >= n) return;
        L = a.context_lens[s];
        q_first = qt * kPfCtaRows;
        nrows = min(n - q_first, kPfCtaRows);
        if (L < 0 || L > a.max_blocks_per_seq * bs || n > L) {
            for (int i = tid; i < nrows * D; i += kPfThreads)
                a.out[((int64_t)(q0 + q_first + i / D) * a.num_heads + h) * D + i % D] =
                    Tag::round1(__int_as_float(0x7fc00000));
            if (tid == 0) report(a.err_word, PA_DEVERR_LEN_RANGE);
            return;
        }
        base_pos = L - n + q_first;
        tok0 = 0;
        tok_end = L;
        kv_head = h / a.group;
        tab = a.block_tables + (int64_t)s * a.max_blocks_per_seq;
    } else {
        // Launched as a programmatic dependent of the decode step's cache write, the
        // grid reads nothing before that write is complete, and lets the decode
        // engine launch only then, so the engine reads the step's new K/V with no
        // wait of its own.  Launched plainly, the wait returns at once.
        asm volatile("griddepcontrol.wait;" ::: "memory");
        // the decode engine that follows may start on the SMs this grid leaves free
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        const int g = blockIdx.z;
        kv_head = blockIdx.y;
        m0 = a.group_offsets[g];
        const int m1 = a.group_offsets[g + 1];
        // the group's offsets and members come from the caller: a group that
        // points outside the batch is skipped whole (every CTA of it agrees)
        bool bad_group = m0 < 0 || m1 < m0 || m1 > a.num_seqs;
        if (!bad_group)
            for (int i = m0 + tid; i < m1; i += kPfThreads) {
                const int mem = __ldg(a.group_members + i);
                bad_group |= mem < 0 || mem >= a.num_seqs;
            }
        if (__syncthreads_or(bad_group)) {
            if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) report(a.err_word, PA_DEVERR_GROUP_RANGE);
            return;
        }
        const int rows = (m1 - m0) * a.group;
        q_first = blockIdx.x * kPfCtaRows;
        if (q_first >= rows) return;
        nrows = min(rows - q_first, kPfCtaRows);
        const int lead = a.group_members[m0];
        L = a.seq_start[lead];  // tokens shared by the group
        const int P = a.partition_tokens;
        if (L <= 0 || L % P != 0 || L > a.max_blocks_per_seq * bs) {  // the group's start is unusable
            if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0) report(a.err_word, PA_DEVERR_LEN_RANGE);
            return;
        }
        // the launch bounds (max_group_size, max_shared_tokens) must cover every group
        if (tid == 0 && ((blockIdx.x == 0 && L > a.max_shared_partitions * P) ||
                         (blockIdx.x == gridDim.x - 1 && rows > (int)gridDim.x * kPfCtaRows)))
            report(a.err_word, PA_DEVERR_LEN_RANGE);
        // One CTA covers the whole shared prefix, all L / P partitions: its result
        // goes into the first partition's slot, and the others are marked absent
        // (running max -inf), which the merge skips.  One CTA per partition would
        // pay the CTA's start-up and epilogue once per partition.
        base_pos = 1 << 29;  // no causal mask: every row sees the whole prefix
        tok0 = 0;
        tok_end = L;
        tab = a.block_tables + (int64_t)lead * a.max_blocks_per_seq;
    }
    // K/V tiles of each query tile: up to the one holding the last token its last row sees
    auto tiles_of = [&](int x) {
        const int nx = min(max(nrows - x * kPfRows, 0), kPfRows);
        const int last = min(base_pos + x * kPfRows + nx - 1, tok_end - 1);
        return nx > 0 ? (last - tok0) / kPfTok + 1 : 0;
    };
    const int nt_a = tiles_of(0), nt_b = tiles_of(1);
    auto ntx = [&](int x) { return x ? nt_b : nt_a; };
    const int ntiles = max(nt_a, nt_b);
    // (member sequence, query head) of CTA row r in shared-prefix mode
    auto shared_row = [&](int r, int& seq, int& head) {
        const int gr = q_first + r;
        seq = a.group_members[m0 + gr / a.group];
        head = kv_head * a.group + gr % a.group;
    };
    // K/V copies of tile j (the load warp): lane i < 128 / box_rows owns box i of
    // every tile and reads that box's table entry; lane 0 posts the byte count first.
    // An entry out of range is never copied and marks the CTA bad.
    const int br = a.box_rows;
    const int nbox = kPfTok / br;
    const uint32_t box_bytes = (uint32_t)(D / 64) * br * 128;
    auto row_of = [&](int j) {  // this lane's cache row for tile j, or -1
        const int tj = tok0 + j * kPfTok + lane * br;
        if (lane >= nbox || tj >= L) return -1;
        const int id = (!kShared && j < 2) ? (j == 0 ? pre0 : pre1) : __ldg(tab + tj / bs);
        const bool in_range = id >= 0 && id < a.num_blocks;
        if (!in_range) *bad_flag = 1;
        return in_range ? id * bs + tj % bs : -1;
    };
    auto load = [&](const CUtensorMap* map, uint8_t* dst0, uint64_t* bar, int row) {
        const uint32_t n = __popc(__ballot_sync(FULL, row >= 0));
        if (lane == 0) mbar_arrive_expect_tx(bar, n * box_bytes);
        __syncwarp();
        if (row >= 0) {
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh)
                tma_load_3d(dst0 + hh * Lay::kTHalf + lane * br * 128, map, hh * 64, kv_head, row, bar);
        }
    };
    // Start-up, overlapped: the load warp sets up the barriers and issues the first
    // two K/V tiles and (prefill) the full query tiles by TMA; the row threads fetch
    // the other q rows.  Shared-prefix mode checks the table range before it goes
    // on; prefill checks each entry as the load warp reads it and turns the CTA's
    // rows into NaN at the end if one was out of range.
    const int early = ntiles < 2 ? ntiles : 2;  // tiles the load warp issues first
    // prefill query tiles of 128 rows come by TMA (rows of a chunk are contiguous in q)
    auto q_by_tma = [&](int x) { return !kShared && nrows >= (x + 1) * kPfRows; };
    if (warp == kPfLoadWarp) {
        if (lane == 0) {
            for (int i = 0; i < Lay::kNumBars; ++i)
                mbar_init(&bars[i], (i == kBarPFull || i == kBarPFull + 1) ? kPfRows / 32 : 1);
            *abort_flag = 0;
            *bad_flag = 0;
            fence_mbar_init();
            if (!kShared) {
                mbar_arrive_expect_tx(&bars[kBarQ], (uint32_t)((q_by_tma(0) + q_by_tma(1)) * Lay::kQTile));
                for (int x = 0; x < 2; ++x)
                    if (q_by_tma(x))
#pragma unroll
                        for (int hh = 0; hh < D / 64; ++hh)
                            tma_load_3d(smem + x * Lay::kQTile + hh * Lay::kQHalf, &qmap, hh * 64, h,
                                        q0 + q_first + x * kPfRows, &bars[kBarQ]);
            }
        }
        __syncwarp();
        for (int j = 0; j < early; ++j) {
            const int row = row_of(j);
            load(&kmap, smem + Lay::kOffK + j * Lay::kTile, &bars[kBarKFull + j], row);
            load(&vmap, smem + Lay::kOffV + j * Lay::kTile, &bars[kBarVFull + j], row);
        }
    }
    const bool q_rows = tid < kPfCtaRows && !q_by_tma(tid / kPfRows);  // this thread stores its q row
    uint4 qv[D / 8];
    const bool q_live = tid < nrows;
    if (q_rows) {
        int64_t qrow;  // row of q in [rows][num_heads * D] units of D
        if constexpr (!kShared) {
            qrow = (int64_t)(q0 + q_first + (q_live ? tid : 0)) * a.num_heads + h;
        } else {
            int seq, head;
            shared_row(q_live ? tid : 0, seq, head);
            qrow = (int64_t)seq * a.num_heads + head;
        }
        const uint4* src = reinterpret_cast<const uint4*>(a.q + qrow * D);
#pragma unroll
        for (int c = 0; c < D / 8; ++c) qv[c] = q_live ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    if constexpr (kShared) {
        const int e0 = tok0 / bs;
        const int nent = (min(tok0 + ntiles * kPfTok, L) + bs - 1) / bs;  // table entries the tiles read
        bool bad = false;
        for (int i = e0 + tid; i < nent; i += kPfThreads) {
            const int id = __ldg(tab + i);
            bad |= id < 0 || id >= a.num_blocks;
        }
        if (__syncthreads_or(bad)) {
            if (warp == kPfLoadWarp && lane == 0)  // the early copies land before the CTA exits
                for (int j = 0; j < early; ++j) {
                    pf_wait(&bars[kBarKFull + j], 0);
                    pf_wait(&bars[kBarVFull + j], 0);
                }
            for (int r = tid; r < nrows; r += kPfThreads) {
                int seq, head;
                shared_row(r, seq, head);
                const int64_t pi = ((int64_t)seq * a.num_heads + head) * a.num_partitions;
                a.ws_m[pi] = __int_as_float(0x7fc00000);
                a.ws_l[pi] = __int_as_float(0x7fc00000);
                for (int k = 1; k < L / a.partition_tokens; ++k) a.ws_m[pi + k] = -INFINITY;
                // merged, so the NaN reaches the row
                if (a.early_merge) count_partial(a, seq, head, L / a.partition_tokens);
            }
            if (tid == 0) report(a.err_word, PA_DEVERR_TABLE_RANGE);
            return;
        }
    }

    // q rows -> K-major swizzled tiles A and B (the 128-byte swizzle TMA applies);
    // rows past the chunk are zero.  A negative scale is moved into the sign of q
    // (exact), so the softmax sees scale >= 0: the row threads flip their own rows
    // here, and the rows TMA brings once they have landed (below).
    const uint32_t flip = a.scale_log2 < 0.f ? 0x80008000u : 0u;
    if (q_rows) {
        uint8_t* qt = smem + (tid / kPfRows) * Lay::kQTile + (tid % kPfRows) * 128;
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
            uint4 v = qv[c];
            v.x ^= flip;
            v.y ^= flip;
            v.z ^= flip;
            v.w ^= flip;
            *reinterpret_cast<uint4*>(qt + (c >> 3) * Lay::kQHalf + (((c & 7) ^ (tid & 7)) << 4)) = v;
        }
        fence_proxy_async_shared();
    }
    if (warp == kPfMmaWarp) umma::alloc(tslot, kPfTmemCols);
    umma::fence_before_sync();
    __syncthreads();
    umma::fence_after_sync();
    if (!kShared && flip) {  // the rows TMA brought (the barriers are initialised now)
        if (tid < kPfCtaRows && !q_rows) {
            if (pf_wait(&bars[kBarQ], 0)) {
                uint4* qt = reinterpret_cast<uint4*>(smem + (tid / kPfRows) * Lay::kQTile + (tid % kPfRows) * 128);
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {  // every 16-byte chunk of the row, wherever the swizzle put it
                    uint4* w = qt + (c >> 3) * (Lay::kQHalf / 16) + (c & 7);
                    uint4 v = *w;
                    v.x ^= flip;
                    v.y ^= flip;
                    v.z ^= flip;
                    v.w ^= flip;
                    *w = v;
                }
                fence_proxy_async_shared();
            } else {
                report(a.err_word, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
        }
        __syncthreads();
    }
    const uint32_t tmem = *tslot;
    const uint32_t tS = tmem + 256;  // S/P of tile X at tS + 128 X; O_X at tmem + X d

    if (warp == kPfLoadWarp) {
        // ---------------------------------------------------------------- loads
        // Tiles `early` .. on (the first ones went out during the start-up); a tile's
        // table entries are read ahead of the wait for its free stage.
        bool ok = true;
        int issued_k = early, issued_v = early;
        int row = early < ntiles ? row_of(early) : -1;
        for (int j = early; j < ntiles; ++j) {
            const int st = j & 1;
            if (j >= 2) ok = __all_sync(FULL, pf_wait(&bars[kBarKEmpty + st], ((j >> 1) + 1) & 1) && !*abort_flag);
            if (!ok) break;
            load(&kmap, smem + Lay::kOffK + st * Lay::kTile, &bars[kBarKFull + st], row);
            issued_k = j + 1;
            const int next = j + 1 < ntiles ? row_of(j + 1) : -1;  // in flight during the wait below
            if (j >= 2) ok = __all_sync(FULL, pf_wait(&bars[kBarVEmpty + st], ((j >> 1) + 1) & 1) && !*abort_flag);
            if (!ok) break;
            load(&vmap, smem + Lay::kOffV + st * Lay::kTile, &bars[kBarVFull + st], row);
            issued_v = j + 1;
            row = next;
        }
        if (lane == 0) {
            if (!ok) {
                report(a.err_word, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            // every copy still in flight lands before the CTA may exit
            if (!kShared) pf_wait(&bars[kBarQ], 0);
            for (int j = max(0, issued_k - 2); j < issued_k; ++j) pf_wait(&bars[kBarKFull + (j & 1)], (j >> 1) & 1);
            for (int j = max(0, issued_v - 2); j < issued_v; ++j) pf_wait(&bars[kBarVFull + (j & 1)], (j >> 1) & 1);
        }
        __syncwarp();
    } else if (warp == kPfMmaWarp) {
        // ----------------------------------------------------------------- MMAs
        // Operand descriptors, built once: an MMA's descriptor is its tile's or
        // stage's plus the byte offset / 16 in the start-address field (no carry:
        // shared addresses stay below 2^18).
        const uint64_t dq0 = umma::desc_sw128(smem_u32(smem), 16, 1024);
        const uint64_t dk0 = umma::desc_sw128(smem_u32(smem + Lay::kOffK), 16, 1024);
        const uint64_t dv0 = umma::desc_sw128(smem_u32(smem + Lay::kOffV), Lay::kTHalf, 1024);
        constexpr uint64_t kQTileStep = Lay::kQTile >> 4;  // tile B's Q
        constexpr uint64_t kStageStep = Lay::kTile >> 4;   // the second stage of a ring
        auto issue_s = [&](int x, int j) {  // lane 0: S_X(j) = Q_X K_j^T
            const uint64_t dq = dq0 + x * kQTileStep;
            const uint64_t bk = dk0 + (j & 1) * kStageStep;
            const uint32_t d = tS + x * 128;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                constexpr int kQStep = Lay::kQHalf >> 4, kTStep = Lay::kTHalf >> 4;
                umma::mma_ss(d, dq + (uint64_t)((kk >> 2) * kQStep + (kk & 3) * 2),
                             bk + (uint64_t)((kk >> 2) * kTStep + (kk & 3) * 2), kIdS, kk > 0 ? 1u : 0u);
            }
            umma::commit(&bars[kBarSFull + x]);
        };
        auto issue_pv = [&](int x, int j) {  // lane 0: O_X += P_X V_j
            const uint64_t bv = dv0 + (j & 1) * kStageStep;
            const uint32_t tp = tS + x * 128, to = tmem + x * D;
#pragma unroll
            for (int kk = 0; kk < kPfTok / 16; ++kk) {
                const uint64_t db = bv + (uint64_t)(kk * (2048 >> 4));  // 16 tokens further
                // tokens 16 kk .. of half kk / 4: P_hi 8 columns in, P_lo 32 further
                const uint32_t ta = tp + (kk >> 2) * kPfHalf + (kk & 3) * 8;
                umma::mma_ts(to, ta, db, kIdO, (j > 0 || kk > 0) ? 1u : 0u);  // P_hi V
                if (kHiLo) umma::mma_ts(to, ta + kPfHalf / 2, db, kIdO, 1u);  // P_lo V
            }
        };
        auto wait = [&](int bar, uint32_t parity) {  // whole warp
            const bool ok = pf_wait(&bars[bar], parity) && !*abort_flag;
            return __all_sync(FULL, ok);
        };
        bool ok = ntiles > 0 && wait(kBarKFull, 0) && (kShared || wait(kBarQ, 0));
        if (ok) {
            umma::fence_after_sync();
            if (lane == 0) {
                for (int x = 0; x < 2; ++x)
                    if (ntx(x) > 0) issue_s(x, 0);
                umma::commit(&bars[kBarKEmpty]);
            }
            __syncwarp();
        }
        for (int j = 0; j < ntiles && ok; ++j) {
            const int st = j & 1;
            bool v_ready = false;
            for (int x = 0; x < 2 && ok; ++x) {
                if (j >= ntx(x)) continue;
                if (!v_ready) {
                    ok = wait(kBarVFull + st, (j >> 1) & 1);
                    if (!ok) break;
                    const int t0 = tok0 + j * kPfTok;
                    if (t0 + kPfTok > L) {  // zero the V rows past the sequence end
                        uint8_t* vt = smem + Lay::kOffV + st * Lay::kTile;
                        const int r0 = L - t0;
#pragma unroll
                        for (int hh = 0; hh < D / 64; ++hh)
                            for (int i = r0 * 8 + lane; i < kPfTok * 8; i += 32)
                                *reinterpret_cast<uint4*>(vt + hh * Lay::kTHalf + i * 16) = make_uint4(0u, 0u, 0u, 0u);
                        fence_proxy_async_shared();
                        __syncwarp();
                    }
                    v_ready = true;
                }
                ok = wait(kBarPFull + x, j & 1);
                if (!ok) break;
                umma::fence_after_sync();
                // the last reader of V_j (tile B, or tile A when B has no tile j)
                // releases the stage; likewise for K_{j+1} below
                const bool v_last = x == 1 || j >= nt_b;
                if (lane == 0) {
                    issue_pv(x, j);
                    if (v_last) umma::commit(&bars[kBarVEmpty + st]);
                    if (j == ntx(x) - 1) umma::commit(&bars[kBarOLast + x]);
                }
                __syncwarp();
                if (j + 1 < ntx(x)) {
                    ok = wait(kBarKFull + ((j + 1) & 1), ((j + 1) >> 1) & 1);
                    if (!ok) break;
                    umma::fence_after_sync();
                    const bool k_last = x == 1 || j + 1 >= nt_b;
                    if (lane == 0) {
                        issue_s(x, j + 1);
                        if (k_last) umma::commit(&bars[kBarKEmpty + ((j + 1) & 1)]);
                    }
                    __syncwarp();
                }
            }
        }
        if (lane == 0) {
            if (!ok && ntiles > 0) {
                report(a.err_word, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            umma::commit(&bars[kBarDrain]);  // every MMA issued completes before TMEM is freed
            pf_wait(&bars[kBarDrain], 0);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------- softmax, one row per thread
        const int x = warp >> 2;             // query tile
        const int r = x * kPfRows + (tid & (kPfRows - 1));  // CTA row
        const int nt = ntx(x);
        const int pos = base_pos + min(r, nrows - 1);
        const int last = min(pos, tok_end - 1);  // last visible token of this row
        const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tSx = tS + x * 128 + lrow, tOx = tmem + x * D + lrow;
        const float c = fabsf(a.scale_log2);
        float m_used = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nt; ++j) {
            ok = __all_sync(FULL, pf_wait(&bars[kBarSFull + x], j & 1) && !*abort_flag);
            if (!ok) break;
            umma::fence_after_sync();
            const int vis = last - (tok0 + j * kPfTok);  // last visible token of the tile, this row
            // one branch per warp: the masked path's tensor-memory stores are
            // warp-aligned instructions, so no lane may take the other path
            const bool diag = __any_sync(FULL, vis < kPfTok - 1);
            float xs[kPfHalf];  // raw scores of one half of the tile
            float mt;
            {
                // the whole row in one round trip; the second half stays in xs
                float x0[kPfHalf];
                uint32_t a[32], b[32], c0[32], c1[32];
                umma::ld32(tSx, a);
                umma::ld32(tSx + 32, b);
                umma::ld32(tSx + 64, c0);
                umma::ld32(tSx + 96, c1);
                umma::wait_ld();
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    x0[t] = __uint_as_float(a[t]);
                    x0[32 + t] = __uint_as_float(b[t]);
                    xs[t] = __uint_as_float(c0[t]);
                    xs[32 + t] = __uint_as_float(c1[t]);
                }
                mt = fmaxf(diag ? half_row_max<true>(x0, vis) : half_row_max<false>(x0, vis),
                           diag ? half_row_max<true>(xs, vis - kPfHalf) : half_row_max<false>(xs, vis - kPfHalf));
            }
            mt = mt == -INFINITY ? -INFINITY : mt * c;  // the tile max in log2 units
            const bool need = mt > m_used + kPfRescaleLog2;  // always on the first tile
            if (__any_sync(FULL, need)) {
                const float m_new = need ? mt : m_used;
                if (j > 0) {  // PV_X(j-1) has landed in O_X (before S_X(j), see above)
                    const float alpha = fast_exp2(m_used - m_new);
#pragma unroll 1
                    for (int cc = 0; cc < D / 8; ++cc) {  // 8 columns at a time: few registers beside the scores
                        uint32_t o[8];
                        umma::ld8(tOx + cc * 8, o);
                        umma::wait_ld();
#pragma unroll
                        for (int k = 0; k < 8; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                        umma::st8(tOx + cc * 8, o);
                    }
                    umma::wait_st();
                    l *= alpha;
                }
                m_used = m_new;
            }
            // the weights of half hf go to its own 64 columns (P_hi of its token t in
            // column 64 hf + t / 2, P_lo 32 columns further), which hold only scores
            // this thread has already read.  The second half's scores are still in
            // registers from the max pass: it goes first, then the first is read again.
#pragma unroll
            for (int hf = 1; hf >= 0; --hf) {
                if (hf == 0) load_half(tSx, xs);
                const uint32_t tHi = tSx + hf * kPfHalf, tLo = tHi + kPfHalf / 2;
                l += diag ? half_row_p<Tag, true, kHiLo>(xs, vis - hf * kPfHalf, c, m_used, tHi, tLo)
                          : half_row_p<Tag, false, kHiLo>(xs, vis - hf * kPfHalf, c, m_used, tHi, tLo);
            }
            umma::wait_st();
            umma::fence_before_sync();
            __syncwarp();  // every lane's P is stored: one arrival per warp
            if (lane == 0) mbar_arrive(&bars[kBarPFull + x]);
        }
        if (ok && nt > 0) ok = __all_sync(FULL, pf_wait(&bars[kBarOLast + x], 0) && !*abort_flag);
        if (ok && nt > 0 && kShared) {
            // partial of the whole prefix for the row's (sequence, head), in the
            // first partition's slot: running max (base-2 units, scores scaled by
            // scale * log2 e), sum, unnormalised o
            umma::fence_after_sync();
            bool write = r < nrows;
            int64_t pi = 0;
            int seq = 0, head = 0;
            if (write) {
                shared_row(r, seq, head);
                const int Ls = a.context_lens[seq];
                // a member must share the group's prefix length and extend past it
                if (a.seq_start[seq] != L || Ls <= L || Ls > a.max_blocks_per_seq * bs) {
                    report(a.err_word, PA_DEVERR_LEN_RANGE);
                    write = false;
                }
                pi = ((int64_t)seq * a.num_heads + head) * a.num_partitions;
            }
            float4* dst = reinterpret_cast<float4*>(a.ws_o + pi * D);
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                umma::ld32(tOx + cc * 32, o);
                umma::wait_ld();
                if (write) {
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        dst[cc * 8 + v] = make_float4(__uint_as_float(o[4 * v]), __uint_as_float(o[4 * v + 1]),
                                                      __uint_as_float(o[4 * v + 2]), __uint_as_float(o[4 * v + 3]));
                }
            }
            if (write) {
                a.ws_m[pi] = m_used;
                a.ws_l[pi] = l;
                for (int k = 1; k < L / a.partition_tokens; ++k) a.ws_m[pi + k] = -INFINITY;  // absent
                if (a.early_merge) count_partial(a, seq, head, L / a.partition_tokens);
            }
        } else if (ok && nt > 0) {
            umma::fence_after_sync();
            const float inv = 1.f / l;
            uint4* dst = reinterpret_cast<uint4*>(
                a.out + ((int64_t)(q0 + q_first + min(r, nrows - 1)) * a.num_heads + h) * D);
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                umma::ld32(tOx + cc * 32, o);
                umma::wait_ld();
                if (r < nrows) {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        const float* f = reinterpret_cast<const float*>(o + 8 * v);
                        dst[cc * 4 + v] = make_uint4(
                            MmaOps<Tag>::pack(f[0] * inv, f[1] * inv), MmaOps<Tag>::pack(f[2] * inv, f[3] * inv),
                            MmaOps<Tag>::pack(f[4] * inv, f[5] * inv), MmaOps<Tag>::pack(f[6] * inv, f[7] * inv));
                    }
                }
            }
        } else if (!ok && lane == 0) {
            report(a.err_word, PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
        }
    }
    umma::fence_before_sync();
    __syncthreads();
    if (warp == kPfMmaWarp) {
        umma::fence_after_sync();
        umma::dealloc(tmem, kPfTmemCols);
    }
    if (!kShared && *bad_flag) {  // a table entry was out of range: the CTA's rows are NaN
        for (int i = tid; i < nrows * D; i += kPfThreads)
            a.out[((int64_t)(q0 + q_first + i / D) * a.num_heads + h) * D + i % D] =
                Tag::round1(__int_as_float(0x7fc00000));
        if (tid == 0) report(a.err_word, PA_DEVERR_TABLE_RANGE);
    }
}

namespace {

template <class Tag, int D>
int launch_prefill(PrefillArgs args, const void* k_cache, const void* v_cache, int num_kv_heads, int num_seqs,
                   int max_query_len, cudaStream_t stream) {
    using Lay = PfLayout<D>;
    static std::atomic<uint64_t> smem_done{0};
    auto kernel = paged_prefill_kernel<Tag, D, false>;
    if (ensure_smem_limit(kernel, Lay::kAlloc, smem_done) != cudaSuccess) return PA_ERR_CUDA;
    args.box_rows = kPfTok < args.block_size ? kPfTok : args.block_size;
    const int64_t total_tokens = (int64_t)args.num_blocks * args.block_size;
    CUtensorMap kmap, vmap;
    if (!encode_cache_map_swizzled(&kmap, k_cache, D, num_kv_heads, total_tokens, args.box_rows) ||
        !encode_cache_map_swizzled(&vmap, v_cache, D, num_kv_heads, total_tokens, args.box_rows))
        return PA_ERR_CUDA;
    // q as [rows][num_heads][D]; the extent covers every row a full query tile may
    // start at (num_seqs * max_query_len bounds the packed rows, which int32
    // query_start keeps below 2^31), and only tiles of 128 rows inside one
    // sequence's chunk are copied
    CUtensorMap qmap;
    const int64_t q_rows = (int64_t)num_seqs * max_query_len;
    if (!encode_cache_map_swizzled(&qmap, args.q, D, args.num_heads, q_rows < INT32_MAX ? q_rows : INT32_MAX, kPfRows))
        return PA_ERR_CUDA;
    dim3 grid((unsigned)((max_query_len + kPfCtaRows - 1) / kPfCtaRows), (unsigned)args.num_heads,
              (unsigned)num_seqs);
    kernel<<<grid, kPfThreads, Lay::kAlloc, stream>>>(args, kmap, vmap, qmap);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

template <class Tag, int D>
int launch_shared(PrefillArgs args, const void* k_cache, const void* v_cache, int num_kv_heads, int num_groups,
                  int max_group_size, bool after_write, cudaStream_t stream) {
    using Lay = PfLayout<D>;
    static std::atomic<uint64_t> smem_done{0};
    auto kernel = paged_prefill_kernel<Tag, D, true>;
    if (ensure_smem_limit(kernel, Lay::kAlloc, smem_done) != cudaSuccess) return PA_ERR_CUDA;
    args.box_rows = kPfTok < args.block_size ? kPfTok : args.block_size;
    const int64_t total_tokens = (int64_t)args.num_blocks * args.block_size;
    CUtensorMap kmap, vmap;
    if (!encode_cache_map_swizzled(&kmap, k_cache, D, num_kv_heads, total_tokens, args.box_rows) ||
        !encode_cache_map_swizzled(&vmap, v_cache, D, num_kv_heads, total_tokens, args.box_rows))
        return PA_ERR_CUDA;
    const int64_t rows = (int64_t)max_group_size * args.group;
    dim3 grid((unsigned)((rows + kPfCtaRows - 1) / kPfCtaRows), (unsigned)num_kv_heads,
              (unsigned)num_groups);
    if (after_write) {  // a programmatic dependent of the cache write launched just before
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(kPfThreads);
        cfg.dynamicSmemBytes = Lay::kAlloc;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, kernel, args, kmap, vmap, kmap) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
    }
    kernel<<<grid, kPfThreads, Lay::kAlloc, stream>>>(args, kmap, vmap, kmap);  // (no q map in this mode)
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace

int launch_shared_prefix(const SharedPrefixLaunch& l, cudaStream_t stream) {
    if (l.partition_tokens % 64 != 0 || l.max_shared_tokens % l.partition_tokens != 0) return PA_ERR_INVALID_ARG;
    const int64_t maxpp = l.max_shared_tokens / l.partition_tokens;
    if (maxpp == 0 || l.num_groups == 0) return PA_OK;
    if (l.num_groups > 65535 || l.num_kv_heads > 65535) return PA_ERR_UNSUPPORTED;
    PrefillArgs args{};
    args.q = static_cast<const uint16_t*>(l.q);
    args.block_tables = l.block_tables;
    args.context_lens = l.context_lens;
    args.err_word = l.err_word;
    args.scale_log2 = l.scale * 1.4426950408889634f;
    args.num_heads = l.num_heads;
    args.group = l.num_heads / l.num_kv_heads;
    args.block_size = l.block_size;
    args.num_blocks = l.num_blocks;
    args.max_blocks_per_seq = l.max_blocks_per_seq;
    args.group_offsets = l.group_offsets;
    args.group_members = l.group_members;
    args.seq_start = l.seq_start;
    args.ws_m = l.ws_m;
    args.ws_l = l.ws_l;
    args.ws_o = l.ws_o;
    args.partition_tokens = l.partition_tokens;
    args.num_partitions = l.num_partitions;
    args.max_shared_partitions = (int)maxpp;
    args.num_seqs = l.num_seqs;
    args.early_merge = l.early_merge;
    args.sched = l.sched;
    args.merge_cnt = l.merge_cnt;
    args.merge_queue = l.merge_queue;
    const bool after = l.after_write != 0;
    if (l.head_dim == 128)
        return l.dtype == PA_F16 ? launch_shared<F16Tag, 128>(args, l.k_cache, l.v_cache, l.num_kv_heads, l.num_groups,
                                                              l.max_group_size, after, stream)
                                 : launch_shared<BF16Tag, 128>(args, l.k_cache, l.v_cache, l.num_kv_heads,
                                                               l.num_groups, l.max_group_size, after, stream);
    return l.dtype == PA_F16 ? launch_shared<F16Tag, 64>(args, l.k_cache, l.v_cache, l.num_kv_heads, l.num_groups,
                                                         l.max_group_size, after, stream)
                             : launch_shared<BF16Tag, 64>(args, l.k_cache, l.v_cache, l.num_kv_heads, l.num_groups,
                                                          l.max_group_size, after, stream);
}

}  // namespace pa

extern "C" int pa_prefill(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                          const int32_t* context_lens, const int32_t* query_start, float scale, int num_kv_heads,
                          void* out, int num_seqs, int num_heads, int head_dim, int block_size, int num_blocks,
                          int max_blocks_per_seq, int max_query_len, int dtype, int32_t* err_word, void* stream) {
    using namespace pa;
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_query_len < 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (block_size != 16 && block_size != 32 && block_size != 64) return PA_ERR_UNSUPPORTED;
    if ((int64_t)num_blocks * block_size > INT32_MAX || (int64_t)max_blocks_per_seq * block_size > INT32_MAX)
        return PA_ERR_UNSUPPORTED;
    if (num_seqs > 65535 || num_heads > 65535) return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0 || max_query_len == 0) return PA_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start || !out)
        return PA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned4(block_tables) ||
        !aligned4(context_lens) || !aligned4(query_start) || (err_word && !aligned4(err_word)))
        return PA_ERR_INVALID_ARG;
    PrefillArgs args{};
    args.q = static_cast<const uint16_t*>(q);
    args.out = static_cast<uint16_t*>(out);
    args.block_tables = block_tables;
    args.context_lens = context_lens;
    args.query_start = query_start;
    args.err_word = err_word;
    args.scale_log2 = scale * 1.4426950408889634f;
    args.num_heads = num_heads;
    args.group = num_heads / num_kv_heads;
    args.block_size = block_size;
    args.num_blocks = num_blocks;
    args.max_blocks_per_seq = max_blocks_per_seq;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (head_dim == 128)
        return dtype == PA_F16
                   ? launch_prefill<F16Tag, 128>(args, k_cache, v_cache, num_kv_heads, num_seqs, max_query_len, st)
                   : launch_prefill<BF16Tag, 128>(args, k_cache, v_cache, num_kv_heads, num_seqs, max_query_len, st);
    return dtype == PA_F16
               ? launch_prefill<F16Tag, 64>(args, k_cache, v_cache, num_kv_heads, num_seqs, max_query_len, st)
               : launch_prefill<BF16Tag, 64>(args, k_cache, v_cache, num_kv_heads, num_seqs, max_query_len, st);
}
