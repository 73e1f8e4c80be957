// K2 + K3: single-query (decode) attention over the paged KV cache.
//
// What is computed (P1 "大模型部署中的PagedAttention：KV Cache显存管理突破", §1, first
// formula; P3 "LLM 推理中的 PageAttention 实现原理", §二 and §三): for sequence s and
// query head h, out = softmax(scale * q K^T) V over the sequence's L tokens taken
// in logical order, token t living in physical block block_tables[s][t / B] at
// offset t % B -- one softmax over all L tokens.
//
// Work decomposition (CUDA cores; fp32 arithmetic throughout):
//   grid = (num_heads * P, num_seqs): one CTA per (query head, context partition,
//   sequence).  A partition is `partition_tokens` consecutive tokens; sequences
//   longer than one partition are split across CTAs whose partial results
//   (running max m, running sum l, unnormalised o) go to the workspace and are
//   merged by K3.  Query heads of one sequence are the fastest grid dimension, so
//   CTAs that run together read the same physical blocks (all heads of a token
//   row sit next to each other) and the CTAs of a GQA group share tiles in L2.
//
// Inside a CTA (4 consumer warps + 1 producer warp):
//   - the producer warp loads the partition's block-table entries with one
//     coalesced warp load per 32 entries (each entry is read once, by one warp),
//     then its lane 0 streams K and V tiles of TOK tokens x head_dim into an
//     NS-deep shared-memory ring with TMA tensor copies (cp.async.bulk.tensor),
//     completion tracked by mbarriers (full / empty per stage);
//   - consumer warp w takes stages w, w+4, ...; per stage it computes the TOK
//     scores with 16-byte shared loads (a token row is split over CH lanes, one
//     16-byte chunk each), reduces them with a reduce-scatter over warp shuffles,
//     updates its online softmax (running max / sum, base-2 exponentials with
//     log2(e) folded into the pre-scaled q) and accumulates p * V;
//   - the four warp states are merged through shared memory at the end.
// Rows past the sequence end inside the last block are never used: their scores
// become -inf and their V rows are skipped (not multiplied by 0, as they may
// hold NaN).  Table entries outside [0, num_blocks) are never dereferenced: the
// stage is dropped, the output row becomes NaN and PA_DEVERR_TABLE_RANGE is set.
#include <cmath>

#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {

constexpr int kConsumerWarps = 4;
constexpr int kDecodeThreads = (kConsumerWarps + 1) * 32;

struct DecodeArgs {
    const uint16_t* q;
    uint16_t* out;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float* ws_m;   // [S*H][P]
    float* ws_l;   // [S*H][P]
    float* ws_o;   // [S*H][P][D]
    int32_t* err_word;
    float scale_log2;  // scale * log2(e)
    int num_heads;
    int group;         // num_heads / num_kv_heads
    int block_size;
    int num_blocks;
    int max_blocks_per_seq;
    int partition_tokens;
    int num_partitions;  // P: partitions allotted per (s, h) in the workspace
};

template <int D, int TOK, int NS>
struct MhaLayout {
    static constexpr int kTileBytes = TOK * D * 2;
    static constexpr int kOffK = 0;
    static constexpr int kOffV = NS * kTileBytes;
    static constexpr int kOffFull = 2 * NS * kTileBytes;
    static constexpr int kOffEmpty = kOffFull + NS * 8;
    static constexpr int kOffBad = kOffEmpty + NS * 8;
    static constexpr int kOffAbort = kOffBad + NS * 4;
    static constexpr int kOffMergeM = (kOffAbort + 4 + 15) / 16 * 16;
    static constexpr int kOffMergeL = kOffMergeM + kConsumerWarps * 4;
    static constexpr int kOffMergeO = kOffMergeL + kConsumerWarps * 4;
    static constexpr int kBytes = kOffMergeO + kConsumerWarps * D * 4;
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
__device__ __forceinline__ void widen8(const uint4& w, float (&f)[8]) {
    float2 a = Tag::widen2(w.x), b = Tag::widen2(w.y), c = Tag::widen2(w.z), d = Tag::widen2(w.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

template <class Tag, int D>
__device__ __forceinline__ void write_row_const(uint16_t* row, float value) {
    for (int i = threadIdx.x; i < D; i += blockDim.x) row[i] = Tag::round1(value);
}

template <class Tag, int D, int TOK, int NS>
__global__ void __launch_bounds__(kDecodeThreads) paged_decode_mha_kernel(const DecodeArgs a,
                                                                          const __grid_constant__ CUtensorMap kmap,
                                                                          const __grid_constant__ CUtensorMap vmap) {
    using Lay = MhaLayout<D, TOK, NS>;
    constexpr int CH = D / 8;       // 16-byte chunks per token row
    constexpr int RPI = 32 / CH;    // token rows covered by one warp-wide 16-byte load
    constexpr int NV = TOK / RPI;   // row groups per stage (values each lane reduces)
    static_assert(NV >= 1 && NV <= CH && CH % NV == 0, "stage shape");
    constexpr int DUP = CH / NV;    // lanes that end up holding the same token's score
    constexpr int SH = DUP == 1 ? 0 : DUP == 2 ? 1 : DUP == 4 ? 2 : DUP == 8 ? 3 : 4;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::kOffFull);
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + Lay::kOffEmpty);
    volatile int* bad = reinterpret_cast<volatile int*>(smem + Lay::kOffBad);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kOffAbort);
    float* merge_m = reinterpret_cast<float*>(smem + Lay::kOffMergeM);
    float* merge_l = reinterpret_cast<float*>(smem + Lay::kOffMergeL);
    float* merge_o = reinterpret_cast<float*>(smem + Lay::kOffMergeO);

    const int h = blockIdx.x % a.num_heads;
    const int part = blockIdx.x / a.num_heads;
    const int s = blockIdx.y;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int bs = a.block_size;
    const int64_t sh = (int64_t)s * a.num_heads + h;
    uint16_t* out_row = a.out + sh * D;

    const int L = a.context_lens[s];
    if (L < 0 || L > a.max_blocks_per_seq * bs) {
        if (part == 0) {
            write_row_const<Tag, D>(out_row, __int_as_float(0x7fc00000));
            if (threadIdx.x == 0) report(a.err_word, PA_DEVERR_LEN_RANGE);
        }
        return;
    }
    if (L == 0) {
        if (part == 0) write_row_const<Tag, D>(out_row, 0.f);
        return;
    }
    const int P = a.partition_tokens;
    const int nparts = (L + P - 1) / P;
    if (part >= nparts) return;
    const int t_begin = part * P;
    const int t_end = min(L, t_begin + P);
    const int nst = (t_end - t_begin + TOK - 1) / TOK;
    const int kv_head = h / a.group;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
            bad[i] = 0;
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------ producer
        constexpr int BR = TOK;  // rows per box: a stage never spans two blocks (TOK <= block_size)
        const int32_t* trow = a.block_tables + (int64_t)s * a.max_blocks_per_seq;
        const int blk0 = t_begin / bs;
        const int nblk = (t_end + bs - 1) / bs - blk0;  // table entries this partition reads
        if (lane == 0) {
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
        }
        int tab = -1, tab_chunk = -1;
        int issued = 0;
        for (int st = 0; st < nst; ++st) {
            const int slot = st % NS;
            const int t0 = t_begin + st * TOK;
            const int e = t0 / bs - blk0;  // warp-uniform
            if ((e >> 5) != tab_chunk) {
                tab_chunk = e >> 5;
                const int idx = (tab_chunk << 5) + lane;
                tab = idx < nblk ? __ldg(trow + blk0 + idx) : -1;
            }
            const int phys = __shfl_sync(0xffffffffu, tab, e & 31);
            bool ok = true;
            if (lane == 0 && st >= NS) ok = mbar_wait(&empty[slot], ((st / NS) - 1) & 1);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok || *abort_flag) {
                if (lane == 0) {
                    if (!ok) report(a.err_word, PA_DEVERR_TIMEOUT);
                    *abort_flag = 1;
                }
                break;
            }
            if (lane == 0) {
                if (phys < 0 || phys >= a.num_blocks) {
                    report(a.err_word, PA_DEVERR_TABLE_RANGE);
                    bad[slot] = 1;
                    mbar_arrive(&full[slot]);
                } else {
                    bad[slot] = 0;
                    const int row = phys * bs + (t0 % bs);
                    mbar_arrive_expect_tx(&full[slot], 2u * BR * D * 2);
                    tma_load_3d(smem + Lay::kOffK + slot * Lay::kTileBytes, &kmap, 0, kv_head, row, &full[slot]);
                    tma_load_3d(smem + Lay::kOffV + slot * Lay::kTileBytes, &vmap, 0, kv_head, row, &full[slot]);
                }
            }
            issued = st + 1;
        }
        // Do not leave while copies into this CTA's shared memory are in flight.
        if (lane == 0) {
            for (int st = issued > NS ? issued - NS : 0; st < issued; ++st)
                if (!mbar_wait(&full[st % NS], (st / NS) & 1)) report(a.err_word, PA_DEVERR_TIMEOUT);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int c = lane % CH;  // 16-byte chunk of the row this lane reads
    const int r = lane / CH;  // row within a warp-wide load
    float qv[8];
    {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(a.q + sh * D) + c);
        widen8<Tag>(w, qv);
#pragma unroll
        for (int k = 0; k < 8; ++k) qv[k] *= a.scale_log2;
    }
    float m = -INFINITY, lsum = 0.f;
    float o[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) o[k] = 0.f;
    bool poisoned = false;

    for (int st = warp; st < nst; st += kConsumerWarps) {
        const int slot = st % NS;
        if (*abort_flag) break;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&full[slot], (st / NS) & 1));
        if (!ok) {
            if (lane == 0) {
                report(a.err_word, PA_DEVERR_TIMEOUT);
                *abort_flag = 1;
            }
            break;
        }
        if (bad[slot]) {
            poisoned = true;
        } else {
            const int ntok = min(TOK, t_end - (t_begin + st * TOK));
            const uint8_t* kt = smem + Lay::kOffK + slot * Lay::kTileBytes;
            const uint8_t* vt = smem + Lay::kOffV + slot * Lay::kTileBytes;
            // scores: lane (c, r) forms the partial dot of row i*RPI + r over its chunk
            float acc[NV];
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int row = i * RPI + r;
                const uint4 w = *reinterpret_cast<const uint4*>(kt + (row * D + c * 8) * 2);
                float kf[8];
                widen8<Tag>(w, kf);
                float d0 = 0.f;
#pragma unroll
                for (int k = 0; k < 8; ++k) d0 = fmaf(qv[k], kf[k], d0);
                acc[i] = d0;
            }
            // reduce-scatter over the CH lanes of a row: after it, lane c holds the
            // full score of row group (c >> SH)
#pragma unroll
            for (int width = NV; width > 1; width >>= 1) {
                const int half = width >> 1;
                const int mask = half << SH;
                const bool upper = (c & mask) != 0;
#pragma unroll
                for (int j = 0; j < half; ++j) {
                    const float keep = upper ? acc[j + half] : acc[j];
                    const float send = upper ? acc[j] : acc[j + half];
                    acc[j] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
                }
            }
            float x = acc[0];
#pragma unroll
            for (int mask = 1; mask < DUP; mask <<= 1) x += __shfl_xor_sync(0xffffffffu, x, mask);
            const int tok = (c >> SH) * RPI + r;
            if (tok >= ntok) x = -INFINITY;
            const float m_new = fmaxf(m, warp_max(x));
            const float alpha = exp2f(m - m_new);
            const float p = exp2f(x - m_new);
            lsum = lsum * alpha + p;
#pragma unroll
            for (int k = 0; k < 8; ++k) o[k] *= alpha;
            m = m_new;
            // o += p_row * V_row for the rows this lane covers
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int row = i * RPI + r;
                const float pr = __shfl_sync(0xffffffffu, p, r * CH + (i << SH));
                if (row < ntok) {
                    const uint4 w = *reinterpret_cast<const uint4*>(vt + (row * D + c * 8) * 2);
                    float vf[8];
                    widen8<Tag>(w, vf);
#pragma unroll
                    for (int k = 0; k < 8; ++k) o[k] = fmaf(pr, vf[k], o[k]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
    }

    // warp state: fold the RPI row groups, then the DUP copies of each p in lsum
#pragma unroll
    for (int off = CH; off < 32; off <<= 1) {
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] += __shfl_xor_sync(0xffffffffu, o[k], off);
    }
    lsum = warp_sum(lsum) * (1.f / DUP);
    poisoned = __any_sync(0xffffffffu, poisoned);
    if (r == 0) {
#pragma unroll
        for (int k = 0; k < 8; ++k) merge_o[warp * D + c * 8 + k] = o[k];
    }
    if (lane == 0) {
        merge_m[warp] = m;
        merge_l[warp] = poisoned ? __int_as_float(0x7fc00000) : lsum;
    }
    named_barrier(1, kConsumerWarps * 32);

    const int tid = threadIdx.x;
    if (tid < D) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, merge_m[w]);
        float l = 0.f, acc = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
            const float mw = merge_m[w];
            const float sc = mw == -INFINITY ? 0.f : exp2f(mw - M);
            l = fmaf(merge_l[w], sc, l);
            acc = fmaf(merge_o[w * D + tid], sc, acc);
        }
        if (nparts == 1) {
            out_row[tid] = Tag::round1(acc / l);
        } else {
            const int64_t pi = sh * a.num_partitions + part;
            a.ws_o[pi * D + tid] = acc;
            if (tid == 0) {
                a.ws_m[pi] = M;
                a.ws_l[pi] = l;
            }
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
        const float w = exp2f(pm[p] - M);
        den = fmaf(pl[p], w, den);
        acc = fmaf(po[(int64_t)p * D + i], w, acc);
    }
    a.out[sh * D + i] = Tag::round1(acc / den);
}

// ------------------------------------------------------------------------ host

namespace {

constexpr int kDefaultPartition = 512;

int64_t num_partitions(int max_blocks_per_seq, int block_size, int ptok) {
    const int64_t max_len = (int64_t)max_blocks_per_seq * block_size;
    return max_len <= 0 ? 1 : (max_len + ptok - 1) / ptok;
}

size_t workspace_bytes_for(int64_t sh, int64_t P, int D) {
    if (P <= 1) return 0;
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    return up(sh * P * 4) * 2 + up(sh * P * D * 4);
}

template <class Tag, int D>
int launch_mha(DecodeArgs args, int num_seqs, const void* k_cache, const void* v_cache, int num_kv_heads,
               cudaStream_t stream) {
    constexpr int TOK = 16;
    constexpr int NS = 8;
    using Lay = MhaLayout<D, TOK, NS>;
    static std::atomic<uint64_t> smem_done{0};
    auto kernel = paged_decode_mha_kernel<Tag, D, TOK, NS>;
    if (ensure_smem_limit(kernel, Lay::kAlloc, smem_done) != cudaSuccess) return PA_ERR_CUDA;
    if (TOK > args.block_size) return PA_ERR_UNSUPPORTED;
    const int64_t total_tokens = (int64_t)args.num_blocks * args.block_size;
    CUtensorMap kmap, vmap;
    if (!encode_cache_map(&kmap, k_cache, D, num_kv_heads, total_tokens, TOK) ||
        !encode_cache_map(&vmap, v_cache, D, num_kv_heads, total_tokens, TOK))
        return PA_ERR_CUDA;
    const int64_t gx = (int64_t)args.num_heads * args.num_partitions;
    dim3 grid((unsigned)gx, (unsigned)num_seqs);
    kernel<<<grid, kDecodeThreads, Lay::kAlloc, stream>>>(args, kmap, vmap);
    if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
    if (args.num_partitions > 1) {
        paged_decode_merge_kernel<Tag, D><<<(unsigned)((int64_t)num_seqs * args.num_heads), D, 0, stream>>>(args);
        if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
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
        max_blocks_per_seq < 0 || partition_tokens < 0 || partition_tokens % 64 != 0)
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
        num_blocks <= 0 || max_blocks_per_seq <= 0 || partition_tokens < 0 || partition_tokens % 64 != 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
    if (head_dim != 64 && head_dim != 128) return PA_ERR_UNSUPPORTED;
    if (block_size != 16 && block_size != 32 && block_size != 64) return PA_ERR_UNSUPPORTED;
    if ((int64_t)num_blocks * block_size > INT32_MAX ||
        (int64_t)max_blocks_per_seq * block_size > INT32_MAX || num_seqs > 65535)
        return PA_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PA_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !out) return PA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        !aligned4(block_tables) || !aligned4(context_lens) || (err_word && !aligned4(err_word)))
        return PA_ERR_INVALID_ARG;
    const int ptok = partition_tokens > 0
                         ? partition_tokens
                         : pa_decode_partition_tokens(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                      max_blocks_per_seq);
    const int64_t P = num_partitions(max_blocks_per_seq, block_size, ptok);
    if ((int64_t)num_heads * P > INT32_MAX) return PA_ERR_UNSUPPORTED;
    const int64_t SH = (int64_t)num_seqs * num_heads;
    const size_t need = workspace_bytes_for(SH, P, head_dim);
    if (need > 0 && (!workspace || !aligned16(workspace) || workspace_bytes < need)) return PA_ERR_INVALID_ARG;

    DecodeArgs args{};
    args.q = static_cast<const uint16_t*>(q);
    args.out = static_cast<uint16_t*>(out);
    args.block_tables = block_tables;
    args.context_lens = context_lens;
    if (need > 0) {
        auto up = [](size_t x) { return (x + 255) / 256 * 256; };
        uint8_t* w = static_cast<uint8_t*>(workspace);
        args.ws_m = reinterpret_cast<float*>(w);
        args.ws_l = reinterpret_cast<float*>(w + up(SH * P * 4));
        args.ws_o = reinterpret_cast<float*>(w + 2 * up(SH * P * 4));
    }
    args.err_word = err_word;
    args.scale_log2 = scale * 1.4426950408889634f;
    args.num_heads = num_heads;
    args.group = num_heads / num_kv_heads;
    args.block_size = block_size;
    args.num_blocks = num_blocks;
    args.max_blocks_per_seq = max_blocks_per_seq;
    args.partition_tokens = ptok;
    args.num_partitions = (int)P;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (head_dim == 128)
        return dtype == PA_F16 ? launch_mha<F16Tag, 128>(args, num_seqs, k_cache, v_cache, num_kv_heads, st)
                               : launch_mha<BF16Tag, 128>(args, num_seqs, k_cache, v_cache, num_kv_heads, st);
    return dtype == PA_F16 ? launch_mha<F16Tag, 64>(args, num_seqs, k_cache, v_cache, num_kv_heads, st)
                           : launch_mha<BF16Tag, 64>(args, num_seqs, k_cache, v_cache, num_kv_heads, st);
}
