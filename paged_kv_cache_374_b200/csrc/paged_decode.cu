// K2 + K3: single-query (decode) attention over the paged KV cache.
//
// What is computed (P1 "大模型部署中的PagedAttention：KV Cache显存管理突破", §1, first
// formula; P3 "LLM 推理中的 PageAttention 实现原理", §二 and §三): for sequence s and
// query head h, out = softmax(scale * q K^T) V over the sequence's L tokens taken
// in logical order, token t living in physical block block_tables[s][t / B] at
// offset t % B -- one softmax over all L tokens.
//
// K2 is the persistent engine of decode_engine.cuh with one of two compute
// policies: CUDA cores per query head (decode_mha.cuh) when each kv head serves
// one query head, tensor cores per kv head (decode_gqa.cuh) when a group of query
// heads shares each kv head.  K3 (below) merges the partials of split sequences.
#include "decode_engine.cuh"
#include "decode_fp8tc.cuh"
#include "decode_gqa.cuh"
#include "decode_mha.cuh"
#include "pa_host.h"

// Tile configuration (compile-time; the defaults are the tuned ones).
#ifndef PA_DECODE_WARPS
#define PA_DECODE_WARPS 12       // warps (streaming engines) per CTA, one CTA per SM
#endif
#ifndef PA_DECODE_SLOTS
#define PA_DECODE_SLOTS 2        // shared-memory slots per warp
#endif
#ifndef PA_FP8TC_WARPS
#define PA_FP8TC_WARPS 12        // warps per CTA of the fp8 tensor-core engine (groups of up to 8)
#endif
#ifndef PA_FP8TC_SLOTS
#define PA_FP8TC_SLOTS 2         // its 32-token slots per warp
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
#ifndef PA_GQA_WARPS
#define PA_GQA_WARPS 12          // GQA path: warps per CTA
#endif
#ifndef PA_GQA_SLOTS
#define PA_GQA_SLOTS 2           // GQA path: shared-memory slots per warp
#endif
#ifndef PA_GQA_TOK
#define PA_GQA_TOK 16            // GQA path: tokens per slot (a multiple of 16)
#endif
#ifndef PA_GQA_MAX_GROUP
#define PA_GQA_MAX_GROUP 16      // largest group served by the tensor-core path
#endif

namespace pa {

// K3: merge the partitions of each (s, h) (base-2 units):
//   M = max_p m_p,  out = sum_p o_p 2^(m_p - M) / sum_p l_p 2^(m_p - M).
// One CTA of 8 warps per (s, h), one pass over the partials: each warp takes
// every 8th partition (each lane 4 dims, 16-byte loads, 4 partitions in flight)
// and keeps its own running max, rescaling its sums when the max grows; the 8
// warp results are combined with the same formula in shared memory.
//
// Launched as a programmatic dependent of K2, in one of two ways:
//   - early merge (DecodeArgs::early_merge): K2 lets this grid launch right after
//     its prologue, so its CTAs take the SMs K2's CTAs leave during K2's tail.
//     CTA b merges the b-th (s, h) whose partitions all landed (K2's merge queue,
//     in completion order), so merges overlap the partitions still streaming;
//     Behind the shared-prefix kernel, that kernel counts and queues the prefix
//     partitions it writes in the same way, and K2 raises its done flag only once
//     that kernel is complete;
//   - otherwise (a shared-prefix batch of more than one engine launch) every CTA
//     waits (griddepcontrol.wait) until K2 and all it waits for are complete, and
//     CTA b merges (s, h) = b.
constexpr int kMergeThreads = 256;

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Early merge, thread 0: the (s*H + h) queued in slot b, or -1 when the queue ends
// before slot b (or the wait gives up after about 2 s, reported as a timeout).
__device__ __forceinline__ int merge_claim(const DecodeArgs& a, int b) {
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0;; ++i) {
        int e = ld_acquire(a.merge_queue + b);
        if (e) return e - 1;
        if (ld_acquire(a.sched + 3)) {  // K2 is done: every entry it queued is visible
            e = ld_acquire(a.merge_queue + b);
            return e ? e - 1 : -1;
        }
        __nanosleep(256);
        if ((i & 63u) == 63u && global_ns() - t0 > 2000000000ull) {
            report(a.err_word, PA_DEVERR_TIMEOUT);
            return -1;
        }
    }
}

// Early merge, thread 0, after the CTA's merge: the last CTA to get here waits for
// K2's done flag, puts the queue state back to zero and does not let this grid
// complete before K2 has.
__device__ __forceinline__ void merge_retire(const DecodeArgs& a) {
    __threadfence();
    if (atomicAdd(a.sched + 4, 1) != (int)gridDim.x - 1) return;
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0; !ld_acquire(a.sched + 3); ++i) {
        __nanosleep(256);
        if ((i & 63u) == 63u && global_ns() - t0 > 2000000000ull) {
            report(a.err_word, PA_DEVERR_TIMEOUT);
            return;
        }
    }
    a.sched[2] = 0;
    a.sched[3] = 0;
    a.sched[4] = 0;
    __threadfence();
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

template <class Tag, int D>
__device__ __forceinline__ void merge_pair(const DecodeArgs& a, int64_t sh) {
    constexpr int NWM = kMergeThreads / 32;
    constexpr int BATCH = 4;
    __shared__ float s_m[NWM], s_l[NWM];
    __shared__ float4 s_acc[NWM][D / 4];
    const int s = (int)(sh / a.num_heads);
    const int L = a.context_lens[s];
    if (L <= 0 || L > a.max_blocks_per_seq * a.block_size) return;  // rows written by K2
    const int nparts = (L + a.partition_tokens - 1) / a.partition_tokens;
    if (nparts <= 1) return;
    const float* pm = a.ws_m + sh * a.num_partitions;
    const float* pl = a.ws_l + sh * a.num_partitions;
    const float4* po = reinterpret_cast<const float4*>(a.ws_o + sh * a.num_partitions * D);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool active = lane < D / 4;

    float m = -INFINITY, l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = warp; p0 < nparts; p0 += NWM * BATCH) {
        float mb[BATCH], lb[BATCH];
        float4 ob[BATCH];
#pragma unroll
        for (int j = 0; j < BATCH; ++j) {  // loads of BATCH partitions first
            const int p = p0 + j * NWM;
            const bool in = p < nparts;
            // L2 loads: with an early merge the partials were written by CTAs that ran
            // beside this one
            mb[j] = in ? __ldcg(pm + p) : -INFINITY;
            lb[j] = in ? __ldcg(pl + p) : 0.f;
            ob[j] = (in && active) ? __ldcg(po + (int64_t)p * (D / 4) + lane) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < BATCH; ++j) {
            if (mb[j] == -INFINITY) continue;  // partition absent (warp-uniform)
            if (mb[j] > m) {
                const float alpha = exp2f(m - mb[j]);
                l *= alpha;
                acc.x *= alpha;
                acc.y *= alpha;
                acc.z *= alpha;
                acc.w *= alpha;
                m = mb[j];
            }
            const float w = exp2f(mb[j] - m);
            l = fmaf(w, lb[j], l);
            acc.x = fmaf(w, ob[j].x, acc.x);
            acc.y = fmaf(w, ob[j].y, acc.y);
            acc.z = fmaf(w, ob[j].z, acc.z);
            acc.w = fmaf(w, ob[j].w, acc.w);
        }
    }
    if (lane == 0) {
        s_m[warp] = m;
        s_l[warp] = l;
    }
    if (active) s_acc[warp][lane] = acc;
    __syncthreads();
    if (tid < D / 4) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NWM; ++w) M = fmaxf(M, s_m[w]);
        float den = 0.f;
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < NWM; ++w) {
            const float sc = s_m[w] == -INFINITY ? 0.f : exp2f(s_m[w] - M);
            den = fmaf(sc, s_l[w], den);
            const float4 v = s_acc[w][tid];
            t.x = fmaf(sc, v.x, t.x);
            t.y = fmaf(sc, v.y, t.y);
            t.z = fmaf(sc, v.z, t.z);
            t.w = fmaf(sc, v.w, t.w);
        }
        const float inv = 1.f / den;
        uint2 packed;
        packed.x = pack2<Tag>(t.x * inv, t.y * inv);
        packed.y = pack2<Tag>(t.z * inv, t.w * inv);
        reinterpret_cast<uint2*>(a.out + sh * D)[tid] = packed;
    }
}

template <class Tag, int D>
__global__ void __launch_bounds__(kMergeThreads) paged_decode_merge_kernel(const DecodeArgs a) {
    // The next step's cache write, launched as a programmatic dependent, may be
    // scheduled now: it waits for this grid to complete before it does anything.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!a.early_merge) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        merge_pair<Tag, D>(a, blockIdx.x);
        return;
    }
    __shared__ int s_sh;
    if (threadIdx.x == 0) s_sh = merge_claim(a, blockIdx.x);
    __syncthreads();
    const int sh = s_sh;
    if (sh >= 0) {
        merge_pair<Tag, D>(a, sh);
        if (threadIdx.x == 0) {  // left zero for the next launch
            a.merge_cnt[sh] = 0;
            a.merge_queue[blockIdx.x] = 0;
        }
    }
    if (threadIdx.x == 0) merge_retire(a);
}

namespace {

constexpr int kDefaultPartition = PA_DECODE_PARTITION;
constexpr size_t kSchedBytes = 256;

int64_t num_partitions(int max_blocks_per_seq, int block_size, int ptok) {
    const int64_t max_len = (int64_t)max_blocks_per_seq * block_size;
    return max_len <= 0 ? 1 : (max_len + ptok - 1) / ptok;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// Counters (left zero by every call) then partials:
//   [0, 256)           scheduling counters (DecodeArgs::sched)
//   when P > 1: merge_cnt int32 [S*H], merge_queue int32 [S*H], then the
//   partials m, l fp32 [S*H][P] and o fp32 [S*H][P][D].
size_t counter_bytes_for(int64_t sh, int64_t P) {
    if (P <= 1) return kSchedBytes;
    return kSchedBytes + 2 * up256(sh * 4);
}

size_t workspace_bytes_for(int64_t sh, int64_t P, int D) {
    if (P <= 1) return kSchedBytes;
    return counter_bytes_for(sh, P) + up256(sh * P * 4) * 2 + up256(sh * P * D * 4);
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

template <class Tag, class CTag, int D, int TOK, int NW, int R, class Policy>
int launch_engine(DecodeArgs args, const void* k_cache, const void* v_cache, int num_kv_heads,
                  cudaStream_t stream) {
    using Lay = Layout<D * CTag::kBytes, TOK, NW, R, Policy::kScratchBytes>;
    static_assert(Lay::kAlloc <= 227 * 1024, "shared memory");
    static std::atomic<uint64_t> smem_done{0};
    auto kernel = paged_decode_kernel<Tag, CTag, D, TOK, NW, R, Policy>;
    if (ensure_smem_limit(kernel, Lay::kAlloc, smem_done) != cudaSuccess) return PA_ERR_CUDA;
    args.box_rows = TOK < args.block_size ? TOK : args.block_size;
    const int64_t total_tokens = (int64_t)args.num_blocks * args.block_size;
    CUtensorMap kmap, vmap;
    if (!encode_cache_map_swizzled(&kmap, k_cache, D, num_kv_heads, total_tokens, args.box_rows, CTag::kBytes) ||
        !encode_cache_map_swizzled(&vmap, v_cache, D, num_kv_heads, total_tokens, args.box_rows, CTag::kBytes))
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
        if (c.seq_start) c.seq_start += s0;
        if (args.num_partitions > 1) {
            c.ws_m += shoff * args.num_partitions;
            c.ws_l += shoff * args.num_partitions;
            c.ws_o += shoff * args.num_partitions * D;
        }
        if ((c.seq_start || c.wait_prior) && s0 == 0) {
            // behind the shared-prefix kernel (start on the SMs it leaves free) or
            // behind the step's cache write (overlap its launch and prologue)
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)sms);
            cfg.blockDim = dim3(NW * 32);
            cfg.dynamicSmemBytes = Lay::kAlloc;
            cfg.stream = stream;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[0].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaLaunchKernelEx(&cfg, kernel, c, kmap, vmap) != cudaSuccess) return PA_ERR_CUDA;
        } else {
            kernel<<<sms, NW * 32, Lay::kAlloc, stream>>>(c, kmap, vmap);
            if (cudaGetLastError() != cudaSuccess) return PA_ERR_CUDA;
        }
        if (args.num_partitions > 1) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3((unsigned)((int64_t)c.num_seqs * args.num_heads));
            cfg.blockDim = dim3(kMergeThreads);
            cfg.stream = stream;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr[0].val.programmaticStreamSerializationAllowed = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            if (cudaLaunchKernelEx(&cfg, paged_decode_merge_kernel<Tag, D>, c) != cudaSuccess) return PA_ERR_CUDA;
        }
    }
    return PA_OK;
}

template <class Tag, int D>
int launch_decode(DecodeArgs args, const void* k_cache, const void* v_cache, int num_kv_heads,
                  cudaStream_t stream) {
    constexpr int R = PA_DECODE_SLOTS;
    if (args.group >= 2 && args.group <= PA_GQA_MAX_GROUP) {
        constexpr int TOK = PA_GQA_TOK;
        constexpr int GR = PA_GQA_SLOTS;
        args.unit_heads = num_kv_heads;
        args.heads_per_unit = args.group;
        if (args.group <= 8)
            return launch_engine<Tag, Tag, D, TOK, PA_GQA_WARPS, GR, GqaPolicy<Tag, D, TOK, 1>>(
                args, k_cache, v_cache, num_kv_heads, stream);
        // two head tiles need more registers per thread: at most 8 warps per CTA
        constexpr int NW2 = PA_GQA_WARPS < 8 ? PA_GQA_WARPS : 8;
        return launch_engine<Tag, Tag, D, TOK, NW2, GR, GqaPolicy<Tag, D, TOK, 2>>(args, k_cache, v_cache,
                                                                                   num_kv_heads, stream);
    }
    constexpr int TOK = D == 128 ? PA_DECODE_TOK128 : PA_DECODE_TOK64;
    args.unit_heads = args.num_heads;
    args.heads_per_unit = 1;
    return launch_engine<Tag, Tag, D, TOK, PA_DECODE_WARPS, R, MhaPolicy<Tag, Tag, D, TOK>>(args, k_cache, v_cache,
                                                                                            num_kv_heads, stream);
}

// fp8 (E4M3) caches.  GQA groups of 2-16: tensor cores, one kv head with its whole
// query group per unit (one fetch of the codes serves the group), codes converted
// from the landed stage straight into MMA fragments.  MHA (and larger groups):
// CUDA cores, one query head per unit: with a single head the tensor-core stage
// carries too little work per byte to keep up.
template <class Tag>
int launch_decode_fp8(DecodeArgs args, const void* k_cache, const void* v_cache, int num_kv_heads,
                      cudaStream_t stream) {
    // 32-token slots of codes (8 KiB for K and V).  Groups of up to 8 run 12 warps (192 KiB
    // of codes in flight per SM, 166 registers); groups of 9-16 hold twice the accumulators
    // (255 registers) and run 8 warps.
    constexpr int TOK = 32;
    if (args.group >= 2 && args.group <= PA_GQA_MAX_GROUP) {
        args.unit_heads = num_kv_heads;
        args.heads_per_unit = args.group;
        if (args.group <= 8)
            return launch_engine<Tag, E4M3Tag, 128, TOK, PA_FP8TC_WARPS, PA_FP8TC_SLOTS, Fp8TcPolicy<Tag, TOK, 1>>(
                args, k_cache, v_cache, num_kv_heads, stream);
        return launch_engine<Tag, E4M3Tag, 128, TOK, 8, 2, Fp8TcPolicy<Tag, TOK, 2>>(args, k_cache, v_cache,
                                                                                       num_kv_heads, stream);
    }
    args.unit_heads = args.num_heads;
    args.heads_per_unit = 1;
    return launch_engine<Tag, E4M3Tag, 128, TOK, PA_DECODE_WARPS, PA_DECODE_SLOTS, MhaPolicy<Tag, E4M3Tag, 128, TOK>>(
        args, k_cache, v_cache, num_kv_heads, stream);
}

}  // namespace
}  // namespace pa

extern "C" int pa_decode_partition_tokens(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                          int block_size, int max_blocks_per_seq) {
    (void)num_seqs; (void)num_heads; (void)num_kv_heads; (void)head_dim; (void)block_size;
    (void)max_blocks_per_seq;
    return pa::kDefaultPartition;
}

namespace pa {
size_t decode_counter_bytes(int num_seqs, int num_heads, int block_size, int max_blocks_per_seq, int partition_tokens) {
    const int ptok = partition_tokens > 0 ? partition_tokens : kDefaultPartition;
    return counter_bytes_for((int64_t)num_seqs * num_heads, num_partitions(max_blocks_per_seq, block_size, ptok));
}
}  // namespace pa

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

namespace pa {
namespace {

// Checks shared by pa_decode and pa_decode_fp8; fills args on success.
int prepare_decode(DecodeArgs& args, const void* q, const void* k_cache, const void* v_cache,
                   const int32_t* block_tables, const int32_t* context_lens, float scale, int num_kv_heads,
                   void* out, int num_seqs, int num_heads, int head_dim, int block_size, int num_blocks,
                   int max_blocks_per_seq, int dtype, int partition_tokens, void* workspace,
                   size_t workspace_bytes, int32_t* err_word) {
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

    args = DecodeArgs{};
    args.q = static_cast<const uint16_t*>(q);
    args.out = static_cast<uint16_t*>(out);
    args.block_tables = block_tables;
    args.context_lens = context_lens;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    args.sched = reinterpret_cast<int32_t*>(w);
    if (P > 1) {
        const size_t c0 = counter_bytes_for(SH, P);
        args.merge_cnt = reinterpret_cast<int32_t*>(w + kSchedBytes);
        args.merge_queue = reinterpret_cast<int32_t*>(w + kSchedBytes + up256(SH * 4));
        args.ws_m = reinterpret_cast<float*>(w + c0);
        args.ws_l = reinterpret_cast<float*>(w + c0 + up256(SH * P * 4));
        args.ws_o = reinterpret_cast<float*>(w + c0 + 2 * up256(SH * P * 4));
        args.early_merge = 1;  // cleared for the shared-prefix path
    }
    args.err_word = err_word;
    args.scale_log2 = scale * 1.4426950408889634f;
    args.k_scale = 1.f;
    args.v_scale = 1.f;
    args.num_seqs = num_seqs;
    args.num_heads = num_heads;
    args.group = num_heads / num_kv_heads;
    args.block_size = block_size;
    args.num_blocks = num_blocks;
    args.max_blocks_per_seq = max_blocks_per_seq;
    args.partition_tokens = ptok;
    args.num_partitions = (int)P;
    return -1;  // ready to launch
}

}  // namespace

int check_decode_call(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                      const int32_t* context_lens, int num_kv_heads, const void* out, int num_seqs, int num_heads,
                      int head_dim, int block_size, int num_blocks, int max_blocks_per_seq, int dtype,
                      int partition_tokens, const int32_t* err_word) {
    // pa_decode's checks with a stand-in workspace that is present, aligned and
    // large enough: no pointer is dereferenced and nothing is launched.
    DecodeArgs args;
    return prepare_decode(args, q, k_cache, v_cache, block_tables, context_lens, 1.f, num_kv_heads,
                          const_cast<void*>(out), num_seqs, num_heads, head_dim, block_size, num_blocks,
                          max_blocks_per_seq, dtype, partition_tokens, reinterpret_cast<void*>(uintptr_t{256}),
                          SIZE_MAX, const_cast<int32_t*>(err_word));
}

}  // namespace pa

extern "C" int pa_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                         const int32_t* context_lens, float scale, int num_kv_heads, void* out, int num_seqs,
                         int num_heads, int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                         int dtype, int partition_tokens, void* workspace, size_t workspace_bytes,
                         int32_t* err_word, void* stream) {
    using namespace pa;
    DecodeArgs args;
    const int rc = prepare_decode(args, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, out,
                                  num_seqs, num_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype,
                                  partition_tokens, workspace, workspace_bytes, err_word);
    if (rc >= 0) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (head_dim == 128)
        return dtype == PA_F16 ? launch_decode<F16Tag, 128>(args, k_cache, v_cache, num_kv_heads, st)
                               : launch_decode<BF16Tag, 128>(args, k_cache, v_cache, num_kv_heads, st);
    return dtype == PA_F16 ? launch_decode<F16Tag, 64>(args, k_cache, v_cache, num_kv_heads, st)
                           : launch_decode<BF16Tag, 64>(args, k_cache, v_cache, num_kv_heads, st);
}

extern "C" int pa_decode_fp8(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                             const int32_t* context_lens, float scale, float k_scale, float v_scale,
                             int num_kv_heads, void* out, int num_seqs, int num_heads, int head_dim, int block_size,
                             int num_blocks, int max_blocks_per_seq, int dtype, int partition_tokens,
                             void* workspace, size_t workspace_bytes, int32_t* err_word, void* stream) {
    using namespace pa;
    if (head_dim != 128) return PA_ERR_UNSUPPORTED;  // 128-byte rows: one swizzled TMA box per row
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !isfinite(k_scale) || !isfinite(v_scale)) return PA_ERR_INVALID_ARG;
    DecodeArgs args;
    const int rc = prepare_decode(args, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, out,
                                  num_seqs, num_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype,
                                  partition_tokens, workspace, workspace_bytes, err_word);
    if (rc >= 0) return rc;
    args.k_scale = k_scale;
    args.v_scale = v_scale;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    return dtype == PA_F16 ? launch_decode_fp8<F16Tag>(args, k_cache, v_cache, num_kv_heads, st)
                           : launch_decode_fp8<BF16Tag>(args, k_cache, v_cache, num_kv_heads, st);
}

namespace pa {
namespace {

// The checks of pa_decode_shared_prefix's group arguments, after prepare_decode
// filled args.  Sets *shared when the prefix kernel runs; returns -1 when the call
// may go on, else the status to return.
int check_shared_prefix(const DecodeArgs& args, const int32_t* seq_start, int num_groups,
                        const int32_t* group_offsets, const int32_t* group_members, int max_group_size,
                        int max_shared_tokens, bool* shared) {
    *shared = num_groups > 0 && max_shared_tokens > 0 && args.num_partitions > 1;
    if (*shared && (!seq_start || !group_offsets || !group_members || !aligned4(seq_start) ||
                    !aligned4(group_offsets) || !aligned4(group_members) || max_group_size <= 0 ||
                    max_shared_tokens % args.partition_tokens != 0))
        return PA_ERR_INVALID_ARG;
    if (*shared && (num_groups > 65535 || args.num_heads / args.group > 65535))
        return PA_ERR_UNSUPPORTED;  // the prefix kernel's grid (groups, kv heads)
    return -1;
}

// The prefix kernel (when *shared) and then the decode engine and merge.
// after_write: the cache write of the same step was launched just before; the
// prefix kernel runs as its programmatic dependent and holds the engine's launch
// until the write is complete, or, with no prefix kernel, the engine waits for it.
int launch_shared_prefix_decode(DecodeArgs args, bool shared, const void* q, const void* k_cache,
                                const void* v_cache, const int32_t* block_tables, const int32_t* context_lens,
                                float scale, int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                                int block_size, int num_blocks, int max_blocks_per_seq, int dtype,
                                const int32_t* seq_start, int num_groups, const int32_t* group_offsets,
                                const int32_t* group_members, int max_group_size, int max_shared_tokens,
                                int32_t* err_word, bool after_write, cudaStream_t st) {
    if (shared) {
        SharedPrefixLaunch l{};
        l.q = q;
        l.k_cache = k_cache;
        l.v_cache = v_cache;
        l.block_tables = block_tables;
        l.context_lens = context_lens;
        l.seq_start = seq_start;
        l.group_offsets = group_offsets;
        l.group_members = group_members;
        l.ws_m = args.ws_m;
        l.ws_l = args.ws_l;
        l.ws_o = args.ws_o;
        l.err_word = err_word;
        l.scale = scale;
        l.num_heads = num_heads;
        l.num_kv_heads = num_kv_heads;
        l.head_dim = head_dim;
        l.block_size = block_size;
        l.num_blocks = num_blocks;
        l.max_blocks_per_seq = max_blocks_per_seq;
        l.dtype = dtype;
        l.partition_tokens = args.partition_tokens;
        l.num_partitions = args.num_partitions;
        l.num_groups = num_groups;
        l.max_group_size = max_group_size;
        l.max_shared_tokens = max_shared_tokens;
        l.num_seqs = num_seqs;
        // both kernels count partitions by (s, h) in one index space only when the
        // engine runs in a single launch
        args.early_merge = num_seqs <= kMaxSeqsPerLaunch ? 1 : 0;
        l.early_merge = args.early_merge;
        l.sched = args.sched;
        l.merge_cnt = args.merge_cnt;
        l.merge_queue = args.merge_queue;
        l.after_write = after_write ? 1 : 0;
        const int r = launch_shared_prefix(l, st);
        if (r != PA_OK) return r;
        args.seq_start = seq_start;
    } else if (after_write) {
        args.wait_prior = 1;
    }
    if (head_dim == 128)
        return dtype == PA_F16 ? launch_decode<F16Tag, 128>(args, k_cache, v_cache, num_kv_heads, st)
                               : launch_decode<BF16Tag, 128>(args, k_cache, v_cache, num_kv_heads, st);
    return dtype == PA_F16 ? launch_decode<F16Tag, 64>(args, k_cache, v_cache, num_kv_heads, st)
                           : launch_decode<BF16Tag, 64>(args, k_cache, v_cache, num_kv_heads, st);
}

}  // namespace
}  // namespace pa

extern "C" int pa_decode_shared_prefix(const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, const int32_t* context_lens, float scale,
                                       int num_kv_heads, void* out, int num_seqs, int num_heads, int head_dim,
                                       int block_size, int num_blocks, int max_blocks_per_seq, int dtype,
                                       const int32_t* seq_start, int num_groups, const int32_t* group_offsets,
                                       const int32_t* group_members, int max_group_size, int max_shared_tokens,
                                       int partition_tokens, void* workspace, size_t workspace_bytes,
                                       int32_t* err_word, void* stream) {
    using namespace pa;
    if (num_groups < 0 || max_group_size < 0 || max_shared_tokens < 0) return PA_ERR_INVALID_ARG;
    DecodeArgs args;
    const int rc = prepare_decode(args, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, out,
                                  num_seqs, num_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype,
                                  partition_tokens, workspace, workspace_bytes, err_word);
    if (rc >= 0) return rc;
    bool shared = false;
    const int rs = check_shared_prefix(args, seq_start, num_groups, group_offsets, group_members, max_group_size,
                                       max_shared_tokens, &shared);
    if (rs >= 0) return rs;
    return launch_shared_prefix_decode(args, shared, q, k_cache, v_cache, block_tables, context_lens, scale,
                                       num_kv_heads, num_seqs, num_heads, head_dim, block_size, num_blocks,
                                       max_blocks_per_seq, dtype, seq_start, num_groups, group_offsets,
                                       group_members, max_group_size, max_shared_tokens, err_word, false,
                                       static_cast<cudaStream_t>(stream));
}

extern "C" int pa_decode_step_shared_prefix(const void* k, const void* v, const int64_t* slot_mapping, const void* q,
                                            void* k_cache, void* v_cache, const int32_t* block_tables,
                                            const int32_t* context_lens, float scale, int num_kv_heads, void* out,
                                            int num_seqs, int num_heads, int head_dim, int block_size,
                                            int num_blocks, int max_blocks_per_seq, int dtype,
                                            const int32_t* seq_start, int num_groups, const int32_t* group_offsets,
                                            const int32_t* group_members, int max_group_size,
                                            int max_shared_tokens, int partition_tokens, void* workspace,
                                            size_t workspace_bytes, int32_t* err_word, void* stream) {
    using namespace pa;
    // every check of both calls before anything is launched
    if (num_groups < 0 || max_group_size < 0 || max_shared_tokens < 0) return PA_ERR_INVALID_ARG;
    const int rk = check_reshape_and_cache(k, v, slot_mapping, k_cache, v_cache, num_seqs, num_kv_heads, head_dim,
                                           block_size, num_blocks, dtype, err_word);
    if (rk > 0) return rk;
    DecodeArgs args;
    const int rc = prepare_decode(args, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, out,
                                  num_seqs, num_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype,
                                  partition_tokens, workspace, workspace_bytes, err_word);
    if (rc >= 0) return rc;  // an error, or an empty batch (num_seqs == 0: nothing to write either)
    bool shared = false;
    const int rs = check_shared_prefix(args, seq_start, num_groups, group_offsets, group_members, max_group_size,
                                       max_shared_tokens, &shared);
    if (rs >= 0) return rs;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int r1 = launch_reshape_and_cache(k, v, slot_mapping, k_cache, v_cache, num_seqs, num_kv_heads, head_dim,
                                            block_size, num_blocks, err_word, st);
    if (r1 != PA_OK) return r1;
    return launch_shared_prefix_decode(args, shared, q, k_cache, v_cache, block_tables, context_lens, scale,
                                       num_kv_heads, num_seqs, num_heads, head_dim, block_size, num_blocks,
                                       max_blocks_per_seq, dtype, seq_start, num_groups, group_offsets,
                                       group_members, max_group_size, max_shared_tokens, err_word, true, st);
}

extern "C" int pa_decode_step(const void* k, const void* v, const int64_t* slot_mapping, const void* q,
                              void* k_cache, void* v_cache, const int32_t* block_tables,
                              const int32_t* context_lens, float scale, int num_kv_heads, void* out, int num_seqs,
                              int num_heads, int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                              int dtype, int partition_tokens, void* workspace, size_t workspace_bytes,
                              int32_t* err_word, void* stream) {
    using namespace pa;
    // every check of both calls before anything is launched
    const int rk = check_reshape_and_cache(k, v, slot_mapping, k_cache, v_cache, num_seqs, num_kv_heads, head_dim,
                                           block_size, num_blocks, dtype, err_word);
    if (rk > 0) return rk;
    DecodeArgs args;
    const int rc = prepare_decode(args, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, out,
                                  num_seqs, num_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype,
                                  partition_tokens, workspace, workspace_bytes, err_word);
    if (rc >= 0) return rc;  // an error, or an empty batch (num_seqs == 0: nothing to write either)
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int r1 = launch_reshape_and_cache(k, v, slot_mapping, k_cache, v_cache, num_seqs, num_kv_heads, head_dim,
                                            block_size, num_blocks, err_word, st);
    if (r1 != PA_OK) return r1;
    args.wait_prior = 1;
    if (head_dim == 128)
        return dtype == PA_F16 ? launch_decode<F16Tag, 128>(args, k_cache, v_cache, num_kv_heads, st)
                               : launch_decode<BF16Tag, 128>(args, k_cache, v_cache, num_kv_heads, st);
    return dtype == PA_F16 ? launch_decode<F16Tag, 64>(args, k_cache, v_cache, num_kv_heads, st)
                           : launch_decode<BF16Tag, 64>(args, k_cache, v_cache, num_kv_heads, st);
}

extern "C" int pa_decode_step_fp8(const void* k, const void* v, const int64_t* slot_mapping, const void* q,
                                  void* k_cache, void* v_cache, const int32_t* block_tables,
                                  const int32_t* context_lens, float scale, float k_scale, float v_scale,
                                  int num_kv_heads, void* out, int num_seqs, int num_heads, int head_dim,
                                  int block_size, int num_blocks, int max_blocks_per_seq, int dtype,
                                  int partition_tokens, void* workspace, size_t workspace_bytes, int32_t* err_word,
                                  void* stream) {
    using namespace pa;
    if (head_dim != 128) return PA_ERR_UNSUPPORTED;
    const int rk = check_reshape_and_cache_fp8(k, v, slot_mapping, k_cache, v_cache, num_seqs, num_kv_heads,
                                               head_dim, block_size, num_blocks, dtype, k_scale, v_scale, err_word);
    if (rk > 0) return rk;
    DecodeArgs args;
    const int rc = prepare_decode(args, q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, out,
                                  num_seqs, num_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype,
                                  partition_tokens, workspace, workspace_bytes, err_word);
    if (rc >= 0) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int r1 = launch_reshape_and_cache_fp8(k, v, slot_mapping, k_cache, v_cache, num_seqs, num_kv_heads,
                                                head_dim, block_size, num_blocks, dtype, k_scale, v_scale, err_word,
                                                st);
    if (r1 != PA_OK) return r1;
    args.k_scale = k_scale;
    args.v_scale = v_scale;
    args.wait_prior = 1;
    return dtype == PA_F16 ? launch_decode_fp8<F16Tag>(args, k_cache, v_cache, num_kv_heads, st)
                           : launch_decode_fp8<BF16Tag>(args, k_cache, v_cache, num_kv_heads, st);
}
