// Paged prefill: causal attention of a chunk of new query tokens over the paged
// cache -- the step before decode (P2 "大模型推理优化：KV Cache与PagedAttention技术详解",
// §2.1: the prompt's K/V enter the cache, then every position attends to the ones
// before it; prefix reuse across requests, P3 §三, makes the chunk start after
// cached tokens).  Query row i of sequence s (chunk of n rows over L tokens) sits
// at position L - n + i and attends to tokens 0 .. L - n + i through the table.
//
// A real dense contraction, run on tensor cores (mma.sync m16n8k16, 16-bit inputs,
// fp32 accumulation): one CTA = 64 query rows of one head (4 warps x 16 rows),
// streaming 64-token K/V tiles of its kv head through a two-stage TMA ring (the
// 128-byte-swizzled tensor maps of the decode path, one mbarrier per stage).  Per
// tile: S = Q K^T (K via ldmatrix), causal mask, online softmax per row in base 2,
// O += P V (V via ldmatrix.trans; P taken straight from the S accumulators and
// fed as two 16-bit terms, hi + lo, so p keeps about 16 significant bits).
// Tokens past the sequence end are zeroed in the V fragments (0 * NaN is NaN in an
// MMA); table entries are checked once, up front.
#include <cmath>

#include "decode_gqa.cuh"
#include "pa_host.h"

namespace pa {

constexpr int kPfRows = 64;          // query rows per CTA
constexpr int kPfTok = 64;           // tokens per K/V tile
constexpr int kPfThreads = 128;
constexpr int kPfMaxEntries = 4096;  // table entries a CTA can hold

struct PrefillArgs {
    const uint16_t* q;    // [T][H][D]
    uint16_t* out;        // [T][H][D]
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* query_start;  // [S + 1]
    int32_t* err_word;
    float scale_log2;
    int num_heads, group, block_size, box_rows, num_blocks, max_blocks_per_seq;
};

template <int D>
struct PfLayout {
    static constexpr int kTile = kPfTok * D * 2;       // one K or V tile
    static constexpr int kHalf = kPfTok * 128;         // one 64-dim half of a tile
    static constexpr int kStage = 2 * kTile;           // K then V
    static constexpr int kOffBars = 2 * kStage;
    static constexpr int kOffTab = kOffBars + 16;
    static constexpr int kBytes = kOffTab + kPfMaxEntries * 4;
    static constexpr int kAlloc = kBytes + 1024;
};

template <class Tag, int D>
__global__ void __launch_bounds__(kPfThreads) paged_prefill_kernel(const PrefillArgs a,
                                                                   const __grid_constant__ CUtensorMap kmap,
                                                                   const __grid_constant__ CUtensorMap vmap) {
    using Lay = PfLayout<D>;
    using Ops = MmaOps<Tag>;
    constexpr int KS = D / 16;  // k-steps of q K^T
    constexpr int DN = D / 8;   // 8-dim output tiles
    constexpr int NT = kPfTok / 8;  // 8-token score tiles per K tile
    constexpr unsigned FULL = 0xffffffffu;

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kOffBars);
    int32_t* s_tab = reinterpret_cast<int32_t*>(smem + Lay::kOffTab);

    const int s = blockIdx.z, h = blockIdx.y;
    const int qt = gridDim.x - 1 - blockIdx.x;  // tiles with the most context first
    const int q0 = a.query_start[s];
    const int n = a.query_start[s + 1] - q0;
    if (qt * kPfRows >= n) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int L = a.context_lens[s];
    const int bs = a.block_size;
    const int q_first = qt * kPfRows;
    const int q_last = min(n, q_first + kPfRows) - 1;
    auto write_rows = [&](float value) {
        for (int i = tid; i < (q_last - q_first + 1) * D; i += kPfThreads) {
            const int r = q_first + i / D;
            a.out[((int64_t)(q0 + r) * a.num_heads + h) * D + i % D] = Tag::round1(value);
        }
    };
    if (L < 0 || L > a.max_blocks_per_seq * bs || n > L) {
        write_rows(__int_as_float(0x7fc00000));
        if (tid == 0) report(a.err_word, PA_DEVERR_LEN_RANGE);
        return;
    }
    const int base_pos = L - n;
    const int pos_last = base_pos + q_last;
    const int ntiles = pos_last / kPfTok + 1;
    const int kv_head = h / a.group;
    const int nent = (min(ntiles * kPfTok, L) + bs - 1) / bs;  // table entries the tiles read

    // table entries, checked once
    bool bad = false;
    for (int i = tid; i < nent; i += kPfThreads) {
        const int id = a.block_tables[(int64_t)s * a.max_blocks_per_seq + i];
        s_tab[i] = id;
        bad |= id < 0 || id >= a.num_blocks;
    }
    if (tid == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
    }
    if (__syncthreads_or(bad)) {
        write_rows(__int_as_float(0x7fc00000));
        if (tid == 0) report(a.err_word, PA_DEVERR_TABLE_RANGE);
        return;
    }

    const int br = a.box_rows;
    auto issue = [&](int tile, int st) {  // thread 0 only
        uint8_t* kd = smem + st * Lay::kStage;
        uint32_t tx = 0;
        for (int j = 0; j * br < kPfTok; ++j)
            if (tile * kPfTok + j * br < L) tx += 2u * (D / 64) * br * 128;
        mbar_arrive_expect_tx(&bars[st], tx);
        for (int j = 0; j * br < kPfTok; ++j) {
            const int tj = tile * kPfTok + j * br;
            if (tj >= L) break;
            const int row = s_tab[tj / bs] * bs + tj % bs;
#pragma unroll
            for (int hh = 0; hh < D / 64; ++hh) {
                uint8_t* dst = kd + hh * Lay::kHalf + j * br * 128;
                tma_load_3d(dst, &kmap, hh * 64, kv_head, row, &bars[st]);
                tma_load_3d(dst + Lay::kTile, &vmap, hh * 64, kv_head, row, &bars[st]);
            }
        }
    };
    if (tid == 0) {
        issue(0, 0);
        if (ntiles > 1) issue(1, 1);
    }

    // this warp's 16 query rows: g and g + 8; rows past the chunk act as its last row
    const int row0 = q_first + warp * 16 + g, row1 = row0 + 8;
    const int pos0 = base_pos + min(row0, n - 1), pos1 = base_pos + min(row1, n - 1);
    uint32_t qa[KS][4];
    {
        const uint32_t* p0 = reinterpret_cast<const uint32_t*>(a.q + ((int64_t)(q0 + min(row0, n - 1)) * a.num_heads + h) * D);
        const uint32_t* p1 = reinterpret_cast<const uint32_t*>(a.q + ((int64_t)(q0 + min(row1, n - 1)) * a.num_heads + h) * D);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            qa[ks][0] = __ldg(p0 + ks * 8 + t);
            qa[ks][1] = __ldg(p1 + ks * 8 + t);
            qa[ks][2] = __ldg(p0 + ks * 8 + 4 + t);
            qa[ks][3] = __ldg(p1 + ks * 8 + 4 + t);
        }
    }
    float o[DN][4];
#pragma unroll
    for (int dn = 0; dn < DN; ++dn) o[dn][0] = o[dn][1] = o[dn][2] = o[dn][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    int stopped_at = -1;  // tile whose wait gave up (the decision is CTA-uniform)

    for (int it = 0; it < ntiles; ++it) {
        const int st = it & 1;
        const bool ok = __all_sync(FULL, mbar_wait(&bars[st], (it >> 1) & 1));
        if (__syncthreads_or(!ok)) {
            stopped_at = it;
            break;
        }
        const uint8_t* kt = smem + st * Lay::kStage;
        const uint8_t* vt = kt + Lay::kTile;
        const int tile_base = it * kPfTok;
        // ---- S = Q K^T
        float sc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
                const int tok = np * 16 + (lane & 7) + ((lane >> 4) & 1) * 8;
                const int ch = ks * 2 + ((lane >> 3) & 1);
                uint32_t b[4];
                ldsm_x4(b, kt + (ch >> 3) * Lay::kHalf + tok * 128 + (((ch & 7) ^ (lane & 7)) << 4));
                Ops::mma(sc[2 * np], qa[ks], b[0], b[1]);
                Ops::mma(sc[2 * np + 1], qa[ks], b[2], b[3]);
            }
        }
        // ---- causal mask, online softmax (rows g and g+8)
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int tk = tile_base + nt * 8 + 2 * t;
            sc[nt][0] = tk <= pos0 ? sc[nt][0] * a.scale_log2 : -INFINITY;
            sc[nt][1] = tk + 1 <= pos0 ? sc[nt][1] * a.scale_log2 : -INFINITY;
            sc[nt][2] = tk <= pos1 ? sc[nt][2] * a.scale_log2 : -INFINITY;
            sc[nt][3] = tk + 1 <= pos1 ? sc[nt][3] * a.scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, fmaxf(sc[nt][0], sc[nt][1]));
            mx1 = fmaxf(mx1, fmaxf(sc[nt][2], sc[nt][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(FULL, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(FULL, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);  // finite: token 0 is always visible
        const float al0 = fast_exp2(m0 - mn0), al1 = fast_exp2(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        l0 *= al0;
        l1 *= al1;
#pragma unroll
        for (int dn = 0; dn < DN; ++dn) {
            o[dn][0] *= al0;
            o[dn][1] *= al0;
            o[dn][2] *= al1;
            o[dn][3] *= al1;
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            sc[nt][0] = fast_exp2(sc[nt][0] - m0);
            sc[nt][1] = fast_exp2(sc[nt][1] - m0);
            sc[nt][2] = fast_exp2(sc[nt][2] - m1);
            sc[nt][3] = fast_exp2(sc[nt][3] - m1);
            l0 += sc[nt][0] + sc[nt][1];
            l1 += sc[nt][2] + sc[nt][3];
        }
        // ---- O += P V, 16 tokens at a time
        const bool tail = tile_base + kPfTok > L;  // some tokens of this tile are past the sequence end
#pragma unroll
        for (int kk = 0; kk < kPfTok / 16; ++kk) {
            uint32_t ph[4], pl[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float* src = &sc[2 * kk + (j >> 1)][(j & 1) * 2];
                ph[j] = Ops::pack(src[0], src[1]);
                const float2 hv = Tag::widen2(ph[j]);
                pl[j] = Ops::pack(src[0] - hv.x, src[1] - hv.y);
            }
            const int tk = tile_base + kk * 16 + 2 * t;
            const uint32_t mlo = tail ? ((tk < L ? 0x0000ffffu : 0u) | (tk + 1 < L ? 0xffff0000u : 0u)) : FULL;
            const uint32_t mhi = tail ? ((tk + 8 < L ? 0x0000ffffu : 0u) | (tk + 9 < L ? 0xffff0000u : 0u)) : FULL;
#pragma unroll
            for (int dp = 0; dp < DN / 2; ++dp) {
                const int tok = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
                const int ch = dp * 2 + ((lane >> 4) & 1);
                uint32_t b[4];
                ldsm_x4_trans(b, vt + (ch >> 3) * Lay::kHalf + tok * 128 + (((ch & 7) ^ (lane & 7)) << 4));
                b[0] &= mlo;
                b[1] &= mhi;
                b[2] &= mlo;
                b[3] &= mhi;
                Ops::mma(o[2 * dp], ph, b[0], b[1]);
                Ops::mma(o[2 * dp], pl, b[0], b[1]);
                Ops::mma(o[2 * dp + 1], ph, b[2], b[3]);
                Ops::mma(o[2 * dp + 1], pl, b[2], b[3]);
            }
        }
        __syncthreads();  // every warp is done with this stage
        if (tid == 0 && it + 2 < ntiles) {
            fence_proxy_async_shared();
            issue(it + 2, st);
        }
    }
    if (stopped_at >= 0) {
        if (tid == 0) {
            report(a.err_word, PA_DEVERR_TIMEOUT);
            // tiles stopped_at and stopped_at + 1 may still be in flight: let them land
            for (int k = stopped_at; k < ntiles && k < stopped_at + 2; ++k) mbar_wait(&bars[k & 1], (k >> 1) & 1);
        }
        return;
    }
    l0 += __shfl_xor_sync(FULL, l0, 1);
    l0 += __shfl_xor_sync(FULL, l0, 2);
    l1 += __shfl_xor_sync(FULL, l1, 1);
    l1 += __shfl_xor_sync(FULL, l1, 2);
    const float inv0 = 1.f / l0, inv1 = 1.f / l1;
    if (row0 < n) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(a.out + ((int64_t)(q0 + row0) * a.num_heads + h) * D);
#pragma unroll
        for (int dn = 0; dn < DN; ++dn) dst[dn * 4 + t] = pack2<Tag>(o[dn][0] * inv0, o[dn][1] * inv0);
    }
    if (row1 < n) {
        uint32_t* dst = reinterpret_cast<uint32_t*>(a.out + ((int64_t)(q0 + row1) * a.num_heads + h) * D);
#pragma unroll
        for (int dn = 0; dn < DN; ++dn) dst[dn * 4 + t] = pack2<Tag>(o[dn][2] * inv1, o[dn][3] * inv1);
    }
}

namespace {

template <class Tag, int D>
int launch_prefill(PrefillArgs args, const void* k_cache, const void* v_cache, int num_kv_heads, int num_seqs,
                   int max_query_len, cudaStream_t stream) {
    using Lay = PfLayout<D>;
    static std::atomic<uint64_t> smem_done{0};
    auto kernel = paged_prefill_kernel<Tag, D>;
    if (ensure_smem_limit(kernel, Lay::kAlloc, smem_done) != cudaSuccess) return PA_ERR_CUDA;
    args.box_rows = kPfTok < args.block_size ? kPfTok : args.block_size;
    const int64_t total_tokens = (int64_t)args.num_blocks * args.block_size;
    CUtensorMap kmap, vmap;
    if (!encode_cache_map_swizzled(&kmap, k_cache, D, num_kv_heads, total_tokens, args.box_rows) ||
        !encode_cache_map_swizzled(&vmap, v_cache, D, num_kv_heads, total_tokens, args.box_rows))
        return PA_ERR_CUDA;
    dim3 grid((unsigned)((max_query_len + kPfRows - 1) / kPfRows), (unsigned)args.num_heads, (unsigned)num_seqs);
    kernel<<<grid, kPfThreads, Lay::kAlloc, stream>>>(args, kmap, vmap);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace
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
    if (max_blocks_per_seq > kPfMaxEntries || num_seqs > 65535 || num_heads > 65535) return PA_ERR_UNSUPPORTED;
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
