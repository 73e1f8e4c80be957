// pa_copy_blocks: whole-block copies inside the paged caches (copy-on-write after
// a beam fork); pa_swap_blocks: the same between two pools (swap-out / swap-in).
// One physical block of one cache is block_size * num_kv_heads * head_dim
// elements, contiguous in the [num_blocks][block_size][num_kv_heads][head_dim]
// layout, so a pair is one contiguous run per cache; threads copy 16-byte
// vectors, K and V alike.
#include <atomic>

#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {

// The (pair, 16-byte vector) space of all pairs is cut into one contiguous,
// equal slice per CTA (every CTA resident at once, no tail wave); a CTA walks its
// slice pair by pair.  The pairs are copied all at once, so a pair that overlaps
// another copying pair -- its destination is another's destination or source, or
// its source is another's destination -- is skipped and reported: a CTA checks
// each pair its slice touches against the whole list (num_pairs comparisons
// spread over its threads).  Pairs that copy nothing (ids out of range, source ==
// destination) conflict with nothing.
__global__ void __launch_bounds__(256, 4) copy_blocks_kernel(uint4* __restrict__ k_cache,
                                                              uint4* __restrict__ v_cache,
                                                              const int32_t* __restrict__ pairs, int num_pairs,
                                                              int64_t block_vecs, int num_blocks, int32_t* err_word) {
    constexpr int U = 4;  // 16-byte vectors in flight per thread and cache
    const int64_t total = (int64_t)num_pairs * block_vecs;
    const int64_t per = (total + gridDim.x - 1) / gridDim.x;
    int64_t lo = (int64_t)blockIdx.x * per;
    const int64_t hi = lo + per < total ? lo + per : total;
    while (lo < hi) {
        const int64_t pi = lo / block_vecs;
        const int64_t c0 = lo - pi * block_vecs;
        const int64_t c1 = c0 + (hi - lo) < block_vecs ? c0 + (hi - lo) : block_vecs;
        lo += c1 - c0;
        const int32_t src = __ldg(pairs + 2 * pi), dst = __ldg(pairs + 2 * pi + 1);
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            if (c0 == 0 && threadIdx.x == 0) report(err_word, PA_DEVERR_TABLE_RANGE);
            continue;
        }
        if (src == dst) continue;
        bool conflict = false;
        for (int j = threadIdx.x; j < num_pairs; j += blockDim.x) {
            const int32_t sj = __ldg(pairs + 2 * (int64_t)j), dj = __ldg(pairs + 2 * (int64_t)j + 1);
            if (j == pi || sj == dj || sj < 0 || sj >= num_blocks || dj < 0 || dj >= num_blocks) continue;
            conflict |= dj == dst || sj == dst || dj == src;
        }
        if (__syncthreads_or(conflict)) {
            if (c0 == 0 && threadIdx.x == 0) report(err_word, PA_DEVERR_PAIR_CONFLICT);
            continue;
        }
        // this slice's part of the pair: n vectors from c0 (a block is far below 2^31 vectors)
        const int n = (int)(c1 - c0);
        const uint4* ks = k_cache + (int64_t)src * block_vecs + c0;
        const uint4* vs = v_cache + (int64_t)src * block_vecs + c0;
        uint4* kd = k_cache + (int64_t)dst * block_vecs + c0;
        uint4* vd = v_cache + (int64_t)dst * block_vecs + c0;
        for (int i = threadIdx.x; i < n; i += 256 * U) {
            uint4 a[U], b[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = i + u * 256;
                if (j < n) {
                    a[u] = __ldcs(ks + j);
                    b[u] = __ldcs(vs + j);
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int j = i + u * 256;
                if (j < n) {
                    kd[j] = a[u];
                    vd[j] = b[u];
                }
            }
        }
    }
}

// Cross-pool variant (swap-out / swap-in): source and destination are different
// pools, either of which may be device-addressable pinned host memory.
__global__ void __launch_bounds__(256) swap_blocks_kernel(const uint4* __restrict__ src_k,
                                                           const uint4* __restrict__ src_v, int src_blocks,
                                                           uint4* __restrict__ dst_k, uint4* __restrict__ dst_v,
                                                           int dst_blocks, const int32_t* __restrict__ pairs,
                                                           int num_pairs, int64_t block_vecs, int32_t* err_word) {
    const int64_t total = (int64_t)num_pairs * block_vecs;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t pi = i / block_vecs;
        const int64_t c = i - pi * block_vecs;
        const int32_t src = __ldg(pairs + 2 * pi), dst = __ldg(pairs + 2 * pi + 1);
        if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
            if (c == 0) report(err_word, PA_DEVERR_TABLE_RANGE);
            continue;
        }
        dst_k[(int64_t)dst * block_vecs + c] = src_k[(int64_t)src * block_vecs + c];
        dst_v[(int64_t)dst * block_vecs + c] = src_v[(int64_t)src * block_vecs + c];
    }
}

}  // namespace pa

extern "C" int pa_swap_blocks(const void* src_k, const void* src_v, int src_num_blocks, void* dst_k, void* dst_v,
                              int dst_num_blocks, const int32_t* pairs, int num_pairs, int num_kv_heads,
                              int head_dim, int block_size, int element_bytes, int32_t* err_word, void* stream) {
    using namespace pa;
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || src_num_blocks < 0 ||
        dst_num_blocks < 0 || (element_bytes != 1 && element_bytes != 2))
        return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!src_k || !src_v || !dst_k || !dst_v || !pairs) return PA_ERR_INVALID_ARG;
    const int64_t block_bytes = (int64_t)block_size * num_kv_heads * head_dim * element_bytes;
    if (block_bytes % 16 != 0) return PA_ERR_UNSUPPORTED;
    if (!aligned16(src_k) || !aligned16(src_v) || !aligned16(dst_k) || !aligned16(dst_v) || !aligned4(pairs) ||
        (err_word && !aligned4(err_word)))
        return PA_ERR_INVALID_ARG;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t total = (int64_t)num_pairs * (block_bytes / 16);
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
    swap_blocks_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(src_k), static_cast<const uint4*>(src_v), src_num_blocks,
        static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v), dst_num_blocks, pairs, num_pairs, block_bytes / 16,
        err_word);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

extern "C" int pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* copy_pairs, int num_pairs,
                              int num_kv_heads, int head_dim, int block_size, int num_blocks, int element_bytes,
                              int32_t* err_word, void* stream) {
    using namespace pa;
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0 ||
        (element_bytes != 1 && element_bytes != 2))
        return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !copy_pairs) return PA_ERR_INVALID_ARG;
    const int64_t block_bytes = (int64_t)block_size * num_kv_heads * head_dim * element_bytes;
    if (block_bytes % 16 != 0) return PA_ERR_UNSUPPORTED;
    if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned4(copy_pairs) || (err_word && !aligned4(err_word)))
        return PA_ERR_INVALID_ARG;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // every CTA resident at once (as many per SM as fit), each with a slice of at
    // least 1024 vectors (16 KiB per cache)
    static std::atomic<int> per_sm{0};
    if (per_sm.load(std::memory_order_relaxed) == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, copy_blocks_kernel, 256, 0) != cudaSuccess || n < 1)
            return PA_ERR_CUDA;
        per_sm.store(n, std::memory_order_relaxed);
    }
    const int64_t block_vecs = block_bytes / 16;
    const int64_t target = (int64_t)sms * per_sm.load(std::memory_order_relaxed);
    const int64_t slices = ((int64_t)num_pairs * block_vecs + 1023) / 1024;
    const int64_t blocks = slices < target ? slices : target;
    copy_blocks_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), copy_pairs, num_pairs, block_vecs, num_blocks,
        err_word);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
