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

// The pairs' blocks are cut into chunks of kChunk 16-byte vectors, in pair order,
// and the CTAs walk them grid-stride, so that at any time they copy one window of
// consecutive chunks (the source blocks are read in the pairs' order).  The pairs
// are copied all at once, so a pair that overlaps another copying pair -- its
// destination is another's destination or source, or its source is another's
// destination -- is skipped and reported: each chunk's CTA checks its pair
// against the whole list, held in shared memory when it fits (kStagedPairs).
// Pairs that copy nothing (ids out of range, source == destination) conflict
// with nothing.
constexpr int kCopyThreads = 256;
constexpr int kCopyUnroll = 4;                              // vectors in flight per thread and cache
constexpr int kChunk = kCopyThreads * kCopyUnroll;          // 16 KiB of each cache
constexpr int kStagedPairs = 2048;                          // 16 KiB of shared memory

__device__ __forceinline__ bool copies(int32_t s, int32_t d, int num_blocks) {
    return s >= 0 && s < num_blocks && d >= 0 && d < num_blocks && s != d;
}

__global__ void __launch_bounds__(kCopyThreads, 4) copy_blocks_kernel(uint4* __restrict__ k_cache,
                                                                       uint4* __restrict__ v_cache,
                                                                       const int32_t* __restrict__ pairs,
                                                                       int num_pairs, int64_t block_vecs,
                                                                       int num_blocks, int32_t* err_word) {
    __shared__ int2 s_pairs[kStagedPairs];
    const bool staged = num_pairs <= kStagedPairs;
    if (staged)
        for (int j = threadIdx.x; j < num_pairs; j += kCopyThreads)
            s_pairs[j] = make_int2(__ldg(pairs + 2 * j), __ldg(pairs + 2 * j + 1));
    __syncthreads();
    const int64_t per_pair = (block_vecs + kChunk - 1) / kChunk;
    const int64_t chunks = (int64_t)num_pairs * per_pair;
    for (int64_t w = blockIdx.x; w < chunks; w += gridDim.x) {
        const int pi = (int)(w / per_pair);
        const int64_t c0 = (w - (int64_t)pi * per_pair) * kChunk;
        const int n = (int)(block_vecs - c0 < kChunk ? block_vecs - c0 : kChunk);
        const int2 me = staged ? s_pairs[pi] : make_int2(__ldg(pairs + 2 * (int64_t)pi), __ldg(pairs + 2 * (int64_t)pi + 1));
        const int32_t src = me.x, dst = me.y;
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            if (c0 == 0 && threadIdx.x == 0) report(err_word, PA_DEVERR_TABLE_RANGE);
            continue;
        }
        if (src == dst) continue;
        // the CTA's threads split the scan (a per-warp scan, without the barrier,
        // measured slower: every warp repeats the whole list)
        bool conflict = false;
        for (int j = threadIdx.x; j < num_pairs; j += kCopyThreads) {
            const int2 o = staged ? s_pairs[j]
                                  : make_int2(__ldg(pairs + 2 * (int64_t)j), __ldg(pairs + 2 * (int64_t)j + 1));
            if (j == pi || !copies(o.x, o.y, num_blocks)) continue;
            conflict |= o.y == dst || o.x == dst || o.y == src;
        }
        if (__syncthreads_or(conflict)) {
            if (c0 == 0 && threadIdx.x == 0) report(err_word, PA_DEVERR_PAIR_CONFLICT);
            continue;
        }
        const uint4* ks = k_cache + (int64_t)src * block_vecs + c0;
        const uint4* vs = v_cache + (int64_t)src * block_vecs + c0;
        uint4* kd = k_cache + (int64_t)dst * block_vecs + c0;
        uint4* vd = v_cache + (int64_t)dst * block_vecs + c0;
        uint4 a[kCopyUnroll], b[kCopyUnroll];
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int j = threadIdx.x + u * kCopyThreads;
            if (j < n) {
                a[u] = __ldcs(ks + j);
                b[u] = __ldcs(vs + j);
            }
        }
#pragma unroll
        for (int u = 0; u < kCopyUnroll; ++u) {
            const int j = threadIdx.x + u * kCopyThreads;
            if (j < n) {
                kd[j] = a[u];
                vd[j] = b[u];
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
    // as many CTAs as are resident at once; they stride over the chunks
    static std::atomic<int> per_sm{0};
    if (per_sm.load(std::memory_order_relaxed) == 0) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, copy_blocks_kernel, kCopyThreads, 0) != cudaSuccess ||
            n < 1)
            return PA_ERR_CUDA;
        per_sm.store(n, std::memory_order_relaxed);
    }
    const int64_t block_vecs = block_bytes / 16;
    const int64_t target = (int64_t)sms * per_sm.load(std::memory_order_relaxed);
    const int64_t chunks = (int64_t)num_pairs * ((block_vecs + kChunk - 1) / kChunk);
    const int64_t blocks = chunks < target ? chunks : target;
    copy_blocks_kernel<<<(unsigned)blocks, kCopyThreads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), copy_pairs, num_pairs, block_vecs, num_blocks,
        err_word);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
