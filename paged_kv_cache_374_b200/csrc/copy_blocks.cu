// pa_copy_blocks: whole-block copies inside the paged caches (copy-on-write after
// a beam fork).  One physical block of one cache is block_size * num_kv_heads *
// head_dim elements, contiguous in the [num_blocks][block_size][num_kv_heads]
// [head_dim] layout, so a pair is one contiguous run per cache; threads copy
// 16-byte vectors, grid-stride over (pair, vector), K and V alike.
#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {

__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                                           const int32_t* __restrict__ pairs, int num_pairs,
                                                           int64_t block_vecs, int num_blocks, int32_t* err_word) {
    const int64_t total = (int64_t)num_pairs * block_vecs;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t pi = i / block_vecs;
        const int64_t c = i - pi * block_vecs;
        const int32_t src = __ldg(pairs + 2 * pi), dst = __ldg(pairs + 2 * pi + 1);
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            if (c == 0) report(err_word, PA_DEVERR_TABLE_RANGE);
            continue;
        }
        if (src == dst) continue;
        k_cache[(int64_t)dst * block_vecs + c] = __ldcs(k_cache + (int64_t)src * block_vecs + c);
        v_cache[(int64_t)dst * block_vecs + c] = __ldcs(v_cache + (int64_t)src * block_vecs + c);
    }
}

}  // namespace pa

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
    const int64_t total = (int64_t)num_pairs * (block_bytes / 16);
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
    copy_blocks_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), copy_pairs, num_pairs, block_bytes / 16,
        num_blocks, err_word);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
