// K1: reshape_and_cache -- scatter each new token's K/V rows into its slot.
//
// Decode step 3 of P2 ("大模型推理优化：KV Cache与PagedAttention技术详解", §2.1):
// the current token's K and V join the cache before attention reads it.  In the
// cache layout [num_blocks][block_size][num_kv_heads][head_dim] one token's rows
// for all kv heads are one contiguous run of num_kv_heads * head_dim * 2 bytes, in
// the source [num_tokens][num_kv_heads][head_dim] as well, so the write is a
// per-token copy of 16-byte vectors: coalesced on both sides, no arithmetic.
#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {

__global__ void __launch_bounds__(256) reshape_and_cache_kernel(const uint4* __restrict__ k,
                                                                 const uint4* __restrict__ v,
                                                                 const int64_t* __restrict__ slot_mapping,
                                                                 uint4* __restrict__ k_cache,
                                                                 uint4* __restrict__ v_cache, int num_tokens,
                                                                 int row_vecs, int64_t num_slots,
                                                                 int32_t* err_word) {
    const int64_t total = (int64_t)num_tokens * row_vecs;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t tok = i / row_vecs;
        const int64_t c = i - tok * row_vecs;
        const int64_t slot = __ldg(slot_mapping + tok);
        if (slot < 0) continue;  // padding token
        if (slot >= num_slots) {
            if (c == 0) report(err_word, PA_DEVERR_SLOT_RANGE);
            continue;
        }
        const uint4 kv = __ldcs(k + i);
        const uint4 vv = __ldcs(v + i);
        k_cache[slot * row_vecs + c] = kv;
        v_cache[slot * row_vecs + c] = vv;
    }
}

}  // namespace pa

extern "C" int pa_reshape_and_cache(const void* k, const void* v, const int64_t* slot_mapping, void* k_cache,
                                    void* v_cache, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                                    int num_blocks, int dtype, int32_t* err_word, void* stream) {
    using namespace pa;
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
    if (head_dim % 8 != 0) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u) || (err_word && !aligned4(err_word)))
        return PA_ERR_INVALID_ARG;
    const int64_t row_vecs64 = (int64_t)num_kv_heads * head_dim / 8;
    if (row_vecs64 > INT32_MAX) return PA_ERR_UNSUPPORTED;
    const int row_vecs = (int)row_vecs64;
    const int64_t total = (int64_t)num_tokens * row_vecs;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    const int64_t cap = (int64_t)sms * 8;
    if (blocks > cap) blocks = cap;
    reshape_and_cache_kernel<<<(unsigned)blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping, static_cast<uint4*>(k_cache),
        static_cast<uint4*>(v_cache), num_tokens, row_vecs, (int64_t)num_blocks * block_size, err_word);
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}
