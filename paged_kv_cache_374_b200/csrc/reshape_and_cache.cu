// K1: reshape_and_cache -- scatter each new token's K/V rows into its slot.
//
// Decode step 3 of P2 ("大模型推理优化：KV Cache与PagedAttention技术详解", §2.1):
// the current token's K and V join the cache before attention reads it.  In the
// cache layout [num_blocks][block_size][num_kv_heads][head_dim] one token's rows
// for all kv heads are one contiguous run of num_kv_heads * head_dim * 2 bytes, in
// the source [num_tokens][num_kv_heads][head_dim] as well, so the write is a
// per-token copy of 16-byte vectors: coalesced on both sides, no arithmetic.
#include <cmath>

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
    // Launched as a programmatic dependent of the kernel before it in the stream,
    // which may have produced k and v: wait for that grid to complete before
    // reading anything.  Then an attention launch that follows as a programmatic
    // dependent (pa_decode_step) may start its prologue; it waits for this grid
    // before it reads the cache.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

// fp8 variant: 16 elements per thread (32 input bytes -> one 16-byte code vector);
// each element is divided by its cache's scale in fp32 (IEEE, round to nearest)
// and rounded to the nearest E4M3 code, saturating at +-448.
template <class Tag>
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(const uint4* __restrict__ k,
                                                                     const uint4* __restrict__ v,
                                                                     const int64_t* __restrict__ slot_mapping,
                                                                     uint4* __restrict__ k_cache,
                                                                     uint4* __restrict__ v_cache, int num_tokens,
                                                                     int row_vecs, int64_t num_slots, float k_scale,
                                                                     float v_scale, int32_t* err_word) {
    asm volatile("griddepcontrol.wait;" ::: "memory");  // as the 16-bit kernel
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t total = (int64_t)num_tokens * row_vecs;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t tok = i / row_vecs;
        const int64_t c = i - tok * row_vecs;
        const int64_t slot = __ldg(slot_mapping + tok);
        if (slot < 0) continue;
        if (slot >= num_slots) {
            if (c == 0) report(err_word, PA_DEVERR_SLOT_RANGE);
            continue;
        }
        uint4 out[2];
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            const uint4* src = t == 0 ? k : v;
            const float sc = t == 0 ? k_scale : v_scale;
            const uint4 a = __ldcs(src + 2 * i), b = __ldcs(src + 2 * i + 1);
            const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
            uint32_t q[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f0 = Tag::widen2(w[2 * j]), f1 = Tag::widen2(w[2 * j + 1]);
                const uint32_t lo = E4M3Tag::encode2(__fdiv_rn(f0.x, sc), __fdiv_rn(f0.y, sc));
                const uint32_t hi = E4M3Tag::encode2(__fdiv_rn(f1.x, sc), __fdiv_rn(f1.y, sc));
                q[j] = lo | (hi << 16);
            }
            out[t] = make_uint4(q[0], q[1], q[2], q[3]);
        }
        k_cache[slot * row_vecs + c] = out[0];
        v_cache[slot * row_vecs + c] = out[1];
    }
}

}  // namespace pa

namespace pa {

int check_reshape_and_cache_fp8(const void* k, const void* v, const int64_t* slot_mapping, const void* k_cache,
                                const void* v_cache, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                                int num_blocks, int dtype, float k_scale, float v_scale, const int32_t* err_word) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0)
        return PA_ERR_INVALID_ARG;
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || !isfinite(k_scale) || !isfinite(v_scale)) return PA_ERR_INVALID_ARG;
    if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
    if (head_dim % 16 != 0) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u) || (err_word && !aligned4(err_word)))
        return PA_ERR_INVALID_ARG;
    if ((int64_t)num_kv_heads * head_dim / 16 > INT32_MAX) return PA_ERR_UNSUPPORTED;
    return -1;
}

int launch_reshape_and_cache_fp8(const void* k, const void* v, const int64_t* slot_mapping, void* k_cache,
                                 void* v_cache, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                                 int num_blocks, int dtype, float k_scale, float v_scale, int32_t* err_word,
                                 cudaStream_t st) {
    const int row_vecs = (int)((int64_t)num_kv_heads * head_dim / 16);
    const int64_t total = (int64_t)num_tokens * row_vecs;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (total + 255) / 256;
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
    const int64_t num_slots = (int64_t)num_blocks * block_size;
    auto kernel = dtype == PA_F16 ? reshape_and_cache_fp8_kernel<F16Tag> : reshape_and_cache_fp8_kernel<BF16Tag>;
    const cudaError_t e = launch_dependent(
        kernel, dim3((unsigned)blocks), dim3(256), 0, st, static_cast<const uint4*>(k), static_cast<const uint4*>(v),
        slot_mapping, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), num_tokens, row_vecs, num_slots,
        k_scale, v_scale, err_word);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa

extern "C" int pa_reshape_and_cache_fp8(const void* k, const void* v, const int64_t* slot_mapping, void* k_cache,
                                        void* v_cache, int num_tokens, int num_kv_heads, int head_dim,
                                        int block_size, int num_blocks, int dtype, float k_scale, float v_scale,
                                        int32_t* err_word, void* stream) {
    using namespace pa;
    const int rc = check_reshape_and_cache_fp8(k, v, slot_mapping, k_cache, v_cache, num_tokens, num_kv_heads,
                                               head_dim, block_size, num_blocks, dtype, k_scale, v_scale, err_word);
    if (rc >= 0) return rc;
    return launch_reshape_and_cache_fp8(k, v, slot_mapping, k_cache, v_cache, num_tokens, num_kv_heads, head_dim,
                                        block_size, num_blocks, dtype, k_scale, v_scale, err_word,
                                        static_cast<cudaStream_t>(stream));
}

namespace pa {

int check_reshape_and_cache(const void* k, const void* v, const int64_t* slot_mapping, const void* k_cache,
                            const void* v_cache, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, int dtype, const int32_t* err_word) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0)
        return PA_ERR_INVALID_ARG;
    if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
    if (head_dim % 8 != 0) return PA_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u) || (err_word && !aligned4(err_word)))
        return PA_ERR_INVALID_ARG;
    if ((int64_t)num_kv_heads * head_dim / 8 > INT32_MAX) return PA_ERR_UNSUPPORTED;
    return -1;
}

int launch_reshape_and_cache(const void* k, const void* v, const int64_t* slot_mapping, void* k_cache,
                             void* v_cache, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                             int num_blocks, int32_t* err_word, cudaStream_t stream) {
    const int row_vecs = (int)((int64_t)num_kv_heads * head_dim / 8);
    const int64_t total = (int64_t)num_tokens * row_vecs;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    const int64_t cap = (int64_t)sms * 8;
    if (blocks > cap) blocks = cap;
    const cudaError_t e = launch_dependent(
        reshape_and_cache_kernel, dim3((unsigned)blocks), dim3(threads), 0, stream, static_cast<const uint4*>(k),
        static_cast<const uint4*>(v), slot_mapping, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
        num_tokens, row_vecs, (int64_t)num_blocks * block_size, err_word);
    return e == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa

extern "C" int pa_reshape_and_cache(const void* k, const void* v, const int64_t* slot_mapping, void* k_cache,
                                    void* v_cache, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                                    int num_blocks, int dtype, int32_t* err_word, void* stream) {
    using namespace pa;
    const int rc = check_reshape_and_cache(k, v, slot_mapping, k_cache, v_cache, num_tokens, num_kv_heads, head_dim,
                                           block_size, num_blocks, dtype, err_word);
    if (rc >= 0) return rc;
    return launch_reshape_and_cache(k, v, slot_mapping, k_cache, v_cache, num_tokens, num_kv_heads, head_dim,
                                    block_size, num_blocks, err_word, static_cast<cudaStream_t>(stream));
}
