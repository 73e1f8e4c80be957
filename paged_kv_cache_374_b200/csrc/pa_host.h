// Host-side helpers for the C ABI: argument checks, tensor-map encoding and the
// one-time per-device kernel attribute set-up.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>

#include "../../include/pa.h"

namespace pa {

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// cuTensorMapEncodeTiled from the driver, fetched through the runtime so that the
// library needs no link-time dependency on libcuda.
inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// Tensor map over a paged cache viewed as [total_tokens][num_kv_heads][head_dim]
// of 16-bit elements, with boxes of `box_rows` consecutive token rows of one head:
// one box is the K (or V) tile of box_rows tokens for one kv head.
inline bool encode_cache_map(CUtensorMap* map, const void* base, int head_dim, int num_kv_heads,
                             int64_t total_tokens, int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_kv_heads, (cuuint64_t)total_tokens};
    cuuint64_t strides[2] = {(cuuint64_t)head_dim * 2, (cuuint64_t)num_kv_heads * head_dim * 2};
    cuuint32_t box[3] = {(cuuint32_t)head_dim, 1u, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Same view, boxes of 128 bytes (64 16-bit or 128 8-bit elements) x box_rows with the 128-byte TMA
// swizzle: 16-byte chunk j of box row r lands at chunk j ^ (r % 8) of that row in
// shared memory, so reading one chunk column of 8 consecutive rows touches all 32
// banks once.  A head_dim of 128 is loaded as two such boxes (x = 0 and x = 64).
inline bool encode_cache_map_swizzled(CUtensorMap* map, const void* base, int head_dim, int num_kv_heads,
                                      int64_t total_tokens, int box_rows, int elem_bytes = 2) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t eb = (cuuint64_t)elem_bytes;
    cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_kv_heads, (cuuint64_t)total_tokens};
    cuuint64_t strides[2] = {(cuuint64_t)head_dim * eb, (cuuint64_t)num_kv_heads * head_dim * eb};
    cuuint32_t box[3] = {(cuuint32_t)(128 / eb), 1u, (cuuint32_t)box_rows};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = enc(map, elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16, 3,
                     const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Raise a kernel's dynamic shared-memory limit once per device.
// Launch `kernel` as a programmatic dependent of the kernel before it in `stream`:
// it may be scheduled before that kernel completes, so it must wait for it
// (griddepcontrol.wait) before it touches memory that kernel may have written.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                   cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename Kernel>
inline cudaError_t ensure_smem_limit(Kernel kernel, int bytes, std::atomic<uint64_t>& done_mask) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (done_mask.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done_mask.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// The host-side checks of pa_decode, without its workspace arguments: a pa_status
// (PA_OK with nothing to launch when num_seqs == 0, else the error pa_decode would
// return) or -1 when the call may go on to launch.  Launches nothing.
int check_decode_call(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                      const int32_t* context_lens, int num_kv_heads, const void* out, int num_seqs, int num_heads,
                      int head_dim, int block_size, int num_blocks, int max_blocks_per_seq, int dtype,
                      int partition_tokens, const int32_t* err_word);

// The same for the fp8 cache write (pa_reshape_and_cache_fp8).
int check_reshape_and_cache_fp8(const void* k, const void* v, const int64_t* slot_mapping, const void* k_cache,
                                const void* v_cache, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                                int num_blocks, int dtype, float k_scale, float v_scale, const int32_t* err_word);
int launch_reshape_and_cache_fp8(const void* k, const void* v, const int64_t* slot_mapping, void* k_cache,
                                 void* v_cache, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                                 int num_blocks, int dtype, float k_scale, float v_scale, int32_t* err_word,
                                 cudaStream_t st);

// Bytes at the start of pa_decode's workspace that hold counters (zero before the
// first call; every call leaves them zero again).
size_t decode_counter_bytes(int num_seqs, int num_heads, int block_size, int max_blocks_per_seq, int partition_tokens);

// K1's host checks (a pa_status, or -1 when it may launch) and its launch; the
// launch assumes the checks passed.
int check_reshape_and_cache(const void* k, const void* v, const int64_t* slot_mapping, const void* k_cache,
                            const void* v_cache, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                            int num_blocks, int dtype, const int32_t* err_word);
int launch_reshape_and_cache(const void* k, const void* v, const int64_t* slot_mapping, void* k_cache,
                             void* v_cache, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                             int num_blocks, int32_t* err_word, cudaStream_t stream);

// The prefix half of a two-level decode (paged_prefill.cu): partials of the
// shared partitions of every group member, written into the decode workspace.
struct SharedPrefixLaunch {
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    const int32_t* seq_start;
    const int32_t* group_offsets;
    const int32_t* group_members;
    float* ws_m;
    float* ws_l;
    float* ws_o;
    int32_t* err_word;
    float scale;
    int num_heads, num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype;
    int partition_tokens, num_partitions, num_groups, max_group_size, max_shared_tokens;
    int num_seqs;  // bounds the group offsets and member indices
    // early merge (see DecodeArgs): the prefix kernel counts the partitions it
    // writes and queues the (s, h) it completes, as the decode engine does
    int early_merge;
    int32_t* sched;
    int32_t* merge_cnt;
    int32_t* merge_queue;
    // nonzero: launched as a programmatic dependent of the step's cache write,
    // which the kernel waits for before the decode engine may launch
    int after_write;
};
int launch_shared_prefix(const SharedPrefixLaunch& l, cudaStream_t stream);

}  // namespace pa
