// pa_decode_noalloc: pa_decode for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc (or any allocating routine)
// at the point where they run attention: code inside a custom allocator or memory
// pool (which would recurse into itself), plug-in hosts that hand out only the
// tensors they own, and launch sequences that must not change the device's memory
// footprint.  This entry point gives them pa_decode with its workspace taken from
// a fixed array in the library's own device memory instead of from the caller.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds it (PA_DECODE_NOALLOC_SCRATCH_BYTES) until the process exits.
// Host code cannot use the array's name as a device address; the address is
// looked up once per device with cudaGetSymbolAddress, with that device current,
// on the first call made on that device.
#include <mutex>

#include "pa_host.h"

namespace {

__device__ __align__(256) static unsigned char g_decode_scratch[PA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Device address of the scratch array on the current device, or nullptr.
void* scratch_address(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace

extern "C" int pa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                 const int32_t* block_tables, const int32_t* context_lens, float scale,
                                 int num_kv_heads, void* out, int num_seqs, int num_heads, int head_dim,
                                 int block_size, int num_blocks, int max_blocks_per_seq, int dtype,
                                 int partition_tokens, int32_t* err_word, void* stream) {
    // pa_decode's own checks first, so that errors (and the early PA_OK of an empty
    // batch) are pa_decode's and nothing is queued on the stream for them
    const int rc = pa::check_decode_call(q, k_cache, v_cache, block_tables, context_lens, num_kv_heads, out,
                                         num_seqs, num_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                                         dtype, partition_tokens, err_word);
    if (rc >= 0) return rc;
    const size_t need = pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                 max_blocks_per_seq, partition_tokens);
    if (need == 0) return PA_ERR_INVALID_ARG;
    if (need > (size_t)PA_DECODE_NOALLOC_SCRATCH_BYTES) return PA_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    void* scratch = scratch_address(dev);
    if (!scratch) return PA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // The scratch keeps whatever the previous call left; the counters at its start
    // must be zero when the kernels start.
    const size_t counters = pa::decode_counter_bytes(num_seqs, num_heads, block_size, max_blocks_per_seq,
                                                     partition_tokens);
    if (cudaMemsetAsync(scratch, 0, counters, st) != cudaSuccess) return PA_ERR_CUDA;
    return pa_decode(q, k_cache, v_cache, block_tables, context_lens, scale, num_kv_heads, out, num_seqs,
                     num_heads, head_dim, block_size, num_blocks, max_blocks_per_seq, dtype, partition_tokens,
                     scratch, (size_t)PA_DECODE_NOALLOC_SCRATCH_BYTES, err_word, stream);
}
