/*
 * pa.h -- C ABI of the B200 paged decode-attention library (libpa.so).
 *
 * The library implements the data-parallel hot path of PagedAttention decoding:
 * the KV cache lives in fixed-size physical blocks of block_size tokens, and each
 * sequence reaches its tokens through a block table that maps logical block j to
 * a physical block id.
 *
 * Pages cited by title and section:
 *   P1  "大模型部署中的PagedAttention：KV Cache显存管理突破" (blog.csdn.net)
 *   P2  "大模型推理优化：KV Cache与PagedAttention技术详解" (intelliparadigm.com)
 *   P3  "LLM 推理中的 PageAttention 实现原理：虚拟内存管理在 KV Cache 中的创新应用"
 *       (dpshk.com)
 *
 * Conventions for every call
 *   - Return value: a pa_status code (PA_OK == 0).  Host-side argument checks run
 *     before anything is launched; on an error nothing is launched or changed.
 *   - Device pointers are owned by the caller and must stay valid until the work
 *     queued on `stream` has finished.  Calls are asynchronous on `stream` (a
 *     cudaStream_t passed as void*; NULL is the legacy default stream) and
 *     allocate no device or pinned memory.
 *   - dtype is PA_F16 or PA_BF16 and is the same for q, k, v, the caches and out.
 *   - Every tensor is contiguous, row-major, in the layout stated, and every
 *     device pointer is 16-byte aligned.
 *   - Cache layout: k_cache and v_cache are [num_blocks][block_size][num_kv_heads]
 *     [head_dim].  Token slot = phys * block_size + offset, so element (slot, h, i)
 *     sits at (slot * num_kv_heads + h) * head_dim + i.  (The pages fix blocks of
 *     block_size tokens, P1 §1 and P3 §一, a per-block tensor of (block_size,
 *     d_model), P1 §2, and a cache of [seq_len, num_heads, head_dim], P2 §2.1; the
 *     order inside a block is this library's choice.)
 *   - Bad indices found on the device never fault: the access is skipped and, if
 *     err_word (a device int32, may be NULL) is given, a PA_DEVERR_* bit is OR-ed
 *     into it.  The caller clears it.
 *   - The block allocator is host-only and single-threaded: callers serialise
 *     access to one allocator (the pages' listing holds a mutex around it, P3 §三).
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned pointer, short workspace, bad id */
    PA_ERR_UNSUPPORTED = 2,   /* no kernel for this head_dim / block_size / dtype / group */
    PA_ERR_OUT_OF_BLOCKS = 3, /* the allocator has too few free blocks; nothing was allocated */
    PA_ERR_REFCOUNT = 4,      /* free or add_ref of a block whose reference count is 0 */
    PA_ERR_CUDA = 5           /* a CUDA runtime call or kernel launch failed */
} pa_status;

enum { PA_F16 = 0, PA_BF16 = 1 };

/* Bits OR-ed into *err_word by the kernels. */
enum {
    PA_DEVERR_SLOT_RANGE = 1,    /* slot_mapping entry >= num_blocks * block_size (write skipped) */
    PA_DEVERR_TABLE_RANGE = 2,   /* block_tables entry outside [0, num_blocks) (output row is NaN) */
    PA_DEVERR_LEN_RANGE = 4,     /* context_len < 0 or > max_blocks_per_seq * block_size (row NaN) */
    PA_DEVERR_TIMEOUT = 8,       /* an in-kernel wait gave up (the output is not valid) */
    PA_DEVERR_GROUP_RANGE = 16,  /* a shared-prefix group's offsets or members out of range (group skipped) */
    PA_DEVERR_PAIR_CONFLICT = 32 /* a block-copy pair overlaps another pair (pair skipped) */
};

/* Human-readable name of a pa_status value (static storage). */
const char* pa_status_string(int status);

/* ------------------------------------------------------------------------ K1 */

/*
 * pa_reshape_and_cache -- write each new token's K and V rows into their slots.
 *
 * Step 3 of a decode step (P2 §2.1: the current token's K/V is added to the
 * cache before attention runs over all t tokens); the slot of a token is
 * table[pos / block_size] * block_size + pos % block_size (P3 §三,
 * BlockTable::get_physical_location).
 *
 *   k, v          [num_tokens][num_kv_heads][head_dim], dtype, device
 *   slot_mapping  [num_tokens] int64, device; a negative entry means "no token"
 *                 (skipped in silence), an entry >= num_blocks * block_size is
 *                 skipped and sets PA_DEVERR_SLOT_RANGE
 *   k_cache, v_cache  [num_blocks][block_size][num_kv_heads][head_dim], device
 *
 * For every i < num_tokens with a valid slot and every h < num_kv_heads:
 *   k_cache[slot_i][h][:] = k[i][h][:], v_cache[slot_i][h][:] = v[i][h][:],
 * a bit-exact copy.  Slots must be distinct (a repeated slot gets one of the rows).
 * head_dim must be a multiple of 8.
 */
int pa_reshape_and_cache(const void* k, const void* v, const int64_t* slot_mapping, void* k_cache,
                         void* v_cache, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, int dtype, int32_t* err_word, void* stream);

/* ------------------------------------------------------------------- K2 + K3 */

/*
 * Context partition used by pa_decode when partition_tokens == 0: the token span
 * of one unit of work.  A sequence longer than this is split across CTAs and the
 * partial results are merged by a second kernel.  Always a multiple of 64.
 */
int pa_decode_partition_tokens(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                               int max_blocks_per_seq);

/*
 * Bytes of device workspace pa_decode needs for these sizes: 256 bytes of
 * scheduling counters, plus, when a sequence can span more than one partition,
 * a merge counter and a merge-queue entry per (sequence, query head) and the
 * partial results of split sequences.  partition_tokens: 0 = the default
 * above, otherwise a positive multiple of 64, at most 65536.  Returns 0 for
 * invalid sizes.
 */
size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                                int max_blocks_per_seq, int partition_tokens);

/*
 * pa_decode -- single-query (decode) attention over the paged cache.
 *
 * For every sequence s and query head h, with g = num_heads / num_kv_heads and
 * h_kv = h / g (g consecutive query heads share one K/V head), L = context_lens[s]
 * tokens in logical order t = 0..L-1, token t at physical block
 * block_tables[s][t / block_size], offset t % block_size (P3 §三):
 *     x_t = scale * sum_i q[s][h][i] * K[t][h_kv][i]
 *     out[s][h][:] = sum_t exp(x_t - M) V[t][h_kv][:] / sum_t exp(x_t - M),  M = max_t x_t
 * i.e. softmax(q K^T * scale) V as one softmax over all L tokens (P1 §1, first
 * formula; the per-block sum printed beside it is not normalised and is not what
 * is computed).  scale is applied as given (1/sqrt(head_dim) is the usual value).
 * Arithmetic is fp32; the result is rounded once to dtype (round to nearest even).
 *
 *   q             [num_seqs][num_heads][head_dim], dtype, device
 *   k_cache, v_cache  cache layout above, device
 *   block_tables  [num_seqs][max_blocks_per_seq] int32, device; entries past
 *                 ceil(L / block_size) are never read
 *   context_lens  [num_seqs] int32, device; L includes this step's new token;
 *                 L == 0 gives a row of zeros
 *   out           [num_seqs][num_heads][head_dim], dtype, device
 *   partition_tokens  0 = default; else a positive multiple of 64
 *   workspace     device scratch of at least pa_decode_workspace_size(...)
 *                 bytes.  It starts with the kernels' counters (work claims and,
 *                 when contexts are split, the merge queue: 256 bytes plus 8 per
 *                 (sequence, query head)): zero the whole workspace once before
 *                 the first call (cudaMemset); every call leaves the counters
 *                 zero again, so a workspace can be reused call after call on one
 *                 stream.  Calls that may run at the same time need separate
 *                 workspaces.  After a PA_DEVERR_TIMEOUT, zero it again.
 *
 * Supported: head_dim in {64, 128}; block_size in {16, 32, 64}; num_heads a
 * multiple of num_kv_heads; any num_seqs >= 0.  Otherwise PA_ERR_UNSUPPORTED or
 * PA_ERR_INVALID_ARG.
 */
int pa_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
              const int32_t* context_lens, float scale, int num_kv_heads, void* out, int num_seqs,
              int num_heads, int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
              int dtype, int partition_tokens, void* workspace, size_t workspace_bytes, int32_t* err_word,
              void* stream);

/*
 * pa_decode_step -- one whole decode step in one call: write each sequence's new
 * token into its slot, then attend over the caches that now hold it (P2 §2.1,
 * decode steps 3-5: the current token's K/V join the cache, then attention runs
 * over all t tokens).  The result is exactly that of
 *     pa_reshape_and_cache(k, v, slot_mapping, ..., num_tokens = num_seqs, ...)
 *     pa_decode(q, ...)
 * in that order on `stream`.  In one call the attention kernel is launched as a
 * programmatic dependent of the cache write: its launch and its scheduling
 * prologue (which read only context_lens, block_tables and q) overlap the write,
 * and every warp waits for the write to complete before its first cache read.
 *
 *   k, v, slot_mapping  as pa_reshape_and_cache, one new token per sequence
 *                       (token i belongs to sequence i; num_tokens = num_seqs)
 *   everything else     as pa_decode (the caches are written, then read)
 * Errors: the checks of both calls run first; on an error nothing is launched.
 */
int pa_decode_step(const void* k, const void* v, const int64_t* slot_mapping, const void* q, void* k_cache,
                   void* v_cache, const int32_t* block_tables, const int32_t* context_lens, float scale,
                   int num_kv_heads, void* out, int num_seqs, int num_heads, int head_dim, int block_size,
                   int num_blocks, int max_blocks_per_seq, int dtype, int partition_tokens, void* workspace,
                   size_t workspace_bytes, int32_t* err_word, void* stream);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate device memory.
 *
 * No counterpart on the pages: this is an interface convenience of the library,
 * not a step of the method.  Some callers cannot call cudaMalloc (or any routine
 * that allocates) where they run attention: code running inside a device memory
 * allocator or pool, which would re-enter itself; plug-in hosts that pass in only
 * the tensors they own; launch sequences that must keep the device memory
 * footprint fixed.  This call takes pa_decode's workspace from a fixed array in the
 * library's own device memory instead, so it allocates nothing.
 *
 * Arguments, results and errors as pa_decode, without workspace/workspace_bytes.
 *   - The array holds PA_DECODE_NOALLOC_SCRATCH_BYTES on every GPU that loads the
 *     library, until the process exits.  Sizes whose pa_decode_workspace_size(...)
 *     exceeds it are refused with PA_ERR_UNSUPPORTED (use pa_decode with a
 *     workspace of your own for those).
 *   - The first call on a device looks up the array's device address on that
 *     device (a one-time set-up); make that first call before any stream capture.
 *   - Every call on a device uses the same array, which keeps the previous call's
 *     contents; the call clears the part that must start at zero.  Calls whose
 *     work may overlap on the GPU (several streams or host threads) race on the
 *     array and give wrong results: serialise them, e.g. on one stream.
 */
#define PA_DECODE_NOALLOC_SCRATCH_BYTES (64u << 20)
int pa_decode_noalloc(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                      const int32_t* context_lens, float scale, int num_kv_heads, void* out, int num_seqs,
                      int num_heads, int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                      int dtype, int partition_tokens, int32_t* err_word, void* stream);

/* ------------------------------------------------------- shared prefixes */

/*
 * pa_decode_shared_prefix -- pa_decode for batches whose sequences share a
 * prefix through the same physical blocks (a beam fork holding the prompt's
 * blocks by reference, P3 §四; requests reusing a cached prompt, P3 §三).  The
 * result is pa_decode's, to rounding: the shared part is attended once per kv
 * head for the whole group (on the tensor cores, the group's queries as the rows
 * of one matrix) instead of once per sequence, and merged with each sequence's
 * own suffix by the same partial-softmax merge that joins split partitions.
 *
 * Arguments as pa_decode, plus (all device arrays):
 *   seq_start      [num_seqs] int32: 0, or the tokens sequence s shares with
 *                  its group -- a multiple of the partition size below
 *                  context_lens[s].  Tokens below it must use the same physical
 *                  blocks as every other member of the group.
 *   num_groups     groups of sequences sharing a prefix (host int; 0 = pa_decode)
 *   group_offsets  [num_groups + 1] int32: group g is
 *   group_members  group_members[group_offsets[g] .. group_offsets[g+1]) (sequence
 *                  indices); every member has the same seq_start.  A group whose
 *                  offsets are not 0 <= offsets[g] <= offsets[g+1] <= num_seqs, or
 *                  that lists a member outside [0, num_seqs), is skipped and
 *                  reported as PA_DEVERR_GROUP_RANGE (its members' outputs are
 *                  then undefined; every other sequence is unaffected)
 *   max_group_size, max_shared_tokens  host ints bounding the group sizes and the
 *                  seq_start values (the launch sizes); a group beyond them is
 *                  reported as PA_DEVERR_LEN_RANGE and its output is undefined
 * pa_find_shared_prefixes builds these from host block tables.  partition_tokens
 * must be the one the workspace was sized with (0 = default).  A seq_start that
 * is not a multiple of the partition below the length is ignored (the whole
 * sequence runs in the per-sequence kernel) and reported as
 * PA_DEVERR_LEN_RANGE; a member whose seq_start differs from its group's gets no
 * shared partials and is reported the same way (its output is then undefined).
 */
int pa_decode_shared_prefix(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                            const int32_t* context_lens, float scale, int num_kv_heads, void* out, int num_seqs,
                            int num_heads, int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                            int dtype, const int32_t* seq_start, int num_groups, const int32_t* group_offsets,
                            const int32_t* group_members, int max_group_size, int max_shared_tokens,
                            int partition_tokens, void* workspace, size_t workspace_bytes, int32_t* err_word,
                            void* stream);

/*
 * pa_decode_step_shared_prefix -- one decode step over shared prefixes: exactly
 *     pa_reshape_and_cache(k, v, slot_mapping, ..., num_tokens = num_seqs, ...)
 *     pa_decode_shared_prefix(q, ...)
 * in one call (P2 §2.1: the step's new K/V enter their slots, then the step's
 * query attends over the whole context; P3 §四: the beams share the prompt).
 * The shared-prefix kernel is launched as a programmatic dependent of the cache
 * write: its launch and start overlap the write, it waits for the write to
 * complete before it reads anything, and only then lets the decode engine launch.
 * The result is exactly that of the two calls.  Arguments, layouts, ownership and
 * errors as those two calls; the checks of both run before anything is launched.
 */
int pa_decode_step_shared_prefix(const void* k, const void* v, const int64_t* slot_mapping, const void* q,
                                 void* k_cache, void* v_cache, const int32_t* block_tables,
                                 const int32_t* context_lens, float scale, int num_kv_heads, void* out, int num_seqs,
                                 int num_heads, int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                                 int dtype, const int32_t* seq_start, int num_groups, const int32_t* group_offsets,
                                 const int32_t* group_members, int max_group_size, int max_shared_tokens,
                                 int partition_tokens, void* workspace, size_t workspace_bytes, int32_t* err_word,
                                 void* stream);

/*
 * pa_find_shared_prefixes -- host-side grouping for pa_decode_shared_prefix.
 * Sequences whose first partition (partition_tokens tokens) maps to the same
 * physical blocks form a group; the group shares the longest run of whole
 * partitions that all members map to the same blocks and that lies strictly
 * below every member's length.  Groups of one sequence are not formed.
 *   block_tables  [num_seqs][max_blocks_per_seq] int32, host;  context_lens host
 *   seq_start     [num_seqs] out (0 outside groups)
 *   group_offsets [num_seqs + 1] out;  group_members [num_seqs] out
 *   num_groups, max_group_size, max_shared_tokens  out
 * partition_tokens must be a positive multiple of block_size (the value passed
 * to the decode call, or pa_decode_partition_tokens(...)).  Table entries are
 * compared, not range-checked (the device kernels check them).
 */
int pa_find_shared_prefixes(const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                            int max_blocks_per_seq, int block_size, int partition_tokens, int32_t* seq_start,
                            int32_t* group_offsets, int32_t* group_members, int* num_groups, int* max_group_size,
                            int* max_shared_tokens);

/* ------------------------------------------------------------ diagnostics */

/*
 * pa_selftest_bounded_wait -- no counterpart on the pages: a check of the
 * library's failure path.  Launches one warp that waits, with the library's
 * bounded mbarrier wait, on a barrier nothing arrives at.  The wait gives up by
 * itself (its bound is about 2 s), OR-s PA_DEVERR_TIMEOUT into *err_word and the
 * kernel returns; the context stays usable.  *outcome (device int32, may be
 * NULL) becomes 0 when the wait gave up (1 would mean the phase completed).
 */
int pa_selftest_bounded_wait(int32_t* err_word, int32_t* outcome, void* stream);

/* ---------------------------------------------------------------- fp8 cache */

/*
 * fp8 (E4M3) KV cache: half the bytes per token.  The pages point at quantising
 * the cache (P1, closing note; P2 §5, memory -64% "with quantisation") without
 * fixing a format; this library stores OCP E4M3 codes ("e4m3fn": 1 sign, 4
 * exponent bits with bias 7, 3 fraction bits, no infinities, largest finite value
 * 448) with one fp32 scale per cache: the stored value of an element is
 * code * k_scale (code * v_scale).  Caches are uint8
 * [num_blocks][block_size][num_kv_heads][head_dim]; q, k, v and out stay fp16 or bf16.
 */

/*
 * pa_reshape_and_cache_fp8 -- pa_reshape_and_cache into fp8 caches.  Each element
 * x of k (v) is stored as the E4M3 code nearest to x / k_scale (x / v_scale),
 * the quotient taken in fp32 (IEEE division, round to nearest) and then rounded to
 * nearest even, saturating at +-448 (NaN stays NaN).  Scales must be positive and
 * finite.  head_dim must be a multiple of 16.
 */
int pa_reshape_and_cache_fp8(const void* k, const void* v, const int64_t* slot_mapping, void* k_cache,
                             void* v_cache, int num_tokens, int num_kv_heads, int head_dim, int block_size,
                             int num_blocks, int dtype, float k_scale, float v_scale, int32_t* err_word,
                             void* stream);

/*
 * pa_decode_fp8 -- pa_decode over fp8 caches: the same softmax(scale * q K^T) V
 * with K = code * k_scale and V = code * v_scale.  The codes widen exactly to f16;
 * q K^T is accumulated in fp32 from exact f16 x f16 products and scaled by
 * scale * k_scale afterwards, and v_scale multiplies the result.  fp16 q enters
 * as it is; bf16 q as q * 2^k in f16, with 2^k chosen per unit from its largest
 * |q| (exact for every element above 2^-31 of that one; smaller ones round to
 * f16's subnormal grid) and undone on the scores.  GQA groups of 2-16 share each
 * K/V fetch and run both products on tensor cores (P^T as a 16-bit hi + lo pair);
 * MHA and larger groups run on CUDA cores, one query head per unit.  head_dim 128
 * only; every other argument, the workspace and the errors as pa_decode.
 */
int pa_decode_fp8(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                  const int32_t* context_lens, float scale, float k_scale, float v_scale, int num_kv_heads, void* out,
                  int num_seqs, int num_heads, int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
                  int dtype, int partition_tokens, void* workspace, size_t workspace_bytes, int32_t* err_word,
                  void* stream);

/*
 * pa_decode_step_fp8 -- pa_decode_step over fp8 caches: exactly
 *     pa_reshape_and_cache_fp8(k, v, slot_mapping, ..., num_tokens = num_seqs, ...)
 *     pa_decode_fp8(q, ...)
 * in one call, the attention launched as a programmatic dependent of the cache
 * write as in pa_decode_step.  Arguments as those two calls; the checks of both
 * run before anything is launched.
 */
int pa_decode_step_fp8(const void* k, const void* v, const int64_t* slot_mapping, const void* q, void* k_cache,
                       void* v_cache, const int32_t* block_tables, const int32_t* context_lens, float scale,
                       float k_scale, float v_scale, int num_kv_heads, void* out, int num_seqs, int num_heads,
                       int head_dim, int block_size, int num_blocks, int max_blocks_per_seq, int dtype,
                       int partition_tokens, void* workspace, size_t workspace_bytes, int32_t* err_word,
                       void* stream);

/* ----------------------------------------------------------------- prefill */

/*
 * pa_prefill -- causal attention of a chunk of new query tokens over the paged
 * cache: the step before decode (P2 §2.1: the prompt's K/V enter the cache and
 * each position attends to the ones before it; with prefix reuse, P3 §三, the
 * chunk starts after tokens already cached).
 *
 * Sequence s contributes n_s = query_start[s+1] - query_start[s] query rows, packed
 * by sequence; its cache already holds all L_s = context_lens[s] tokens, the
 * chunk's own K/V included (written by pa_reshape_and_cache with the slots of
 * pa_prefill_slots).  Query row i of sequence s sits at position L_s - n_s + i and
 * attends, with one softmax, to tokens 0 .. L_s - n_s + i through the block table:
 *     out[row][h] = softmax(scale * q[row][h] K[0..pos]^T) V[0..pos]   (h_kv = h / g)
 *
 *   q, out        [T][num_heads][head_dim], T = query_start[num_seqs], dtype, device
 *   query_start   int32 [num_seqs + 1], device; n_s <= context_lens[s]
 *   max_query_len the largest n_s (sizes the grid)
 * Caches, tables, lengths, dtype and supported sizes as pa_decode.  Runs on the
 * 5th-generation tensor cores (tcgen05 MMAs, fp32 accumulators in tensor
 * memory).  The softmax weights p (at most 2^8 by construction) enter P.V as one
 * f16 term for f16 inputs, or as two bf16 terms (hi + lo) for bf16 inputs.
 * Bad lengths or table entries give NaN rows and PA_DEVERR_* bits.
 */
int pa_prefill(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
               const int32_t* context_lens, const int32_t* query_start, float scale, int num_kv_heads, void* out,
               int num_seqs, int num_heads, int head_dim, int block_size, int num_blocks, int max_blocks_per_seq,
               int max_query_len, int dtype, int32_t* err_word, void* stream);

/* ---------------------------------------------------------- host allocator */

/*
 * Refcounted block allocator over num_blocks physical block ids, after the block
 * pool of P3 §三 (BlockPool, BlockTable, PageAttentionManager) and the beam-search
 * fork of P3 §四:
 *   - free ids wait in a FIFO queue: allocation takes the front and sets the
 *     reference count to 1; a block whose count drops to 0 goes to the back;
 *   - add_ref / fork add one reference per block (prefix sharing, beam fork);
 *   - multi-block allocation is all-or-nothing.
 * Unlike the listing's saturating free, freeing or add_ref-ing a block whose
 * count is 0 is an error (PA_ERR_REFCOUNT) so that double frees surface.
 * Every call that fails leaves the allocator unchanged.
 */
typedef struct pa_allocator pa_allocator;

/* initial_order: NULL for 0..num_blocks-1, else a permutation giving the initial
 * order of the free queue.  Returns NULL on a bad argument or out of memory. */
pa_allocator* pa_allocator_create(int num_blocks, const int32_t* initial_order);
void pa_allocator_destroy(pa_allocator* a);

/* BlockTable::num_required_blocks (P3 §三): ceil(num_tokens / block_size); -1 on bad input. */
int pa_num_required_blocks(int num_tokens, int block_size);

int pa_alloc(pa_allocator* a, int32_t* out_id);                     /* one block */
int pa_alloc_n(pa_allocator* a, int n, int32_t* out_ids);           /* n blocks, all or nothing */
int pa_free(pa_allocator* a, int32_t id);                           /* drop one reference */
int pa_free_n(pa_allocator* a, int n, const int32_t* ids);          /* drop one reference each (free_request) */
int pa_add_ref(pa_allocator* a, int32_t id);                        /* one more reference */
/* dst[i] = src[i] with one more reference each: a beam fork or a shared prefix
 * (P3 §三 share_prefix_blocks; P3 §四, beam search).  dst may equal src. */
int pa_fork(pa_allocator* a, const int32_t* src, int n, int32_t* dst);
int pa_refcount(const pa_allocator* a, int32_t id);                 /* -1 for an id out of range */
int pa_num_free(const pa_allocator* a);
int pa_num_blocks(const pa_allocator* a);
double pa_usage(const pa_allocator* a);                             /* allocated / total (usage_ratio) */

/*
 * pa_append_slots -- slot resolution for one decode step (host; step a1).
 *
 * For each sequence s, n = context_lens[s] tokens are stored before this step.
 * The new token goes to position n: when n % block_size == 0 a block is
 * allocated first and written to block_tables[s][n / block_size]
 * (PageAttentionManager::append_slot, P3 §三).  Then
 *     slot_mapping[s] = block_tables[s][n / block_size] * block_size + n % block_size
 * and context_lens[s] becomes n + 1, the length pa_decode takes.
 *
 *   block_tables  host int32 [num_seqs][max_blocks_per_seq], in/out
 *   context_lens  host int32 [num_seqs], in/out
 *   slot_mapping  host int64 [num_seqs], out
 * All or nothing: PA_ERR_OUT_OF_BLOCKS (too few free blocks for every sequence on
 * a boundary) or PA_ERR_INVALID_ARG (a table full, an id out of range) leaves all
 * three arrays and the allocator unchanged.
 */
int pa_append_slots(pa_allocator* a, int32_t* block_tables, int max_blocks_per_seq, int32_t* context_lens,
                    int num_seqs, int block_size, int64_t* slot_mapping);

/*
 * pa_prefill_slots -- slot resolution for a chunk of new tokens per sequence
 * (host; the prefill analogue of pa_append_slots).
 *
 * Sequence s holds n = context_lens[s] tokens and appends m = new_tokens[s]: its
 * new tokens take positions n .. n+m-1, a block being allocated each time a
 * position opens one (P3 §三, allocate_for_request / append_slot), and
 *     slot_mapping[k] = block_tables[s][pos / block_size] * block_size + pos % block_size
 * for the k-th new token overall, sequences in order.  context_lens[s] becomes
 * n + m.  All or nothing (PA_ERR_OUT_OF_BLOCKS, PA_ERR_INVALID_ARG).
 *   slot_mapping  host int64 [sum of new_tokens], out
 */
int pa_prefill_slots(pa_allocator* a, int32_t* block_tables, int max_blocks_per_seq, int32_t* context_lens,
                     const int32_t* new_tokens, int num_seqs, int block_size, int64_t* slot_mapping);

/* ------------------------------------------------------------ copy-on-write */

/*
 * pa_cow_prepare -- copy-on-write before appending into a shared block (host).
 *
 * A beam fork copies block references, each shared block's count going up by one
 * (P3 §四, beam search; P3 §三, share_prefix_blocks).  When a sequence then appends
 * into a shared block that is only partly filled, it must first get a private copy
 * (the pages stop at the fork; this is the plainest completion of it).  For each
 * sequence s with n = context_lens[s] stored tokens and n % block_size != 0, the
 * next token goes into block j = n / block_size; if that block's reference count
 * is above 1, a fresh block is allocated into block_tables[s][j], one reference of
 * the shared block is dropped, and the pair (shared, fresh) is appended to
 * copy_pairs.  Sequences are handled in order, so of c sequences appending into
 * one block held by exactly c references, the last keeps the original.
 *
 *   block_tables  host int32 [num_seqs][max_blocks_per_seq], in/out
 *   context_lens  host int32 [num_seqs] (stored tokens, not changed)
 *   copy_pairs    host int32 [2 * num_seqs] out: (src, dst) pairs; *num_copies pairs
 * All or nothing: PA_ERR_OUT_OF_BLOCKS or PA_ERR_INVALID_ARG change nothing.  Run
 * pa_copy_blocks on the pairs before the step's pa_reshape_and_cache.
 */
int pa_cow_prepare(pa_allocator* a, int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                   int num_seqs, int block_size, int32_t* copy_pairs, int* num_copies);

/*
 * pa_copy_blocks -- copy whole physical blocks of both caches on the device.
 *
 * For i < num_pairs: k_cache[dst_i] = k_cache[src_i] and v_cache[dst_i] =
 * v_cache[src_i], all block_size x num_kv_heads x head_dim elements, bit for bit.
 *   copy_pairs  device int32 [2 * num_pairs]: (src, dst) per pair
 *   element_bytes  bytes per cache element (2 for fp16/bf16, 1 for 8-bit caches)
 * The pairs are copied all at once, so they must not overlap: a pair whose
 * destination is another pair's destination or source, or whose source is
 * another pair's destination, is skipped and sets PA_DEVERR_PAIR_CONFLICT (a
 * chained list such as (a, b), (b, c) is refused rather than copied in some
 * order; pa_cow_prepare never produces one).  Several pairs may share a source.
 * A pair with an id outside [0, num_blocks) is skipped and sets
 * PA_DEVERR_TABLE_RANGE.
 */
int pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* copy_pairs, int num_pairs, int num_kv_heads,
                   int head_dim, int block_size, int num_blocks, int element_bytes, int32_t* err_word,
                   void* stream);

/* ---------------------------------------------------------------- swapping */

/*
 * pa_swap_plan -- move one sequence's blocks from one pool to another (host).
 *
 * When no block is free for an append, a sequence is preempted: its KV blocks go to
 * host memory and come back when the device has room (P3 §三, append_slot's
 * "Preemption required"; P3 §五, swap to CPU memory and back).  With one allocator
 * per pool (device pool, pinned host pool), this allocates num_blocks blocks in
 * `to`, drops one reference of each listed block in `from` (a block shared with
 * other sequences stays allocated for them), writes the (old, new) id pairs to
 * `pairs` (int32 [2 * num_blocks]) and rewrites table_row with the new ids.
 * All or nothing.  Copy the data with pa_swap_blocks before the freed blocks can
 * be written again (stream order does this when both run on one stream).
 */
int pa_swap_plan(pa_allocator* from, pa_allocator* to, int32_t* table_row, int num_blocks, int32_t* pairs);

/*
 * pa_swap_blocks -- copy blocks between two block pools of the same geometry.
 *
 * For i < num_pairs: dst pool block pairs[2i+1] := src pool block pairs[2i], K and
 * V, bit for bit.  Either pool may be pinned host memory that the device can
 * address (cudaHostAlloc / cudaMallocHost memory under unified addressing), so
 * one kernel moves a preempted sequence's blocks out to host memory or back in,
 * without a staging buffer.  Pools are [num_blocks][block_size][num_kv_heads]
 * [head_dim] of element_bytes each; pairs is int32 [2 * num_pairs] in device-
 * readable memory.  Ids outside their pool are skipped and set PA_DEVERR_TABLE_RANGE.
 */
int pa_swap_blocks(const void* src_k, const void* src_v, int src_num_blocks, void* dst_k, void* dst_v,
                   int dst_num_blocks, const int32_t* pairs, int num_pairs, int num_kv_heads, int head_dim,
                   int block_size, int element_bytes, int32_t* err_word, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
