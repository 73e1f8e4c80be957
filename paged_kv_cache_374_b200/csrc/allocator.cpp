// Host block allocator behind the pa_allocator_* / pa_append_slots calls.
//
// The block pool of P3 ("LLM 推理中的 PageAttention 实现原理", §三: BlockPool,
// BlockTable, PageAttentionManager) as a flat C++ structure: one int32 reference
// count per physical block and a ring buffer holding the FIFO free queue.  The
// ring has exactly num_blocks slots, enough because a block sits in the queue only
// while its count is zero.  Every operation validates first and mutates second, so
// a failing call leaves the allocator as it was.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstdlib>
#include <new>
#include <vector>

#include "../../include/pa.h"

struct pa_allocator {
    int32_t n = 0;
    std::vector<int32_t> ref;    // reference count per block
    std::vector<int32_t> ring;   // free queue storage
    int32_t head = 0;            // index of the queue's front in `ring`
    int32_t count = 0;           // blocks in the queue

    int32_t pop_front() {
        int32_t id = ring[head];
        head = head + 1 == n ? 0 : head + 1;
        --count;
        return id;
    }
    void push_back(int32_t id) {
        int32_t tail = head + count;
        if (tail >= n) tail -= n;
        ring[tail] = id;
        ++count;
    }
    bool valid(int32_t id) const { return id >= 0 && id < n; }
};

extern "C" {

pa_allocator* pa_allocator_create(int num_blocks, const int32_t* initial_order) {
    if (num_blocks < 0) return nullptr;
    pa_allocator* a = new (std::nothrow) pa_allocator();
    if (!a) return nullptr;
    try {
        a->n = num_blocks;
        a->ref.assign(num_blocks, 0);
        a->ring.resize(num_blocks);
    } catch (...) {
        delete a;
        return nullptr;
    }
    std::vector<char> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
        int32_t id = initial_order ? initial_order[i] : i;
        if (id < 0 || id >= num_blocks || seen[id]) {  // not a permutation
            delete a;
            return nullptr;
        }
        seen[id] = 1;
        a->ring[i] = id;
    }
    a->head = 0;
    a->count = num_blocks;
    return a;
}

void pa_allocator_destroy(pa_allocator* a) { delete a; }

int pa_num_required_blocks(int num_tokens, int block_size) {
    if (num_tokens < 0 || block_size <= 0) return -1;
    return (int)(((int64_t)num_tokens + block_size - 1) / block_size);
}

int pa_alloc(pa_allocator* a, int32_t* out_id) {
    if (!a || !out_id) return PA_ERR_INVALID_ARG;
    if (a->count == 0) return PA_ERR_OUT_OF_BLOCKS;
    int32_t id = a->pop_front();
    a->ref[id] = 1;
    *out_id = id;
    return PA_OK;
}

int pa_alloc_n(pa_allocator* a, int n, int32_t* out_ids) {
    if (!a || n < 0 || (n > 0 && !out_ids)) return PA_ERR_INVALID_ARG;
    if (a->count < n) return PA_ERR_OUT_OF_BLOCKS;  // checked before anything is taken
    for (int i = 0; i < n; ++i) {
        int32_t id = a->pop_front();
        a->ref[id] = 1;
        out_ids[i] = id;
    }
    return PA_OK;
}

int pa_free(pa_allocator* a, int32_t id) {
    if (!a || !a->valid(id)) return PA_ERR_INVALID_ARG;
    if (a->ref[id] == 0) return PA_ERR_REFCOUNT;
    if (--a->ref[id] == 0) a->push_back(id);
    return PA_OK;
}

int pa_free_n(pa_allocator* a, int n, const int32_t* ids) {
    if (!a || n < 0 || (n > 0 && !ids)) return PA_ERR_INVALID_ARG;
    // Validate against the counts the sequence of frees would see (an id may repeat).
    std::vector<int32_t> drops;
    try {
        drops.assign(n, 0);
    } catch (...) {
        return PA_ERR_INVALID_ARG;
    }
    for (int i = 0; i < n; ++i) {
        if (!a->valid(ids[i])) return PA_ERR_INVALID_ARG;
        int seen = 0;
        for (int j = 0; j < i; ++j) seen += ids[j] == ids[i];
        if (a->ref[ids[i]] - seen <= 0) return PA_ERR_REFCOUNT;
    }
    for (int i = 0; i < n; ++i) {
        int32_t id = ids[i];
        if (--a->ref[id] == 0) a->push_back(id);
    }
    return PA_OK;
}

int pa_add_ref(pa_allocator* a, int32_t id) {
    if (!a || !a->valid(id)) return PA_ERR_INVALID_ARG;
    if (a->ref[id] == 0) return PA_ERR_REFCOUNT;
    ++a->ref[id];
    return PA_OK;
}

int pa_fork(pa_allocator* a, const int32_t* src, int n, int32_t* dst) {
    if (!a || n < 0 || (n > 0 && (!src || !dst))) return PA_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        if (!a->valid(src[i])) return PA_ERR_INVALID_ARG;
        if (a->ref[src[i]] == 0) return PA_ERR_REFCOUNT;
    }
    for (int i = 0; i < n; ++i) {
        int32_t id = src[i];
        ++a->ref[id];
        dst[i] = id;
    }
    return PA_OK;
}

int pa_refcount(const pa_allocator* a, int32_t id) {
    if (!a || !a->valid(id)) return -1;
    return a->ref[id];
}

int pa_num_free(const pa_allocator* a) { return a ? a->count : -1; }

int pa_num_blocks(const pa_allocator* a) { return a ? a->n : -1; }

double pa_usage(const pa_allocator* a) {
    if (!a || a->n == 0) return 0.0;
    return (double)(a->n - a->count) / (double)a->n;
}

int pa_append_slots(pa_allocator* a, int32_t* block_tables, int max_blocks_per_seq, int32_t* context_lens,
                    int num_seqs, int block_size, int64_t* slot_mapping) {
    if (!a || num_seqs < 0 || max_blocks_per_seq < 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
    if (num_seqs > 0 && (!block_tables || !context_lens || !slot_mapping)) return PA_ERR_INVALID_ARG;
    // Pass 1: validate and count the sequences that sit on a block boundary.
    int need = 0;
    for (int s = 0; s < num_seqs; ++s) {
        int64_t n = context_lens[s];
        if (n < 0 || n == INT32_MAX) return PA_ERR_INVALID_ARG;
        int64_t j = n / block_size;
        if (j >= max_blocks_per_seq) return PA_ERR_INVALID_ARG;  // the table row is full
        if (n % block_size == 0) {
            ++need;
        } else {
            int32_t id = block_tables[(int64_t)s * max_blocks_per_seq + j];
            if (!a->valid(id) || a->ref[id] == 0) return PA_ERR_INVALID_ARG;
        }
    }
    if (a->count < need) return PA_ERR_OUT_OF_BLOCKS;  // "Preemption required"
    // Pass 2: allocate in sequence order and resolve each new token's slot.
    for (int s = 0; s < num_seqs; ++s) {
        int64_t n = context_lens[s];
        int64_t j = n / block_size;
        int32_t* row = block_tables + (int64_t)s * max_blocks_per_seq;
        if (n % block_size == 0) {
            int32_t id = a->pop_front();
            a->ref[id] = 1;
            row[j] = id;
        }
        slot_mapping[s] = (int64_t)row[j] * block_size + n % block_size;
        context_lens[s] = (int32_t)(n + 1);
    }
    return PA_OK;
}

int pa_prefill_slots(pa_allocator* a, int32_t* block_tables, int max_blocks_per_seq, int32_t* context_lens,
                     const int32_t* new_tokens, int num_seqs, int block_size, int64_t* slot_mapping) {
    if (!a || num_seqs < 0 || max_blocks_per_seq < 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
    if (num_seqs > 0 && (!block_tables || !context_lens || !new_tokens || !slot_mapping)) return PA_ERR_INVALID_ARG;
    // Pass 1: validate and count the blocks the chunks open.
    int64_t need = 0;
    for (int s = 0; s < num_seqs; ++s) {
        const int64_t n = context_lens[s], m = new_tokens[s];
        if (n < 0 || m < 0 || n + m > INT32_MAX) return PA_ERR_INVALID_ARG;
        const int64_t have = (n + block_size - 1) / block_size;
        const int64_t want = (n + m + block_size - 1) / block_size;
        if (want > max_blocks_per_seq) return PA_ERR_INVALID_ARG;  // the table row is too short
        if (n % block_size != 0 && m > 0) {  // the chunk starts inside the last held block
            const int32_t id = block_tables[(int64_t)s * max_blocks_per_seq + n / block_size];
            if (!a->valid(id) || a->ref[id] == 0) return PA_ERR_INVALID_ARG;
        }
        need += want - have;
    }
    if (a->count < need) return PA_ERR_OUT_OF_BLOCKS;
    // Pass 2: open the blocks in sequence order and resolve every new token's slot.
    int64_t k = 0;
    for (int s = 0; s < num_seqs; ++s) {
        const int64_t n = context_lens[s], m = new_tokens[s];
        int32_t* row = block_tables + (int64_t)s * max_blocks_per_seq;
        for (int64_t pos = n; pos < n + m; ++pos) {
            if (pos % block_size == 0) {
                const int32_t id = a->pop_front();
                a->ref[id] = 1;
                row[pos / block_size] = id;
            }
            slot_mapping[k++] = (int64_t)row[pos / block_size] * block_size + pos % block_size;
        }
        context_lens[s] = (int32_t)(n + m);
    }
    return PA_OK;
}

int pa_cow_prepare(pa_allocator* a, int32_t* block_tables, int max_blocks_per_seq, const int32_t* context_lens,
                   int num_seqs, int block_size, int32_t* copy_pairs, int* num_copies) {
    if (!a || num_seqs < 0 || max_blocks_per_seq < 0 || block_size <= 0 || !num_copies) return PA_ERR_INVALID_ARG;
    if (num_seqs > 0 && (!block_tables || !context_lens || !copy_pairs)) return PA_ERR_INVALID_ARG;
    // Pass 1: validate, and count per shared block how many sequences append into it.
    std::vector<int32_t> appenders;
    try {
        appenders.assign(a->n, 0);
    } catch (...) {
        return PA_ERR_INVALID_ARG;
    }
    for (int s = 0; s < num_seqs; ++s) {
        const int64_t n = context_lens[s];
        if (n < 0) return PA_ERR_INVALID_ARG;
        if (n % block_size == 0) continue;  // the next token opens a new block: nothing shared to copy
        const int64_t j = n / block_size;
        if (j >= max_blocks_per_seq) return PA_ERR_INVALID_ARG;
        const int32_t id = block_tables[(int64_t)s * max_blocks_per_seq + j];
        if (!a->valid(id) || a->ref[id] == 0) return PA_ERR_INVALID_ARG;
        ++appenders[id];
    }
    // A block with r references and c appenders in this batch needs c copies when
    // r > c (someone outside the batch keeps the original), else c - 1 (the last
    // appender keeps it).
    int64_t need = 0;
    for (int32_t id = 0; id < a->n; ++id) {
        const int32_t c = appenders[id];
        if (c == 0) continue;
        if (a->ref[id] < c) return PA_ERR_INVALID_ARG;  // a table lists a block it does not hold
        need += a->ref[id] > c ? c : c - 1;
    }
    if (a->count < need) return PA_ERR_OUT_OF_BLOCKS;
    // Pass 2: in sequence order, move each appender off a still-shared block.
    int k = 0;
    for (int s = 0; s < num_seqs; ++s) {
        const int64_t n = context_lens[s];
        if (n % block_size == 0) continue;
        int32_t* slot = block_tables + (int64_t)s * max_blocks_per_seq + n / block_size;
        const int32_t src = *slot;
        if (a->ref[src] <= 1) continue;
        const int32_t dst = a->pop_front();
        a->ref[dst] = 1;
        --a->ref[src];
        *slot = dst;
        copy_pairs[2 * k] = src;
        copy_pairs[2 * k + 1] = dst;
        ++k;
    }
    *num_copies = k;
    return PA_OK;
}

int pa_swap_plan(pa_allocator* from, pa_allocator* to, int32_t* table_row, int num_blocks, int32_t* pairs) {
    if (!from || !to || from == to || num_blocks < 0 || (num_blocks > 0 && (!table_row || !pairs)))
        return PA_ERR_INVALID_ARG;
    for (int i = 0; i < num_blocks; ++i) {
        const int32_t id = table_row[i];
        if (!from->valid(id) || from->ref[id] == 0) return PA_ERR_INVALID_ARG;
        int seen = 0;  // a row listing one block twice would drop two references
        for (int j = 0; j < i; ++j) seen += table_row[j] == id;
        if (from->ref[id] - seen <= 0) return PA_ERR_REFCOUNT;
    }
    if (to->count < num_blocks) return PA_ERR_OUT_OF_BLOCKS;
    for (int i = 0; i < num_blocks; ++i) {
        const int32_t old = table_row[i];
        const int32_t fresh = to->pop_front();
        to->ref[fresh] = 1;
        if (--from->ref[old] == 0) from->push_back(old);
        pairs[2 * i] = old;
        pairs[2 * i + 1] = fresh;
        table_row[i] = fresh;
    }
    return PA_OK;
}

int pa_find_shared_prefixes(const int32_t* block_tables, const int32_t* context_lens, int num_seqs,
                            int max_blocks_per_seq, int block_size, int partition_tokens, int32_t* seq_start,
                            int32_t* group_offsets, int32_t* group_members, int* num_groups, int* max_group_size,
                            int* max_shared_tokens) {
    if (num_seqs < 0 || max_blocks_per_seq < 0 || block_size <= 0 || partition_tokens <= 0 ||
        partition_tokens % block_size != 0 || !num_groups || !max_group_size || !max_shared_tokens)
        return PA_ERR_INVALID_ARG;
    if (num_seqs > 0 && (!block_tables || !context_lens || !seq_start || !group_offsets || !group_members))
        return PA_ERR_INVALID_ARG;
    const int P = partition_tokens, epp = partition_tokens / block_size;  // table entries per partition
    const int64_t maxlen = (int64_t)max_blocks_per_seq * block_size;
    auto row = [&](int s) { return block_tables + (int64_t)s * max_blocks_per_seq; };
    auto same = [&](int x, int y, int k) {  // partition k of x and y uses the same blocks
        return std::equal(row(x) + (int64_t)k * epp, row(x) + (int64_t)(k + 1) * epp, row(y) + (int64_t)k * epp);
    };
    // candidates: at least one whole partition strictly below the length
    std::vector<int> cand;
    for (int s = 0; s < num_seqs; ++s) {
        seq_start[s] = 0;
        if (context_lens[s] > P && context_lens[s] <= maxlen) cand.push_back(s);
    }
    int ng = 0, pos = 0, maxg = 0, maxtok = 0;
    group_offsets[0] = 0;
    auto kmax = [&](int x) { return (context_lens[x] - 1) / P; };  // whole partitions below the length
    auto emit = [&](std::vector<int>& mem, int k) {
        std::sort(mem.begin(), mem.end());
        for (int x : mem) {
            seq_start[x] = k * P;
            group_members[pos++] = x;
        }
        group_offsets[++ng] = pos;
        maxg = std::max(maxg, (int)mem.size());
        maxtok = std::max(maxtok, k * P);
    };
    // `mem` (two or more) share partitions [0, k).  Members that also share
    // partition k with at least one other member split off with a longer prefix;
    // the rest form a group sharing k partitions.
    std::vector<std::pair<std::vector<int>, int>> work;
    auto split = [&](std::vector<int> mem, int k) {
        std::vector<int> rest, ext;
        for (int x : mem) (kmax(x) > k ? ext : rest).push_back(x);
        std::sort(ext.begin(), ext.end(), [&](int x, int y) {
            const int32_t *a = row(x) + (int64_t)k * epp, *b = row(y) + (int64_t)k * epp;
            for (int i = 0; i < epp; ++i)
                if (a[i] != b[i]) return a[i] < b[i];
            return x < y;
        });
        for (size_t i = 0; i < ext.size();) {
            size_t j = i + 1;
            while (j < ext.size() && same(ext[i], ext[j], k)) ++j;
            if (j - i >= 2)
                work.emplace_back(std::vector<int>(ext.begin() + i, ext.begin() + j), k + 1);
            else
                rest.push_back(ext[i]);
            i = j;
        }
        if (rest.size() >= 2 && k > 0) emit(rest, k);
    };
    work.emplace_back(cand, 0);
    while (!work.empty()) {
        auto item = std::move(work.back());
        work.pop_back();
        split(std::move(item.first), item.second);
    }
    *num_groups = ng;
    *max_group_size = maxg;
    *max_shared_tokens = maxtok;
    return PA_OK;
}

const char* pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_OUT_OF_BLOCKS: return "PA_ERR_OUT_OF_BLOCKS";
        case PA_ERR_REFCOUNT: return "PA_ERR_REFCOUNT";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        default: return "PA_ERR_UNKNOWN";
    }
}

}  // extern "C"
