// Host block allocator: a pool of fixed-size physical blocks handed out
// slab-style from a free stack, with per-block reference counts, immediate
// reclamation at count zero, fork (prefix sharing) and copy-on-write.
//
// Sources: "PagedAttention技术解析" 2.1 (Block {ref_count, is_allocated},
// O(1) allocation, fork-like sharing), 4.2 (reclaim at ref_count 0, keep a
// free pool); "VLLM中PagedAttention如何降低显存碎片？" 三 items 7-8 (slab-style
// frames, shared prefix pages); "vLLM内存管理与PagedAttention精讲" ch.2 2.4
// (a new block only when the current one is full; copy-on-write when a
// shared block is written).
//
// Compaction ("PagedAttention技术解析" 2.1: defragmentation moves block
// pointers; 4.2 item 2: periodic defragmentation): with fixed-size blocks a
// free block serves any request, so the useful form is packing the live
// blocks below a target so the pool's tail can be released; the caller
// copies the moved blocks' data (pa_copy_blocks) and rewrites its tables
// (pa_seq_remap).
//
// Every operation is O(1) per block touched; failing calls change nothing.
#include <cstdint>
#include <cstring>
#include <unordered_map>
#include <vector>

#include "internal.h"

struct pa_allocator {
    int num_blocks;
    int block_size;
    std::vector<int32_t> stack;   // free blocks; back() is the top
    std::vector<int32_t> ref;     // reference count per block (0 = free)
};

namespace {

inline int blocks_for(int64_t tokens, int bs) { return (int)((tokens + bs - 1) / bs); }

inline bool valid_block(const pa_allocator* a, int32_t b) {
    return b >= 0 && b < a->num_blocks;
}

inline int32_t pop_block(pa_allocator* a) {
    int32_t b = a->stack.back();
    a->stack.pop_back();
    a->ref[b] = 1;
    return b;
}

inline void drop_ref(pa_allocator* a, int32_t b) {
    if (--a->ref[b] == 0) a->stack.push_back(b);
}

// Core of one append; the caller has already checked that a free block
// exists if one is needed.
inline void append_one(pa_allocator* a, int32_t* table, int* length, int64_t* slot,
                       int32_t* cow_src, int32_t* cow_dst) {
    const int bs = a->block_size;
    const int len = *length;
    const int idx = len / bs;
    *cow_src = -1;
    *cow_dst = -1;
    if (len % bs == 0) {
        table[idx] = pop_block(a);
    } else if (a->ref[table[idx]] > 1) {
        const int32_t old = table[idx];
        const int32_t fresh = pop_block(a);
        drop_ref(a, old);
        table[idx] = fresh;
        *cow_src = old;
        *cow_dst = fresh;
    }
    *slot = (int64_t)table[idx] * bs + len % bs;
    *length = len + 1;
}

// The table entry an append reads: the block holding the last token, when
// that block still has room (a full last block is not read: a fresh one
// follows).  An append touches nothing else, so this is the only entry it
// needs to trust; checking the whole table on every step would cost a random
// read per block of every sequence.
pa_status check_last_entry(const pa_allocator* a, const int32_t* table, int len) {
    const int bs = a->block_size;
    if (len % bs == 0) return PA_OK;
    const int32_t b = table[len / bs];
    if (!valid_block(a, b) || a->ref[b] <= 0)
        return pa::fail(PA_ERR_BAD_BLOCK_ID, "table entry %d (%d) is not an allocated block",
                        len / bs, (int)b);
    return PA_OK;
}

pa_status check_table(const pa_allocator* a, const int32_t* table, int n) {
    for (int i = 0; i < n; ++i) {
        if (!valid_block(a, table[i]) || a->ref[table[i]] <= 0)
            return pa::fail(PA_ERR_BAD_BLOCK_ID, "table entry %d (%d) is not an allocated block",
                            i, (int)table[i]);
    }
    return PA_OK;
}

}  // namespace

extern "C" {

pa_allocator* pa_alloc_create(int num_blocks, int block_size, const int32_t* order) {
    if (num_blocks <= 0 || block_size <= 0) {
        pa::fail(PA_ERR_INVALID_ARG, "num_blocks and block_size must be positive");
        return nullptr;
    }
    auto* a = new pa_allocator;
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->ref.assign(num_blocks, 0);
    a->stack.resize(num_blocks);
    std::vector<uint8_t> seen(num_blocks, 0);
    for (int i = 0; i < num_blocks; ++i) {
        const int32_t b = order ? order[i] : i;
        if (b < 0 || b >= num_blocks || seen[b]) {
            delete a;
            pa::fail(PA_ERR_INVALID_ARG, "initial_free_order is not a permutation (entry %d)", i);
            return nullptr;
        }
        seen[b] = 1;
        a->stack[num_blocks - 1 - i] = b;   // element 0 ends on top
    }
    return a;
}

void pa_alloc_destroy(pa_allocator* a) { delete a; }

pa_status pa_alloc_allocate(pa_allocator* a, int32_t* out) {
    if (!a || !out) return pa::fail(PA_ERR_INVALID_ARG, "null argument");
    if (a->stack.empty()) return pa::fail(PA_ERR_OUT_OF_BLOCKS, "no free block");
    *out = pop_block(a);
    return PA_OK;
}

pa_status pa_alloc_incref(pa_allocator* a, int32_t b) {
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "null allocator");
    if (!valid_block(a, b) || a->ref[b] <= 0)
        return pa::fail(PA_ERR_BAD_BLOCK_ID, "incref of unallocated block %d", (int)b);
    ++a->ref[b];
    return PA_OK;
}

pa_status pa_alloc_decref(pa_allocator* a, int32_t b) {
    if (!a) return pa::fail(PA_ERR_INVALID_ARG, "null allocator");
    if (!valid_block(a, b) || a->ref[b] <= 0)
        return pa::fail(PA_ERR_BAD_BLOCK_ID, "decref of unallocated block %d", (int)b);
    drop_ref(a, b);
    return PA_OK;
}

int pa_alloc_num_free(const pa_allocator* a) { return a ? (int)a->stack.size() : -1; }
int pa_alloc_num_blocks(const pa_allocator* a) { return a ? a->num_blocks : -1; }
int pa_alloc_block_size(const pa_allocator* a) { return a ? a->block_size : -1; }

int pa_alloc_ref_count(const pa_allocator* a, int32_t b) {
    if (!a || !valid_block(a, b)) return -1;
    return a->ref[b];
}

pa_status pa_alloc_free_order(const pa_allocator* a, int32_t* out, int capacity, int* count) {
    if (!a || (!out && capacity > 0)) return pa::fail(PA_ERR_INVALID_ARG, "null argument");
    const int n = (int)a->stack.size();
    if (count) *count = n;
    const int m = n < capacity ? n : capacity;
    for (int i = 0; i < m; ++i) out[i] = a->stack[n - 1 - i];
    return PA_OK;
}

pa_status pa_seq_append_slot(pa_allocator* a, int32_t* table, int capacity, int* length,
                             int64_t* slot, int32_t* cow_src, int32_t* cow_dst) {
    if (!a || !table || !length || !slot || !cow_src || !cow_dst || *length < 0)
        return pa::fail(PA_ERR_INVALID_ARG, "null argument or negative length");
    const int bs = a->block_size;
    const int len = *length;
    if (pa_status s = check_last_entry(a, table, len)) return s;
    const bool fresh = len % bs == 0;
    if (fresh && len / bs >= capacity)
        return pa::fail(PA_ERR_INVALID_ARG, "block table full (capacity %d)", capacity);
    const bool cow = !fresh && a->ref[table[len / bs]] > 1;
    if ((fresh || cow) && a->stack.empty())
        return pa::fail(PA_ERR_OUT_OF_BLOCKS, "no free block");
    append_one(a, table, length, slot, cow_src, cow_dst);
    return PA_OK;
}

pa_status pa_seq_append_slots(pa_allocator* a, int32_t* tables, int stride, int* lengths,
                              int num_seqs, int64_t* slots, int32_t* cow_pairs, int* num_cow) {
    if (!a || num_seqs < 0 || (num_seqs > 0 && (!tables || !lengths || !slots || !cow_pairs)))
        return pa::fail(PA_ERR_INVALID_ARG, "null argument");
    const int bs = a->block_size;
    // Count the blocks this batch needs, in processing order, without
    // touching the state (so OUT_OF_BLOCKS leaves everything unchanged).
    std::unordered_map<int32_t, int> pending;
    int64_t need = 0;
    for (int i = 0; i < num_seqs; ++i) {
        const int len = lengths[i];
        if (len < 0) return pa::fail(PA_ERR_INVALID_ARG, "negative length for sequence %d", i);
        int32_t* t = tables + (int64_t)i * stride;
        if (pa_status s = check_last_entry(a, t, len)) return s;
        if (len % bs == 0) {
            if (len / bs >= stride)
                return pa::fail(PA_ERR_INVALID_ARG, "block table %d full (stride %d)", i, stride);
            ++need;
        } else {
            const int32_t last = t[len / bs];
            auto it = pending.find(last);
            int count = it == pending.end() ? a->ref[last] : it->second;
            if (count > 1) {
                ++need;
                pending[last] = count - 1;
            }
        }
    }
    if (need > (int64_t)a->stack.size())
        return pa::fail(PA_ERR_OUT_OF_BLOCKS, "batch needs %lld blocks, %d free",
                        (long long)need, (int)a->stack.size());
    int ncow = 0;
    for (int i = 0; i < num_seqs; ++i) {
        int32_t src, dst;
        append_one(a, tables + (int64_t)i * stride, &lengths[i], &slots[i], &src, &dst);
        if (src >= 0) {
            cow_pairs[2 * ncow] = src;
            cow_pairs[2 * ncow + 1] = dst;
            ++ncow;
        }
    }
    if (num_cow) *num_cow = ncow;
    return PA_OK;
}

pa_status pa_seq_extend(pa_allocator* a, int32_t* table, int capacity, int* length,
                        int num_tokens, int64_t* slots, int32_t* cow_src, int32_t* cow_dst) {
    if (!a || !table || !length || !cow_src || !cow_dst || *length < 0 || num_tokens < 0)
        return pa::fail(PA_ERR_INVALID_ARG, "null argument or negative size");
    const int bs = a->block_size;
    const int len = *length;
    *cow_src = -1;
    *cow_dst = -1;
    if (num_tokens == 0) return PA_OK;
    const int have = blocks_for(len, bs);
    if (pa_status s = check_table(a, table, have)) return s;
    const int want = blocks_for((int64_t)len + num_tokens, bs);
    if (want > capacity)
        return pa::fail(PA_ERR_INVALID_ARG, "needs %d table entries, capacity %d", want, capacity);
    const bool cow = len % bs != 0 && a->ref[table[len / bs]] > 1;
    if ((int64_t)(want - have) + (cow ? 1 : 0) > (int64_t)a->stack.size())
        return pa::fail(PA_ERR_OUT_OF_BLOCKS, "extend needs %d blocks, %d free",
                        want - have + (cow ? 1 : 0), (int)a->stack.size());
    for (int k = 0; k < num_tokens; ++k) {
        int64_t s;
        int32_t src, dst;
        append_one(a, table, length, &s, &src, &dst);
        if (slots) slots[k] = s;
        if (k == 0) {
            *cow_src = src;
            *cow_dst = dst;
        }
    }
    return PA_OK;
}

pa_status pa_seq_fork(pa_allocator* a, const int32_t* parent, int n, int32_t* child) {
    if (!a || n < 0 || (n > 0 && (!parent || !child)))
        return pa::fail(PA_ERR_INVALID_ARG, "null argument");
    if (pa_status s = check_table(a, parent, n)) return s;
    for (int i = 0; i < n; ++i) {
        ++a->ref[parent[i]];
        child[i] = parent[i];
    }
    return PA_OK;
}

pa_status pa_alloc_compact(pa_allocator* a, int target, int32_t* moves, int capacity,
                           int* num_moves) {
    if (!a || !num_moves || target < 0 || target > a->num_blocks || capacity < 0 ||
        (capacity > 0 && !moves))
        return pa::fail(PA_ERR_INVALID_ARG, "bad compaction arguments");
    std::vector<int32_t> high, low;
    for (int32_t b = target; b < a->num_blocks; ++b)
        if (a->ref[b] > 0) high.push_back(b);
    for (int32_t b = 0; b < target; ++b)
        if (a->ref[b] == 0) low.push_back(b);       // ascending id
    if (high.size() > low.size())
        return pa::fail(PA_ERR_OUT_OF_BLOCKS, "%zu live blocks above %d, %zu free below", high.size(),
                        target, low.size());
    if ((int)high.size() > capacity)
        return pa::fail(PA_ERR_INVALID_ARG, "moves need %zu entries, capacity %d", high.size(),
                        capacity);
    std::vector<uint8_t> taken(target, 0);
    for (size_t i = 0; i < high.size(); ++i) {
        moves[2 * i] = high[i];
        moves[2 * i + 1] = low[i];
        a->ref[low[i]] = a->ref[high[i]];
        a->ref[high[i]] = 0;
        taken[low[i]] = 1;
    }
    // free stack keeps its order, minus blocks at or above the target and
    // the destinations just taken
    std::vector<int32_t> stack;
    stack.reserve(a->stack.size());
    for (int32_t b : a->stack)
        if (b < target && !taken[b]) stack.push_back(b);
    a->stack.swap(stack);
    a->ref.resize(target);
    a->num_blocks = target;
    *num_moves = (int)high.size();
    return PA_OK;
}

pa_status pa_seq_remap(int32_t* table, int n, const int32_t* moves, int num_moves) {
    if (n < 0 || num_moves < 0 || (n > 0 && !table) || (num_moves > 0 && !moves))
        return pa::fail(PA_ERR_INVALID_ARG, "null argument");
    std::unordered_map<int32_t, int32_t> where;
    where.reserve((size_t)num_moves * 2);
    for (int i = 0; i < num_moves; ++i) where[moves[2 * i]] = moves[2 * i + 1];
    for (int i = 0; i < n; ++i) {
        auto it = where.find(table[i]);
        if (it != where.end()) table[i] = it->second;
    }
    return PA_OK;
}

pa_status pa_seq_remap_batch(int32_t* tables, int stride, const int* lengths_in_blocks,
                             int num_seqs, const int32_t* moves, int num_moves) {
    if (num_seqs < 0 || num_moves < 0 || stride < 0 || (num_seqs > 0 && (!tables || !lengths_in_blocks)) ||
        (num_moves > 0 && !moves))
        return pa::fail(PA_ERR_INVALID_ARG, "null argument");
    for (int s = 0; s < num_seqs; ++s)
        if (lengths_in_blocks[s] < 0 || lengths_in_blocks[s] > stride)
            return pa::fail(PA_ERR_INVALID_ARG, "sequence %d: %d table entries, stride %d", s,
                            lengths_in_blocks[s], stride);
    // a dense map from every moved block to its new id (moves name blocks of
    // the pool before compaction, so the largest source bounds its size)
    int32_t top = -1;
    for (int i = 0; i < num_moves; ++i) {
        if (moves[2 * i] < 0 || moves[2 * i + 1] < 0)
            return pa::fail(PA_ERR_INVALID_ARG, "move %d names a negative block", i);
        if (moves[2 * i] > top) top = moves[2 * i];
    }
    std::vector<int32_t> where((size_t)top + 1, -1);
    for (int i = 0; i < num_moves; ++i) where[moves[2 * i]] = moves[2 * i + 1];
    for (int s = 0; s < num_seqs; ++s) {
        int32_t* t = tables + (size_t)s * stride;
        for (int j = 0; j < lengths_in_blocks[s]; ++j) {
            const int32_t b = t[j];
            if (b >= 0 && b <= top && where[b] >= 0) t[j] = where[b];
        }
    }
    return PA_OK;
}

pa_status pa_seq_free(pa_allocator* a, const int32_t* table, int n) {
    if (!a || n < 0 || (n > 0 && !table)) return pa::fail(PA_ERR_INVALID_ARG, "null argument");
    // a table may name one block more than once only through misuse; check
    // the counts cover every entry before dropping any
    std::unordered_map<int32_t, int> uses;
    for (int i = 0; i < n; ++i) {
        if (!valid_block(a, table[i]))
            return pa::fail(PA_ERR_BAD_BLOCK_ID, "table entry %d out of range", i);
        if (++uses[table[i]] > a->ref[table[i]])
            return pa::fail(PA_ERR_BAD_BLOCK_ID, "block %d freed more often than held",
                            (int)table[i]);
    }
    for (int i = 0; i < n; ++i) drop_ref(a, table[i]);
    return PA_OK;
}

}  // extern "C"
