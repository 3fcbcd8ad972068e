// Host-side refcounted block allocator with fork and copy-on-write.
//
// Semantics follow "Walk through paged attention end to end" (append step:
// a fresh block when next_pos % block_size == 0), "What is PagedAttention
// and how does it manage KV cache" (BlockTable.append_token; blocks return
// to the pool when a request finishes) and "PagedAttention & vLLM"
// (Copy-on-write sharing: a shared block is duplicated before a write).
// A fork shares every block of the parent, the partial last one included.
//
// Free blocks sit on a stack: the most recently freed block is reused first
// (it is the likeliest to still be warm in L2); a fresh allocator hands out
// blocks in the order it was given.
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/pa.h"

namespace {

struct Seq {
    std::vector<int32_t> blocks;
    int64_t tokens = 0;
    bool live = false;
};

// One undo record of a batched append.
struct Undo {
    int32_t seq;
    int32_t taken;    // block taken from the free stack, or -1
    int32_t replaced; // block the copy replaced (CoW), or -1
};

}  // namespace

struct pa_allocator {
    int32_t num_blocks = 0;
    int32_t block_size = 0;
    std::vector<int32_t> free_stack;  // back() is handed out next
    std::vector<int32_t> ref;
    std::vector<Seq> seqs;

    bool valid_seq(int id) const { return id >= 0 && id < (int)seqs.size() && seqs[id].live; }

    // Append one token to sequence `id`.  Returns PA_OK or PA_ERR_OOM; on OOM
    // nothing changed.  `undo` (optional) records how to revert the step.
    int append(int id, int32_t *slot, int32_t *cow_src, int32_t *cow_dst, Undo *undo) {
        Seq &s = seqs[id];
        const int64_t n = s.tokens;
        const int64_t j = n / block_size;
        const int32_t row = (int32_t)(n % block_size);
        int32_t src = -1, dst = -1, taken = -1, replaced = -1;
        if (row == 0) {
            if (free_stack.empty()) return PA_ERR_OOM;
            taken = free_stack.back();
            free_stack.pop_back();
            ref[taken] = 1;
            s.blocks.push_back(taken);
        } else {
            const int32_t cur = s.blocks[j];
            if (ref[cur] > 1) {
                if (free_stack.empty()) return PA_ERR_OOM;
                taken = free_stack.back();
                free_stack.pop_back();
                ref[taken] = 1;
                ref[cur] -= 1;
                s.blocks[j] = taken;
                replaced = cur;
                src = cur;
                dst = taken;
            }
        }
        s.tokens = n + 1;
        *slot = s.blocks[j] * block_size + row;
        if (cow_src) *cow_src = src;
        if (cow_dst) *cow_dst = dst;
        if (undo) *undo = Undo{id, taken, replaced};
        return PA_OK;
    }

    void revert(const Undo &u) {
        Seq &s = seqs[u.seq];
        s.tokens -= 1;
        if (u.taken >= 0) {
            if (u.replaced >= 0) {  // copy-on-write: restore the shared block
                const int64_t j = s.tokens / block_size;
                s.blocks[j] = u.replaced;
                ref[u.replaced] += 1;
            } else {
                s.blocks.pop_back();
            }
            ref[u.taken] = 0;
            free_stack.push_back(u.taken);
        }
    }
};

namespace {

// Appends one token to each of ids[0..n) in order, all or nothing: on any
// failure (out of blocks, or a table growing past max_blocks) every append
// of the call is reverted.  Copy-on-write pairs go to pairs[2k], pairs[2k+1];
// slots (optional) receive each new token's slot.
int append_all(pa_allocator *a, const int32_t *ids, int n, int32_t *slots, int32_t *pairs, int *ncow,
               int64_t max_blocks) {
    std::vector<Undo> log;
    log.reserve((size_t)n);
    int count = 0;
    int st = PA_OK;
    for (int i = 0; i < n && st == PA_OK; ++i) {
        int32_t slot, src, dst;
        Undo u;
        st = a->append(ids[i], &slot, &src, &dst, &u);
        if (st != PA_OK) break;
        log.push_back(u);
        if (slots) slots[i] = slot;
        if (src >= 0) {
            pairs[2 * count] = src;
            pairs[2 * count + 1] = dst;
            ++count;
        }
        if ((int64_t)a->seqs[ids[i]].blocks.size() > max_blocks) st = PA_ERR_INVALID_ARG;
    }
    if (st != PA_OK) {
        for (auto it = log.rbegin(); it != log.rend(); ++it) a->revert(*it);
        return st;
    }
    *ncow = count;
    return PA_OK;
}

}  // namespace

extern "C" {

int pa_alloc_create_ordered(int num_blocks, int block_size, const int32_t *order,
                            pa_allocator **out) {
    if (!out || num_blocks <= 0 || block_size <= 0) return PA_ERR_INVALID_ARG;
    *out = nullptr;
    // Block sizes the kernels address (8, 16, 32, 64 tokens).
    if (block_size != 8 && block_size != 16 && block_size != 32 && block_size != 64) return PA_ERR_UNSUPPORTED;
    // A slot is block * block_size + row in int32: every slot of the pool must fit.
    if ((int64_t)num_blocks * block_size > (int64_t)INT32_MAX) return PA_ERR_INVALID_ARG;
    pa_allocator *a = new (std::nothrow) pa_allocator();
    if (!a) return PA_ERR_OOM;
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->ref.assign((size_t)num_blocks, 0);
    a->free_stack.resize((size_t)num_blocks);
    if (order) {
        std::vector<char> seen((size_t)num_blocks, 0);
        for (int i = 0; i < num_blocks; ++i) {
            const int32_t b = order[i];
            if (b < 0 || b >= num_blocks || seen[b]) {
                delete a;
                return PA_ERR_INVALID_ARG;
            }
            seen[b] = 1;
            a->free_stack[(size_t)(num_blocks - 1 - i)] = b;
        }
    } else {
        for (int i = 0; i < num_blocks; ++i) a->free_stack[(size_t)(num_blocks - 1 - i)] = i;
    }
    *out = a;
    return PA_OK;
}

int pa_alloc_create(int num_blocks, int block_size, pa_allocator **out) {
    return pa_alloc_create_ordered(num_blocks, block_size, nullptr, out);
}

void pa_alloc_destroy(pa_allocator *alloc) { delete alloc; }

int pa_seq_create(pa_allocator *alloc, int *seq_id) {
    if (!alloc || !seq_id) return PA_ERR_INVALID_ARG;
    alloc->seqs.emplace_back();
    alloc->seqs.back().live = true;
    *seq_id = (int)alloc->seqs.size() - 1;
    return PA_OK;
}

int pa_seq_append(pa_allocator *alloc, int seq_id, int32_t *slot_out, int32_t *cow_src,
                  int32_t *cow_dst) {
    if (!alloc || !slot_out) return PA_ERR_INVALID_ARG;
    if (!alloc->valid_seq(seq_id)) return PA_ERR_BAD_INDEX;
    int32_t s = -1, d = -1;
    const int st = alloc->append(seq_id, slot_out, &s, &d, nullptr);
    if (st != PA_OK) return st;
    if (s >= 0 && (!cow_src || !cow_dst)) {
        // The caller cannot receive the copy it must perform: undo and refuse.
        alloc->revert(Undo{seq_id, d, s});
        return PA_ERR_INVALID_ARG;
    }
    if (cow_src) *cow_src = s;
    if (cow_dst) *cow_dst = d;
    return PA_OK;
}

int pa_seq_append_batch(pa_allocator *alloc, const int32_t *seq_ids, int n, int32_t *slots_out,
                        int32_t *cow_pairs_out, int *n_cow) {
    if (!alloc || n < 0 || (n > 0 && (!seq_ids || !slots_out || !cow_pairs_out)) || !n_cow)
        return PA_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (!alloc->valid_seq(seq_ids[i])) return PA_ERR_BAD_INDEX;
    return append_all(alloc, seq_ids, n, slots_out, cow_pairs_out, n_cow, INT64_MAX);
}

int pa_alloc_step(pa_allocator *alloc, const int32_t *seq_ids, int n, int32_t *tables, int max_blocks,
                  int32_t pad, int32_t *seq_lens, int32_t *cow_pairs_out, int *n_cow, int *max_seq_len) {
    if (!alloc || n < 0 || max_blocks < 0 || !n_cow || !max_seq_len) return PA_ERR_INVALID_ARG;
    if (n > 0 && (!seq_ids || !tables || !seq_lens || !cow_pairs_out)) return PA_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i)
        if (!alloc->valid_seq(seq_ids[i])) return PA_ERR_BAD_INDEX;
    int ncow = 0;
    const int st = append_all(alloc, seq_ids, n, nullptr, cow_pairs_out, &ncow, max_blocks);
    if (st != PA_OK) return st;
    int64_t longest = 0;
    for (int i = 0; i < n; ++i) {
        const Seq &s = alloc->seqs[seq_ids[i]];
        int32_t *row = tables + (size_t)i * (size_t)max_blocks;
        const size_t nb = s.blocks.size();
        if (nb) std::memcpy(row, s.blocks.data(), nb * sizeof(int32_t));
        for (size_t j = nb; j < (size_t)max_blocks; ++j) row[j] = pad;
        seq_lens[i] = (int32_t)s.tokens;
        if (s.tokens > longest) longest = s.tokens;
    }
    *n_cow = ncow;
    *max_seq_len = (int)longest;
    return PA_OK;
}

int pa_seq_fork(pa_allocator *alloc, int parent_id, int *child_id) {
    if (!alloc || !child_id) return PA_ERR_INVALID_ARG;
    if (!alloc->valid_seq(parent_id)) return PA_ERR_BAD_INDEX;
    Seq child;
    child.blocks = alloc->seqs[parent_id].blocks;
    child.tokens = alloc->seqs[parent_id].tokens;
    child.live = true;
    for (int32_t b : child.blocks) alloc->ref[b] += 1;
    alloc->seqs.push_back(std::move(child));
    *child_id = (int)alloc->seqs.size() - 1;
    return PA_OK;
}

int pa_seq_free(pa_allocator *alloc, int seq_id) {
    if (!alloc) return PA_ERR_INVALID_ARG;
    if (!alloc->valid_seq(seq_id)) return PA_ERR_BAD_INDEX;
    Seq &s = alloc->seqs[seq_id];
    for (int32_t b : s.blocks) {
        if (--alloc->ref[b] == 0) alloc->free_stack.push_back(b);
    }
    s.blocks.clear();
    s.blocks.shrink_to_fit();
    s.tokens = 0;
    s.live = false;
    return PA_OK;
}

int pa_seq_block_table(const pa_allocator *alloc, int seq_id, int32_t *out, int cap,
                       int *n_blocks, int *n_tokens) {
    if (!alloc || !n_blocks || !n_tokens) return PA_ERR_INVALID_ARG;
    if (!alloc->valid_seq(seq_id)) return PA_ERR_BAD_INDEX;
    const Seq &s = alloc->seqs[seq_id];
    *n_blocks = (int)s.blocks.size();
    *n_tokens = (int)s.tokens;
    if (cap < (int)s.blocks.size() || (!out && !s.blocks.empty())) return PA_ERR_INVALID_ARG;
    if (!s.blocks.empty()) std::memcpy(out, s.blocks.data(), s.blocks.size() * sizeof(int32_t));
    return PA_OK;
}

int pa_alloc_export(const pa_allocator *alloc, const int32_t *seq_ids, int n, int32_t *tables,
                    int max_blocks, int32_t pad, int32_t *seq_lens) {
    if (!alloc || n < 0 || max_blocks < 0) return PA_ERR_INVALID_ARG;
    if (n > 0 && (!seq_ids || !tables || !seq_lens)) return PA_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        if (!alloc->valid_seq(seq_ids[i])) return PA_ERR_BAD_INDEX;
        if ((int)alloc->seqs[seq_ids[i]].blocks.size() > max_blocks) return PA_ERR_INVALID_ARG;
    }
    for (int i = 0; i < n; ++i) {
        const Seq &s = alloc->seqs[seq_ids[i]];
        int32_t *row = tables + (size_t)i * (size_t)max_blocks;
        const size_t nb = s.blocks.size();
        if (nb) std::memcpy(row, s.blocks.data(), nb * sizeof(int32_t));
        for (size_t j = nb; j < (size_t)max_blocks; ++j) row[j] = pad;
        seq_lens[i] = (int32_t)s.tokens;
    }
    return PA_OK;
}

int pa_validate_tables(const int32_t *tables, int batch, int max_blocks, const int32_t *seq_lens,
                       int64_t num_blocks, int block_size, int *bad_seq, int *bad_entry) {
    if (batch < 0 || max_blocks < 0 || num_blocks <= 0 || block_size <= 0 || !bad_seq || !bad_entry)
        return PA_ERR_INVALID_ARG;
    *bad_seq = -1;
    *bad_entry = -1;
    if (batch == 0) return PA_OK;
    if (!tables || !seq_lens) return PA_ERR_INVALID_ARG;
    // seen[id] == b + 1: block id already used by row b (a repeat within a row)
    std::vector<int32_t> seen;
    try {
        seen.assign((size_t)num_blocks, 0);
    } catch (...) {
        return PA_ERR_OOM;
    }
    for (int b = 0; b < batch; ++b) {
        const int64_t L = seq_lens[b];
        if (L < 0 || L > (int64_t)max_blocks * block_size) {
            *bad_seq = b;
            return PA_ERR_BAD_INDEX;
        }
        const int64_t used = (L + block_size - 1) / block_size;
        const int32_t *row = tables + (size_t)b * (size_t)max_blocks;
        for (int64_t j = 0; j < used; ++j) {
            const int32_t id = row[j];
            if (id < 0 || id >= num_blocks || seen[(size_t)id] == b + 1) {
                *bad_seq = b;
                *bad_entry = (int)j;
                return PA_ERR_BAD_INDEX;
            }
            seen[(size_t)id] = b + 1;
        }
    }
    return PA_OK;
}

int pa_alloc_num_free(const pa_allocator *alloc) {
    return alloc ? (int)alloc->free_stack.size() : -1;
}

int pa_block_refcount(const pa_allocator *alloc, int32_t block) {
    if (!alloc || block < 0 || block >= alloc->num_blocks) return -1;
    return alloc->ref[block];
}

}  // extern "C"
