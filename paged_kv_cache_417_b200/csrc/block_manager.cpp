// block_manager.cpp - host block manager of a paged KV cache
// (include/pagedkv_block_manager.h): free list, reference counts, block
// tables, fork, append with copy-on-write, and the decode-step inputs.
#include "pagedkv_block_manager.h"

#include <algorithm>
#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "last_error.h"

using pagedkv::fail;
using pagedkv::ok;

struct pa_block_manager {
    struct Seq {
        std::vector<int32_t> table;
        int32_t tokens = 0;
    };
    int32_t num_blocks = 0, block_size = 0;
    std::vector<int32_t> free_list; // back() is handed out next
    std::vector<int32_t> ref;
    std::unordered_map<int64_t, Seq> seqs;

    int32_t take()
    {
        const int32_t b = free_list.back();
        free_list.pop_back();
        ref[b] = 1;
        return b;
    }

    void release(int32_t b)
    {
        if (--ref[b] == 0)
            free_list.push_back(b);
    }

    Seq *find(int64_t id)
    {
        auto it = seqs.find(id);
        return it == seqs.end() ? nullptr : &it->second;
    }
};

namespace {

int64_t blocks_for(int64_t tokens, int32_t bs) { return (tokens + bs - 1) / bs; }

} // namespace

extern "C" {

pa_block_manager *pa_bm_create(int32_t num_blocks, int32_t block_size, const int32_t *free_order)
{
    if (num_blocks < 0 || block_size <= 0)
        return nullptr;
    pa_block_manager *bm = new (std::nothrow) pa_block_manager();
    if (!bm)
        return nullptr;
    try {
        bm->num_blocks = num_blocks;
        bm->block_size = block_size;
        bm->ref.assign(num_blocks, 0);
        bm->free_list.resize(num_blocks);
        std::vector<char> seen(num_blocks, 0);
        for (int32_t i = 0; i < num_blocks; ++i) {
            const int32_t b = free_order ? free_order[i] : i;
            if (b < 0 || b >= num_blocks || seen[b]) {
                delete bm;
                return nullptr;
            }
            seen[b] = 1;
            bm->free_list[num_blocks - 1 - i] = b; // order[0] is handed out first
        }
    } catch (...) {
        delete bm;
        return nullptr;
    }
    return bm;
}

void pa_bm_destroy(pa_block_manager *bm) { delete bm; }

int32_t pa_bm_num_free(const pa_block_manager *bm)
{
    return bm ? (int32_t)bm->free_list.size() : 0;
}

int32_t pa_bm_can_allocate(const pa_block_manager *bm, int32_t n)
{
    return bm && n >= 0 && (size_t)n <= bm->free_list.size() ? 1 : 0;
}

int32_t pa_bm_ref_count(const pa_block_manager *bm, int32_t block)
{
    if (!bm || block < 0 || block >= bm->num_blocks)
        return -1;
    return bm->ref[block];
}

pa_status pa_bm_add_sequence(pa_block_manager *bm, int64_t seq)
{
    if (!bm)
        return fail(PA_ERR_INVALID_ARG, "NULL block manager");
    if (bm->seqs.count(seq))
        return fail(PA_ERR_INVALID_ARG, "sequence %lld exists", (long long)seq);
    bm->seqs.emplace(seq, pa_block_manager::Seq());
    return ok();
}

pa_status pa_bm_allocate_tokens(pa_block_manager *bm, int64_t seq, int32_t n)
{
    if (!bm)
        return fail(PA_ERR_INVALID_ARG, "NULL block manager");
    pa_block_manager::Seq *s = bm->find(seq);
    if (!s)
        return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq);
    if (n < 0)
        return fail(PA_ERR_INVALID_ARG, "negative token count");
    if (n == 0)
        return ok();
    const int32_t bs = bm->block_size;
    if (s->tokens % bs && bm->ref[s->table.back()] > 1)
        return fail(PA_ERR_INVALID_ARG, "sequence %lld: last block is shared", (long long)seq);
    const int64_t need = blocks_for((int64_t)s->tokens + n, bs) - blocks_for(s->tokens, bs);
    if ((size_t)need > bm->free_list.size())
        return fail(PA_ERR_INVALID_ARG, "pool exhausted: need %lld blocks, %zu free",
                    (long long)need, bm->free_list.size());
    for (int64_t i = 0; i < need; ++i)
        s->table.push_back(bm->take());
    s->tokens += n;
    return ok();
}

pa_status pa_bm_fork(pa_block_manager *bm, int64_t parent, int64_t child)
{
    if (!bm)
        return fail(PA_ERR_INVALID_ARG, "NULL block manager");
    pa_block_manager::Seq *p = bm->find(parent);
    if (!p)
        return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)parent);
    if (bm->seqs.count(child))
        return fail(PA_ERR_INVALID_ARG, "sequence %lld exists", (long long)child);
    pa_block_manager::Seq c = *p; // copy before the map may rehash
    for (int32_t b : c.table)
        ++bm->ref[b];
    bm->seqs.emplace(child, std::move(c));
    return ok();
}

pa_status pa_bm_append_token(pa_block_manager *bm, int64_t seq, int64_t *slot, int64_t *cow_src,
                             int64_t *cow_dst)
{
    if (!bm)
        return fail(PA_ERR_INVALID_ARG, "NULL block manager");
    pa_block_manager::Seq *s = bm->find(seq);
    if (!s)
        return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq);
    const int32_t bs = bm->block_size;
    const int32_t offset = s->tokens % bs;
    const bool needs_block = offset == 0 || bm->ref[s->table.back()] > 1;
    if (needs_block && bm->free_list.empty())
        return fail(PA_ERR_INVALID_ARG, "pool exhausted");
    int64_t src = -1, dst = -1;
    if (offset == 0) {
        s->table.push_back(bm->take());
    } else if (bm->ref[s->table.back()] > 1) {
        src = s->table.back();
        dst = bm->take();
        bm->release((int32_t)src);
        s->table.back() = (int32_t)dst;
    }
    if (slot)
        *slot = (int64_t)s->table.back() * bs + offset;
    if (cow_src)
        *cow_src = src;
    if (cow_dst)
        *cow_dst = dst;
    ++s->tokens;
    return ok();
}

pa_status pa_bm_free_sequence(pa_block_manager *bm, int64_t seq)
{
    if (!bm)
        return fail(PA_ERR_INVALID_ARG, "NULL block manager");
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end())
        return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seq);
    for (int32_t b : it->second.table)
        bm->release(b);
    bm->seqs.erase(it);
    return ok();
}

int32_t pa_bm_num_tokens(const pa_block_manager *bm, int64_t seq)
{
    if (!bm)
        return -1;
    auto it = bm->seqs.find(seq);
    return it == bm->seqs.end() ? -1 : it->second.tokens;
}

int32_t pa_bm_block_table(const pa_block_manager *bm, int64_t seq, int32_t *out, int32_t cap)
{
    if (!bm)
        return -1;
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end())
        return -1;
    const std::vector<int32_t> &t = it->second.table;
    for (int32_t i = 0; i < cap && (size_t)i < t.size(); ++i)
        out[i] = t[i];
    return (int32_t)t.size();
}

pa_status pa_bm_prepare_decode(pa_block_manager *bm, const int64_t *seqs, int32_t n,
                               int32_t max_blocks_per_seq, int32_t *block_tables,
                               int32_t *context_lens, int64_t *slot_mapping,
                               int64_t *copy_pairs, int32_t *num_pairs)
{
    if (!bm)
        return fail(PA_ERR_INVALID_ARG, "NULL block manager");
    if (n < 0 || max_blocks_per_seq < 1)
        return fail(PA_ERR_INVALID_ARG, "bad size argument");
    if (n > 0 && (!seqs || !block_tables || !context_lens || !slot_mapping || !copy_pairs))
        return fail(PA_ERR_INVALID_ARG, "NULL pointer argument");
    // Check the whole step first: known, distinct sequences; tables that fit;
    // enough free blocks, counting copy-on-write in batch order (a shared
    // block copied by one holder may be exclusive for the next).
    std::unordered_set<int64_t> seen;
    std::unordered_map<int32_t, int32_t> drops; // ref-count drops from earlier copies
    int64_t need = 0;
    const int32_t bs = bm->block_size;
    for (int32_t i = 0; i < n; ++i) {
        pa_block_manager::Seq *s = bm->find(seqs[i]);
        if (!s)
            return fail(PA_ERR_INVALID_ARG, "unknown sequence %lld", (long long)seqs[i]);
        if (!seen.insert(seqs[i]).second)
            return fail(PA_ERR_INVALID_ARG, "sequence %lld twice in one step",
                        (long long)seqs[i]);
        if (blocks_for((int64_t)s->tokens + 1, bs) > max_blocks_per_seq)
            return fail(PA_ERR_INVALID_ARG, "sequence %lld outgrows max_blocks_per_seq %d",
                        (long long)seqs[i], max_blocks_per_seq);
        if (s->tokens % bs == 0) {
            ++need;
        } else {
            const int32_t last = s->table.back();
            if (bm->ref[last] - drops[last] > 1) {
                ++need;
                ++drops[last];
            }
        }
    }
    if ((size_t)need > bm->free_list.size())
        return fail(PA_ERR_INVALID_ARG, "pool exhausted: the step needs %lld blocks, %zu free",
                    (long long)need, bm->free_list.size());
    int32_t pairs = 0;
    for (int32_t i = 0; i < n; ++i) {
        int64_t src, dst;
        pa_bm_append_token(bm, seqs[i], &slot_mapping[i], &src, &dst);
        if (src >= 0) {
            copy_pairs[2 * pairs] = src;
            copy_pairs[2 * pairs + 1] = dst;
            ++pairs;
        }
        const pa_block_manager::Seq *s = bm->find(seqs[i]);
        context_lens[i] = s->tokens;
        int32_t *row = block_tables + (size_t)i * max_blocks_per_seq;
        std::copy(s->table.begin(), s->table.end(), row);
        std::fill(row + s->table.size(), row + max_blocks_per_seq, -1);
    }
    if (num_pairs)
        *num_pairs = pairs;
    return ok();
}

} // extern "C"
