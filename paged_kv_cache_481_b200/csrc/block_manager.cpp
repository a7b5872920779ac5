// Host-side KV block manager (declared in include/pa_block_manager.h): the
// shared free pool, per-block reference counts, slot allocation for each
// decode step, the copy-on-write decision for shared blocks, and the
// swap-out / swap-in of whole sequence groups to a host block pool.
#include <algorithm>
#include <cstdint>
#include <mutex>
#include <new>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "../../include/pa_block_manager.h"

struct pa_block_manager {
    // A free-block stack with reference counts; one for the device pool and
    // one for the host (swap) pool.
    struct Pool {
        std::vector<int32_t> free_stack;  // back() is handed out next
        std::vector<int32_t> refcount;    // per physical block

        void init(int n)
        {
            refcount.assign(size_t(n), 0);
            free_stack.resize(size_t(n));
            for (int i = 0; i < n; ++i)  // hands out 0, 1, 2, ...
                free_stack[size_t(i)] = n - 1 - i;
        }

        int32_t take()
        {
            const int32_t b = free_stack.back();
            free_stack.pop_back();
            refcount[size_t(b)] = 1;
            return b;
        }

        void release(int32_t b)
        {
            if (--refcount[size_t(b)] == 0)
                free_stack.push_back(b);
        }
    };

    struct Sequence {
        std::vector<int32_t> blocks;  // logical block i -> physical id
        int64_t len = 0;              // tokens held
        bool swapped = false;         // blocks are ids of the host pool
    };

    int num_blocks = 0;
    int block_size = 0;
    Pool gpu, cpu;
    std::unordered_map<int64_t, Sequence> seqs;
    mutable std::mutex mu;

    int32_t take() { return gpu.take(); }
    void release(int32_t b) { gpu.release(b); }
    Pool &pool_of(const Sequence &s) { return s.swapped ? cpu : gpu; }

    // Move a group of sequences from pool `from` to pool `to` (swap-out when
    // from is the device pool, swap-in otherwise).  Every block the group
    // holds must be held by group members only, so that the whole group
    // leaves together (all-or-nothing preemption).  Each distinct block gets
    // one block of `to`, in order of first appearance (sequences in the
    // given order, each table front to back), with its reference count; the
    // (from, to) pairs are written to `pairs` ([max_pairs, 2]).
    pa_status move_group(const int64_t *ids, int n, bool to_cpu, int64_t *pairs, int max_pairs,
                         int *num_pairs)
    {
        Pool &from = to_cpu ? gpu : cpu;
        Pool &to = to_cpu ? cpu : gpu;
        std::unordered_set<int64_t> seen;
        std::unordered_map<int32_t, int> holders;  // block -> holders within the group
        std::vector<int32_t> order;                // distinct blocks, first appearance
        for (int i = 0; i < n; ++i) {
            auto it = seqs.find(ids[i]);
            if (it == seqs.end() || !seen.insert(ids[i]).second || it->second.swapped == to_cpu)
                return PA_ERR_INVALID_ARG;
            for (int32_t b : it->second.blocks)
                if (holders[b]++ == 0)
                    order.push_back(b);
        }
        for (const auto &h : holders)
            if (from.refcount[size_t(h.first)] != h.second)
                return PA_ERR_INVALID_ARG;  // shared with a sequence outside the group
        *num_pairs = int(order.size());
        if (int64_t(order.size()) > int64_t(max_pairs))
            return PA_ERR_INVALID_ARG;
        if (order.size() > to.free_stack.size())
            return PA_ERR_OUT_OF_BLOCKS;
        std::unordered_map<int32_t, int32_t> moved;
        for (size_t k = 0; k < order.size(); ++k) {
            const int32_t b = order[k];
            const int32_t nb = to.take();
            to.refcount[size_t(nb)] = from.refcount[size_t(b)];
            moved[b] = nb;
            pairs[2 * k] = b;
            pairs[2 * k + 1] = nb;
        }
        for (int32_t b : order) {
            from.refcount[size_t(b)] = 0;
            from.free_stack.push_back(b);
        }
        for (int i = 0; i < n; ++i) {
            Sequence &s = seqs[ids[i]];
            for (int32_t &b : s.blocks)
                b = moved[b];
            s.swapped = to_cpu;
        }
        return PA_OK;
    }
};

namespace {

int64_t blocks_for(int64_t tokens, int block_size)
{
    return (tokens + block_size - 1) / block_size;
}

} // namespace

extern "C" {

pa_block_manager *pa_bm_create_with_swap(int num_blocks, int num_cpu_blocks, int block_size)
{
    if (num_blocks <= 0 || num_cpu_blocks < 0 || block_size <= 0)
        return nullptr;
    pa_block_manager *bm = new (std::nothrow) pa_block_manager;
    if (!bm)
        return nullptr;
    try {
        bm->num_blocks = num_blocks;
        bm->block_size = block_size;
        bm->gpu.init(num_blocks);
        bm->cpu.init(num_cpu_blocks);
    } catch (...) {
        delete bm;
        return nullptr;
    }
    return bm;
}

pa_block_manager *pa_bm_create(int num_blocks, int block_size)
{
    return pa_bm_create_with_swap(num_blocks, 0, block_size);
}

void pa_bm_destroy(pa_block_manager *bm)
{
    delete bm;
}

int pa_bm_num_free(const pa_block_manager *bm)
{
    if (!bm)
        return -1;
    std::lock_guard<std::mutex> g(bm->mu);
    return int(bm->gpu.free_stack.size());
}

int pa_bm_num_free_cpu(const pa_block_manager *bm)
{
    if (!bm)
        return -1;
    std::lock_guard<std::mutex> g(bm->mu);
    return int(bm->cpu.free_stack.size());
}

int pa_bm_refcount(const pa_block_manager *bm, int block)
{
    if (!bm || block < 0 || block >= bm->num_blocks)
        return -1;
    std::lock_guard<std::mutex> g(bm->mu);
    return bm->gpu.refcount[size_t(block)];
}

int pa_bm_cpu_refcount(const pa_block_manager *bm, int block)
{
    if (!bm || block < 0)
        return -1;
    std::lock_guard<std::mutex> g(bm->mu);
    if (size_t(block) >= bm->cpu.refcount.size())
        return -1;
    return bm->cpu.refcount[size_t(block)];
}

int pa_bm_is_swapped(const pa_block_manager *bm, int64_t seq)
{
    if (!bm)
        return -1;
    std::lock_guard<std::mutex> g(bm->mu);
    auto it = bm->seqs.find(seq);
    return it == bm->seqs.end() ? -1 : int(it->second.swapped);
}

pa_status pa_bm_swap_out(pa_block_manager *bm, const int64_t *seqs, int n, int64_t *pairs,
                         int max_pairs, int *num_pairs)
{
    if (!bm || n <= 0 || !seqs || !num_pairs || max_pairs < 0 || (max_pairs > 0 && !pairs))
        return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(bm->mu);
    return bm->move_group(seqs, n, true, pairs, max_pairs, num_pairs);
}

pa_status pa_bm_swap_in(pa_block_manager *bm, const int64_t *seqs, int n, int64_t *pairs,
                        int max_pairs, int *num_pairs)
{
    if (!bm || n <= 0 || !seqs || !num_pairs || max_pairs < 0 || (max_pairs > 0 && !pairs))
        return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(bm->mu);
    return bm->move_group(seqs, n, false, pairs, max_pairs, num_pairs);
}

pa_status pa_bm_add_sequence(pa_block_manager *bm, int64_t seq, int prompt_len)
{
    if (!bm || prompt_len < 0)
        return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(bm->mu);
    if (bm->seqs.count(seq))
        return PA_ERR_INVALID_ARG;
    const int64_t need = blocks_for(prompt_len, bm->block_size);
    if (need > int64_t(bm->gpu.free_stack.size()))
        return PA_ERR_OUT_OF_BLOCKS;
    pa_block_manager::Sequence s;
    s.len = prompt_len;
    s.blocks.reserve(size_t(need));
    for (int64_t i = 0; i < need; ++i)
        s.blocks.push_back(bm->take());
    bm->seqs.emplace(seq, std::move(s));
    return PA_OK;
}

pa_status pa_bm_fork(pa_block_manager *bm, int64_t parent, int64_t child)
{
    if (!bm)
        return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(bm->mu);
    auto it = bm->seqs.find(parent);
    if (it == bm->seqs.end() || it->second.swapped || bm->seqs.count(child))
        return PA_ERR_INVALID_ARG;
    pa_block_manager::Sequence s = it->second;  // same table, same length
    for (int32_t b : s.blocks)
        ++bm->gpu.refcount[size_t(b)];
    bm->seqs.emplace(child, std::move(s));
    return PA_OK;
}

pa_status pa_bm_free_sequence(pa_block_manager *bm, int64_t seq)
{
    if (!bm)
        return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(bm->mu);
    auto it = bm->seqs.find(seq);
    if (it == bm->seqs.end())
        return PA_ERR_INVALID_ARG;
    pa_block_manager::Pool &pool = bm->pool_of(it->second);
    for (int32_t b : it->second.blocks)
        pool.release(b);
    bm->seqs.erase(it);
    return PA_OK;
}

pa_status pa_bm_append_slots(pa_block_manager *bm, const int64_t *seqs, int n, int64_t *slots,
                             int64_t *cow_pairs, int *num_pairs)
{
    if (!bm || n < 0 || (n > 0 && (!seqs || !slots || !cow_pairs)) || !num_pairs)
        return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(bm->mu);
    const int bs = bm->block_size;
    // Validate and count the blocks the whole step needs before changing anything.
    // A shared last block is copied once per writer that is not its last owner
    // in this step, so count copies with the reference counts as they will be.
    std::unordered_set<int64_t> seen;
    std::unordered_map<int32_t, int> pending_refs;
    int64_t need = 0;
    for (int i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seqs[i]);
        if (it == bm->seqs.end() || it->second.swapped || !seen.insert(seqs[i]).second)
            return PA_ERR_INVALID_ARG;
        const pa_block_manager::Sequence &s = it->second;
        if (s.len % bs == 0) {
            ++need;  // last block full (or none): a fresh block
        } else {
            const int32_t last = s.blocks.back();
            auto pr = pending_refs.find(last);
            int refs = pr == pending_refs.end() ? bm->gpu.refcount[size_t(last)] : pr->second;
            if (refs > 1) {
                ++need;  // shared: this writer gets a copy
                pending_refs[last] = refs - 1;
            }
        }
    }
    if (need > int64_t(bm->gpu.free_stack.size()))
        return PA_ERR_OUT_OF_BLOCKS;

    int pairs = 0;
    for (int i = 0; i < n; ++i) {
        pa_block_manager::Sequence &s = bm->seqs[seqs[i]];
        const int64_t pos = s.len;
        if (pos % bs == 0) {
            s.blocks.push_back(bm->take());
        } else {
            const int32_t last = s.blocks.back();
            if (bm->gpu.refcount[size_t(last)] > 1) {  // copy-on-write of the shared last block
                const int32_t fresh = bm->take();
                --bm->gpu.refcount[size_t(last)];
                s.blocks.back() = fresh;
                cow_pairs[2 * pairs] = last;
                cow_pairs[2 * pairs + 1] = fresh;
                ++pairs;
            }
        }
        slots[i] = int64_t(s.blocks[size_t(pos / bs)]) * bs + pos % bs;
        s.len = pos + 1;
    }
    *num_pairs = pairs;
    return PA_OK;
}

pa_status pa_bm_block_tables(const pa_block_manager *bm, const int64_t *seqs, int n,
                             int32_t *block_tables, int max_blocks, int32_t *context_lens)
{
    if (!bm || n < 0 || max_blocks < 0 || (n > 0 && (!seqs || !block_tables || !context_lens)))
        return PA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(bm->mu);
    for (int i = 0; i < n; ++i) {
        auto it = bm->seqs.find(seqs[i]);
        if (it == bm->seqs.end() || it->second.swapped ||
            int64_t(it->second.blocks.size()) > max_blocks ||
            it->second.len > INT32_MAX)
            return PA_ERR_INVALID_ARG;
    }
    for (int i = 0; i < n; ++i) {
        const pa_block_manager::Sequence &s = bm->seqs.find(seqs[i])->second;
        int32_t *row = block_tables + size_t(i) * size_t(max_blocks);
        std::fill(row, row + max_blocks, -1);
        std::copy(s.blocks.begin(), s.blocks.end(), row);
        context_lens[i] = int32_t(s.len);
    }
    return PA_OK;
}

} // extern "C"
