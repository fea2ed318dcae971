// Host block allocator for the paged KV pool (C ABI in include/pagedkv.h).
//
// Free pool, per-block reference counts, per-sequence block tables, shared
// prefixes, forks and the copy-on-write trigger:
//   openeuler.csdn.net PagedAttention explainer 4.1-4.3 (fixed blocks, block
//   table, growth only when the last block is full), 6.1 (shared prefix),
//   6.2 (copy only the block being written);
//   agent.csdn.net PagedAttention blog 2.2 (forked samples/beams share blocks),
//   3.1 (allocate a free block on demand);
//   aiknowledge.cn "2.2 PagedAttention 与 KV Cache 分页管理" 2.2.2 (free on
//   finish/preemption), 2.2.3 (worked example), 2.2.13 (monitoring counters).
//
// Every call checks all preconditions and counts the blocks it needs before it
// changes anything, so a failing call leaves the state untouched.
#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <deque>
#include <iterator>
#include <list>
#include <string>
#include <unordered_map>
#include <vector>

#include "../../include/pagedkv.h"

namespace pkv_host {
void set_error(const std::string& msg);
}

// Automatic prefix caching (openeuler.csdn.net explainer 7.4: a prompt
// prefix computed once is reused and its prefill skipped; aiknowledge.cn
// 2.2.3 shared blocks, 2.2.8 only byte-identical prefixes share, 2.2.13 hit
// rate).  Only full blocks are cached.  A block's key is (node id of the
// cached block before it on its sequence -- kRoot for the first block --,
// its block_size token ids), so equal keys mean identical whole prefixes.
// Each registration gets a fresh node id.  Cached blocks whose count drops
// to zero stay cached at the back of an LRU list; fresh blocks come from the
// free queue first, then by evicting the LRU front (its key is dropped).
constexpr int64_t kRoot = -1;
constexpr int64_t kBroken = -2;  // chain unknown: this sequence registers nothing

struct CacheKey {
    int64_t parent;
    std::vector<int32_t> toks;
    bool operator==(const CacheKey& o) const { return parent == o.parent && toks == o.toks; }
};
struct CacheKeyHash {
    size_t operator()(const CacheKey& k) const {
        uint64_t h = 1469598103934665603ull ^ (uint64_t)k.parent;
        for (int32_t t : k.toks) h = (h ^ (uint32_t)t) * 1099511628211ull;
        return (size_t)h;
    }
};

struct pkv_alloc {
    struct Seq {
        std::vector<int32_t> table;  // logical block -> physical block
        int64_t len = 0;             // tokens cached
        int64_t chain = kRoot;       // node of its last cached block (prefix caching)
        std::vector<int32_t> tail;   // token ids of its partly filled last block
    };
    int num_blocks = 0;
    int block_size = 0;
    std::deque<int32_t> free_q;
    std::vector<int32_t> ref;
    std::unordered_map<int64_t, Seq> seqs;
    int64_t alloc_failures = 0;
    int64_t cow_copies = 0;

    bool caching = false;
    std::unordered_map<CacheKey, int32_t, CacheKeyHash> cache;
    std::vector<CacheKey> key_of;  // per block, valid while node_of >= 0
    std::vector<int64_t> node_of;  // per block, -1 if not cached
    std::list<int32_t> lru;        // cached blocks with count 0, oldest first
    std::vector<std::list<int32_t>::iterator> lru_it;
    std::vector<char> in_lru;
    int64_t next_node = 0, lookups = 0, hits = 0, evictions = 0;

    int64_t available() const { return (int64_t)free_q.size() + (int64_t)lru.size(); }

    // A write into block b goes to a private copy when another sequence holds
    // b, or when b is cached: a cached block's tokens are never overwritten
    // (a sequence can hold a cached block with fewer of its tokens when it
    // was given a prefix that ends part-way into it).
    bool must_copy(int32_t b) const { return ref[b] > 1 || node_of[b] >= 0; }

    // A fresh block: the free queue's front, else the least recently released
    // cached block (its key is dropped).  Callers check available() first.
    int32_t take() {
        if (!free_q.empty()) {
            int32_t b = free_q.front();
            free_q.pop_front();
            return b;
        }
        int32_t b = lru.front();
        lru.pop_front();
        in_lru[b] = 0;
        cache.erase(key_of[b]);
        key_of[b].toks.clear();
        node_of[b] = -1;
        evictions += 1;
        return b;
    }

    void release(int32_t b) {
        if (--ref[b] != 0) return;
        if (caching && node_of[b] >= 0) {
            lru.push_back(b);
            lru_it[b] = std::prev(lru.end());
            in_lru[b] = 1;
        } else {
            free_q.push_back(b);
        }
    }

    void revive(int32_t b) {  // a cached block with count 0 found by a lookup
        if (in_lru[b]) {
            lru.erase(lru_it[b]);
            in_lru[b] = 0;
        }
        ref[b] += 1;
    }

    void register_block(Seq& s, int32_t b) {
        if (s.chain == kBroken) return;
        CacheKey k{s.chain, s.tail};
        if (cache.count(k)) {  // this prefix was computed elsewhere: stop this chain
            s.chain = kBroken;
            return;
        }
        const int64_t node = next_node++;
        cache.emplace(k, b);
        key_of[b] = std::move(k);
        node_of[b] = node;
        s.chain = node;
    }
};

using pkv_host::set_error;

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

extern "C" {

pkv_alloc* pkv_alloc_create(int num_blocks, int block_size, const int32_t* free_order) {
    if (num_blocks <= 0 || block_size <= 0) {
        set_error("pkv_alloc_create: num_blocks and block_size must be positive");
        return nullptr;
    }
    pkv_alloc* a = new (std::nothrow) pkv_alloc();
    if (!a) return nullptr;
    a->num_blocks = num_blocks;
    a->block_size = block_size;
    a->ref.assign(num_blocks, 0);
    a->key_of.resize(num_blocks);
    a->node_of.assign(num_blocks, -1);
    a->lru_it.resize(num_blocks);
    a->in_lru.assign(num_blocks, 0);
    if (free_order) {
        std::vector<char> seen(num_blocks, 0);
        for (int i = 0; i < num_blocks; ++i) {
            int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || seen[b]) {
                set_error("pkv_alloc_create: free_order is not a permutation of the pool");
                delete a;
                return nullptr;
            }
            seen[b] = 1;
            a->free_q.push_back(b);
        }
    } else {
        for (int i = 0; i < num_blocks; ++i) a->free_q.push_back(i);
    }
    return a;
}

void pkv_alloc_destroy(pkv_alloc* a) { delete a; }

pkv_status pkv_seq_add(pkv_alloc* a, int64_t seq_id) {
    if (!a) return PKV_ERR_INVALID;
    if (a->seqs.count(seq_id)) {
        set_error("pkv_seq_add: sequence already registered");
        return PKV_ERR_INVALID;
    }
    a->seqs.emplace(seq_id, pkv_alloc::Seq());
    return PKV_OK;
}

pkv_status pkv_seq_share_prefix(pkv_alloc* a, int64_t seq_id, const int32_t* blocks, int nblocks,
                                int num_tokens) {
    if (!a) return PKV_ERR_INVALID;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end() || it->second.len != 0 || !it->second.table.empty()) {
        set_error("pkv_seq_share_prefix: sequence must be registered and empty");
        return PKV_ERR_INVALID;
    }
    if (num_tokens < 0 || nblocks != ceil_div(num_tokens, a->block_size) || (nblocks > 0 && !blocks)) {
        set_error("pkv_seq_share_prefix: nblocks must equal ceil(num_tokens / block_size)");
        return PKV_ERR_INVALID;
    }
    std::vector<int32_t> sorted(blocks, blocks + nblocks);
    std::sort(sorted.begin(), sorted.end());
    for (int i = 0; i < nblocks; ++i) {
        int32_t b = sorted[i];
        if (b < 0 || b >= a->num_blocks || a->ref[b] == 0 || (i > 0 && sorted[i - 1] == b)) {
            set_error("pkv_seq_share_prefix: blocks must be distinct and in use");
            return PKV_ERR_INVALID;
        }
    }
    for (int i = 0; i < nblocks; ++i) a->ref[blocks[i]] += 1;
    it->second.table.assign(blocks, blocks + nblocks);
    it->second.len = num_tokens;
    it->second.chain = kBroken;  // token ids unknown
    it->second.tail.clear();
    return PKV_OK;
}

pkv_status pkv_seq_fork(pkv_alloc* a, int64_t parent, int64_t child) {
    if (!a) return PKV_ERR_INVALID;
    auto p = a->seqs.find(parent);
    if (p == a->seqs.end() || a->seqs.count(child)) {
        set_error("pkv_seq_fork: parent must exist and child must not");
        return PKV_ERR_INVALID;
    }
    pkv_alloc::Seq c = p->second;
    for (int32_t b : c.table) a->ref[b] += 1;
    a->seqs.emplace(child, std::move(c));
    return PKV_OK;
}

}  // extern "C"

// Reserve slots for ntok tokens of s (tokens: their ids, or nullptr if
// unknown -- then the sequence registers no more blocks).
static pkv_status append_impl(pkv_alloc* a, pkv_alloc::Seq& s, int ntok, const int32_t* tokens, int64_t* slots_out,
                              int32_t* cow_out, int cow_cap, int* n_cow) {
    const int64_t bs = a->block_size;
    const int64_t L = s.len;
    // Only the first new token can land in an existing block (the partly
    // filled last one); it needs a private copy if that block is shared.
    bool cow = ntok > 0 && (L % bs) != 0 && a->must_copy(s.table[L / bs]);
    int64_t fresh = ceil_div(L + ntok, bs) - (int64_t)s.table.size();
    if (cow && (cow_cap < 1 || !cow_out)) {
        set_error("pkv_seq_append_slots: a copy-on-write pair is due but cow_cap < 1");
        return PKV_ERR_INVALID;
    }
    // The copy is taken first; when this sequence was the last holder of the
    // (cached) original, the original becomes evictable for the fresh blocks.
    int64_t avail = a->available();
    bool short_of_blocks = false;
    if (cow) {
        if (avail == 0) short_of_blocks = true;
        else avail += (a->ref[s.table[L / bs]] == 1) ? 0 : -1;
    }
    if (short_of_blocks || fresh > avail) {
        a->alloc_failures += 1;
        set_error("pkv_seq_append_slots: free pool exhausted");
        return PKV_ERR_NO_FREE_BLOCK;
    }
    int ncow = 0;
    for (int64_t t = L; t < L + ntok; ++t) {
        int64_t j = t / bs;
        if (j == (int64_t)s.table.size()) {
            int32_t b = a->take();
            a->ref[b] = 1;
            s.table.push_back(b);
        } else if (a->must_copy(s.table[j])) {
            int32_t src = s.table[j];
            int32_t dst = a->take();
            cow_out[2 * ncow] = src;
            cow_out[2 * ncow + 1] = dst;
            ++ncow;
            a->release(src);
            a->ref[dst] = 1;
            s.table[j] = dst;
            a->cow_copies += 1;
        }
        slots_out[t - L] = (int64_t)s.table[j] * bs + t % bs;
        if (a->caching) {
            if (!tokens) {
                s.chain = kBroken;
                s.tail.clear();
            } else if (s.chain != kBroken) {
                s.tail.push_back(tokens[t - L]);
                if (t % bs == bs - 1) {  // block j just filled
                    a->register_block(s, s.table[j]);
                    s.tail.clear();
                }
            }
        }
    }
    s.len = L + ntok;
    if (n_cow) *n_cow = ncow;
    return PKV_OK;
}

extern "C" {

pkv_status pkv_seq_append_slots(pkv_alloc* a, int64_t seq_id, int ntok, int64_t* slots_out,
                                int32_t* cow_out, int cow_cap, int* n_cow) {
    if (!a) return PKV_ERR_INVALID;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end() || ntok < 0 || (ntok > 0 && !slots_out)) {
        set_error("pkv_seq_append_slots: unknown sequence or bad arguments");
        return PKV_ERR_INVALID;
    }
    return append_impl(a, it->second, ntok, nullptr, slots_out, cow_out, cow_cap, n_cow);
}

pkv_status pkv_seq_append_tokens(pkv_alloc* a, int64_t seq_id, const int32_t* tokens, int ntok,
                                 int64_t* slots_out, int32_t* cow_out, int cow_cap, int* n_cow) {
    if (!a) return PKV_ERR_INVALID;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end() || ntok < 0 || (ntok > 0 && (!slots_out || !tokens))) {
        set_error("pkv_seq_append_tokens: unknown sequence or bad arguments");
        return PKV_ERR_INVALID;
    }
    return append_impl(a, it->second, ntok, tokens, slots_out, cow_out, cow_cap, n_cow);
}

pkv_status pkv_seq_add_with_prompt(pkv_alloc* a, int64_t seq_id, const int32_t* tokens, int ntok,
                                   int64_t* slots_out, int* n_cached) {
    if (n_cached) *n_cached = 0;
    if (!a || ntok < 0 || (ntok > 0 && (!tokens || !slots_out)) || a->seqs.count(seq_id)) {
        set_error("pkv_seq_add_with_prompt: sequence exists or bad arguments");
        return PKV_ERR_INVALID;
    }
    const int bs = a->block_size;
    const int nfull = ntok / bs;
    std::vector<int32_t> hit;
    int64_t node = kRoot;
    if (a->caching) {
        CacheKey k{kRoot, {}};
        for (int j = 0; j < nfull; ++j) {
            k.parent = node;
            k.toks.assign(tokens + (int64_t)j * bs, tokens + (int64_t)(j + 1) * bs);
            auto f = a->cache.find(k);
            if (f == a->cache.end()) break;
            hit.push_back(f->second);
            node = a->node_of[f->second];
        }
    }
    int64_t revived = 0;
    for (int32_t b : hit) revived += a->ref[b] == 0 ? 1 : 0;
    const int64_t cached = (int64_t)hit.size() * bs;
    if (ceil_div(ntok - cached, bs) > a->available() - revived) {
        a->alloc_failures += 1;
        set_error("pkv_seq_add_with_prompt: free pool exhausted");
        return PKV_ERR_NO_FREE_BLOCK;
    }
    for (int32_t b : hit) a->revive(b);
    pkv_alloc::Seq s;
    s.table = hit;
    s.len = cached;
    s.chain = node;
    auto ins = a->seqs.emplace(seq_id, std::move(s));
    int dummy = 0;
    append_impl(a, ins.first->second, (int)(ntok - cached), tokens + cached, slots_out, nullptr, 0, &dummy);
    if (a->caching) {
        a->lookups += nfull;
        a->hits += (int64_t)hit.size();
    }
    if (n_cached) *n_cached = (int)cached;
    return PKV_OK;
}

pkv_status pkv_alloc_set_prefix_caching(pkv_alloc* a, int enable) {
    if (!a || !a->seqs.empty()) {
        set_error("pkv_alloc_set_prefix_caching: only before any sequence is registered");
        return PKV_ERR_INVALID;
    }
    a->caching = enable != 0;
    return PKV_OK;
}

pkv_status pkv_prefix_cache_stats(const pkv_alloc* a, int64_t* lookups, int64_t* hits, int* cached_blocks,
                                  int* evictable_blocks, int64_t* evictions) {
    if (!a) return PKV_ERR_INVALID;
    if (lookups) *lookups = a->lookups;
    if (hits) *hits = a->hits;
    if (cached_blocks) *cached_blocks = (int)a->cache.size();
    if (evictable_blocks) *evictable_blocks = (int)a->lru.size();
    if (evictions) *evictions = a->evictions;
    return PKV_OK;
}

pkv_status pkv_seq_append_slots_batch(pkv_alloc* a, const int64_t* seq_ids, int n, int64_t* slots_out,
                                      int32_t* cow_out, int cow_cap, int* n_cow) {
    if (n_cow) *n_cow = 0;
    if (!a || n < 0 || (n > 0 && (!seq_ids || !slots_out))) {
        set_error("pkv_seq_append_slots_batch: bad arguments");
        return PKV_ERR_INVALID;
    }
    // Dry run, in call order: every block the batch takes must be available
    // when it is taken.  A sequence listed twice sees its own first
    // reservation (its length grows); a copy made by the last holder of a
    // cached block leaves that block evictable, so later takes may use it.
    std::unordered_map<int64_t, int64_t> extra;      // tokens already reserved in this call
    std::unordered_map<int32_t, int32_t> ref_drop;   // references given up by copies made in this call
    int64_t avail = a->available(), ncow = 0;
    bool short_of_blocks = false;
    for (int i = 0; i < n; ++i) {
        auto it = a->seqs.find(seq_ids[i]);
        if (it == a->seqs.end()) {
            set_error("pkv_seq_append_slots_batch: unknown sequence");
            return PKV_ERR_INVALID;
        }
        const pkv_alloc::Seq& s = it->second;
        const int64_t bs = a->block_size;
        int64_t& k = extra[seq_ids[i]];
        const int64_t L = s.len + k;
        if (L % bs == 0) {  // a fresh block
            if (avail == 0) short_of_blocks = true;
            else avail -= 1;
        } else if (k == 0) {
            const int32_t b = s.table[L / bs];
            int32_t& drop = ref_drop[b];
            const int32_t holders = a->ref[b] - drop;
            if (holders > 1 || a->node_of[b] >= 0) {  // still shared, or cached, when this sequence writes
                if (avail == 0) short_of_blocks = true;
                else avail -= 1;
                ncow += 1;
                drop += 1;
                if (holders == 1) avail += 1;  // the cached original is released, evictable from now on
            }
        }
        k += 1;
    }
    if (ncow > 0 && (!cow_out || cow_cap < ncow)) {
        set_error("pkv_seq_append_slots_batch: cow_cap too small");
        return PKV_ERR_INVALID;
    }
    if (short_of_blocks) {
        a->alloc_failures += 1;
        set_error("pkv_seq_append_slots_batch: free pool exhausted");
        return PKV_ERR_NO_FREE_BLOCK;
    }
    int done = 0;
    for (int i = 0; i < n; ++i) {
        int c = 0;
        pkv_status st = pkv_seq_append_slots(a, seq_ids[i], 1, slots_out + i, cow_out ? cow_out + 2 * done : nullptr,
                                             cow_cap - done, &c);
        if (st != PKV_OK) return st;  // unreachable: the dry run checked every condition
        done += c;
    }
    if (n_cow) *n_cow = done;
    return PKV_OK;
}

pkv_status pkv_seq_block_tables_batch(const pkv_alloc* a, const int64_t* seq_ids, int n, int32_t* out,
                                      int max_blocks, int32_t* lens_out) {
    if (!a || n < 0 || max_blocks < 0 || (n > 0 && (!seq_ids || !out || !lens_out))) {
        set_error("pkv_seq_block_tables_batch: bad arguments");
        return PKV_ERR_INVALID;
    }
    std::vector<const pkv_alloc::Seq*> rows(n);
    for (int i = 0; i < n; ++i) {
        auto it = a->seqs.find(seq_ids[i]);
        if (it == a->seqs.end() || (int64_t)it->second.table.size() > max_blocks || it->second.len > INT32_MAX) {
            set_error("pkv_seq_block_tables_batch: unknown sequence or table longer than max_blocks");
            return PKV_ERR_INVALID;
        }
        rows[i] = &it->second;
    }
    for (int i = 0; i < n; ++i) {
        int32_t* row = out + (int64_t)i * max_blocks;
        const auto& t = rows[i]->table;
        std::copy(t.begin(), t.end(), row);
        std::fill(row + t.size(), row + max_blocks, -1);
        lens_out[i] = (int32_t)rows[i]->len;
    }
    return PKV_OK;
}

pkv_status pkv_seq_lens_batch(const pkv_alloc* a, const int64_t* seq_ids, int n, int64_t* lens_out) {
    if (!a || n < 0 || (n > 0 && (!seq_ids || !lens_out))) {
        set_error("pkv_seq_lens_batch: bad arguments");
        return PKV_ERR_INVALID;
    }
    for (int i = 0; i < n; ++i) {
        if (a->seqs.find(seq_ids[i]) == a->seqs.end()) {
            set_error("pkv_seq_lens_batch: unknown sequence");
            return PKV_ERR_INVALID;
        }
    }
    for (int i = 0; i < n; ++i) lens_out[i] = a->seqs.find(seq_ids[i])->second.len;
    return PKV_OK;
}

pkv_status pkv_seq_free(pkv_alloc* a, int64_t seq_id) {
    if (!a) return PKV_ERR_INVALID;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) {
        set_error("pkv_seq_free: unknown sequence");
        return PKV_ERR_INVALID;
    }
    for (int32_t b : it->second.table) a->release(b);
    a->seqs.erase(it);
    return PKV_OK;
}

pkv_status pkv_seq_block_table(const pkv_alloc* a, int64_t seq_id, int32_t* out, int cap, int* n,
                               int64_t* len_tokens) {
    if (!a) return PKV_ERR_INVALID;
    auto it = a->seqs.find(seq_id);
    if (it == a->seqs.end()) {
        set_error("pkv_seq_block_table: unknown sequence");
        return PKV_ERR_INVALID;
    }
    int nb = (int)it->second.table.size();
    if (n) *n = nb;
    if (len_tokens) *len_tokens = it->second.len;
    if (cap < nb || (nb > 0 && !out)) {
        set_error("pkv_seq_block_table: output capacity too small");
        return PKV_ERR_INVALID;
    }
    if (nb > 0) std::memcpy(out, it->second.table.data(), sizeof(int32_t) * nb);
    return PKV_OK;
}

pkv_status pkv_alloc_stats(const pkv_alloc* a, int* free_blocks, int* used_blocks,
                           int64_t* alloc_failures, int64_t* cow_copies) {
    if (!a) return PKV_ERR_INVALID;
    int nfree = (int)a->available();  // evictable cached blocks are free to reuse
    if (free_blocks) *free_blocks = nfree;
    if (used_blocks) *used_blocks = a->num_blocks - nfree;
    if (alloc_failures) *alloc_failures = a->alloc_failures;
    if (cow_copies) *cow_copies = a->cow_copies;
    return PKV_OK;
}

int pkv_block_refcount(const pkv_alloc* a, int block) {
    if (!a || block < 0 || block >= a->num_blocks) return -1;
    return a->ref[block];
}

pkv_status pkv_find_shared_prefix_groups(const int32_t* block_tables, const int32_t* context_lens, int n,
                                         int max_blocks, int block_size, int min_group_size,
                                         int32_t* group_first, int32_t* group_shared, int max_groups,
                                         int* n_groups) {
    if (n_groups) *n_groups = 0;
    if (n < 0 || max_blocks < 0 || block_size <= 0 || !n_groups || max_groups < n ||
        (n > 0 && (!block_tables || !context_lens || !group_first || !group_shared))) {
        set_error("pkv_find_shared_prefix_groups: bad arguments (max_groups must be >= n)");
        return PKV_ERR_INVALID;
    }
    if (min_group_size < 2) min_group_size = 2;
    // The output partitions [0, n) into runs: groups (shared > 0) and the gaps
    // between them (shared = 0); there are at most n runs.
    int ng = 0;
    auto full_blocks = [&](int i) {
        const int L = context_lens[i] < 0 ? 0 : context_lens[i];
        return std::min(L / block_size, max_blocks);
    };
    int gap_begin = -1;
    int i = 0;
    while (i < n) {
        int k = full_blocks(i);
        int j = i + 1;
        const int32_t* lead = block_tables + (int64_t)i * max_blocks;
        while (j < n && k >= 1) {
            const int32_t* row = block_tables + (int64_t)j * max_blocks;
            const int lim = std::min(k, full_blocks(j));
            int c = 0;
            while (c < lim && row[c] == lead[c]) ++c;
            if (c < 1) break;
            k = c;
            ++j;
        }
        if (j - i >= min_group_size && k >= 1) {
            if (gap_begin >= 0) {
                group_first[ng] = gap_begin;
                group_shared[ng++] = 0;
                gap_begin = -1;
            }
            group_first[ng] = i;
            group_shared[ng++] = k * block_size;
            i = j;
        } else {
            if (gap_begin < 0) gap_begin = i;
            ++i;
        }
    }
    if (gap_begin >= 0) {
        group_first[ng] = gap_begin;
        group_shared[ng++] = 0;
    }
    if (ng > 0) group_first[ng] = n;  // group_first holds max_groups + 1 entries
    *n_groups = ng;
    return PKV_OK;
}

}  // extern "C"
