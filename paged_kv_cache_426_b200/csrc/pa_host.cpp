// Host block allocator and block-table manager behind the C ABI (pa.h).
//
// "Paged Attention" (velog @junegood), 구현 세부사항: a BlockAllocator hands out
// a free physical block (allocate_block) and takes freed ones back into the
// reuse pool (free_block).  Same page, 작동 예시 / 동적 할당: a request gets a
// new block only when its last block is full.  Same page, 메모리 공유: beams
// share the prompt's blocks and continue on blocks of their own; a shared
// block that is written is copied first ("KV Cache & PagedAttention"
// studynote, II).  "09. PagedAttention" (119-ai-studio), 해법: the per-request
// block table maps logical to physical blocks; only the last block may be
// partly filled.
//
// Prefix caching ("vLLM PagedAttention" studynote, prefix caching; "09.
// PagedAttention" (119-ai-studio), 다음 장): the full blocks of a prompt are
// registered under a key that identifies the whole token prefix up to the
// block's end; a later prompt that starts with the same tokens maps the same
// physical blocks instead of storing them again.  The cache holds one
// reference per cached block, so a cached block outlives the sequences that
// used it, and is evicted (least recently used first, and only while nothing
// else references it) when the free pool runs dry.
//
// Pure host code: nothing here touches device memory.
#include <algorithm>
#include <cstdint>
#include <deque>
#include <iterator>
#include <list>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa.h"

struct pa_allocator {
    std::deque<int32_t> free_ids;      // FIFO pool: pop front, push back
    std::vector<int32_t> refcount;     // per physical block
};

struct pa_manager {
    struct Seq {
        std::vector<int32_t> table;    // logical block -> physical block
        int32_t len = 0;               // tokens held
        uint64_t stamp = 0;            // last append_step call that named it
    };
    // One cached block: the key of its whole prefix, the key of the prefix
    // before it (0 for a first block) and its own tokens (checked on a hit).
    struct Cached {
        uint64_t key, parent;
        std::vector<int32_t> tokens;
        std::list<int32_t>::iterator lru;   // position in `lru`
    };
    pa_allocator* alloc = nullptr;
    int block_size = 0;
    std::unordered_map<int64_t, Seq> seqs;
    bool prefix_cache = false;
    std::unordered_multimap<uint64_t, int32_t> by_key;   // prefix key -> block
    std::unordered_map<int32_t, Cached> cached;          // block -> entry
    std::list<int32_t> lru;                              // least recently used first
    int64_t hits = 0, misses = 0, evictions = 0;
    uint64_t step_calls = 0;                             // append_step calls so far
};

namespace {

bool valid_id(const pa_allocator* a, int32_t b) {
    return b >= 0 && b < static_cast<int32_t>(a->refcount.size());
}

int32_t take(pa_allocator* a) {        // caller checked the pool is not empty
    int32_t b = a->free_ids.front();
    a->free_ids.pop_front();
    a->refcount[b] = 1;
    return b;
}

void drop(pa_allocator* a, int32_t b) {  // caller checked refcount > 0
    if (--a->refcount[b] == 0) a->free_ids.push_back(b);
}

// Prefix key of a block: FNV-1a over the key of the prefix before it and the
// block's tokens (a 64-bit fingerprint of the whole token prefix).
uint64_t block_key(uint64_t parent, const int32_t* tokens, int n) {
    uint64_t h = 1469598103934665603ull ^ (parent * 0x9E3779B97F4A7C15ull);
    for (int i = 0; i < n; ++i) {
        uint32_t t = static_cast<uint32_t>(tokens[i]);
        for (int k = 0; k < 4; ++k) {
            h ^= (t >> (8 * k)) & 0xffu;
            h *= 1099511628211ull;
        }
    }
    return h;
}

// The cached block holding exactly this prefix (key, the key before it and
// the block's own tokens), or -1.  At most one block per prefix is cached.
int32_t lookup(const pa_manager* m, uint64_t key, uint64_t parent, const int32_t* t) {
    auto range = m->by_key.equal_range(key);
    for (auto k = range.first; k != range.second; ++k) {
        const auto& c = m->cached.at(k->second);
        if (c.parent == parent && std::equal(c.tokens.begin(), c.tokens.end(), t)) return k->second;
    }
    return -1;
}

// Take block b out of the cache (the cache's reference is dropped).
void uncache(pa_manager* m, int32_t b) {
    auto c = m->cached.find(b);
    auto range = m->by_key.equal_range(c->second.key);
    for (auto k = range.first; k != range.second; ++k)
        if (k->second == b) { m->by_key.erase(k); break; }
    m->lru.erase(c->second.lru);
    m->cached.erase(c);
    drop(m->alloc, b);
}

// Free one cached block that only the cache still references (least recently
// used first).  Returns false if there is none.
bool evict_one(pa_manager* m) {
    for (auto it = m->lru.begin(); it != m->lru.end(); ++it) {
        const int32_t b = *it;
        if (m->alloc->refcount[b] != 1) continue;
        uncache(m, b);                // back to the free pool
        ++m->evictions;
        return true;
    }
    return false;
}

// A block for a new table entry: from the free pool, else by evicting.
bool have_free(pa_manager* m) {
    if (!m->alloc->free_ids.empty()) return true;
    return m->prefix_cache && evict_one(m) && !m->alloc->free_ids.empty();
}

// One append, with enough recorded to undo it.
struct Undo {
    pa_manager::Seq* seq;
    int32_t taken;     // block taken by this append (-1 if none)
    int32_t cow_src;   // block whose reference was dropped by a copy (-1)
    bool grew;         // the table got a new entry
};

int append_one(pa_manager* m, pa_manager::Seq& s, int64_t* slot, Undo* u,
               int64_t* cow_src, int64_t* cow_dst) {
    pa_allocator* a = m->alloc;
    const int bs = m->block_size;
    const int32_t p = s.len;
    *u = Undo{&s, -1, -1, false};
    *cow_src = -1;
    *cow_dst = -1;
    if (p % bs == 0) {
        if (!have_free(m)) return PA_ERR_OOM;
        u->taken = take(a);
        s.table.push_back(u->taken);
        u->grew = true;
    } else {
        int32_t last = s.table.back();
        if (a->refcount[last] > 1) {
            if (!have_free(m)) return PA_ERR_OOM;
            u->taken = take(a);
            u->cow_src = last;
            drop(a, last);
            s.table.back() = u->taken;
            *cow_src = last;
            *cow_dst = u->taken;
        }
    }
    s.len = p + 1;
    *slot = static_cast<int64_t>(s.table[p / bs]) * bs + p % bs;
    return PA_OK;
}

// Reverse one append (applied newest first).  A block this append took is
// still referenced only by this sequence, so it goes back to the front of the
// pool; undoing newest first restores the pool's order as the appends found
// it.  A copy never sends its source to the pool (its count was above 1).
// With the prefix cache on, taking a block may first have evicted cached
// blocks (have_free); those evictions are not reversed: the blocks stay in the
// pool and their cache entries are gone.
void undo_one(pa_manager* m, const Undo& u) {
    pa_allocator* a = m->alloc;
    pa_manager::Seq& s = *u.seq;
    s.len -= 1;
    if (u.grew) {
        s.table.pop_back();
    } else if (u.cow_src >= 0) {
        s.table.back() = u.cow_src;
        a->refcount[u.cow_src] += 1;
    }
    if (u.taken >= 0) {
        a->refcount[u.taken] = 0;
        // put it back at the front so the next allocation gets it again
        a->free_ids.push_front(u.taken);
    }
}

}  // namespace

extern "C" {

const char* pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID: return "PA_ERR_INVALID";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        case PA_ERR_OOM: return "PA_ERR_OOM";
        case PA_ERR_STATE: return "PA_ERR_STATE";
        default: return "unknown pa_status";
    }
}

int pa_version(void) { return 200; }

int pa_allocator_create(int num_blocks, const int32_t* free_order, int num_free,
                        pa_allocator** out) {
    if (!out || num_blocks <= 0) return PA_ERR_INVALID;
    *out = nullptr;
    if (free_order && (num_free < 0 || num_free > num_blocks)) return PA_ERR_INVALID;
    pa_allocator* a = new (std::nothrow) pa_allocator;
    if (!a) return PA_ERR_OOM;
    if (!free_order) {
        a->refcount.assign(num_blocks, 0);
        for (int32_t b = 0; b < num_blocks; ++b) a->free_ids.push_back(b);
    } else {
        a->refcount.assign(num_blocks, 1);      // held by an outside owner ...
        for (int i = 0; i < num_free; ++i) {
            int32_t b = free_order[i];
            if (b < 0 || b >= num_blocks || a->refcount[b] == 0) {
                delete a;
                return PA_ERR_INVALID;          // out of range or listed twice
            }
            a->refcount[b] = 0;                 // ... unless listed as free
            a->free_ids.push_back(b);
        }
    }
    *out = a;
    return PA_OK;
}

void pa_allocator_destroy(pa_allocator* a) { delete a; }

int pa_allocator_allocate(pa_allocator* a, int32_t* block_id) {
    if (!a || !block_id) return PA_ERR_INVALID;
    if (a->free_ids.empty()) return PA_ERR_OOM;
    *block_id = take(a);
    return PA_OK;
}

int pa_allocator_incref(pa_allocator* a, int32_t b) {
    if (!a || !valid_id(a, b)) return PA_ERR_INVALID;
    if (a->refcount[b] <= 0) return PA_ERR_STATE;
    a->refcount[b] += 1;
    return PA_OK;
}

int pa_allocator_free(pa_allocator* a, int32_t b) {
    if (!a || !valid_id(a, b)) return PA_ERR_INVALID;
    if (a->refcount[b] <= 0) return PA_ERR_STATE;
    drop(a, b);
    return PA_OK;
}

int pa_allocator_refcount(const pa_allocator* a, int32_t b, int32_t* rc) {
    if (!a || !rc || !valid_id(a, b)) return PA_ERR_INVALID;
    *rc = a->refcount[b];
    return PA_OK;
}

int pa_allocator_num_free(const pa_allocator* a, int32_t* n) {
    if (!a || !n) return PA_ERR_INVALID;
    *n = static_cast<int32_t>(a->free_ids.size());
    return PA_OK;
}

int pa_manager_create(pa_allocator* alloc, int block_size, pa_manager** out) {
    if (!out) return PA_ERR_INVALID;
    *out = nullptr;
    if (!alloc || block_size <= 0) return PA_ERR_INVALID;
    pa_manager* m = new (std::nothrow) pa_manager;
    if (!m) return PA_ERR_OOM;
    m->alloc = alloc;
    m->block_size = block_size;
    *out = m;
    return PA_OK;
}

void pa_manager_destroy(pa_manager* m) { delete m; }

int pa_manager_add_seq(pa_manager* m, int64_t seq_id) {
    if (!m) return PA_ERR_INVALID;
    if (m->seqs.count(seq_id)) return PA_ERR_STATE;
    m->seqs.emplace(seq_id, pa_manager::Seq{});
    return PA_OK;
}

int pa_manager_fork(pa_manager* m, int64_t parent, int64_t child) {
    if (!m) return PA_ERR_INVALID;
    auto it = m->seqs.find(parent);
    if (it == m->seqs.end() || m->seqs.count(child)) return PA_ERR_STATE;
    for (int32_t b : it->second.table) m->alloc->refcount[b] += 1;
    pa_manager::Seq copy = it->second;   // copy before emplace may rehash
    m->seqs.emplace(child, std::move(copy));
    return PA_OK;
}

int pa_manager_free_seq(pa_manager* m, int64_t seq_id) {
    if (!m) return PA_ERR_INVALID;
    auto it = m->seqs.find(seq_id);
    if (it == m->seqs.end()) return PA_ERR_STATE;
    for (int32_t b : it->second.table) drop(m->alloc, b);
    m->seqs.erase(it);
    return PA_OK;
}

int pa_manager_append(pa_manager* m, int64_t seq_id, int num_tokens, int64_t* slots,
                      int64_t* cow_pairs, int* num_cow) {
    if (!m || num_tokens < 0 || (num_tokens > 0 && (!slots || !cow_pairs)) || !num_cow)
        return PA_ERR_INVALID;
    auto it = m->seqs.find(seq_id);
    if (it == m->seqs.end()) return PA_ERR_STATE;
    *num_cow = 0;
    std::vector<Undo> log(num_tokens);
    for (int i = 0; i < num_tokens; ++i) {
        int64_t src, dst;
        int st = append_one(m, it->second, &slots[i], &log[i], &src, &dst);
        if (st != PA_OK) {
            for (int k = i - 1; k >= 0; --k) undo_one(m, log[k]);
            *num_cow = 0;
            return st;
        }
        if (src >= 0) {   // only the first write into a shared block copies
            cow_pairs[0] = src;
            cow_pairs[1] = dst;
            *num_cow = 1;
        }
    }
    return PA_OK;
}

int pa_manager_append_step(pa_manager* m, const int64_t* seq_ids, int num_seqs,
                           int64_t* slots, int64_t* cow_pairs, int* num_cow) {
    if (!m || num_seqs < 0 || !num_cow || (num_seqs > 0 && (!seq_ids || !slots || !cow_pairs)))
        return PA_ERR_INVALID;
    std::vector<pa_manager::Seq*> ss(num_seqs);
    const uint64_t stamp = ++m->step_calls;   // a sequence may append once per step
    for (int i = 0; i < num_seqs; ++i) {
        auto it = m->seqs.find(seq_ids[i]);
        if (it == m->seqs.end()) return PA_ERR_STATE;
        if (it->second.stamp == stamp) return PA_ERR_INVALID;
        it->second.stamp = stamp;
        ss[i] = &it->second;
    }
    std::vector<Undo> log(num_seqs);
    int n = 0;
    for (int i = 0; i < num_seqs; ++i) {
        int64_t src, dst;
        int st = append_one(m, *ss[i], &slots[i], &log[i], &src, &dst);
        if (st != PA_OK) {
            for (int k = i - 1; k >= 0; --k) undo_one(m, log[k]);
            *num_cow = 0;
            return st;
        }
        if (src >= 0) {
            cow_pairs[2 * n] = src;
            cow_pairs[2 * n + 1] = dst;
            ++n;
        }
    }
    *num_cow = n;
    return PA_OK;
}

int pa_manager_seq_len(const pa_manager* m, int64_t seq_id, int32_t* len) {
    if (!m || !len) return PA_ERR_INVALID;
    auto it = m->seqs.find(seq_id);
    if (it == m->seqs.end()) return PA_ERR_STATE;
    *len = it->second.len;
    return PA_OK;
}

int pa_manager_block_tables(const pa_manager* m, const int64_t* seq_ids, int num_seqs,
                            int32_t* block_tables, int max_blocks, int32_t* context_lens) {
    if (!m || num_seqs < 0 || max_blocks <= 0 ||
        (num_seqs > 0 && (!seq_ids || !block_tables || !context_lens)))
        return PA_ERR_INVALID;
    for (int i = 0; i < num_seqs; ++i) {
        auto it = m->seqs.find(seq_ids[i]);
        if (it == m->seqs.end()) return PA_ERR_STATE;
        const auto& t = it->second.table;
        if (static_cast<int>(t.size()) > max_blocks) return PA_ERR_INVALID;
        int32_t* row = block_tables + static_cast<int64_t>(i) * max_blocks;
        std::copy(t.begin(), t.end(), row);
        std::fill(row + t.size(), row + max_blocks, int32_t(-1));
        context_lens[i] = it->second.len;
    }
    return PA_OK;
}

int pa_manager_enable_prefix_cache(pa_manager* m) {
    if (!m) return PA_ERR_INVALID;
    if (!m->seqs.empty()) return PA_ERR_STATE;
    m->prefix_cache = true;
    return PA_OK;
}

int pa_manager_add_seq_prompt(pa_manager* m, int64_t seq_id, const int32_t* tokens,
                              int num_tokens, int64_t* slots, int* num_cached) {
    if (!m || num_tokens < 0 || !num_cached || (num_tokens > 0 && (!tokens || !slots)))
        return PA_ERR_INVALID;
    if (!m->prefix_cache) return PA_ERR_STATE;
    if (m->seqs.count(seq_id)) return PA_ERR_STATE;
    pa_allocator* a = m->alloc;
    const int bs = m->block_size;
    pa_manager::Seq s;
    // 1. the longest run of leading full blocks already cached, leaving at
    // least the prompt's last token to compute (its attention output is what
    // the first generated token needs): a prompt that is a whole number of
    // blocks looks up all but its last block
    uint64_t parent = 0;
    int hit = 0;
    const int full = num_tokens / bs;
    const int lookable = num_tokens > 0 ? (num_tokens - 1) / bs : 0;
    for (; hit < lookable; ++hit) {
        const int32_t* t = tokens + static_cast<int64_t>(hit) * bs;
        const uint64_t key = block_key(parent, t, bs);
        const int32_t found = lookup(m, key, parent, t);
        if (found < 0) break;
        a->refcount[found] += 1;
        auto& c = m->cached.at(found);
        m->lru.splice(m->lru.end(), m->lru, c.lru);     // most recently used
        s.table.push_back(found);
        parent = key;
    }
    s.len = hit * bs;
    // 2. the rest is appended; every prompt block it fills is registered
    std::vector<int32_t> registered;   // blocks this call put in the cache
    for (int i = s.len; i < num_tokens; ++i) {
        if (i % bs == 0) {
            if (!have_free(m)) {
                // nothing of this call stays: its blocks will never be written
                for (int32_t b : registered) uncache(m, b);
                for (int32_t b : s.table) drop(a, b);   // hits and new blocks alike
                return PA_ERR_OOM;
            }
            s.table.push_back(take(a));
        }
        s.len = i + 1;
        if ((i + 1) % bs == 0) {                         // a full prompt block
            const int32_t blk = s.table.back();
            const int32_t* t = tokens + static_cast<int64_t>(i + 1 - bs);
            const uint64_t key = block_key(parent, t, bs);
            if (lookup(m, key, parent, t) >= 0) {        // this prefix is cached already
                parent = key;
                continue;
            }
            m->lru.push_back(blk);
            m->cached.emplace(blk, pa_manager::Cached{key, parent,
                                                      std::vector<int32_t>(t, t + bs),
                                                      std::prev(m->lru.end())});
            m->by_key.emplace(key, blk);
            a->refcount[blk] += 1;                       // the cache's reference
            registered.push_back(blk);
            parent = key;
        }
    }
    m->hits += hit;
    m->misses += full - hit;
    for (int i = 0; i < num_tokens; ++i)
        slots[i] = i < hit * bs ? -1
                                : static_cast<int64_t>(s.table[i / bs]) * bs + i % bs;
    *num_cached = hit * bs;
    m->seqs.emplace(seq_id, std::move(s));
    return PA_OK;
}

int pa_manager_prefix_cache_stats(const pa_manager* m, int64_t* stats) {
    if (!m || !stats) return PA_ERR_INVALID;
    stats[0] = static_cast<int64_t>(m->cached.size());
    stats[1] = m->hits;
    stats[2] = m->misses;
    stats[3] = m->evictions;
    return PA_OK;
}

}  // extern "C"
