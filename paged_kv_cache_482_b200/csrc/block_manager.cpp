// block_manager.cpp -- the host-side block manager of libpagedkv.so (C ABI in
// include/pagedkv_blocks.h).
//
// It assigns the physical blocks of the paged KV pool to sequences, shares
// full blocks between sequences whose token prefixes are equal, and produces
// the block tables, context lengths and slot mappings the kernels read
// ("Nano-vLLM：轻量高效的大模型推理框架", sections 三.1 and 三.2 (1);
// "DeepSeek复刻vLLM反超原版", section "vLLM：大模型推理的加速引擎与挑战").
//
// Data structures, all sized once at creation:
//  * tokens_[b * bs + i]: the token each slot of block b holds (what a hit
//    is verified against, and what a filled block's key is computed from);
//  * a doubly linked FIFO queue of free blocks (O(1) removal when a hit
//    lands on a free block that still holds a cached prefix);
//  * a 128-bit chain key per cached full block, key(b_i) = mix(key(b_{i-1}),
//    tokens of b_i), plus the parent's key, in an open-addressing table
//    (linear probing, backward-shift deletion, load <= 1/2) indexed by the
//    key's first 64 bits. A hit compares the other 64 bits, the parent key
//    and the block's tokens.
// Every call checks all it needs before it changes anything.
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "pagedkv_blocks.h"

namespace {

struct Key {
    uint64_t a = 0, b = 0;
    bool operator==(const Key &o) const { return a == o.a && b == o.b; }
};

// Root of every chain (the key of the empty prefix).
constexpr Key kRoot{0x243f6a8885a308d3ull, 0x13198a2e03707344ull};

inline uint64_t rotl(uint64_t x, int r) { return (x << r) | (x >> (64 - r)); }

// Final avalanche: the splitmix64 output function (Steele, Lea, Flood,
// "Fast splittable pseudorandom number generators", OOPSLA 2014).
inline uint64_t fmix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
}

// Key of a block from its parent's key and its tokens: two independent
// multiply-rotate lanes over the tokens, each finished with fmix.
Key chain_key(const Key &parent, const int32_t *tok, int n) {
    uint64_t a = parent.a ^ 0x9e3779b97f4a7c15ull, b = parent.b ^ 0xc2b2ae3d27d4eb4full;
    for (int i = 0; i < n; ++i) {
        const uint64_t t = static_cast<uint32_t>(tok[i]);
        a = rotl((a ^ t) * 0xff51afd7ed558ccdull, 29);
        b = rotl((b + t) * 0xc4ceb9fe1a85ec53ull, 37) ^ (b >> 17);
    }
    return Key{fmix(a ^ static_cast<uint64_t>(n)), fmix(b + parent.a)};
}

struct Seq {
    std::vector<int32_t> table;
    int64_t num_tokens = 0;
    int32_t off = 0;        // num_tokens % block_size, kept so that appends divide nothing
    Key last_full = kRoot;  // key of the last full block (the next block's parent)
    uint64_t stamp = 0;     // repeated-id check in batch calls (64 bits: never wraps)
};

// Live sequences by id: open addressing with linear probing and
// backward-shift deletion over a power-of-two table, the records in a slab
// whose slots are reused. A decode step looks every sequence up twice
// (append, then the table row), so the lookup is a multiply, a mask and
// usually one compare. Pointers into the slab stay valid until the next
// insert.
class SeqTable {
  public:
    Seq *find(int64_t id) {
        if (count_ == 0) return nullptr;
        for (uint64_t i = home(id);; i = (i + 1) & mask_) {
            if (val_[i] < 0) return nullptr;
            if (key_[i] == id) return &slab_[val_[i]];
        }
    }
    const Seq *find(int64_t id) const { return const_cast<SeqTable *>(this)->find(id); }

    // id must be absent. Throws std::bad_alloc before any change.
    Seq *insert(int64_t id) {
        if ((count_ + 1) * 2 > val_.size()) grow();
        int32_t slot;
        if (!free_.empty()) {
            slot = free_.back();
            free_.pop_back();
        } else {
            free_.reserve(slab_.size() + 1);  // so that erase never allocates
            slab_.emplace_back();
            slot = static_cast<int32_t>(slab_.size() - 1);
        }
        uint64_t i = home(id);
        while (val_[i] >= 0) i = (i + 1) & mask_;
        key_[i] = id;
        val_[i] = slot;
        ++count_;
        return &slab_[slot];
    }

    // Removes id (nothing happens when it is absent).
    void erase(int64_t id) {
        if (count_ == 0) return;
        uint64_t i = home(id);
        for (;; i = (i + 1) & mask_) {
            if (val_[i] < 0) return;
            if (key_[i] == id) break;
        }
        slab_[val_[i]] = Seq{};
        free_.push_back(val_[i]);
        val_[i] = -1;
        --count_;
        // pull later entries of the probe run back over the hole when their
        // home is at or before it
        for (uint64_t j = (i + 1) & mask_; val_[j] >= 0; j = (j + 1) & mask_) {
            if (((j - home(key_[j])) & mask_) >= ((j - i) & mask_)) {
                key_[i] = key_[j];
                val_[i] = val_[j];
                val_[j] = -1;
                i = j;
            }
        }
    }

  private:
    uint64_t home(int64_t id) const {
        const uint64_t h = static_cast<uint64_t>(id) * 0x9E3779B97F4A7C15ull;
        return (h ^ (h >> 29)) & mask_;
    }
    void grow() {
        const size_t cap = val_.empty() ? 64 : 2 * val_.size();
        std::vector<int64_t> key(cap);
        std::vector<int32_t> val(cap, -1);
        const uint64_t mask = cap - 1;
        std::swap(key, key_);
        std::swap(val, val_);
        mask_ = mask;
        for (size_t i = 0; i < val.size(); ++i) {
            if (val[i] < 0) continue;
            uint64_t k = home(key[i]);
            while (val_[k] >= 0) k = (k + 1) & mask_;
            key_[k] = key[i];
            val_[k] = val[i];
        }
    }

    std::vector<int64_t> key_;
    std::vector<int32_t> val_;  // slab slot, -1 empty
    uint64_t mask_ = 0;
    size_t count_ = 0;
    std::vector<Seq> slab_;
    std::vector<int32_t> free_;
};

}  // namespace

struct pkv_block_manager {
    int64_t nb;
    int bs;
    std::vector<int32_t> tokens;  // [nb * bs]
    std::vector<int32_t> ref;     // users of each block
    std::vector<int32_t> fill;    // tokens written into each block
    // free queue
    std::vector<int32_t> prev, next;
    int32_t head = -1, tail = -1;
    int64_t nfree = 0;
    std::vector<uint8_t> in_queue;
    // cache entries
    std::vector<uint8_t> has_key;
    std::vector<Key> key, parent;
    std::vector<int32_t> slot_of;  // block -> index in `table` (for deletion)
    std::vector<int32_t> table;    // open addressing: block id or -1
    uint64_t mask;
    SeqTable seqs;
    std::vector<Seq *> step;  // scratch of the batch calls
    uint64_t stamp = 0;       // batch-call counter; records start at 0, calls at 1

    pkv_block_manager(int64_t n, int b) : nb(n), bs(b) {
        tokens.assign(static_cast<size_t>(n) * b, 0);
        ref.assign(n, 0);
        fill.assign(n, 0);
        prev.resize(n);
        next.resize(n);
        in_queue.assign(n, 1);
        for (int64_t i = 0; i < n; ++i) {
            prev[i] = static_cast<int32_t>(i - 1);
            next[i] = i + 1 < n ? static_cast<int32_t>(i + 1) : -1;
        }
        head = 0;
        tail = static_cast<int32_t>(n - 1);
        nfree = n;
        has_key.assign(n, 0);
        key.resize(n);
        parent.resize(n);
        slot_of.assign(n, -1);
        uint64_t cap = 16;
        while (cap < 2 * static_cast<uint64_t>(n)) cap <<= 1;
        table.assign(cap, -1);
        mask = cap - 1;
    }

    // ---------------------------------------------------------- free queue
    void q_remove(int32_t b) {
        const int32_t p = prev[b], x = next[b];
        if (p >= 0) next[p] = x; else head = x;
        if (x >= 0) prev[x] = p; else tail = p;
        in_queue[b] = 0;
        --nfree;
    }
    void q_push_back(int32_t b) {
        prev[b] = tail;
        next[b] = -1;
        if (tail >= 0) next[tail] = b; else head = b;
        tail = b;
        in_queue[b] = 1;
        ++nfree;
    }

    // -------------------------------------------------------- cache table
    bool matches(int32_t b, const Key &k, const Key &par, const int32_t *tok) const {
        return key[b] == k && parent[b] == par && std::memcmp(&tokens[static_cast<size_t>(b) * bs], tok,
                                                              sizeof(int32_t) * bs) == 0;
    }
    // Cached block with this key, parent and tokens, or -1.
    int32_t lookup(const Key &k, const Key &par, const int32_t *tok) const {
        for (uint64_t i = k.a & mask;; i = (i + 1) & mask) {
            const int32_t b = table[i];
            if (b < 0) return -1;
            if (key[b].a == k.a) return matches(b, k, par, tok) ? b : -1;
        }
    }
    void erase(int32_t b) {
        uint64_t i = static_cast<uint64_t>(slot_of[b]);
        has_key[b] = 0;
        slot_of[b] = -1;
        // backward-shift deletion keeps every probe run unbroken
        for (uint64_t j = (i + 1) & mask;; j = (j + 1) & mask) {
            const int32_t c = table[j];
            if (c < 0) break;
            const uint64_t home = key[c].a & mask;
            // c may move to i if its home does not lie cyclically in (i, j]
            const bool stay = (j > i) ? (home > i && home <= j) : (home > i || home <= j);
            if (!stay) {
                table[i] = c;
                slot_of[c] = static_cast<int32_t>(i);
                i = j;
            }
        }
        table[i] = -1;
    }
    // Cache block b (full, tokens in place) under key k with parent par. An
    // entry with the same first 64 key bits (the same prefix, or a
    // different one that collides there) gives way to the newer block.
    void insert(int32_t b, const Key &k, const Key &par) {
        if (has_key[b]) erase(b);
        uint64_t i = k.a & mask;
        for (;; i = (i + 1) & mask) {
            const int32_t c = table[i];
            if (c < 0) break;
            if (key[c].a == k.a) {
                erase(c);
                insert(b, k, par);
                return;
            }
        }
        key[b] = k;
        parent[b] = par;
        has_key[b] = 1;
        table[i] = b;
        slot_of[b] = static_cast<int32_t>(i);
    }

    // A free block for new content: from the queue's front; whatever it
    // cached is about to be overwritten.
    int32_t take_free() {
        const int32_t b = head;
        q_remove(b);
        if (has_key[b]) erase(b);
        fill[b] = 0;
        return b;
    }

    void release(Seq &s) {
        for (auto it = s.table.rbegin(); it != s.table.rend(); ++it) {
            if (--ref[*it] == 0) q_push_back(*it);
        }
    }

    // Appends one token to s (a free block must exist when one is needed).
    int32_t append(Seq &s, int32_t tok) {
        const int off = s.off;
        if (off == 0) {  // the sequence's blocks are all full: open one
            const int32_t b = take_free();
            ref[b] = 1;
            s.table.push_back(b);
        }
        const int32_t b = s.table.back();  // the block holding position num_tokens
        tokens[static_cast<size_t>(b) * bs + off] = tok;
        fill[b] = off + 1;
        s.num_tokens += 1;
        if (off + 1 == bs) {
            const Key k = chain_key(s.last_full, &tokens[static_cast<size_t>(b) * bs], bs);
            insert(b, k, s.last_full);
            s.last_full = k;
            s.off = 0;
        } else {
            s.off = off + 1;
        }
        return static_cast<int32_t>(static_cast<int64_t>(b) * bs + off);
    }
};

extern "C" {

pkv_block_manager *pkv_bm_create(int64_t num_blocks, int block_size) {
    if (num_blocks < 1 || block_size < 1) return nullptr;
    if (num_blocks > INT32_MAX / block_size) return nullptr;  // slots are int32
    try {
        return new pkv_block_manager(num_blocks, block_size);
    } catch (...) {
        return nullptr;
    }
}

void pkv_bm_destroy(pkv_block_manager *bm) { delete bm; }

int pkv_bm_add_sequence(pkv_block_manager *bm, int64_t seq_id, const int32_t *tokens, int num_tokens,
                        int *num_cached_tokens) {
    if (!bm || !tokens || !num_cached_tokens || num_tokens < 1) return PKV_ERR_INVALID_ARG;
    if (bm->seqs.find(seq_id)) return PKV_ERR_INVALID_ARG;
    const int bs = bm->bs;
    const int64_t n_blocks = (static_cast<int64_t>(num_tokens) + bs - 1) / bs;
    if (n_blocks > bm->nb) return PKV_ERR_WORKSPACE;
    // leading full blocks that are cached
    std::vector<int32_t> hits;
    std::vector<Key> keys;
    Key par = kRoot;
    int64_t free_hits = 0;
    for (int64_t i = 0; i < num_tokens / bs; ++i) {
        const int32_t *tok = tokens + i * bs;
        const Key k = chain_key(par, tok, bs);
        const int32_t b = bm->lookup(k, par, tok);
        if (b < 0) break;
        hits.push_back(b);
        keys.push_back(k);
        free_hits += bm->ref[b] == 0;
        par = k;
    }
    const int64_t need = n_blocks - static_cast<int64_t>(hits.size());
    if (bm->nfree - free_hits < need) return PKV_ERR_WORKSPACE;
    try {
        Seq s;
        s.table.reserve(n_blocks + 1);  // appends below stay within it: nothing throws after the insert
        Seq &q = *bm->seqs.insert(seq_id);
        q = std::move(s);
        for (int32_t b : hits) {
            if (bm->ref[b] == 0) bm->q_remove(b);
            ++bm->ref[b];
            q.table.push_back(b);
        }
        q.num_tokens = static_cast<int64_t>(hits.size()) * bs;
        q.last_full = hits.empty() ? kRoot : keys.back();
        for (int64_t p = q.num_tokens; p < num_tokens; ++p) bm->append(q, tokens[p]);
    } catch (const std::bad_alloc &) {
        return PKV_ERR_WORKSPACE;
    }
    *num_cached_tokens = static_cast<int>(hits.size()) * bs;
    return PKV_OK;
}

int pkv_bm_append_token(pkv_block_manager *bm, int64_t seq_id, int32_t token, int64_t *slot) {
    if (!bm || !slot) return PKV_ERR_INVALID_ARG;
    Seq *sp = bm->seqs.find(seq_id);
    if (!sp) return PKV_ERR_INVALID_ARG;
    Seq &s = *sp;
    if (s.off == 0 && bm->nfree == 0) return PKV_ERR_WORKSPACE;
    if (s.num_tokens >= INT32_MAX) return PKV_ERR_INVALID_ARG;
    *slot = bm->append(s, token);
    return PKV_OK;
}

int pkv_bm_free_sequence(pkv_block_manager *bm, int64_t seq_id) {
    if (!bm) return PKV_ERR_INVALID_ARG;
    Seq *sp = bm->seqs.find(seq_id);
    if (!sp) return PKV_ERR_INVALID_ARG;
    bm->release(*sp);
    bm->seqs.erase(seq_id);
    return PKV_OK;
}

int pkv_bm_block_table(const pkv_block_manager *bm, int64_t seq_id, int32_t *row, int max_blocks,
                       int *num_tokens) {
    if (!bm || !num_tokens || max_blocks < 0 || (max_blocks > 0 && !row)) return PKV_ERR_INVALID_ARG;
    const Seq *sp = bm->seqs.find(seq_id);
    if (!sp) return PKV_ERR_INVALID_ARG;
    const Seq &s = *sp;
    const int n = static_cast<int>(s.table.size());
    *num_tokens = static_cast<int>(s.num_tokens);
    if (n > max_blocks) return PKV_ERR_INVALID_ARG;
    std::memcpy(row, s.table.data(), sizeof(int32_t) * n);
    for (int i = n; i < max_blocks; ++i) row[i] = -1;
    return PKV_OK;
}

int pkv_bm_slots(const pkv_block_manager *bm, int64_t seq_id, int start, int count, int32_t *slots) {
    if (!bm || start < 0 || count < 0 || (count > 0 && !slots)) return PKV_ERR_INVALID_ARG;
    const Seq *sp = bm->seqs.find(seq_id);
    if (!sp) return PKV_ERR_INVALID_ARG;
    const Seq &s = *sp;
    if (static_cast<int64_t>(start) + count > s.num_tokens) return PKV_ERR_INVALID_ARG;
    const int bs = bm->bs;
    for (int i = 0; i < count; ++i) {
        const int p = start + i;
        slots[i] = s.table[p / bs] * bs + p % bs;
    }
    return PKV_OK;
}

int64_t pkv_bm_num_free_blocks(const pkv_block_manager *bm) { return bm ? bm->nfree : -1; }

int pkv_bm_block_refcount(const pkv_block_manager *bm, int64_t block, int *refcount) {
    if (!bm || !refcount || block < 0 || block >= bm->nb) return PKV_ERR_INVALID_ARG;
    *refcount = bm->ref[block];
    return PKV_OK;
}

int pkv_bm_append_tokens(pkv_block_manager *bm, const int64_t *seq_ids, const int32_t *tokens, int n,
                         int32_t *slots) {
    if (!bm || n < 0 || (n > 0 && (!seq_ids || !tokens || !slots))) return PKV_ERR_INVALID_ARG;
    if (n == 0) return PKV_OK;
    // pass 1: every id live and distinct; count the blocks the step needs
    std::vector<Seq *> &ss = bm->step;
    try {
        ss.resize(n);
    } catch (const std::bad_alloc &) {
        return PKV_ERR_WORKSPACE;
    }
    const uint64_t st = ++bm->stamp;
    int64_t need = 0;
    int bad = 0;
    for (int i = 0; i < n; ++i) {
        Seq *q = bm->seqs.find(seq_ids[i]);
        if (!q || q->stamp == st || q->num_tokens >= INT32_MAX) {
            bad = 1;
            break;
        }
        q->stamp = st;
        ss[i] = q;
        need += q->off == 0;
    }
    if (bad) return PKV_ERR_INVALID_ARG;
    if (need > bm->nfree) return PKV_ERR_WORKSPACE;
    // pass 2: apply
    for (int i = 0; i < n; ++i) slots[i] = bm->append(*ss[i], tokens[i]);
    return PKV_OK;
}

int pkv_bm_block_tables(const pkv_block_manager *bm, const int64_t *seq_ids, int n, int32_t *block_tables,
                        int max_blocks, int32_t *context_lens) {
    if (!bm || n < 0 || max_blocks < 0) return PKV_ERR_INVALID_ARG;
    if (n > 0 && (!seq_ids || !block_tables || !context_lens)) return PKV_ERR_INVALID_ARG;
    for (int i = 0; i < n; ++i) {
        const Seq *sp = bm->seqs.find(seq_ids[i]);
        if (!sp) return PKV_ERR_INVALID_ARG;
        const Seq &s = *sp;
        const int nb = static_cast<int>(s.table.size());
        if (nb > max_blocks) return PKV_ERR_INVALID_ARG;
        int32_t *row = block_tables + static_cast<size_t>(i) * max_blocks;
        std::memcpy(row, s.table.data(), sizeof(int32_t) * nb);
        for (int j = nb; j < max_blocks; ++j) row[j] = -1;
        context_lens[i] = static_cast<int32_t>(s.num_tokens);
    }
    return PKV_OK;
}

}  // extern "C"
