// Host-side block manager; see block_manager.h for the rules it follows.
#include "block_manager.h"

#include <algorithm>
#include <limits>

namespace pkv {

BlockManager::BlockManager(int num_blocks, int block_size)
    : num_blocks_(num_blocks), block_size_(block_size), next_(num_blocks, -1),
      prev_(num_blocks, -1), ref_(num_blocks, 0), hashed_(num_blocks, 0), hash_(num_blocks, 0) {
    reset(nullptr);
}

pkv_status BlockManager::reset(const int32_t* order) {
    if (order) {
        std::vector<char> seen(num_blocks_, 0);
        for (int i = 0; i < num_blocks_; ++i) {
            int32_t b = order[i];
            if (b < 0 || b >= num_blocks_ || seen[b]) return PKV_ERR_INVALID_ARG;
            seen[b] = 1;
        }
    }
    head_ = tail_ = -1;
    count_ = 0;
    for (int i = 0; i < num_blocks_; ++i) push_back(order ? order[i] : i);
    std::fill(ref_.begin(), ref_.end(), 0);
    seqs_.clear();
    cow_count_ = 0;
    std::fill(hashed_.begin(), hashed_.end(), 0);
    by_hash_.clear();
    hit_tokens_ = 0;
    return PKV_OK;
}

int BlockManager::fill_of_last(const Sequence& s) const {
    if (s.blocks.empty()) return 0;
    return (int)(s.length - (int64_t)(s.blocks.size() - 1) * block_size_);
}

void BlockManager::push_back(int32_t b) {
    next_[b] = -1;
    prev_[b] = tail_;
    if (tail_ >= 0) next_[tail_] = b; else head_ = b;
    tail_ = b;
    ++count_;
}

void BlockManager::remove_free(int32_t b) {
    if (prev_[b] >= 0) next_[prev_[b]] = next_[b]; else head_ = next_[b];
    if (next_[b] >= 0) prev_[next_[b]] = prev_[b]; else tail_ = prev_[b];
    next_[b] = prev_[b] = -1;
    --count_;
}

// a block handed out as a fresh block loses its registration
int32_t BlockManager::pop_front() {
    const int32_t b = head_;
    remove_free(b);
    unregister(b);
    ref_[b] = 1;
    return b;
}

void BlockManager::unpop_front(int32_t b) {
    next_[b] = head_;
    prev_[b] = -1;
    if (head_ >= 0) prev_[head_] = b; else tail_ = b;
    head_ = b;
    ++count_;
    ref_[b] = 0;
}

void BlockManager::unregister(int32_t b) {
    if (!hashed_[b]) return;
    auto it = by_hash_.find(hash_[b]);
    if (it != by_hash_.end() && it->second == b) by_hash_.erase(it);
    hashed_[b] = 0;
    dropped_.emplace_back(b, hash_[b]);
}

void BlockManager::restore_dropped() {
    for (auto r = dropped_.rbegin(); r != dropped_.rend(); ++r) {
        hashed_[r->first] = 1;
        hash_[r->first] = r->second;
        by_hash_[r->second] = r->first;
    }
    dropped_.clear();
}

int32_t BlockManager::lookup(uint64_t h, const int32_t* tokens) const {
    auto it = by_hash_.find(h);
    if (it == by_hash_.end()) return -1;
    const int32_t b = it->second;
    const int32_t* bt = block_tokens_.data() + (size_t)b * block_size_;
    for (int i = 0; i < block_size_; ++i)
        if (bt[i] != tokens[i]) return -1;   // a hash collision: not the same tokens
    return b;
}

void BlockManager::set_prefix_caching(bool on) {
    caching_ = on;
    if (on && block_tokens_.empty()) block_tokens_.assign((size_t)num_blocks_ * block_size_, 0);
    if (!on) {
        std::fill(hashed_.begin(), hashed_.end(), 0);
        by_hash_.clear();
    }
}

namespace {
// FNV-1a, 64 bit (offset basis 14695981039346656037, prime 1099511628211),
// over the parent hash (8 bytes, little endian) and the block's token ids
// (4 bytes each, little endian): the chain hash of a full block.
uint64_t chain_hash(uint64_t parent, const int32_t* tokens, int n) {
    uint64_t h = 14695981039346656037ull;
    auto eat = [&h](uint8_t byte) {
        h ^= byte;
        h *= 1099511628211ull;
    };
    for (int i = 0; i < 8; ++i) eat((uint8_t)(parent >> (8 * i)));
    for (int t = 0; t < n; ++t) {
        const uint32_t v = (uint32_t)tokens[t];
        for (int i = 0; i < 4; ++i) eat((uint8_t)(v >> (8 * i)));
    }
    return h;
}
}  // namespace

pkv_status BlockManager::alloc_prefix(int64_t seq, const int32_t* tokens, int n_tokens,
                                      int32_t* slots, int32_t* n_cached) {
    if (n_tokens < 0 || (n_tokens > 0 && (!slots || !tokens)) || !n_cached)
        return PKV_ERR_INVALID_ARG;
    if (!caching_) {
        const pkv_status st = alloc(seq, n_tokens, slots);
        if (st == PKV_OK) *n_cached = 0;
        return st;
    }
    dropped_.clear();
    if (seqs_.count(seq)) return PKV_ERR_SEQ_EXISTS;
    const int bs = block_size_;
    const int need = (n_tokens + bs - 1) / bs;
    const int full = n_tokens / bs;
    // leading full blocks already registered with the same tokens
    std::vector<int32_t> hits;
    std::vector<uint64_t> hashes((size_t)full);
    uint64_t parent = 0;
    int free_hits = 0;
    bool hitting = true;
    for (int i = 0; i < full; ++i) {
        hashes[i] = chain_hash(parent, tokens + (size_t)i * bs, bs);
        parent = hashes[i];
        if (hitting) {
            const int32_t b = lookup(hashes[i], tokens + (size_t)i * bs);
            if (b >= 0) {
                hits.push_back(b);
                free_hits += ref_[b] == 0;
            } else {
                hitting = false;
            }
        }
    }
    const int fresh = need - (int)hits.size();
    if (fresh > count_ - free_hits) return PKV_ERR_NO_BLOCKS;
    Sequence s;
    s.blocks.reserve((size_t)need);
    for (int32_t b : hits) {
        if (ref_[b] == 0) remove_free(b);
        ++ref_[b];
        s.blocks.push_back(b);
    }
    for (int i = (int)hits.size(); i < need; ++i) {
        const int32_t b = pop_front();
        s.blocks.push_back(b);
        if (i < full && !by_hash_.count(hashes[i])) {
            hashed_[b] = 1;
            hash_[b] = hashes[i];
            by_hash_[hashes[i]] = b;
            std::copy(tokens + (size_t)i * bs, tokens + (size_t)(i + 1) * bs,
                      block_tokens_.begin() + (size_t)b * bs);
        }
    }
    s.length = n_tokens;
    s.epoch = next_epoch_++;
    for (int t = 0; t < n_tokens; ++t) slots[t] = s.blocks[t / bs] * bs + t % bs;
    *n_cached = (int32_t)hits.size() * bs;
    hit_tokens_ += *n_cached;
    seqs_.emplace(seq, std::move(s));
    return PKV_OK;
}

pkv_status BlockManager::alloc(int64_t seq, int n_tokens, int32_t* slots) {
    dropped_.clear();
    if (n_tokens < 0 || (n_tokens > 0 && !slots)) return PKV_ERR_INVALID_ARG;
    if (seqs_.count(seq)) return PKV_ERR_SEQ_EXISTS;
    const int64_t need = ((int64_t)n_tokens + block_size_ - 1) / block_size_;
    if (need > count_) return PKV_ERR_NO_BLOCKS;
    Sequence s;
    s.blocks.reserve((size_t)need);
    for (int64_t i = 0; i < need; ++i) s.blocks.push_back(pop_front());
    s.length = n_tokens;
    s.epoch = next_epoch_++;
    for (int t = 0; t < n_tokens; ++t)
        slots[t] = s.blocks[t / block_size_] * block_size_ + t % block_size_;
    seqs_.emplace(seq, std::move(s));
    return PKV_OK;
}

pkv_status BlockManager::append_one(int64_t seq, int32_t* slot, int32_t* src, int32_t* dst,
                                    Undo* undo) {
    auto it = seqs_.find(seq);
    if (it == seqs_.end()) return PKV_ERR_UNKNOWN_SEQ;
    Sequence& s = it->second;
    int fill = fill_of_last(s);
    int32_t csrc = -1, cdst = -1;
    int kind = 0;
    int32_t old = -1;
    if (s.blocks.empty() || fill == block_size_) {
        // the last block is full (or there is none): take a fresh block
        if (count_ == 0) return PKV_ERR_NO_BLOCKS;
        s.blocks.push_back(pop_front());
        fill = 0;
        kind = 1;
    } else if (ref_[s.blocks.back()] > 1) {
        // partially filled and shared: copy on write into a fresh block
        if (count_ == 0) return PKV_ERR_NO_BLOCKS;
        old = s.blocks.back();
        int32_t fresh = pop_front();
        --ref_[old];
        s.blocks.back() = fresh;
        csrc = old;
        cdst = fresh;
        ++cow_count_;
        kind = 2;
    }
    *slot = s.blocks.back() * block_size_ + fill;
    s.length += 1;
    if (src) *src = csrc;
    if (dst) *dst = cdst;
    if (undo) *undo = Undo{seq, kind, old};
    return PKV_OK;
}

void BlockManager::undo_one(const Undo& u) {
    Sequence& s = seqs_.at(u.seq);
    s.length -= 1;
    if (u.kind == 1) {
        int32_t b = s.blocks.back();
        s.blocks.pop_back();
        unpop_front(b);
    } else if (u.kind == 2) {
        int32_t fresh = s.blocks.back();
        s.blocks.back() = u.old_block;
        ++ref_[u.old_block];
        unpop_front(fresh);
        --cow_count_;
    }
}

pkv_status BlockManager::append(int64_t seq, int32_t* slot, int32_t* cow_src, int32_t* cow_dst) {
    if (!slot) return PKV_ERR_INVALID_ARG;
    return append_one(seq, slot, cow_src, cow_dst, nullptr);
}

pkv_status BlockManager::append_batch(const int64_t* seqs, int n, int32_t* slots, int32_t* cow_src,
                                      int32_t* cow_dst, int* n_cow) {
    if (n < 0 || (n > 0 && (!seqs || !slots || !cow_src || !cow_dst)) || !n_cow)
        return PKV_ERR_INVALID_ARG;
    dropped_.clear();
    std::vector<Undo> log;
    log.reserve((size_t)n);
    int pairs = 0;
    for (int i = 0; i < n; ++i) {
        int32_t src = -1, dst = -1;
        Undo u;
        pkv_status st = append_one(seqs[i], &slots[i], &src, &dst, &u);
        if (st != PKV_OK) {
            for (auto r = log.rbegin(); r != log.rend(); ++r) undo_one(*r);
            restore_dropped();
            return st;
        }
        log.push_back(u);
        if (src >= 0) {
            cow_src[pairs] = src;
            cow_dst[pairs] = dst;
            ++pairs;
        }
    }
    *n_cow = pairs;
    return PKV_OK;
}

pkv_status BlockManager::fork(int64_t parent, int64_t child) {
    auto it = seqs_.find(parent);
    if (it == seqs_.end()) return PKV_ERR_UNKNOWN_SEQ;
    if (seqs_.count(child)) return PKV_ERR_SEQ_EXISTS;
    Sequence c = it->second;  // copy of the table and the length
    c.epoch = next_epoch_++;
    for (int32_t b : c.blocks) ++ref_[b];
    seqs_.emplace(child, std::move(c));
    return PKV_OK;
}

pkv_status BlockManager::release(int64_t seq) {
    auto it = seqs_.find(seq);
    if (it == seqs_.end()) return PKV_ERR_UNKNOWN_SEQ;
    for (int32_t b : it->second.blocks)
        if (--ref_[b] == 0) push_back(b);
    seqs_.erase(it);
    return PKV_OK;
}

void BlockManager::undo_alloc(int64_t seq) {
    auto it = seqs_.find(seq);
    if (it == seqs_.end()) return;
    const std::vector<int32_t>& b = it->second.blocks;
    for (auto r = b.rbegin(); r != b.rend(); ++r) unpop_front(*r);
    seqs_.erase(it);
    restore_dropped();
}

pkv_status BlockManager::export_tables(const int64_t* seqs, int n, int max_blocks, int32_t* tables,
                                       int32_t* lens, int32_t* fills) const {
    if (n < 0 || max_blocks < 0 || (n > 0 && (!seqs || !lens || (max_blocks > 0 && !tables))))
        return PKV_ERR_INVALID_ARG;
    // validate everything first so that nothing is written on error
    for (int i = 0; i < n; ++i) {
        auto it = seqs_.find(seqs[i]);
        if (it == seqs_.end()) return PKV_ERR_UNKNOWN_SEQ;
        if ((int64_t)it->second.blocks.size() > max_blocks) return PKV_ERR_INVALID_ARG;
        if (it->second.length > std::numeric_limits<int32_t>::max()) return PKV_ERR_INVALID_ARG;
    }
    for (int i = 0; i < n; ++i) {
        const Sequence& s = seqs_.at(seqs[i]);
        int32_t* row = tables + (size_t)i * max_blocks;
        size_t nb = s.blocks.size();
        std::copy(s.blocks.begin(), s.blocks.end(), row);
        std::fill(row + nb, row + max_blocks, -1);
        lens[i] = (int32_t)s.length;
        if (fills) fills[i] = fill_of_last(s);
    }
    return PKV_OK;
}

pkv_status BlockManager::num_blocks_of(int64_t seq, int32_t* out) const {
    if (!out) return PKV_ERR_INVALID_ARG;
    auto it = seqs_.find(seq);
    if (it == seqs_.end()) return PKV_ERR_UNKNOWN_SEQ;
    *out = (int32_t)it->second.blocks.size();
    return PKV_OK;
}

pkv_status BlockManager::blocks_after_append(int64_t seq, int32_t* out) const {
    if (!out) return PKV_ERR_INVALID_ARG;
    auto it = seqs_.find(seq);
    if (it == seqs_.end()) return PKV_ERR_UNKNOWN_SEQ;
    const Sequence& s = it->second;
    const int nb = (int)s.blocks.size();
    *out = (nb == 0 || fill_of_last(s) == block_size_) ? nb + 1 : nb;
    return PKV_OK;
}

pkv_status BlockManager::refcount_of(int32_t block, int32_t* out) const {
    if (!out || block < 0 || block >= num_blocks_) return PKV_ERR_INVALID_ARG;
    *out = ref_[block];
    return PKV_OK;
}

pkv_status BlockManager::free_queue(int32_t* out, int cap, int* n_out) const {
    if (!n_out || cap < count_ || (count_ > 0 && !out)) return PKV_ERR_INVALID_ARG;
    int i = 0;
    for (int32_t b = head_; b >= 0; b = next_[b]) out[i++] = b;
    *n_out = count_;
    return PKV_OK;
}

void BlockManager::stats(pkv_stats* out) const {
    pkv_stats st{};
    st.num_blocks = num_blocks_;
    st.block_size = block_size_;
    st.free_blocks = count_;
    int used = 0;
    for (int32_t r : ref_) used += r > 0;
    st.used_blocks = used;
    st.num_seqs = (int32_t)seqs_.size();
    // every sequence that references a block agrees on its fill
    std::vector<int32_t> fill(num_blocks_, 0);
    for (const auto& kv : seqs_) {
        const Sequence& s = kv.second;
        size_t nb = s.blocks.size();
        for (size_t i = 0; i < nb; ++i)
            fill[s.blocks[i]] = (i + 1 < nb) ? block_size_ : fill_of_last(s);
        st.logical_tokens += s.length;
        st.table_slots += (int64_t)nb * block_size_;
    }
    for (int32_t f : fill) st.stored_slots += f;
    st.cow_count = cow_count_;
    st.prefix_hit_tokens = hit_tokens_;
    for (uint8_t h : hashed_) st.cached_blocks += h;
    *out = st;
}

}  // namespace pkv
