// Host-side block manager of the paged KV pool.
//
// Implements the block-table rules of "KV 缓存与分页注意力" §块表 (one table per
// sequence: physical block per logical block, fill count of the last block; a
// new block only when the last one is full; blocks returned when a sequence
// finishes), the copy-on-write rule of its FAQ 08 and of "读懂PagedAttention"
// §同一提示生成两个回答的假想例子 (a partially filled last block that is still
// shared is copied before the write; full shared blocks stay shared), with a
// FIFO free queue.  Optional automatic prefix caching ("KV 缓存与分页注意力"
// §后来的做法): a full prompt block is registered under a hash of its tokens and
// everything before it; a later prompt that starts with the same tokens takes
// the registered blocks instead of new ones.  A freed registered block stays
// registered (and in the free queue) until it is handed out again.
// Not thread-safe: calls on one pool must be serialised.
#pragma once

#include <cstdint>
#include <unordered_map>
#include <vector>

#include "pagedkv.h"

namespace pkv {

struct Sequence {
    std::vector<int32_t> blocks;  // logical block i -> physical block id
    int64_t length = 0;           // tokens stored (the fill count is derived)
    uint64_t epoch = 0;           // unique per admission / fork: between two appends
                                  // of the same epoch only the last entry changes
};

class BlockManager {
  public:
    BlockManager(int num_blocks, int block_size);

    pkv_status reset(const int32_t* free_order);
    pkv_status alloc(int64_t seq, int n_tokens, int32_t* slots);
    pkv_status append(int64_t seq, int32_t* slot, int32_t* cow_src, int32_t* cow_dst);
    pkv_status append_batch(const int64_t* seqs, int n, int32_t* slots, int32_t* cow_src,
                            int32_t* cow_dst, int* n_cow);
    // admission with prompt token ids: reuses registered blocks for the longest
    // run of matching full leading blocks (when prefix caching is on)
    pkv_status alloc_prefix(int64_t seq, const int32_t* tokens, int n_tokens, int32_t* slots,
                            int32_t* n_cached);
    void set_prefix_caching(bool on);
    pkv_status fork(int64_t parent, int64_t child);
    pkv_status release(int64_t seq);
    // undo the most recent alloc(seq): its blocks go back to the front of the
    // free queue in their original order (only valid right after that alloc)
    void undo_alloc(int64_t seq);
    pkv_status export_tables(const int64_t* seqs, int n, int max_blocks, int32_t* tables,
                             int32_t* lens, int32_t* fills) const;
    pkv_status num_blocks_of(int64_t seq, int32_t* out) const;
    // table length after one more append (the last block full -> one more)
    pkv_status blocks_after_append(int64_t seq, int32_t* out) const;
    pkv_status refcount_of(int32_t block, int32_t* out) const;
    pkv_status free_queue(int32_t* out, int cap, int* n_out) const;
    void stats(pkv_stats* out) const;
    const Sequence* find(int64_t seq) const {
        auto it = seqs_.find(seq);
        return it == seqs_.end() ? nullptr : &it->second;
    }

    int num_blocks() const { return num_blocks_; }
    int block_size() const { return block_size_; }

  private:
    // one undo record per successful append inside a batch
    struct Undo {
        int64_t seq;
        int kind;        // 0 = in place, 1 = fresh block pushed, 2 = copy-on-write
        int32_t old_block;
    };

    int fill_of_last(const Sequence& s) const;
    int32_t pop_front();
    void unpop_front(int32_t b);
    void push_back(int32_t b);
    void remove_free(int32_t b);
    void unregister(int32_t b);
    int32_t lookup(uint64_t hash, const int32_t* tokens) const;
    pkv_status append_one(int64_t seq, int32_t* slot, int32_t* src, int32_t* dst, Undo* undo);
    void undo_one(const Undo& u);

    int num_blocks_;
    int block_size_;
    // FIFO free queue as a doubly linked list over block ids (-1 = none)
    std::vector<int32_t> next_, prev_;
    int32_t head_ = -1, tail_ = -1;
    int count_ = 0;
    // prefix cache
    bool caching_ = false;
    std::vector<uint8_t> hashed_;          // block registered?
    std::vector<uint64_t> hash_;           // its chain hash
    std::vector<int32_t> block_tokens_;    // [num_blocks][block_size] token ids
    std::unordered_map<uint64_t, int32_t> by_hash_;
    int64_t hit_tokens_ = 0;
    // registrations dropped since the start of the current call, so that an
    // undone call can restore them
    std::vector<std::pair<int32_t, uint64_t>> dropped_;
    void restore_dropped();
    std::vector<int32_t> ref_;
    std::unordered_map<int64_t, Sequence> seqs_;
    int64_t cow_count_ = 0;
    uint64_t next_epoch_ = 1;
};

}  // namespace pkv
