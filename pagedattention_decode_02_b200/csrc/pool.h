// The pool object behind the opaque pkv_pool handle.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>

#include "block_manager.h"
#include "pagedkv.h"

struct pkv_pool {
    pkv_pool(int num_blocks, int block_size) : bm(num_blocks, block_size) {}

    int num_blocks = 0;
    int block_size = 0;
    int n_kv_heads = 0;
    int head_dim = 0;
    pkv_dtype dtype = PKV_F32;
    float k_scale = 1.f;
    float v_scale = 1.f;
    bool host_only = false;
    bool owns_buffers = false;
    int device = -1;
    int sm_count = 0;       // streaming multiprocessors of `device` (0: unknown)
    uint8_t* k = nullptr;   // device [num_blocks][n_kv_heads][block_size][head_dim]
    uint8_t* v = nullptr;
    size_t bytes = 0;       // bytes of one of the two buffers
    // buffers the pool allocated itself: one guard block (rounded up to 256
    // bytes) before and after each, filled with kGuardByte and never written
    // by the library; k_alloc / v_alloc are the allocations (k = k_alloc + guard)
    static constexpr unsigned char kGuardByte = 0xA5;
    uint8_t* k_alloc = nullptr;
    uint8_t* v_alloc = nullptr;
    size_t guard = 0;
    uint32_t* d_err = nullptr;
    // work counters of the prompt kernel's dynamic schedule: kPrefillSlots
    // pairs {next item, CTAs done}, one pair per launch in flight (launch i
    // takes pair i % kPrefillSlots); each launch's last CTA zeroes its pair
    static constexpr int kPrefillSlots = 64;
    unsigned long long* d_sched = nullptr;
    std::atomic<unsigned> prefill_seq{0};
    // budget of the kernels' main-loop waits on a copy (pkv_set_wait_budget)
    unsigned long long wait_ns = 2000000000ull;
    pkv::BlockManager bm;
    // TMA descriptors of the K and V pools (CUtensorMap, 128 bytes each) for
    // the tensor-core decode path; valid when has_tmaps.
    alignas(64) unsigned char tmap_k[128] = {};
    alignas(64) unsigned char tmap_v[128] = {};
    bool has_tmaps = false;
};

namespace pkv {
// device-side extras set up after the buffers exist (tensor maps)
void pool_init_device_extras(pkv_pool* p);
// places the static decode scratch on `device` (the current device) and looks
// up its address; false if that failed
bool static_scratch_prepare(int device);
// automatic partition length (tokens) for this batch shape, and the workspace
// of the partitioned decode kernels for a partition request (0 = automatic),
// not counting the stage-balanced kernel's
int decode_auto_partition(const pkv_pool* pool, int B, int n_q_heads, int max_blocks);
size_t decode_workspace_bytes_partitioned(const pkv_pool* pool, int B, int n_q_heads,
                                          int max_blocks, int partition_tokens);
}  // namespace pkv
