// Host-side launchers of the decode-path kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "kernels_common.cuh"

namespace pkv {

// CUDA-core decode (any grouping, any storage type) + partition merge.
int simt_heads_per_cta(int group);
// mid (may be null) is recorded on st after the decode kernel, before the merge.
cudaError_t launch_decode_simt(const DecodeParams& p, int kv_dtype, int q_dtype, int head_dim,
                               int heads_per_cta, cudaStream_t st, cudaEvent_t mid = nullptr);

// Log-sum-exp merge of the partitions (a no-op grid when max_parts <= 1).
cudaError_t launch_merge(const DecodeParams& p, int q_dtype, int head_dim, cudaStream_t st);

}  // namespace pkv
struct pkv_pool;
namespace pkv {
// Tensor-core decode of grouped heads (F16/BF16 pools with TMA descriptors,
// 1 < G <= 128) + partition merge.
bool tensor_path_supported(const pkv_pool* pool, int q_dtype, int group);
bool pool_has_row_maps(const pkv_pool* pool);

// CUDA-core decode with swizzled TMA staging, one query head per CTA (pools
// with row tensor maps) + partition merge.
bool simt2_supported(const pkv_pool* pool, int group);
cudaError_t launch_decode_simt2(const DecodeParams& p, const void* tmap_k, const void* tmap_v,
                                int kv_dtype, int q_dtype, int head_dim, int bs_shift,
                                cudaStream_t st, cudaEvent_t mid = nullptr);
cudaError_t launch_decode_tensor(const DecodeParams& p, const void* tmap_k, const void* tmap_v,
                                 int kv_dtype, int head_dim, cudaStream_t st,
                                 cudaEvent_t mid = nullptr);

// Stage-balanced tensor-core decode (one persistent wave; a split pair merged
// in the kernel by the worker that finishes its last piece): F16/BF16 pools with row tensor
// maps, q in the pool dtype, head_dim 64/128, 1 <= G <= 128, B <= 2048.  The
// workspace holds the pieces' partial states; the per-pair merge counters are
// p.counters when given (zeroed once by the caller; every launch leaves them
// zero), else carved from the workspace and zeroed by a memset on st.  mid
// (may be null) is recorded after the launch.
bool lean_supported(const pkv_pool* pool, int q_dtype, int group, int B, int max_blocks);
size_t lean_workspace_bytes(const pkv_pool* pool, int B, int n_q_heads);
cudaError_t launch_decode_lean(DecodeParams p, const pkv_pool* pool, void* ws, cudaStream_t st,
                               cudaEvent_t mid = nullptr);

// Prompt-phase attention (F16/BF16 pools with row tensor maps, q in the pool
// dtype, head_dim 64/128).  Sequence i's queries are rows
// q_starts[i] .. q_starts[i+1]-1 of q/out ([rows][H_q][D]); they are the last
// n_i of its lens[i] cached tokens and attend causally.
struct PrefillParams {
    const void* q;
    void* out;
    const int32_t* q_starts;   // [B + 1]
    const int32_t* tables;     // [B][max_blocks]
    const int32_t* lens;       // [B]
    uint32_t* err;
    int B, H_q, H_kv, G;
    int max_blocks, block_size, num_blocks;
    int max_q_len;             // >= every n_i (sizes the grid)
    float q_scale;             // scale * log2(e)
    unsigned long long wait_ns;// budget of the main loops' waits (the pool's)
    // the tcgen05 kernel's work counters {next item, CTAs done}: zero at the
    // launch, zero again after it (its last CTA resets them)
    unsigned long long* sched;
};
bool prefill_supported(const pkv_pool* pool, int q_dtype);
// the mma.sync kernel (m16n8k16, register accumulators)
cudaError_t launch_prefill(const PrefillParams& p, const pkv_pool* pool, cudaStream_t st);
// the tcgen05 kernel (tensor-memory accumulators, persistent heaviest-first schedule)
cudaError_t launch_prefill_tc05(const PrefillParams& p, const pkv_pool* pool, cudaStream_t st);

// One decode round's small host-side results, passed by value as kernel
// parameters (no separate host-to-device copy):
//   data = slots[B] | lens[B] | rows[B] | order[B] | cow_src[n_cow]
//          | cow_dst[n_cow] | cow_rows[n_cow] | upd_idx[n_upd] | upd_val[n_upd]
// slots[i] = append slot of the caller's sequence i; lens, rows and order are
// by launch slot (longest context first): order[z] = the caller's index of
// launch slot z, rows[z] = its persistent table row; cow_rows[j] = rows of
// the shared block to copy (the fill before the write); upd_* = changed
// block-table entries (flat index into [table rows][max_blocks]).
constexpr int kStepArgInts = 990;   // the whole parameter block stays under 4 KB
struct StepArgs {
    int32_t B, n_cow, n_upd, table_cap;
    int32_t data[kStepArgInts];
};

// The round's prologue in one launch: lengths, rows and launch order by
// launch slot and table updates into the persistent device tables,
// copy-on-write of the shared rows, append of the B new rows (FP8 pools
// quantise).
cudaError_t launch_step_prologue(const StepArgs& a, uint8_t* k_pool, uint8_t* v_pool,
                                 const void* k, const void* v, int in_dtype, int kv_dtype,
                                 int32_t* tables, int32_t* lens, int32_t* rows, int32_t* order,
                                 int n_kv_heads, int head_dim, int block_size, int num_blocks,
                                 float k_scale, float v_scale, uint32_t* err, cudaStream_t st);

// Copy staged full tables ([B][max_blocks]) into their persistent rows.
cudaError_t launch_scatter_rows(const int32_t* staged, const int32_t* rows, int B, int max_blocks,
                                int32_t* tables, cudaStream_t st);

// Store new rows into their slots (FP8 pools quantise).
cudaError_t launch_kv_append(uint8_t* k_pool, uint8_t* v_pool, const int32_t* slots, int n_tokens,
                             const void* k, const void* v, int in_dtype, int kv_dtype,
                             int n_kv_heads, int head_dim, int block_size, int num_blocks,
                             float k_scale, float v_scale, uint32_t* err, cudaStream_t st);

// One CTA waiting, with budget_ns, on a barrier that nothing completes; sets
// PKV_DEVERR_TIMEOUT in *err when the wait gives up.
cudaError_t launch_wait_probe(uint32_t* err, unsigned long long budget_ns, cudaStream_t st);

// Whole-block copies src[i] -> dst[i] of K and V.
cudaError_t launch_block_copy(uint8_t* k_pool, uint8_t* v_pool, const int32_t* src,
                              const int32_t* dst, int n_pairs, long long block_bytes,
                              int num_blocks, uint32_t* err, cudaStream_t st);

}  // namespace pkv
