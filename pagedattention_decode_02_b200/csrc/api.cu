// The C ABI declared in include/pagedkv.h: pool lifetime, block-table calls
// (forwarded to the host BlockManager), argument validation and kernel
// dispatch for the device calls.
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>
#include <limits>
#include <unordered_map>
#include <algorithm>

#include "block_manager.h"
#include "decode_launch.h"
#include "pagedkv.h"
#include "pool.h"
#include "trace.h"

using pkv::BlockManager;

namespace {

int elem_bytes(int dt) {
    switch (dt) {
        case PKV_F32: return 4;
        case PKV_F16: return 2;
        case PKV_BF16: return 2;
        case PKV_FP8_E4M3: return 1;
        default: return 0;
    }
}

bool valid_dtype(int dt) { return dt >= PKV_F32 && dt <= PKV_FP8_E4M3; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool same_device(const pkv_pool* pool) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    return dev == pool->device;
}

// Tokens per partition when the caller leaves it to the library.  Contexts up
// to kNoSplitTokens run as one partition per (sequence, head group); longer
// ones are cut into kAutoPartition-token partitions so that long and short
// sequences give CTAs of similar size and the grid fills all SMs.
constexpr int kNoSplitTokens = 512;
constexpr int kAutoPartition = 512;

// With G query heads per KV head, a partition's partial state is G * (d + 2)
// floats against partition * 2 * d * elem bytes of K/V, so the automatic
// partition grows with G; grouped heads take three times the one-head length
// per 8 heads (measured on the Llama-2-70B-shaped batch with equal-length
// partitions launched longest first: 1536 tokens 0.78 of the copy peak,
// against 0.72 for 1024 and 1280 and 0.70 for 2048).
//
// units: CTAs of the unsplit grid (0: unknown).  With at least two waves of
// them (three CTAs per SM) the batch alone fills the GPU and is not split:
// no partial states, no merge (measured on the OPT-13B-shaped batch, 1,200
// one-head CTAs: unsplit 0.97 of the copy peak against 0.92-0.93 for 512 to
// 1024-token partitions).
int pool_sms(const pkv_pool* pool) { return pool->sm_count > 0 ? pool->sm_count : 148; }

long long unsplit_units(const pkv_pool* pool, int B, int n_q_heads) {
    const int G = n_q_heads / pool->n_kv_heads;
    return (long long)B * (G <= 1 ? n_q_heads : (long long)pool->n_kv_heads * ((G + 7) / 8));
}

int resolve_partition(const pkv_pool* pool, int max_blocks, int requested, int group = 1,
                      long long units = 0) {
    const long long max_ctx = (long long)max_blocks * pool->block_size;
    const int whole = (int)(((max_ctx + 15) / 16) * 16);
    if (requested < 0) return whole < 16 ? 16 : whole;
    if (requested > 0) return requested;
    if (units > 0 && units >= 6LL * pool_sms(pool)) return whole < 16 ? 16 : whole;
    const long long auto_p =
        (long long)kAutoPartition * (group > 1 ? 3 : 1) * ((group + 7) / 8);
    if (max_ctx <= (group > 8 ? auto_p : kNoSplitTokens)) return whole < 16 ? 16 : whole;
    return (int)(auto_p < (1 << 30) ? auto_p : (1 << 30));
}

int parts_for(const pkv_pool* pool, int max_blocks, int part_tokens) {
    const long long max_ctx = (long long)max_blocks * pool->block_size;
    return (int)((max_ctx + part_tokens - 1) / part_tokens);
}

size_t workspace_for(const pkv_pool* pool, int B, int n_q_heads, int max_parts) {
    if (max_parts <= 1) return 0;
    const size_t rows = (size_t)B * n_q_heads * max_parts;
    const size_t ml = ((rows * 2 * sizeof(float)) + 255) & ~(size_t)255;
    return ml + rows * pool->head_dim * sizeof(float);
}

}  // namespace

namespace pkv {
// The automatic partition length and the workspace the partitioned kernels
// need for it, without the stage-balanced kernel's share (used by the
// no-allocation call to keep the library's own choice when only that share
// would not fit its scratch).
int decode_auto_partition(const pkv_pool* pool, int B, int n_q_heads, int max_blocks) {
    return resolve_partition(pool, max_blocks, 0, n_q_heads / pool->n_kv_heads,
                             unsplit_units(pool, B, n_q_heads));
}
size_t decode_workspace_bytes_partitioned(const pkv_pool* pool, int B, int n_q_heads,
                                          int max_blocks, int partition_tokens) {
    const int P = resolve_partition(pool, max_blocks, partition_tokens,
                                    n_q_heads / pool->n_kv_heads,
                                    unsplit_units(pool, B, n_q_heads));
    if (P <= 0 || P % 16) return 0;
    return workspace_for(pool, B, n_q_heads, parts_for(pool, max_blocks, P));
}
}  // namespace pkv

extern "C" {

const char* pkv_status_str(pkv_status s) {
    switch (s) {
        case PKV_OK: return "OK";
        case PKV_ERR_INVALID_ARG: return "INVALID_ARG";
        case PKV_ERR_NO_BLOCKS: return "NO_BLOCKS";
        case PKV_ERR_UNKNOWN_SEQ: return "UNKNOWN_SEQ";
        case PKV_ERR_SEQ_EXISTS: return "SEQ_EXISTS";
        case PKV_ERR_CUDA: return "CUDA";
        case PKV_ERR_DEVICE: return "DEVICE";
        case PKV_ERR_SCRATCH_LIMIT: return "SCRATCH_LIMIT";
        default: return "UNKNOWN_STATUS";
    }
}

pkv_status kv_pool_create(int num_blocks, int block_size, int n_kv_heads, int head_dim,
                          pkv_dtype dtype, float k_scale, float v_scale, void* k_buf, void* v_buf,
                          unsigned flags, size_t* bytes_needed_out, pkv_pool** out) {
    if (num_blocks < 1 || block_size < 1 || n_kv_heads < 1) return PKV_ERR_INVALID_ARG;
    if (head_dim != 32 && head_dim != 64 && head_dim != 128) return PKV_ERR_INVALID_ARG;
    if (!valid_dtype(dtype)) return PKV_ERR_INVALID_ARG;
    if ((flags & ~PKV_POOL_HOST_ONLY) != 0) return PKV_ERR_INVALID_ARG;
    if (dtype == PKV_FP8_E4M3 &&
        !(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f))
        return PKV_ERR_INVALID_ARG;
    // slots are int32: num_blocks * block_size must fit
    if ((long long)num_blocks * block_size > 0x7fffffffLL) return PKV_ERR_INVALID_ARG;
    const size_t bytes = (size_t)num_blocks * n_kv_heads * block_size * head_dim * elem_bytes(dtype);
    if (bytes_needed_out) *bytes_needed_out = bytes;
    if (!out) return PKV_OK;
    const bool host_only = flags & PKV_POOL_HOST_ONLY;
    if (!host_only && ((k_buf == nullptr) != (v_buf == nullptr))) return PKV_ERR_INVALID_ARG;
    if (!host_only && k_buf && (!aligned16(k_buf) || !aligned16(v_buf))) return PKV_ERR_INVALID_ARG;

    pkv_pool* p = new (std::nothrow) pkv_pool(num_blocks, block_size);
    if (!p) return PKV_ERR_INVALID_ARG;
    p->num_blocks = num_blocks;
    p->block_size = block_size;
    p->n_kv_heads = n_kv_heads;
    p->head_dim = head_dim;
    p->dtype = dtype;
    p->k_scale = dtype == PKV_FP8_E4M3 ? k_scale : 1.f;
    p->v_scale = dtype == PKV_FP8_E4M3 ? v_scale : 1.f;
    p->host_only = host_only;
    p->bytes = bytes;
    if (!host_only) {
        if (cudaGetDevice(&p->device) != cudaSuccess ||
            cudaDeviceGetAttribute(&p->sm_count, cudaDevAttrMultiProcessorCount, p->device) !=
                cudaSuccess) {
            delete p;
            return PKV_ERR_CUDA;
        }
        if (k_buf) {
            p->k = static_cast<uint8_t*>(k_buf);
            p->v = static_cast<uint8_t*>(v_buf);
            p->owns_buffers = false;
        } else {
            // each buffer between two guard blocks of a known byte
            const size_t g = ((bytes / num_blocks) + 255) & ~(size_t)255;
            if (cudaMalloc(&p->k_alloc, bytes + 2 * g) != cudaSuccess) {
                delete p;
                return PKV_ERR_CUDA;
            }
            if (cudaMalloc(&p->v_alloc, bytes + 2 * g) != cudaSuccess) {
                cudaFree(p->k_alloc);
                delete p;
                return PKV_ERR_CUDA;
            }
            p->guard = g;
            p->k = p->k_alloc + g;
            p->v = p->v_alloc + g;
            p->owns_buffers = true;
            if (cudaMemset(p->k_alloc, pkv_pool::kGuardByte, g) != cudaSuccess ||
                cudaMemset(p->k + bytes, pkv_pool::kGuardByte, g) != cudaSuccess ||
                cudaMemset(p->v_alloc, pkv_pool::kGuardByte, g) != cudaSuccess ||
                cudaMemset(p->v + bytes, pkv_pool::kGuardByte, g) != cudaSuccess) {
                cudaFree(p->k_alloc);
                cudaFree(p->v_alloc);
                delete p;
                return PKV_ERR_CUDA;
            }
        }
        // the error word, then (256 bytes in) the prompt kernel's counters
        constexpr size_t kSchedOff = 256;
        const size_t err_bytes = kSchedOff + 2 * sizeof(unsigned long long) * pkv_pool::kPrefillSlots;
        if (cudaMalloc(&p->d_err, err_bytes) != cudaSuccess ||
            cudaMemset(p->d_err, 0, err_bytes) != cudaSuccess) {
            if (p->owns_buffers) {
                cudaFree(p->k_alloc);
                cudaFree(p->v_alloc);
            }
            if (p->d_err) cudaFree(p->d_err);
            delete p;
            return PKV_ERR_CUDA;
        }
        p->d_sched = reinterpret_cast<unsigned long long*>(reinterpret_cast<uint8_t*>(p->d_err) +
                                                           kSchedOff);
        pkv::pool_init_device_extras(p);
        // the no-allocation decode call's scratch array: placed on this device
        // now, while allocating is allowed (a failure here is not fatal; that
        // call looks it up again and reports PKV_ERR_CUDA if it still fails)
        (void)pkv::static_scratch_prepare(p->device);
    }
    *out = p;
    return PKV_OK;
}

void kv_pool_destroy(pkv_pool* p) {
    if (!p) return;
    if (!p->host_only) {
        if (p->owns_buffers) {
            cudaFree(p->k_alloc);
            cudaFree(p->v_alloc);
        }
        cudaFree(p->d_err);
    }
    delete p;
}

pkv_status kv_pool_check_guards(const pkv_pool* p, int* intact) {
    if (!p || !intact) return PKV_ERR_INVALID_ARG;
    *intact = 1;
    if (p->host_only || !p->owns_buffers || p->guard == 0) return PKV_OK;
    if (!same_device(p)) return PKV_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return PKV_ERR_CUDA;
    std::vector<uint8_t> h(p->guard);
    const uint8_t* regions[4] = {p->k_alloc, p->k + p->bytes, p->v_alloc, p->v + p->bytes};
    for (const uint8_t* r : regions) {
        if (cudaMemcpy(h.data(), r, p->guard, cudaMemcpyDeviceToHost) != cudaSuccess)
            return PKV_ERR_CUDA;
        for (uint8_t b : h)
            if (b != pkv_pool::kGuardByte) {
                *intact = 0;
                return PKV_OK;
            }
    }
    return PKV_OK;
}

pkv_status kv_pool_get_info(const pkv_pool* p, pkv_pool_info* info) {
    if (!p || !info) return PKV_ERR_INVALID_ARG;
    info->num_blocks = p->num_blocks;
    info->block_size = p->block_size;
    info->n_kv_heads = p->n_kv_heads;
    info->head_dim = p->head_dim;
    info->dtype = p->dtype;
    info->host_only = p->host_only;
    info->k_scale = p->k_scale;
    info->v_scale = p->v_scale;
    info->k_buf = p->k;
    info->v_buf = p->v;
    info->bytes_per_buffer = p->bytes;
    info->error_word = p->d_err;
    return PKV_OK;
}

// ---------------------------------------------------------------------------
// block tables
// ---------------------------------------------------------------------------
pkv_status bt_reset(pkv_pool* p, const int32_t* order) {
    if (!p) return PKV_ERR_INVALID_ARG;
    return p->bm.reset(order);
}
pkv_status bt_alloc(pkv_pool* p, int64_t seq, int n_tokens, int32_t* slots) {
    if (!p) return PKV_ERR_INVALID_ARG;
    return p->bm.alloc(seq, n_tokens, slots);
}
pkv_status bt_append(pkv_pool* p, int64_t seq, int32_t* slot, int32_t* src, int32_t* dst) {
    if (!p) return PKV_ERR_INVALID_ARG;
    return p->bm.append(seq, slot, src, dst);
}
pkv_status bt_append_batch(pkv_pool* p, const int64_t* seqs, int n, int32_t* slots, int32_t* src,
                           int32_t* dst, int* n_cow) {
    if (!p) return PKV_ERR_INVALID_ARG;
    return p->bm.append_batch(seqs, n, slots, src, dst, n_cow);
}
pkv_status bt_set_prefix_caching(pkv_pool* p, int enable) {
    if (!p || (enable != 0 && enable != 1)) return PKV_ERR_INVALID_ARG;
    p->bm.set_prefix_caching(enable != 0);
    return PKV_OK;
}
pkv_status bt_alloc_prefix(pkv_pool* p, int64_t seq, const int32_t* tokens, int n_tokens,
                           int32_t* slots, int32_t* n_cached) {
    if (!p) return PKV_ERR_INVALID_ARG;
    return p->bm.alloc_prefix(seq, tokens, n_tokens, slots, n_cached);
}
pkv_status bt_fork(pkv_pool* p, int64_t parent, int64_t child) {
    if (!p) return PKV_ERR_INVALID_ARG;
    return p->bm.fork(parent, child);
}
pkv_status bt_free(pkv_pool* p, int64_t seq) {
    if (!p) return PKV_ERR_INVALID_ARG;
    return p->bm.release(seq);
}
pkv_status bt_export(pkv_pool* p, const int64_t* seqs, int n, int max_blocks, int32_t* tables,
                     int32_t* lens, int32_t* fills) {
    if (!p) return PKV_ERR_INVALID_ARG;
    return p->bm.export_tables(seqs, n, max_blocks, tables, lens, fills);
}
pkv_status bt_num_blocks(const pkv_pool* p, int64_t seq, int32_t* n) {
    if (!p) return PKV_ERR_INVALID_ARG;
    return p->bm.num_blocks_of(seq, n);
}
pkv_status bt_refcount(const pkv_pool* p, int32_t block, int32_t* r) {
    if (!p) return PKV_ERR_INVALID_ARG;
    return p->bm.refcount_of(block, r);
}
pkv_status bt_free_queue(const pkv_pool* p, int32_t* out, int cap, int* n) {
    if (!p) return PKV_ERR_INVALID_ARG;
    return p->bm.free_queue(out, cap, n);
}
pkv_status bt_stats(const pkv_pool* p, pkv_stats* out) {
    if (!p || !out) return PKV_ERR_INVALID_ARG;
    p->bm.stats(out);
    return PKV_OK;
}

// ---------------------------------------------------------------------------
// device calls
// ---------------------------------------------------------------------------
pkv_status kv_append(pkv_pool* p, const int32_t* slots, int n_tokens, const void* k, const void* v,
                     pkv_dtype in_dtype, void* stream) {
    PKV_TRACE("kv_append");
    if (!p || p->host_only || n_tokens < 0) return PKV_ERR_INVALID_ARG;
    if (!valid_dtype(in_dtype)) return PKV_ERR_INVALID_ARG;
    if (p->dtype == PKV_FP8_E4M3 ? in_dtype == PKV_FP8_E4M3 : in_dtype != p->dtype)
        return PKV_ERR_INVALID_ARG;
    if (n_tokens == 0) return PKV_OK;
    if (!slots || !k || !v || !aligned16(k) || !aligned16(v)) return PKV_ERR_INVALID_ARG;
    if (!same_device(p)) return PKV_ERR_INVALID_ARG;
    cudaError_t e = pkv::launch_kv_append(p->k, p->v, slots, n_tokens, k, v, in_dtype, p->dtype,
                                          p->n_kv_heads, p->head_dim, p->block_size, p->num_blocks,
                                          p->k_scale, p->v_scale, p->d_err,
                                          static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status block_copy(pkv_pool* p, const int32_t* src, const int32_t* dst, int n_pairs,
                      void* stream) {
    PKV_TRACE("block_copy");
    if (!p || p->host_only || n_pairs < 0) return PKV_ERR_INVALID_ARG;
    if (n_pairs == 0) return PKV_OK;
    if (!src || !dst) return PKV_ERR_INVALID_ARG;
    if (!same_device(p)) return PKV_ERR_INVALID_ARG;
    const long long block_bytes = (long long)p->n_kv_heads * p->block_size * p->head_dim *
                                  elem_bytes(p->dtype);
    cudaError_t e = pkv::launch_block_copy(p->k, p->v, src, dst, n_pairs, block_bytes,
                                           p->num_blocks, p->d_err,
                                           static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

size_t paged_decode_workspace_bytes_ex(const pkv_pool* p, int B, int n_q_heads, int max_blocks,
                                       int partition_tokens) {
    if (!p || B <= 0 || n_q_heads <= 0 || max_blocks <= 0) return 0;
    const int P = resolve_partition(p, max_blocks, partition_tokens, n_q_heads / p->n_kv_heads,
                                    unsplit_units(p, B, n_q_heads));
    if (P <= 0 || P % 16) return 0;
    const size_t part = workspace_for(p, B, n_q_heads, parts_for(p, max_blocks, P));
    // the automatic choice may take the stage-balanced kernel: room for it too
    if (partition_tokens == 0 && !p->host_only && n_q_heads % p->n_kv_heads == 0 &&
        pkv::lean_supported(p, p->dtype, n_q_heads / p->n_kv_heads, B, max_blocks))
        return std::max(part, pkv::lean_workspace_bytes(p, B, n_q_heads));
    return part;
}

size_t paged_decode_workspace_bytes(const pkv_pool* p, int B, int n_q_heads, int max_blocks) {
    return paged_decode_workspace_bytes_ex(p, B, n_q_heads, max_blocks, 0);
}

}  // extern "C"

namespace {
// paged_decode_attention_ex with optional events recorded on the stream right
// before the decode kernel (ev_begin), between it and the merge (ev_mid) and
// after the last launch (ev_end).
pkv_status decode_attention_impl(pkv_pool* p, const void* q, pkv_dtype q_dtype,
                                 const int32_t* tables, int max_blocks, const int32_t* lens, int B,
                                 int n_q_heads, float scale, void* out, void* ws, size_t ws_bytes,
                                 int partition_tokens, int kernel, void* stream,
                                 cudaEvent_t ev_begin, cudaEvent_t ev_mid, cudaEvent_t ev_end,
                                 int* counters = nullptr, bool pdl = false,
                                 const int32_t* table_rows = nullptr, int n_table_rows = 0,
                                 int* n_launches = nullptr, int* kernel_used = nullptr,
                                 const int32_t* order = nullptr,
                                 const pkv::StepPrefetch* pre = nullptr) {
    if (n_launches) *n_launches = 0;
    if (kernel_used) *kernel_used = 0;
    if (!p || p->host_only || B < 0) return PKV_ERR_INVALID_ARG;
    if (B == 0) return PKV_OK;
    if (!q || !out || !tables || !lens || max_blocks < 1) return PKV_ERR_INVALID_ARG;
    if (n_q_heads < p->n_kv_heads || n_q_heads % p->n_kv_heads) return PKV_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PKV_ERR_INVALID_ARG;
    if (p->dtype == PKV_FP8_E4M3) {
        if (q_dtype != PKV_F16 && q_dtype != PKV_BF16) return PKV_ERR_INVALID_ARG;
    } else if (q_dtype != p->dtype) {
        return PKV_ERR_INVALID_ARG;
    }
    if (partition_tokens != 0 && partition_tokens != -1 &&
        (partition_tokens < 16 || partition_tokens % 16))
        return PKV_ERR_INVALID_ARG;
    if (kernel < PKV_KERNEL_AUTO || kernel > PKV_KERNEL_LEAN) return PKV_ERR_INVALID_ARG;
    if ((long long)max_blocks * p->block_size > 0x7fffffffLL) return PKV_ERR_INVALID_ARG;
    if (!same_device(p)) return PKV_ERR_INVALID_ARG;

    const int G = n_q_heads / p->n_kv_heads;
    const bool lean_ok = pkv::lean_supported(p, q_dtype, G, B, max_blocks);
    const size_t lean_need = lean_ok ? pkv::lean_workspace_bytes(p, B, n_q_heads) : 0;
    const bool lean_fits = lean_ok && ws && ws_bytes >= lean_need && aligned16(ws);
    const bool tc_ok = pkv::tensor_path_supported(p, q_dtype, G);
    const bool s2_ok = pkv::simt2_supported(p, G);
    int use = kernel;
    // automatic: large groups (one KV head shared by many query heads, a
    // small latency-bound batch) take the stage-balanced kernel; up to 16
    // heads per KV head the partitioned tensor-core kernel measured faster,
    // and FP8 pools take it from one head per KV head (the CUDA-core kernel
    // is issue-bound on the conversions), except with one token per block,
    // where its 16 one-row boxes per stage made it slower (OPT-13B-shaped
    // FP8 batch: 0.28 of the copy peak against 0.40 on the CUDA cores).
    const bool tc_auto =
        tc_ok && !(p->dtype == PKV_FP8_E4M3 && G == 1 && p->block_size == 1);
    if (use == PKV_KERNEL_AUTO)
        use = (lean_fits && G > 16 && partition_tokens == 0)
                  ? PKV_KERNEL_LEAN
                  : (tc_auto ? PKV_KERNEL_TENSOR : PKV_KERNEL_SIMT);
    if (use == PKV_KERNEL_SIMT) use = s2_ok ? PKV_KERNEL_SIMT_TMA : PKV_KERNEL_SIMT_BULK;
    if (use == PKV_KERNEL_TENSOR && !tc_ok) return PKV_ERR_INVALID_ARG;
    if (use == PKV_KERNEL_SIMT_TMA && !s2_ok) return PKV_ERR_INVALID_ARG;
    if (use == PKV_KERNEL_LEAN && !lean_fits) return PKV_ERR_INVALID_ARG;

    const int P = resolve_partition(p, max_blocks, partition_tokens, G, unsplit_units(p, B, n_q_heads));
    const int max_parts = use == PKV_KERNEL_LEAN ? 1 : parts_for(p, max_blocks, P);
    const size_t need = workspace_for(p, B, n_q_heads, max_parts);
    if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return PKV_ERR_INVALID_ARG;
    if ((long long)max_parts > 0x7fffffffLL || B > 65535) return PKV_ERR_INVALID_ARG;

    pkv::DecodeParams dp{};
    dp.q = q;
    dp.out = out;
    dp.k_pool = p->k;
    dp.v_pool = p->v;
    dp.tables = tables;
    dp.lens = lens;
    dp.err = p->d_err;
    dp.B = B;
    dp.H_q = n_q_heads;
    dp.H_kv = p->n_kv_heads;
    dp.G = G;
    dp.max_blocks = max_blocks;
    dp.block_size = p->block_size;
    dp.num_blocks = p->num_blocks;
    dp.part_tokens = P;
    dp.max_parts = max_parts;
    const size_t rows = (size_t)B * n_q_heads * max_parts;
    dp.ws_ml = need ? static_cast<float*>(ws) : nullptr;
    dp.ws_acc = need ? reinterpret_cast<float*>(static_cast<uint8_t*>(ws) +
                                                ((rows * 2 * sizeof(float) + 255) & ~(size_t)255))
                     : nullptr;
    // the tensor-core kernel merges a split KV head's G query heads in the CTA
    // that finishes last (one handshake per G heads); the one-head CUDA-core
    // kernels leave it to the merge kernel, launched right behind them
    dp.counters = (need && use == PKV_KERNEL_TENSOR) ? counters : nullptr;
    dp.pdl = pdl ? 1 : 0;
    dp.table_rows = table_rows;
    dp.n_table_rows = n_table_rows;
    dp.order = order;
    dp.pre = pre;
    const float log2e = 1.4426950408889634f;
    dp.q_scale = scale * log2e * p->k_scale;
    dp.v_scale = p->v_scale;
    dp.head_stride = (long long)p->block_size * p->head_dim * elem_bytes(p->dtype);
    dp.block_stride = dp.head_stride * p->n_kv_heads;
    dp.wait_ns = p->wait_ns;

    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = ev_begin ? cudaEventRecord(ev_begin, st) : cudaSuccess;
    if (e != cudaSuccess) return PKV_ERR_CUDA;
    if (use == PKV_KERNEL_LEAN) {
        dp.counters = counters;
        dp.max_parts = 1;
        e = pkv::launch_decode_lean(dp, p, ws, st, ev_mid);
        if (n_launches) *n_launches = 1 + (counters ? 0 : 1);   // + the counter memset
    } else if (use == PKV_KERNEL_TENSOR) {
        e = pkv::launch_decode_tensor(dp, p->tmap_k, p->tmap_v, p->dtype, p->head_dim, st, ev_mid);
    } else if (use == PKV_KERNEL_SIMT_TMA) {
        e = pkv::launch_decode_simt2(dp, p->tmap_k, p->tmap_v, p->dtype, q_dtype, p->head_dim,
                                     __builtin_ctz((unsigned)p->block_size), st, ev_mid);
    } else {
        e = pkv::launch_decode_simt(dp, p->dtype, q_dtype, p->head_dim, pkv::simt_heads_per_cta(G),
                                    st, ev_mid);
    }
    if (kernel_used) *kernel_used = use;
    if (use != PKV_KERNEL_LEAN && n_launches)
        *n_launches = 1 + (max_parts > 1 && !(use == PKV_KERNEL_TENSOR && counters) ? 1 : 0);
    if (e == cudaSuccess && ev_end) e = cudaEventRecord(ev_end, st);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
}  // namespace

extern "C" {

pkv_status paged_decode_attention_ex(pkv_pool* p, const void* q, pkv_dtype q_dtype,
                                     const int32_t* tables, int max_blocks, const int32_t* lens,
                                     int B, int n_q_heads, float scale, void* out, void* ws,
                                     size_t ws_bytes, int partition_tokens, int kernel,
                                     void* stream) {
    PKV_TRACE("paged_decode_attention_ex");
    return decode_attention_impl(p, q, q_dtype, tables, max_blocks, lens, B, n_q_heads, scale, out,
                                 ws, ws_bytes, partition_tokens, kernel, stream, nullptr, nullptr,
                                 nullptr);
}

pkv_status paged_decode_attention(pkv_pool* p, const void* q, pkv_dtype q_dtype,
                                  const int32_t* tables, int max_blocks, const int32_t* lens, int B,
                                  int n_q_heads, float scale, void* out, void* ws, size_t ws_bytes,
                                  void* stream) {
    return paged_decode_attention_ex(p, q, q_dtype, tables, max_blocks, lens, B, n_q_heads, scale,
                                     out, ws, ws_bytes, 0, PKV_KERNEL_AUTO, stream);
}

pkv_status paged_prefill_attention_ex(pkv_pool* p, const void* q, pkv_dtype q_dtype,
                                      const int32_t* q_starts, int max_q_len,
                                      const int32_t* tables, int max_blocks, const int32_t* lens,
                                      int B, int n_q_heads, float scale, void* out, int kernel,
                                      void* stream) {
    PKV_TRACE("paged_prefill_attention_ex");
    if (!p || p->host_only || B < 0 || max_q_len < 0) return PKV_ERR_INVALID_ARG;
    if (kernel < PKV_PREFILL_AUTO || kernel > PKV_PREFILL_MMA_SYNC) return PKV_ERR_INVALID_ARG;
    if (B == 0 || max_q_len == 0) return PKV_OK;
    if (!q || !out || !q_starts || !tables || !lens || max_blocks < 1) return PKV_ERR_INVALID_ARG;
    if (n_q_heads < p->n_kv_heads || n_q_heads % p->n_kv_heads) return PKV_ERR_INVALID_ARG;
    if (!std::isfinite(scale) || B > 65535 || p->n_kv_heads > 65535) return PKV_ERR_INVALID_ARG;
    if ((long long)max_blocks * p->block_size > 0x7fffffffLL) return PKV_ERR_INVALID_ARG;
    if ((long long)max_q_len * (n_q_heads / p->n_kv_heads) > 0x7fffffffLL) return PKV_ERR_INVALID_ARG;
    if (!pkv::prefill_supported(p, q_dtype)) return PKV_ERR_INVALID_ARG;
    if (!same_device(p)) return PKV_ERR_INVALID_ARG;
    pkv::PrefillParams pp{};
    pp.q = q;
    pp.out = out;
    pp.q_starts = q_starts;
    pp.tables = tables;
    pp.lens = lens;
    pp.err = p->d_err;
    pp.B = B;
    pp.H_q = n_q_heads;
    pp.H_kv = p->n_kv_heads;
    pp.G = n_q_heads / p->n_kv_heads;
    pp.max_blocks = max_blocks;
    pp.block_size = p->block_size;
    pp.num_blocks = p->num_blocks;
    pp.max_q_len = max_q_len;
    pp.q_scale = scale * 1.4426950408889634f;
    pp.wait_ns = p->wait_ns;
    pp.sched = p->d_sched + 2 * (p->prefill_seq.fetch_add(1) % pkv_pool::kPrefillSlots);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const cudaError_t e = kernel == PKV_PREFILL_MMA_SYNC ? pkv::launch_prefill(pp, p, st)
                                                         : pkv::launch_prefill_tc05(pp, p, st);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status paged_prefill_attention(pkv_pool* p, const void* q, pkv_dtype q_dtype,
                                   const int32_t* q_starts, int max_q_len, const int32_t* tables,
                                   int max_blocks, const int32_t* lens, int B, int n_q_heads,
                                   float scale, void* out, void* stream) {
    return paged_prefill_attention_ex(p, q, q_dtype, q_starts, max_q_len, tables, max_blocks, lens,
                                      B, n_q_heads, scale, out, PKV_PREFILL_AUTO, stream);
}

pkv_status pkv_set_wait_budget(pkv_pool* p, uint64_t budget_ns) {
    if (!p || budget_ns > pkv::kWaitBudgetNs) return PKV_ERR_INVALID_ARG;
    p->wait_ns = budget_ns == 0 ? pkv::kWaitBudgetNs : budget_ns;
    return PKV_OK;
}

pkv_status pkv_wait_probe(pkv_pool* p, void* stream) {
    PKV_TRACE("pkv_wait_probe");
    if (!p || p->host_only || !same_device(p)) return PKV_ERR_INVALID_ARG;
    return pkv::launch_wait_probe(p->d_err, p->wait_ns, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? PKV_OK
               : PKV_ERR_CUDA;
}

pkv_status pkv_device_error(pkv_pool* p, void* stream, uint32_t* bits_out) {
    if (!p || p->host_only) return PKV_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t bits = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess) return PKV_ERR_CUDA;
    if (cudaMemcpy(&bits, p->d_err, sizeof(bits), cudaMemcpyDeviceToHost) != cudaSuccess)
        return PKV_ERR_CUDA;
    if (bits && cudaMemset(p->d_err, 0, sizeof(uint32_t)) != cudaSuccess) return PKV_ERR_CUDA;
    if (bits_out) *bits_out = bits;
    return bits ? PKV_ERR_DEVICE : PKV_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// decode-step runtime
// ---------------------------------------------------------------------------
struct pkv_step {
    static constexpr int kRing = 3;   // pinned staging slots in flight
    pkv_pool* pool = nullptr;
    int max_batch = 0, max_seqs = 0, max_blocks = 0, n_q_heads = 0;
    pkv_dtype q_dtype = PKV_F16;
    int partition_tokens = 0, kernel = PKV_KERNEL_AUTO;
    // device: slots | cow src | cow dst | lens | rows | order  (max_batch each)
    //         | staged tables [max_batch][max_blocks]  (fallback path)
    int32_t* h_stage[kRing] = {};
    cudaEvent_t ev[kRing] = {};
    bool pending[kRing] = {};
    int ring = 0;
    int32_t* d_stage = nullptr;
    int32_t* d_tables = nullptr;      // persistent [max_seqs][max_blocks], one row per sequence
    void* d_ws = nullptr;
    size_t ws_bytes = 0;
    int* d_counters = nullptr;        // [max_batch][n_q_heads], zero between launches
    uint8_t* d_io = nullptr;          // pkv_decode_step_host: q | k | v | out, made on first use
    int max_parts = 1;
    int last_launches = 0;
    int last_kernel = 0;              // decode kernel of the last round (after the auto choice)
    // host mirror of the persistent rows
    std::vector<int64_t> row_seq;     // sequence held, or INT64_MIN
    std::vector<uint64_t> row_epoch;
    std::vector<int32_t> row_nb;      // entries the device row holds
    std::vector<long long> row_used;  // last round that used the row
    std::unordered_map<int64_t, int> row_of;
    std::vector<int32_t> mirror;      // [max_seqs][max_blocks]
    // one round's host scratch
    std::vector<int32_t> h_slots, h_src, h_dst, h_rows, h_cow_rows, h_upd_idx, h_upd_val;
    std::vector<int32_t> h_lens, h_order, h_key;   // fast path: lengths, launch order, sort key
    std::vector<int32_t> h_stable;    // fast path: leading row entries the prologue keeps
    pkv::StepArgs args;
    pkv::StepPrefetch pre{};          // fast path: per launch slot, for the decode kernel
    long long fast_rounds = 0, slow_rounds = 0;
    // profiling: every prof_every-th round records four events (before the
    // prologue, before the decode kernel, between it and the merge, after the
    // merge) into a ring of prof_n entries
    int prof_n = 0;
    int prof_every = 1;
    long long prof_count = 0;
    long long round = 0;              // rounds run (row recency)
    long long prof_start = 0;         // round count when profiling was (re)armed
    cudaEvent_t* prof_ev = nullptr;
};

namespace {
void prof_free(pkv_step* s) {
    if (s->prof_ev) {
        for (int i = 0; i < 4 * s->prof_n; ++i)
            if (s->prof_ev[i]) cudaEventDestroy(s->prof_ev[i]);
        delete[] s->prof_ev;
    }
    s->prof_ev = nullptr;
    s->prof_n = 0;
    s->prof_count = 0;
}

void step_free(pkv_step* s) {
    prof_free(s);
    for (int i = 0; i < pkv_step::kRing; ++i) {
        if (s->ev[i]) {
            cudaEventSynchronize(s->ev[i]);
            cudaEventDestroy(s->ev[i]);
        }
        if (s->h_stage[i]) cudaFreeHost(s->h_stage[i]);
    }
    if (s->d_stage) cudaFree(s->d_stage);
    if (s->d_tables) cudaFree(s->d_tables);
    if (s->d_ws) cudaFree(s->d_ws);
    if (s->d_counters) cudaFree(s->d_counters);
    if (s->d_io) cudaFree(s->d_io);
    delete s;
}

// Persistent table row of `seq` for this round: its own row if it has one,
// else a free row or the least recently used row no sequence of this round
// holds (max_seqs >= max_batch guarantees one).  A new or evicted row holds
// nothing (nb = 0), so the whole table is sent.
int row_for(pkv_step* s, int64_t seq) {
    auto it = s->row_of.find(seq);
    int r = -1;
    if (it != s->row_of.end()) {
        r = it->second;
    } else {
        long long oldest = std::numeric_limits<long long>::max();
        for (int i = 0; i < s->max_seqs; ++i) {
            if (s->row_seq[i] == std::numeric_limits<int64_t>::min()) {
                r = i;
                break;
            }
            if (s->row_used[i] < s->round && s->row_used[i] < oldest) {
                oldest = s->row_used[i];
                r = i;
            }
        }
        if (r < 0) return -1;
        if (s->row_seq[r] != std::numeric_limits<int64_t>::min()) s->row_of.erase(s->row_seq[r]);
        s->row_seq[r] = seq;
        s->row_epoch[r] = 0;
        s->row_nb[r] = 0;
        s->row_of[seq] = r;
    }
    s->row_used[r] = s->round;
    return r;
}
}  // namespace

extern "C" {

pkv_status pkv_step_create(pkv_pool* pool, int max_batch, int max_seqs, int max_blocks,
                           int n_q_heads, pkv_dtype q_dtype, int partition_tokens, int kernel,
                           pkv_step** out) {
    if (!pool || pool->host_only || !out || max_batch < 1 || max_batch > 65535 || max_blocks < 1)
        return PKV_ERR_INVALID_ARG;
    if (max_seqs < max_batch || (long long)max_seqs * max_blocks > (1LL << 31) - 1)
        return PKV_ERR_INVALID_ARG;
    if (n_q_heads < pool->n_kv_heads || n_q_heads % pool->n_kv_heads) return PKV_ERR_INVALID_ARG;
    if (pool->dtype == PKV_FP8_E4M3 ? (q_dtype != PKV_F16 && q_dtype != PKV_BF16)
                                    : q_dtype != pool->dtype)
        return PKV_ERR_INVALID_ARG;
    if (partition_tokens != 0 && partition_tokens != -1 &&
        (partition_tokens < 16 || partition_tokens % 16))
        return PKV_ERR_INVALID_ARG;
    if (kernel < PKV_KERNEL_AUTO || kernel > PKV_KERNEL_LEAN) return PKV_ERR_INVALID_ARG;
    if (!same_device(pool)) return PKV_ERR_INVALID_ARG;
    pkv_step* s = new (std::nothrow) pkv_step();
    if (!s) return PKV_ERR_INVALID_ARG;
    s->pool = pool;
    s->max_batch = max_batch;
    s->max_seqs = max_seqs;
    s->max_blocks = max_blocks;
    s->n_q_heads = n_q_heads;
    s->q_dtype = q_dtype;
    s->partition_tokens = partition_tokens;
    s->kernel = kernel;
    const size_t stage_ints = (size_t)6 * max_batch + (size_t)max_batch * max_blocks;
    bool ok = true;
    for (int i = 0; i < pkv_step::kRing && ok; ++i) {
        ok &= cudaMallocHost(&s->h_stage[i], stage_ints * sizeof(int32_t)) == cudaSuccess;
        ok &= ok && cudaEventCreateWithFlags(&s->ev[i], cudaEventDisableTiming) == cudaSuccess;
    }
    ok &= ok && cudaMalloc(&s->d_stage, stage_ints * sizeof(int32_t)) == cudaSuccess;
    ok &= ok && cudaMalloc(&s->d_tables, (size_t)max_seqs * max_blocks * sizeof(int32_t)) ==
                    cudaSuccess;
    s->row_seq.assign(max_seqs, std::numeric_limits<int64_t>::min());
    s->row_epoch.assign(max_seqs, 0);
    s->row_nb.assign(max_seqs, 0);
    s->row_used.assign(max_seqs, -1);
    s->mirror.assign((size_t)max_seqs * max_blocks, -1);
    const int P = resolve_partition(pool, max_blocks, partition_tokens,
                                    n_q_heads / pool->n_kv_heads);
    s->max_parts = parts_for(pool, max_blocks, P);
    s->ws_bytes = workspace_for(pool, max_batch, n_q_heads, s->max_parts);
    if ((kernel == PKV_KERNEL_AUTO || kernel == PKV_KERNEL_LEAN) &&
        pkv::lean_supported(pool, q_dtype, n_q_heads / pool->n_kv_heads, max_batch, max_blocks))
        s->ws_bytes = std::max(s->ws_bytes, pkv::lean_workspace_bytes(pool, max_batch, n_q_heads));
    if (ok && s->ws_bytes) ok &= cudaMalloc(&s->d_ws, s->ws_bytes) == cudaSuccess;
    if (ok && s->ws_bytes) {
        const size_t cb = (size_t)max_batch * n_q_heads * sizeof(int);
        ok &= cudaMalloc(&s->d_counters, cb) == cudaSuccess;
        ok &= ok && cudaMemset(s->d_counters, 0, cb) == cudaSuccess;
    }
    if (!ok) {
        step_free(s);
        return PKV_ERR_CUDA;
    }
    *out = s;
    return PKV_OK;
}

void pkv_step_destroy(pkv_step* s) {
    if (s) step_free(s);
}

pkv_status pkv_decode_step_host(pkv_step* s, const int64_t* seq_ids, int B, const void* h_q,
                                const void* h_k_new, const void* h_v_new, float scale,
                                void* h_out, void* stream) {
    PKV_TRACE("pkv_decode_step_host");
    if (!s || B < 0 || B > s->max_batch) return PKV_ERR_INVALID_ARG;
    if (B == 0) {
        s->last_launches = 0;
        s->last_kernel = 0;
        return PKV_OK;
    }
    if (!seq_ids || !h_q || !h_k_new || !h_v_new || !h_out) return PKV_ERR_INVALID_ARG;
    pkv_pool* pool = s->pool;
    if (!same_device(pool)) return PKV_ERR_INVALID_ARG;
    const size_t elem = s->q_dtype == PKV_F32 ? 4 : 2;
    const size_t q_row = (size_t)s->n_q_heads * pool->head_dim * elem;
    const size_t kv_row = (size_t)pool->n_kv_heads * pool->head_dim * elem;
    auto up16 = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t q_cap = up16(q_row * s->max_batch), kv_cap = up16(kv_row * s->max_batch);
    if (!s->d_io && cudaMalloc(&s->d_io, 2 * q_cap + 2 * kv_cap) != cudaSuccess) {
        s->d_io = nullptr;
        return PKV_ERR_CUDA;
    }
    // q | k | v back to back on the device (rows are multiples of 16 bytes), so
    // that a caller's packed host buffer travels in one copy
    uint8_t* d_q = s->d_io;
    uint8_t* d_k = d_q + q_row * B;
    uint8_t* d_v = d_k + kv_row * B;
    uint8_t* d_out = s->d_io + q_cap + 2 * kv_cap;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const uint8_t* hq8 = static_cast<const uint8_t*>(h_q);
    const bool packed = static_cast<const uint8_t*>(h_k_new) == hq8 + q_row * B &&
                        static_cast<const uint8_t*>(h_v_new) == hq8 + q_row * B + kv_row * B;
    // on any failure, wait for copies already queued: they read or write the
    // caller's buffers, which the caller may release once the call returns
    auto fail = [&](pkv_status e) {
        cudaStreamSynchronize(st);
        return e;
    };
    if (packed) {
        if (cudaMemcpyAsync(d_q, h_q, (q_row + 2 * kv_row) * B, cudaMemcpyHostToDevice, st) !=
            cudaSuccess)
            return fail(PKV_ERR_CUDA);
    } else if (cudaMemcpyAsync(d_q, h_q, q_row * B, cudaMemcpyHostToDevice, st) != cudaSuccess ||
               cudaMemcpyAsync(d_k, h_k_new, kv_row * B, cudaMemcpyHostToDevice, st) !=
                   cudaSuccess ||
               cudaMemcpyAsync(d_v, h_v_new, kv_row * B, cudaMemcpyHostToDevice, st) !=
                   cudaSuccess) {
        return fail(PKV_ERR_CUDA);
    }
    const pkv_status ps = pkv_decode_step(s, seq_ids, B, d_q, d_k, d_v, scale, d_out, stream);
    if (ps != PKV_OK) return fail(ps);
    if (cudaMemcpyAsync(h_out, d_out, q_row * B, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return fail(PKV_ERR_CUDA);
    return cudaStreamSynchronize(st) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

int pkv_step_last_launches(const pkv_step* s) { return s ? s->last_launches : 0; }

int pkv_step_last_kernel(const pkv_step* s) { return s ? s->last_kernel : 0; }

pkv_status pkv_decode_step(pkv_step* s, const int64_t* seq_ids, int B, const void* q,
                           const void* k_new, const void* v_new, float scale, void* out,
                           void* stream) {
    PKV_TRACE("pkv_decode_step");
    if (!s || B < 0 || B > s->max_batch) return PKV_ERR_INVALID_ARG;
    s->last_launches = 0;
    s->last_kernel = 0;
    if (B == 0) return PKV_OK;
    if (!seq_ids || !q || !k_new || !v_new || !out) return PKV_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new)) return PKV_ERR_INVALID_ARG;
    pkv_pool* pool = s->pool;
    if (!same_device(pool)) return PKV_ERR_INVALID_ARG;
    // every table must still fit after the append: checked before anything changes
    for (int i = 0; i < B; ++i) {
        int32_t nb = 0;
        pkv_status st = pool->bm.blocks_after_append(seq_ids[i], &nb);
        if (st != PKV_OK) return st;
        if (nb > s->max_blocks) return PKV_ERR_INVALID_ARG;
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int mb = s->max_batch;
    const int bs = pool->block_size;
    int n_cow = 0;
    s->h_slots.resize(B);
    s->h_src.resize(B);
    s->h_dst.resize(B);
    pkv_status ps = pool->bm.append_batch(seq_ids, B, s->h_slots.data(), s->h_src.data(),
                                          s->h_dst.data(), &n_cow);
    if (ps != PKV_OK) return ps;
    ++s->round;
    // rows of each shared block to copy: the fill before the write, i.e. the
    // offset of the slot that the copying sequence writes into the copy
    s->h_cow_rows.resize(n_cow);
    for (int j = 0; j < n_cow; ++j) {
        s->h_cow_rows[j] = bs;
        for (int i = 0; i < B; ++i)
            if (s->h_slots[i] / bs == s->h_dst[j]) {
                s->h_cow_rows[j] = s->h_slots[i] % bs;
                break;
            }
    }
    // each sequence's persistent row, and the entries of it the device lacks
    s->h_rows.resize(B);
    s->h_upd_idx.clear();
    s->h_upd_val.clear();
    s->h_stable.resize(B);
    for (int i = 0; i < B; ++i) {
        const int r = row_for(s, seq_ids[i]);
        if (r < 0) return PKV_ERR_INVALID_ARG;   // cannot happen: max_seqs >= max_batch
        s->h_rows[i] = r;
    }
    const size_t limit = (size_t)pkv::kStepArgInts;
    const size_t fixed = (size_t)4 * B + 3 * (size_t)n_cow;
    bool fits = fixed <= limit;
    for (int i = 0; i < B && fits; ++i) {
        const pkv::Sequence* sq = pool->bm.find(seq_ids[i]);
        const int r = s->h_rows[i];
        const int nb = (int)sq->blocks.size();
        const bool same = s->row_epoch[r] == sq->epoch;
        const int from = same ? (s->row_nb[r] > 0 ? s->row_nb[r] - 1 : 0) : 0;
        s->h_stable[i] = from;   // entries below `from` stay as the device holds them
        const int32_t* m = s->mirror.data() + (size_t)r * s->max_blocks;
        for (int e = from; e < nb; ++e) {
            if (same && e < s->row_nb[r] && m[e] == sq->blocks[e]) continue;
            s->h_upd_idx.push_back(r * s->max_blocks + e);
            s->h_upd_val.push_back(sq->blocks[e]);
        }
        fits = fixed + 2 * s->h_upd_idx.size() <= limit;
    }
    int launches = 0;
    int32_t* d_lens = s->d_stage + 3 * mb;
    int32_t* d_rows = s->d_stage + 4 * mb;
    int32_t* d_order = s->d_stage + 5 * mb;
    cudaEvent_t e_pre = nullptr, e0 = nullptr, e1 = nullptr, e2 = nullptr;
    const bool profiled =
        s->prof_n > 0 && ((s->round - 1 - s->prof_start) % s->prof_every) == 0;
    if (profiled) {
        const int i = (int)(s->prof_count % s->prof_n);
        e_pre = s->prof_ev[4 * i];
        e0 = s->prof_ev[4 * i + 1];
        e1 = s->prof_ev[4 * i + 2];
        e2 = s->prof_ev[4 * i + 3];
        if (cudaEventRecord(e_pre, st) != cudaSuccess) return PKV_ERR_CUDA;
    }
    if (fits) {
        // fast path: everything of this round travels as kernel parameters
        pkv::StepArgs& a = s->args;
        a.B = B;
        a.n_cow = n_cow;
        a.n_upd = (int32_t)s->h_upd_idx.size();
        a.table_cap = s->max_seqs * s->max_blocks;
        // launch slots by partition length, longest first: a sequence's
        // partitions are equally long, so the grid runs the longest
        // partitions in the first waves and the short ones fill the last
        s->h_lens.resize(B);
        s->h_order.resize(B);
        s->h_key.resize(B);
        // the partition length this round's launch resolves to
        const int P_round = resolve_partition(pool, s->max_blocks, s->partition_tokens,
                                              s->n_q_heads / pool->n_kv_heads,
                                              unsplit_units(pool, B, s->n_q_heads));
        for (int i = 0; i < B; ++i) {
            s->h_lens[i] = (int32_t)pool->bm.find(seq_ids[i])->length;
            s->h_key[i] = pkv::balanced_part_tokens(s->h_lens[i], P_round);
            s->h_order[i] = i;
        }
        std::stable_sort(s->h_order.begin(), s->h_order.end(),
                         [&](int32_t x, int32_t y) { return s->h_key[x] > s->h_key[y]; });
        int32_t* d = a.data;
        for (int i = 0; i < B; ++i) d[i] = s->h_slots[i];
        d += B;
        for (int z = 0; z < B; ++z) d[z] = s->h_lens[s->h_order[z]];
        d += B;
        for (int z = 0; z < B; ++z) d[z] = s->h_rows[s->h_order[z]];
        d += B;
        for (int z = 0; z < B; ++z) d[z] = s->h_order[z];
        d += B;
        for (int j = 0; j < n_cow; ++j) d[j] = s->h_src[j];
        d += n_cow;
        for (int j = 0; j < n_cow; ++j) d[j] = s->h_dst[j];
        d += n_cow;
        for (int j = 0; j < n_cow; ++j) d[j] = s->h_cow_rows[j];
        d += n_cow;
        for (int32_t u = 0; u < a.n_upd; ++u) d[u] = s->h_upd_idx[u];
        d += a.n_upd;
        for (int32_t u = 0; u < a.n_upd; ++u) d[u] = s->h_upd_val[u];
        // what the prologue will leave in the launch slots' lengths, rows and
        // leading table entries, for the decode kernel to start from
        s->pre.n = B <= pkv::kPreSlots ? B : 0;
        for (int z = 0; z < s->pre.n; ++z) {
            s->pre.lens[z] = s->h_lens[s->h_order[z]];
            s->pre.rows[z] = s->h_rows[s->h_order[z]];
            s->pre.order[z] = s->h_order[z];
            s->pre.stable[z] = s->h_stable[s->h_order[z]];
        }
        cudaError_t e = pkv::launch_step_prologue(
            a, pool->k, pool->v, k_new, v_new, s->q_dtype, pool->dtype, s->d_tables, d_lens,
            d_rows, d_order, pool->n_kv_heads, pool->head_dim, bs, pool->num_blocks, pool->k_scale,
            pool->v_scale, pool->d_err, st);
        if (e != cudaSuccess) return PKV_ERR_CUDA;
        launches = 1;
        for (size_t u = 0; u < s->h_upd_idx.size(); ++u) s->mirror[s->h_upd_idx[u]] = s->h_upd_val[u];
        ++s->fast_rounds;
    } else {
        // large rounds: one packed upload of slots, copy pairs, lengths, rows and
        // the batch's full tables from pinned staging; the tables are scattered
        // into their persistent rows, then the copy and the append
        const int r = s->ring;
        if (s->pending[r] && cudaEventSynchronize(s->ev[r]) != cudaSuccess) return PKV_ERR_CUDA;
        s->pending[r] = false;
        int32_t* h = s->h_stage[r];
        for (int i = 0; i < B; ++i) h[i] = s->h_slots[i];
        for (int j = 0; j < n_cow; ++j) {
            h[mb + j] = s->h_src[j];
            h[2 * mb + j] = s->h_dst[j];
        }
        for (int i = 0; i < B; ++i) h[4 * mb + i] = s->h_rows[i];
        int32_t* ht = h + 6 * mb;
        ps = pool->bm.export_tables(seq_ids, B, s->max_blocks, ht, h + 3 * mb, nullptr);
        if (ps != PKV_OK) return ps;   // cannot happen after the checks above
        const size_t ints = (size_t)6 * mb + (size_t)B * s->max_blocks;
        if (cudaMemcpyAsync(s->d_stage, h, ints * sizeof(int32_t), cudaMemcpyHostToDevice, st) !=
                cudaSuccess ||
            cudaEventRecord(s->ev[r], st) != cudaSuccess)
            return PKV_ERR_CUDA;
        s->pending[r] = true;
        s->ring = (r + 1) % pkv_step::kRing;
        if (pkv::launch_scatter_rows(s->d_stage + 6 * mb, d_rows, B, s->max_blocks, s->d_tables,
                                     st) != cudaSuccess)
            return PKV_ERR_CUDA;
        ++launches;
        if (n_cow > 0) {
            ps = block_copy(pool, s->d_stage + mb, s->d_stage + 2 * mb, n_cow, stream);
            if (ps != PKV_OK) return ps;
            ++launches;
        }
        ps = kv_append(pool, s->d_stage, B, k_new, v_new, s->q_dtype, stream);
        if (ps != PKV_OK) return ps;
        ++launches;
        for (int i = 0; i < B; ++i)
            std::copy(ht + (size_t)i * s->max_blocks, ht + (size_t)(i + 1) * s->max_blocks,
                      s->mirror.begin() + (size_t)s->h_rows[i] * s->max_blocks);
        ++s->slow_rounds;
    }
    for (int i = 0; i < B; ++i) {
        const pkv::Sequence* sq = pool->bm.find(seq_ids[i]);
        const int r = s->h_rows[i];
        s->row_epoch[r] = sq->epoch;
        s->row_nb[r] = (int32_t)sq->blocks.size();
    }
    // the decode kernel starts its launch while the prologue runs (programmatic
    // dependent launch), except in profiled rounds whose events sit between
    int decode_launches = 0;
    ps = decode_attention_impl(pool, q, s->q_dtype, s->d_tables, s->max_blocks, d_lens, B,
                               s->n_q_heads, scale, out, s->d_ws, s->ws_bytes, s->partition_tokens,
                               s->kernel, stream, e0, e1, e2, s->d_counters, fits && !profiled,
                               d_rows, s->max_seqs, &decode_launches, &s->last_kernel,
                               fits ? d_order : nullptr, fits ? &s->pre : nullptr);
    if (ps != PKV_OK) return ps;
    if (profiled) ++s->prof_count;
    launches += decode_launches;
    s->last_launches = launches;
    return PKV_OK;
}

}  // extern "C"

extern "C" {

pkv_status pkv_step_profile(pkv_step* s, int n, int every) {
    if (!s || n < 0 || every < 1) return PKV_ERR_INVALID_ARG;
    prof_free(s);
    if (n == 0) return PKV_OK;
    s->prof_ev = new (std::nothrow) cudaEvent_t[4 * (size_t)n]();
    if (!s->prof_ev) return PKV_ERR_INVALID_ARG;
    s->prof_n = n;
    s->prof_every = every;
    s->prof_start = s->round;   // the next round is profiled
    for (int i = 0; i < 4 * n; ++i)
        if (cudaEventCreate(&s->prof_ev[i]) != cudaSuccess) {
            prof_free(s);
            return PKV_ERR_CUDA;
        }
    return PKV_OK;
}

pkv_status pkv_step_profile_read(pkv_step* s, float* prologue_ms, float* decode_ms,
                                 float* merge_ms, int cap, int* n_out) {
    if (!s || !n_out || cap < 0) return PKV_ERR_INVALID_ARG;
    const int have = (int)(s->prof_count < s->prof_n ? s->prof_count : s->prof_n);
    if (cap < have || (have > 0 && (!prologue_ms || !decode_ms || !merge_ms)))
        return PKV_ERR_INVALID_ARG;
    const long long first = s->prof_count - have;
    for (int j = 0; j < have; ++j) {
        const int i = (int)((first + j) % s->prof_n);
        cudaEvent_t* ev = s->prof_ev + 4 * i;
        if (cudaEventSynchronize(ev[3]) != cudaSuccess) return PKV_ERR_CUDA;
        float a = 0.f, b = 0.f, c = 0.f;
        if (cudaEventElapsedTime(&a, ev[0], ev[1]) != cudaSuccess ||
            cudaEventElapsedTime(&b, ev[1], ev[2]) != cudaSuccess ||
            cudaEventElapsedTime(&c, ev[2], ev[3]) != cudaSuccess)
            return PKV_ERR_CUDA;
        prologue_ms[j] = a;
        decode_ms[j] = b;
        merge_ms[j] = c;
    }
    *n_out = have;
    return PKV_OK;
}

}  // extern "C"
