// Appending new K/V rows into their slots, and copy-on-write block copies.
//
// "KV 缓存与分页注意力" §一次写一个词元: each round computes only the new token's
// key and value and stores it; §块表 / "读懂PagedAttention" §分离逻辑顺序与实际存储位置:
// it goes into the next free slot of the sequence's last block.  The slot
// (physical block * block_size + offset) comes from the host block manager.
// The exhibit's FAQ 08 (共用，写时复制): a block that is still shared is copied
// before the write; block_copy makes that copy on the device.
//
// Both kernels move 16-byte chunks: one thread per chunk of a destination row
// (kv_append) or of a block (block_copy), so every access is a coalesced
// 16-byte load/store.  FP8 pools quantise on the way in: 16 input values ->
// float -> divided by the per-tensor scale (IEEE round-to-nearest) ->
// e4m3 with round-to-nearest-even and saturation -> one 16-byte store.
#include "decode_launch.h"
#include "kernels_common.cuh"

namespace pkv {

namespace {

template <typename IN>
__device__ __forceinline__ void load16(const IN* src, float* f) {
    // 16 consecutive input elements as floats
    if constexpr (sizeof(IN) == 4) {
#pragma unroll
        for (int i = 0; i < 4; ++i) VecLoad<float, 4>::run(src + 4 * i, f + 4 * i);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) VecLoad<IN, 4>::run(src + 4 * i, f + 4 * i);
    }
}

// One 16-byte chunk of one destination row.  `which` 0 = K, 1 = V; `t` the
// token, `h` the KV head, `ch` the chunk of the row.  FP8 pools: 16 input
// values -> x / scale (IEEE division) -> e4m3, round to nearest even,
// saturating.
template <typename IN>
__device__ __forceinline__ void append_chunk_fp8(uint8_t* k_pool, uint8_t* v_pool, const IN* k,
                                                 const IN* v, int which, int t, int h, int ch,
                                                 int slot, int H, int D, int bs, float k_scale,
                                                 float v_scale) {
    const IN* src = (which ? v : k) + ((long long)t * H + h) * D + ch * 16;
    const float scale = which ? v_scale : k_scale;
    float f[16];
    load16<IN>(src, f);
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float2 a = make_float2(__fdiv_rn(f[4 * j], scale), __fdiv_rn(f[4 * j + 1], scale));
        float2 b = make_float2(__fdiv_rn(f[4 * j + 2], scale), __fdiv_rn(f[4 * j + 3], scale));
        const uint32_t lo = __nv_cvt_float2_to_fp8x2(a, __NV_SATFINITE, __NV_E4M3);
        const uint32_t hi = __nv_cvt_float2_to_fp8x2(b, __NV_SATFINITE, __NV_E4M3);
        w[j] = (lo & 0xFFFFu) | (hi << 16);
    }
    const long long b = slot / bs, off = slot % bs;
    uint8_t* dst = (which ? v_pool : k_pool) + (((b * H + h) * bs + off) * D + ch * 16);
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void append_chunk_copy(uint8_t* k_pool, uint8_t* v_pool,
                                                  const uint8_t* k, const uint8_t* v, int which,
                                                  int t, int h, int ch, int slot, int H,
                                                  int row_bytes, int bs) {
    const uint4 val = *reinterpret_cast<const uint4*>((which ? v : k) +
                                                      ((long long)t * H + h) * row_bytes + ch * 16);
    const long long b = slot / bs, off = slot % bs;
    uint8_t* dst = (which ? v_pool : k_pool) + ((b * H + h) * bs + off) * row_bytes + ch * 16;
    *reinterpret_cast<uint4*>(dst) = val;
}

// one thread = one 16-byte chunk of one destination row (K or V)
template <typename IN>
__global__ void kv_append_fp8_kernel(uint8_t* k_pool, uint8_t* v_pool, const int32_t* slots,
                                     int n_tokens, const IN* k, const IN* v, int H, int D, int bs,
                                     int num_blocks, float k_scale, float v_scale, uint32_t* err) {
    const int chunks = D / 16;                      // 16 fp8 codes per chunk
    const long long per_tok = (long long)H * chunks;
    const long long total = 2LL * n_tokens * per_tok;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int which = (int)(i / (n_tokens * per_tok));
        const long long r = i - which * (n_tokens * per_tok);
        const int t = (int)(r / per_tok);
        const int h = (int)((r / chunks) % H);
        const int ch = (int)(r % chunks);
        const int slot = slots[t];
        if (slot < 0) continue;
        if ((long long)slot >= (long long)num_blocks * bs) {
            if (which == 0 && h == 0 && ch == 0) report_error(err, PKV_DEVERR_SLOT);
            continue;
        }
        append_chunk_fp8<IN>(k_pool, v_pool, k, v, which, t, h, ch, slot, H, D, bs, k_scale, v_scale);
    }
}

// same dtype in and out: plain 16-byte copies
__global__ void kv_append_copy_kernel(uint8_t* k_pool, uint8_t* v_pool, const int32_t* slots,
                                      int n_tokens, const uint8_t* k, const uint8_t* v, int H,
                                      int row_bytes, int bs, int num_blocks, uint32_t* err) {
    const int chunks = row_bytes / 16;
    const long long per_tok = (long long)H * chunks;
    const long long total = 2LL * n_tokens * per_tok;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int which = (int)(i / (n_tokens * per_tok));
        const long long r = i - which * (n_tokens * per_tok);
        const int t = (int)(r / per_tok);
        const int h = (int)((r / chunks) % H);
        const int ch = (int)(r % chunks);
        const int slot = slots[t];
        if (slot < 0) continue;
        if ((long long)slot >= (long long)num_blocks * bs) {
            if (which == 0 && h == 0 && ch == 0) report_error(err, PKV_DEVERR_SLOT);
            continue;
        }
        append_chunk_copy(k_pool, v_pool, k, v, which, t, h, ch, slot, H, row_bytes, bs);
    }
}

// The decode round's prologue (see StepArgs).  blockIdx.y == 0: lengths,
// table updates and the appends; blockIdx.y == 1 + j: copy-on-write pair j,
// rows [0, cow_rows[j]) of every KV head's tile, K and V.  The copied rows
// and the appended row (row cow_rows[j] of the new block) are disjoint, and
// no append writes a row below the fill of a shared block, so the two kinds
// of work need no ordering inside the launch.
template <typename IN, bool FP8>
__global__ void step_prologue_kernel(const __grid_constant__ StepArgs a, uint8_t* k_pool,
                                     uint8_t* v_pool, const IN* k, const IN* v, int32_t* tables,
                                     int32_t* lens, int32_t* rows, int32_t* order, int H, int D,
                                     int bs, int num_blocks, float k_scale, float v_scale,
                                     uint32_t* err) {
    allow_dependent_launch();   // the decode kernel may start its launch now
    const int B = a.B;
    const int32_t* slots = a.data;
    const int32_t* lens_in = a.data + B;
    const int32_t* rows_in = a.data + 2 * B;
    const int32_t* order_in = a.data + 3 * B;
    const int32_t* cow_src = a.data + 4 * B;
    const int32_t* cow_dst = cow_src + a.n_cow;
    const int32_t* cow_rows = cow_dst + a.n_cow;
    const int32_t* upd_idx = cow_rows + a.n_cow;
    const int32_t* upd_val = upd_idx + a.n_upd;
    const int eb = FP8 ? 1 : (int)sizeof(IN);
    const int row_bytes = D * eb;
    const long long stride = (long long)gridDim.x * blockDim.x;
    const long long first = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    if (blockIdx.y == 0) {
        for (long long i = first; i < B; i += stride) {
            lens[i] = lens_in[i];
            rows[i] = rows_in[i];
            order[i] = order_in[i];
        }
        for (long long u = first; u < a.n_upd; u += stride) {
            const int idx = upd_idx[u];
            if (idx >= 0 && idx < a.table_cap) tables[idx] = upd_val[u];
        }
        const int chunks = FP8 ? D / 16 : row_bytes / 16;
        const long long per_tok = (long long)H * chunks;
        const long long total = 2LL * B * per_tok;
        for (long long i = first; i < total; i += stride) {
            const int which = (int)(i / (B * per_tok));
            const long long r = i - which * (B * per_tok);
            const int t = (int)(r / per_tok);
            const int h = (int)((r / chunks) % H);
            const int ch = (int)(r % chunks);
            const int slot = slots[t];
            if (slot < 0) continue;
            if ((long long)slot >= (long long)num_blocks * bs) {
                if (which == 0 && h == 0 && ch == 0) report_error(err, PKV_DEVERR_SLOT);
                continue;
            }
            if constexpr (FP8)
                append_chunk_fp8<IN>(k_pool, v_pool, k, v, which, t, h, ch, slot, H, D, bs,
                                     k_scale, v_scale);
            else
                append_chunk_copy(k_pool, v_pool, reinterpret_cast<const uint8_t*>(k),
                                  reinterpret_cast<const uint8_t*>(v), which, t, h, ch, slot, H,
                                  row_bytes, bs);
        }
        return;
    }
    const int j = blockIdx.y - 1;
    const int s = cow_src[j], d = cow_dst[j], n_rows = cow_rows[j];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks || n_rows < 0 || n_rows > bs) {
        if (first == 0) report_error(err, PKV_DEVERR_BLOCK_ID);
        return;
    }
    const long long tile = (long long)bs * row_bytes;             // one (block, head) tile
    const long long per_head = (long long)n_rows * row_bytes / 16; // chunks copied per tile
    const long long total = 2LL * H * per_head;
    for (long long i = first; i < total; i += stride) {
        const int which = (int)(i / (H * per_head));
        const long long r = i - which * (H * per_head);
        const int h = (int)(r / per_head);
        const long long c = r % per_head;
        uint8_t* pool = which ? v_pool : k_pool;
        const uint4 val = reinterpret_cast<const uint4*>(pool + ((long long)s * H + h) * tile)[c];
        reinterpret_cast<uint4*>(pool + ((long long)d * H + h) * tile)[c] = val;
    }
}

__global__ void block_copy_kernel(uint8_t* k_pool, uint8_t* v_pool, const int32_t* src,
                                  const int32_t* dst, long long block_bytes, int num_blocks,
                                  uint32_t* err) {
    const int pair = blockIdx.x;
    const int s = src[pair], d = dst[pair];
    if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0) report_error(err, PKV_DEVERR_BLOCK_ID);
        return;
    }
    const long long chunks = block_bytes / 16;
    for (long long c = blockIdx.y * (long long)blockDim.x + threadIdx.x; c < 2 * chunks;
         c += (long long)gridDim.y * blockDim.x) {
        const int which = c >= chunks;
        const long long cc = which ? c - chunks : c;
        uint8_t* pool = which ? v_pool : k_pool;
        const uint4 val = reinterpret_cast<const uint4*>(pool + s * block_bytes)[cc];
        reinterpret_cast<uint4*>(pool + d * block_bytes)[cc] = val;
    }
}

int grid_for(long long items, int threads) {
    long long g = (items + threads - 1) / threads;
    if (g > 148LL * 32) g = 148LL * 32;
    return (int)(g < 1 ? 1 : g);
}

}  // namespace

cudaError_t launch_kv_append(uint8_t* k_pool, uint8_t* v_pool, const int32_t* slots, int n_tokens,
                             const void* k, const void* v, int in_dtype, int kv_dtype,
                             int n_kv_heads, int head_dim, int block_size, int num_blocks,
                             float k_scale, float v_scale, uint32_t* err, cudaStream_t st) {
    if (n_tokens <= 0) return cudaSuccess;
    constexpr int kThreads = 256;
    if (kv_dtype == PKV_FP8_E4M3) {
        const long long items = 2LL * n_tokens * n_kv_heads * (head_dim / 16);
        const int grid = grid_for(items, kThreads);
        switch (in_dtype) {
            case PKV_F32:
                kv_append_fp8_kernel<float><<<grid, kThreads, 0, st>>>(
                    k_pool, v_pool, slots, n_tokens, (const float*)k, (const float*)v, n_kv_heads,
                    head_dim, block_size, num_blocks, k_scale, v_scale, err);
                break;
            case PKV_F16:
                kv_append_fp8_kernel<__half><<<grid, kThreads, 0, st>>>(
                    k_pool, v_pool, slots, n_tokens, (const __half*)k, (const __half*)v, n_kv_heads,
                    head_dim, block_size, num_blocks, k_scale, v_scale, err);
                break;
            case PKV_BF16:
                kv_append_fp8_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(
                    k_pool, v_pool, slots, n_tokens, (const __nv_bfloat16*)k,
                    (const __nv_bfloat16*)v, n_kv_heads, head_dim, block_size, num_blocks, k_scale,
                    v_scale, err);
                break;
            default:
                return cudaErrorInvalidValue;
        }
        return cudaGetLastError();
    }
    const int eb = kv_dtype == PKV_F32 ? 4 : 2;
    const int row = head_dim * eb;
    const long long items = 2LL * n_tokens * n_kv_heads * (row / 16);
    kv_append_copy_kernel<<<grid_for(items, kThreads), kThreads, 0, st>>>(
        k_pool, v_pool, slots, n_tokens, (const uint8_t*)k, (const uint8_t*)v, n_kv_heads, row,
        block_size, num_blocks, err);
    return cudaGetLastError();
}

cudaError_t launch_block_copy(uint8_t* k_pool, uint8_t* v_pool, const int32_t* src,
                              const int32_t* dst, int n_pairs, long long block_bytes,
                              int num_blocks, uint32_t* err, cudaStream_t st) {
    if (n_pairs <= 0) return cudaSuccess;
    constexpr int kThreads = 256;
    const long long chunks = 2 * block_bytes / 16;
    long long gy = (chunks + kThreads * 4 - 1) / (kThreads * 4);
    if (gy > 65535) gy = 65535;
    block_copy_kernel<<<dim3(n_pairs, (unsigned)gy), kThreads, 0, st>>>(k_pool, v_pool, src, dst,
                                                                        block_bytes, num_blocks, err);
    return cudaGetLastError();
}

}  // namespace pkv

namespace pkv {

cudaError_t launch_step_prologue(const StepArgs& a, uint8_t* k_pool, uint8_t* v_pool,
                                 const void* k, const void* v, int in_dtype, int kv_dtype,
                                 int32_t* tables, int32_t* lens, int32_t* rows, int32_t* order,
                                 int H, int D, int bs, int num_blocks, float k_scale,
                                 float v_scale, uint32_t* err, cudaStream_t st) {
    constexpr int kThreads = 256;
    const int eb = kv_dtype == PKV_F32 ? 4 : kv_dtype == PKV_FP8_E4M3 ? 1 : 2;
    const int chunks_per_row = kv_dtype == PKV_FP8_E4M3 ? D / 16 : D * eb / 16;
    const long long append_items = 2LL * a.B * H * chunks_per_row;
    const long long copy_items = 2LL * H * bs * D * eb / 16;
    long long items = append_items > copy_items ? append_items : copy_items;
    long long gx = (items + kThreads - 1) / kThreads;
    if (gx > 148 * 4) gx = 148 * 4;
    if (gx < 1) gx = 1;
    const dim3 grid((unsigned)gx, 1 + a.n_cow);
    if (kv_dtype == PKV_FP8_E4M3) {
        switch (in_dtype) {
            case PKV_F32:
                step_prologue_kernel<float, true><<<grid, kThreads, 0, st>>>(
                    a, k_pool, v_pool, (const float*)k, (const float*)v, tables, lens, rows, order, H, D, bs,
                    num_blocks, k_scale, v_scale, err);
                break;
            case PKV_F16:
                step_prologue_kernel<__half, true><<<grid, kThreads, 0, st>>>(
                    a, k_pool, v_pool, (const __half*)k, (const __half*)v, tables, lens, rows, order, H, D, bs,
                    num_blocks, k_scale, v_scale, err);
                break;
            case PKV_BF16:
                step_prologue_kernel<__nv_bfloat16, true><<<grid, kThreads, 0, st>>>(
                    a, k_pool, v_pool, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, tables,
                    lens, rows, order, H, D, bs, num_blocks, k_scale, v_scale, err);
                break;
            default:
                return cudaErrorInvalidValue;
        }
    } else if (kv_dtype == PKV_F32) {
        step_prologue_kernel<float, false><<<grid, kThreads, 0, st>>>(
            a, k_pool, v_pool, (const float*)k, (const float*)v, tables, lens, rows, order, H, D, bs,
            num_blocks, k_scale, v_scale, err);
    } else {
        step_prologue_kernel<__half, false><<<grid, kThreads, 0, st>>>(
            a, k_pool, v_pool, (const __half*)k, (const __half*)v, tables, lens, rows, order, H, D, bs,
            num_blocks, k_scale, v_scale, err);
    }
    return cudaGetLastError();
}

}  // namespace pkv

namespace pkv {
namespace {
__global__ void scatter_rows_kernel(const int32_t* staged, const int32_t* rows, int B,
                                    int max_blocks, int32_t* tables) {
    const long long total = (long long)B * max_blocks;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int b = (int)(i / max_blocks);
        tables[(long long)rows[b] * max_blocks + i % max_blocks] = staged[i];
    }
}
}  // namespace

cudaError_t launch_scatter_rows(const int32_t* staged, const int32_t* rows, int B, int max_blocks,
                                int32_t* tables, cudaStream_t st) {
    const long long total = (long long)B * max_blocks;
    long long grid = (total + 255) / 256;
    grid = grid < 1 ? 1 : (grid > 148 * 8 ? 148 * 8 : grid);
    scatter_rows_kernel<<<(unsigned)grid, 256, 0, st>>>(staged, rows, B, max_blocks, tables);
    return cudaGetLastError();
}

namespace {
// One thread waits, with the given budget, on a barrier phase that nothing
// completes (no arrival, no copy), the same bounded wait the decode and
// prompt kernels use; when it gives up it reports PKV_DEVERR_TIMEOUT.
__global__ void wait_probe_kernel(uint32_t* err, unsigned long long budget_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, budget_ns)) report_error(err, PKV_DEVERR_TIMEOUT);
}
}  // namespace

cudaError_t launch_wait_probe(uint32_t* err, unsigned long long budget_ns, cudaStream_t st) {
    wait_probe_kernel<<<1, 32, 0, st>>>(err, budget_ns);
    return cudaGetLastError();
}

}  // namespace pkv
