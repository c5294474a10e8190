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
        const uint4 val = *reinterpret_cast<const uint4*>((which ? v : k) +
                                                          ((long long)t * H + h) * row_bytes + ch * 16);
        const long long b = slot / bs, off = slot % bs;
        uint8_t* dst = (which ? v_pool : k_pool) + ((b * H + h) * bs + off) * row_bytes + ch * 16;
        *reinterpret_cast<uint4*>(dst) = val;
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
