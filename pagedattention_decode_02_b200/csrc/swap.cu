// Swapping a sequence's KV blocks out to host memory and back.
//
// "KV 缓存与分页注意力" §放不下的时候: when blocks run out, the latest-started
// sequence gives up all of its blocks (a sequence's blocks are kept or given
// up together); one way back is to move them to CPU memory and, when its turn
// comes, move them back.  kv_swap_out copies every block of the sequence, in
// logical order, into caller-owned pinned host buffers and releases the
// sequence; kv_swap_in admits it again with fresh blocks and copies the rows
// back.  Blocks the sequence shared with others are copied out like the rest
// and come back as private blocks.
//
// The copy is one kernel per launch of up to kSwapBlocks blocks: each thread
// moves 16-byte chunks between a pool tile and pinned host memory (reached
// through its device mapping), so no device staging buffer is needed.
#include <algorithm>
#include <memory>
#include <new>
#include <vector>

#include "decode_launch.h"
#include "kernels_common.cuh"
#include "pool.h"
#include "trace.h"

namespace pkv {
namespace {

constexpr int kSwapBlocks = 960;   // block ids per launch (kernel parameters < 4 KB)

struct SwapArgs {
    int32_t n;
    int32_t first;   // index of blocks[0] in the host buffer, in blocks
    int32_t blocks[kSwapBlocks];
};

// out = true: pool -> host; false: host -> pool.  K and V, all KV heads of a block.
__global__ void swap_kernel(const __grid_constant__ SwapArgs a, uint8_t* k_pool, uint8_t* v_pool,
                            uint8_t* h_k, uint8_t* h_v, long long block_bytes, int num_blocks,
                            bool out, uint32_t* err) {
    const long long chunks = block_bytes / 16;
    const long long total = 2LL * a.n * chunks;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int which = (int)(i / (a.n * chunks));
        const long long r = i - which * a.n * chunks;
        const int j = (int)(r / chunks);
        const long long c = r % chunks;
        const int b = a.blocks[j];
        if (b < 0 || b >= num_blocks) {
            if (c == 0 && which == 0) report_error(err, PKV_DEVERR_BLOCK_ID);
            continue;
        }
        uint4* dev = reinterpret_cast<uint4*>((which ? v_pool : k_pool) + (long long)b * block_bytes) + c;
        uint4* host = reinterpret_cast<uint4*>((which ? h_v : h_k) +
                                               (long long)(a.first + j) * block_bytes) + c;
        if (out)
            *host = *dev;
        else
            *dev = *host;
    }
}

// device address of a pinned host buffer, or null if it is not pinned
void* mapped(const void* host) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, host) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (at.type != cudaMemoryTypeHost || !at.devicePointer) return nullptr;
    return at.devicePointer;
}

cudaError_t launch_swap(pkv_pool* p, const std::vector<int32_t>& blocks, void* dk, void* dv,
                        bool out, cudaStream_t st) {
    const long long block_bytes = (long long)p->n_kv_heads * p->block_size * p->head_dim *
                                  (p->dtype == PKV_F32 ? 4 : p->dtype == PKV_FP8_E4M3 ? 1 : 2);
    std::unique_ptr<SwapArgs> holder(new (std::nothrow) SwapArgs);
    if (!holder) return cudaErrorMemoryAllocation;
    SwapArgs& a = *holder;
    for (size_t s = 0; s < blocks.size(); s += kSwapBlocks) {
        a.n = (int32_t)std::min<size_t>(kSwapBlocks, blocks.size() - s);
        a.first = (int32_t)s;
        std::copy(blocks.begin() + s, blocks.begin() + s + a.n, a.blocks);
        const long long items = 2LL * a.n * (block_bytes / 16);
        long long grid = (items + 255) / 256;
        grid = std::max(1LL, std::min(grid, 148LL * 8));
        swap_kernel<<<(unsigned)grid, 256, 0, st>>>(a, p->k, p->v, static_cast<uint8_t*>(dk),
                                                    static_cast<uint8_t*>(dv), block_bytes,
                                                    p->num_blocks, out, p->d_err);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace
}  // namespace pkv

extern "C" {

pkv_status kv_swap_out(pkv_pool* p, int64_t seq_id, void* h_k, void* h_v, size_t capacity_bytes,
                       int32_t* n_blocks_out, int64_t* n_tokens_out, void* stream) {
    PKV_TRACE("kv_swap_out");
    if (!p || p->host_only || !h_k || !h_v) return PKV_ERR_INVALID_ARG;
    const pkv::Sequence* s = p->bm.find(seq_id);
    if (!s) return PKV_ERR_UNKNOWN_SEQ;
    const size_t block_bytes = (size_t)p->n_kv_heads * p->block_size * p->head_dim *
                               (p->dtype == PKV_F32 ? 4 : p->dtype == PKV_FP8_E4M3 ? 1 : 2);
    if (s->blocks.size() * block_bytes > capacity_bytes) return PKV_ERR_INVALID_ARG;
    void* dk = pkv::mapped(h_k);
    void* dv = pkv::mapped(h_v);
    if (!dk || !dv) return PKV_ERR_INVALID_ARG;
    const std::vector<int32_t> blocks = s->blocks;
    const int64_t n_tokens = s->length;
    if (pkv::launch_swap(p, blocks, dk, dv, true, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return PKV_ERR_CUDA;
    // the copies are queued on `stream` ahead of any later work that reuses the blocks
    const pkv_status st = p->bm.release(seq_id);
    if (st != PKV_OK) return st;
    if (n_blocks_out) *n_blocks_out = (int32_t)blocks.size();
    if (n_tokens_out) *n_tokens_out = n_tokens;
    return PKV_OK;
}

pkv_status kv_swap_in(pkv_pool* p, int64_t seq_id, const void* h_k, const void* h_v,
                      size_t capacity_bytes, int64_t n_tokens, void* stream) {
    PKV_TRACE("kv_swap_in");
    if (!p || p->host_only || !h_k || !h_v || n_tokens < 0 || n_tokens > 0x7fffffff)
        return PKV_ERR_INVALID_ARG;
    const size_t block_bytes = (size_t)p->n_kv_heads * p->block_size * p->head_dim *
                               (p->dtype == PKV_F32 ? 4 : p->dtype == PKV_FP8_E4M3 ? 1 : 2);
    const size_t n_blocks = (size_t)((n_tokens + p->block_size - 1) / p->block_size);
    if (n_blocks * block_bytes > capacity_bytes) return PKV_ERR_INVALID_ARG;
    void* dk = pkv::mapped(h_k);
    void* dv = pkv::mapped(h_v);
    if (!dk || !dv) return PKV_ERR_INVALID_ARG;
    std::vector<int32_t> slots((size_t)n_tokens);
    const pkv_status st = p->bm.alloc(seq_id, (int)n_tokens, slots.data());
    if (st != PKV_OK) return st;
    const std::vector<int32_t> blocks = p->bm.find(seq_id)->blocks;
    if (pkv::launch_swap(p, blocks, dk, dv, false, static_cast<cudaStream_t>(stream)) !=
        cudaSuccess) {
        p->bm.undo_alloc(seq_id);   // state exactly as before the call
        return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

}  // extern "C"
