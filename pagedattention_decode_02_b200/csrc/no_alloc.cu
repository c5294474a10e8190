// paged_decode_attention_static: the decode attention call for callers that
// must not allocate device memory.
//
// Who needs it: a process whose device memory is already reserved by another
// allocator (a framework's caching allocator that took the GPU up front, where
// a direct cudaMalloc fails or fragments), and latency-critical loops that
// allow no cudaMalloc/cudaFree once warmed up, because cudaFree - and often
// cudaMalloc - synchronises the whole device.  Such callers cannot provide the
// workspace that paged_decode_attention needs for split contexts.
//
// What it does: the split-context scratch (per-partition max, sum and
// accumulator) lives in one file-scope device array of kScratchBytes, part of
// the library image: every GPU that loads the library holds it until the
// process exits.  Its device address is looked up once per device with
// cudaGetSymbolAddress (the array's name in host code is only a host-side
// stand-in) and handed to the regular decode launch as its workspace.
#include <mutex>

#include "pagedkv.h"

namespace {

constexpr size_t kScratchBytes = 8u << 20;   // 8 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// device address of the scratch array on the current device (looked up on the
// first call for that device); nullptr on failure
void* scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess) return nullptr;
        g_scratch_addr[dev] = ptr;
    }
    return g_scratch_addr[dev];
}

}  // namespace

extern "C" {

size_t paged_decode_static_scratch_bytes(void) { return kScratchBytes; }

pkv_status paged_decode_attention_static(pkv_pool* pool, const void* d_q, pkv_dtype q_dtype,
                                         const int32_t* d_block_tables, int max_blocks,
                                         const int32_t* d_context_lens, int B, int n_q_heads,
                                         float scale, void* d_out, int partition_tokens,
                                         void* stream) {
    if (!pool || B < 0 || max_blocks < 1 || n_q_heads < 1) return PKV_ERR_INVALID_ARG;
    if (B == 0) return PKV_OK;
    int part = partition_tokens;
    size_t need = paged_decode_workspace_bytes_ex(pool, B, n_q_heads, max_blocks, part);
    if (part == 0) {
        // automatic: the library's own choice, or longer partitions (less
        // scratch) until the scratch fits; an unsplit pass needs none
        for (int p = 1024; need > kScratchBytes && p <= (1 << 29); p *= 2) {
            part = p;
            need = paged_decode_workspace_bytes_ex(pool, B, n_q_heads, max_blocks, part);
        }
        if (need > kScratchBytes) {
            part = -1;
            need = 0;
        }
    } else if (need > kScratchBytes) {
        return PKV_ERR_SCRATCH_LIMIT;
    }
    void* ws = nullptr;
    if (need > 0) {
        ws = scratch_for_current_device();
        if (!ws) return PKV_ERR_CUDA;
    }
    return paged_decode_attention_ex(pool, d_q, q_dtype, d_block_tables, max_blocks,
                                     d_context_lens, B, n_q_heads, scale, d_out, ws,
                                     need > 0 ? kScratchBytes : 0, part, PKV_KERNEL_AUTO, stream);
}

}  // extern "C"
