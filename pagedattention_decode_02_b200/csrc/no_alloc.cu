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
// the library image.  The array's name in host code is only a host-side
// stand-in; its device address is looked up once per device with
// cudaGetSymbolAddress and handed to the regular decode launch as its
// workspace.  With CUDA's lazy module loading the array is placed on a device
// only when its module is first touched there - and placing it is itself an
// allocation.  kv_pool_create (which allocates anyway) therefore performs the
// lookup for the pool's device, so the array is in place before a caller's
// allocator takes the GPU; from then on the device holds it until the process
// exits.  The lookup on the first static call is only a fallback for a device
// no pool was created on.
#include <mutex>

#include "pagedkv.h"
#include "pool.h"
#include "trace.h"

namespace {

constexpr size_t kScratchBytes = 8u << 20;   // 8 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// device address of the scratch array on device `dev`, which must be the
// current device (looked up on first use for that device); nullptr on failure
void* scratch_for_device(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_addr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess) {
            cudaGetLastError();   // leave no sticky error for the caller's next call
            return nullptr;
        }
        g_scratch_addr[dev] = ptr;
    }
    return g_scratch_addr[dev];
}

void* scratch_for_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    return scratch_for_device(dev);
}

}  // namespace

namespace pkv {
// called by kv_pool_create with the pool's device current
bool static_scratch_prepare(int device) { return scratch_for_device(device) != nullptr; }
}  // namespace pkv

extern "C" {

size_t paged_decode_static_scratch_bytes(void) { return kScratchBytes; }

pkv_status paged_decode_attention_static(pkv_pool* pool, const void* d_q, pkv_dtype q_dtype,
                                         const int32_t* d_block_tables, int max_blocks,
                                         const int32_t* d_context_lens, int B, int n_q_heads,
                                         float scale, void* d_out, int partition_tokens,
                                         void* stream) {
    PKV_TRACE("paged_decode_attention_static");
    if (!pool || B < 0 || max_blocks < 1 || n_q_heads < 1) return PKV_ERR_INVALID_ARG;
    if (B == 0) return PKV_OK;
    if (pool->host_only || n_q_heads % pool->n_kv_heads) return PKV_ERR_INVALID_ARG;
    int part = partition_tokens;
    size_t need = paged_decode_workspace_bytes_ex(pool, B, n_q_heads, max_blocks, part);
    if (part == 0 && need > kScratchBytes) {
        // automatic: the library's own choice as paged_decode_attention makes
        // it - without the stage-balanced kernel when only its share does not
        // fit (the automatic selection skips that kernel when the workspace
        // is too small for it) - else partitions lengthened from the
        // automatic length (less scratch) until the scratch fits; an unsplit
        // pass needs none
        need = pkv::decode_workspace_bytes_partitioned(pool, B, n_q_heads, max_blocks, 0);
        if (need > kScratchBytes) {
            const long long auto_p = pkv::decode_auto_partition(pool, B, n_q_heads, max_blocks);
            for (long long p = 2 * auto_p; need > kScratchBytes && p <= (1 << 29); p *= 2) {
                part = (int)p;
                need = pkv::decode_workspace_bytes_partitioned(pool, B, n_q_heads, max_blocks,
                                                               part);
            }
        }
        if (need > kScratchBytes) {
            part = -1;
            need = 0;
        }
    } else if (part != 0 && need > kScratchBytes) {
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
