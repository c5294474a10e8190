// Device helpers shared by the paged-KV kernels (sm_100a).
//
// - mbarrier + 1-D bulk copies (cp.async.bulk, no multicast, this GPU's own
//   memory only) for staging K/V rows into shared memory;
// - bounded waits: every wait on a copy gives up after a fixed wall-clock
//   budget, sets a bit in the pool's device error word and lets the kernel
//   finish instead of hanging;
// - element conversions for the four storage types.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "pagedkv.h"

namespace pkv {

// ---------------------------------------------------------------------------
// element types
// ---------------------------------------------------------------------------
struct fp8e4m3 {
    uint8_t x;
};

template <typename T>
struct Elem;
template <>
struct Elem<float> {
    static constexpr int bytes = 4;
    static constexpr int id = PKV_F32;
    __device__ static float to_f(float v) { return v; }
    __device__ static float from_f(float v) { return v; }
};
template <>
struct Elem<__half> {
    static constexpr int bytes = 2;
    static constexpr int id = PKV_F16;
    __device__ static float to_f(__half v) { return __half2float(v); }
    __device__ static __half from_f(float v) { return __float2half_rn(v); }
};
template <>
struct Elem<__nv_bfloat16> {
    static constexpr int bytes = 2;
    static constexpr int id = PKV_BF16;
    __device__ static float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    __device__ static __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};
template <>
struct Elem<fp8e4m3> {
    static constexpr int bytes = 1;
    static constexpr int id = PKV_FP8_E4M3;
};

// Load N consecutive elements of type T from shared/global memory as floats.
// N * sizeof(T) is 4, 8 or 16 bytes; the address is aligned to that size.
template <typename T, int N>
struct VecLoad;

template <int N>
struct VecLoad<float, N> {
    __device__ static void run(const void* p, float* out) {
        if constexpr (N == 4) {
            float4 v = *reinterpret_cast<const float4*>(p);
            out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
        } else if constexpr (N == 2) {
            float2 v = *reinterpret_cast<const float2*>(p);
            out[0] = v.x; out[1] = v.y;
        } else {
            static_assert(N == 1, "");
            out[0] = *reinterpret_cast<const float*>(p);
        }
    }
};

template <int N>
struct VecLoad<__half, N> {
    __device__ static void run(const void* p, float* out) {
        if constexpr (N == 4) {
            uint2 u = *reinterpret_cast<const uint2*>(p);
            float2 a = __half22float2(*reinterpret_cast<__half2*>(&u.x));
            float2 b = __half22float2(*reinterpret_cast<__half2*>(&u.y));
            out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
        } else if constexpr (N == 2) {
            uint32_t u = *reinterpret_cast<const uint32_t*>(p);
            float2 a = __half22float2(*reinterpret_cast<__half2*>(&u));
            out[0] = a.x; out[1] = a.y;
        } else {
            static_assert(N == 1, "");
            out[0] = __half2float(*reinterpret_cast<const __half*>(p));
        }
    }
};

template <int N>
struct VecLoad<__nv_bfloat16, N> {
    __device__ static void run(const void* p, float* out) {
        if constexpr (N == 4) {
            uint2 u = *reinterpret_cast<const uint2*>(p);
            out[0] = __uint_as_float(u.x << 16); out[1] = __uint_as_float(u.x & 0xFFFF0000u);
            out[2] = __uint_as_float(u.y << 16); out[3] = __uint_as_float(u.y & 0xFFFF0000u);
        } else if constexpr (N == 2) {
            uint32_t u = *reinterpret_cast<const uint32_t*>(p);
            out[0] = __uint_as_float(u << 16); out[1] = __uint_as_float(u & 0xFFFF0000u);
        } else {
            static_assert(N == 1, "");
            uint32_t u = *reinterpret_cast<const uint16_t*>(p);
            out[0] = __uint_as_float(u << 16);
        }
    }
};

// two FP8-E4M3 codes -> two floats, exact (through the hardware e4m3x2 -> f16x2 convert)
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two, __NV_E4M3);
    return __half22float2(*reinterpret_cast<__half2*>(&h));
}

template <int N>
struct VecLoad<fp8e4m3, N> {
    __device__ static void run(const void* p, float* out) {
        if constexpr (N == 4) {
            uint32_t u = *reinterpret_cast<const uint32_t*>(p);
            float2 a = e4m3x2_to_float2((uint16_t)(u & 0xFFFF));
            float2 b = e4m3x2_to_float2((uint16_t)(u >> 16));
            out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
        } else if constexpr (N == 2) {
            float2 a = e4m3x2_to_float2(*reinterpret_cast<const uint16_t*>(p));
            out[0] = a.x; out[1] = a.y;
        } else {
            static_assert(N == 1, "");
            uint16_t u = *reinterpret_cast<const uint8_t*>(p);
            out[0] = e4m3x2_to_float2(u).x;
        }
    }
};

// ---------------------------------------------------------------------------
// error word
// ---------------------------------------------------------------------------
__device__ __forceinline__ void report_error(uint32_t* err, uint32_t bits) {
    if (err) atomicOr(err, bits);
}

// ---------------------------------------------------------------------------
// mbarrier and bulk copies
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// make barrier initialisation visible to the async (bulk copy) proxy
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (bulk copy) writes to the same memory
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// non-blocking test of the phase with the given parity
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for the barrier phase with the given parity.  Gives up after
// budget_ns of wall-clock time and returns false.  A healthy copy of a few KB
// completes in microseconds; the default budget only ends a wait that would
// otherwise never end.  Kernels pass their pool's budget (pkv_set_wait_budget)
// for the waits of their main loops, and keep the default for the waits that
// make sure no copy is still in flight when they give up.  A shortened budget
// polls without blocking (try_wait may suspend the thread until the phase
// completes), so that the wait can give up while the copy is still on its way.
constexpr uint64_t kWaitBudgetNs = 2000000000ull;  // 2 s

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          uint64_t budget_ns = kWaitBudgetNs) {
    if (budget_ns < kWaitBudgetNs) {
        const uint64_t t0 = global_timer_ns();
        while (true) {
            if (mbar_test_wait(bar, parity)) return true;
            if (global_timer_ns() - t0 > budget_ns) return false;
        }
    }
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > budget_ns) return false;
    }
}

// 1-D bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned)
// from this GPU's global memory into this CTA's shared memory; completion is
// counted on `bar` in bytes.  The L2 policy marks the lines evict-first: the
// KV stream is read once per step.
__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src_gmem, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ---------------------------------------------------------------------------
// kernel parameter blocks
// ---------------------------------------------------------------------------
// programmatic dependent launch: wait until the preceding kernel of the
// stream has completed and its writes are visible (a no-op when the kernel
// was launched without the programmatic-serialization attribute) / allow the
// next kernel of the stream to start launching
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependent_launch() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

struct DecodeParams {
    const void* q;
    void* out;
    const uint8_t* k_pool;
    const uint8_t* v_pool;
    const int32_t* tables;
    const int32_t* lens;
    float* ws_ml;    // [B][H_q][max_parts][2]  (running max in log2 units, sum)
    float* ws_acc;   // [B][H_q][max_parts][D]  (unnormalised accumulator)
    const int32_t* table_rows;  // [B] row of `tables` holding launch slot i's table, or null
                                // (row i); rows outside [0, n_table_rows) are rejected
    const int32_t* order;       // [B] launch slot -> the caller's sequence index (q, out,
                                // partials), or null (identity); lens and table_rows are
                                // indexed by launch slot
    int n_table_rows;
    int pdl;         // host side: launch with programmatic stream serialization
    int* counters;   // [B][H_q] partitions finished, or null: when set, the last
                     // CTA of a split (sequence, head) merges in the decode
                     // kernel itself and resets its counter to 0
    uint32_t* err;
    int B, H_q, H_kv, G;
    int max_blocks, block_size, num_blocks;
    int part_tokens;  // longest partition (multiple of 16): ceil(c / part_tokens) partitions
    int max_parts;    // partitions of the longest possible context
    float q_scale;    // scale * log2(e) * k_scale: folded into q
    float v_scale;    // FP8 V dequantisation (1 otherwise)
    long long head_stride;   // bytes of one (block, kv head) tile: bs * D * elem
    long long block_stride;  // bytes of one block: H_kv * head_stride
    unsigned long long wait_ns;  // budget of the main loops' waits (the pool's)
    const struct StepPrefetch* pre;   // host side only: see StepPrefetch (null: none)
};

// What the decode-step runtime knows on the host about each launch slot
// before the round's prologue kernel runs: the context length, the table row,
// the caller's sequence index, and how many leading entries of the row the
// prologue leaves unchanged (their blocks hold no token it writes and no
// copy-on-write target).  Passed to the decode kernel by value, so that a CTA
// can read those entries, start loading their blocks and load its query
// before the prologue has finished (the query is not the prologue's output:
// it was written before the prologue, which starts only once all preceding
// work on the stream has completed).
constexpr int kPreSlots = 128;
struct StepPrefetch {
    int n;                        // launch slots covered: 0 .. n - 1 (0: none)
    int32_t lens[kPreSlots];
    int32_t rows[kPreSlots];
    int32_t order[kPreSlots];
    int32_t stable[kPreSlots];
};

// The launch's prefetch block, or an empty one.
inline const StepPrefetch& prefetch_of(const DecodeParams& p) {
    static const StepPrefetch none{};
    return p.pre ? *p.pre : none;
}

}  // namespace pkv

namespace pkv {

// Row of the block-table array that holds launch slot `slot`'s table; -1 if
// the row index is out of range.
__device__ __forceinline__ long long table_row(const DecodeParams& p, int slot) {
    if (!p.table_rows) return slot;
    const int r = p.table_rows[slot];
    return (r >= 0 && r < p.n_table_rows) ? r : -1;
}

// The caller's sequence index of launch slot `slot`.
__device__ __forceinline__ int seq_of(const DecodeParams& p, int slot) {
    return p.order ? p.order[slot] : slot;
}

// Allow the kernel the device's whole opt-in shared memory per block (minus
// its static shared memory), once per device and kernel; occupancy follows
// the dynamic size given at each launch.
template <typename Kernel>
inline cudaError_t allow_large_smem(Kernel kern, unsigned long long* done_mask) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (__atomic_load_n(done_mask, __ATOMIC_ACQUIRE) & bit) return cudaSuccess;
    int optin = 0;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - (int)fa.sharedSizeBytes);
    if (e == cudaSuccess) __atomic_fetch_or(done_mask, bit, __ATOMIC_RELEASE);
    return e;
}

// Launch with or without programmatic dependent launch.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t st, bool pdl, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// After every thread of the CTA wrote its partition's partial state: count
// the partition as done; returns true in the CTA that finished last (it then
// sees every partial and has reset the counter for the next launch).
__device__ __forceinline__ bool finish_partition(int* counter, int nparts, int* flag_smem) {
    // the CTA barrier orders every thread's partial-state stores before thread
    // 0's device-scope fence (fences are cumulative), which orders them
    // before the counter update that other CTAs observe
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int prev = atomicAdd(counter, 1);
        const int last = prev == nparts - 1;
        if (last) {
            atomicExch(counter, 0);
            __threadfence();
        }
        *flag_smem = last;
    }
    __syncthreads();
    return *flag_smem != 0;
}

// Merge the partitions of heads h0 .. h0 + nh - 1 of one sequence inside the
// decode kernel (the CTA that finished last), with all partial (max, sum)
// pairs staged in shared memory first: two rounds of global loads in total.
// `scratch` holds at least 3 * nh * nparts + nh floats, else the heads are
// merged one after the other.
template <typename QT, int D>
__device__ void merge_in_cta(const DecodeParams& p, int seq, int h, int nparts);

template <typename QT, int D>
__device__ void merge_group_in_cta(const DecodeParams& p, int seq, int h0, int nh, int nparts,
                                   float* scratch, int scratch_floats) {
    const int n = nh * nparts;
    if (3 * n + nh > scratch_floats) {
        for (int hh = 0; hh < nh; ++hh) merge_in_cta<QT, D>(p, seq, h0 + hh, nparts);
        return;
    }
    float* ml = scratch;        // [nh][nparts][2]
    float* w = scratch + 2 * n; // [nh][nparts]
    float* linv = w + n;        // [nh]
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const size_t row = ((size_t)seq * p.H_q + h0 + i / nparts) * p.max_parts + i % nparts;
        ml[2 * i] = __ldcg(p.ws_ml + row * 2);
        ml[2 * i + 1] = __ldcg(p.ws_ml + row * 2 + 1);
    }
    __syncthreads();
    for (int hh = threadIdx.x; hh < nh; hh += blockDim.x) {
        float M = -INFINITY;
        for (int q = 0; q < nparts; ++q) M = fmaxf(M, ml[2 * (hh * nparts + q)]);
        float L = 0.f;
        for (int q = 0; q < nparts; ++q) {
            const int i = hh * nparts + q;
            const float wq = M == -INFINITY ? 0.f : exp2f(ml[2 * i] - M);
            w[i] = wq;
            L = fmaf(wq, ml[2 * i + 1], L);
        }
        linv[hh] = L > 0.f ? 1.f / L : 0.f;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < nh * D; i += blockDim.x) {
        const int hh = i / D, d = i % D;
        const size_t row0 = ((size_t)seq * p.H_q + h0 + hh) * p.max_parts;
        float O = 0.f;
        for (int q = 0; q < nparts; ++q)
            O = fmaf(w[hh * nparts + q], __ldcg(p.ws_acc + (row0 + q) * D + d), O);
        reinterpret_cast<QT*>(p.out)[((size_t)seq * p.H_q + h0 + hh) * D + d] =
            Elem<QT>::from_f(O * linv[hh]);
    }
}

// One head at a time (the fallback of merge_group_in_cta): threads stride
// over the D columns.
template <typename QT, int D>
__device__ void merge_in_cta(const DecodeParams& p, int seq, int h, int nparts) {
    const size_t row0 = ((size_t)seq * p.H_q + h) * p.max_parts;
    float M = -INFINITY;
    for (int q = 0; q < nparts; ++q) M = fmaxf(M, __ldcg(p.ws_ml + (row0 + q) * 2));
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
        float L = 0.f, O = 0.f;
        for (int q = 0; q < nparts && M != -INFINITY; ++q) {
            const float w = exp2f(__ldcg(p.ws_ml + (row0 + q) * 2) - M);
            L = fmaf(__ldcg(p.ws_ml + (row0 + q) * 2 + 1), w, L);
            O = fmaf(__ldcg(p.ws_acc + (row0 + q) * D + d), w, O);
        }
        reinterpret_cast<QT*>(p.out)[((size_t)seq * p.H_q + h) * D + d] =
            Elem<QT>::from_f(L > 0.f ? O / L : 0.f);
    }
}

// Tokens per partition of a c-token context split into n = ceil(c / P)
// partitions of equal length, rounded up to a whole 16-token stage (the last
// partition is shorter by less than 16 n tokens; (n - 1) * result < c since the
// result is at most P).  All partitions of a sequence then cost the same, so
// launching sequences in decreasing order of this length schedules the
// partitions longest first.  Host and device use the same formula.
__host__ __device__ __forceinline__ int balanced_part_tokens(int c, int P) {
    const int n = (c + P - 1) / P;
    const int per = (c + n - 1) / n;
    return (per + 15) & ~15;
}

}  // namespace pkv
