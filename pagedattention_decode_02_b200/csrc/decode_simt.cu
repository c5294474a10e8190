// Paged decode attention on CUDA cores, and the log-sum-exp merge of
// split-context partitions.
//
// The operation ("KV 缓存与分页注意力" §一次写一个词元, §块表): for sequence i and
// query head h (KV head g = h / G) over the c_i stored tokens
//     out = sum_j softmax_j(scale * <q, K_j>) V_j,
// with K_j, V_j read block by block through the block table.
//
// Work decomposition: one CTA per (partition of the context, group of HPC
// query heads sharing one KV head, sequence).  Inside a CTA each of the 4
// warps owns every 4th stage of 16 tokens and runs its own ring of
// kStages shared-memory slots: one lane arms the slot's mbarrier with the
// stage's byte count, up to 32 lanes issue one 1-D bulk copy each (one per
// run of tokens inside one physical block, K and V), and the whole warp waits
// on the barrier.  Warps never synchronise with each other until the final
// combine.  Each (block, KV head) tile is contiguous in the pool
// ([num_blocks][H_kv][bs][d]), so a stage of 16 tokens at bs >= 16 is one
// copy for K and one for V.
//
// Scores: each lane owns d/32 consecutive elements of a row (q pre-scaled by
// scale * log2(e) in registers), so the row reads are conflict-free; the 16
// per-token partial dot products are combined with a butterfly
// reduce-scatter (8 + 4 + 2 + 1 + 1 shuffles), after which lane l holds the
// score of token l / 2.  Online softmax (running max and sum per warp) in
// base 2; V is accumulated with the probabilities broadcast by shuffles.
//
// Split context: with more than one partition, each CTA writes its
// (max, sum, unnormalised accumulator) to the workspace and the merge kernel
// combines them: M = max_p m_p, out = sum_p 2^(m_p - M) acc_p / sum_p 2^(m_p - M) l_p.
#include <cfloat>

#include "decode_launch.h"
#include "kernels_common.cuh"

namespace pkv {

namespace {

constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kStageTokens = 16;
constexpr int kStages = 3;

__device__ __forceinline__ float warp_max_xor2_16(float v) {
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
    return v;
}
__device__ __forceinline__ float warp_sum_xor2_16(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    v += __shfl_xor_sync(0xffffffffu, v, 16);
    return v;
}

// 16 per-lane partial sums (one per token) -> lane l holds the full sum of
// token l >> 1 (lanes l and l ^ 1 hold the same token).
__device__ __forceinline__ float reduce_scatter16(float (&p)[16], int lane) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const bool hi = lane & 16;
        float send = hi ? p[j] : p[j + 8];
        float keep = hi ? p[j + 8] : p[j];
        p[j] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const bool hi = lane & 8;
        float send = hi ? p[j] : p[j + 4];
        float keep = hi ? p[j + 4] : p[j];
        p[j] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const bool hi = lane & 4;
        float send = hi ? p[j] : p[j + 2];
        float keep = hi ? p[j + 2] : p[j];
        p[j] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    {
        const bool hi = lane & 2;
        float send = hi ? p[0] : p[1];
        float keep = hi ? p[1] : p[0];
        p[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
    return p[0] + __shfl_xor_sync(0xffffffffu, p[0], 1);
}

template <typename QT>
__device__ __forceinline__ float load_q(const QT* q, int i) {
    return Elem<QT>::to_f(q[i]);
}
template <>
__device__ __forceinline__ float load_q<float>(const float* q, int i) {
    return q[i];
}

template <typename KV, int D, int HPC>
struct SimtSmem {
    static constexpr int kRow = D * Elem<KV>::bytes;
    static constexpr int kTile = kStageTokens * kRow;                    // K or V of one stage
    static constexpr int kTilesBytes = kWarps * kStages * 2 * kTile;
    static constexpr int kBarOffset = kTilesBytes;
    static constexpr int kTableOffset = kBarOffset + kWarps * kStages * 8;
    __host__ __device__ static int comb_offset(int table_entries) {
        return (kTableOffset + table_entries * 4 + 15) & ~15;
    }
    __host__ __device__ static int bytes(int table_entries) {
        return comb_offset(table_entries) + kWarps * HPC * (D + 2) * 4;
    }
};

template <typename KV, typename QT, int D, int HPC>
__global__ void __launch_bounds__(kThreads)
decode_simt_kernel(const DecodeParams p, int table_entries) {
    using L = SimtSmem<KV, D, HPC>;
    constexpr int VEC = D / 32;
    constexpr int ROW = L::kRow;
    constexpr int TILE = L::kTile;
    static_assert(D % 32 == 0 && VEC >= 1 && VEC <= 4, "head_dim must be 32, 64 or 128");

    extern __shared__ __align__(1024) uint8_t smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
    int32_t* blk = reinterpret_cast<int32_t*>(smem + L::kTableOffset);
    float* comb = reinterpret_cast<float*>(smem + L::comb_offset(table_entries));

    const int part = blockIdx.x;
    const int h0 = blockIdx.y * HPC;
    const int slot = blockIdx.z;   // launch slot: length and table row
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int g = h0 / p.G;
    const int bs = p.block_size;
    const int P = p.part_tokens;

    const int c = p.lens[slot];
    const int seq = seq_of(p, slot);   // the caller's sequence: q, out, partials
    const int max_ctx = p.max_blocks * bs;
    if (c < 1 || c > max_ctx) {
        // invalid length: partition 0 zeroes the output, nothing is read
        if (part == 0) {
            if (tid == 0 && blockIdx.y == 0) report_error(p.err, PKV_DEVERR_CONTEXT_LEN);
            QT* out = reinterpret_cast<QT*>(p.out);
            for (int i = tid; i < HPC * D; i += kThreads)
                out[((size_t)seq * p.H_q + h0 + i / D) * D + i % D] = Elem<QT>::from_f(0.f);
        }
        return;
    }
    const int nparts = (c + P - 1) / P;
    if (part >= nparts) return;
    const int t_begin = part * P;
    const int t_end = min(c, t_begin + P);
    const int lb0 = t_begin / bs;
    const int n_lb = (t_end - 1) / bs - lb0 + 1;

    // the partition's block ids, validated once
    const long long trow = table_row(p, slot);
    bool bad = trow < 0;
    for (int i = tid; i < n_lb && trow >= 0; i += kThreads) {
        int32_t b = p.tables[trow * p.max_blocks + lb0 + i];
        bad |= (b < 0 || b >= p.num_blocks);
        blk[i] = b;
    }
    if (tid == 0) {
        for (int i = 0; i < kWarps * kStages; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    const bool any_bad = __syncthreads_or(bad);
    const bool split = nparts > 1;
    if (any_bad) {
        if (tid == 0 && blockIdx.y == 0) report_error(p.err, PKV_DEVERR_BLOCK_ID);
        // the partition contributes nothing
        for (int i = tid; i < HPC * D; i += kThreads) {
            const int h = h0 + i / D, d = i % D;
            const size_t row = ((size_t)seq * p.H_q + h) * p.max_parts + part;
            if (split) {
                p.ws_acc[row * D + d] = 0.f;
                if (d == 0) { p.ws_ml[row * 2] = -INFINITY; p.ws_ml[row * 2 + 1] = 0.f; }
            } else {
                reinterpret_cast<QT*>(p.out)[((size_t)seq * p.H_q + h) * D + d] = Elem<QT>::from_f(0.f);
            }
        }
        return;
    }

    const int n_stages = (t_end - t_begin + kStageTokens - 1) / kStageTokens;
    const int my_n = n_stages > warp ? (n_stages - warp + kWarps - 1) / kWarps : 0;
    uint8_t* my_tiles = smem + warp * kStages * 2 * TILE;
    uint64_t* my_bars = bars + warp * kStages;
    const uint64_t policy = l2_evict_first_policy();
    const uint8_t* kbase = p.k_pool + (long long)g * p.head_stride;
    const uint8_t* vbase = p.v_pool + (long long)g * p.head_stride;

    auto issue = [&](int k_local, int slot) {
        const int s = warp + k_local * kWarps;
        const int a = t_begin + s * kStageTokens;
        const int n = min(kStageTokens, t_end - a);
        uint8_t* kd = my_tiles + slot * 2 * TILE;
        uint8_t* vd = kd + TILE;
        if (lane == 0) mbar_arrive_expect_tx(&my_bars[slot], (uint32_t)(2 * n * ROW));
        __syncwarp();
        const int lb_first = a / bs;
        const int nch = (a + n - 1) / bs - lb_first + 1;  // <= 16
        if (lane < 2 * nch) {
            const int which = lane >= nch;
            const int lb = lb_first + (which ? lane - nch : lane);
            const int ta = max(a, lb * bs);
            const int tb = min(a + n, (lb + 1) * bs);
            const long long off = (long long)blk[lb - lb0] * p.block_stride + (long long)(ta - lb * bs) * ROW;
            fence_proxy_async_smem();
            bulk_load((which ? vd : kd) + (ta - a) * ROW, (which ? vbase : kbase) + off,
                      (uint32_t)((tb - ta) * ROW), &my_bars[slot], policy);
        }
    };

    // q of this CTA's heads, pre-scaled (scale * log2 e * FP8 K scale)
    float qf[HPC][VEC];
    const QT* qp = reinterpret_cast<const QT*>(p.q);
#pragma unroll
    for (int h = 0; h < HPC; ++h)
#pragma unroll
        for (int v = 0; v < VEC; ++v)
            qf[h][v] = load_q<QT>(qp, ((size_t)seq * p.H_q + h0 + h) * D + lane * VEC + v) * p.q_scale;

    float m[HPC], l[HPC], acc[HPC][VEC];
#pragma unroll
    for (int h = 0; h < HPC; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[h][v] = 0.f;
    }

    const int pro = min(kStages, my_n);
    for (int k = 0; k < pro; ++k) issue(k, k);

    int k = 0;
    bool timed_out = false;
    for (; k < my_n; ++k) {
        const int slot = k % kStages;
        if (!mbar_wait(&my_bars[slot], (uint32_t)((k / kStages) & 1), p.wait_ns)) {
            timed_out = true;
            break;
        }
        const int s = warp + k * kWarps;
        const int a = t_begin + s * kStageTokens;
        const int n = min(kStageTokens, t_end - a);
        const uint8_t* kt = my_tiles + slot * 2 * TILE;
        const uint8_t* vt = kt + TILE;
        const int tok = lane >> 1;
#pragma unroll
        for (int h = 0; h < HPC; ++h) {
            float part_s[kStageTokens];
#pragma unroll
            for (int t = 0; t < kStageTokens; ++t) {
                float kf[VEC];
                if (t < n) {
                    VecLoad<KV, VEC>::run(kt + t * ROW + lane * VEC * Elem<KV>::bytes, kf);
                } else {
#pragma unroll
                    for (int v = 0; v < VEC; ++v) kf[v] = 0.f;
                }
                float acc_t = 0.f;
#pragma unroll
                for (int v = 0; v < VEC; ++v) acc_t = fmaf(qf[h][v], kf[v], acc_t);
                part_s[t] = acc_t;
            }
            float sc = reduce_scatter16(part_s, lane);
            sc = tok < n ? sc : -INFINITY;
            const float m_new = fmaxf(m[h], warp_max_xor2_16(sc));
            const float alpha = exp2f(m[h] - m_new);
            const float pr = tok < n ? exp2f(sc - m_new) : 0.f;
            l[h] = l[h] * alpha + warp_sum_xor2_16(pr);
#pragma unroll
            for (int v = 0; v < VEC; ++v) acc[h][v] *= alpha;
#pragma unroll
            for (int t = 0; t < kStageTokens; ++t) {
                const float pt = __shfl_sync(0xffffffffu, pr, 2 * t);
                if (t < n) {
                    float vf[VEC];
                    VecLoad<KV, VEC>::run(vt + t * ROW + lane * VEC * Elem<KV>::bytes, vf);
#pragma unroll
                    for (int v = 0; v < VEC; ++v) acc[h][v] = fmaf(pt, vf[v], acc[h][v]);
                }
            }
            m[h] = m_new;
        }
        __syncwarp();
        if (k + kStages < my_n) issue(k + kStages, slot);
    }
    if (timed_out) {
        if (lane == 0) report_error(p.err, PKV_DEVERR_TIMEOUT);
        // let the copies still in flight land before the CTA exits (bounded)
        for (int j = k; j < min(my_n, k + kStages); ++j)
            (void)mbar_wait(&my_bars[j % kStages], (uint32_t)((j / kStages) & 1));
    }

    // combine the warps' softmax states
#pragma unroll
    for (int h = 0; h < HPC; ++h) {
        float* cw = comb + (warp * HPC + h) * (D + 2);
#pragma unroll
        for (int v = 0; v < VEC; ++v) cw[lane * VEC + v] = acc[h][v];
        if (lane == 0) {
            cw[D] = m[h];
            cw[D + 1] = l[h];
        }
    }
    __syncthreads();
    for (int i = tid; i < HPC * D; i += kThreads) {
        const int h = i / D, d = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, comb[(w * HPC + h) * (D + 2) + D]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float* cw = comb + (w * HPC + h) * (D + 2);
            const float wt = exp2f(cw[D] - M);
            L = fmaf(cw[D + 1], wt, L);
            O = fmaf(cw[d], wt, O);
        }
        O *= p.v_scale;
        if (split) {
            const size_t row = ((size_t)seq * p.H_q + h0 + h) * p.max_parts + part;
            p.ws_acc[row * D + d] = O;
            if (d == 0) {
                p.ws_ml[row * 2] = M;
                p.ws_ml[row * 2 + 1] = L;
            }
        } else {
            reinterpret_cast<QT*>(p.out)[((size_t)seq * p.H_q + h0 + h) * D + d] = Elem<QT>::from_f(O / L);
        }
    }
}

// Merge the partitions of one (sequence, head) per warp, 8 heads per CTA:
// M = max_p m_p, out = sum_p 2^(m_p - M) acc_p / sum_p 2^(m_p - M) l_p.  Lane
// l holds D/32 consecutive columns; the partitions' (m, l) pairs are read 32
// at a time, one per lane, and broadcast by shuffles.
constexpr int kMergeWarps = 8;

template <typename QT, int D>
__global__ void __launch_bounds__(kMergeWarps * 32)
merge_kernel(const DecodeParams p) {
    constexpr int VEC = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x * kMergeWarps + warp;
    const int slot = blockIdx.y;
    grid_dependency_wait();   // the decode kernel's partials (programmatic launch)
    if (h >= p.H_q) return;
    const int c = p.lens[slot];
    const int seq = seq_of(p, slot);
    if (c < 1 || c > p.max_blocks * p.block_size) return;   // zeroed by the decode kernel
    const int nparts = (c + p.part_tokens - 1) / p.part_tokens;
    if (nparts <= 1) return;                                   // written by the decode kernel
    const size_t row0 = ((size_t)seq * p.H_q + h) * p.max_parts;
    float M = -INFINITY;
    for (int q0 = 0; q0 < nparts; q0 += 32) {
        const float m = q0 + lane < nparts ? p.ws_ml[(row0 + q0 + lane) * 2] : -INFINITY;
        M = fmaxf(M, m);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
    if (M != -INFINITY) {
        for (int q0 = 0; q0 < nparts; q0 += 32) {
            const int qi = q0 + lane;
            float w = 0.f, lw = 0.f;
            if (qi < nparts) {
                w = exp2f(p.ws_ml[(row0 + qi) * 2] - M);
                lw = w * p.ws_ml[(row0 + qi) * 2 + 1];
            }
            L += lw;
            const int cnt = min(32, nparts - q0);
            for (int j = 0; j < cnt; ++j) {
                const float wj = __shfl_sync(0xffffffffu, w, j);
                const float* a = p.ws_acc + (row0 + q0 + j) * D + lane * VEC;
                float f[VEC];
                if constexpr (VEC == 4) {
                    const float4 u = *reinterpret_cast<const float4*>(a);
                    f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
                } else if constexpr (VEC == 2) {
                    const float2 u = *reinterpret_cast<const float2*>(a);
                    f[0] = u.x; f[1] = u.y;
                } else {
                    f[0] = a[0];
                }
#pragma unroll
                for (int v = 0; v < VEC; ++v) acc[v] = fmaf(wj, f[v], acc[v]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    }
    QT* out = reinterpret_cast<QT*>(p.out) + ((size_t)seq * p.H_q + h) * D + lane * VEC;
#pragma unroll
    for (int v = 0; v < VEC; ++v) out[v] = Elem<QT>::from_f(L > 0.f ? acc[v] / L : 0.f);
}

template <typename KV, typename QT, int D, int HPC>
cudaError_t launch_simt_t(const DecodeParams& p, cudaStream_t st, cudaEvent_t mid) {
    using L = SimtSmem<KV, D, HPC>;
    const int table_entries = p.part_tokens / p.block_size + 2;
    const int smem = L::bytes(table_entries);
    auto kern = decode_simt_kernel<KV, QT, D, HPC>;
    static unsigned long long attr_done = 0;
    cudaError_t e = allow_large_smem(kern, &attr_done);
    if (e != cudaSuccess) return e;
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    dim3 grid(p.max_parts, p.H_q / HPC, p.B);
    kern<<<grid, kThreads, smem, st>>>(p, table_entries);
    e = cudaGetLastError();
    if (e == cudaSuccess && mid) e = cudaEventRecord(mid, st);
    if (e != cudaSuccess || p.max_parts <= 1) return e;
    return launch_merge(p, Elem<QT>::id, D, st);
}

template <typename KV, typename QT, int D>
cudaError_t launch_simt_d(const DecodeParams& p, int hpc, cudaStream_t st, cudaEvent_t mid) {
    switch (hpc) {
        case 1: return launch_simt_t<KV, QT, D, 1>(p, st, mid);
        case 2: return launch_simt_t<KV, QT, D, 2>(p, st, mid);
        case 4: return launch_simt_t<KV, QT, D, 4>(p, st, mid);
        case 8: return launch_simt_t<KV, QT, D, 8>(p, st, mid);
        default: return cudaErrorInvalidValue;
    }
}

template <typename KV, typename QT>
cudaError_t launch_simt_q(const DecodeParams& p, int D, int hpc, cudaStream_t st, cudaEvent_t mid) {
    switch (D) {
        case 32: return launch_simt_d<KV, QT, 32>(p, hpc, st, mid);
        case 64: return launch_simt_d<KV, QT, 64>(p, hpc, st, mid);
        case 128: return launch_simt_d<KV, QT, 128>(p, hpc, st, mid);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_merge(const DecodeParams& p, int q_dtype, int D, cudaStream_t st) {
    const dim3 grid((p.H_q + kMergeWarps - 1) / kMergeWarps, p.B);
    cudaError_t e = cudaSuccess;
#define PKV_MERGE(QT, DD) \
    e = launch_kernel(merge_kernel<QT, DD>, grid, dim3(kMergeWarps * 32), 0, st, p.pdl != 0, p)
    if (q_dtype == PKV_F32) {
        if (D == 32) PKV_MERGE(float, 32); else if (D == 64) PKV_MERGE(float, 64); else PKV_MERGE(float, 128);
    } else if (q_dtype == PKV_F16) {
        if (D == 32) PKV_MERGE(__half, 32); else if (D == 64) PKV_MERGE(__half, 64); else PKV_MERGE(__half, 128);
    } else {
        if (D == 32) PKV_MERGE(__nv_bfloat16, 32); else if (D == 64) PKV_MERGE(__nv_bfloat16, 64);
        else PKV_MERGE(__nv_bfloat16, 128);
    }
#undef PKV_MERGE
    return e;
}

int simt_heads_per_cta(int group) {
    for (int h : {8, 4, 2})
        if (group % h == 0) return h;
    return 1;
}

size_t simt_smem_bytes(int kv_dtype, int D, int hpc, int part_tokens, int block_size) {
    const int te = part_tokens / block_size + 2;
    const int eb = kv_dtype == PKV_F32 ? 4 : kv_dtype == PKV_FP8_E4M3 ? 1 : 2;
    const int tiles = kWarps * kStages * 2 * kStageTokens * D * eb;
    const int comb = ((tiles + kWarps * kStages * 8 + te * 4) + 15) & ~15;
    return (size_t)comb + (size_t)kWarps * hpc * (D + 2) * 4;
}

cudaError_t launch_decode_simt(const DecodeParams& p, int kv_dtype, int q_dtype, int D, int hpc,
                               cudaStream_t st, cudaEvent_t mid) {
    switch (kv_dtype) {
        case PKV_F32: return launch_simt_q<float, float>(p, D, hpc, st, mid);
        case PKV_F16: return launch_simt_q<__half, __half>(p, D, hpc, st, mid);
        case PKV_BF16: return launch_simt_q<__nv_bfloat16, __nv_bfloat16>(p, D, hpc, st, mid);
        case PKV_FP8_E4M3:
            if (q_dtype == PKV_F16) return launch_simt_q<fp8e4m3, __half>(p, D, hpc, st, mid);
            if (q_dtype == PKV_BF16) return launch_simt_q<fp8e4m3, __nv_bfloat16>(p, D, hpc, st, mid);
            return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkv
