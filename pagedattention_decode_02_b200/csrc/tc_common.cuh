// Tensor-core building blocks of the grouped-head decode kernels (sm_100a):
// mma.sync m16n8k16 wrappers for f16/bf16 inputs with fp32 accumulation,
// ldmatrix loads, the 2-D tiled TMA load and the 128-byte swizzle of a staged
// 16-token tile, and the per-stage body (scores, online softmax, P.V) that the
// partitioned and the stage-balanced kernels share.
#pragma once

#include <cuda.h>

#include "kernels_common.cuh"

namespace pkv {
namespace tc {

constexpr int kStageTokens = 16;

template <typename T>
struct MmaType;
template <>
struct MmaType<__half> {
    __device__ static uint32_t pack(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __device__ static void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
};
template <>
struct MmaType<__nv_bfloat16> {
    __device__ static uint32_t pack(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __device__ static void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
            "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// 2-D tiled TMA load of one box into shared memory, completion on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Byte offset of 16-byte chunk c (of the row's d / 8 chunks) in row r of a
// swizzled stage tile: [d / 64 halves][16 rows][128 B], chunk index XOR (r % 8).
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)((c >> 3) * (kStageTokens * 128) + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}


// Q fragments (mma A operand) of one warp's 16 query-head rows: rows
// r0 = row_base + lane / 4 and r0 + 8 of the [rows][D] block at q, zero for
// rows >= n_rows.
template <typename T, int D>
__device__ __forceinline__ void load_q_frags(uint32_t (&qa)[D / 16][4], const T* q, int row_base,
                                             int n_rows, int lane) {
    const int r0 = row_base + (lane >> 2), r1 = r0 + 8;
    const int tq = lane & 3;
    const T* q0 = q + (size_t)r0 * D;
    const T* q1 = q + (size_t)r1 * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int c0 = kk * 16 + 2 * tq;
        qa[kk][0] = r0 < n_rows ? *reinterpret_cast<const uint32_t*>(q0 + c0) : 0u;
        qa[kk][1] = r1 < n_rows ? *reinterpret_cast<const uint32_t*>(q1 + c0) : 0u;
        qa[kk][2] = r0 < n_rows ? *reinterpret_cast<const uint32_t*>(q0 + c0 + 8) : 0u;
        qa[kk][3] = r1 < n_rows ? *reinterpret_cast<const uint32_t*>(q1 + c0 + 8) : 0u;
    }
}

// One 16-token stage for one warp's 16 head rows:
//     S = Q K_stage^T (q_scale folds the softmax scale and log2 e), online
//     softmax per row in base 2, O = alpha O + P V_stage.
// kt / vt: the stage's swizzled K and V tiles; n (1..16) tokens are valid.
// V rows past n hold stale bytes and are zeroed first (every warp zeroes its
// own view; the values are identical, so overlapping writes are harmless),
// then a proxy fence, since the async proxy refills the slot later.  Scores
// of tokens past n are -inf, so P is exactly 0 there.
template <typename T, int D>
__device__ __forceinline__ void stage_body(const uint32_t (&qa)[D / 16][4], uint8_t* kt,
                                           uint8_t* vt, int n, float q_scale,
                                           float (&o)[D / 8][4], float (&m_run)[2],
                                           float (&l_run)[2], int lane) {
    constexpr int KSTEPS = D / 16;
    constexpr int DTILES = D / 8;
    const int tq = lane & 3;
    if (n < kStageTokens) {
        for (int i = lane; i < (kStageTokens - n) * (D / 8); i += 32) {
            const int r = n + i / (D / 8), cc = i % (D / 8);
            *reinterpret_cast<uint4*>(vt + swz(r, cc)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
    }
    const uint32_t kbase = smem_addr(kt);
    const uint32_t vbase = smem_addr(vt);

    // S = Q K^T : two n-tiles of 8 tokens; even and odd k-steps go to
    // separate accumulators to halve the dependent mma chain
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
        float s2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const int mi = lane >> 3, r = lane & 7;
        const int tok = (mi >> 1) * 8 + r;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(kbase + swz(tok, 2 * kk + (mi & 1)), b0, b1, b2, b3);
            if (kk & 1) {
                MmaType<T>::mma(s2[0], qa[kk], b0, b1);
                MmaType<T>::mma(s2[1], qa[kk], b2, b3);
            } else {
                MmaType<T>::mma(s[0], qa[kk], b0, b1);
                MmaType<T>::mma(s[1], qa[kk], b2, b3);
            }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) s[j][e] += s2[j][e];
    }
    // online softmax over this stage's tokens, per head row (lane / 4, + 8)
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int tok = 8 * j + 2 * tq + (e & 1);
            float v = s[j][e] * q_scale;
            v = tok < n ? v : -INFINITY;
            s[j][e] = v;
            mx[e >> 1] = fmaxf(mx[e >> 1], v);
        }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
        mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
        const float m_new = fmaxf(m_run[r], mx[r]);
        alpha[r] = exp2f(m_run[r] - m_new);
        m_run[r] = m_new;
        l_run[r] *= alpha[r];
    }
    uint32_t pa[4];
    {
        float pr[2][4];
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                pr[j][e] = exp2f(s[j][e] - m_run[e >> 1]);
                l_run[e >> 1] += pr[j][e];
            }
        pa[0] = MmaType<T>::pack(pr[0][0], pr[0][1]);
        pa[1] = MmaType<T>::pack(pr[0][2], pr[0][3]);
        pa[2] = MmaType<T>::pack(pr[1][0], pr[1][1]);
        pa[3] = MmaType<T>::pack(pr[1][2], pr[1][3]);
    }
    // rescale the accumulator only when some row's running max moved
    // (alpha == 1 exactly otherwise): late in a sequence it rarely does
    if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
        for (int j = 0; j < DTILES; ++j) {
            o[j][0] *= alpha[0];
            o[j][1] *= alpha[0];
            o[j][2] *= alpha[1];
            o[j][3] *= alpha[1];
        }
    }
    // O += P V : V^T fragments by transposed ldmatrix, two d-tiles per load
    {
        const int mi = lane >> 3, r = lane & 7;
        const int tok = (mi & 1) * 8 + r;
#pragma unroll
        for (int j = 0; j < DTILES; j += 2) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(vbase + swz(tok, j + (mi >> 1)), b0, b1, b2, b3);
            MmaType<T>::mma(o[j], pa, b0, b1);
            MmaType<T>::mma(o[j + 1], pa, b2, b3);
        }
    }
}


// Transpose of an 8x8 b16 matrix held one 32-bit pair per lane in the mma
// fragment layout (row lane / 4, columns 2 (lane % 4) and + 1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

// Q^T fragments (mma B operand, K = d, N = 8 heads) of heads head_base ..
// head_base + 7 of the [heads][D] block at q: per 16-wide k-step, the pairs
// (d = 16 kk + 2 (lane % 4), + 1) and (+ 8, + 9) of head head_base + lane / 4;
// zero for heads >= n_heads.
template <typename T, int D>
__device__ __forceinline__ void load_qT_frags(uint32_t (&qb)[D / 16][2], const T* q, int head_base,
                                              int n_heads, int lane) {
    const int h = head_base + (lane >> 2);
    const int tq = lane & 3;
    const T* qh = q + (size_t)h * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        const int c0 = kk * 16 + 2 * tq;
        qb[kk][0] = h < n_heads ? *reinterpret_cast<const uint32_t*>(qh + c0) : 0u;
        qb[kk][1] = h < n_heads ? *reinterpret_cast<const uint32_t*>(qh + c0 + 8) : 0u;
    }
}

// One 16-token stage for one warp's 8 query heads, in transposed form (no
// padded rows when a KV head has 8 or fewer query heads):
//     S^T [16 tokens][8 heads] = K_stage Q^T,
//     online softmax per head (column) in base 2,
//     O^T [D][8 heads] = alpha O^T + V_stage^T P^T.
// P^T moves from the accumulator layout to the B-operand layout with two 8x8
// transposes (movmatrix).  This lane holds heads 2 (lane % 4) and + 1:
// m_run / l_run (l partial over this lane's tokens, summed over the lanes of
// the same lane % 4 at the end), o[mt] = O^T rows d = 16 mt + lane / 4 (and
// + 8) for those two heads.  Same staging and zeroing rules as stage_body.
template <typename T, int D>
__device__ __forceinline__ void stage_body_t(const uint32_t (&qb)[D / 16][2], uint8_t* kt,
                                             uint8_t* vt, int n, float q_scale,
                                             float (&o)[D / 16][4], float (&m_run)[2],
                                             float (&l_run)[2], int lane) {
    constexpr int KSTEPS = D / 16;
    const int gq = lane >> 2;
    if (n < kStageTokens) {
        for (int i = lane; i < (kStageTokens - n) * (D / 8); i += 32) {
            const int r = n + i / (D / 8), cc = i % (D / 8);
            *reinterpret_cast<uint4*>(vt + swz(r, cc)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
    }
    const uint32_t kbase = smem_addr(kt);
    const uint32_t vbase = smem_addr(vt);
    const int mi = lane >> 3, r8 = lane & 7;

    // S^T = K Q^T over the d k-steps, four interleaved accumulators
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = acc[a][2] = acc[a][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
        uint32_t a[4];
        ldsm_x4(kbase + swz((mi & 1) * 8 + r8, 2 * kk + (mi >> 1)), a[0], a[1], a[2], a[3]);
        MmaType<T>::mma(acc[kk & 3], a, qb[kk][0], qb[kk][1]);
    }
    float s[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) s[e] = ((acc[0][e] + acc[1][e]) + (acc[2][e] + acc[3][e])) * q_scale;
    // tokens gq (s[0], s[1]) and gq + 8 (s[2], s[3]); heads 2 tq (even e), 2 tq + 1
    if (gq >= n) s[0] = s[1] = -INFINITY;
    if (gq + 8 >= n) s[2] = s[3] = -INFINITY;
    float mx[2] = {fmaxf(s[0], s[2]), fmaxf(s[1], s[3])};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 4));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 8));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 16));
    }
    float alpha[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const float m_new = fmaxf(m_run[h], mx[h]);
        alpha[h] = exp2f(m_run[h] - m_new);
        m_run[h] = m_new;
    }
    const float p0 = exp2f(s[0] - m_run[0]);
    const float p1 = exp2f(s[1] - m_run[1]);
    const float p2 = exp2f(s[2] - m_run[0]);
    const float p3 = exp2f(s[3] - m_run[1]);
    l_run[0] = l_run[0] * alpha[0] + (p0 + p2);
    l_run[1] = l_run[1] * alpha[1] + (p1 + p3);
    // P^T as the B operand: b0 = tokens 0-7, b1 = tokens 8-15
    const uint32_t pb0 = movmatrix_trans(MmaType<T>::pack(p0, p1));
    const uint32_t pb1 = movmatrix_trans(MmaType<T>::pack(p2, p3));
    if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            o[mt][0] *= alpha[0];
            o[mt][1] *= alpha[1];
            o[mt][2] *= alpha[0];
            o[mt][3] *= alpha[1];
        }
    }
    // O^T += V^T P^T: one m-tile of 16 d rows per transposed ldmatrix
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) {
        uint32_t a[4];
        ldsm_x4_t(vbase + swz((mi >> 1) * 8 + r8, 2 * mt + (mi & 1)), a[0], a[1], a[2], a[3]);
        MmaType<T>::mma(o[mt], a, pb0, pb1);
    }
}

}  // namespace tc
}  // namespace pkv
