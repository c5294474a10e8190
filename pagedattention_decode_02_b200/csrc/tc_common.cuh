// Tensor-core building blocks of the grouped-head decode kernels (sm_100a):
// mma.sync m16n8k16 wrappers for f16/bf16 inputs with fp32 accumulation,
// ldmatrix loads, the 2-D tiled TMA load and the 128-byte swizzle of a staged
// 16-token tile, and the per-stage math (scores, online softmax, P.V) that the
// partitioned and the stage-balanced kernels share, for f16/bf16 pools and,
// converted in registers, FP8-E4M3 pools.
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
// Two 16 x 16 byte matrices, transposed: lanes 0-15 address the rows of the
// first, lanes 16-31 those of the second; per matrix this lane receives rows
// 4 (lane % 4) .. + 3 of column lane / 4 (one byte per row, in row order) in
// the first register and of column lane / 4 + 8 in the second.
__device__ __forceinline__ void ldsm_x2_t_b8(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                             uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m16n16.x2.trans.shared.b8 {%0,%1,%2,%3}, [%4];"
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

// The A fragments of one staged 16-token tile, read out of shared memory so
// that the ring slot can be refilled while the math uses them.
//   k[kk]: K rows (tokens) x d columns 16 kk .. 16 kk + 15 (S^T = K Q^T);
//   v[mt]: V^T rows d = 16 mt .. 16 mt + 15 x tokens (O^T += V^T P^T).
template <int D>
struct StageFrags {
    uint32_t k[D / 16][4];
    uint32_t v[D / 16][4];
};

// Fill f from the swizzled K and V tiles of a stage with n valid tokens.  V of
// the tokens past n may hold anything (stale or never-written rows): its
// values are replaced by 0, so that 0-weight tokens add 0 (not NaN).
template <int D>
__device__ __forceinline__ void stage_frags_t(const uint8_t* kt, const uint8_t* vt, int n,
                                              StageFrags<D>& f, int lane) {
    const uint32_t kbase = smem_addr(kt);
    const uint32_t vbase = smem_addr(vt);
    const int mi = lane >> 3, r8 = lane & 7;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
        ldsm_x4(kbase + swz((mi & 1) * 8 + r8, 2 * kk + (mi >> 1)), f.k[kk][0], f.k[kk][1],
                f.k[kk][2], f.k[kk][3]);
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt)
        ldsm_x4_t(vbase + swz((mi >> 1) * 8 + r8, 2 * mt + (mi & 1)), f.v[mt][0], f.v[mt][1],
                  f.v[mt][2], f.v[mt][3]);
    if (n < kStageTokens) {
        // registers 0/1 hold tokens 2 tq (low half) and 2 tq + 1 (high half),
        // registers 2/3 tokens 2 tq + 8 and 2 tq + 9
        const int t0 = 2 * (lane & 3);
        const uint32_t m01 = (t0 < n ? 0x0000ffffu : 0u) | (t0 + 1 < n ? 0xffff0000u : 0u);
        const uint32_t m23 = (t0 + 8 < n ? 0x0000ffffu : 0u) | (t0 + 9 < n ? 0xffff0000u : 0u);
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            f.v[mt][0] &= m01;
            f.v[mt][1] &= m01;
            f.v[mt][2] &= m23;
            f.v[mt][3] &= m23;
        }
    }
}

// Scores of one stage: S^T fragment (tokens gq, gq + 8; heads 2 tq, 2 tq + 1)
// scaled to base 2, tokens past n at -inf.
__device__ __forceinline__ void mask_scores(float (&s)[4], int n, int lane) {
    const int gq = lane >> 2;
    if (gq >= n) s[0] = s[1] = -INFINITY;
    if (gq + 8 >= n) s[2] = s[3] = -INFINITY;
}

// 2^x on the special-function unit (ex2.approx, flush-to-zero): its relative
// error (a few units in the last place of fp32) is far below the f16/bf16
// rounding of the probabilities it feeds; 2^-inf = 0.
__device__ __forceinline__ float ex2_fast(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Online-softmax update of one stage for this lane's two heads; returns P^T
// as the B operand of the P.V product (pb0 = tokens 0-7, pb1 = tokens 8-15)
// and rescales o and l when the running maxima move (lazily: only when a
// score exceeds its head's maximum by more than 2^8).
template <typename T, int MTILES>
__device__ __forceinline__ void softmax_step(const float (&s)[4], float (&o)[MTILES][4],
                                             float (&m_run)[2], float (&l_run)[2], uint32_t& pb0,
                                             uint32_t& pb1) {
    float mx[2] = {fmaxf(s[0], s[2]), fmaxf(s[1], s[3])};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 4));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 8));
        mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 16));
    }
    // lazy rescaling: the running maximum moves only when a new score
    // exceeds it by more than 2^8 (probabilities stay below 256, exact to the
    // f16/bf16 rounding of P); the whole warp moves together
    if (__any_sync(0xffffffffu, mx[0] > m_run[0] + 8.f || mx[1] > m_run[1] + 8.f)) {
        float alpha[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float m_new = fmaxf(m_run[h], mx[h]);
            alpha[h] = ex2_fast(m_run[h] - m_new);
            m_run[h] = m_new;
            l_run[h] *= alpha[h];
        }
#pragma unroll
        for (int mt = 0; mt < MTILES; ++mt) {
            o[mt][0] *= alpha[0];
            o[mt][1] *= alpha[1];
            o[mt][2] *= alpha[0];
            o[mt][3] *= alpha[1];
        }
    }
    const float p0 = ex2_fast(s[0] - m_run[0]);
    const float p1 = ex2_fast(s[1] - m_run[1]);
    const float p2 = ex2_fast(s[2] - m_run[0]);
    const float p3 = ex2_fast(s[3] - m_run[1]);
    l_run[0] += p0 + p2;
    l_run[1] += p1 + p3;
    pb0 = movmatrix_trans(MmaType<T>::pack(p0, p1));
    pb1 = movmatrix_trans(MmaType<T>::pack(p2, p3));
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
// + 8) for those two heads.
template <typename T, int D>
__device__ __forceinline__ void stage_math_t(const uint32_t (&qb)[D / 16][2],
                                             const StageFrags<D>& f, int n, float q_scale,
                                             float (&o)[D / 16][4], float (&m_run)[2],
                                             float (&l_run)[2], int lane) {
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = acc[a][2] = acc[a][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) MmaType<T>::mma(acc[kk & 3], f.k[kk], qb[kk][0], qb[kk][1]);
    float s[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) s[e] = ((acc[0][e] + acc[1][e]) + (acc[2][e] + acc[3][e])) * q_scale;
    if (n < 16) mask_scores(s, n, lane);
    uint32_t pb0, pb1;
    softmax_step<T, D / 16>(s, o, m_run, l_run, pb0, pb1);
#pragma unroll
    for (int mt = 0; mt < D / 16; ++mt) MmaType<T>::mma(o[mt], f.v[mt], pb0, pb1);
}

// stage_frags_t + stage_math_t with each fragment loaded next to its use
// (fewer live registers; the slot is released after the whole stage).
template <typename T, int D>
__device__ __forceinline__ void stage_body_t(const uint32_t (&qb)[D / 16][2], const uint8_t* kt,
                                             const uint8_t* vt, int n, float q_scale,
                                             float (&o)[D / 16][4], float (&m_run)[2],
                                             float (&l_run)[2], int lane) {
    const uint32_t kbase = smem_addr(kt);
    const uint32_t vbase = smem_addr(vt);
    const int mi = lane >> 3, r8 = lane & 7;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = acc[a][2] = acc[a][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t a[4];
        ldsm_x4(kbase + swz((mi & 1) * 8 + r8, 2 * kk + (mi >> 1)), a[0], a[1], a[2], a[3]);
        MmaType<T>::mma(acc[kk & 3], a, qb[kk][0], qb[kk][1]);
    }
    float s[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) s[e] = ((acc[0][e] + acc[1][e]) + (acc[2][e] + acc[3][e])) * q_scale;
    if (n < 16) mask_scores(s, n, lane);
    uint32_t pb0, pb1;
    softmax_step<T, D / 16>(s, o, m_run, l_run, pb0, pb1);
    if (n == kStageTokens) {
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            uint32_t a[4];
            ldsm_x4_t(vbase + swz((mi >> 1) * 8 + r8, 2 * mt + (mi & 1)), a[0], a[1], a[2], a[3]);
            MmaType<T>::mma(o[mt], a, pb0, pb1);
        }
    } else {
        // V of the tokens past n replaced by 0 (see stage_frags_t)
        const int t0 = 2 * (lane & 3);
        const uint32_t m01 = (t0 < n ? 0x0000ffffu : 0u) | (t0 + 1 < n ? 0xffff0000u : 0u);
        const uint32_t m23 = (t0 + 8 < n ? 0x0000ffffu : 0u) | (t0 + 9 < n ? 0xffff0000u : 0u);
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) {
            uint32_t a[4];
            ldsm_x4_t(vbase + swz((mi >> 1) * 8 + r8, 2 * mt + (mi & 1)), a[0], a[1], a[2], a[3]);
            a[0] &= m01;
            a[1] &= m01;
            a[2] &= m23;
            a[3] &= m23;
            MmaType<T>::mma(o[mt], a, pb0, pb1);
        }
    }
}

// ---------------------------------------------------------------------------
// FP8-E4M3 pools (d = 128, f16 queries): the stage's K and V tiles hold codes
// in 128-byte rows, converted to f16 in registers.  K: each lane reads its
// codes with four 16-byte loads, contiguous and free of bank conflicts, with
// the d index of the score contraction permuted (a sum over d in any order):
//   S^T k-step kk, fragment columns 2 tq + {0, 1} / 2 tq + {8, 9}
//       <-> d = 32 tq + 4 kk + {0, 1} / + {2, 3}.
// V: four transposing byte-matrix loads give each lane, per 16-column
// d-block, four consecutive tokens of one column, which are the A fragment's
// contraction indices 2 tq, + 1, + 8, + 9 once the stage's tokens are taken
// in that order on both products (fp8_token_of; K rows follow it too).
// ---------------------------------------------------------------------------

// Four FP8-E4M3 codes (one word, low byte first) -> two f16x2: lo = codes 0
// and 1, hi = codes 2 and 3; exact (every e4m3 value is an f16 value).  The
// word's 16-bit halves go to the converts as they are, with no shifts or masks.
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
    asm("{\n\t.reg .b16 a, b;\n\t"
        "mov.b32 {a, b}, %2;\n\t"
        "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
        "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
        : "=r"(lo), "=r"(hi)
        : "r"(w));
}

// Byte offset of the 16-byte chunk c (0..7) of row r in a 16-row tile of
// 128-byte rows staged with the 128-byte swizzle.
__device__ __forceinline__ uint32_t swz_chunk(int r, int c) {
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

// The contraction index r (0..15) of an FP8 stage and its token: the order
// in which the transposed byte-matrix load hands a lane a column's tokens
// (4 (lane % 4) .. + 3 = the indices 2 (lane % 4), + 1, + 8, + 9 of the
// f16 A fragment).
__device__ __forceinline__ int fp8_token_of(int r) {
    return 4 * ((r >> 1) & 3) + 2 * (r >> 3) + (r & 1);
}

// This lane's codes of one stage:
//   k[i][j]: K row fp8_token_of(gq + 8 i), bytes 32 tq + 16 j .. + 15;
//   v[jj]:   V transposed, d-blocks 2 jj (.x, .y) and 2 jj + 1 (.z, .w) of 16
//            columns: .x tokens 4 tq .. + 3 of column 16 (2 jj) + gq, .y the
//            same tokens of that column + 8 (likewise .z, .w); codes of
//            tokens at or past n are zero.
struct Fp8Raw {
    uint4 k[2][2];
    uint4 v[4];
};

__device__ __forceinline__ void stage_raw_fp8(const uint8_t* kt, const uint8_t* vt, int n,
                                              Fp8Raw& r, int lane) {
    const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j)
            r.k[i][j] = *reinterpret_cast<const uint4*>(
                kt + swz_chunk(fp8_token_of(gq + 8 * i), 2 * tq + j));
    const uint32_t vbase = smem_addr(vt);
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
        ldsm_x2_t_b8(vbase + swz_chunk(lane & 15, 2 * jj + (lane >> 4)), r.v[jj].x, r.v[jj].y,
                     r.v[jj].z, r.v[jj].w);
    if (n < kStageTokens) {
        const int valid = min(max(n - 4 * tq, 0), 4);   // of this lane's tokens 4 tq .. + 3
        const uint32_t m = valid >= 4 ? 0xffffffffu : ((1u << (8 * valid)) - 1u);
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            r.v[jj].x &= m;
            r.v[jj].y &= m;
            r.v[jj].z &= m;
            r.v[jj].w &= m;
        }
    }
}

// Q^T fragments for the permuted contraction: k-step kk, b0 = q[head][32 tq
// + 4 kk + {0, 1}], b1 = q[head][32 tq + 4 kk + {2, 3}], head = head_base +
// lane / 4, zero for heads >= n_heads.
__device__ __forceinline__ void load_qT_frags_fp8(uint32_t (&qb)[8][2], const __half* q,
                                                  int head_base, int n_heads, int lane) {
    const int h = head_base + (lane >> 2);
    const uint32_t* src = reinterpret_cast<const uint32_t*>(q + (size_t)h * 128 + 32 * (lane & 3));
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        qb[kk][0] = h < n_heads ? src[2 * kk] : 0u;
        qb[kk][1] = h < n_heads ? src[2 * kk + 1] : 0u;
    }
}

// The stage math of stage_math_t on an FP8 stage (scales folded by the
// caller: q_scale includes k_scale, the output is multiplied by v_scale), the
// stage's tokens taken in fp8_token_of order on both products.
// o[mt] = O^T rows d = 16 mt + gq (o[mt][0..1]) and + 8 (o[mt][2..3]).
__device__ __forceinline__ void stage_math_fp8(const uint32_t (&qb)[8][2], const Fp8Raw& r, int n,
                                               float q_scale, float (&o)[8][4],
                                               float (&m_run)[2], float (&l_run)[2], int lane) {
    float acc[2][4];
#pragma unroll
    for (int a = 0; a < 2; ++a) acc[a][0] = acc[a][1] = acc[a][2] = acc[a][3] = 0.f;
    const uint32_t* k0 = reinterpret_cast<const uint32_t*>(&r.k[0][0]);   // row gq, 8 words
    const uint32_t* k1 = reinterpret_cast<const uint32_t*>(&r.k[1][0]);   // row gq + 8
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        // word kk: d = 32 tq + 4 kk .. + 3
        uint32_t a[4];
        e4m3x4_to_f16x2(k0[kk], a[0], a[2]);
        e4m3x4_to_f16x2(k1[kk], a[1], a[3]);
        MmaType<__half>::mma(acc[kk & 1], a, qb[kk][0], qb[kk][1]);
    }
    float s[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) s[e] = (acc[0][e] + acc[1][e]) * q_scale;
    if (n < 16) {
        // rows gq and gq + 8 of S^T are tokens fp8_token_of(gq) and that + 2
        const int t0 = fp8_token_of(lane >> 2);
        if (t0 >= n) s[0] = s[1] = -INFINITY;
        if (t0 + 2 >= n) s[2] = s[3] = -INFINITY;
    }
    uint32_t pb0, pb1;
    softmax_step<__half, 8>(s, o, m_run, l_run, pb0, pb1);
    // V^T fragments straight from the transposed codes: a word's low and high
    // halves are a column's tokens at contraction indices 2 tq, + 1 and + 8, + 9
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
        uint32_t a[4];
        e4m3x4_to_f16x2(r.v[jj].x, a[0], a[2]);
        e4m3x4_to_f16x2(r.v[jj].y, a[1], a[3]);
        MmaType<__half>::mma(o[2 * jj], a, pb0, pb1);
        e4m3x4_to_f16x2(r.v[jj].z, a[0], a[2]);
        e4m3x4_to_f16x2(r.v[jj].w, a[1], a[3]);
        MmaType<__half>::mma(o[2 * jj + 1], a, pb0, pb1);
    }
}

}  // namespace tc
}  // namespace pkv
