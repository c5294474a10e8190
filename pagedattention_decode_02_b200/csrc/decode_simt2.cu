// Paged decode attention on CUDA cores, one query head per CTA, with
// swizzled TMA staging (the kernel used when the pool has row tensor maps:
// rows of 128, 256 or 512 bytes and a power-of-two block size).
//
// The operation is the one of decode_simt.cu ("KV 缓存与分页注意力"
// §一次写一个词元, §块表): out = sum_j softmax_j(scale <q, K_j>) V_j over the
// sequence's stored tokens, read block by block through the table.
//
// What changes against decode_simt.cu is the mapping of work to lanes, made
// possible by the 128-byte swizzle of the staged tiles:
// * scores: lane l takes token l % 16 and half of its row (l / 16), so no
//   cross-lane reduction is needed beyond one shuffle joining the two halves;
//   the 8 lanes of a shared-memory phase read 8 consecutive rows at the same
//   logical 16-byte chunk, which the swizzle spreads over 8 bank groups;
// * values: lane l owns d/32 consecutive columns of every row (also
//   conflict-free), the 16 probabilities reach every lane through a 64-byte
//   broadcast buffer in shared memory instead of 16 shuffles;
// * products are accumulated with packed fp32x2 FMAs.
// Each warp still owns every W-th 16-token stage of its CTA's partition and a
// private ring of S slots filled by 2-D TMA boxes (K and V, 128-byte inner
// box, min(bs, 16) rows), armed by one lane and issued by up to 32 lanes.
#include <cuda.h>

#include <cfloat>

#include "decode_launch.h"
#include "kernels_common.cuh"

namespace pkv {

namespace {

constexpr int kTok = 16;   // tokens per stage

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// 16 bytes of a row as floats (8 halves / 4 floats / 16 fp8 codes)
template <typename KV>
struct Chunk;
template <>
struct Chunk<__half> {
    static constexpr int N = 8;
    __device__ static void load(const uint8_t* p, float* f) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
            f[2 * i] = a.x;
            f[2 * i + 1] = a.y;
        }
    }
};
template <>
struct Chunk<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const uint8_t* p, float* f) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
    }
};
template <>
struct Chunk<float> {
    static constexpr int N = 4;
    __device__ static void load(const uint8_t* p, float* f) {
        const float4 u = *reinterpret_cast<const float4*>(p);
        f[0] = u.x; f[1] = u.y; f[2] = u.z; f[3] = u.w;
    }
};
template <>
struct Chunk<fp8e4m3> {
    static constexpr int N = 16;
    __device__ static void load(const uint8_t* p, float* f) {
        const uint4 u = *reinterpret_cast<const uint4*>(p);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 a = e4m3x2_to_float2((uint16_t)(w[i] & 0xFFFF));
            const float2 b = e4m3x2_to_float2((uint16_t)(w[i] >> 16));
            f[4 * i] = a.x; f[4 * i + 1] = a.y; f[4 * i + 2] = b.x; f[4 * i + 3] = b.y;
        }
    }
};

template <typename KV, int D, int W, int S>
struct Simt2Smem {
    static constexpr int kRow = D * Elem<KV>::bytes;
    static constexpr int kParts = kRow / 128;           // 128-byte column boxes per row
    static constexpr int kTile = kTok * kRow;           // K (or V) of one stage
    static constexpr int kSlot = 2 * kTile;
    static constexpr int kTiles = W * S * kSlot;
    static constexpr int kBars = kTiles;                 // W * S mbarriers
    static constexpr int kPbuf = kBars + W * S * 8;      // W x 16 floats
    static constexpr int kTable = kPbuf + W * kTok * 4;
    __host__ __device__ static int comb(int te) { return (kTable + te * 4 + 15) & ~15; }
    __host__ __device__ static int bytes(int te) { return 1024 + comb(te) + W * (D + 2) * 4; }
};

template <typename KV, typename QT, int D, int W, int S>
__global__ void __launch_bounds__(W * 32)
decode_simt2_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p,
                    const __grid_constant__ StepPrefetch pf, int table_entries, int bs_shift) {
    using L = Simt2Smem<KV, D, W, S>;
    constexpr int NT = W * 32;
    constexpr int PARTS = L::kParts;                 // 1, 2 or 4
    constexpr int TILE = L::kTile;
    constexpr int SLOT = L::kSlot;
    constexpr int EB = Elem<KV>::bytes;
    constexpr int CPR = PARTS * 8;                   // 16-byte chunks per row
    constexpr int CPL = CPR / 2;                     // chunks per lane for the scores
    constexpr int EPC = Chunk<KV>::N;                // elements per chunk
    constexpr int VEC = D / 32;                      // value columns per lane
    static_assert(PARTS == 1 || PARTS == 2 || PARTS == 4, "row of 128/256/512 bytes");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
    float* pbuf_all = reinterpret_cast<float*>(smem + L::kPbuf);
    int32_t* blk = reinterpret_cast<int32_t*>(smem + L::kTable);
    float* comb = reinterpret_cast<float*>(smem + L::comb(table_entries));

    const int part = blockIdx.x;
    const int h = blockIdx.y;
    const int slot = blockIdx.z;   // launch slot: length and table row
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int g = h / p.G;
    const int bs = 1 << bs_shift;
    const int P = p.part_tokens;

    __shared__ int last_flag;
    // Lengths, tables, rows and the launch order come from the preceding
    // kernel.  A launch slot that the host's prefetch block covers takes its
    // length, row and sequence from there, and loads the table entries below
    // its stable count, the stages they cover and its query before waiting
    // for that kernel.
    const bool pre = slot < pf.n;
    long long trow;
    int c, seq;   // seq: the caller's sequence (q, out, partials)
    if (pre) {
        const int r = pf.rows[slot];
        trow = (r >= 0 && r < p.n_table_rows) ? r : -1;
        c = pf.lens[slot];
        seq = pf.order[slot];
    } else {
        grid_dependency_wait();
        trow = table_row(p, slot);   // issued together with the length load
        c = p.lens[slot];
        seq = seq_of(p, slot);
    }
    if (c < 1 || c > p.max_blocks * bs) {
        if (pre) grid_dependency_wait();
        if (part == 0) {
            if (tid == 0 && h == 0) report_error(p.err, PKV_DEVERR_CONTEXT_LEN);
            QT* out = reinterpret_cast<QT*>(p.out);
            for (int i = tid; i < D; i += NT)
                out[((size_t)seq * p.H_q + h) * D + i] = Elem<QT>::from_f(0.f);
        }
        return;
    }
    const int nparts = (c + P - 1) / P;
    if (part >= nparts) return;
    const int Ps = balanced_part_tokens(c, P);
    const int t_begin = part * Ps;
    const int t_end = min(c, t_begin + Ps);
    const int lb0 = t_begin >> bs_shift;
    const int n_lb = ((t_end - 1) >> bs_shift) - lb0 + 1;
    // table entries final before the preceding kernel ends
    const int n_pre = pre ? max(0, min(n_lb, pf.stable[slot] - lb0)) : n_lb;

    bool bad = trow < 0;
    for (int i = tid; i < n_pre && trow >= 0; i += NT) {
        const int32_t b = p.tables[trow * p.max_blocks + lb0 + i];
        bad |= (b < 0 || b >= p.num_blocks);
        blk[i] = b;
    }
    if (tid == 0) {
        for (int i = 0; i < W * S; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    bad = __syncthreads_or(bad);

    const int n_stages = (t_end - t_begin + kTok - 1) / kTok;
    const int my_n = n_stages > warp ? (n_stages - warp + W - 1) / W : 0;
    uint8_t* ring = smem + warp * S * SLOT;
    uint64_t* my_bars = bars + warp * S;
    float* pbuf = pbuf_all + warp * kTok;
    const uint64_t policy = l2_evict_first_policy();
    const int rpb_shift = bs_shift < 4 ? bs_shift : 4;   // rows per box = min(bs, 16)
    const int rpb = 1 << rpb_shift;

    auto issue = [&](int k_local, int slot) {
        const int a = t_begin + (warp + k_local * W) * kTok;
        const int n = min(kTok, t_end - a);
        const int n_boxes = (n + rpb - 1) >> rpb_shift;
        uint8_t* kd = ring + slot * SLOT;
        if (lane == 0)
            mbar_arrive_expect_tx(&my_bars[slot], (uint32_t)(2 * n_boxes * rpb * D * EB));
        __syncwarp();
        const int total = 2 * n_boxes * PARTS;
        for (int i = lane; i < total; i += 32) {
            const int which = i >= n_boxes * PARTS;
            const int r = which ? i - n_boxes * PARTS : i;
            const int bx = r / PARTS, cp = r % PARTS;
            const int t0 = a + (bx << rpb_shift);
            const int lb = t0 >> bs_shift;
            const int y = ((blk[lb - lb0] * p.H_kv + g) << bs_shift) + (t0 & (bs - 1));
            uint8_t* dst = kd + which * TILE + cp * (kTok * 128) + (bx << rpb_shift) * 128;
            tma_load_2d(dst, which ? &tmap_v : &tmap_k, cp * (128 / EB), y, &my_bars[slot], policy);
        }
    };

    // this lane's half of q (score chunks), pre-scaled; loaded while the first
    // stages are in flight
    const int tok = lane & 15;
    const int side = lane >> 4;
    float qk[CPL * EPC];
    auto load_q = [&]() {
        const QT* qp = reinterpret_cast<const QT*>(p.q) + ((size_t)seq * p.H_q + h) * D;
#pragma unroll
        for (int j = 0; j < CPL * EPC; ++j)
            qk[j] = Elem<QT>::to_f(qp[side * (D / 2) + j]) * p.q_scale;
    };

    const int pro = min(S, my_n);
    int issued = 0;   // first stages in flight before the wait
    if (pre) {
        if (!bad)
            for (; issued < pro; ++issued) {
                const int a = t_begin + (warp + issued * W) * kTok;
                if (((min(a + kTok, t_end) - 1) >> bs_shift) - lb0 >= n_pre) break;
                issue(issued, issued);
            }
        load_q();
        grid_dependency_wait();
        if (n_pre < n_lb) {
            bool bad2 = false;
            for (int i = n_pre + tid; i < n_lb && trow >= 0; i += NT) {
                const int32_t b = p.tables[trow * p.max_blocks + lb0 + i];
                bad2 |= (b < 0 || b >= p.num_blocks);
                blk[i] = b;
            }
            bad = __syncthreads_or(bad2) || bad;
        }
    }
    const bool split = nparts > 1;
    if (bad) {
        // copies issued before the wait land before the CTA leaves
        for (int j = 0; j < issued; ++j) (void)mbar_wait(&my_bars[j], 0u);
        if (tid == 0 && h == 0) report_error(p.err, PKV_DEVERR_BLOCK_ID);
        for (int d = tid; d < D; d += NT) {
            const size_t row = ((size_t)seq * p.H_q + h) * p.max_parts + part;
            if (split) {
                p.ws_acc[row * D + d] = 0.f;
                if (d == 0) { p.ws_ml[row * 2] = -INFINITY; p.ws_ml[row * 2 + 1] = 0.f; }
            } else {
                reinterpret_cast<QT*>(p.out)[((size_t)seq * p.H_q + h) * D + d] = Elem<QT>::from_f(0.f);
            }
        }
        if (split && p.counters &&
            finish_partition(&p.counters[(size_t)seq * p.H_q + h], nparts, &last_flag))
            merge_group_in_cta<QT, D>(p, seq, h, 1, nparts, reinterpret_cast<float*>(smem),
                                      L::kTiles / 4);
        return;
    }

    for (int k = issued; k < pro; ++k) issue(k, k);
    if (!pre) load_q();

    float m_run = -INFINITY, l_run = 0.f;
    float acc[VEC];
#pragma unroll
    for (int v = 0; v < VEC; ++v) acc[v] = 0.f;
    // byte offset of this lane's value columns within a row, as (chunk, offset)
    const int vbyte = lane * VEC * EB;
    const int vch = vbyte >> 4, voff = vbyte & 15;

    int k = 0;
    bool timed_out = false;
    for (; k < my_n; ++k) {
        const int slot = k % S;
        if (!mbar_wait(&my_bars[slot], (uint32_t)((k / S) & 1), p.wait_ns)) {
            timed_out = true;
            break;
        }
        const int a = t_begin + (warp + k * W) * kTok;
        const int n = min(kTok, t_end - a);
        const uint8_t* kt = ring + slot * SLOT;
        const uint8_t* vt = kt + TILE;

        // score of token `tok`, this lane's half of the row
        float s;
        {
            float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int cc = 0; cc < CPL; ++cc) {
                const int chunk = side * CPL + cc;
                const uint8_t* src = kt + (chunk >> 3) * (kTok * 128) + tok * 128 +
                                     (((chunk & 7) ^ (tok & 7)) << 4);
                float f[EPC];
                Chunk<KV>::load(src, f);
#pragma unroll
                for (int e = 0; e < EPC; e += 2)
                    acc2 = __ffma2_rn(make_float2(qk[cc * EPC + e], qk[cc * EPC + e + 1]),
                                      make_float2(f[e], f[e + 1]), acc2);
            }
            s = acc2.x + acc2.y;
            s += __shfl_xor_sync(0xffffffffu, s, 16);
        }
        s = tok < n ? s : -INFINITY;
        float mx = s;
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        const float m_new = fmaxf(m_run, mx);
        const float alpha = exp2f(m_run - m_new);
        const float pr = tok < n ? exp2f(s - m_new) : 0.f;
        float sum = pr;
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        sum += __shfl_xor_sync(0xffffffffu, sum, 4);
        sum += __shfl_xor_sync(0xffffffffu, sum, 8);
        l_run = l_run * alpha + sum;
        m_run = m_new;
        if (lane < kTok) pbuf[lane] = pr;
        __syncwarp();
        float pv[kTok];
#pragma unroll
        for (int i = 0; i < kTok; i += 4) {
            const float4 q4 = *reinterpret_cast<const float4*>(pbuf + i);
            pv[i] = q4.x; pv[i + 1] = q4.y; pv[i + 2] = q4.z; pv[i + 3] = q4.w;
        }
#pragma unroll
        for (int v = 0; v < VEC; ++v) acc[v] *= alpha;
#pragma unroll
        for (int t = 0; t < kTok; ++t) {
            if (t < n) {
                const uint8_t* src = vt + (vch >> 3) * (kTok * 128) + t * 128 +
                                     (((vch & 7) ^ (t & 7)) << 4) + voff;
                float vf[VEC];
                VecLoad<KV, VEC>::run(src, vf);
                if constexpr (VEC % 2 == 0) {
#pragma unroll
                    for (int v = 0; v < VEC; v += 2) {
                        float2 r = __ffma2_rn(make_float2(pv[t], pv[t]), make_float2(vf[v], vf[v + 1]),
                                              make_float2(acc[v], acc[v + 1]));
                        acc[v] = r.x;
                        acc[v + 1] = r.y;
                    }
                } else {
                    acc[0] = fmaf(pv[t], vf[0], acc[0]);
                }
            }
        }
        __syncwarp();   // every lane done with this slot and with pbuf
        if (k + S < my_n) {
            fence_proxy_async_smem();
            issue(k + S, slot);
        }
    }
    if (timed_out) {
        if (lane == 0) report_error(p.err, PKV_DEVERR_TIMEOUT);
        for (int j = k; j < min(my_n, k + S); ++j)
            (void)mbar_wait(&my_bars[j % S], (uint32_t)((j / S) & 1));
    }

    // combine the warps
    {
        float* cw = comb + warp * (D + 2);
#pragma unroll
        for (int v = 0; v < VEC; ++v) cw[lane * VEC + v] = acc[v];
        if (lane == 0) {
            cw[D] = m_run;
            cw[D + 1] = l_run;
        }
    }
    __syncthreads();
    for (int d = tid; d < D; d += NT) {
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < W; ++w) M = fmaxf(M, comb[w * (D + 2) + D]);
        float Lsum = 0.f, O = 0.f;
#pragma unroll
        for (int w = 0; w < W; ++w) {
            const float* cw = comb + w * (D + 2);
            const float wt = exp2f(cw[D] - M);
            Lsum = fmaf(cw[D + 1], wt, Lsum);
            O = fmaf(cw[d], wt, O);
        }
        O *= p.v_scale;
        if (split) {
            const size_t row = ((size_t)seq * p.H_q + h) * p.max_parts + part;
            p.ws_acc[row * D + d] = O;
            if (d == 0) {
                p.ws_ml[row * 2] = M;
                p.ws_ml[row * 2 + 1] = Lsum;
            }
        } else {
            reinterpret_cast<QT*>(p.out)[((size_t)seq * p.H_q + h) * D + d] = Elem<QT>::from_f(O / Lsum);
        }
    }
    if (split && p.counters &&
        finish_partition(&p.counters[(size_t)seq * p.H_q + h], nparts, &last_flag))
        merge_group_in_cta<QT, D>(p, seq, h, 1, nparts, reinterpret_cast<float*>(smem),
                                  L::kTiles / 4);
}

template <typename KV, typename QT, int D, int W, int S>
cudaError_t launch_t(const DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv,
                     int q_dtype, int bs_shift, cudaStream_t st, cudaEvent_t mid) {
    using L = Simt2Smem<KV, D, W, S>;
    const int te = (p.part_tokens >> bs_shift) + 2;
    const int smem = L::bytes(te);
    if (smem > 227 * 1024) return cudaErrorInvalidValue;
    auto kern = decode_simt2_kernel<KV, QT, D, W, S>;
    static unsigned long long attr_done = 0;
    cudaError_t e = allow_large_smem(kern, &attr_done);
    if (e != cudaSuccess) return e;
    e = launch_kernel(kern, dim3(p.max_parts, p.H_q, p.B), dim3(W * 32), smem, st, p.pdl != 0,
                      *tk, *tv, p, prefetch_of(p), te, bs_shift);
    if (e == cudaSuccess && mid) e = cudaEventRecord(mid, st);
    if (e != cudaSuccess || p.max_parts <= 1 || p.counters) return e;
    return launch_merge(p, q_dtype, D, st);
}

template <typename KV, typename QT>
cudaError_t launch_q(const DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv, int D,
                     int q_dtype, int bs_shift, cudaStream_t st, cudaEvent_t mid) {
    constexpr int EB = Elem<KV>::bytes;
    // rows of 128, 256 or 512 bytes
    if (D * EB == 128 || D * EB == 256 || D * EB == 512) {
        switch (D) {
            case 32: if constexpr (32 * EB >= 128) return launch_t<KV, QT, 32, 4, 3>(p, tk, tv, q_dtype, bs_shift, st, mid); break;
            case 64: if constexpr (64 * EB >= 128) return launch_t<KV, QT, 64, 4, 3>(p, tk, tv, q_dtype, bs_shift, st, mid); break;
            case 128: return launch_t<KV, QT, 128, 4, (128 * EB >= 256 ? 2 : 3)>(p, tk, tv, q_dtype, bs_shift, st, mid);
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace

bool simt2_supported(const pkv_pool* pool, int group) {
    (void)group;
    return pool_has_row_maps(pool);
}

cudaError_t launch_decode_simt2(const DecodeParams& p, const void* tmap_k, const void* tmap_v,
                                int kv_dtype, int q_dtype, int D, int bs_shift, cudaStream_t st,
                                cudaEvent_t mid) {
    const CUtensorMap* tk = reinterpret_cast<const CUtensorMap*>(tmap_k);
    const CUtensorMap* tv = reinterpret_cast<const CUtensorMap*>(tmap_v);
    switch (kv_dtype) {
        case PKV_F32: return launch_q<float, float>(p, tk, tv, D, q_dtype, bs_shift, st, mid);
        case PKV_F16: return launch_q<__half, __half>(p, tk, tv, D, q_dtype, bs_shift, st, mid);
        case PKV_BF16:
            return launch_q<__nv_bfloat16, __nv_bfloat16>(p, tk, tv, D, q_dtype, bs_shift, st, mid);
        case PKV_FP8_E4M3:
            if (q_dtype == PKV_F16) return launch_q<fp8e4m3, __half>(p, tk, tv, D, q_dtype, bs_shift, st, mid);
            if (q_dtype == PKV_BF16)
                return launch_q<fp8e4m3, __nv_bfloat16>(p, tk, tv, D, q_dtype, bs_shift, st, mid);
            return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pkv
