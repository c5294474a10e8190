// Paged decode attention for grouped query heads on tensor cores.
//
// With G = H_q / H_kv > 1 query heads per KV head ("KV 缓存与分页注意力"
// §后来的做法: Llama-2-70B puts 64 heads on 8 K/V groups, Falcon-7B all heads on
// one), every K/V element read from HBM is used G times, so one KV head's
// group is a small dense contraction per 16-token stage:
//     S[G x 16]  = Q_group[G x d] . K_stage^T[d x 16]
//     O[G x d]  += P[G x 16] . V_stage[16 x d]
// done with mma.sync m16n8k16 (f16/bf16 in, fp32 accumulate).  The path stays
// HBM-bound (8 flop/B at G = 8, 71 at G = 71); the tensor cores only remove
// the CUDA-core FMA bound that G scalar dot products per element would hit.
//
// Staging: the pool is viewed by two TMA tensor maps (K and V) as a 2-D
// tensor [num_blocks * H_kv * bs rows][d] with 128-byte swizzle; one stage is
// min(bs, 16)-row boxes per 64-column half (bs a power of two), so each
// 8 x 16-byte ldmatrix read hits 8 different bank groups.  Loads are plain
// (no multicast) from this GPU's own memory.
//
// CTA = (partition, KV head, sequence).  Warps: MT warps of 8 query heads
// (MT = ceil(G / 8)) x TS token groups.  Each token group owns a ring of
// kStages slots; its first warp issues the copies (one box per lane), every warp of the
// group consumes every stage, and with MT > 1 an "empty" mbarrier per slot
// (MT arrivals) tells the producer when all of them are done with it.
// A warp computes S^T = K Q^T and O^T += V^T P^T (16 tokens or 16 d-rows by
// its 8 heads, so no padded rows up to 8 heads per KV head), P^T moving to
// the B-operand layout by register transposes; online softmax in base 2 per
// head.  The token groups' states are combined through shared memory.
#include <cuda.h>

#include <cfloat>
#include <type_traits>

#include "decode_launch.h"
#include "kernels_common.cuh"
#include "pool.h"
#include "tc_common.cuh"

namespace pkv {

namespace {

using tc::kStageTokens;
using tc::mbar_arrive;
using tc::tma_load_2d;

// EB: bytes per stored K/V element (2: f16/bf16 pools, 1: FP8 pools)
template <int D, int EB>
struct TcSmem {
    static constexpr int kTile = kStageTokens * D * EB;   // bytes of K (or V) of one stage
    static constexpr int kSlot = 2 * kTile;
};

template <int D, int MT, int TS, int S, int EB>
__host__ __device__ constexpr int tc_union_bytes() {
    const int tiles = TS * S * TcSmem<D, EB>::kSlot;
    const int comb = MT * TS * 8 * (D + 2) * 4;
    return ((tiles > comb ? tiles : comb) + 15) & ~15;
}

template <typename T, int D, int MT, int TS, int S, int EB>
__global__ void __launch_bounds__(MT * TS * 32)
decode_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                 const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p,
                 const __grid_constant__ StepPrefetch pf) {
    constexpr int kStages = S;
    constexpr int NW = MT * TS;
    constexpr int NT = NW * 32;
    constexpr int TILE = TcSmem<D, EB>::kTile;
    constexpr int SLOT = TcSmem<D, EB>::kSlot;
    constexpr int KSTEPS = D / 16;       // k-steps of S = Q K^T
    constexpr int HALVES = D * EB / 128;   // 128-byte column boxes per row
    static_assert(EB == 2 || (EB == 1 && D == 128), "FP8 stages have 128-byte rows");
    // early slot release holds a whole stage's fragments in registers: with
    // up to 8 warps (255 registers a thread) and for FP8 (raw codes, 32 registers)
    constexpr bool kEarly = EB == 1 || NT <= 256;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment of the swizzled tiles; the combine area reuses the
    // tile ring once every stage has been consumed
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* tiles = smem;                                            // [TS][kStages][SLOT]
    float* comb = reinterpret_cast<float*>(smem);                     // [NW][8][D + 2]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + tc_union_bytes<D, MT, TS, S, EB>());
    uint64_t* empty = full + TS * kStages;
    int32_t* blk = reinterpret_cast<int32_t*>(empty + TS * kStages);   // the partition's block ids

    const int part = blockIdx.x;
    const int g = blockIdx.y;
    const int slot = blockIdx.z;   // launch slot: length and table row
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int mt = warp % MT;       // m-tile of this warp
    const int ts = warp / MT;       // token group of this warp
    const int G = p.G;
    const int bs = p.block_size;   // a power of two (row tensor maps)
    const int bs_shift = __ffs(bs) - 1;
    const int P = p.part_tokens;
    const int h_base = g * G;       // first query head of the group

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
            if (tid == 0 && g == 0) report_error(p.err, PKV_DEVERR_CONTEXT_LEN);
            T* out = reinterpret_cast<T*>(p.out);
            for (int i = tid; i < G * D; i += NT)
                out[((size_t)seq * p.H_q + h_base + i / D) * D + i % D] = Elem<T>::from_f(0.f);
        }
        return;
    }
    const int nparts = (c + P - 1) / P;
    if (part >= nparts) return;
    const int Ps = balanced_part_tokens(c, P);
    const int t_begin = part * Ps;
    const int t_end = min(c, t_begin + Ps);
    const int32_t* table = p.tables + (trow < 0 ? 0 : trow) * p.max_blocks;

    const int lb0 = t_begin >> bs_shift;
    const int n_lb = ((t_end - 1) >> bs_shift) - lb0 + 1;
    // table entries final before the preceding kernel ends
    const int n_pre = pre ? max(0, min(n_lb, pf.stable[slot] - lb0)) : n_lb;
    bool bad = trow < 0;
    for (int i = tid; i < n_pre && trow >= 0; i += NT) {
        const int32_t b = table[lb0 + i];
        bad |= (b < 0 || b >= p.num_blocks);
        blk[i] = b;
    }
    if (tid == 0) {
        for (int i = 0; i < TS * kStages; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], MT);
        }
        fence_mbar_init();
    }
    bad = __syncthreads_or(bad);

    const int n_stages = (t_end - t_begin + kStageTokens - 1) / kStageTokens;
    const int my_n = n_stages > ts ? (n_stages - ts + TS - 1) / TS : 0;
    uint8_t* ring = tiles + ts * kStages * SLOT;
    uint64_t* my_full = full + ts * kStages;
    uint64_t* my_empty = empty + ts * kStages;
    const bool producer = (mt == 0);
    const uint64_t policy = l2_evict_first_policy();
    const int rpb_shift = bs_shift < 4 ? bs_shift : 4;   // rows per box: min(bs, 16)
    const int rows_per_box = 1 << rpb_shift;

    // issue stage k_local (this group's k-th) into `slot`; called by the
    // producer warp (all lanes)
    auto issue = [&](int k_local, int slot) {
        const int a = t_begin + (ts + k_local * TS) * kStageTokens;
        const int n = min(kStageTokens, t_end - a);
        const int n_boxes = (n + rows_per_box - 1) >> rpb_shift;   // boxes per half
        uint8_t* kd = ring + slot * SLOT;
        uint8_t* vd = kd + TILE;
        if (lane == 0)
            mbar_arrive_expect_tx(&my_full[slot], (uint32_t)(2 * HALVES * n_boxes * rows_per_box * 128));
        __syncwarp();
        // one (box, half, K or V) copy per lane: the copies' issue latencies
        // overlap instead of adding up
        for (int i = lane; i < 2 * HALVES * n_boxes; i += 32) {
            const int bx = i / (2 * HALVES), hf = (i >> 1) % HALVES, kv = i & 1;
            const int t0 = a + (bx << rpb_shift);
            const int lb = t0 >> bs_shift;
            const int y = ((blk[lb - lb0] * p.H_kv + g) << bs_shift) + (t0 & (bs - 1));
            const int off = hf * (kStageTokens * 128) + (bx << rpb_shift) * 128;
            tma_load_2d((kv ? vd : kd) + off, kv ? &tmap_v : &tmap_k, hf * (128 / EB), y,
                        &my_full[slot], policy);
        }
        __syncwarp();
    };

    // Q^T fragments (B operand) of this warp's 8 heads, zero past the group
    const int gq = lane >> 2;       // fragment row: d (and d + 8) of O^T
    const int tq = lane & 3;        // this lane's heads: 2 tq, 2 tq + 1 of the warp's 8
    uint32_t qb[KSTEPS][2];
    auto load_q = [&]() {
        if constexpr (EB == 1)
            tc::load_qT_frags_fp8(qb, reinterpret_cast<const __half*>(p.q) + ((size_t)seq * p.H_q + h_base) * D,
                                  mt * 8, G, lane);
        else
            tc::load_qT_frags<T, D>(qb, reinterpret_cast<const T*>(p.q) + ((size_t)seq * p.H_q + h_base) * D,
                                    mt * 8, G, lane);
    };

    const int pro = min(kStages, my_n);
    int issued = 0;   // first stages in flight before the wait (producer warps)
    if (pre) {
        if (!bad && producer)
            for (; issued < pro; ++issued) {
                const int a = t_begin + (ts + issued * TS) * kStageTokens;
                if (((min(a + kStageTokens, t_end) - 1) >> bs_shift) - lb0 >= n_pre) break;
                issue(issued, issued);
            }
        load_q();
        grid_dependency_wait();
        if (n_pre < n_lb) {
            bool bad2 = false;
            for (int i = n_pre + tid; i < n_lb && trow >= 0; i += NT) {
                const int32_t b = table[lb0 + i];
                bad2 |= (b < 0 || b >= p.num_blocks);
                blk[i] = b;
            }
            bad = __syncthreads_or(bad2) || bad;
        }
    }
    const bool split = nparts > 1;
    if (bad) {
        // copies issued before the wait land before the CTA leaves
        for (int j = 0; j < issued; ++j) (void)mbar_wait(&my_full[j], 0u);
        __syncthreads();
        if (tid == 0 && g == 0) report_error(p.err, PKV_DEVERR_BLOCK_ID);
        for (int i = tid; i < G * D; i += NT) {
            const int h = h_base + i / D, d = i % D;
            const size_t row = ((size_t)seq * p.H_q + h) * p.max_parts + part;
            if (split) {
                p.ws_acc[row * D + d] = 0.f;
                if (d == 0) { p.ws_ml[row * 2] = -INFINITY; p.ws_ml[row * 2 + 1] = 0.f; }
            } else {
                reinterpret_cast<T*>(p.out)[((size_t)seq * p.H_q + h) * D + d] = Elem<T>::from_f(0.f);
            }
        }
        if (split && p.counters &&
            finish_partition(&p.counters[(size_t)seq * p.H_kv + g], nparts, &last_flag))
            merge_group_in_cta<T, D>(p, seq, h_base, G, nparts, reinterpret_cast<float*>(smem),
                                     tc_union_bytes<D, MT, TS, S, EB>() / 4);
        return;
    }

    if (!pre) load_q();

    float o[D / 16][4];
#pragma unroll
    for (int j = 0; j < D / 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};

    if (producer)
        for (int k = issued; k < pro; ++k) issue(k, k);

    int k = 0;
    bool timed_out = false;
    int rslot = 0;         // ring slot: k % kStages
    uint32_t phase = 0;    // its parity: (k / kStages) & 1
    for (; k < my_n; ++k) {
        if (k > 0 && ++rslot == kStages) {
            rslot = 0;
            phase ^= 1u;
        }
        if (!mbar_wait(&my_full[rslot], phase, p.wait_ns)) {
            timed_out = true;
            break;
        }
        const int a = t_begin + (ts + k * TS) * kStageTokens;
        const int n = min(kStageTokens, t_end - a);
        const uint8_t* kt = ring + rslot * SLOT;
        const uint8_t* vt = kt + TILE;
        // hand the slot back for the next copy: the producer waits (MT > 1)
        // until every warp of the group has read it
        auto release = [&]() -> bool {
            fence_proxy_async_smem();   // these reads before the async proxy's refill
            __syncwarp();
            if constexpr (MT > 1) {
                if (lane == 0) mbar_arrive(&my_empty[rslot]);
            }
            if (producer && k + kStages < my_n) {
                if constexpr (MT > 1) {
                    if (!mbar_wait(&my_empty[rslot], phase, p.wait_ns)) return false;
                }
                issue(k + kStages, rslot);
            }
            return true;
        };
        if constexpr (kEarly) {
            // the stage moves into registers, the rslot is released, and the
            // math runs while the next copy is in flight
            using Frags = std::conditional_t<EB == 1, tc::Fp8Raw, tc::StageFrags<D>>;
            Frags f;
            if constexpr (EB == 1)
                tc::stage_raw_fp8(kt, vt, n, f, lane);
            else
                tc::stage_frags_t<D>(kt, vt, n, f, lane);
            if (!release()) {
                timed_out = true;
                ++k;
                break;
            }
            if constexpr (EB == 1)
                tc::stage_math_fp8(qb, f, n, p.q_scale, o, m_run, l_run, lane);
            else
                tc::stage_math_t<T, D>(qb, f, n, p.q_scale, o, m_run, l_run, lane);
        } else {
            tc::stage_body_t<T, D>(qb, kt, vt, n, p.q_scale, o, m_run, l_run, lane);
            if (!release()) {
                timed_out = true;
                ++k;
                break;
            }
        }
    }
    if (timed_out) {
        if (lane == 0) report_error(p.err, PKV_DEVERR_TIMEOUT);
        // bounded wait for copies this group may still have in flight
        if (producer)
            for (int j = k; j < min(my_n, k + kStages); ++j)
                (void)mbar_wait(&my_full[j % kStages], (uint32_t)((j / kStages) & 1));
    }

    if constexpr (EB == 1) {
        // FP8 V was used as codes: its scale applies to the accumulator
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
            o[j][0] *= p.v_scale;
            o[j][1] *= p.v_scale;
            o[j][2] *= p.v_scale;
            o[j][3] *= p.v_scale;
        }
    }
    // head sums: the lanes with the same lane % 4 hold disjoint tokens
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 4);
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 8);
        l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 16);
    }
    __syncthreads();   // every ring slot consumed: the combine area may be written
    // per-warp state -> shared memory [NW][8 heads][D + 2]
    {
        float* cw = comb + warp * 8 * (D + 2);
        const int ra = 2 * tq, rb = ra + 1;
        // o[j] rows: d = 16 j + gq and + 8
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
            const int d0 = 16 * j + gq;
            const int d1 = d0 + 8;
            cw[ra * (D + 2) + d0] = o[j][0];
            cw[rb * (D + 2) + d0] = o[j][1];
            cw[ra * (D + 2) + d1] = o[j][2];
            cw[rb * (D + 2) + d1] = o[j][3];
        }
        if (gq == 0) {
            cw[ra * (D + 2) + D] = m_run[0];
            cw[ra * (D + 2) + D + 1] = l_run[0];
            cw[rb * (D + 2) + D] = m_run[1];
            cw[rb * (D + 2) + D + 1] = l_run[1];
        }
    }
    __syncthreads();
    // combine the token groups of each 8-head group and write the G real heads
    for (int i = tid; i < MT * 8 * D; i += NT) {
        const int m_tile = i / (8 * D);
        const int row = (i / D) % 8;
        const int d = i % D;
        const int hrow = m_tile * 8 + row;
        if (hrow >= G) continue;
        float M = -INFINITY;
#pragma unroll
        for (int t = 0; t < TS; ++t)
            M = fmaxf(M, comb[((t * MT + m_tile) * 8 + row) * (D + 2) + D]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int t = 0; t < TS; ++t) {
            const float* cw = comb + ((t * MT + m_tile) * 8 + row) * (D + 2);
            const float w = M == -INFINITY ? 0.f : exp2f(cw[D] - M);
            L = fmaf(cw[D + 1], w, L);
            O = fmaf(cw[d], w, O);
        }
        const int h = h_base + hrow;
        if (split) {
            const size_t prow = ((size_t)seq * p.H_q + h) * p.max_parts + part;
            p.ws_acc[prow * D + d] = O;
            if (d == 0) {
                p.ws_ml[prow * 2] = M;
                p.ws_ml[prow * 2 + 1] = L;
            }
        } else {
            reinterpret_cast<T*>(p.out)[((size_t)seq * p.H_q + h) * D + d] =
                Elem<T>::from_f(L > 0.f ? O / L : 0.f);
        }
    }
    if (split && p.counters &&
        finish_partition(&p.counters[(size_t)seq * p.H_kv + g], nparts, &last_flag))
        merge_group_in_cta<T, D>(p, seq, h_base, G, nparts, reinterpret_cast<float*>(smem),
                                 tc_union_bytes<D, MT, TS, S, EB>() / 4);
}

template <int D, int MT, int TS, int S, int EB>
constexpr int tc_smem_bytes() {
    return 1024 + tc_union_bytes<D, MT, TS, S, EB>() + 2 * TS * S * 8;
}
// plus the partition's block ids: part_tokens / bs + 2 entries
inline int tc_table_bytes(const DecodeParams& p) {
    return ((p.part_tokens / p.block_size + 2) * 4 + 15) & ~15;
}

template <typename T, int D, int MT, int TS, int S = (D == 128 ? 2 : 3), int EB = 2>
cudaError_t launch_tc_t(const DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv,
                        int q_dtype, cudaStream_t st, cudaEvent_t mid) {
    constexpr int base = tc_smem_bytes<D, MT, TS, S, EB>();
    static_assert(base <= 227 * 1024 - 64, "shared memory budget");
    const int smem = base + tc_table_bytes(p);
    if (smem > 227 * 1024 - 64) return cudaErrorInvalidValue;
    auto kern = decode_tc_kernel<T, D, MT, TS, S, EB>;
    static unsigned long long attr_done = 0;
    cudaError_t e = allow_large_smem(kern, &attr_done);
    if (e != cudaSuccess) return e;
    const dim3 grid(p.max_parts, p.H_kv, p.B);
    e = launch_kernel(kern, grid, dim3(MT * TS * 32), smem, st, p.pdl != 0, *tk, *tv, p,
                      prefetch_of(p));
    if (e == cudaSuccess && mid) e = cudaEventRecord(mid, st);
    if (e != cudaSuccess || p.max_parts <= 1 || p.counters) return e;
    return launch_merge(p, q_dtype, D, st);
}

template <typename T, int D>
cudaError_t launch_tc_d(const DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv,
                        int q_dtype, cudaStream_t st, cudaEvent_t mid) {
    const int mt = (p.G + 7) / 8;
    switch (mt) {
        // warps of 8 heads x token groups
        case 1: return launch_tc_t<T, D, 1, 4>(p, tk, tv, q_dtype, st, mid);
        case 2: return launch_tc_t<T, D, 2, 4>(p, tk, tv, q_dtype, st, mid);
        case 3: return launch_tc_t<T, D, 3, 3>(p, tk, tv, q_dtype, st, mid);
        case 4: return launch_tc_t<T, D, 4, 2>(p, tk, tv, q_dtype, st, mid);
        case 5: return launch_tc_t<T, D, 5, 2>(p, tk, tv, q_dtype, st, mid);
        case 6: return launch_tc_t<T, D, 6, 2>(p, tk, tv, q_dtype, st, mid);
        case 7: return launch_tc_t<T, D, 7, 1>(p, tk, tv, q_dtype, st, mid);
        case 8: return launch_tc_t<T, D, 8, 1>(p, tk, tv, q_dtype, st, mid);
        case 9: return launch_tc_t<T, D, 9, 1>(p, tk, tv, q_dtype, st, mid);
        case 10: return launch_tc_t<T, D, 10, 1>(p, tk, tv, q_dtype, st, mid);
        case 11: return launch_tc_t<T, D, 11, 1>(p, tk, tv, q_dtype, st, mid);
        case 12: return launch_tc_t<T, D, 12, 1>(p, tk, tv, q_dtype, st, mid);
        case 13: return launch_tc_t<T, D, 13, 1>(p, tk, tv, q_dtype, st, mid);
        case 14: return launch_tc_t<T, D, 14, 1>(p, tk, tv, q_dtype, st, mid);
        case 15: return launch_tc_t<T, D, 15, 1>(p, tk, tv, q_dtype, st, mid);
        case 16: return launch_tc_t<T, D, 16, 1>(p, tk, tv, q_dtype, st, mid);
        default: return cudaErrorInvalidValue;
    }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// dependency on libcuda)
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

bool encode_pool_map(CUtensorMap* map, void* base, int dtype, int D, long long rows, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const int eb = dtype == PKV_F32 ? 4 : dtype == PKV_FP8_E4M3 ? 1 : 2;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * eb};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / eb), (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUtensorMapDataType t = CU_TENSOR_MAP_DATA_TYPE_UINT8;
    if (dtype == PKV_F32) t = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    if (dtype == PKV_F16) t = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    if (dtype == PKV_BF16) t = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    return fn(map, t, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// Row tensor maps of the K and V pools: a 2-D view [num_blocks * H_kv * bs
// rows][d] with 128-byte inner boxes of min(bs, 16) rows and 128-byte swizzle.
// Made when a row is 128, 256 or 512 bytes and bs is a power of two (then a
// 16-token stage is a whole number of boxes, none crossing a block).
void pool_init_device_extras(pkv_pool* p) {
    p->has_tmaps = false;
    const int eb = p->dtype == PKV_F32 ? 4 : p->dtype == PKV_FP8_E4M3 ? 1 : 2;
    const int row = p->head_dim * eb;
    if (row != 128 && row != 256 && row != 512) return;
    if (p->block_size & (p->block_size - 1)) return;
    const long long rows = (long long)p->num_blocks * p->n_kv_heads * p->block_size;
    if (rows >= (1LL << 31)) return;
    const int box_rows = p->block_size < kStageTokens ? p->block_size : kStageTokens;
    static_assert(sizeof(CUtensorMap) == 128, "tensor map size");
    p->has_tmaps = encode_pool_map(reinterpret_cast<CUtensorMap*>(p->tmap_k), p->k, p->dtype,
                                   p->head_dim, rows, box_rows) &&
                   encode_pool_map(reinterpret_cast<CUtensorMap*>(p->tmap_v), p->v, p->dtype,
                                   p->head_dim, rows, box_rows);
}

bool pool_has_row_maps(const pkv_pool* pool) { return pool->has_tmaps; }

bool tensor_path_supported(const pkv_pool* pool, int q_dtype, int group) {
    if (!pool->has_tmaps) return false;
    // FP8 codes are converted to f16 in registers: f16 queries, 128-byte rows,
    // one warp of up to 8 heads per KV head
    if (pool->dtype == PKV_FP8_E4M3)
        return q_dtype == PKV_F16 && pool->head_dim == 128 && group >= 1 && group <= 8;
    return (pool->dtype == PKV_F16 || pool->dtype == PKV_BF16) && q_dtype == pool->dtype &&
           (pool->head_dim == 64 || pool->head_dim == 128) && group > 1 && group <= 128;
}

cudaError_t launch_decode_tensor(const DecodeParams& p, const void* tmap_k, const void* tmap_v,
                                 int kv_dtype, int D, cudaStream_t st, cudaEvent_t mid) {
    const CUtensorMap* tk = reinterpret_cast<const CUtensorMap*>(tmap_k);
    const CUtensorMap* tv = reinterpret_cast<const CUtensorMap*>(tmap_v);
    if (kv_dtype == PKV_FP8_E4M3) {
        // 4 KB stages, 3-slot rings per token group: 48 KB a CTA, four CTAs
        // (16 warps) per SM to hide the conversion and softmax latency
        // (measured: 0.84 of the copy peak on the OPT-13B-shaped FP8 batch
        // against 0.78 with 4-slot rings at three CTAs per SM)
        if (D == 128 && p.G <= 8) return launch_tc_t<__half, 128, 1, 4, 3, 1>(p, tk, tv, PKV_F16, st, mid);
        return cudaErrorInvalidValue;
    }
    if (kv_dtype == PKV_F16) {
        if (D == 64) return launch_tc_d<__half, 64>(p, tk, tv, PKV_F16, st, mid);
        if (D == 128) return launch_tc_d<__half, 128>(p, tk, tv, PKV_F16, st, mid);
    } else if (kv_dtype == PKV_BF16) {
        if (D == 64) return launch_tc_d<__nv_bfloat16, 64>(p, tk, tv, PKV_BF16, st, mid);
        if (D == 128) return launch_tc_d<__nv_bfloat16, 128>(p, tk, tv, PKV_BF16, st, mid);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pkv
