// Stage-balanced paged decode on tensor cores (one persistent wave).
//
// The decode step reads every cached K/V row of the batch once
// ("KV 缓存与分页注意力" §块表: the kernel follows each sequence's block table
// to blocks scattered over the pool).  A batch of ragged contexts cut into
// per-(sequence, head) CTAs leaves SMs idle in every CTA's start-up and tail
// and at the end of the grid; here the work is instead laid out as one line of
// 16-token stages - pairs (sequence, KV head) in sequence-major order, each
// pair ceil(c / 16) stages - and every worker of a one-wave persistent grid
// takes an equal contiguous share of it.  A share crosses pair boundaries; the
// part of a pair inside one share is a "piece".  A pair held by one piece is
// written out directly; a pair split over several workers leaves one partial
// softmax state (running max in log2 units, sum, unnormalised accumulator) per
// piece in the workspace, and the worker that finishes the pair's last piece
// merges them by log-sum-exp (the split-context merge of the decode step).
//
// Worker = MT warps (16 query heads of the KV head's group each, as mma.sync
// m16n8k16 m-tiles); a CTA holds TS workers.  Each worker owns a ring of RG
// 16-token stage slots filled by 2-D TMA loads (128-byte swizzle, plain loads
// of this GPU's own memory) that its first warp issues, RG stages ahead of
// the one being consumed; with MT > 1 an "empty" mbarrier per slot tells the
// issuing warp when every warp of the worker is done with it.  Many
// independent workers per SM hide each one's serial chain (scores, softmax,
// P.V) and the copies' latency.  A stage whose block id is out of range is not
// loaded (the piece's contribution becomes zero and the device error word
// records it).  Every wait is bounded.
#include <cuda.h>

#include <algorithm>
#include <cfloat>

#include "decode_launch.h"
#include "kernels_common.cuh"
#include "pool.h"
#include "tc_common.cuh"

namespace pkv {

namespace {

using tc::kStageTokens;

constexpr int kLeanMaxBatch = 2048;      // stage prefix sums of the batch sit in shared memory
constexpr int kLeanMaxWorkersPerSm = 16; // bounds the workspace
constexpr unsigned kFull = 0xffffffffu;

template <int D>
struct LeanCfg {
    static constexpr int kSlot = 2 * kStageTokens * D * 2;   // K and V of one stage
};

// Workers per CTA, ring slots per worker and merge scratch per worker (floats)
// for MT m-tile warps per worker.
template <int D, int MT>
struct LeanShape {
    static constexpr int TS = MT == 1 ? 4 : (MT == 2 ? 2 : 1);
    static constexpr int RG = D == 128 ? 3 : 4;
    static constexpr int kMerge = MT == 1 ? 512 : 2048;
};

// The part of one (sequence, KV head) pair inside a worker's share.
struct Piece {
    int seq, g;
    int s0, s1;         // stages [s0, s1) of the pair
    int n_st;           // stages of the pair
    long long start;    // position of the pair's first stage on the stage line
};

// The stage line: pair (seq, g) starts at H_kv * pre[seq] + g * n_st(seq),
// pre[] = exclusive prefix sums of the stages per sequence.  Worker w owns
// [floor(w T / n), floor((w + 1) T / n)) of the n workers, non-empty for n <= T.
struct Schedule {
    const int* pre;
    int B, H_kv, n;
    long long T;
    __device__ long long lo(int w) const { return (long long)w * T / n; }
    // the worker whose share holds position x (the largest w with lo(w) <= x)
    __device__ int worker_of(long long x) const { return (int)(((x + 1) * n - 1) / T); }
    // the piece starting at position pos of a share ending at hi
    __device__ Piece at(long long pos, long long hi) const {
        int a = 0, b = B - 1;   // the largest s with H_kv * pre[s] <= pos
        while (a < b) {
            const int m = (a + b + 1) >> 1;
            if ((long long)H_kv * pre[m] <= pos)
                a = m;
            else
                b = m - 1;
        }
        Piece pc;
        pc.seq = a;
        pc.n_st = pre[a + 1] - pre[a];
        const long long off = pos - (long long)H_kv * pre[a];
        pc.g = (int)(off / pc.n_st);
        pc.s0 = (int)(off - (long long)pc.g * pc.n_st);
        pc.start = pos - pc.s0;
        const long long room = hi - pos;
        pc.s1 = room < pc.n_st - pc.s0 ? pc.s0 + (int)room : pc.n_st;
        return pc;
    }
};

// Barrier over the MT warps of one worker (named barrier 1 + worker).
template <int MT>
__device__ __forceinline__ void worker_sync(int worker) {
    if constexpr (MT == 1) {
        __syncwarp();
    } else {
        asm volatile("bar.sync %0, %1;" ::"r"(1 + worker), "r"(MT * 32) : "memory");
    }
}

// Merge the pieces' partial states of pair (seq, g) into the output, run by
// the threads of the worker that finished the pair last.  Round trip 1: every
// piece's running max per head row -> weights in shared memory; round trip 2:
// the sums; round trip 3: the accumulators, all loads independent.  `scratch`
// holds k_merge floats; more pieces than fit take the one-element-at-a-time
// path.
template <typename T, int D, int MT>
__device__ void merge_pieces(const DecodeParams& p, int seq, int g, int first, int n_pieces,
                             float* scratch, int k_merge, int wtid, int worker) {
    constexpr int n_thr = MT * 32;
    const int G = p.G;
    const size_t slot0 = (size_t)seq * p.H_kv + g + first;
    T* out = reinterpret_cast<T*>(p.out) + ((size_t)seq * p.H_q + (size_t)g * G) * D;
    if (n_pieces * G + G <= k_merge) {
        float* w = scratch;                    // [n_pieces][G] weights
        float* rowv = scratch + n_pieces * G;  // [G] row max, then 1 / L
        for (int i = wtid; i < n_pieces * G; i += n_thr)
            w[i] = __ldcg(p.ws_ml + ((slot0 + i / G) * G + i % G) * 2);
        worker_sync<MT>(worker);
        for (int r = wtid; r < G; r += n_thr) {
            float M = -INFINITY;
            for (int j = 0; j < n_pieces; ++j) M = fmaxf(M, w[j * G + r]);
            rowv[r] = M;
        }
        worker_sync<MT>(worker);
        for (int i = wtid; i < n_pieces * G; i += n_thr) {
            const float m = w[i];
            w[i] = (m == -INFINITY) ? 0.f : exp2f(m - rowv[i % G]);
        }
        worker_sync<MT>(worker);
        for (int r = wtid; r < G; r += n_thr) {
            float L = 0.f;
            for (int j = 0; j < n_pieces; ++j)
                L = fmaf(w[j * G + r], __ldcg(p.ws_ml + ((slot0 + j) * G + r) * 2 + 1), L);
            rowv[r] = L > 0.f ? 1.f / L : 0.f;
        }
        worker_sync<MT>(worker);
        for (int i = wtid; i < G * (D / 4); i += n_thr) {
            const int r = i / (D / 4), d4 = i % (D / 4);
            float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
            for (int j = 0; j < n_pieces; ++j) {
                const float wj = w[j * G + r];
                const float4 a = __ldcg(
                    reinterpret_cast<const float4*>(p.ws_acc + ((slot0 + j) * G + r) * D) + d4);
                O.x = fmaf(wj, a.x, O.x);
                O.y = fmaf(wj, a.y, O.y);
                O.z = fmaf(wj, a.z, O.z);
                O.w = fmaf(wj, a.w, O.w);
            }
            const float inv = rowv[r];
            T* o = out + (size_t)r * D + 4 * d4;
            o[0] = Elem<T>::from_f(O.x * inv);
            o[1] = Elem<T>::from_f(O.y * inv);
            o[2] = Elem<T>::from_f(O.z * inv);
            o[3] = Elem<T>::from_f(O.w * inv);
        }
        worker_sync<MT>(worker);   // the scratch is free again
        return;
    }
    for (int i = wtid; i < G * (D / 4); i += n_thr) {
        const int r = i / (D / 4), d4 = i % (D / 4);
        float M = -INFINITY, L = 0.f;
        float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < n_pieces; ++j) {
            const size_t row = (slot0 + j) * G + r;
            const float m = __ldcg(p.ws_ml + row * 2);
            const float l = __ldcg(p.ws_ml + row * 2 + 1);
            const float4 a = __ldcg(reinterpret_cast<const float4*>(p.ws_acc + row * D) + d4);
            if (m == -INFINITY) continue;
            const float Mn = fmaxf(M, m);
            const float so = exp2f(M - Mn), sn = exp2f(m - Mn);
            L = L * so + l * sn;
            O.x = O.x * so + a.x * sn;
            O.y = O.y * so + a.y * sn;
            O.z = O.z * so + a.z * sn;
            O.w = O.w * so + a.w * sn;
            M = Mn;
        }
        const float inv = L > 0.f ? 1.f / L : 0.f;
        T* o = out + (size_t)r * D + 4 * d4;
        o[0] = Elem<T>::from_f(O.x * inv);
        o[1] = Elem<T>::from_f(O.y * inv);
        o[2] = Elem<T>::from_f(O.z * inv);
        o[3] = Elem<T>::from_f(O.w * inv);
    }
}

template <int D, int MT>
__host__ __device__ constexpr int lean_fixed_smem() {
    using S = LeanShape<D, MT>;
    // rings (1024-aligned) + full/empty barriers + slot token counts + per
    // worker flags + merge scratch + per-warp scan totals; prefix sums follow
    return 1024 + S::TS * S::RG * LeanCfg<D>::kSlot + 2 * S::TS * S::RG * 8 + S::TS * S::RG * 4 +
           S::TS * 4 + S::TS * S::kMerge * 4 + 16 * 4;
}

// The issuing side of a worker: walks the share RG stages ahead of the
// consumption; held by the worker's first warp (all lanes).
struct Issuer {
    long long pos;       // the next piece starts at pos
    int seq, g;          // piece being issued
    int s, s1;           // next stage of it to issue, its end (s == s1: take the next piece)
    int trow;            // its table row (-1: invalid)
    int c;               // its context length
    int wb, wid;         // table entries wb .. wb + 31, one per lane
    int issued;          // stages issued so far
};

template <int D>
__device__ __forceinline__ void issue_stage(Issuer& is, long long hi, const Schedule& sc,
                                            const DecodeParams& p, const CUtensorMap* tk,
                                            const CUtensorMap* tv, uint8_t* slot_mem,
                                            uint64_t* full, volatile int* slot_n, uint64_t policy,
                                            int lane) {
    constexpr int TILE = LeanCfg<D>::kSlot / 2;
    constexpr int HALVES = D / 64;
    if (is.s == is.s1) {
        const Piece pc = sc.at(is.pos, hi);
        is.pos = pc.start + pc.s1;
        is.seq = pc.seq;
        is.g = pc.g;
        is.s = pc.s0;
        is.s1 = pc.s1;
        is.trow = (int)table_row(p, pc.seq);
        is.c = p.lens[pc.seq];
        is.wb = -1;
    }
    const int bs = p.block_size;
    const int rpb = bs < kStageTokens ? bs : kStageTokens;   // rows per box
    const int a = is.s * kStageTokens;
    const int n = min(kStageTokens, is.c - a);
    const int nb = (n + rpb - 1) / rpb;
    const int lb0 = a / bs;
    const int lb1 = (a + n - 1) / bs;
    if (is.wb < 0 || lb1 >= is.wb + 32) {
        is.wb = lb0;
        is.wid = (is.trow >= 0 && is.wb + lane < p.max_blocks)
                     ? p.tables[(long long)is.trow * p.max_blocks + is.wb + lane]
                     : -1;
    }
    bool bad = is.trow < 0;
    for (int bx = 0; bx < nb; ++bx) {
        const int id = __shfl_sync(kFull, is.wid, (a + bx * rpb) / bs - is.wb);
        bad |= id < 0 || id >= p.num_blocks;
    }
    if (lane == 0) {
        *slot_n = bad ? -1 : n;
        if (bad) {
            report_error(p.err, PKV_DEVERR_BLOCK_ID);
            tc::mbar_arrive(full);
        } else {
            mbar_arrive_expect_tx(full, (uint32_t)(2 * HALVES * nb * rpb * 128));
        }
    }
    if (!bad) {
        for (int bx = 0; bx < nb; ++bx) {
            const int t0 = a + bx * rpb;
            const int lb = t0 / bs;
            const int id = __shfl_sync(kFull, is.wid, lb - is.wb);
            if (lane == 0) {
                const int y = (id * p.H_kv + is.g) * bs + (t0 - lb * bs);
#pragma unroll
                for (int hf = 0; hf < HALVES; ++hf) {
                    const int off = hf * (kStageTokens * 128) + bx * rpb * 128;
                    tc::tma_load_2d(slot_mem + off, tk, hf * 64, y, full, policy);
                    tc::tma_load_2d(slot_mem + TILE + off, tv, hf * 64, y, full, policy);
                }
            }
        }
    }
    __syncwarp();
    ++is.s;
    ++is.issued;
}

template <typename T, int D, int MT>
__global__ void __launch_bounds__(LeanShape<D, MT>::TS * MT * 32)
decode_lean_kernel(const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
    using S = LeanShape<D, MT>;
    constexpr int TS = S::TS;
    constexpr int RG = S::RG;
    constexpr int SLOT = LeanCfg<D>::kSlot;
    constexpr int TILE = SLOT / 2;
    constexpr int DTILES = D / 8;
    constexpr int NT = TS * MT * 32;
    static_assert(NT / 32 <= 16, "scan totals");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* rings = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t* fulls = reinterpret_cast<uint64_t*>(rings + TS * RG * SLOT);   // [TS][RG]
    uint64_t* empties = fulls + TS * RG;                                     // [TS][RG]
    volatile int* slot_ns = reinterpret_cast<volatile int*>(empties + TS * RG);   // [TS][RG]
    volatile int* flags = slot_ns + TS * RG;                                 // [TS] last-piece flag
    float* merge_scr = reinterpret_cast<float*>(const_cast<int*>(flags + TS));   // [TS][kMerge]
    int* wsum = reinterpret_cast<int*>(merge_scr + TS * S::kMerge);          // [16]
    int* pre = wsum + 16;                                                    // [B + 1]

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int B = p.B;
    const int H_kv = p.H_kv;
    const int G = p.G;
    const int max_ctx = p.max_blocks * p.block_size;   // fits int: checked by the host

    if (tid == 0) {
        for (int i = 0; i < TS * RG; ++i) {
            mbar_init(&fulls[i], 1);
            mbar_init(&empties[i], MT);
        }
        fence_mbar_init();
    }
    grid_dependency_wait();   // lengths and tables may come from the preceding kernel

    // stages per sequence (0 for an invalid length), then an in-place
    // inclusive scan: every thread one contiguous chunk
    for (int i = tid; i < B; i += NT) {
        const int c = p.lens[i];
        pre[i + 1] = (c >= 1 && c <= max_ctx) ? (c + kStageTokens - 1) / kStageTokens : 0;
    }
    if (tid == 0) pre[0] = 0;
    __syncthreads();
    {
        const int chunk = (B + NT - 1) / NT;
        const int a = 1 + tid * chunk;
        const int b = min(B + 1, a + chunk);
        int sum = 0;
        for (int i = a; i < b; ++i) sum += pre[i];
        int x = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(kFull, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[warp] = x;
        __syncthreads();
        int run = x - sum;
        for (int w = 0; w < warp; ++w) run += wsum[w];
        for (int i = a; i < b; ++i) {
            run += pre[i];
            pre[i] = run;
        }
        __syncthreads();
    }

    // sequences with an invalid length: zero output, error bit
    for (int seq = blockIdx.x; seq < B; seq += gridDim.x) {
        if (pre[seq + 1] != pre[seq]) continue;
        if (tid == 0) report_error(p.err, PKV_DEVERR_CONTEXT_LEN);
        T* out = reinterpret_cast<T*>(p.out) + (size_t)seq * p.H_q * D;
        for (int i = tid; i < p.H_q * D; i += NT) out[i] = Elem<T>::from_f(0.f);
    }

    // with fewer stages than workers the surplus workers stay idle, so that
    // every share is non-empty and a pair's pieces sit in consecutive workers
    const long long total = (long long)H_kv * pre[B];
    const long long n_workers = (long long)gridDim.x * TS;
    const Schedule sc{pre, B, H_kv, (int)(total < n_workers ? total : n_workers), total};
    const int worker = warp / MT;
    const int mt = warp % MT;
    const int vw = blockIdx.x * TS + worker;   // this worker's index on the stage line
    if (vw >= sc.n) return;
    const long long lo = sc.lo(vw);
    const long long hi = sc.lo(vw + 1);
    const int n_stages = (int)(hi - lo);

    uint8_t* ring = rings + worker * RG * SLOT;
    uint64_t* full = fulls + worker * RG;
    uint64_t* empty = empties + worker * RG;
    volatile int* slot_n = slot_ns + worker * RG;
    float* scratch = merge_scr + worker * S::kMerge;
    const bool issuer = mt == 0;
    const uint64_t policy = l2_evict_first_policy();

    Issuer is;
    is.pos = lo;
    is.s = is.s1 = 0;
    is.issued = 0;
    if (issuer) {
        const int pro = min(RG, n_stages);
        for (int k = 0; k < pro; ++k)
            issue_stage<D>(is, hi, sc, p, &tmap_k, &tmap_v, ring + k * SLOT, &full[k], &slot_n[k],
                           policy, lane);
    }

    const int gq = lane >> 2;
    const int tq = lane & 3;
    const int r0 = mt * 16 + gq;
    const int r1 = r0 + 8;
    const int wtid = mt * 32 + lane;
    long long pos = lo;
    int it = 0;
    bool abort = false;
    while (pos < hi) {
        const Piece pc = sc.at(pos, hi);
        pos = pc.start + pc.s1;
        const int h0 = pc.g * G;
        uint32_t qa[D / 16][4];
        tc::load_q_frags<T, D>(qa, reinterpret_cast<const T*>(p.q) + ((size_t)pc.seq * p.H_q + h0) * D,
                               mt * 16, G, lane);
        float o[DTILES][4];
#pragma unroll
        for (int j = 0; j < DTILES; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        float m_run[2] = {-INFINITY, -INFINITY};
        float l_run[2] = {0.f, 0.f};
        bool bad = false;
        for (int s = pc.s0; s < pc.s1; ++s, ++it) {
            const int slot = it % RG;
            const uint32_t par = (uint32_t)((it / RG) & 1);
            if (!abort) {
                const bool ok = mbar_wait(&full[slot], par);
                if (!__all_sync(kFull, ok)) {
                    abort = true;
                    if (lane == 0) report_error(p.err, PKV_DEVERR_TIMEOUT);
                }
            }
            if (!abort) {
                const int n = slot_n[slot];
                uint8_t* kt = ring + slot * SLOT;
                if (n < 0)
                    bad = true;
                else
                    tc::stage_body<T, D>(qa, kt, kt + TILE, n, p.q_scale, o, m_run, l_run, lane);
                __syncwarp();
            }
            if constexpr (MT > 1) {
                if (lane == 0) tc::mbar_arrive(&empty[slot]);
            }
            if (issuer && it + RG < n_stages) {
                bool ok = !abort;
                if constexpr (MT > 1) ok = ok && mbar_wait(&empty[slot], par);
                if (__all_sync(kFull, ok)) {
                    issue_stage<D>(is, hi, sc, p, &tmap_k, &tmap_v, ring + slot * SLOT, &full[slot],
                                   &slot_n[slot], policy, lane);
                } else if (!abort) {
                    abort = true;
                    if (lane == 0) report_error(p.err, PKV_DEVERR_TIMEOUT);
                }
            }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l_run[r] += __shfl_xor_sync(kFull, l_run[r], 1);
            l_run[r] += __shfl_xor_sync(kFull, l_run[r], 2);
        }
        if (bad || abort) {
            // the piece contributes nothing
            m_run[0] = m_run[1] = -INFINITY;
            l_run[0] = l_run[1] = 0.f;
#pragma unroll
            for (int j = 0; j < DTILES; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        }
        const int first = sc.worker_of(pc.start);
        const int n_pieces = sc.worker_of(pc.start + pc.n_st - 1) - first + 1;
        if (n_pieces == 1) {
            T* out = reinterpret_cast<T*>(p.out) + ((size_t)pc.seq * p.H_q + h0) * D;
            const float i0 = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
            const float i1 = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
#pragma unroll
            for (int j = 0; j < DTILES; ++j) {
                const int col = 8 * j + 2 * tq;
                if (r0 < G) {
                    out[(size_t)r0 * D + col] = Elem<T>::from_f(o[j][0] * i0);
                    out[(size_t)r0 * D + col + 1] = Elem<T>::from_f(o[j][1] * i0);
                }
                if (r1 < G) {
                    out[(size_t)r1 * D + col] = Elem<T>::from_f(o[j][2] * i1);
                    out[(size_t)r1 * D + col + 1] = Elem<T>::from_f(o[j][3] * i1);
                }
            }
            continue;
        }
        // partial state of this piece -> its workspace slot
        const size_t slot_id = (size_t)pc.seq * H_kv + pc.g + vw;
        float* acc = p.ws_acc + slot_id * G * D;
        float* ml = p.ws_ml + slot_id * G * 2;
#pragma unroll
        for (int j = 0; j < DTILES; ++j) {
            const int col = 8 * j + 2 * tq;
            if (r0 < G)
                *reinterpret_cast<float2*>(acc + (size_t)r0 * D + col) = make_float2(o[j][0], o[j][1]);
            if (r1 < G)
                *reinterpret_cast<float2*>(acc + (size_t)r1 * D + col) = make_float2(o[j][2], o[j][3]);
        }
        if (tq == 0) {
            if (r0 < G) {
                ml[r0 * 2] = m_run[0];
                ml[r0 * 2 + 1] = l_run[0];
            }
            if (r1 < G) {
                ml[r1 * 2] = m_run[1];
                ml[r1 * 2 + 1] = l_run[1];
            }
        }
        // the worker barrier orders every warp's stores before the leader's
        // device-scope fence, which orders them before the counter update
        worker_sync<MT>(worker);
        if (wtid == 0) {
            __threadfence();
            int* counter = p.counters + (size_t)pc.seq * H_kv + pc.g;
            const int last = atomicAdd(counter, 1) == n_pieces - 1;
            if (last) {
                atomicExch(counter, 0);
                __threadfence();
            }
            flags[worker] = last;
        }
        worker_sync<MT>(worker);
        if (flags[worker])
            merge_pieces<T, D, MT>(p, pc.seq, pc.g, first, n_pieces, scratch, S::kMerge, wtid,
                                   worker);
    }
    // no copy may outlive the CTA: after an abort, wait (bounded) for the
    // last stages issued
    if (abort && issuer)
        for (int j = max(0, is.issued - RG); j < is.issued; ++j)
            (void)mbar_wait(&full[j % RG], (uint32_t)((j / RG) & 1));
}

int sm_count(int device) {
    static int cached[64] = {};
    if (device < 0 || device >= 64) return 0;
    if (!cached[device]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        cached[device] = n;
    }
    return cached[device];
}

template <typename T, int D, int MT>
cudaError_t launch_lean_t(const DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv,
                          int device, cudaStream_t st) {
    using S = LeanShape<D, MT>;
    constexpr int threads = S::TS * MT * 32;
    const int smem = (lean_fixed_smem<D, MT>() + (p.B + 1) * 4 + 15) & ~15;
    auto kern = decode_lean_kernel<T, D, MT>;
    static unsigned long long attr_done = 0;
    cudaError_t e = allow_large_smem(kern, &attr_done);
    if (e != cudaSuccess) return e;
    // one wave of persistent CTAs
    static int last_smem = -1, last_per_sm = 0;
    if (smem != last_smem) {
        int n = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem);
        if (e != cudaSuccess) return e;
        last_per_sm = std::max(1, std::min(n, kLeanMaxWorkersPerSm / S::TS));
        last_smem = smem;
    }
    const int grid = std::max(1, sm_count(device)) * last_per_sm;
    return launch_kernel(kern, dim3(grid), dim3(threads), smem, st, p.pdl != 0, *tk, *tv, p);
}

template <typename T, int D>
cudaError_t launch_lean_d(const DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv,
                          int device, cudaStream_t st) {
    switch ((p.G + 15) / 16) {
        case 1: return launch_lean_t<T, D, 1>(p, tk, tv, device, st);
        case 2: return launch_lean_t<T, D, 2>(p, tk, tv, device, st);
        case 3: return launch_lean_t<T, D, 3>(p, tk, tv, device, st);
        case 4: return launch_lean_t<T, D, 4>(p, tk, tv, device, st);
        case 5: return launch_lean_t<T, D, 5>(p, tk, tv, device, st);
        case 6: return launch_lean_t<T, D, 6>(p, tk, tv, device, st);
        case 7: return launch_lean_t<T, D, 7>(p, tk, tv, device, st);
        case 8: return launch_lean_t<T, D, 8>(p, tk, tv, device, st);
        default: return cudaErrorInvalidValue;
    }
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

bool lean_supported(const pkv_pool* pool, int q_dtype, int group, int B, int max_blocks) {
    if (!pool_has_row_maps(pool) || (pool->dtype != PKV_F16 && pool->dtype != PKV_BF16)) return false;
    if (q_dtype != pool->dtype || (pool->head_dim != 64 && pool->head_dim != 128)) return false;
    if (group < 1 || group > 128 || B < 1 || B > kLeanMaxBatch) return false;
    // stage counts of the whole batch stay within int
    const long long stages = ((long long)max_blocks * pool->block_size + kStageTokens - 1) /
                             kStageTokens;
    return (long long)B * stages < (1LL << 31) && sm_count(pool->device) > 0;
}

size_t lean_workspace_bytes(const pkv_pool* pool, int B, int n_q_heads) {
    const int G = n_q_heads / pool->n_kv_heads;
    const size_t pairs = (size_t)B * pool->n_kv_heads;
    const size_t slots = pairs + (size_t)sm_count(pool->device) * kLeanMaxWorkersPerSm;
    return align256(slots * G * 2 * sizeof(float)) +
           align256(slots * G * pool->head_dim * sizeof(float)) + align256(pairs * sizeof(int));
}

cudaError_t launch_decode_lean(DecodeParams p, const pkv_pool* pool, void* ws, cudaStream_t st) {
    const size_t pairs = (size_t)p.B * p.H_kv;
    const size_t slots = pairs + (size_t)sm_count(pool->device) * kLeanMaxWorkersPerSm;
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.ws_ml = reinterpret_cast<float*>(w);
    w += align256(slots * p.G * 2 * sizeof(float));
    p.ws_acc = reinterpret_cast<float*>(w);
    w += align256(slots * p.G * pool->head_dim * sizeof(float));
    if (!p.counters) {
        // no persistent zeroed counters from the caller: use the workspace's
        p.counters = reinterpret_cast<int*>(w);
        cudaError_t e = cudaMemsetAsync(p.counters, 0, pairs * sizeof(int), st);
        if (e != cudaSuccess) return e;
    }
    const CUtensorMap* tk = reinterpret_cast<const CUtensorMap*>(pool->tmap_k);
    const CUtensorMap* tv = reinterpret_cast<const CUtensorMap*>(pool->tmap_v);
    if (pool->dtype == PKV_F16) {
        if (pool->head_dim == 64) return launch_lean_d<__half, 64>(p, tk, tv, pool->device, st);
        if (pool->head_dim == 128) return launch_lean_d<__half, 128>(p, tk, tv, pool->device, st);
    } else if (pool->dtype == PKV_BF16) {
        if (pool->head_dim == 64) return launch_lean_d<__nv_bfloat16, 64>(p, tk, tv, pool->device, st);
        if (pool->head_dim == 128)
            return launch_lean_d<__nv_bfloat16, 128>(p, tk, tv, pool->device, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pkv
