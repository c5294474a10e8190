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
// Worker = MT warps of 8 query heads of the KV head's group each; a warp
// computes S^T = K Q^T and O^T += V^T P^T with mma.sync m16n8k16 (16 tokens
// or 16 d-rows by 8 heads: no padded rows up to 8 heads per KV head); a CTA
// holds TS workers.  Each worker owns a ring of RG
// 16-token stage slots filled by 2-D TMA loads (128-byte swizzle, plain loads
// of this GPU's own memory) that its first warp issues, RG stages ahead of
// the one being consumed; with MT > 1 an "empty" mbarrier per slot tells the
// issuing warp when every warp of the worker is done with it.  Many
// independent workers per SM hide each one's serial chain (scores, softmax,
// P.V) and the copies' latency.  A stage whose block id is out of range is not
// loaded (the piece's contribution becomes zero and the device error word
// records it).  Every wait is bounded.
#include <cuda.h>

#include <atomic>

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

// Workers per CTA and ring slots per worker for MT warps (of 8 query heads)
// per worker.
template <int D, int MT>
struct LeanShape {
    static constexpr int TS = MT == 1 ? 4 : (MT == 2 ? 2 : 1);   // <= 16 warps per CTA
    static constexpr int RG = D == 128 ? 3 : 4;
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

// Merge of a split pair by the worker that finished its last piece (NTH
// threads, t = 0 .. NTH - 1): the pair's pieces left (running max, sum,
// accumulator) per head in consecutive workspace slots (pair + first worker
// .. pair + last worker), combined by log-sum-exp.  Each thread takes 4
// float4 outputs per pass, two pieces at a time; all loads of a step are
// issued before any is used.  Kept out of line so that its registers do not
// count against the streaming loop's.
template <typename T, int D, int NTH>
__device__ __noinline__ void merge_pair(const DecodeParams& p, int pair, int first, int n_pieces,
                                        int t) {
    constexpr int E = 4;
    const int G = p.G;
    const int seq = seq_of(p, pair / p.H_kv), g = pair % p.H_kv;
    const int total = G * (D / 4);
    const size_t slot0 = (size_t)pair + first;
    const float2* ml = reinterpret_cast<const float2*>(p.ws_ml) + slot0 * G;
    const float4* acc = reinterpret_cast<const float4*>(p.ws_acc) + slot0 * G * (D / 4);
    T* out = reinterpret_cast<T*>(p.out) + ((size_t)seq * p.H_q + (size_t)g * G) * D;
    for (int base = t; base < total; base += NTH * E) {
        float M[E], L[E];
        float4 O[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            M[e] = -INFINITY;
            L[e] = 0.f;
            O[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll 2
        for (int j = 0; j < n_pieces; ++j) {
            float2 v[E];
            float4 a[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int i = min(base + e * NTH, total - 1);
                v[e] = __ldcg(ml + (size_t)j * G + i / (D / 4));
                a[e] = __ldcg(acc + (size_t)j * G * (D / 4) + i);
            }
#pragma unroll
            for (int e = 0; e < E; ++e) {
                if (v[e].x == -INFINITY) continue;
                const float Mn = fmaxf(M[e], v[e].x);
                const float so = exp2f(M[e] - Mn), sn = exp2f(v[e].x - Mn);
                L[e] = L[e] * so + v[e].y * sn;
                O[e].x = O[e].x * so + a[e].x * sn;
                O[e].y = O[e].y * so + a[e].y * sn;
                O[e].z = O[e].z * so + a[e].z * sn;
                O[e].w = O[e].w * so + a[e].w * sn;
                M[e] = Mn;
            }
        }
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int i = base + e * NTH;
            if (i >= total) break;
            const float s = L[e] > 0.f ? 1.f / L[e] : 0.f;
            T* o = out + (size_t)i * 4;
            o[0] = Elem<T>::from_f(O[e].x * s);
            o[1] = Elem<T>::from_f(O[e].y * s);
            o[2] = Elem<T>::from_f(O[e].z * s);
            o[3] = Elem<T>::from_f(O[e].w * s);
        }
    }
}

template <int D, int MT>
__host__ __device__ constexpr int lean_fixed_smem() {
    using S = LeanShape<D, MT>;
    // rings (1024-aligned) + full/empty barriers + slot token counts + per
    // worker flags + per-warp scan totals; prefix sums follow
    return 1024 + S::TS * S::RG * LeanCfg<D>::kSlot + 2 * S::TS * S::RG * 8 + S::TS * S::RG * 4 +
           S::TS * 4 + 32 * 4;
}

// A walk over a worker's share, one 16-token stage at a time, RG stages ahead
// of the consumption; held by the worker's first warp (all lanes).
struct Cursor {
    long long pos;       // the next piece starts at pos
    int seq, g;          // piece being walked
    int s, s1;           // its next stage and its end (s == s1: take the next piece)
    int trow;            // its table row (-1: invalid)
    int c;               // its context length
    int wb, wid;         // table entries wb .. wb + 31, one per lane
    int count;           // stages walked so far
};

__device__ __forceinline__ void cursor_init(Cursor& cu, long long lo) {
    cu.pos = lo;
    cu.s = cu.s1 = 0;
    cu.count = 0;
}

// Moves the cursor over its next stage.  Returns the stage's box count nb
// (2-D TMA boxes of min(bs, 16) rows each) and, for lane < nb, that box's
// TMA row in *y (-1 when its block id is out of range, or the table row is
// invalid); *n = valid tokens of the stage.
__device__ __forceinline__ int cursor_stage(Cursor& cu, long long hi, const Schedule& sc,
                                            const DecodeParams& p, int lane, int* y, int* n) {
    if (cu.s == cu.s1) {
        const Piece pc = sc.at(cu.pos, hi);
        cu.pos = pc.start + pc.s1;
        cu.seq = pc.seq;
        cu.g = pc.g;
        cu.s = pc.s0;
        cu.s1 = pc.s1;
        cu.trow = (int)table_row(p, pc.seq);
        cu.c = p.lens[pc.seq];
        cu.wb = -1;
    }
    const int bs = p.block_size;
    const int rpb = bs < kStageTokens ? bs : kStageTokens;   // rows per box
    const int a = cu.s * kStageTokens;
    *n = min(kStageTokens, cu.c - a);
    const int nb = (*n + rpb - 1) / rpb;
    const int lb1 = (a + *n - 1) / bs;
    if (cu.wb < 0 || lb1 >= cu.wb + 32) {
        cu.wb = a / bs;
        cu.wid = (cu.trow >= 0 && cu.wb + lane < p.max_blocks)
                     ? p.tables[(long long)cu.trow * p.max_blocks + cu.wb + lane]
                     : -1;
    }
    const int t0 = a + (lane < nb ? lane : 0) * rpb;
    const int lb = t0 / bs;
    const int id = __shfl_sync(kFull, cu.wid, lb - cu.wb);
    *y = (cu.trow >= 0 && id >= 0 && id < p.num_blocks) ? (id * p.H_kv + cu.g) * bs + (t0 - lb * bs)
                                                         : -1;
    ++cu.s;
    ++cu.count;
    return nb;
}

// Load the cursor's next stage into a ring slot: one box per lane < nb, K
// and V, every 64-column half; a stage with an out-of-range block id is not
// loaded (slot_n = -1) and its barrier phase completes without bytes.
template <int D>
__device__ __forceinline__ void issue_stage(Cursor& cu, long long hi, const Schedule& sc,
                                            const DecodeParams& p, const CUtensorMap* tk,
                                            const CUtensorMap* tv, uint8_t* slot_mem,
                                            uint64_t* full, volatile int* slot_n, uint64_t policy,
                                            int lane) {
    constexpr int TILE = LeanCfg<D>::kSlot / 2;
    constexpr int HALVES = D / 64;
    int y, n;
    const int nb = cursor_stage(cu, hi, sc, p, lane, &y, &n);
    const int rpb = p.block_size < kStageTokens ? p.block_size : kStageTokens;
    const bool bad = __any_sync(kFull, lane < nb && y < 0);
    if (lane == 0) {
        *slot_n = bad ? -1 : n;
        if (bad) {
            report_error(p.err, PKV_DEVERR_BLOCK_ID);
            tc::mbar_arrive(full);
        } else {
            mbar_arrive_expect_tx(full, (uint32_t)(2 * HALVES * nb * rpb * 128));
        }
    }
    __syncwarp();
    if (!bad && lane < nb) {
#pragma unroll
        for (int hf = 0; hf < HALVES; ++hf) {
            const int off = hf * (kStageTokens * 128) + lane * rpb * 128;
            tc::tma_load_2d(slot_mem + off, tk, hf * 64, y, full, policy);
            tc::tma_load_2d(slot_mem + TILE + off, tv, hf * 64, y, full, policy);
        }
    }
    __syncwarp();
}

// Barrier over the MT warps of one worker (named barrier 1 + worker).
template <int MT>
__device__ __forceinline__ void worker_sync(int worker) {
    if constexpr (MT == 1) {
        __syncwarp();
    } else {
        asm volatile("bar.sync %0, %1;" ::"r"(1 + worker), "r"(MT * 32) : "memory");
    }
}

template <typename T, int D, int MT>
__global__ void __launch_bounds__(LeanShape<D, MT>::TS * MT * 32, MT <= 2 ? 2 : 1)
decode_lean_kernel(const __grid_constant__ CUtensorMap tmap_k,
                   const __grid_constant__ CUtensorMap tmap_v, const DecodeParams p) {
    using S = LeanShape<D, MT>;
    constexpr int TS = S::TS;
    constexpr int RG = S::RG;
    constexpr int SLOT = LeanCfg<D>::kSlot;
    constexpr int TILE = SLOT / 2;
    constexpr int NT = TS * MT * 32;
    static_assert(NT / 32 <= 32, "scan totals");

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* rings = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint64_t* fulls = reinterpret_cast<uint64_t*>(rings + TS * RG * SLOT);   // [TS][RG]
    uint64_t* empties = fulls + TS * RG;                                     // [TS][RG]
    volatile int* slot_ns = reinterpret_cast<volatile int*>(empties + TS * RG);   // [TS][RG]
    volatile int* flags = slot_ns + TS * RG;                                 // [TS] last-piece flag
    int* wsum = const_cast<int*>(flags + TS);                                // [32]
    int* pre = wsum + 32;                                                    // [B + 1]

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
    for (int slot = blockIdx.x; slot < B; slot += gridDim.x) {
        if (pre[slot + 1] != pre[slot]) continue;
        if (tid == 0) report_error(p.err, PKV_DEVERR_CONTEXT_LEN);
        T* out = reinterpret_cast<T*>(p.out) + (size_t)seq_of(p, slot) * p.H_q * D;
        for (int i = tid; i < p.H_q * D; i += NT) out[i] = Elem<T>::from_f(0.f);
    }

    // with fewer stages than workers the surplus workers stay idle, so that
    // every share is non-empty and a pair's pieces sit in consecutive workers
    const long long total = (long long)H_kv * pre[B];
    if (total == 0) return;
    const long long n_workers = (long long)gridDim.x * TS;
    const Schedule sc{pre, B, H_kv, (int)(total < n_workers ? total : n_workers), total};

    // ------------------------------------------------------------- workers
    const int worker = warp / MT;
    const int mt = warp % MT;
    const int vw = blockIdx.x * TS + worker;   // this worker's index on the stage line
    const long long lo = vw < sc.n ? sc.lo(vw) : 0;
    const long long hi = vw < sc.n ? sc.lo(vw + 1) : 0;
    const int n_stages = (int)(hi - lo);

    uint8_t* ring = rings + worker * RG * SLOT;
    uint64_t* full = fulls + worker * RG;
    uint64_t* empty = empties + worker * RG;
    volatile int* slot_n = slot_ns + worker * RG;
    const bool issuer = mt == 0;
    const uint64_t policy = l2_evict_first_policy();

    Cursor is;
    cursor_init(is, lo);
    if (issuer) {
        const int pro = min(RG, n_stages);
        for (int k = 0; k < pro; ++k)
            issue_stage<D>(is, hi, sc, p, &tmap_k, &tmap_v, ring + k * SLOT, &full[k], &slot_n[k],
                           policy, lane);
    }

    const int gq = lane >> 2;
    const int tq = lane & 3;
    const int hw = mt * 8;                    // this warp's first head of the group
    const int ha = hw + 2 * tq, hb = ha + 1;  // this lane's two heads
    long long pos = lo;
    int it = 0;
    bool abort = false;
    while (pos < hi) {
        const Piece pc = sc.at(pos, hi);
        pos = pc.start + pc.s1;
        const int h0 = pc.g * G;
        const int oseq = seq_of(p, pc.seq);   // pieces walk launch slots
        uint32_t qb[D / 16][2];
        tc::load_qT_frags<T, D>(qb, reinterpret_cast<const T*>(p.q) + ((size_t)oseq * p.H_q + h0) * D,
                                hw, G, lane);
        float o[D / 16][4];
#pragma unroll
        for (int j = 0; j < D / 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        float m_run[2] = {-INFINITY, -INFINITY};
        float l_run[2] = {0.f, 0.f};
        bool bad = false;
        for (int s = pc.s0; s < pc.s1; ++s, ++it) {
            const int slot = it % RG;
            const uint32_t par = (uint32_t)((it / RG) & 1);
            if (!abort) {
                const bool ok = mbar_wait(&full[slot], par, p.wait_ns);
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
                    tc::stage_body_t<T, D>(qb, kt, kt + TILE, n, p.q_scale, o, m_run, l_run, lane);
                __syncwarp();
            }
            if constexpr (MT > 1) {
                if (lane == 0) tc::mbar_arrive(&empty[slot]);
            }
            if (issuer && it + RG < n_stages) {
                bool ok = !abort;
                if constexpr (MT > 1) ok = ok && mbar_wait(&empty[slot], par, p.wait_ns);
                if (__all_sync(kFull, ok)) {
                    issue_stage<D>(is, hi, sc, p, &tmap_k, &tmap_v, ring + slot * SLOT, &full[slot],
                                   &slot_n[slot], policy, lane);
                } else if (!abort) {
                    abort = true;
                    if (lane == 0) report_error(p.err, PKV_DEVERR_TIMEOUT);
                }
            }
        }
        // sums over the lanes holding the same heads (one per token pair)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            l_run[h] += __shfl_xor_sync(kFull, l_run[h], 4);
            l_run[h] += __shfl_xor_sync(kFull, l_run[h], 8);
            l_run[h] += __shfl_xor_sync(kFull, l_run[h], 16);
        }
        if (bad || abort) {
            // the piece contributes nothing
            m_run[0] = m_run[1] = -INFINITY;
            l_run[0] = l_run[1] = 0.f;
#pragma unroll
            for (int j = 0; j < D / 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
        }
        const int first = sc.worker_of(pc.start);
        const int n_pieces = sc.worker_of(pc.start + pc.n_st - 1) - first + 1;
        if (n_pieces == 1) {
            T* out = reinterpret_cast<T*>(p.out) + ((size_t)oseq * p.H_q + h0) * D;
            const float ia = l_run[0] > 0.f ? 1.f / l_run[0] : 0.f;
            const float ib = l_run[1] > 0.f ? 1.f / l_run[1] : 0.f;
#pragma unroll
            for (int j = 0; j < D / 16; ++j) {
                const int d = 16 * j + gq;
                if (ha < G) {
                    out[(size_t)ha * D + d] = Elem<T>::from_f(o[j][0] * ia);
                    out[(size_t)ha * D + d + 8] = Elem<T>::from_f(o[j][2] * ia);
                }
                if (hb < G) {
                    out[(size_t)hb * D + d] = Elem<T>::from_f(o[j][1] * ib);
                    out[(size_t)hb * D + d + 8] = Elem<T>::from_f(o[j][3] * ib);
                }
            }
            continue;
        }
        // partial state of this piece -> its workspace slot; the worker that
        // finishes the pair's last piece merges them all (counter below)
        const int pair = pc.seq * H_kv + pc.g;
        const size_t slot_id = (size_t)pair + vw;
        float* acc = p.ws_acc + slot_id * G * D;
        float* ml = p.ws_ml + slot_id * G * 2;
#pragma unroll
        for (int j = 0; j < D / 16; ++j) {
            const int d = 16 * j + gq;
            if (ha < G) {
                acc[(size_t)ha * D + d] = o[j][0];
                acc[(size_t)ha * D + d + 8] = o[j][2];
            }
            if (hb < G) {
                acc[(size_t)hb * D + d] = o[j][1];
                acc[(size_t)hb * D + d + 8] = o[j][3];
            }
        }
        if (gq == 0) {
            if (ha < G) {
                ml[ha * 2] = m_run[0];
                ml[ha * 2 + 1] = l_run[0];
            }
            if (hb < G) {
                ml[hb * 2] = m_run[1];
                ml[hb * 2 + 1] = l_run[1];
            }
        }
        // the worker barrier orders every warp's stores before the leader's
        // device-scope fence, which orders them before the counter update
        worker_sync<MT>(worker);
        if (mt == 0 && lane == 0) {
            __threadfence();
            int* counter = p.counters + pair;
            const int last = atomicAdd(counter, 1) == n_pieces - 1;
            if (last) {
                atomicExch(counter, 0);
                __threadfence();
            }
            flags[worker] = last;
        }
        worker_sync<MT>(worker);
        if (flags[worker]) merge_pair<T, D, MT * 32>(p, pair, first, n_pieces, mt * 32 + lane);
        worker_sync<MT>(worker);   // the flag is read by every warp before it is reused
    }
    // no copy may outlive the CTA: after an abort, wait (bounded) for the
    // last stages issued
    if (abort && issuer)
        for (int j = max(0, is.count - RG); j < is.count; ++j)
            (void)mbar_wait(&full[j % RG], (uint32_t)((j / RG) & 1));
}

template <typename T, int D, int MT>
cudaError_t launch_lean_t(const DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv,
                          int sms, cudaStream_t st, cudaEvent_t mid) {
    using S = LeanShape<D, MT>;
    constexpr int threads = S::TS * MT * 32;
    const int smem = (lean_fixed_smem<D, MT>() + (p.B + 1) * 4 + 15) & ~15;
    auto kern = decode_lean_kernel<T, D, MT>;
    static unsigned long long attr_done = 0;
    cudaError_t e = allow_large_smem(kern, &attr_done);
    if (e != cudaSuccess) return e;
    // one wave of persistent CTAs; the occupancy of the last shared-memory
    // size is cached as one atomic word (size << 32 | CTAs per SM), so that
    // calls from several host threads never see a half-written pair
    static std::atomic<unsigned long long> occ_cache{~0ull};
    unsigned long long occ = occ_cache.load(std::memory_order_acquire);
    int per_sm = (int)(occ & 0xffffffffull);
    if ((occ >> 32) != (unsigned long long)(unsigned)smem) {
        int n = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem);
        if (e != cudaSuccess) return e;
        per_sm = std::max(1, std::min(n, kLeanMaxWorkersPerSm / S::TS));
        occ_cache.store(((unsigned long long)(unsigned)smem << 32) | (unsigned)per_sm,
                        std::memory_order_release);
    }
    const int grid = std::max(1, sms) * per_sm;
    e = launch_kernel(kern, dim3(grid), dim3(threads), smem, st, p.pdl != 0, *tk, *tv, p);
    if (e == cudaSuccess && mid) e = cudaEventRecord(mid, st);
    return e;
}

template <typename T, int D>
cudaError_t launch_lean_d(const DecodeParams& p, const CUtensorMap* tk, const CUtensorMap* tv,
                          int sms, cudaStream_t st, cudaEvent_t mid) {
    // warps of 8 query heads each
    switch ((p.G + 7) / 8) {
        case 1: return launch_lean_t<T, D, 1>(p, tk, tv, sms, st, mid);
        case 2: return launch_lean_t<T, D, 2>(p, tk, tv, sms, st, mid);
        case 3: return launch_lean_t<T, D, 3>(p, tk, tv, sms, st, mid);
        case 4: return launch_lean_t<T, D, 4>(p, tk, tv, sms, st, mid);
        case 5: return launch_lean_t<T, D, 5>(p, tk, tv, sms, st, mid);
        case 6: return launch_lean_t<T, D, 6>(p, tk, tv, sms, st, mid);
        case 7: return launch_lean_t<T, D, 7>(p, tk, tv, sms, st, mid);
        case 8: return launch_lean_t<T, D, 8>(p, tk, tv, sms, st, mid);
        case 9: return launch_lean_t<T, D, 9>(p, tk, tv, sms, st, mid);
        case 10: return launch_lean_t<T, D, 10>(p, tk, tv, sms, st, mid);
        case 11: return launch_lean_t<T, D, 11>(p, tk, tv, sms, st, mid);
        case 12: return launch_lean_t<T, D, 12>(p, tk, tv, sms, st, mid);
        case 13: return launch_lean_t<T, D, 13>(p, tk, tv, sms, st, mid);
        case 14: return launch_lean_t<T, D, 14>(p, tk, tv, sms, st, mid);
        case 15: return launch_lean_t<T, D, 15>(p, tk, tv, sms, st, mid);
        case 16: return launch_lean_t<T, D, 16>(p, tk, tv, sms, st, mid);
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
    return (long long)B * stages < (1LL << 31) && pool->sm_count > 0;
}

// piece slots: pair + worker index
size_t lean_slots(const pkv_pool* pool, int B) {
    const size_t pairs = (size_t)B * pool->n_kv_heads;
    return pairs + (size_t)pool->sm_count * kLeanMaxWorkersPerSm;
}

size_t lean_workspace_bytes(const pkv_pool* pool, int B, int n_q_heads) {
    const int G = n_q_heads / pool->n_kv_heads;
    const size_t slots = lean_slots(pool, B);
    return align256(slots * G * 2 * sizeof(float)) +
           align256(slots * G * pool->head_dim * sizeof(float)) +
           align256((size_t)B * pool->n_kv_heads * sizeof(int));
}

cudaError_t launch_decode_lean(DecodeParams p, const pkv_pool* pool, void* ws, cudaStream_t st,
                               cudaEvent_t mid) {
    const size_t slots = lean_slots(pool, p.B);
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.ws_ml = reinterpret_cast<float*>(w);
    w += align256(slots * p.G * 2 * sizeof(float));
    p.ws_acc = reinterpret_cast<float*>(w);
    w += align256(slots * p.G * pool->head_dim * sizeof(float));
    if (!p.counters) {
        // no persistent zeroed counters from the caller: the workspace's
        p.counters = reinterpret_cast<int*>(w);
        cudaError_t e = cudaMemsetAsync(p.counters, 0, (size_t)p.B * p.H_kv * sizeof(int), st);
        if (e != cudaSuccess) return e;
    }
    const CUtensorMap* tk = reinterpret_cast<const CUtensorMap*>(pool->tmap_k);
    const CUtensorMap* tv = reinterpret_cast<const CUtensorMap*>(pool->tmap_v);
    if (pool->dtype == PKV_F16) {
        if (pool->head_dim == 64) return launch_lean_d<__half, 64>(p, tk, tv, pool->sm_count, st, mid);
        if (pool->head_dim == 128) return launch_lean_d<__half, 128>(p, tk, tv, pool->sm_count, st, mid);
    } else if (pool->dtype == PKV_BF16) {
        if (pool->head_dim == 64) return launch_lean_d<__nv_bfloat16, 64>(p, tk, tv, pool->sm_count, st, mid);
        if (pool->head_dim == 128)
            return launch_lean_d<__nv_bfloat16, 128>(p, tk, tv, pool->sm_count, st, mid);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pkv
