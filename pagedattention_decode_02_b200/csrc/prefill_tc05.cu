// Prompt-phase (prefill) attention over the paged cache on the fifth-generation
// tensor cores (tcgen05.mma, accumulators in tensor memory).
//
// "KV 缓存与分页注意力" §一次写一个词元: the prompt phase computes a whole prompt
// at once.  Sequence i's n_i prompt tokens are the last n_i of its c_i cached
// tokens (their keys and values already appended, after a prefix that may come
// from the prefix cache, §后来的做法, or from a recomputed history,
// §放不下的时候); token t, at position c_i - n_i + t, attends causally to
// positions 0 .. c_i - n_i + t through the block table.
//
// Work item = 256 query rows of one (sequence, KV head g), as two 128-row
// tiles that share every K/V tile: the rows of a (sequence, g) are its
// (token, query head of the group) pairs in token-major order.  Items are
// ordered group by group - all items of one (sequence, g) next to each other,
// its last rows (the most keys) first - so that the CTAs working at the same
// time re-read the same K/V from L2; one persistent CTA per SM claims them in
// that order from a global counter, one at a time, so that every CTA finishes
// within about one item of the others.  Per CTA:
//   warps 0-3, 4-7  softmax of tile 0 and tile 1: read each score tile
//              S = Q K^T from tensor memory (one row per thread), mask
//              causally, online softmax in base 2, write P (f16/bf16) back
//              over S in tensor memory, and rescale the O accumulator there
//              when the running maximum grew by more than 2^8; finally O / l
//              to global memory.  The next item's Q rows are copied into
//              shared memory (cp.async) as soon as the tile's last S of the
//              current item is done, and handed to the tensor cores before
//              the current item's output is written, so that the next S runs
//              under that epilogue;
//   warps 8, 10  producers of the 128-key K tiles and V tiles (warp 8 also
//              claims the items and hands their indices to every role through
//              a small shared-memory ring), each through
//              a two-deep ring: 2-D TMA boxes (128-byte swizzle) of up to 16
//              rows of one block and one 64-column half, read through the
//              block table from this GPU's own pool, every lane issuing its
//              own boxes;
//   warp 9     MMA: one thread issues, per tile x, S_x = Q_x K^T (M 128,
//              N 128, K = d; both operands in shared memory) and O_x += P_x V
//              (M 128, N = d, K 128; P from tensor memory, V from shared memory
//              as an MN-major operand), completion by tcgen05.commit.  Per key
//              tile: P_0 V, S_0 of the next key tile, P_1 V, S_1 of the next
//              (each S after its tile's P.V completed: S overwrites P).
// Tensor memory: tile x owns columns [256 x, 256 x + 128) for S (P packed
// into the first 64 of them) and [256 x + 128, 256 x + 128 + d) for O.
// Every wait is bounded; a wait that gives up sets PKV_DEVERR_TIMEOUT, the CTA
// stops issuing work, waits (with the default budget) for its copies and
// tensor-core operations in flight, frees its tensor memory and exits.
#include <cuda.h>

#include <type_traits>

#include "decode_launch.h"
#include "kernels_common.cuh"
#include "pool.h"
#include "tc05.cuh"
#include "tc_common.cuh"

namespace pkv {

namespace {

constexpr int kM = 128;              // rows per query tile (tensor-memory lanes)
constexpr int kTiles = 2;            // query tiles per work item
constexpr int kRows = kTiles * kM;   // rows per work item
constexpr int kN = 128;              // keys per K/V tile
constexpr int kRingK = 2;            // K ring depth
constexpr int kRingV = 2;            // V ring depth
constexpr int kProducerWarp = 8;     // K tiles
constexpr int kMmaWarp = 9;
constexpr int kProducerVWarp = 10;   // V tiles
constexpr int kThreads = 11 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTileCols = 256;  // per query tile: S (P) then O
constexpr float kRescaleLog2 = 8.f;  // keep a stale maximum while the new one is within 2^8
constexpr unsigned kFull = 0xffffffffu;
// sequences for which the group-major order and shared copies of q_starts
// and context lengths are kept in shared memory
constexpr int kMaxSchedSeqs = 1024;
// Work items are claimed at run time from a global counter (one claim per
// item, in the group-major order): the K producer claims and publishes each
// item index through a ring of kItemRing shared-memory slots, which the V
// producer, the MMA warp and the eight softmax warps each read.
constexpr int kItemRing = 4;
constexpr int kItemReaders = 10;

enum Bar {
    kKFull = 0,
    kKEmpty = kKFull + kRingK,
    kVFull = kKEmpty + kRingK,
    kVEmpty = kVFull + kRingV,
    kSFull = kVEmpty + kRingV,        // per tile: S_x computed
    kPFull = kSFull + kTiles,        // per tile: P_x written, O_x rescaled (4 warps)
    kPvDone = kPFull + kTiles,       // per tile: O_x += P_x V done
    kQFull = kPvDone + kTiles,       // per tile: Q_x rows written (4 warps)
    kItemFull = kQFull + kTiles,     // per ring slot: item index written
    kItemEmpty = kItemFull + kItemRing,   // per ring slot: read by every reader
    kDrain = kItemEmpty + kItemRing,
    kNumBars = kDrain + 1
};

template <int D>
struct Layout5 {
    static constexpr int kHalves = D / 64;
    static constexpr int kQBytes = kHalves * kM * 128;   // Q tile [half][row][128 B]
    static constexpr int kTileBytes = kHalves * kN * 128;// K or V tile [half][key][128 B]
    static constexpr int kQ = 0;                          // [kTiles][kQBytes]
    static constexpr int kK = kQ + kTiles * kQBytes;
    static constexpr int kV = kK + kRingK * kTileBytes;
    static constexpr int kBars = kV + kRingV * kTileBytes;
    // int prefix[kMaxSchedSeqs + 1], q_starts[kMaxSchedSeqs + 1], lens[kMaxSchedSeqs],
    // partial[kThreads]
    static constexpr int kItems = kBars + kNumBars * 8 + 16;   // long long [kItemRing]
    static constexpr int kSched = kItems + kItemRing * 8;
    static constexpr int kEnd = kSched + (3 * kMaxSchedSeqs + 2 + kThreads) * 4;
    // at least 116 KB, so that a second CTA never shares an SM (each CTA
    // takes all 512 tensor-memory columns)
    static constexpr int kSmem = (1024 + kEnd) > 118784 ? (1024 + kEnd) : 118784;
};

// Item parameters, computed identically by every role.
struct Item {
    int seq, g, q0, n, c, row0, base;
    int row_end[kTiles];             // exclusive row end of each query tile
    int n_kt[kTiles];                // key tiles each query tile sees (0: empty tile)
    int n_kt_all, kv_end;
    bool valid;
};

// The work order and the sequences' row offsets and lengths: shared-memory
// copies when the batch has at most kMaxSchedSeqs sequences, else global.
struct Sched {
    const int* prefix;               // items of the sequences before s; null: rank-major
    const int* q_starts;
    const int* lens;
    long long max_tiles;
};

__device__ __forceinline__ int items_of(int n, int G, int H_kv) {
    if (n <= 0) return 0;
    const long long rows = (long long)n * G;
    return (int)((rows + kRows - 1) / kRows) * H_kv;
}

// Item `it` -> (sequence, g, tile), the tile counted from the last rows.
__device__ __forceinline__ bool load_item(const PrefillParams& p, long long it, const Sched& sc,
                                          Item& x) {
    int rank;
    if (sc.prefix) {
        int lo = 0, hi = p.B - 1;          // the last s with prefix[s] <= it
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sc.prefix[mid] <= it) lo = mid; else hi = mid - 1;
        }
        x.seq = lo;
        const int local = (int)(it - sc.prefix[lo]);
        const int per_g = (sc.prefix[lo + 1] - sc.prefix[lo]) / p.H_kv;
        if (per_g <= 0) return false;
        x.g = local / per_g;
        rank = local % per_g;
    } else {
        const long long per_rank = (long long)p.B * p.H_kv;
        rank = (int)(it / per_rank);
        const int sg = (int)(it % per_rank);
        x.seq = sg / p.H_kv;
        x.g = sg % p.H_kv;
        if (rank >= sc.max_tiles) return false;
    }
    x.q0 = sc.q_starts[x.seq];
    x.n = sc.q_starts[x.seq + 1] - x.q0;
    x.c = sc.lens[x.seq];
    if (x.n <= 0) return false;
    const long long rows = (long long)x.n * p.G;
    const int n_tiles = (int)((rows + kRows - 1) / kRows);
    if (rank >= n_tiles) return false;
    const int tile = n_tiles - 1 - rank;          // last rows (most keys) first
    x.row0 = tile * kRows;
    x.valid = x.c >= 1 && (long long)x.c <= (long long)p.max_blocks * p.block_size &&
              x.n <= x.c && x.n <= p.max_q_len;
    x.base = x.c - x.n;
    x.n_kt_all = 0;
    x.kv_end = 0;
#pragma unroll
    for (int t = 0; t < kTiles; ++t) {
        const long long r0 = (long long)x.row0 + t * kM;
        if (r0 >= rows) {
            x.row_end[t] = (int)rows;
            x.n_kt[t] = 0;
            continue;
        }
        x.row_end[t] = (int)min(rows, r0 + kM);
        const int kv_end = x.base + (x.row_end[t] - 1) / p.G + 1;
        x.n_kt[t] = (kv_end + kN - 1) / kN;
        x.kv_end = max(x.kv_end, kv_end);
        x.n_kt_all = max(x.n_kt_all, x.n_kt[t]);
    }
    return true;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc05_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const PrefillParams p,
                    long long max_tiles, int allow_grouped) {
    using L = Layout5<D>;
    constexpr int HALVES = L::kHalves;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    uint8_t* sQ = sm + L::kQ;
    uint8_t* sK = sm + L::kK;
    uint8_t* sV = sm + L::kV;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::kBars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile long long* items = reinterpret_cast<volatile long long*>(sm + L::kItems);
    int* prefix = reinterpret_cast<int*>(sm + L::kSched);
    int* qs_c = prefix + kMaxSchedSeqs + 1;
    int* len_c = qs_c + kMaxSchedSeqs + 1;
    int* partial = len_c + kMaxSchedSeqs;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < kRingK; ++i) {
            mbar_init(&bar[kKFull + i], 1);
            mbar_init(&bar[kKEmpty + i], 1);
        }
        for (int i = 0; i < kRingV; ++i) {
            mbar_init(&bar[kVFull + i], 1);
            mbar_init(&bar[kVEmpty + i], 1);
        }
        for (int t = 0; t < kTiles; ++t) {
            mbar_init(&bar[kSFull + t], 1);
            mbar_init(&bar[kPFull + t], 4);
            mbar_init(&bar[kPvDone + t], 1);
            mbar_init(&bar[kQFull + t], 4);
        }
        for (int i = 0; i < kItemRing; ++i) {
            mbar_init(&bar[kItemFull + i], 1);
            mbar_init(&bar[kItemEmpty + i], kItemReaders);
        }
        mbar_init(&bar[kDrain], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tc05::tmem_alloc(tmem_slot, kTmemCols);
        tc05::tmem_relinquish();
    }
    grid_dependency_wait();
    // the work order: items per sequence and their prefix sums (every CTA
    // computes the same), with the sequences' offsets and lengths copied
    const bool grouped = allow_grouped && p.B <= kMaxSchedSeqs;
    int s0 = 0, s1 = 0;
    if (grouped) {
        for (int s = tid; s <= p.B; s += kThreads) qs_c[s] = p.q_starts[s];
        for (int s = tid; s < p.B; s += kThreads) len_c[s] = p.lens[s];
    }
    __syncthreads();
    if (grouped) {
        const int per = (p.B + kThreads - 1) / kThreads;
        s0 = min(p.B, tid * per);
        s1 = min(p.B, s0 + per);
        int sum = 0;
        for (int s = s0; s < s1; ++s) sum += items_of(qs_c[s + 1] - qs_c[s], p.G, p.H_kv);
        partial[tid] = sum;
    }
    __syncthreads();
    if (grouped && tid == 0) {
        int run = 0;
        for (int i = 0; i < kThreads; ++i) {
            const int v = partial[i];
            partial[i] = run;
            run += v;
        }
        prefix[p.B] = run;
    }
    __syncthreads();
    if (grouped) {
        int run = partial[tid];
        for (int s = s0; s < s1; ++s) {
            prefix[s] = run;
            run += items_of(qs_c[s + 1] - qs_c[s], p.G, p.H_kv);
        }
    }
    tc05::fence_before();
    __syncthreads();
    tc05::fence_after();
    const long long n_items = grouped ? (long long)prefix[p.B] : max_tiles * p.B * p.H_kv;
    const Sched sc{grouped ? prefix : nullptr, grouped ? qs_c : p.q_starts,
                   grouped ? len_c : p.lens, max_tiles};
    const uint32_t tmem = *tmem_slot;

    if (warp == kProducerWarp || warp == kProducerVWarp) {
        // ----------------------------------------------------------- producers
        // the other work items of the same (sequence, KV head), running on
        // other SMs at about the same time, read the same K/V tiles: keep them
        // in L2
        const uint64_t policy = tc05::l2_evict_last_policy();
        const int bs = p.block_size;
        const int rpb = bs < 16 ? bs : 16;          // rows per TMA box
        const int boxes = kN / rpb;                  // boxes per half-tile (<= 128)
        const int kv = warp == kProducerVWarp ? 1 : 0;   // this warp's tiles: K or V
        const int ring = kv ? kRingV : kRingK;
        long long armed = 0;                         // tiles whose barrier was armed
        bool ok = true;
        auto wait_ok = [&](uint64_t* b, uint32_t ph) {
            const bool w = mbar_wait(b, ph, p.wait_ns);
            if (!__all_sync(kFull, w) || *abort_flag) {
                if (lane == 0 && !w) report_error(p.err, PKV_DEVERR_TIMEOUT);
                if (lane == 0) *abort_flag = 1;
                ok = false;
            }
            return ok;
        };
        // the K producer's claim of the item after the one it publishes next:
        // the atomic's round trip overlaps a whole item's loads
        unsigned long long ahead = 0;
        if (kv == 0 && lane == 0) ahead = atomicAdd(p.sched, 1ull);
        for (long long kn = 0; ok; ++kn) {
            const int s_it = (int)(kn % kItemRing);
            long long it;
            if (kv == 0) {
                // publish this CTA's next item (n_items: no more), claim the
                // one after it
                if (kn >= kItemRing &&
                    !wait_ok(&bar[kItemEmpty + s_it], (uint32_t)(((kn / kItemRing) - 1) & 1)))
                    break;
                unsigned long long c = 0;
                if (lane == 0) {
                    c = ahead;
                    if (c < (unsigned long long)n_items) ahead = atomicAdd(p.sched, 1ull);
                    else c = (unsigned long long)n_items;
                    items[s_it] = (long long)c;
                    tc::mbar_arrive(&bar[kItemFull + s_it]);
                }
                it = (long long)__shfl_sync(kFull, c, 0);
            } else {
                if (!wait_ok(&bar[kItemFull + s_it], (uint32_t)((kn / kItemRing) & 1))) break;
                it = items[s_it];
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bar[kItemEmpty + s_it]);
            }
            if (it >= n_items) break;
            Item x;
            if (!load_item(p, it, sc, x) || !x.valid) continue;
            const int32_t* table = p.tables + (long long)x.seq * p.max_blocks;
            for (int kt = 0; kt < x.n_kt_all && ok; ++kt) {
                const int a0 = kt * kN;
                // the block ids of this lane's boxes (l, l + 32, ...), read
                // before waiting for the slot; -1: past the end or out of range
                // (skipped; the softmax warps zero such an item's output)
                int ids[4];
                uint32_t good = 0;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int b = lane + 32 * i;
                    const int t0 = a0 + b * rpb;
                    int id = -1;
                    if (b < boxes && t0 < x.kv_end) {
                        id = table[t0 / bs];
                        if (id < 0 || id >= p.num_blocks) id = -1;
                    }
                    ids[i] = id;
                    good += id >= 0 ? 1u : 0u;
                }
                good = __reduce_add_sync(kFull, good);
                {
                    const long long j = armed;
                    const int st = (int)(j % ring);
                    if (j >= ring && !wait_ok(&bar[(kv ? kVEmpty : kKEmpty) + st],
                                              (uint32_t)(((j / ring) - 1) & 1)))
                        break;
                    uint64_t* full = &bar[(kv ? kVFull : kKFull) + st];
                    if (tc05::elect_one())
                        mbar_arrive_expect_tx(full, good * (uint32_t)(rpb * 128 * HALVES));
                    __syncwarp();
                    armed = j + 1;
                    uint8_t* dst = (kv ? sV : sK) + st * L::kTileBytes;
                    const CUtensorMap* map = kv ? &tmap_v : &tmap_k;
                    // every lane issues its own boxes: the copies' issue
                    // latencies overlap instead of adding up
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        if (ids[i] < 0) continue;
                        const int b = lane + 32 * i;
                        const int t0 = a0 + b * rpb;
                        const int y = (ids[i] * p.H_kv + x.g) * bs + (t0 % bs);
#pragma unroll
                        for (int hf = 0; hf < HALVES; ++hf)
                            tc::tma_load_2d(dst + hf * (kN * 128) + b * rpb * 128, map, hf * 64, y,
                                            full, policy);
                    }
                    __syncwarp();
                }
            }
        }
        // no copy may outlive the CTA: the last armed tiles of this ring may
        // still be in flight (an earlier tile's slot was reused only after the
        // MMA warp had waited for it to land)
        for (long long j = armed - ring < 0 ? 0 : armed - ring; j < armed; ++j)
            (void)mbar_wait(&bar[(kv ? kVFull : kKFull) + (int)(j % ring)],
                            (uint32_t)((j / ring) & 1));
    } else if (warp == kMmaWarp) {
        // ----------------------------------------------------------------- MMA
        constexpr bool kBf16 = std::is_same<T, __nv_bfloat16>::value;
        constexpr uint32_t idS = tc05::idesc_f16(kBf16, false, kM, kN);
        constexpr uint32_t idPV = tc05::idesc_f16(kBf16, true, kM, D);
        // descriptors of the operands' first 16-element K step; later steps add
        // their byte offset / 16 to the start-address field (the addresses
        // stay below 256 KB, so the field never carries over)
        const uint64_t dQ = tc05::sdesc_sw128(smem_addr(sQ), 16, 1024);
        const uint64_t dK = tc05::sdesc_sw128(smem_addr(sK), 16, 1024);
        const uint64_t dV = tc05::sdesc_sw128(smem_addr(sV), kN * 128, 1024);
        long long kc = 0;                  // K/V tiles consumed
        long long cnt0 = 0, cnt1 = 0;      // P.V issued per query tile
        long long qc0 = 0, qc1 = 0;        // items started per query tile
        bool ok = true;
        auto wait_ok = [&](uint64_t* b, uint32_t ph) {
            const bool w = mbar_wait(b, ph, p.wait_ns);
            if (!__all_sync(kFull, w) || *abort_flag) {
                if (lane == 0 && !w) report_error(p.err, PKV_DEVERR_TIMEOUT);
                if (lane == 0) *abort_flag = 1;
                ok = false;
            }
            return ok;
        };
        // S_x of a key tile whose K sits in ring slot st
        auto issue_s = [&](int x, int st) {
            // this tile's last P.V (of this item or, at its first key tile, of
            // the previous one) is done: its P, in S_x's columns, was read.
            // Tensor-core operations on different accumulators are not
            // ordered among themselves, so issue order alone does not keep S
            // from overwriting P early.
            const long long c = x ? cnt1 : cnt0;
            if (c > 0 && !wait_ok(&bar[kPvDone + x], (uint32_t)((c - 1) & 1))) return;
            tc05::fence_after();
            const uint64_t a0 = dQ + (uint64_t)((x * L::kQBytes) >> 4);
            const uint64_t b0 = dK + (uint64_t)((st * L::kTileBytes) >> 4);
            const uint32_t d = tmem + x * kTileCols;
            if (tc05::elect_one()) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t q_off = ((kk >> 2) * (kM * 128) + (kk & 3) * 32) >> 4;
                    const uint32_t k_off = ((kk >> 2) * (kN * 128) + (kk & 3) * 32) >> 4;
                    tc05::mma_ss(d, a0 + q_off, b0 + k_off, idS, kk > 0 ? 1u : 0u);
                }
                tc05::commit(&bar[kSFull + x]);
            }
            __syncwarp();
        };
        // O_x += P_x V of a key tile whose V sits in ring slot st
        auto issue_pv = [&](int x, int st, int ksteps, bool first) {
            long long& c = x ? cnt1 : cnt0;
            if (!wait_ok(&bar[kPFull + x], (uint32_t)(c & 1))) return;
            tc05::fence_after();
            const uint64_t b0 = dV + (uint64_t)((st * L::kTileBytes) >> 4);
            const uint32_t a = tmem + x * kTileCols;
            const uint32_t d = a + kM;
            if (tc05::elect_one()) {
                if (ksteps == kN / 16) {
#pragma unroll
                    for (int kk = 0; kk < kN / 16; ++kk)
                        tc05::mma_ts(d, a + kk * 8, b0 + (uint64_t)((kk * 16 * 128) >> 4), idPV,
                                     (!first || kk > 0) ? 1u : 0u);
                } else {
                    for (int kk = 0; kk < ksteps; ++kk)
                        tc05::mma_ts(d, a + kk * 8, b0 + (uint64_t)((kk * 16 * 128) >> 4), idPV,
                                     (!first || kk > 0) ? 1u : 0u);
                }
                tc05::commit(&bar[kPvDone + x]);
            }
            __syncwarp();
            ++c;
        };
        for (long long kn = 0; ok; ++kn) {
            const int s_it = (int)(kn % kItemRing);
            if (!wait_ok(&bar[kItemFull + s_it], (uint32_t)((kn / kItemRing) & 1))) break;
            const long long it = items[s_it];
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bar[kItemEmpty + s_it]);
            if (it >= n_items) break;
            Item x;
            if (!load_item(p, it, sc, x) || !x.valid) continue;
            if (x.n_kt[0] > 0 && wait_ok(&bar[kQFull + 0], (uint32_t)(qc0 & 1))) ++qc0;
            if (ok && x.n_kt[1] > 0 && wait_ok(&bar[kQFull + 1], (uint32_t)(qc1 & 1))) ++qc1;
            if (!ok) break;
            // key tile 0: S_0, S_1
            {
                const int st = (int)(kc % kRingK);
                if (!wait_ok(&bar[kKFull + st], (uint32_t)((kc / kRingK) & 1))) break;
                if (x.n_kt[0] > 0) issue_s(0, st);
                if (ok && x.n_kt[1] > 0) issue_s(1, st);
                if (!ok) break;
                if (tc05::elect_one()) tc05::commit(&bar[kKEmpty + st]);
                __syncwarp();
            }
            for (int kt = 0; kt < x.n_kt_all && ok; ++kt) {
                const int st = (int)(kc % kRingV);          // V of this key tile
                const int st1 = (int)((kc + 1) % kRingK);   // K of the next
                const bool more = kt + 1 < x.n_kt_all;
                if (!wait_ok(&bar[kVFull + st], (uint32_t)((kc / kRingV) & 1))) break;
                if (more && !wait_ok(&bar[kKFull + st1], (uint32_t)(((kc + 1) / kRingK) & 1))) break;
                tc05::fence_after();
                const int keys = min(kN, x.kv_end - kt * kN);
                const int ksteps = (keys + 15) >> 4;
                if (keys < ksteps * 16) {
                    // keys past the end inside the last 16-key step carry P = 0;
                    // their V rows may hold anything, so make them 0 (0 * NaN
                    // would poison the sum)
                    uint8_t* vt = sV + st * L::kTileBytes;
                    const int rows = ksteps * 16 - keys;
                    for (int i = lane; i < rows * HALVES * 8; i += 32) {
                        const int r = keys + i / (HALVES * 8);
                        const int cc = i % (HALVES * 8);
                        *reinterpret_cast<uint4*>(vt + (cc >> 3) * (kN * 128) + r * 128 +
                                                  (((cc & 7) ^ (r & 7)) << 4)) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                // per tile, P.V of this key tile and then S of the next: tile
                // 0's S does not wait for tile 1's P, so the two softmax
                // groups fall half a step apart and take turns on the
                // exponential units while the tensor cores serve the other
                if (kt < x.n_kt[0]) issue_pv(0, st, ksteps, kt == 0);
                if (ok && more && kt + 1 < x.n_kt[0]) issue_s(0, st1);
                if (ok && kt < x.n_kt[1]) issue_pv(1, st, ksteps, kt == 0);
                if (!ok) break;
                if (tc05::elect_one()) tc05::commit(&bar[kVEmpty + st]);
                __syncwarp();
                if (more) {
                    if (kt + 1 < x.n_kt[1]) issue_s(1, st1);
                    if (!ok) break;
                    if (tc05::elect_one()) tc05::commit(&bar[kKEmpty + st1]);
                    __syncwarp();
                }
                ++kc;
            }
        }
        // every tensor-core operation issued has completed before the CTA
        // frees tensor memory and exits
        if (tc05::elect_one()) tc05::commit(&bar[kDrain]);
        __syncwarp();
        (void)mbar_wait(&bar[kDrain], 0);
    } else {
        // ------------------------------------------------------------- softmax
        const int t = warp >> 2;                   // query tile of this warp
        const int r = tid & (kM - 1);              // tensor-memory lane = tile row
        const uint32_t t_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16) + t * kTileCols;
        uint8_t* sQt = sQ + t * L::kQBytes;
        long long cnt = 0;
        bool ok = true;
        auto wait_ok = [&](uint64_t* b, uint32_t ph) {
            const bool w = mbar_wait(b, ph, p.wait_ns);
            if (!__all_sync(kFull, w) || *abort_flag) {
                if (lane == 0 && !w) report_error(p.err, PKV_DEVERR_TIMEOUT);
                if (lane == 0) *abort_flag = 1;
                ok = false;
            }
            return ok;
        };
        T* out = reinterpret_cast<T*>(p.out);
        const T* qg = reinterpret_cast<const T*>(p.q);
        // this thread's row of an item: position in the (sequence, g) rows,
        // whether it exists, and its token and query head
        struct Row {
            int row0, row_end, n_kt, tok, head;
            bool ok;
        };
        auto row_of = [&](const Item& x) {
            Row w;
            w.row0 = x.row0 + t * kM;
            w.row_end = t ? x.row_end[1] : x.row_end[0];
            w.n_kt = t ? x.n_kt[1] : x.n_kt[0];
            const int gr = w.row0 + r;
            w.ok = gr < w.row_end;
            const int last = w.ok ? gr : w.row_end - 1;
            w.tok = last / p.G;
            w.head = x.g * p.G + last % p.G;
            return w;
        };
        // the next item this tile takes part in; items with a bad length have
        // their rows zeroed on the way
        // 1: the next item, 0: no more (or gave up), -1: not published yet
        // (only without blocking).  Inside a key step this never blocks: the
        // K producer publishes the next item only after the MMA warp issued
        // this item's S tiles, which may wait for this step's P.
        long long kn = 0;
        auto next_item = [&](Item& x, bool block) -> int {
            for (;; ++kn) {
                const int s_it = (int)(kn % kItemRing);
                const uint32_t ph = (uint32_t)((kn / kItemRing) & 1);
                if (!block) {
                    if (!__all_sync(kFull, mbar_test_wait(&bar[kItemFull + s_it], ph))) return -1;
                } else if (!wait_ok(&bar[kItemFull + s_it], ph)) {
                    return 0;
                }
                const long long it = items[s_it];
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bar[kItemEmpty + s_it]);
                if (it >= n_items) return 0;
                if (!load_item(p, it, sc, x)) continue;
                const Row w = row_of(x);
                if (w.n_kt == 0) continue;                 // this tile is past the rows
                if (!x.valid) {
                    if (r == 0 && t == 0) report_error(p.err, PKV_DEVERR_CONTEXT_LEN);
                    if (x.n <= p.max_q_len && w.ok) {
                        T* orow = out + ((size_t)(x.q0 + w.tok) * p.H_q + w.head) * D;
                        for (int i = 0; i < D; i += 8)
                            *reinterpret_cast<uint4*>(orow + i) = make_uint4(0, 0, 0, 0);
                    }
                    continue;
                }
                ++kn;
                return 1;
            }
        };
        // this thread's Q row of item x -> shared memory (128-byte swizzle),
        // without passing through registers; rows past the end are zero
        auto fetch_q = [&](const Item& x) {
            const Row w = row_of(x);
            const T* qrow = qg + ((size_t)(x.q0 + w.tok) * p.H_q + w.head) * D;
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                uint8_t* dst = sQt + (c >> 3) * (kM * 128) + (r >> 3) * 1024 + (r & 7) * 128 +
                               (((c & 7) ^ (r & 7)) << 4);
                if (w.ok)
                    tc05::cp_async16(dst, qrow + c * 8);
                else
                    *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
            }
            tc05::cp_async_commit();
        };
        // hand the fetched Q rows to the tensor cores
        auto publish_q = [&]() {
            tc05::cp_async_wait_all();
            fence_proxy_async_smem();
            tc05::fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bar[kQFull + t]);
        };

        Item nxt;
        bool have = next_item(nxt, true) == 1;
        if (have) {
            fetch_q(nxt);
            publish_q();
        }
        while (have && ok) {
            const Item x = nxt;
            const Row w = row_of(x);
            T* orow = out + ((size_t)(x.q0 + w.tok) * p.H_q + w.head) * D;
            // block ids of the item in range? (the producer skipped bad ones;
            // checked here, while the tensor cores compute the first S, each
            // warp on its own: no CTA-wide barrier inside the roles, which a
            // warp that gave up could leave unreached)
            bool bad = false;
            {
                const int n_blk = (x.kv_end + p.block_size - 1) / p.block_size;
                const int32_t* table = p.tables + (long long)x.seq * p.max_blocks;
                for (int j = lane; j < n_blk; j += 32) {
                    const int id = table[j];
                    bad |= id < 0 || id >= p.num_blocks;
                }
                bad = __any_sync(kFull, bad);
                if (bad && r == 0 && t == 0) report_error(p.err, PKV_DEVERR_BLOCK_ID);
            }
            const int lim = x.base + w.tok;                // last visible key of this row
            const int min_lim = x.base + w.row0 / p.G;
            float m_run = -INFINITY, l_run = 0.f;
            int nx = 0;
            for (int kt = 0; kt < w.n_kt; ++kt) {
                if (!wait_ok(&bar[kSFull + t], (uint32_t)(cnt & 1))) break;
                tc05::fence_after();
                if (kt == w.n_kt - 1) {
                    // the item's last S of this tile is done: its Q rows are no
                    // longer read, so the next item's can come in
                    nx = next_item(nxt, false);
                    if (nx == 1) fetch_q(nxt);
                }
                // pass 1 over S: the largest scaled score of each row.  Keys
                // past the row's position are masked, which only the tile on
                // the diagonal needs; the scale may be negative, then the
                // smallest raw score counts.
                const int k0 = kt * kN;
                const bool full_tile = k0 + kN - 1 <= min_lim;
                const bool up = p.q_scale >= 0.f;
                float ext = up ? -INFINITY : INFINITY;
#pragma unroll 1
                for (int c = 0; c < kN / 64; ++c) {
                    uint32_t u[64];
                    tc05::tmem_ld64(t_lane + c * 64, u);
                    const int vis = lim - k0 - c * 64;     // columns j <= vis are visible
                    if (full_tile) {
                        // eight independent chains, then a tree
                        float e8[8];
#pragma unroll
                        for (int a = 0; a < 8; ++a) e8[a] = ext;
                        if (up) {
#pragma unroll
                            for (int j = 0; j < 64; ++j) e8[j & 7] = fmaxf(e8[j & 7], __uint_as_float(u[j]));
#pragma unroll
                            for (int a = 4; a > 0; a >>= 1)
#pragma unroll
                                for (int b = 0; b < a; ++b) e8[b] = fmaxf(e8[b], e8[b + a]);
                        } else {
#pragma unroll
                            for (int j = 0; j < 64; ++j) e8[j & 7] = fminf(e8[j & 7], __uint_as_float(u[j]));
#pragma unroll
                            for (int a = 4; a > 0; a >>= 1)
#pragma unroll
                                for (int b = 0; b < a; ++b) e8[b] = fminf(e8[b], e8[b + a]);
                        }
                        ext = e8[0];
                    } else {
#pragma unroll
                        for (int j = 0; j < 64; ++j) {
                            const float v = __uint_as_float(u[j]);
                            if (j <= vis) ext = up ? fmaxf(ext, v) : fminf(ext, v);
                        }
                    }
                }
                const float mt = fabsf(ext) == INFINITY ? -INFINITY : ext * p.q_scale;
                const float m_new = (mt > m_run + kRescaleLog2) ? mt : m_run;
                const float alpha = tc05::ex2(m_run - m_new);   // 0 on the first tile
                // O of this tile is idle: the MMA warp issued this S only after
                // the previous P.V had completed
                if (kt > 0 && __any_sync(kFull, m_new != m_run)) {
#pragma unroll 1
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tc05::tmem_ld32(t_lane + kM + c * 32, o);
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                        tc05::tmem_st32(t_lane + kM + c * 32, o);
                    }
                }
                m_run = m_new;
                // pass 2: probabilities -> P (f16/bf16 pairs) over S's first 64
                // columns; chunk c's P lands in columns 32 c .. 32 c + 31, all
                // of them S values already read
                const float neg_m = -m_new;
                float rs4[4] = {0.f, 0.f, 0.f, 0.f};   // independent partial sums
                // the full tile's scaling and sums two lanes at a time (packed
                // f32x2 FMA and add: half the issue slots)
                const float2 sc2 = make_float2(p.q_scale, p.q_scale);
                const float2 nm2 = make_float2(neg_m, neg_m);
                float2 rs2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll 1
                for (int c = 0; c < kN / 32; ++c) {
                    uint32_t u[32];
                    tc05::tmem_ld32(t_lane + c * 32, u);
                    uint32_t pk[16];
                    if (full_tile) {
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const float2 x2 = __ffma2_rn(
                                make_float2(__uint_as_float(u[j]), __uint_as_float(u[j + 1])), sc2, nm2);
                            const float2 e = make_float2(tc05::ex2(x2.x), tc05::ex2(x2.y));
                            rs2[(j >> 1) & 1] = __fadd2_rn(rs2[(j >> 1) & 1], e);
                            pk[j / 2] = tc::MmaType<T>::pack(e.x, e.y);
                        }
                    } else {
                        const int vis = lim - k0 - c * 32;   // columns j <= vis are visible
#pragma unroll
                        for (int j = 0; j < 32; j += 2) {
                            const float a = j <= vis
                                ? tc05::ex2(fmaf(__uint_as_float(u[j]), p.q_scale, neg_m)) : 0.f;
                            const float b = j + 1 <= vis
                                ? tc05::ex2(fmaf(__uint_as_float(u[j + 1]), p.q_scale, neg_m)) : 0.f;
                            rs4[(j >> 1) & 3] += a + b;
                            pk[j / 2] = tc::MmaType<T>::pack(a, b);
                        }
                    }
                    tc05::tmem_st16(t_lane + c * 16, pk);
                }
                tc05::tmem_st_wait();
                l_run = l_run * alpha + (((rs4[0] + rs4[1]) + (rs4[2] + rs4[3])) +
                                         ((rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y)));
                tc05::fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bar[kPFull + t]);
                ++cnt;
            }
            if (!ok) break;
            // the next item's Q goes to the tensor cores before this item's
            // epilogue, which its first S can then overlap
            if (nx == -1) {
                // not published during the last step: wait for it now that
                // this tile's P has been handed over
                nx = next_item(nxt, true);
                if (nx == 1) fetch_q(nxt);
            }
            if (!ok) break;
            const bool have_next = nx == 1;
            if (have_next) publish_q();
            // epilogue: O / l of the item's last P.V
            if (!wait_ok(&bar[kPvDone + t], (uint32_t)((cnt - 1) & 1))) break;
            tc05::fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tc05::tmem_ld32(t_lane + kM + c * 32, o);
                if (bad) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) o[j] = 0u;   // the item's keys were not read
                }
                if (w.ok) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint4 v;
                        v.x = tc::MmaType<T>::pack(__uint_as_float(o[j]) * inv, __uint_as_float(o[j + 1]) * inv);
                        v.y = tc::MmaType<T>::pack(__uint_as_float(o[j + 2]) * inv, __uint_as_float(o[j + 3]) * inv);
                        v.z = tc::MmaType<T>::pack(__uint_as_float(o[j + 4]) * inv, __uint_as_float(o[j + 5]) * inv);
                        v.w = tc::MmaType<T>::pack(__uint_as_float(o[j + 6]) * inv, __uint_as_float(o[j + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + c * 32 + j) = v;
                    }
                }
            }
            tc05::fence_before();
            have = have_next;
        }
        // a fetch still in flight (after giving up) must land before the CTA exits
        tc05::cp_async_wait_all();
    }

    // every role is done: free tensor memory
    tc05::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc05::fence_after();
        tc05::tmem_dealloc(tmem, kTmemCols);
    }
    // this CTA claims no more items: the last CTA to get here zeroes the
    // launch's counters for the launch that next takes them
    if (tid == 0) {
        __threadfence();
        if (atomicAdd(p.sched + 1, 1ull) == gridDim.x - 1) {
            __threadfence();
            p.sched[0] = 0;
            p.sched[1] = 0;
        }
    }
}

template <typename T, int D>
cudaError_t launch_t(const PrefillParams& p, const pkv_pool* pool, cudaStream_t st) {
    using L = Layout5<D>;
    static_assert(L::kSmem <= 227 * 1024, "shared memory budget");
    auto kern = prefill_tc05_kernel<T, D>;
    static unsigned long long attr_done = 0;
    cudaError_t e = allow_large_smem(kern, &attr_done);
    if (e != cudaSuccess) return e;
    const long long max_tiles = ((long long)p.max_q_len * p.G + kRows - 1) / kRows;
    const long long n_items = max_tiles * p.B * p.H_kv;   // an upper bound
    if (n_items <= 0) return cudaSuccess;
    const int sms = pool->sm_count > 0 ? pool->sm_count : 148;
    const int grid = (int)(n_items < sms ? n_items : sms);
    // the group-major order counts items in 32-bit prefix sums
    const int allow_grouped = n_items < (1LL << 31) ? 1 : 0;
    return launch_kernel(kern, dim3(grid), dim3(kThreads), L::kSmem, st, false,
                         *reinterpret_cast<const CUtensorMap*>(pool->tmap_k),
                         *reinterpret_cast<const CUtensorMap*>(pool->tmap_v), p, max_tiles,
                         allow_grouped);
}

}  // namespace

cudaError_t launch_prefill_tc05(const PrefillParams& p, const pkv_pool* pool, cudaStream_t st) {
    if (pool->dtype == PKV_F16) {
        if (pool->head_dim == 64) return launch_t<__half, 64>(p, pool, st);
        if (pool->head_dim == 128) return launch_t<__half, 128>(p, pool, st);
    } else if (pool->dtype == PKV_BF16) {
        if (pool->head_dim == 64) return launch_t<__nv_bfloat16, 64>(p, pool, st);
        if (pool->head_dim == 128) return launch_t<__nv_bfloat16, 128>(p, pool, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pkv
