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
// Work item = 128 query rows of one (sequence, KV head g): the rows of a
// (sequence, g) are its (token, query head of the group) pairs in token-major
// order, so all 128 rows share one stream of K/V tiles.  A persistent CTA per
// SM walks the items heaviest first (the last rows of the longest prompts see
// the most keys) in a grid-stride order.  Per CTA:
//   warps 0-3  softmax: load the item's Q tile into shared memory, read each
//              score tile S = Q K^T from tensor memory (one row per thread),
//              mask causally, online softmax in base 2, write P (f16/bf16) to
//              shared memory and rescale the O accumulator in tensor memory
//              when the running maximum grew by more than 2^8; finally
//              O / l to global memory;
//   warp 4     producer: 128-key K and V tiles through two-deep rings, each
//              tile 16-key stages of 2-D TMA boxes (128-byte swizzle) read
//              through the block table from this GPU's own pool;
//   warp 5     MMA: one thread issues S_j = Q K_j^T (M 128, N 128, K = d)
//              into one of two tensor-memory score buffers and O += P_j V_j
//              (M 128, N = d, K 128) with tcgen05.mma, completion signalled
//              by tcgen05.commit; S_{j+1} is issued before P_j is ready so
//              the tensor pipe computes it while the softmax warps work.
// Tensor memory: S buffers in columns [0, 128) and [128, 256), O in [256,
// 256 + d).  Every wait is bounded; a wait that gives up sets
// PKV_DEVERR_TIMEOUT, the CTA stops issuing work, waits (with the normal
// budget) for its copies and tensor-core operations in flight, frees its
// tensor memory and exits.
#include <cuda.h>

#include <type_traits>

#include "decode_launch.h"
#include "kernels_common.cuh"
#include "pool.h"
#include "tc05.cuh"
#include "tc_common.cuh"

namespace pkv {

namespace {

constexpr int kM = 128;             // query rows per item (tensor-memory lanes)
constexpr int kN = 128;             // keys per K/V tile
constexpr int kRing = 2;            // K ring and V ring depth
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 6 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;       // two score buffers of kN columns
constexpr uint32_t kColO = 2 * kN;  // the output accumulator
constexpr float kRescaleLog2 = 8.f; // keep a stale maximum while the new one is within 2^8
constexpr unsigned kFull = 0xffffffffu;

enum Bar {
    kKFull = 0,
    kKEmpty = kKFull + kRing,
    kVFull = kKEmpty + kRing,
    kVEmpty = kVFull + kRing,
    kSFull = kVEmpty + kRing,
    kSEmpty = kSFull + 2,
    kPFull = kSEmpty + 2,
    kPvDone = kPFull + 1,
    kQFull = kPvDone + 1,
    kDrain = kQFull + 1,
    kNumBars = kDrain + 1
};

template <int D>
struct Layout5 {
    static constexpr int kHalves = D / 64;
    static constexpr int kQBytes = kHalves * kM * 128;   // Q tile [half][row][128 B]
    static constexpr int kPBytes = 2 * kM * 128;         // P tile [key half][row][128 B]
    static constexpr int kTileBytes = kHalves * kN * 128;// K or V tile [half][key][128 B]
    static constexpr int kQ = 0;
    static constexpr int kP = kQ + kQBytes;
    static constexpr int kK = kP + kPBytes;
    static constexpr int kV = kK + kRing * kTileBytes;
    static constexpr int kBars = kV + kRing * kTileBytes;
    static constexpr int kEnd = kBars + kNumBars * 8 + 16;
    // at least 116 KB, so that a second CTA never shares an SM (each CTA
    // takes all 512 tensor-memory columns)
    static constexpr int kSmem = (1024 + kEnd) > 118784 ? (1024 + kEnd) : 118784;
};

// Item parameters, computed identically by every role.
struct Item {
    int seq, g, q0, n, c, row0, row_end, base, kv_end, n_kt;
    bool valid;
};

__device__ __forceinline__ bool load_item(const PrefillParams& p, long long it,
                                          long long per_rank, Item& x) {
    const int rank = (int)(it / per_rank);
    const int sg = (int)(it % per_rank);
    x.seq = sg / p.H_kv;
    x.g = sg % p.H_kv;
    x.q0 = p.q_starts[x.seq];
    x.n = p.q_starts[x.seq + 1] - x.q0;
    x.c = p.lens[x.seq];
    if (x.n <= 0) return false;
    const long long rows = (long long)x.n * p.G;
    const int n_tiles = (int)((rows + kM - 1) / kM);
    if (rank >= n_tiles) return false;
    const int tile = n_tiles - 1 - rank;          // heaviest (last rows) first
    x.row0 = tile * kM;
    x.row_end = (int)min(rows, (long long)x.row0 + kM);
    x.valid = x.c >= 1 && (long long)x.c <= (long long)p.max_blocks * p.block_size &&
              x.n <= x.c && x.n <= p.max_q_len;
    x.base = x.c - x.n;
    x.kv_end = x.base + (x.row_end - 1) / p.G + 1;
    x.n_kt = (x.kv_end + kN - 1) / kN;
    return true;
}

template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc05_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v, const PrefillParams p,
                    long long n_items) {
    using L = Layout5<D>;
    constexpr int HALVES = L::kHalves;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    uint8_t* sQ = sm + L::kQ;
    uint8_t* sP = sm + L::kP;
    uint8_t* sK = sm + L::kK;
    uint8_t* sV = sm + L::kV;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + L::kBars);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + kNumBars);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (tid == 0) {
        for (int i = 0; i < kRing; ++i) {
            mbar_init(&bar[kKFull + i], 1);
            mbar_init(&bar[kKEmpty + i], 1);
            mbar_init(&bar[kVFull + i], 1);
            mbar_init(&bar[kVEmpty + i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bar[kSFull + i], 1);
            mbar_init(&bar[kSEmpty + i], kSoftmaxWarps);
        }
        mbar_init(&bar[kPFull], kSoftmaxWarps);
        mbar_init(&bar[kPvDone], 1);
        mbar_init(&bar[kQFull], kSoftmaxWarps);
        mbar_init(&bar[kDrain], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tc05::tmem_alloc(tmem_slot, kTmemCols);
        tc05::tmem_relinquish();
    }
    tc05::fence_before();
    __syncthreads();
    tc05::fence_after();
    const uint32_t tmem = *tmem_slot;

    grid_dependency_wait();
    const long long per_rank = (long long)p.B * p.H_kv;

    if (warp == kProducerWarp) {
        // ------------------------------------------------------------ producer
        const uint64_t policy = l2_evict_first_policy();
        const int bs = p.block_size;
        const int rpb = bs < 16 ? bs : 16;          // rows per TMA box
        const int boxes = kN / rpb;                  // boxes per half-tile
        long long armed[2] = {0, 0};                 // K, V tiles whose barrier was armed
        bool ok = true;
        for (long long it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            Item x;
            if (!load_item(p, it, per_rank, x) || !x.valid) continue;
            const int32_t* table = p.tables + (long long)x.seq * p.max_blocks;
            for (int kt = 0; kt < x.n_kt && ok; ++kt) {
                const int a0 = kt * kN;
                for (int kv = 0; kv < 2; ++kv) {
                    const long long j = armed[kv];
                    const int st = (int)(j % kRing);
                    if (j >= kRing) {
                        const bool w = mbar_wait(&bar[(kv ? kVEmpty : kKEmpty) + st],
                                                 (uint32_t)(((j / kRing) - 1) & 1), p.wait_ns);
                        if (!__all_sync(kFull, w) || *abort_flag) {
                            if (lane == 0 && !w) report_error(p.err, PKV_DEVERR_TIMEOUT);
                            if (lane == 0) *abort_flag = 1;
                            ok = false;
                            break;
                        }
                    }
                    // lane l handles boxes l, l + 32, ...; ids out of range are
                    // skipped (the softmax warps zero such an item's output)
                    uint32_t good = 0;
                    for (int b = lane; b < boxes; b += 32) {
                        const int t0 = a0 + b * rpb;
                        if (t0 >= x.kv_end) break;
                        const int id = table[t0 / bs];
                        good += (id >= 0 && id < p.num_blocks) ? 1u : 0u;
                    }
                    good = __reduce_add_sync(kFull, good);
                    uint64_t* full = &bar[(kv ? kVFull : kKFull) + st];
                    if (lane == 0)
                        mbar_arrive_expect_tx(full, good * (uint32_t)(rpb * 128 * HALVES));
                    __syncwarp();
                    armed[kv] = j + 1;
                    uint8_t* dst = (kv ? sV : sK) + st * L::kTileBytes;
                    const CUtensorMap* map = kv ? &tmap_v : &tmap_k;
                    for (int b = lane; b < boxes; b += 32) {
                        const int t0 = a0 + b * rpb;
                        if (t0 >= x.kv_end) break;
                        const int id = table[t0 / bs];
                        if (id < 0 || id >= p.num_blocks) continue;
                        const int y = (id * p.H_kv + x.g) * bs + (t0 % bs);
#pragma unroll
                        for (int hf = 0; hf < HALVES; ++hf)
                            tc::tma_load_2d(dst + hf * (kN * 128) + b * rpb * 128, map, hf * 64, y,
                                            full, policy);
                    }
                    __syncwarp();
                }
            }
        }
        // no copy may outlive the CTA: the last armed tiles of each ring may
        // still be in flight (an earlier tile's slot was reused only after the
        // MMA warp had waited for it to land)
        for (int kv = 0; kv < 2; ++kv)
            for (long long j = armed[kv] - kRing < 0 ? 0 : armed[kv] - kRing; j < armed[kv]; ++j)
                (void)mbar_wait(&bar[(kv ? kVFull : kKFull) + (int)(j % kRing)],
                                (uint32_t)((j / kRing) & 1));
    } else if (warp == kMmaWarp) {
        // ----------------------------------------------------------------- MMA
        constexpr uint32_t idS = tc05::idesc_f16(std::is_same<T, __nv_bfloat16>::value, false, kM, kN);
        constexpr uint32_t idPV = tc05::idesc_f16(std::is_same<T, __nv_bfloat16>::value, true, kM, D);
        const uint32_t aQ = smem_addr(sQ), aP = smem_addr(sP);
        const uint32_t aK = smem_addr(sK), aV = smem_addr(sV);
        long long sc = 0, pc = 0, ic = 0;   // S issued, PV issued, items started
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
        auto issue_s = [&]() {
            const int sb = (int)(sc & 1);
            const int st = (int)(sc % kRing);
            if (sc >= 2 && !wait_ok(&bar[kSEmpty + sb], (uint32_t)(((sc >> 1) - 1) & 1))) return;
            if (!wait_ok(&bar[kKFull + st], (uint32_t)((sc / kRing) & 1))) return;
            tc05::fence_after();
            if (lane == 0) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (uint32_t)((kk & 3) * 32);
                    const uint64_t a = tc05::sdesc_sw128(aQ + (kk >> 2) * (kM * 128) + off, 16, 1024);
                    const uint64_t b = tc05::sdesc_sw128(aK + st * L::kTileBytes +
                                                             (kk >> 2) * (kN * 128) + off, 16, 1024);
                    tc05::mma_ss(tmem + kColS + sb * kN, a, b, idS, kk > 0 ? 1u : 0u);
                }
                tc05::commit(&bar[kSFull + sb]);
                tc05::commit(&bar[kKEmpty + st]);
            }
            __syncwarp();
            ++sc;
        };
        for (long long it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            Item x;
            if (!load_item(p, it, per_rank, x) || !x.valid) continue;
            if (!wait_ok(&bar[kQFull], (uint32_t)(ic & 1))) break;
            ++ic;
            tc05::fence_after();
            issue_s();
            for (int kt = 0; kt < x.n_kt && ok; ++kt) {
                if (kt + 1 < x.n_kt) {
                    issue_s();
                    if (!ok) break;
                }
                // O += P_kt V_kt
                const int st = (int)(pc % kRing);
                if (!wait_ok(&bar[kPFull], (uint32_t)(pc & 1))) break;
                if (!wait_ok(&bar[kVFull + st], (uint32_t)((pc / kRing) & 1))) break;
                tc05::fence_after();
                const int a0 = kt * kN;
                const int keys = min(kN, x.kv_end - a0);
                const int ksteps = (keys + 15) >> 4;
                uint8_t* vt = sV + st * L::kTileBytes;
                if (keys < ksteps * 16) {
                    // keys past the end inside the last 16-key step carry P = 0;
                    // their V rows may hold anything, so make them 0 (0 * NaN
                    // would poison the sum)
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
                if (lane == 0) {
                    for (int kk = 0; kk < ksteps; ++kk) {
                        const uint64_t a = tc05::sdesc_sw128(
                            aP + (kk >> 2) * (kM * 128) + (uint32_t)((kk & 3) * 32), 16, 1024);
                        const uint64_t b = tc05::sdesc_sw128(
                            aV + st * L::kTileBytes + (uint32_t)(kk * 16 * 128), kN * 128, 1024);
                        tc05::mma_ss(tmem + kColO, a, b, idPV, (kt > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc05::commit(&bar[kVEmpty + st]);
                    tc05::commit(&bar[kPvDone]);
                }
                __syncwarp();
                ++pc;
            }
        }
        // every tensor-core operation issued has completed before the CTA
        // frees tensor memory and exits
        if (lane == 0) tc05::commit(&bar[kDrain]);
        __syncwarp();
        (void)mbar_wait(&bar[kDrain], 0);
    } else {
        // ------------------------------------------------------------- softmax
        const int r = tid;                         // tensor-memory lane = tile row
        const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
        long long sc = 0, pc = 0;
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
        for (long long it = blockIdx.x; it < n_items && ok; it += gridDim.x) {
            Item x;
            if (!load_item(p, it, per_rank, x)) continue;
            const int gr = x.row0 + r;             // this thread's row of (seq, g)
            const bool row_ok = gr < x.row_end;
            const int tok = (row_ok ? gr : x.row_end - 1) / p.G;
            const int head = x.g * p.G + (row_ok ? gr : x.row_end - 1) % p.G;
            T* orow = out + ((size_t)(x.q0 + tok) * p.H_q + head) * D;
            if (!x.valid) {
                if (r == 0) report_error(p.err, PKV_DEVERR_CONTEXT_LEN);
                if (x.n <= p.max_q_len && row_ok)
                    for (int i = 0; i < D; i += 8)
                        *reinterpret_cast<uint4*>(orow + i) = make_uint4(0, 0, 0, 0);
                continue;
            }
            // block ids of the item in range? (the producer skipped bad ones)
            // (each warp checks on its own: no CTA-wide barrier inside the
            // roles, which a warp that gave up could leave unreached)
            bool bad = false;
            const int n_blk = (x.kv_end + p.block_size - 1) / p.block_size;
            const int32_t* table = p.tables + (long long)x.seq * p.max_blocks;
            for (int j = lane; j < n_blk; j += 32) {
                const int id = table[j];
                bad |= id < 0 || id >= p.num_blocks;
            }
            bad = __any_sync(kFull, bad);
            if (bad && r == 0) report_error(p.err, PKV_DEVERR_BLOCK_ID);
            // Q row -> shared memory, 128-byte swizzle
            {
                const T* qrow = qg + ((size_t)(x.q0 + tok) * p.H_q + head) * D;
#pragma unroll
                for (int c = 0; c < D / 8; ++c) {
                    uint4 v = row_ok ? *reinterpret_cast<const uint4*>(qrow + c * 8)
                                     : make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4*>(sQ + (c >> 3) * (kM * 128) + (r >> 3) * 1024 +
                                              (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4)) = v;
                }
            }
            fence_proxy_async_smem();
            tc05::fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&bar[kQFull]);

            const int lim = x.base + tok;          // last visible key of this row
            const int min_lim = x.base + x.row0 / p.G;
            float m_run = -INFINITY, l_run = 0.f;
            for (int kt = 0; kt < x.n_kt; ++kt) {
                const int sb = (int)(sc & 1);
                if (!wait_ok(&bar[kSFull + sb], (uint32_t)((sc >> 1) & 1))) break;
                tc05::fence_after();
                float s[kN];
#pragma unroll
                for (int c = 0; c < kN / 32; ++c) {
                    uint32_t u[32];
                    tc05::tmem_ld32(t_lane + kColS + sb * kN + c * 32, u);
#pragma unroll
                    for (int j = 0; j < 32; ++j) s[c * 32 + j] = __uint_as_float(u[j]);
                }
                tc05::fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bar[kSEmpty + sb]);
                ++sc;
                // scale into the base-2 domain, causal mask, tile maximum
                const int k0 = kt * kN;
                float mt = -INFINITY;
                if (k0 + kN - 1 <= min_lim) {
#pragma unroll
                    for (int j = 0; j < kN; ++j) {
                        s[j] *= p.q_scale;
                        mt = fmaxf(mt, s[j]);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < kN; ++j) {
                        s[j] = (k0 + j <= lim) ? s[j] * p.q_scale : -INFINITY;
                        mt = fmaxf(mt, s[j]);
                    }
                }
                const float m_new = (mt > m_run + kRescaleLog2) ? mt : m_run;
                const float alpha = tc05::ex2(m_run - m_new);   // 0 on the first tile
                // probabilities, row sum, P row (f16/bf16 pairs) in registers
                uint32_t pk[kN / 2];
                float rs = 0.f;
#pragma unroll
                for (int j = 0; j < kN; j += 2) {
                    const float a = tc05::ex2(s[j] - m_new);
                    const float b = tc05::ex2(s[j + 1] - m_new);
                    rs += a + b;
                    pk[j / 2] = tc::MmaType<T>::pack(a, b);
                }
                l_run = l_run * alpha + rs;
                // the previous P.V must be done: P's buffer is reused and O is
                // rescaled below
                if (pc > 0 && !wait_ok(&bar[kPvDone], (uint32_t)((pc - 1) & 1))) break;
                tc05::fence_after();
                if (kt > 0 && __any_sync(kFull, m_new != m_run)) {
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t u[32];
                        tc05::tmem_ld32(t_lane + kColO + c * 32, u);
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            u[j] = __float_as_uint(__uint_as_float(u[j]) * alpha);
                        tc05::tmem_st32(t_lane + kColO + c * 32, u);
                    }
                }
                m_run = m_new;
#pragma unroll
                for (int c = 0; c < kN / 8; ++c) {
                    // keys 8c .. 8c + 7: half c / 8 of the P tile, chunk c % 8
                    *reinterpret_cast<uint4*>(sP + (c >> 3) * (kM * 128) + (r >> 3) * 1024 +
                                              (r & 7) * 128 + (((c & 7) ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                }
                fence_proxy_async_smem();
                tc05::fence_before();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(&bar[kPFull]);
                ++pc;
            }
            if (!ok) break;
            // epilogue: O / l of the item's last P.V
            if (!wait_ok(&bar[kPvDone], (uint32_t)((pc - 1) & 1))) break;
            tc05::fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t u[32];
                tc05::tmem_ld32(t_lane + kColO + c * 32, u);
                if (bad) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) u[j] = 0u;   // the item's keys were not read
                }
                if (row_ok) {
#pragma unroll
                    for (int j = 0; j < 32; j += 8) {
                        uint4 v;
                        v.x = tc::MmaType<T>::pack(__uint_as_float(u[j]) * inv, __uint_as_float(u[j + 1]) * inv);
                        v.y = tc::MmaType<T>::pack(__uint_as_float(u[j + 2]) * inv, __uint_as_float(u[j + 3]) * inv);
                        v.z = tc::MmaType<T>::pack(__uint_as_float(u[j + 4]) * inv, __uint_as_float(u[j + 5]) * inv);
                        v.w = tc::MmaType<T>::pack(__uint_as_float(u[j + 6]) * inv, __uint_as_float(u[j + 7]) * inv);
                        *reinterpret_cast<uint4*>(orow + c * 32 + j) = v;
                    }
                }
            }
            tc05::fence_before();
        }
    }

    // every role is done: free tensor memory
    tc05::fence_before();
    __syncthreads();
    if (warp == 0) {
        tc05::fence_after();
        tc05::tmem_dealloc(tmem, kTmemCols);
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
    const long long max_tiles = ((long long)p.max_q_len * p.G + kM - 1) / kM;
    const long long n_items = max_tiles * p.B * p.H_kv;
    if (n_items <= 0) return cudaSuccess;
    const int sms = pool->sm_count > 0 ? pool->sm_count : 148;
    const int grid = (int)(n_items < sms ? n_items : sms);
    return launch_kernel(kern, dim3(grid), dim3(kThreads), L::kSmem, st, false,
                         *reinterpret_cast<const CUtensorMap*>(pool->tmap_k),
                         *reinterpret_cast<const CUtensorMap*>(pool->tmap_v), p, n_items);
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
