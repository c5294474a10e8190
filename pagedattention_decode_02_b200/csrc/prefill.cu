// Prompt-phase (prefill) attention over the paged cache on tensor cores.
//
// "KV 缓存与分页注意力" §一次写一个词元: the prompt phase computes a whole prompt
// at once, every prompt token's key and value together.  Here sequence i's n_i
// prompt tokens are the last n_i of its c_i cached tokens - their keys and
// values already appended (kv_append), after a prefix that may come from the
// prefix cache (§后来的做法) or from a recomputed history (§放不下的时候) - and
// token t, at position c_i - n_i + t, attends causally to positions
// 0 .. c_i - n_i + t through the block table.
//
// CTA = (64 query rows, KV head g, sequence).  The rows of a (sequence, g)
// are its (token, query head of the group) pairs in token-major order, so a
// CTA's 64 rows share one stream of K/V tiles (G query heads per KV head read
// each tile once).  One producer warp streams 64-token K/V tiles (four
// 16-token stages of 2-D TMA boxes, 128-byte swizzle, plain loads of this
// GPU's own memory) through a double buffer; four consumer warps (16 rows
// each) compute S = Q K^T and O += P V with mma.sync m16n8k16 (fp32
// accumulation) and an online softmax in base 2, masking keys past each row's
// position.  CTAs are launched heaviest tile (latest tokens) first.
#include <cuda.h>

#include <cfloat>

#include "decode_launch.h"
#include "kernels_common.cuh"
#include "pool.h"
#include "tc_common.cuh"

namespace pkv {

namespace {

using tc::kStageTokens;
using tc::swz;

constexpr int kRows = 64;                // query rows per CTA
constexpr int kTileStages = 4;           // 16-token stages per K/V tile
constexpr int kTileKeys = kTileStages * kStageTokens;
constexpr int kBufs = 2;                 // K/V tiles in flight
constexpr int kConsumers = kRows / 16;   // consumer warps
constexpr unsigned kFull = 0xffffffffu;

template <int D>
struct PfCfg {
    static constexpr int kStage = kStageTokens * D * 2;        // K (or V) of one stage
    static constexpr int kTile = kTileStages * 2 * kStage;     // K and V of one tile
};

template <int D>
constexpr int prefill_smem_bytes() {
    return 1024 + kBufs * PfCfg<D>::kTile + 2 * kBufs * 8 + kBufs * 4;
}

template <typename T, int D>
__global__ void __launch_bounds__((kConsumers + 1) * 32, 2)
prefill_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, const PrefillParams p) {
    constexpr int STAGE = PfCfg<D>::kStage;
    constexpr int TILE = PfCfg<D>::kTile;
    constexpr int KSTEPS = D / 16;
    constexpr int DTILES = D / 8;
    constexpr int HALVES = D / 64;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* bufs = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    // buffer b: K stages [4][STAGE] then V stages [4][STAGE]
    uint64_t* full = reinterpret_cast<uint64_t*>(bufs + kBufs * TILE);
    uint64_t* empty = full + kBufs;
    volatile int* buf_bad = reinterpret_cast<volatile int*>(empty + kBufs);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int g = blockIdx.y;
    const int seq = blockIdx.z;
    const int G = p.G;
    const int bs = p.block_size;

    grid_dependency_wait();
    const int q0 = p.q_starts[seq];
    const int n = p.q_starts[seq + 1] - q0;
    const int c = p.lens[seq];
    const int rows = n * G;
    const int n_tiles = (rows + kRows - 1) / kRows;
    if (n <= 0 || (int)blockIdx.x >= n_tiles) return;
    const int tile = n_tiles - 1 - blockIdx.x;   // heaviest first
    const int row0 = tile * kRows;
    const int row_end = min(rows, row0 + kRows);
    const bool valid = c >= 1 && c <= p.max_blocks * bs && n <= c && n <= p.max_q_len;
    if (!valid) {
        if (tid == 0) report_error(p.err, PKV_DEVERR_CONTEXT_LEN);
        T* out = reinterpret_cast<T*>(p.out);
        if (n <= p.max_q_len)
            for (int i = tid; i < (row_end - row0) * D; i += blockDim.x) {
                const int r = row0 + i / D;
                out[((size_t)(q0 + r / G) * p.H_q + (size_t)g * G + r % G) * D + i % D] =
                    Elem<T>::from_f(0.f);
            }
        return;
    }
    const int base = c - n;                                // position of prompt token 0
    const int kv_end = base + (row_end - 1) / G + 1;       // keys any row of the CTA sees
    const int n_kt = (kv_end + kTileKeys - 1) / kTileKeys;

    if (tid == 0) {
        for (int i = 0; i < kBufs; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kConsumers);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumers) {
        // ------------------------------------------------------------ producer
        const uint64_t policy = l2_evict_first_policy();
        const int rpb = bs < kStageTokens ? bs : kStageTokens;
        const int32_t* table = p.tables + (long long)seq * p.max_blocks;
        int wb = -1, wid = -1;
        int kt = 0;
        for (; kt < n_kt; ++kt) {
            const int b = kt % kBufs;
            if (kt >= kBufs) {
                const bool ok = mbar_wait(&empty[b], (uint32_t)(((kt / kBufs) - 1) & 1), p.wait_ns);
                if (!__all_sync(kFull, ok)) {
                    if (lane == 0) report_error(p.err, PKV_DEVERR_TIMEOUT);
                    break;
                }
            }
            // boxes of this tile and whether every block id is in range; the
            // issue pass below walks the same boxes from the same window
            const int wb_tile = wb, wid_tile = wid;
            uint32_t bytes = 0;
            bool bad = false;
            for (int st = 0; st < kTileStages; ++st) {
                const int a = kt * kTileKeys + st * kStageTokens;
                if (a >= kv_end) break;
                const int ns = min(kStageTokens, kv_end - a);
                const int nb = (ns + rpb - 1) / rpb;
                const int lb1 = (a + ns - 1) / bs;
                if (wb < 0 || lb1 >= wb + 32) {
                    wb = a / bs;
                    wid = wb + lane < p.max_blocks ? table[wb + lane] : -1;
                }
                for (int bx = 0; bx < nb; ++bx) {
                    const int id = __shfl_sync(kFull, wid, (a + bx * rpb) / bs - wb);
                    bad |= id < 0 || id >= p.num_blocks;
                }
                bytes += (uint32_t)(2 * HALVES * nb * rpb * 128);
            }
            if (lane == 0) {
                buf_bad[b] = bad;
                if (bad) {
                    report_error(p.err, PKV_DEVERR_BLOCK_ID);
                    tc::mbar_arrive(&full[b]);
                } else {
                    mbar_arrive_expect_tx(&full[b], bytes);
                }
            }
            wb = wb_tile;
            wid = wid_tile;
            if (!bad) {
                uint8_t* kd = bufs + b * TILE;
                uint8_t* vd = kd + kTileStages * STAGE;
                for (int st = 0; st < kTileStages; ++st) {
                    const int a = kt * kTileKeys + st * kStageTokens;
                    if (a >= kv_end) break;
                    const int ns = min(kStageTokens, kv_end - a);
                    const int nb = (ns + rpb - 1) / rpb;
                    const int lb1 = (a + ns - 1) / bs;
                    if (wb < 0 || lb1 >= wb + 32) {
                        wb = a / bs;
                        wid = wb + lane < p.max_blocks ? table[wb + lane] : -1;
                    }
                    for (int bx = 0; bx < nb; ++bx) {
                        const int t0 = a + bx * rpb;
                        const int lb = t0 / bs;
                        const int id = __shfl_sync(kFull, wid, lb - wb);
                        if (lane == 0) {
                            const int y = (id * p.H_kv + g) * bs + (t0 - lb * bs);
#pragma unroll
                            for (int hf = 0; hf < HALVES; ++hf) {
                                const int off = st * STAGE + hf * (kStageTokens * 128) + bx * rpb * 128;
                                tc::tma_load_2d(kd + off, &tmap_k, hf * 64, y, &full[b], policy);
                                tc::tma_load_2d(vd + off, &tmap_v, hf * 64, y, &full[b], policy);
                            }
                        }
                    }
                }
            }
            __syncwarp();
        }
        // no copy may outlive the CTA
        for (int j = max(0, kt - kBufs); j < kt; ++j)
            (void)mbar_wait(&full[j % kBufs], (uint32_t)((j / kBufs) & 1));
        return;
    }

    // --------------------------------------------------------------- consumers
    const int gq = lane >> 2;
    const int tq = lane & 3;
    const int ra = row0 + warp * 16 + gq;   // this lane's two rows
    const int rb = ra + 8;
    const int last_row = row_end - 1;
    // each row's last visible key; rows past the CTA's end take the last
    // row's (their output is not written)
    const int lim_a = base + min(ra, last_row) / G;
    const int lim_b = base + min(rb, last_row) / G;
    const int min_lim = base + row0 / G;

    uint32_t qa[KSTEPS][4];
    {
        const T* qp = reinterpret_cast<const T*>(p.q);
        const T* qra = qp + ((size_t)(q0 + ra / G) * p.H_q + (size_t)g * G + ra % G) * D;
        const T* qrb = qp + ((size_t)(q0 + rb / G) * p.H_q + (size_t)g * G + rb % G) * D;
        const bool va = ra < row_end, vb = rb < row_end;
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
            const int c0 = kk * 16 + 2 * tq;
            qa[kk][0] = va ? *reinterpret_cast<const uint32_t*>(qra + c0) : 0u;
            qa[kk][1] = vb ? *reinterpret_cast<const uint32_t*>(qrb + c0) : 0u;
            qa[kk][2] = va ? *reinterpret_cast<const uint32_t*>(qra + c0 + 8) : 0u;
            qa[kk][3] = vb ? *reinterpret_cast<const uint32_t*>(qrb + c0 + 8) : 0u;
        }
    }
    float o[DTILES][4];
#pragma unroll
    for (int j = 0; j < DTILES; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY};
    float l_run[2] = {0.f, 0.f};
    bool bad = false;
    bool abort = false;
    const int mi = lane >> 3, r8 = lane & 7;

    for (int kt = 0; kt < n_kt; ++kt) {
        const int b = kt % kBufs;
        if (!abort) {
            const bool ok = mbar_wait(&full[b], (uint32_t)((kt / kBufs) & 1), p.wait_ns);
            if (!__all_sync(kFull, ok)) {
                abort = true;
                if (lane == 0) report_error(p.err, PKV_DEVERR_TIMEOUT);
            }
        }
        if (!abort && buf_bad[b]) bad = true;
        if (!abort && !bad) {
            uint8_t* kd = bufs + b * TILE;
            uint8_t* vd = kd + kTileStages * STAGE;
            const int k_first = kt * kTileKeys;
            const int valid_keys = min(kTileKeys, kv_end - k_first);
            if (valid_keys < kTileKeys) {
                // rows past the last key hold stale bytes: zero V there (all
                // consumer warps write the same zeros)
                for (int i = lane; i < (kTileKeys - valid_keys) * (D / 8); i += 32) {
                    const int key = valid_keys + i / (D / 8), cc = i % (D / 8);
                    *reinterpret_cast<uint4*>(vd + (key / kStageTokens) * STAGE +
                                              swz(key % kStageTokens, cc)) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();
                __syncwarp();
            }
            const uint32_t kbase = smem_addr(kd);
            const uint32_t vbase = smem_addr(vd);
            // S = Q K^T over 64 keys: 8 n-tiles of 8
            float s[8][4];
#pragma unroll
            for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KSTEPS; ++kk) {
#pragma unroll
                for (int st = 0; st < kTileStages; ++st) {
                    uint32_t b0, b1, b2, b3;
                    tc::ldsm_x4(kbase + st * STAGE + swz((mi >> 1) * 8 + r8, 2 * kk + (mi & 1)), b0,
                                b1, b2, b3);
                    tc::MmaType<T>::mma(s[2 * st], qa[kk], b0, b1);
                    tc::MmaType<T>::mma(s[2 * st + 1], qa[kk], b2, b3);
                }
            }
            // scale, causal mask, online softmax per row
            const bool need_mask = k_first + kTileKeys - 1 > min_lim;
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float v = s[j][e] * p.q_scale;
                    if (need_mask) {
                        const int key = k_first + 8 * j + 2 * tq + (e & 1);
                        v = key <= ((e >> 1) ? lim_b : lim_a) ? v : -INFINITY;
                    }
                    s[j][e] = v;
                    mx[e >> 1] = fmaxf(mx[e >> 1], v);
                }
            float alpha[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(kFull, mx[r], 1));
                mx[r] = fmaxf(mx[r], __shfl_xor_sync(kFull, mx[r], 2));
                const float m_new = fmaxf(m_run[r], mx[r]);
                alpha[r] = exp2f(m_run[r] - m_new);
                m_run[r] = m_new;
                l_run[r] *= alpha[r];
            }
            uint32_t pa[kTileStages][4];
#pragma unroll
            for (int st = 0; st < kTileStages; ++st) {
                float pr[2][4];
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        pr[h][e] = exp2f(s[2 * st + h][e] - m_run[e >> 1]);
                        l_run[e >> 1] += pr[h][e];
                    }
                pa[st][0] = tc::MmaType<T>::pack(pr[0][0], pr[0][1]);
                pa[st][1] = tc::MmaType<T>::pack(pr[0][2], pr[0][3]);
                pa[st][2] = tc::MmaType<T>::pack(pr[1][0], pr[1][1]);
                pa[st][3] = tc::MmaType<T>::pack(pr[1][2], pr[1][3]);
            }
            if (__any_sync(kFull, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
                for (int j = 0; j < DTILES; ++j) {
                    o[j][0] *= alpha[0];
                    o[j][1] *= alpha[0];
                    o[j][2] *= alpha[1];
                    o[j][3] *= alpha[1];
                }
            }
            // O += P V, one 16-key stage per k-step
#pragma unroll
            for (int st = 0; st < kTileStages; ++st) {
#pragma unroll
                for (int j = 0; j < DTILES; j += 2) {
                    uint32_t b0, b1, b2, b3;
                    tc::ldsm_x4_t(vbase + st * STAGE + swz((mi & 1) * 8 + r8, j + (mi >> 1)), b0, b1,
                                  b2, b3);
                    tc::MmaType<T>::mma(o[j], pa[st], b0, b1);
                    tc::MmaType<T>::mma(o[j + 1], pa[st], b2, b3);
                }
            }
        }
        __syncwarp();
        // a warp that gave up hands no buffer back: its copy may still be in
        // flight, so the producer must not refill it (the producer's own wait
        // for the buffer then gives up too, and it waits for its last copies)
        if (lane == 0 && !abort) tc::mbar_arrive(&empty[b]);
    }

#pragma unroll
    for (int r = 0; r < 2; ++r) {
        l_run[r] += __shfl_xor_sync(kFull, l_run[r], 1);
        l_run[r] += __shfl_xor_sync(kFull, l_run[r], 2);
    }
    const bool zero = bad || abort;
    const float ia = (!zero && l_run[0] > 0.f) ? 1.f / l_run[0] : 0.f;
    const float ib = (!zero && l_run[1] > 0.f) ? 1.f / l_run[1] : 0.f;
    T* out = reinterpret_cast<T*>(p.out);
    T* oa = out + ((size_t)(q0 + ra / G) * p.H_q + (size_t)g * G + ra % G) * D;
    T* ob = out + ((size_t)(q0 + rb / G) * p.H_q + (size_t)g * G + rb % G) * D;
#pragma unroll
    for (int j = 0; j < DTILES; ++j) {
        const int col = 8 * j + 2 * tq;
        if (ra < row_end) {
            oa[col] = Elem<T>::from_f(zero ? 0.f : o[j][0] * ia);
            oa[col + 1] = Elem<T>::from_f(zero ? 0.f : o[j][1] * ia);
        }
        if (rb < row_end) {
            ob[col] = Elem<T>::from_f(zero ? 0.f : o[j][2] * ib);
            ob[col + 1] = Elem<T>::from_f(zero ? 0.f : o[j][3] * ib);
        }
    }
}

template <typename T, int D>
cudaError_t launch_prefill_t(const PrefillParams& p, const pkv_pool* pool, cudaStream_t st) {
    constexpr int smem = prefill_smem_bytes<D>();
    static_assert(smem <= 227 * 1024, "shared memory budget");
    auto kern = prefill_tc_kernel<T, D>;
    static unsigned long long attr_done = 0;
    cudaError_t e = allow_large_smem(kern, &attr_done);
    if (e != cudaSuccess) return e;
    const long long tiles = ((long long)p.max_q_len * p.G + kRows - 1) / kRows;
    if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)tiles, p.H_kv, p.B);
    return launch_kernel(kern, grid, dim3((kConsumers + 1) * 32), smem, st, false,
                         *reinterpret_cast<const CUtensorMap*>(pool->tmap_k),
                         *reinterpret_cast<const CUtensorMap*>(pool->tmap_v), p);
}

}  // namespace

bool prefill_supported(const pkv_pool* pool, int q_dtype) {
    return pool_has_row_maps(pool) && (pool->dtype == PKV_F16 || pool->dtype == PKV_BF16) &&
           q_dtype == pool->dtype && (pool->head_dim == 64 || pool->head_dim == 128);
}

cudaError_t launch_prefill(const PrefillParams& p, const pkv_pool* pool, cudaStream_t st) {
    if (pool->dtype == PKV_F16) {
        if (pool->head_dim == 64) return launch_prefill_t<__half, 64>(p, pool, st);
        if (pool->head_dim == 128) return launch_prefill_t<__half, 128>(p, pool, st);
    } else if (pool->dtype == PKV_BF16) {
        if (pool->head_dim == 64) return launch_prefill_t<__nv_bfloat16, 64>(p, pool, st);
        if (pool->head_dim == 128) return launch_prefill_t<__nv_bfloat16, 128>(p, pool, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace pkv
