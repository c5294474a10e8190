/*
 * pagedkv.h - C ABI of the paged KV cache and its decode-step kernels (sm_100a).
 *
 * What the library does, and where each call comes from
 * ------------------------------------------------------
 * Pages cited (by title and section):
 *   [F55]   "KV 缓存与分页注意力" (world.lapla.si, exhibit F55)
 *   [TOPIC] "KV 缓存" topic page (aiinfact.com), levels 1-3
 *   [IPLEX] "读懂PagedAttention：vLLM的KV缓存与GPU显存管理" (iplexlaw.co.kr)
 *
 * The KV pool is one region of device memory cut into equal physical blocks
 * ([F55] §像内存分页): no external fragmentation.  Each sequence owns a block
 * table: logical block -> physical block id, plus the fill count of the last
 * block ([F55] §块表).  A block is taken only when the last one is full
 * ([F55] §块表), shared blocks carry a reference count and are copied on write
 * ([F55] FAQ 08 共用，写时复制; [IPLEX] §同一提示生成两个回答的假想例子), and a finished
 * sequence's blocks are returned ([F55] §块表).  Each decode round stores the
 * new token's key and value and then attends over the whole history, reading
 * it block by block through the table ([F55] §一次写一个词元, §块表; [TOPIC]
 * level 3, cached generation).
 *
 * Layouts (all row-major, no padding):
 *   pool K, pool V     [num_blocks][n_kv_heads][block_size][head_dim]  (pool dtype)
 *   q, out             [B][n_q_heads][head_dim]                        (q dtype)
 *   new k, new v       [n_tokens][n_kv_heads][head_dim]                (input dtype)
 *   block_tables       [B][max_blocks] int32, unused entries -1
 *   context_lens       [B] int32, tokens per sequence *including* the new one
 *   slot_mapping       [n_tokens] int32, slot = physical_block * block_size + offset
 * Query head h reads KV head floor(h / (n_q_heads / n_kv_heads)).
 *
 * Conventions
 *   - Nothing throws or aborts across this ABI; every call returns a status.
 *   - Host calls (kv_pool_*, bt_*) are all-or-nothing: on any error the state
 *     is exactly as before the call.
 *   - Device calls are asynchronous on the given stream (a cudaStream_t passed
 *     as void*, NULL = legacy default stream).  Argument errors visible on the
 *     host return PKV_ERR_INVALID_ARG before anything is launched; errors only
 *     visible on the device (a context length or block id out of range, a
 *     bounded wait that gave up) set bits in the pool's device error word,
 *     which pkv_device_error() reads and clears.  Kernels never trap.
 *   - Ownership: the caller owns every pointer it passes (q, out, k, v,
 *     tables, lengths, slot mapping, workspace).  The pool owns its host
 *     bookkeeping, its device error word and - when it allocated them - its
 *     K/V buffers.
 */
#ifndef PAGEDKV_H
#define PAGEDKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1,  /* bad argument; nothing done */
    PKV_ERR_NO_BLOCKS = 2,    /* not enough free blocks; nothing done */
    PKV_ERR_UNKNOWN_SEQ = 3,  /* sequence id not in the pool */
    PKV_ERR_SEQ_EXISTS = 4,   /* sequence id already in the pool */
    PKV_ERR_CUDA = 5,         /* a CUDA runtime call failed */
    PKV_ERR_DEVICE = 6,       /* the device error word was set (see pkv_device_error) */
    PKV_ERR_SCRATCH_LIMIT = 7 /* the request needs more than the static scratch of
                                 paged_decode_attention_static; nothing launched */
} pkv_status;

typedef enum {
    PKV_F32 = 0,
    PKV_F16 = 1,
    PKV_BF16 = 2,
    PKV_FP8_E4M3 = 3          /* OCP FP8 E4M3, per-tensor scale ([F55] §后来的做法) */
} pkv_dtype;

/* bits of the device error word */
#define PKV_DEVERR_CONTEXT_LEN 0x1u  /* context_len < 1 or > max_blocks * block_size */
#define PKV_DEVERR_BLOCK_ID    0x2u  /* block id outside [0, num_blocks) */
#define PKV_DEVERR_SLOT        0x4u  /* slot outside [0, num_blocks * block_size) */
#define PKV_DEVERR_TIMEOUT     0x8u  /* a bounded wait on a copy gave up */

/* kv_pool_create flags */
#define PKV_POOL_HOST_ONLY 0x1u      /* bookkeeping only: no device memory, device calls refused */

typedef struct pkv_pool pkv_pool;

typedef struct {
    int32_t num_blocks;
    int32_t block_size;
    int32_t free_blocks;
    int32_t used_blocks;      /* blocks with refcount > 0 */
    int32_t num_seqs;
    int32_t pad_;
    int64_t stored_slots;     /* filled slots over used blocks (a shared block counts once) */
    int64_t logical_tokens;   /* sum of sequence lengths (a shared token counts per sequence) */
    int64_t table_slots;      /* sum over sequences of |table| * block_size */
    int64_t cow_count;        /* copy-on-write events since the last bt_reset */
    int64_t prefix_hit_tokens;/* prompt tokens found in the prefix cache since the last bt_reset */
    int64_t cached_blocks;    /* blocks registered in the prefix cache (in use or free) */
} pkv_stats;

typedef struct {
    int32_t num_blocks, block_size, n_kv_heads, head_dim;
    int32_t dtype;            /* pkv_dtype */
    int32_t host_only;
    float k_scale, v_scale;
    void* k_buf;              /* device pointers (NULL for host-only pools) */
    void* v_buf;
    size_t bytes_per_buffer;  /* num_blocks * n_kv_heads * block_size * head_dim * elem bytes */
    uint32_t* error_word;     /* device pointer */
} pkv_pool_info;

/* ---------------------------------------------------------------------------
 * Pool
 * ------------------------------------------------------------------------- */

/* kv_pool_create - the KV pool of equal physical blocks ([F55] §像内存分页).
 *   num_blocks >= 1, block_size >= 1, n_kv_heads >= 1, head_dim in {32, 64, 128}.
 *   dtype: storage type.  k_scale, v_scale: FP8 dequantisation scales (stored
 *   value = code * scale); must be finite and > 0 for PKV_FP8_E4M3, ignored
 *   otherwise.
 *   k_buf, v_buf: both NULL -> the pool allocates both buffers itself (and
 *   frees them in kv_pool_destroy); both non-NULL -> caller-owned device
 *   buffers of at least *bytes_needed_out bytes each, 16-byte aligned.
 *   flags: PKV_POOL_HOST_ONLY for a bookkeeping-only pool (k_buf/v_buf ignored).
 *   bytes_needed_out (may be NULL): receives the size of one buffer.
 *   out: receives the pool; if NULL, only *bytes_needed_out is computed.
 *   The free queue starts in identity order (see bt_reset).
 *   Errors: INVALID_ARG, CUDA (allocation failed; nothing leaked). */
pkv_status kv_pool_create(int num_blocks, int block_size, int n_kv_heads, int head_dim,
                          pkv_dtype dtype, float k_scale, float v_scale,
                          void* k_buf, void* v_buf, unsigned flags,
                          size_t* bytes_needed_out, pkv_pool** out);

/* kv_pool_destroy - frees the bookkeeping, the error word and self-allocated
 *   buffers.  NULL is accepted.  The caller must make sure no kernel using the
 *   pool is still running. */
void kv_pool_destroy(pkv_pool* pool);

/* kv_pool_get_info - fills *info (device pointers, sizes, scales). */
pkv_status kv_pool_get_info(const pkv_pool* pool, pkv_pool_info* info);

/* kv_pool_check_guards - a debugging check of the pool's own buffers.  A pool
 *   that allocated its K and V buffers keeps one guard block (the block size
 *   rounded up to 256 bytes) of a fixed byte before and after each of them;
 *   no call of the library writes there, so a changed byte means a write out
 *   of the pool's bounds.  Waits for all work on the pool's device
 *   (cudaDeviceSynchronize), copies the four guard regions to the host and
 *   sets *intact to 1 if every byte still holds the guard value, else 0.
 *   Pools on caller-owned buffers and host-only pools have no guards:
 *   *intact = 1.  Errors: INVALID_ARG (NULL argument, another current
 *   device), CUDA (the wait or a copy failed). */
pkv_status kv_pool_check_guards(const pkv_pool* pool, int* intact);

/* ---------------------------------------------------------------------------
 * Block tables (host; [F55] §块表, FAQ 08; [IPLEX] §分离逻辑顺序与实际存储位置,
 * §同一提示生成两个回答的假想例子).  Free-queue policy: FIFO; a block is taken from
 * the front and returned to the back when its refcount reaches zero.
 * ------------------------------------------------------------------------- */

/* bt_reset - drops every sequence and refills the free queue in the given
 *   order (free_order: host array of num_blocks distinct ids; NULL = identity).
 *   Resets cow_count.  Errors: INVALID_ARG (not a permutation). */
pkv_status bt_reset(pkv_pool* pool, const int32_t* free_order);

/* bt_alloc - admits a new sequence with n_tokens >= 0 prompt tokens: takes
 *   ceil(n_tokens / block_size) blocks and writes the n_tokens slots, in token
 *   order, to slot_mapping_out (host, n_tokens entries; may be NULL when
 *   n_tokens == 0).  Errors: INVALID_ARG, SEQ_EXISTS, NO_BLOCKS. */
pkv_status bt_alloc(pkv_pool* pool, int64_t seq_id, int n_tokens, int32_t* slot_mapping_out);

/* bt_append - reserves the slot of one new token of seq_id: the next slot of
 *   the last block; a fresh block if the last is full (or there is none); if
 *   the last block is partially filled and shared (refcount > 1), a fresh
 *   block receives a copy first: *cow_src_out / *cow_dst_out get the pair
 *   (else -1), the old block's count drops by one, and the caller must run
 *   block_copy(src -> dst) before kv_append writes the slot.
 *   Errors: UNKNOWN_SEQ, NO_BLOCKS. */
pkv_status bt_append(pkv_pool* pool, int64_t seq_id, int32_t* slot_out,
                     int32_t* cow_src_out, int32_t* cow_dst_out);

/* bt_append_batch - bt_append for seq_ids[0..n) in that order, all-or-nothing.
 *   slots_out: host [n]; cow_src_out, cow_dst_out: host arrays of capacity n,
 *   *n_cow_out receives the number of copy pairs written (in the order made).
 *   Errors: INVALID_ARG, UNKNOWN_SEQ, NO_BLOCKS (state unchanged). */
pkv_status bt_append_batch(pkv_pool* pool, const int64_t* seq_ids, int n, int32_t* slots_out,
                           int32_t* cow_src_out, int32_t* cow_dst_out, int* n_cow_out);

/* bt_set_prefix_caching - turns automatic prefix caching on (1) or off (0,
 *   which forgets every registration) ([F55] §后来的做法: each full block is
 *   hashed over its tokens and everything before it; a new request with the
 *   same beginning uses the existing blocks; it saves prompt processing only).
 *   Off by default.  Errors: INVALID_ARG. */
pkv_status bt_set_prefix_caching(pkv_pool* pool, int enable);

/* bt_alloc_prefix - bt_alloc with the prompt's token ids (host [n_tokens]).
 *   With prefix caching on, the longest run of leading full blocks whose
 *   tokens - and all tokens before them - match a registered block is taken
 *   over (refcount + 1; a registered free block leaves the free queue), the
 *   rest comes from the free queue, and the new full blocks are registered.
 *   Registration key: FNV-1a 64 over (parent key, 8 bytes little endian, 0 for
 *   the first block) followed by the block's token ids (4 bytes little endian
 *   each); a hit is confirmed against the stored token ids.  A block handed
 *   out as a fresh block loses its registration.  *n_cached_out receives the
 *   number of leading tokens whose keys and values are already in the pool
 *   (a multiple of block_size): the caller appends only tokens
 *   [*n_cached_out, n_tokens).  slot_mapping_out gets all n_tokens slots.
 *   Errors: INVALID_ARG, SEQ_EXISTS, NO_BLOCKS (nothing changed). */
pkv_status bt_alloc_prefix(pkv_pool* pool, int64_t seq_id, const int32_t* token_ids, int n_tokens,
                           int32_t* slot_mapping_out, int32_t* n_cached_out);

/* bt_fork - child_id gets parent_id's table; every block's refcount + 1
 *   ([IPLEX]: two samples of one prompt point at the same input blocks).
 *   Errors: UNKNOWN_SEQ (parent), SEQ_EXISTS (child). */
pkv_status bt_fork(pkv_pool* pool, int64_t parent_id, int64_t child_id);

/* bt_free - a finished sequence releases its blocks in logical order; blocks
 *   whose count reaches zero return to the free queue.  Errors: UNKNOWN_SEQ. */
pkv_status bt_free(pkv_pool* pool, int64_t seq_id);

/* bt_export - block tables and lengths of seq_ids[0..n) for the kernels:
 *   block_tables_out host [n][max_blocks] (entries past a table's end = -1),
 *   context_lens_out host [n], fill_of_last_out host [n] (may be NULL; 0 for a
 *   sequence without blocks).  Errors: INVALID_ARG (a table longer than
 *   max_blocks), UNKNOWN_SEQ. */
pkv_status bt_export(pkv_pool* pool, const int64_t* seq_ids, int n, int max_blocks,
                     int32_t* block_tables_out, int32_t* context_lens_out,
                     int32_t* fill_of_last_out);

/* bt_num_blocks - number of blocks in seq_id's table. */
pkv_status bt_num_blocks(const pkv_pool* pool, int64_t seq_id, int32_t* n_out);

/* bt_refcount - refcount of one physical block. */
pkv_status bt_refcount(const pkv_pool* pool, int32_t block_id, int32_t* refcount_out);

/* bt_free_queue - copies the free queue front-to-back into out (capacity cap);
 *   *n_out receives its length.  INVALID_ARG if cap is too small. */
pkv_status bt_free_queue(const pkv_pool* pool, int32_t* out, int cap, int* n_out);

/* bt_stats - pool counters; utilisation = logical_tokens / table_slots
 *   ([F55] §块表: blocks actually storing tokens). */
pkv_status bt_stats(const pkv_pool* pool, pkv_stats* out);

/* ---------------------------------------------------------------------------
 * Device calls
 * ------------------------------------------------------------------------- */

/* kv_append - stores new keys and values into their slots ([F55] §一次写一个词元;
 *   [IPLEX] §分离逻辑顺序与实际存储位置: later tokens go into the free slots of the
 *   last block).  pool K[slot / bs][h][slot % bs][:] = d_k[t][h][:], same for V.
 *   d_slot_mapping: device int32 [n_tokens]; slot < 0 skips the token.
 *   d_k, d_v: device [n_tokens][n_kv_heads][head_dim] in in_dtype.
 *   in_dtype must equal the pool dtype, except for FP8 pools, which take
 *   F32/F16/BF16 rows and store e4m3(round-to-nearest-even, saturating) of
 *   (x / scale) with the quotient formed in float32.
 *   A slot >= num_blocks * block_size sets PKV_DEVERR_SLOT and is skipped.
 *   n_tokens == 0 is a no-op.  Errors: INVALID_ARG, CUDA. */
pkv_status kv_append(pkv_pool* pool, const int32_t* d_slot_mapping, int n_tokens,
                     const void* d_k, const void* d_v, pkv_dtype in_dtype, void* stream);

/* block_copy - copy-on-write: copies whole physical blocks (all KV heads, K
 *   and V) d_src[i] -> d_dst[i] ([F55] FAQ 08: copy the block, then write the
 *   copy).  d_src, d_dst: device int32 [n_pairs]; destinations must be
 *   distinct and no destination may be a source.  Ids out of range set
 *   PKV_DEVERR_BLOCK_ID and the pair is skipped.  Errors: INVALID_ARG, CUDA. */
pkv_status block_copy(pkv_pool* pool, const int32_t* d_src, const int32_t* d_dst, int n_pairs,
                      void* stream);

/* paged_decode_attention - one decode step's attention ([F55] §块表: the kernel
 *   fetches K and V block by block following the table; blocks need not be
 *   adjacent).  For sequence i and query head h, with g = floor(h / G):
 *     out[i][h] = sum_j softmax_j(scale * <q[i][h], K_i[g][j]>) V_i[g][j],  j < c_i
 *   where K_i[g][j] lives in block d_block_tables[i][j / bs], slot j % bs.
 *   d_q: device [B][n_q_heads][head_dim] in q_dtype; q_dtype = pool dtype for
 *   F32/F16/BF16 pools, F16 or BF16 for FP8 pools.  d_out: same shape/dtype.
 *   d_block_tables: device int32 [B][max_blocks]; d_context_lens: device [B].
 *   n_q_heads must be a multiple of n_kv_heads.
 *   Long contexts are split into partitions whose partial softmax states are
 *   merged by log-sum-exp (unless the unsplit grid already has two waves of
 *   CTAs at three per SM: B * n_q_heads CTAs for one head per KV head,
 *   B * n_kv_heads * ceil(G / 8) for grouped heads); that needs d_workspace (device,
 *   ws_bytes >= paged_decode_workspace_bytes(...), 16-byte aligned, caller
 *   owned, contents scratch).  Without enough workspace the call returns
 *   INVALID_ARG.  A context length outside [1, max_blocks * bs] sets
 *   PKV_DEVERR_CONTEXT_LEN and that sequence's output is zero; a table entry
 *   outside [0, num_blocks) sets PKV_DEVERR_BLOCK_ID and the output of the
 *   affected partition is zero.  B == 0 is a no-op.  Errors: INVALID_ARG, CUDA. */
pkv_status paged_decode_attention(pkv_pool* pool, const void* d_q, pkv_dtype q_dtype,
                                  const int32_t* d_block_tables, int max_blocks,
                                  const int32_t* d_context_lens, int B, int n_q_heads,
                                  float scale, void* d_out, void* d_workspace, size_t ws_bytes,
                                  void* stream);

/* paged_decode_workspace_bytes - workspace paged_decode_attention needs for
 *   this batch shape (max_blocks as passed to it). */
size_t paged_decode_workspace_bytes(const pkv_pool* pool, int B, int n_q_heads, int max_blocks);

/* Kernel selection for paged_decode_attention_ex. */
#define PKV_KERNEL_AUTO 0          /* LEAN for large groups (G > 16) when supported, the workspace
                                      holds its state and partition_tokens is 0; else TENSOR when
                                      supported (not for FP8 pools with G = 1 and block size 1);
                                      else SIMT */
#define PKV_KERNEL_SIMT 1          /* CUDA-core dot products: SIMT_TMA when supported, else SIMT_BULK */
#define PKV_KERNEL_TENSOR 2        /* tensor-core contraction of grouped heads: F16/BF16 pools with
                                      q in the pool dtype, head_dim 64 or 128, power-of-two block
                                      size, 1 < G <= 128; FP8-E4M3 pools with F16 q, head_dim 128,
                                      power-of-two block size, 1 <= G <= 8 (codes converted to f16
                                      in registers) */
#define PKV_KERNEL_SIMT_BULK 3     /* CUDA-core, 1-D bulk copies per block run (any shape) */
#define PKV_KERNEL_SIMT_TMA 4      /* CUDA-core, swizzled 2-D TMA boxes, one query head per CTA:
                                      rows of 128/256/512 bytes, power-of-two block size */
#define PKV_KERNEL_LEAN 5          /* tensor cores, one wave of persistent workers sharing the batch's
                                      16-token stages equally, a split pair merged in the kernel by
                                      the worker that finishes its last piece:
                                      F16/BF16 pools with head_dim 64 or 128, power-of-two block
                                      size, 1 <= G <= 128, B <= 2048; ignores partition_tokens */

/* paged_decode_attention_ex - paged_decode_attention with explicit choices:
 *   partition_tokens: 0 = automatic, > 0 = the longest partition (a multiple
 *   of 16), -1 = never split; kernel: PKV_KERNEL_*.  A context of c tokens is
 *   split into ceil(c / P) partitions; the tensor-core and TMA kernels give
 *   them equal lengths (rounded up to 16 tokens, the last one shorter), the
 *   bulk-copy kernel cuts at multiples of P.  The workspace needed for the
 *   same choices is paged_decode_workspace_bytes_ex(). */
pkv_status paged_decode_attention_ex(pkv_pool* pool, const void* d_q, pkv_dtype q_dtype,
                                     const int32_t* d_block_tables, int max_blocks,
                                     const int32_t* d_context_lens, int B, int n_q_heads,
                                     float scale, void* d_out, void* d_workspace, size_t ws_bytes,
                                     int partition_tokens, int kernel, void* stream);
size_t paged_decode_workspace_bytes_ex(const pkv_pool* pool, int B, int n_q_heads, int max_blocks,
                                       int partition_tokens);

/* ---------------------------------------------------------------------------
 * Decode-step runtime: one call per generation round for a batch of running
 * sequences ([F55] §一次写一个词元: each round every running sequence stores its
 * new token's key and value and attends over its history).
 * ------------------------------------------------------------------------- */
typedef struct pkv_step pkv_step;

/* pkv_step_create - runtime state for decode rounds on a pool: batches of up
 *   to max_batch sequences whose tables hold up to max_blocks blocks, with
 *   device-resident block tables kept for up to max_seqs distinct sequences
 *   (max_seqs >= max_batch; a sequence not seen for the longest time gives
 *   its row up first), pinned host staging and the attention workspace.  All
 *   memory is allocated here, none in pkv_decode_step.  q_dtype: dtype of q,
 *   of the new K/V rows and of the output.  partition_tokens / kernel as in
 *   paged_decode_attention_ex.  Errors: INVALID_ARG, CUDA. */
pkv_status pkv_step_create(pkv_pool* pool, int max_batch, int max_seqs, int max_blocks,
                           int n_q_heads, pkv_dtype q_dtype, int partition_tokens, int kernel,
                           pkv_step** out);

/* pkv_step_destroy - synchronises on the runtime's outstanding copies and
 *   frees its buffers.  NULL is accepted. */
void pkv_step_destroy(pkv_step* step);

/* pkv_decode_step - one decode round for seq_ids[0..B), B <= max_batch:
 *   1. host: bt_append_batch (slots, copy-on-write pairs; all-or-nothing -
 *      on error nothing is launched and the tables are unchanged);
 *   2. host: the batch's block tables and context lengths into pinned staging,
 *      one asynchronous host-to-device copy on `stream`;
 *   3. device: copy-on-write of the shared blocks, append of the B new rows,
 *      then paged decode attention into d_out.
 *   The device keeps each sequence's table in a row of its own between calls;
 *   a round sends only what changed (slots, lengths, rows, copy pairs, new
 *   table entries) as the parameters of one prologue kernel, falling back to
 *   a packed host-to-device copy of the batch's full tables when that does not
 *   fit (first sight of many long sequences).  On the parameter path (up to
 *   128 sequences) the decode kernel also receives each launch slot's length,
 *   row, sequence index and the count of leading table entries the prologue
 *   leaves unchanged, and starts loading those blocks and its queries while
 *   the prologue still runs (programmatic dependent launch); the block that
 *   takes the new token, and any copy-on-write target, are read only after
 *   the prologue has finished.  With split contexts the
 *   decode kernel merges the partitions itself (counters in the runtime's
 *   workspace, zero between calls) when the tensor-core or swizzled-TMA
 *   kernel runs.
 *   d_q: device [B][n_q_heads][head_dim]; d_k_new, d_v_new: device
 *   [B][n_kv_heads][head_dim]; d_out: device [B][n_q_heads][head_dim]; all in
 *   q_dtype.  Returns INVALID_ARG if a table would exceed max_blocks (nothing
 *   changed).  The host returns once the work is queued; staging slots are
 *   reused only after their copies completed.
 *   Errors: INVALID_ARG, UNKNOWN_SEQ, NO_BLOCKS - returned by step 1 or
 *   before it, with nothing changed; CUDA - a copy or launch of steps 2-3
 *   failed after step 1 had been applied: the block manager then holds the
 *   round's appends (lengths, new blocks, copy-on-write) although no key or
 *   value was written, so the caller must bt_free (or bt_reset) the batch's
 *   sequences before using them again.  A failed launch usually means the
 *   CUDA context itself is lost. */
pkv_status pkv_decode_step(pkv_step* step, const int64_t* seq_ids, int B, const void* d_q,
                           const void* d_k_new, const void* d_v_new, float scale, void* d_out,
                           void* stream);

/* pkv_decode_step_host - pkv_decode_step with the round's q, new K/V rows and
 *   output in HOST memory, for callers whose data lives on the host: the call
 *   copies h_q, h_k_new and h_v_new into the runtime's own device buffers
 *   (one cudaMemcpyAsync each on `stream`; made on the first call, sized for
 *   max_batch; when h_k_new and h_v_new directly follow h_q in one packed
 *   host buffer q | k | v, the three travel in a single copy), runs the round
 *   as pkv_decode_step, copies the output into
 *   h_out and waits for the stream: h_out holds the round's attention output
 *   when the call returns.  Pinned host buffers make the copies asynchronous
 *   and fastest; pageable ones work too.  Shapes and dtype as pkv_decode_step:
 *   h_q, h_out [B][n_q_heads][head_dim]; h_k_new, h_v_new
 *   [B][n_kv_heads][head_dim]; all in the step's q_dtype.  Errors as
 *   pkv_decode_step (nothing changed when it rejects the batch), CUDA for a
 *   failed copy or allocation. */
pkv_status pkv_decode_step_host(pkv_step* step, const int64_t* seq_ids, int B, const void* h_q,
                                const void* h_k_new, const void* h_v_new, float scale,
                                void* h_out, void* stream);

/* pkv_step_last_launches - number of kernels the last pkv_decode_step call
 *   launched (copy-on-write copy, append, decode, merge). */
int pkv_step_last_launches(const pkv_step* step);

/* pkv_step_last_kernel - the decode kernel (PKV_KERNEL_LEAN, _TENSOR,
 *   _SIMT_TMA or _SIMT_BULK) the last pkv_decode_step call ran, after the
 *   automatic choice; 0 before the first call or for an empty batch. */
int pkv_step_last_kernel(const pkv_step* step);

/* pkv_step_profile - n > 0: every `every`-th later pkv_decode_step call (the
 *   first one included) records CUDA events on its stream before the round's
 *   prologue (copy/append), before the decode kernel, between it and the
 *   partition merge kernel, and after it, into a ring of n entries; those
 *   rounds run their kernels strictly one after the other.  n == 0 turns this
 *   off.  Errors: INVALID_ARG, CUDA. */
pkv_status pkv_step_profile(pkv_step* step, int n, int every);

/* pkv_step_profile_read - milliseconds of the prologue, of the decode kernel
 *   and of the merge (~0 when the decode kernel merged in-kernel) for the most
 *   recent min(recorded rounds, n) rounds, oldest first (capacity cap each);
 *   *n_out receives the count.  Waits for those events.
 *   Errors: INVALID_ARG (cap too small), CUDA. */
pkv_status pkv_step_profile_read(pkv_step* step, float* prologue_ms, float* decode_ms,
                                 float* merge_ms, int cap, int* n_out);

/* ---------------------------------------------------------------------------
 * Swapping a sequence out to host memory and back ([F55] §放不下的时候: when
 * blocks run out a sequence gives up all of its blocks; they can move to CPU
 * memory and come back when its turn comes).
 * ------------------------------------------------------------------------- */

/* kv_swap_out - queues on `stream` a copy of every block of seq_id, in
 *   logical order, into h_k and h_v (pinned host buffers, e.g. cudaHostAlloc,
 *   layout [n_blocks][n_kv_heads][block_size][head_dim] in the pool dtype,
 *   capacity_bytes each), then releases the sequence like bt_free.  Returns
 *   the block and token counts.  The blocks may be handed out again at once:
 *   device work that writes them must be queued on the same stream (after
 *   the copy).  h_k/h_v must stay valid until the copy has run.
 *   Errors: INVALID_ARG (not pinned, too small), UNKNOWN_SEQ, CUDA. */
pkv_status kv_swap_out(pkv_pool* pool, int64_t seq_id, void* h_k, void* h_v,
                       size_t capacity_bytes, int32_t* n_blocks_out, int64_t* n_tokens_out,
                       void* stream);

/* kv_swap_in - admits seq_id again with n_tokens tokens (fresh blocks, as
 *   bt_alloc) and queues on `stream` the copy of its rows from h_k/h_v
 *   (pinned, the layout kv_swap_out wrote, capacity_bytes each; the call reads
 *   ceil(n_tokens / block_size) blocks' worth and refuses smaller buffers).
 *   Errors: INVALID_ARG, SEQ_EXISTS, NO_BLOCKS (nothing changed), CUDA. */
pkv_status kv_swap_in(pkv_pool* pool, int64_t seq_id, const void* h_k, const void* h_v,
                      size_t capacity_bytes, int64_t n_tokens, void* stream);

/* paged_decode_attention_static - paged_decode_attention for callers that
 *   cannot allocate device memory: processes whose GPU memory is already held
 *   by another allocator (a direct cudaMalloc would fail or fragment it), and
 *   latency-bound loops that allow no cudaMalloc/cudaFree after warm-up
 *   because those calls can synchronise the whole device.  The pages have no
 *   counterpart: this is a deployment variant of the same computation.
 *   Arguments and results as paged_decode_attention_ex with kernel = AUTO,
 *   except that no workspace is passed: the split-context scratch is a
 *   file-scope device array of paged_decode_static_scratch_bytes() (8 MiB).
 *   Placing that array on a device is itself an allocation (CUDA loads the
 *   library's device code lazily), so kv_pool_create does it for the pool's
 *   device, while allocating is still allowed: from the first pool created
 *   on a device, that device holds the array until the process exits, and
 *   this call allocates nothing there.  Create the pool before another
 *   allocator takes the GPU.  On a device with no pool created yet, the
 *   first call looks the array up itself (cudaGetSymbolAddress, with that
 *   device current), which places it - make such a call before any stream
 *   capture; if that fails the call returns PKV_ERR_CUDA.
 *   partition_tokens: 0 = automatic - the library's choice as
 *   paged_decode_attention makes it (without the stage-balanced kernel when
 *   only its share exceeds the scratch), else partitions lengthened from the
 *   automatic length (less scratch) until the scratch fits, down to an
 *   unsplit pass that needs none; > 0 (a multiple of 16) or -1 as in
 *   paged_decode_attention_ex, and a request whose scratch exceeds the limit
 *   returns PKV_ERR_SCRATCH_LIMIT without launching anything.
 *   All calls share the one array and it
 *   keeps the last call's contents; nothing in it needs to start at zero
 *   (every partition's state is written before the merge reads it), but calls
 *   whose kernels overlap on the GPU - on different streams, or from several
 *   host threads - race on it: order them on one stream.
 *   Errors: INVALID_ARG, SCRATCH_LIMIT, CUDA. */
pkv_status paged_decode_attention_static(pkv_pool* pool, const void* d_q, pkv_dtype q_dtype,
                                         const int32_t* d_block_tables, int max_blocks,
                                         const int32_t* d_context_lens, int B, int n_q_heads,
                                         float scale, void* d_out, int partition_tokens,
                                         void* stream);

/* paged_prefill_attention - the prompt phase's attention over the paged cache
 *   ([F55] §一次写一个词元: the whole prompt is computed at once).  Sequence i's
 *   prompt tokens are rows d_q_starts[i] .. d_q_starts[i+1]-1 of d_q and
 *   d_out; with n_i = d_q_starts[i+1] - d_q_starts[i] they are the last n_i of
 *   its d_context_lens[i] = c_i cached tokens, whose keys and values are
 *   already stored (bt_alloc / bt_alloc_prefix slots, kv_append).  Tokens
 *   before them - a cached prefix ([F55] §后来的做法) or a recomputed history -
 *   are attended as well.  For row t of sequence i and query head h, with
 *   g = floor(h / G) and position P = c_i - n_i + t:
 *     out[t][h] = sum_{j <= P} softmax_j(scale * <q[t][h], K_i[g][j]>) V_i[g][j].
 *   d_q, d_out: device [d_q_starts[B]][n_q_heads][head_dim] in the pool dtype
 *   (F16 or BF16 pools with head_dim 64 or 128 and a power-of-two block size;
 *   other pools return INVALID_ARG).  d_q_starts: device int32 [B + 1],
 *   non-decreasing from 0.  d_block_tables: device int32 [B][max_blocks];
 *   d_context_lens: device int32 [B].  max_q_len >= every n_i (it sizes the
 *   grid).  n_i == 0 writes nothing.  A length outside [1, max_blocks * bs],
 *   n_i > c_i or n_i > max_q_len sets PKV_DEVERR_CONTEXT_LEN (that sequence's
 *   rows are zero where the grid covers them); a block id outside
 *   [0, num_blocks) sets PKV_DEVERR_BLOCK_ID and zeroes the affected work
 *   item's rows (256 rows with the tcgen05 kernel, 64 with mma.sync).  No
 *   workspace: the tcgen05 kernel's work counters live in the pool (one pair
 *   per launch in flight, taken in turn from 64), so at most 64 prompt
 *   launches on one pool may run at the same time.  Runs the tcgen05 kernel
 *   (see paged_prefill_attention_ex).
 *   Errors: INVALID_ARG, CUDA. */
pkv_status paged_prefill_attention(pkv_pool* pool, const void* d_q, pkv_dtype q_dtype,
                                   const int32_t* d_q_starts, int max_q_len,
                                   const int32_t* d_block_tables, int max_blocks,
                                   const int32_t* d_context_lens, int B, int n_q_heads,
                                   float scale, void* d_out, void* stream);

/* Kernel selection for paged_prefill_attention_ex. */
#define PKV_PREFILL_AUTO 0         /* PKV_PREFILL_TCGEN05 */
#define PKV_PREFILL_TCGEN05 1      /* fifth-generation tensor cores: 256 query rows (two 128-row
                                      tiles) per work item, S = Q K^T and O += P V by tcgen05.mma
                                      into tensor memory, one persistent CTA per SM claiming items
                                      from a global counter (each sequence's heaviest first) */
#define PKV_PREFILL_MMA_SYNC 2     /* warp-level mma.sync m16n8k16, register accumulators, one CTA
                                      per 64 query rows */

/* paged_prefill_attention_ex - paged_prefill_attention with an explicit kernel
 *   (PKV_PREFILL_*); same arguments, results and errors.  Both kernels compute
 *   the same attention. */
pkv_status paged_prefill_attention_ex(pkv_pool* pool, const void* d_q, pkv_dtype q_dtype,
                                      const int32_t* d_q_starts, int max_q_len,
                                      const int32_t* d_block_tables, int max_blocks,
                                      const int32_t* d_context_lens, int B, int n_q_heads,
                                      float scale, void* d_out, int kernel, void* stream);

/* paged_decode_static_scratch_bytes - size of the static scratch array. */
size_t paged_decode_static_scratch_bytes(void);

/* ---------------------------------------------------------------------------
 * The exhibit's allocation bench on the host ([F55] §实验台): requests arrive,
 * write their prompt at once and one token per round, and leave; those that
 * do not fit wait (first come, first served).  Paged memory (block_size > 0,
 * the block manager's rules) against the contiguous reservations of
 * [F55] §先占好最长的位置 / §三种浪费, each one run of slots taken up front at
 * the first place it fits:
 *   PKV_SIM_MAX    (0)  max_len slots per request;
 *   PKV_SIM_POW2   (-1) the next power of two >= the request's final length,
 *                       at most max_len (over-reserves by less than 2x);
 *   PKV_SIM_ORACLE (-2) exactly the final length (needs the output length in
 *                       advance, which a real server does not know).
 * ------------------------------------------------------------------------- */
#define PKV_SIM_MAX 0
#define PKV_SIM_POW2 (-1)
#define PKV_SIM_ORACLE (-2)

typedef struct {
    int32_t arrival;   /* round the request arrives (non-decreasing over the array) */
    int32_t prompt;    /* prompt tokens, >= 1 */
    int32_t output;    /* tokens to generate, >= 1; prompt + output <= max_len */
} pkv_sim_request;

typedef struct {
    int32_t rounds;             /* rounds until every request has left */
    int32_t peak_running;       /* most requests holding memory in one round */
    int32_t preemptions;        /* paged: requests that gave up their blocks */
    int32_t admitted;           /* admissions (a preempted request is admitted again) */
    int64_t stored_token_rounds;   /* sum over rounds of tokens stored */
    int64_t reserved_slot_rounds;  /* sum over rounds of slots held */
    int64_t future_slot_rounds;    /* ... of held slots its request writes later
                                      (the "reservation" waste) */
    int64_t internal_frag_slot_rounds; /* ... of held slots its request never
                                          writes (internal fragmentation) */
    double mean_utilisation;    /* mean over rounds (with slots held) of stored / held */
} pkv_sim_result;

/* pkv_simulate - runs the bench.  Each round: (1) admission in arrival order
 *   while the head fits; (2) every request admitted earlier writes one token -
 *   paged growth that finds no block preempts the most recently admitted
 *   running request ([F55] §放不下的时候), which rejoins the head of the queue
 *   and comes back with its written tokens as its new prompt (recomputation);
 *   (3) finished requests leave.  Readouts are taken after (2).
 *   block_size: > 0 paged, or one of PKV_SIM_MAX / _POW2 / _ORACLE.
 *   running_per_round (may be NULL) receives the number of requests holding
 *   memory in each round (capacity max_rounds).
 *   Errors: INVALID_ARG (bad request, num_slots not a multiple of block_size,
 *   unknown mode, or not finished within max_rounds). */
pkv_status pkv_simulate(const pkv_sim_request* requests, int n, int num_slots, int block_size,
                        int max_len, int max_rounds, pkv_sim_result* out,
                        int32_t* running_per_round);

/* pkv_set_wait_budget - how long a kernel launched on this pool waits for
 *   one copy (or one tensor-core result) in its main loop before it gives up:
 *   it then sets PKV_DEVERR_TIMEOUT, stops issuing work, waits with the
 *   default budget for its copies and tensor-core operations still in flight,
 *   frees what it holds and returns (the affected outputs are zero or stale).
 *   budget_ns: 1 .. 2e9 ns; 0 restores the default of 2 s, long enough that
 *   only a wait that would otherwise never end gives up.  A short budget
 *   makes waits give up while their copies are still on the way: it exists
 *   to exercise that path.  The library has no counterpart in the pages: it
 *   is this implementation's failure handling.  Errors: INVALID_ARG. */
pkv_status pkv_set_wait_budget(pkv_pool* pool, uint64_t budget_ns);

/* pkv_wait_probe - queues one small kernel on `stream` that waits, with the
 *   pool's wait budget, on a barrier that nothing ever completes, and sets
 *   PKV_DEVERR_TIMEOUT when that wait gives up (read it with
 *   pkv_device_error): a check that the bounded wait and its error report
 *   work on this device.  Takes about the budget to run.  Errors:
 *   INVALID_ARG, CUDA. */
pkv_status pkv_wait_probe(pkv_pool* pool, void* stream);

/* pkv_device_error - synchronises the stream, returns the device error word's
 *   bits in *bits_out (may be NULL) and clears it.  Returns PKV_ERR_DEVICE if
 *   any bit was set, PKV_OK otherwise. */
pkv_status pkv_device_error(pkv_pool* pool, void* stream, uint32_t* bits_out);

/* pkv_status_str - a static, human-readable name of a status. */
const char* pkv_status_str(pkv_status status);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H */
