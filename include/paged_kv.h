/*
 * paged_kv.h — C ABI of the B200 (sm_100a) paged KV-cache library.
 *
 * The operation follows four web pages on LLM inference (cited by title and
 * section):
 *   [T1] "LLM推理优化实战：从KV Cache到Speculative Decoding，把延迟打下来"
 *   [T2] "大模型推理加速：从 KV Cache 到投机采样的工程实践"
 *   [T3] "LLM 推理优化：KV Cache、PagedAttention 与量化"
 *   [T4] "大模型推理加速与显存黑科技 (Inference Acceleration & KV Cache)"
 *
 * Data layout (the pages fix none; all device arrays are row-major, dense):
 *   k_pool, v_pool  fp16 [num_blocks][Hkv][block_size][head_dim]
 *                   (one (block, kv-head) tile is block_size*head_dim*2
 *                   contiguous bytes; base 16-byte aligned, head_dim*2 a
 *                   multiple of 16)
 *   block_tables    int32 [B][max_blocks_per_seq]; entry b of row s is the
 *                   physical block holding tokens [b*bs, b*bs+bs) of sequence s
 *   context_lens    int32 [B]; tokens of sequence s already in the cache
 *                   (including any token appended this step)
 *   q, out          fp16 [B][q_len][Hq][head_dim]  (q_len = 1 for decode)
 *   k_new, v_new    fp16 [T][Hkv][head_dim]
 *   slot_mapping    int64 [T]; slot = physical_block*block_size + offset,
 *                   negative = padding (skipped)
 * Query head h reads KV head h / (Hq / Hkv) (contiguous GQA groups).
 *
 * Ownership: the caller allocates and owns every device buffer (pools, q,
 * out, tables, lengths, workspace) and every host array it passes.  The
 * library owns only the host bookkeeping behind an opaque kv_pool*.  Device
 * calls are asynchronous on the caller's stream (a cudaStream_t passed as
 * void*; NULL = legacy default stream); they never allocate device memory.
 *
 * Errors: every call returns a status.  On KV_ERR_INVALID nothing was
 * launched or changed; KV_ERR_CUDA means a CUDA call failed (text in
 * kv_last_error_string()).  Kernels never trap: an out-of-range block id or
 * slot met on the device is skipped and recorded in a per-device error word
 * read by kv_device_error().
 */
#ifndef PAGED_KV_H
#define PAGED_KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KV_OK 0
#define KV_ERR_INVALID 1     /* bad argument, shape, id or state */
#define KV_ERR_OOM 2         /* pool exhausted: the pages' preemption trigger */
#define KV_ERR_DOUBLE_FREE 3 /* a free would take a refcount below zero */
#define KV_ERR_CUDA 4        /* a CUDA runtime call failed */
#define KV_ERR_TIMEOUT 5     /* unused by the host; device-word bit, see below */

/* Bits of the device error word. */
#define KV_DEV_BAD_BLOCK 1   /* a block-table entry outside [0, num_blocks) */
#define KV_DEV_BAD_SLOT 2    /* an append slot beyond the pool */
#define KV_DEV_TIMEOUT 4     /* a pipeline wait ran past its limit */
#define KV_DEV_BAD_SCALE 8   /* a K scale that is not positive and finite */

/* Text of the last error raised on the calling thread ("" if none). */
const char* kv_last_error_string(void);

/* Library version, for the binding's load check. */
int kv_version(void);

/* ---------------------------------------------------------------------------
 * Pool configuration and sizing.
 * [T2] §"KV Cache的内存挑战" and [T4] §2.1: KV bytes =
 * 2 x layers x heads x head_dim x seq_len x batch x dtype_size.  For a pool,
 * seq_len x batch is its capacity num_blocks x block_size tokens and heads are
 * the KV heads (under MQA/GQA only KV heads are cached, [T2] §"主流优化策略").
 */
typedef struct kv_pool_config {
    int32_t num_blocks;   /* physical blocks in the pool, > 0 */
    int32_t block_size;   /* tokens per block: 16 (default) or 8 ([T3] §2.2) */
    int32_t num_kv_heads; /* Hkv */
    int32_t head_dim;     /* D: 64 or 128 on the decode path */
    int32_t num_layers;   /* layers sharing one block table (sizing only) */
    int32_t dtype_bytes;  /* 2 (fp16) */
} kv_pool_config;

/* per_layer_bytes = K+V bytes of one layer's pools; total_bytes = per layer x
 * num_layers.  Either output may be NULL. */
int kv_pool_bytes(const kv_pool_config* cfg, uint64_t* per_layer_bytes, uint64_t* total_bytes);

/* ---------------------------------------------------------------------------
 * Host block manager ([T3] §2.3 (1)-(3)): fixed-capacity pool, on-demand
 * allocation, immediate reuse of freed blocks, per-block reference counts,
 * block-level copy-on-write, prefix sharing by pointing several tables at the
 * same blocks.  Policy (fixed so results are bit-exact and testable):
 *   - the free list is a LIFO stack; it first pops ids in ascending order, or
 *     in the order of `order` (a permutation of 0..num_blocks-1) if given;
 *     freed blocks are pushed on top and reused first;
 *   - block_alloc is all-or-nothing (KV_ERR_OOM and no change on shortage);
 *   - block_free drops one reference per listed id, pushing ids whose count
 *     reaches zero in list order; KV_ERR_DOUBLE_FREE (no change) if any count
 *     would go below zero;
 *   - block_fork adds one reference per listed (live) id.
 * A kv_pool is not thread-safe; use one per thread or lock around it.
 */
typedef struct kv_pool kv_pool;

int kv_pool_create(const kv_pool_config* cfg, const int32_t* order /* nullable */,
                   kv_pool** out);
int kv_pool_destroy(kv_pool* pool);
int kv_pool_num_free(const kv_pool* pool, int32_t* n_out);
int block_alloc(kv_pool* pool, int32_t n, int32_t* ids_out /* [n] */);
int block_free(kv_pool* pool, const int32_t* ids, int32_t n);
int block_fork(kv_pool* pool, const int32_t* ids, int32_t n);
int block_refcount(const kv_pool* pool, int32_t id, int32_t* rc_out);

/* Reserve the cache slot of token number ctx_len (0-based) of one sequence
 * whose table holds *n_blocks == ceil(ctx_len / block_size) entries
 * ([T3] §2.3 (1) on-demand allocation, (2) copy-on-write):
 *   - ctx_len % block_size == 0: a new block is allocated and appended;
 *   - the last block is shared (refcount > 1): a new block replaces it in the
 *     table, one reference to the old block is dropped and (*cow_src_out,
 *     *cow_dst_out) = (old, new): the caller must copy that block on the
 *     device (paged_kv_copy_blocks) before appending;
 *   - otherwise the token goes into the last block.
 * cow_* are -1 when no copy is needed.  table_capacity bounds the table. */
int kv_seq_reserve_slot(kv_pool* pool, int32_t* table, int32_t table_capacity,
                        int32_t* n_blocks, int32_t ctx_len, int64_t* slot_out,
                        int32_t* cow_src_out, int32_t* cow_dst_out);

/* The same for B sequences in order (table row s = tables + s*table_capacity).
 * Copy pairs are written as (src, dst) into cow_pairs_out[2*k], [2*k+1] and
 * counted in *n_cow_out.  On an error at sequence i the earlier sequences keep
 * their reservations, *n_done_out = i and the error is returned. */
int kv_batch_reserve_slots(kv_pool* pool, int32_t B, int32_t* tables, int32_t table_capacity,
                           int32_t* n_blocks /* [B] */, const int32_t* ctx_lens /* [B] */,
                           int64_t* slots_out /* [B] */, int32_t* cow_pairs_out /* [2B] */,
                           int32_t* n_cow_out, int32_t* n_done_out);

/* Beam-search step ([T3] §2.3 (2): a fork copies only the block table; blocks
 * stay shared until a beam writes, then copy-on-write).  tables [n_beams]
 * [table_capacity] with n_blocks[b] live entries each; new beam i continues
 * old beam parents[i]: new_tables[i] (same capacity, -1 padded; must not
 * overlap tables) is a copy of its table and each of those blocks gets one
 * more reference; then every old beam's references are dropped, beam by beam
 * in order (a block reaching zero goes on the free list).  Nothing is copied
 * on the device: the next kv_batch_reserve_slots emits the copy-on-write pairs
 * for the beams whose shared last block is partial.  KV_ERR_INVALID (nothing
 * changes) on a parent out of range or a table entry that is not live. */
int kv_beam_reorder(kv_pool* pool, const int32_t* tables, const int32_t* n_blocks, int32_t n_beams,
                    int32_t table_capacity, const int32_t* parents, int32_t n_new,
                    int32_t* new_tables, int32_t* new_n_blocks);

/* Prefix cache ([T3] §2.3 (3): requests sharing a prompt prefix are found by
 * hashing block contents and point their tables at the same physical blocks;
 * §2.3 (1): blocks nothing references are kept in LRU order).  A cached block
 * is keyed by (parent, tokens): the cached block holding the previous
 * block_size tokens (-1 for a first block) and its own block_size token ids,
 * compared exactly; a match of block i therefore implies blocks 0..i-1.  Only
 * full blocks are cached.  The cache holds one reference on each cached
 * block (callers must not free that reference); host-only, not thread-safe.
 *
 * kv_prefix_match: walks the full blocks of tokens[0..n_tokens) from the
 * start and stops at the first miss or after table_capacity blocks; each hit
 * gets one more reference (for the new request) and is written to
 * table_out[i]; *n_matched_out = hits.  The request then holds
 * n_matched * block_size tokens of K/V and allocates the rest as usual. */
int kv_prefix_match(kv_pool* pool, const int32_t* tokens, int32_t n_tokens, int32_t* table_out,
                    int32_t table_capacity, int32_t* n_matched_out);
/* kv_prefix_register: caches the full blocks of a request whose K/V are in
 * the pool (table[i] holds tokens[i*bs .. i*bs+bs)), in order.  A block
 * already cached under the same key is only marked used; the walk stops at a
 * key cached in another block or at a block cached under another key.
 * *n_cached_out (nullable) = leading blocks of table now cached under this
 * prefix.  KV_ERR_INVALID if a table entry is not a live block (nothing
 * changes). */
int kv_prefix_register(kv_pool* pool, const int32_t* tokens, int32_t n_tokens, const int32_t* table,
                       int32_t n_blocks, int32_t* n_cached_out);
/* kv_prefix_evict: frees up to n cached blocks that only the cache still
 * references and that have no cached child, least recently used first
 * (matched or registered counts as a use); their ids go to ids_out[k]
 * (nullable), in eviction order, and to the top of the free list. */
int kv_prefix_evict(kv_pool* pool, int32_t n, int32_t* ids_out, int32_t* n_evicted_out);
int kv_prefix_num_cached(const kv_pool* pool, int32_t* n_out);

/* ---------------------------------------------------------------------------
 * Device calls.
 */

/* Cache append: for each t with slot_mapping[t] >= 0,
 *   k_pool[slot/bs][h][slot%bs][:] = k_new[t][h][:]  (and V), every h.
 * Bit-exact copy.  Slots >= num_blocks*bs are skipped and flag
 * KV_DEV_BAD_SLOT.  Distinct tokens must target distinct slots. */
int paged_kv_append(const void* k_new, const void* v_new, const int64_t* slot_mapping,
                    void* k_pool, void* v_pool, int32_t T, int32_t Hkv, int32_t head_dim,
                    int32_t block_size, int32_t num_blocks, void* stream);

/* Copy-on-write block copy ([T3] §2.3 (2)): for each i, physical block
 * pairs[2i+1] of both pools becomes a copy of block pairs[2i] (all heads and
 * slots).  pairs is a DEVICE int32 array [n][2]; destinations must be
 * distinct and no destination may also be a source.  Out-of-range ids are
 * skipped and flag KV_DEV_BAD_BLOCK. */
int paged_kv_copy_blocks(void* k_pool, void* v_pool, const int32_t* pairs, int32_t n,
                         int32_t Hkv, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                         void* stream);

/* Quantised K pool ([T2] §"KV Cache量化": INT8 KV caches, keys quantised per
 * channel as in KVQuant; [T3] §4.2: keys per channel at low bit width, values
 * kept in FP16).  The K pool holds int8 codes [num_blocks][Hkv][bs][D] (half
 * the bytes of fp16), the V pool stays fp16; one fp32 scale per (KV head,
 * channel), k_scales [Hkv][D], fixed by the caller (e.g. from calibration
 * tokens with paged_kv_k_scales).  Key t of head h is code * k_scales[h][d].
 *
 * paged_kv_k_scales: k_scales[h][d] = max_t |k[t][h][d]| / 127 over the
 * DEVICE fp16 tokens k [T][Hkv][D] (1 for an all-zero channel); fp32,
 * correctly rounded division. */
int paged_kv_k_scales(const void* k, int64_t T, int32_t Hkv, int32_t head_dim, float* k_scales,
                      void* stream);
/* paged_kv_append_q8k: paged_kv_append with K written as codes
 *   code = clamp(rint(k / k_scales[h][d]), -128, 127)
 * (fp32, correctly rounded division, round half to even: bit-exact and
 * reproducible on the host) and V copied; a NaN key stores code 0.  A scale
 * that is not positive and finite writes code 0 and flags KV_DEV_BAD_SCALE. */
int paged_kv_append_q8k(const void* k_new, const void* v_new, const int64_t* slot_mapping,
                        const float* k_scales, void* kq_pool, void* v_pool, int32_t T, int32_t Hkv,
                        int32_t head_dim, int32_t block_size, int32_t num_blocks, void* stream);
/* paged_kv_copy_blocks_q8k: paged_kv_copy_blocks for an int8 K pool (K blocks
 * of Hkv*bs*D bytes) and its fp16 V pool; head_dim a multiple of 16. */
int paged_kv_copy_blocks_q8k(void* kq_pool, void* v_pool, const int32_t* pairs, int32_t n,
                             int32_t Hkv, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                             void* stream);
/* paged_attention_q8k: paged_verify_attention (q_len = 1: decode) over an int8
 * K pool: scores use key t = code * k_scales[kvh][:].  The scales are folded
 * into q once per (sequence, kv head) segment (q_d * k_scales[d], rounded to
 * fp16); codes are exact fp16 integers, so the products stay exact in fp32.
 * Requires head_dim 128; k_scales device, 16-byte aligned; workspace as for
 * paged_attention_workspace_size.  Otherwise as paged_verify_attention. */
int paged_attention_q8k(const void* q, const void* kq_pool, const float* k_scales,
                        const void* v_pool, const int32_t* block_tables, int32_t max_blocks_per_seq,
                        const int32_t* context_lens, int32_t q_len, float scale, void* out,
                        int32_t B, int32_t Hq, int32_t Hkv, int32_t head_dim, int32_t block_size,
                        int32_t num_blocks, void* workspace, size_t workspace_bytes, void* stream);

/* Block swap between the pools and host memory ([T3] §2.3 (1): when the pool
 * is full, a preempted request's blocks are moved to CPU memory and brought
 * back when it resumes).  staging (device) and host hold
 * [2 (K, V)][n][Hkv][block_size][head_dim] fp16: 2*n*Hkv*bs*D*2 bytes,
 * staging 16-byte aligned; host should be pinned (cudaHostAlloc) for the
 * copy to be asynchronous; both are owned by the caller.  block_ids is a
 * DEVICE int32 array [n], n <= 65535.
 *   swap_out: a gather kernel copies K and V of block_ids[i] to staging row
 *     i, then one cudaMemcpyAsync copies staging to host (host may be NULL:
 *     the blocks then stay in staging).
 *   swap_in: one cudaMemcpyAsync copies host to staging (skipped if host is
 *     NULL), then a scatter kernel writes row i to block_ids[i].
 * Both are stream-ordered and bit-exact; the host buffer must stay valid
 * until the stream reaches the copy.  Out-of-range ids are skipped and flag
 * KV_DEV_BAD_BLOCK.  The host block manager is not touched: free the
 * swapped-out ids, and allocate fresh ids for the swap-in, with block_free /
 * block_alloc. */
int paged_kv_swap_out(const void* k_pool, const void* v_pool, const int32_t* block_ids, int32_t n,
                      void* staging, void* host, int32_t Hkv, int32_t head_dim, int32_t block_size,
                      int32_t num_blocks, void* stream);
int paged_kv_swap_in(void* k_pool, void* v_pool, const int32_t* block_ids, int32_t n, void* staging,
                     const void* host, int32_t Hkv, int32_t head_dim, int32_t block_size,
                     int32_t num_blocks, void* stream);

/* Bytes of device workspace paged_decode_attention / paged_verify_attention
 * (and the int8-K entries) need for these head counts on the current device
 * (partial results of context splits; a shape the kernel may serve as pairs
 * of KV heads, two 8-row tiles, is sized for that form whatever the block
 * size or pool type).  grid_ctas: 0 for the default launch, else the value
 * given in paged_attention_opts.grid_ctas.  The workspace holds no state
 * between calls and needs no initialisation. */
int paged_attention_workspace_size(int32_t Hq, int32_t Hkv, int32_t q_len, int32_t head_dim,
                                   int32_t grid_ctas, size_t* bytes_out);

/* Paged decode attention ([T4] §2, Attention(Q,K,V) = softmax(QK^T/sqrt(d_k))V;
 * paging per [T3] §2.2 and [T4] §3.2; tiling with an online softmax per
 * [T4] §4.2): for every sequence s and query head h,
 *   out[s][0][h] = softmax(scale * q[s][0][h] . K_t) V_t over t < context_lens[s],
 * K_t / V_t gathered from the pools through block_tables[s][t / bs], row t % bs.
 * fp16 in, fp32 accumulation, fp16 (round-to-nearest-even) out; a sequence of
 * length 0 gives zeros.  Long contexts are split across CTAs and merged by
 * log-sum-exp on the device.  Requirements: head_dim in {64, 128},
 * block_size in {8, 16}, Hq % Hkv == 0, (Hq/Hkv)*q_len <= 32; workspace of at
 * least paged_attention_workspace_size() bytes, 16-byte aligned. */
int paged_decode_attention(const void* q, const void* k_pool, const void* v_pool,
                           const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* context_lens, float scale, void* out, int32_t B,
                           int32_t Hq, int32_t Hkv, int32_t head_dim, int32_t block_size,
                           int32_t num_blocks, void* workspace, size_t workspace_bytes,
                           void* stream);

/* Causal verify window for speculative decoding ([T1] §"Speculative
 * Decoding：用草稿模型加速": the target scores prompt + drafts in one pass;
 * [T3] §6.2): q holds q_len rows per sequence, context_lens counts the drafts,
 * and row j attends to tokens 0 .. context_lens[s] - q_len + j.  q_len = 1 is
 * paged_decode_attention. */
int paged_verify_attention(const void* q, const void* k_pool, const void* v_pool,
                           const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* context_lens, int32_t q_len, float scale, void* out,
                           int32_t B, int32_t Hq, int32_t Hkv, int32_t head_dim,
                           int32_t block_size, int32_t num_blocks, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Paged (chunked) prefill ([T4] §1: the prompt is processed in parallel;
 * same formula, paging and GQA grouping as above): q holds a chunk of q_len
 * new tokens per sequence whose K/V are already in the cache; context_lens
 * counts them; row j of sequence s attends causally to tokens
 * 0 .. context_lens[s] - q_len + j.  Tensor cores (tcgen05, fp32 accumulators
 * in tensor memory); requires head_dim 128, block_size 8 or 16, Hq/Hkv a
 * divisor of 128.  Needs no workspace.  A row that sees no token gives zeros. */
int paged_prefill_attention(const void* q, const void* k_pool, const void* v_pool,
                            const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* context_lens, int32_t q_len, float scale, void* out,
                            int32_t B, int32_t Hq, int32_t Hkv, int32_t head_dim,
                            int32_t block_size, int32_t num_blocks, void* stream);

/* Launch knobs for tuning and tests; zero fields mean "default".
 *   grid_ctas        persistent CTAs (default: SMs x CTAs per SM);
 *   min_split_blocks smallest run of work units one CTA takes (default 16),
 *                    lower values force more context splits (and merges);
 *   use_pdl          1 (default): programmatic dependent launch for both
 *                    launches: the attention kernel may start its set-up
 *                    (reading context_lens and block_tables) while the
 *                    preceding kernel in the stream runs, if that kernel
 *                    allows it (the library's append kernels do), and waits
 *                    for that kernel before its first read of q or the pools;
 *                    the split merge overlaps the attention kernel's tail.
 *                    -1: plain launches (use it when a preceding kernel of
 *                    your own triggers dependents early and writes
 *                    context_lens or block_tables after that);
 *   seg_cost_blocks  fixed cost, in blocks, charged to every (sequence,
 *                    kv-head) when work is divided among CTAs (default: 128
 *                    tokens' worth, 256 over an int8 K pool with several
 *                    query rows per KV head; -1 for none);
 *   producer_wait_ns limit, in nanoseconds, of the loading warp's waits for
 *                    a free pipeline stage (default 2 s; below 1000 the
 *                    loader gives up at the first stage that is not already
 *                    free, as the device timer is too coarse to measure
 *                    less).  Meant for failure-detection tests: with a limit
 *                    shorter than a stage's turnaround the loader gives up,
 *                    the CTA finishes the
 *                    stages already loaded and stops, KV_DEV_TIMEOUT is set
 *                    in the device error word and the output is undefined;
 *                    the call still returns and later calls are unaffected.
 *                    The compute warps' waits keep the default limit (they
 *                    meet at a barrier at the end of every sequence, so they
 *                    must all stop at the same stage);
 *   consumer         the compute path for more than one query row per KV
 *                    head at head_dim 128: 1 = warp-level tensor-core MMAs
 *                    (mma.sync, accumulators in registers), 2 = tcgen05 MMAs
 *                    with accumulators in tensor memory, 0 = default (the
 *                    warp-level MMAs).  Both compute the same attention;
 *                    other values are rejected with KV_ERR_INVALID. */
typedef struct paged_attention_opts {
    int32_t grid_ctas;
    int32_t min_split_blocks;
    int32_t use_pdl;
    int32_t seg_cost_blocks;
    int32_t producer_wait_ns;
    int32_t consumer;
    int32_t reserved[2];
} paged_attention_opts;

int paged_attention_ex(const void* q, const void* k_pool, const void* v_pool,
                       const int32_t* block_tables, int32_t max_blocks_per_seq,
                       const int32_t* context_lens, int32_t q_len, float scale, void* out,
                       int32_t B, int32_t Hq, int32_t Hkv, int32_t head_dim, int32_t block_size,
                       int32_t num_blocks, void* workspace, size_t workspace_bytes,
                       const paged_attention_opts* opts, void* stream);

/* paged_prefill_attention with launch knobs (opts may be NULL): only
 * producer_wait_ns is read, as the limit of the loading warp's wait without
 * progress (a free ring slot); below 1000 it gives up at the first wait.  On
 * a give-up the kernel stops, sets KV_DEV_TIMEOUT and leaves the output
 * undefined; the compute warps reach their own 2 s limits first, so the call
 * returns within a few seconds; later calls are unaffected. */
int paged_prefill_attention_ex(const void* q, const void* k_pool, const void* v_pool,
                               const int32_t* block_tables, int32_t max_blocks_per_seq,
                               const int32_t* context_lens, int32_t q_len, float scale, void* out,
                               int32_t B, int32_t Hq, int32_t Hkv, int32_t head_dim,
                               int32_t block_size, int32_t num_blocks,
                               const paged_attention_opts* opts, void* stream);

/* paged_attention_q8k with the launch knobs of paged_attention_ex (opts may
 * be NULL: defaults). */
int paged_attention_q8k_ex(const void* q, const void* kq_pool, const float* k_scales,
                           const void* v_pool, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t q_len,
                           float scale, void* out, int32_t B, int32_t Hq, int32_t Hkv,
                           int32_t head_dim, int32_t block_size, int32_t num_blocks,
                           void* workspace, size_t workspace_bytes,
                           const paged_attention_opts* opts, void* stream);

/* paged_decode_attention without a workspace argument: for callers that may
 * not allocate device memory themselves (their device memory is owned by
 * another allocator, they receive tensors but no way to allocate, or a
 * cudaMalloc on their hot path is not allowed).  The pages have no
 * counterpart to this call; it exists for those callers only.
 *   - Scratch for context splits comes from a fixed 8 MiB array inside the
 *     library, present on every device that loads it until process exit.
 *     Shapes that would need more return KV_ERR_INVALID (use
 *     paged_decode_attention with a workspace instead).
 *   - The call allocates nothing.  Its first call on each device looks up the
 *     array's device address (a host-side runtime query, done once per
 *     device with that device current); make that first call before any
 *     stream capture.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents; nothing in it needs to start at zero.  Calls that overlap on
 *     the GPU (different streams running at the same time) race on it:
 *     serialise them.
 * Arguments and results are those of paged_decode_attention. */
int paged_decode_attention_static_ws(const void* q, const void* k_pool, const void* v_pool,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* context_lens, float scale, void* out,
                                     int32_t B, int32_t Hq, int32_t Hkv, int32_t head_dim,
                                     int32_t block_size, int32_t num_blocks, void* stream);

/* Read the current device's error word (bits KV_DEV_*) after synchronizing
 * `stream`; reset != 0 clears it. */
int kv_device_error(int32_t* word_out, int32_t reset, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_H */
