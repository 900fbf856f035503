/*
 * msa.h -- C ABI of libmsa: MiniMax Sparse Attention (MSA) over grouped query attention,
 * the data-parallel hot path, for NVIDIA B200 (sm_100a).
 *
 * The method (sources, by page title and section):
 *  - youmind article "MiniMax M3 sparse attention agents", paragraph "The mechanism that
 *    changes this" and figure 1 caption: before attention a light Index Branch scores the
 *    key-value context in blocks and keeps the top-k blocks per query and GQA group; the
 *    main branch attends only to those blocks.
 *  - same article, bullet "Predictable cost at every length": Bk = 128 tokens per block and
 *    k = 16 blocks, a fixed budget of 2,048 key-value tokens per query and GQA group.
 *  - same article, paragraph "Why this comes now": the kernels split the context into blocks
 *    and read each block once with contiguous memory access.
 *  - KuCoin flash "MiniMax launches MSA sparse attention method and MiniMax-M3 model",
 *    summary: MSA is built on GQA; the index branch picks 16 blocks of (default) 128 tokens
 *    per GQA group, the main branch runs exact softmax attention over those blocks, and the
 *    top-k selection is exp-free.
 *
 * The pages do not give the scoring function. This library computes:
 *   pooled key of full block j:   kbar_j = mean of the Bk index keys k_I of block j (fp32)
 *   score of fully-past block j:  s_j = q_I . kbar_j / sqrt(d_I), for j < c = floor(t / Bk)
 *   selection for the query at t: {c} plus the k-1 best j < c, ordered by (s desc, j asc);
 *                                 every block 0..c when c + 1 <= k
 *   output of query head h:       softmax(q_h . k_u / sqrt(d)) weighted sum of v_u over the
 *                                 keys u <= t of the selected blocks; all heads of a group
 *                                 share the group's selection; head h is in group h/(Hq/G).
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library allocates
 *    nothing. Tensors are dense row-major with the shapes stated below (innermost last).
 *    bf16 tensors are passed as void*; 16-byte alignment is required for every pointer.
 *  - Every call validates its arguments on the host first and returns an error without
 *    launching anything when they are wrong; otherwise it only enqueues work on `stream`
 *    (asynchronous, no synchronisation, safe to capture in a CUDA graph).
 *  - MSA_ERR_CUDA reports a launch error (the CUDA error is kept for msa_last_cuda_error).
 *  - Problems only the device can see (a selection id out of range, a position beyond the
 *    cache) are recorded in the workspace's error word and read by msa_get_device_status.
 *  - Workspaces are device buffers of msa_workspace_size() bytes that must be zero-filled
 *    before their first use; the library leaves them ready for the next call. Calls that
 *    share a workspace must be ordered on one stream.
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (NULL = the legacy default stream). */
typedef struct CUstream_st *msa_stream_t;

typedef enum {
    MSA_OK = 0,
    MSA_ERR_INVALID_ARGUMENT = 1, /* null/misaligned pointer, bad size or shape */
    MSA_ERR_UNSUPPORTED = 2,      /* constants other than d=128, d_I=64, Bk=128, k=16, or Hq/G not in {1,2,4,8,16} */
    MSA_ERR_WORKSPACE = 3,        /* workspace missing or smaller than msa_workspace_size() */
    MSA_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed */
    MSA_ERR_TIMEOUT = 5,          /* (device) a bounded wait expired */
    MSA_ERR_DEVICE_BOUNDS = 6     /* (device) an index or position was out of range */
} msa_status_t;

typedef struct {
    int32_t batch;       /* B: sequences */
    int32_t n_q_heads;   /* Hq: query heads */
    int32_t n_kv_groups; /* G: key-value heads (GQA groups); Hq % G == 0 */
    int32_t head_dim;    /* d: must be 128 */
    int32_t index_dim;   /* d_I: index-branch dimension per group, must be 64 */
    int32_t block_size;  /* Bk: must be 128 */
    int32_t top_k;       /* k: blocks per query and group, must be 16 */
} msa_shape_t;

/* Operation ids for msa_workspace_size. */
enum {
    MSA_OP_INDEX_SELECT_PREFILL = 0,
    MSA_OP_INDEX_SELECT_DECODE = 1,
    MSA_OP_ATTN_PREFILL = 2,
    MSA_OP_ATTN_DECODE = 3,
    MSA_OP_ATTN_PREFILL_BACKWARD = 4
};

/* Version of this ABI (bumped on any incompatible change). */
int32_t msa_abi_version(void);

const char *msa_status_string(msa_status_t status);

/* The CUDA error code behind the last MSA_ERR_CUDA returned on this host thread. */
int32_t msa_last_cuda_error(void);

/* Number of kernels this library has enqueued in this process (all threads), for launch
 * accounting in benchmarks. Kernels enqueued while a stream is being captured are counted
 * once, at capture; graph replays are not counted. */
uint64_t msa_kernel_launches(void);

/* Kernel ids: workspace error records (info[0] of msa_get_device_status) and timing records. */
enum {
    MSA_KERNEL_POOL = 1,             /* pooling (and its chunked form), running-sum reset */
    MSA_KERNEL_SELECT_PREFILL = 2,   /* prefill block scores + exp-free top-k (tensor cores) */
    MSA_KERNEL_SELECT_DECODE = 3,    /* decode block scores + exp-free top-k */
    MSA_KERNEL_APPEND = 4,           /* decode append and pooled-key update */
    MSA_KERNEL_ATTN_DECODE = 5,      /* decode main branch (bf16 or FP8 cache) */
    MSA_KERNEL_ATTN_PREFILL = 6,     /* prefill main branch, key-value-major attention */
    MSA_KERNEL_INVERTED_INDEX = 7,   /* prefill / backward: inverted index of the selection */
    MSA_KERNEL_COMBINE = 8,          /* prefill: log-sum-exp merge of the partials */
    MSA_KERNEL_SELFTEST = 9,
    MSA_KERNEL_FP8 = 10,             /* FP8 cache: block quantisation */
    MSA_KERNEL_SPLIT_KEYS = 11,      /* prefill selection: pooled keys split into bf16 terms */
    MSA_KERNEL_ATTN_BACKWARD = 12,   /* main-branch backward: dQ, dK, dV */
    MSA_KERNEL_BACKWARD_DOT = 13,    /* main-branch backward: D = dO . o per row */
    MSA_KERNEL_TOPK = 14             /* msa_topk_rows */
};

/*
 * Per-kernel device time, for benchmarks and profiling. While timing is on, every kernel this
 * library enqueues on a stream that is not being captured is bracketed by two CUDA events on
 * that stream (kernels enqueued during a stream capture, and graph replays, are not timed).
 * The records are kept, in launch order, until read.
 *   msa_kernel_timing_enable(on): on != 0 switches timing on, 0 off; returns the previous state.
 *   msa_kernel_timing_read(kernel, ms, cap): waits for the recorded events, writes up to cap
 *     records -- kernel[i] an MSA_KERNEL_* id, ms[i] that launch's device time in milliseconds
 *     -- then drops every record and its events; returns the number written, or -1 after a
 *     CUDA error (the records are dropped all the same). Host arrays; NULL with cap 0 only
 *     drops the records.
 */
int32_t msa_kernel_timing_enable(int32_t on);
int32_t msa_kernel_timing_read(int32_t *kernel, float *ms, int32_t cap);

/*
 * Workspace bytes needed by one operation.
 *  op = MSA_OP_INDEX_SELECT_PREFILL: n = one past the last query position (the number of query
 *                                    tokens per sequence for a whole prefill, P + n for a chunk);
 *                                    the workspace holds the pooled keys of the fully-past
 *                                    blocks split into three bf16 terms (384 B per block and group)
 *  op = MSA_OP_INDEX_SELECT_DECODE:  n = max_pos (largest query position)
 *  op = MSA_OP_ATTN_PREFILL:         n = number of tokens per sequence
 *  op = MSA_OP_ATTN_DECODE:          n = max_pos
 *  op = MSA_OP_ATTN_PREFILL_BACKWARD: n = number of tokens per sequence
 * Returns 0 for an invalid shape or op.
 */
size_t msa_workspace_size(const msa_shape_t *shape, int32_t op, int64_t n);

/*
 * Index Branch, step 1 -- block pooling (sources: youmind article, figure 1 caption and
 * bullet "Predictable cost at every length"; the mean is this library's reading).
 *   k_idx    bf16 [B, n_tokens, G, d_I]   index keys
 *   pooled   fp32 [B, G, nb_cap, d_I]     out: pooled[b,g,j] = mean of k_idx[b, j*Bk:(j+1)*Bk, g]
 *                                         for every full block j < n_tokens / Bk (must be <= nb_cap);
 *                                         other rows are not touched
 *   tail_sum fp32 [B, G, d_I] or NULL     out: plain sum of the index keys of the trailing
 *                                         partial block (zeros when n_tokens % Bk == 0); this is
 *                                         the running sum msa_pooled_keys_append continues
 */
msa_status_t msa_pool_index_keys(const msa_shape_t *shape, const void *k_idx, int64_t n_tokens,
                                 float *pooled, int64_t nb_cap, float *tail_sum,
                                 msa_stream_t stream);

/*
 * Index Branch, steps 2-3 -- block scores and exp-free top-k selection (sources: youmind
 * article, paragraph "The mechanism that changes this"; KuCoin MSA launch flash, summary).
 *   q_idx   bf16 [B, n_queries, G, d_I]   index queries
 *   q_pos   NULL for prefill: query i of every sequence sits at position i;
 *           else device int32 [B] for decode: the single query (n_queries must be 1) of
 *           sequence b sits at position q_pos[b] (the position of the new token)
 *   max_pos host bound on every query position (prefill: n_queries - 1); sizes the grid;
 *           a q_pos above it is a device bounds error
 *   pooled  fp32 [B, G, nb_cap, d_I]      pooled keys; rows j < floor(pos / Bk) are read
 *   sel     int32 [B, n_queries, G, k]    out: selected block ids in ascending order, padded
 *                                         with -1 (the query's own block is always included)
 *   workspace of msa_workspace_size(op = MSA_OP_INDEX_SELECT_PREFILL or _DECODE)
 */
msa_status_t msa_index_select(const msa_shape_t *shape, const void *q_idx, int64_t n_queries,
                              const int32_t *q_pos, int64_t max_pos, const float *pooled,
                              int64_t nb_cap, int32_t *sel, void *workspace,
                              size_t workspace_bytes, msa_stream_t stream);

/*
 * Decode selection without a workspace. The paper has no counterpart: this is an interface
 * for callers that cannot allocate device memory when they select blocks -- a serving
 * engine that gives all device memory to its own pool at start-up and allows no allocation
 * per step, or a host thread that must not wait on the allocator. It computes exactly what
 * msa_index_select computes in decode mode (same arguments, n_queries = 1), but keeps its
 * scratch in a 2 MiB array that libmsa holds on every GPU that loads it, until exit.
 *  - Limit: B * G * (min(ceil((max_pos / 128) / 1024), 64) * 120 + 4) bytes plus at most
 *    512 must fit in the 2 MiB: any B * G <= 272 fits at every supported max_pos (B = 16,
 *    G = 8 included); B * G = 1024 fits up to max_pos = 2,228,351. Larger problems return
 *    MSA_ERR_WORKSPACE without launching.
 *  - The first call on a device looks up the array's device address (once per device); make
 *    that first call before any stream capture. The address is kept for the life of the
 *    process: do not call this entry point after a cudaDeviceReset (or any other teardown of
 *    the device's primary context) in the same process, since the array may then live
 *    elsewhere.
 *  - Every call shares the one array: calls that may overlap on the GPU (other streams,
 *    other host threads on the same device) race and must be serialised by the caller.
 *  - sel rows are preset to -1; a row left all -1 means the device found its q_pos out of
 *    range (this variant has no workspace error word).
 *  - Allocates nothing: no cudaMalloc/cudaFree; two cudaMemsetAsync calls and one kernel on
 *    `stream`.
 */
msa_status_t msa_index_select_decode_noalloc(const msa_shape_t *shape, const void *q_idx,
                                             const int32_t *q_pos, int64_t max_pos,
                                             const float *pooled, int64_t nb_cap, int32_t *sel,
                                             msa_stream_t stream);

/*
 * Main Branch, prefill -- exact softmax attention over the selected blocks, causal inside
 * the query's own block (sources: youmind article, figure 1 caption; KuCoin MSA launch
 * flash, summary: exact softmax attention only over the selected blocks).
 *   q    bf16 [B, N, Hq, d]     k, v bf16 [B, G, N, d]  (a block of one group is contiguous)
 *   sel  int32 [B, N, G, k]     from msa_index_select (prefill)
 *   out  bf16 [B, N, Hq, d]     out
 *   lse  fp32 [B, N, Hq] or NULL  out: natural log of the softmax denominator of the scaled
 *                                 scores q.k/sqrt(d)
 *   workspace of msa_workspace_size(MSA_OP_ATTN_PREFILL, N)
 * Size limits (device indices are 32-bit): B*N*Hq*k < 2^31 (one partial row per token, query
 * head and selected block), B*N*G*(k-1) < 2^31, B*G*N + Bk < 2^31 and N/Bk <= 49152, else
 * MSA_ERR_UNSUPPORTED before any launch.
 */
msa_status_t msa_sparse_attn_prefill(const msa_shape_t *shape, const void *q, const void *k,
                                     const void *v, int64_t n_tokens, const int32_t *sel,
                                     void *out, float *lse, void *workspace,
                                     size_t workspace_bytes, msa_stream_t stream);

/*
 * Chunked prefill: a chunk of n new tokens at positions P .. P + n - 1 (P = q_start) of every
 * sequence, against caches that already hold positions 0 .. P - 1. Source: youmind article
 * "MiniMax M3 sparse attention agents", bullet "Predictable cost at every length" (every query
 * reads the same fixed budget of 16 blocks = 2,048 key-value tokens, whatever the length); the
 * chunk is this library's reading of the step between a prefill and decode. Every query of the
 * chunk selects among all fully-past blocks -- cached ones and those the chunk itself completes
 * -- exactly as in a whole prefill, so the chunked results equal rows P .. P + n - 1 of a
 * prefill of the whole sequence (up to the order of the fp32 sums in the pooled keys).
 * Order of a chunk: msa_pool_index_keys_chunk, msa_index_select_chunk, then (once the chunk's
 * K and V rows are in the caches) msa_sparse_attn_prefill_chunk.
 */

/* Pool the chunk's index keys k_idx [B, n, G, d_I] (positions P .. P + n - 1) into pooled
 * [B, G, nb_cap, d_I] for every block the chunk completes, and keep tail_sum [B, G, d_I] -- the
 * plain sum of the open block's positions, which must hold positions Bk floor(P / Bk) .. P - 1
 * on entry (zeros when P is a multiple of Bk) -- current. pooled may be NULL when no block
 * completes. (P + n) / Bk <= nb_cap. */
msa_status_t msa_pool_index_keys_chunk(const msa_shape_t *shape, const void *k_idx, int64_t q_start, int64_t n,
                                       float *pooled, int64_t nb_cap, float *tail_sum, msa_stream_t stream);

/* Block scores and exp-free top-k selection for the chunk's index queries q_idx [B, n, G, d_I]
 * (row i at position P + i); sel [B, n, G, k] as msa_index_select. pooled must hold every full
 * block below P + n (after msa_pool_index_keys_chunk). Workspace (16-byte aligned) of
 * msa_workspace_size(MSA_OP_INDEX_SELECT_PREFILL, P + n). */
msa_status_t msa_index_select_chunk(const msa_shape_t *shape, const void *q_idx, int64_t q_start, int64_t n,
                                    const float *pooled, int64_t nb_cap, int32_t *sel, void *workspace,
                                    size_t workspace_bytes, msa_stream_t stream);

/* Main Branch for the chunk: q [B, n, Hq, d] (row i at position P + i), k_cache, v_cache
 * [B, G, l_cap, d] holding positions 0 .. P + n - 1 (P + n <= l_cap), sel from
 * msa_index_select_chunk; out [B, n, Hq, d], lse [B, n, Hq] or NULL. Workspace of
 * msa_prefill_chunk_workspace_size(shape, P, n) bytes. Size limits as msa_sparse_attn_prefill
 * with N = n, plus B*G*l_cap + Bk < 2^31 and (P + n) / Bk <= 49152. */
msa_status_t msa_sparse_attn_prefill_chunk(const msa_shape_t *shape, const void *q, const void *k_cache,
                                           const void *v_cache, int64_t l_cap, int64_t q_start, int64_t n,
                                           const int32_t *sel, void *out, float *lse, void *workspace,
                                           size_t workspace_bytes, msa_stream_t stream);

/* Workspace bytes of msa_sparse_attn_prefill_chunk (0 for an invalid shape, P < 0 or n < 1). */
size_t msa_prefill_chunk_workspace_size(const msa_shape_t *shape, int64_t q_start, int64_t n_queries);

/*
 * Main Branch, backward pass of a prefill: the gradient of the outputs with respect to q, k and
 * v, the selection held fixed (a discrete choice). Sources: youmind article "MiniMax M3 sparse
 * attention agents", bullet on MSA-CPT, and KuCoin MSA launch flash, "ME AI News" (MSA-PT):
 * the model is trained through the sparse attention. With z_u = q . k_u / sqrt(d) over the
 * keys u of the forward (selected blocks, u <= t), p = softmax(z), o = sum p_u v_u and the
 * upstream gradient dO of o: dV_u += p_u dO, dS_u = p_u (dO . v_u - dO . o),
 * dQ = sum_u dS_u k_u / sqrt(d), dK_u += dS_u q / sqrt(d) (summed over heads and queries).
 *   q, k, v, sel      as msa_sparse_attn_prefill (N = n_tokens)
 *   out, lse          the forward's outputs (bf16 [B, N, Hq, d], fp32 [B, N, Hq]; lse required)
 *   d_out             bf16 [B, N, Hq, d]  upstream gradient of out
 *   dq                fp32 [B, N, Hq, d]  out
 *   dk, dv            fp32 [B, G, N, d]   out (every row written; rows no query attends are 0)
 *   workspace of msa_workspace_size(MSA_OP_ATTN_PREFILL_BACKWARD, N)
 * Sums over blocks and queries run in fp32 with atomic adds, so the low bits of the results
 * may differ between runs. Size limits as msa_sparse_attn_prefill.
 */
msa_status_t msa_sparse_attn_prefill_backward(const msa_shape_t *shape, const void *q, const void *k,
                                              const void *v, int64_t n_tokens, const int32_t *sel,
                                              const void *out, const float *lse, const void *d_out,
                                              float *dq, float *dk, float *dv, void *workspace,
                                              size_t workspace_bytes, msa_stream_t stream);

/*
 * Decode: append the new token to the caches and keep the pooled keys current (the pages
 * fix only the block size; the incremental update is this library's reading of it).
 *   ctx_len   device int32 [B]: tokens already cached (L_b); the new token goes to position L_b
 *   k_idx_new bf16 [B, G, d_I]  the new token's index keys
 *   k_new, v_new bf16 [B, G, d] or both NULL  -> written to k_cache/v_cache [B, G, l_cap, d]
 *   tail_sum  fp32 [B, G, d_I]  running sum of the open block: set to k_idx_new when L_b is a
 *                               multiple of Bk, else incremented by it
 *   pooled    fp32 [B, G, nb_cap, d_I]: when L_b + 1 completes block j = L_b / Bk,
 *                               pooled[b,g,j] = tail_sum / Bk
 * The kernel is launched with programmatic dependent launch: it may start during the tail of
 * the previous kernel of this library on the stream (the step's msa_index_select, which reads
 * only the pooled keys of blocks below L_b / Bk) and completes only after that kernel, so a
 * decode step may run selection, append, attention in that order; the attention needs the
 * appended key and value.
 */
msa_status_t msa_pooled_keys_append(const msa_shape_t *shape, const void *k_idx_new,
                                    const void *k_new, const void *v_new, const int32_t *ctx_len,
                                    void *k_cache, void *v_cache, int64_t l_cap, float *tail_sum,
                                    float *pooled, int64_t nb_cap, void *workspace,
                                    size_t workspace_bytes, msa_stream_t stream);

/*
 * Main Branch, decode -- one query token per sequence, split over the selected blocks and
 * merged by log-sum-exp (sources as msa_sparse_attn_prefill).
 *   q        bf16 [B, Hq, d]
 *   k_cache, v_cache bf16 [B, G, l_cap, d]; positions 0..q_pos[b] must be filled
 *   q_pos    device int32 [B]: the query's position (= L_b, after msa_pooled_keys_append)
 *   max_pos  host bound on q_pos; q_pos[b] must be < l_cap
 *   sel      int32 [B, G, k]  from msa_index_select (decode)
 *   out      bf16 [B, Hq, d]  out;   lse fp32 [B, Hq] or NULL
 *   workspace of msa_workspace_size(MSA_OP_ATTN_DECODE, max_pos)
 */
msa_status_t msa_sparse_attn_decode(const msa_shape_t *shape, const void *q, const void *k_cache,
                                    const void *v_cache, int64_t l_cap, const int32_t *q_pos,
                                    int64_t max_pos, const int32_t *sel, void *out, float *lse,
                                    void *workspace, size_t workspace_bytes,
                                    msa_stream_t stream);

/*
 * A whole decode step in one call: msa_index_select (decode, q_pos = ctx_len), then
 * msa_pooled_keys_append, then msa_sparse_attn_decode, on the stream in that order, with the
 * same arguments, kernels and results as those three calls (sources as theirs). The three
 * workspaces are theirs: msa_workspace_size(MSA_OP_INDEX_SELECT_DECODE, max_pos), at least 256
 * bytes, and msa_workspace_size(MSA_OP_ATTN_DECODE, max_pos); each records its own kernels'
 * device errors (msa_get_device_status). k_new and v_new are required. Every argument of the
 * three steps is checked before the first launch, so a rejected call changes nothing.
 */
msa_status_t msa_decode_step(const msa_shape_t *shape, const void *q, const void *q_idx,
                             const void *k_idx_new, const void *k_new, const void *v_new,
                             const int32_t *ctx_len, void *k_cache, void *v_cache, int64_t l_cap,
                             float *tail_sum, float *pooled, int64_t nb_cap, int64_t max_pos,
                             int32_t *sel, void *out, float *lse, void *ws_select,
                             size_t ws_select_bytes, void *ws_append, size_t ws_append_bytes,
                             void *ws_attn, size_t ws_attn_bytes, msa_stream_t stream);

/*
 * FP8 (e4m3) key-value cache of the decode step. Source: KuCoin flash "MiniMax launches MSA
 * sparse attention method and MiniMax-M3 model", "ME AI News" paragraph (the SM100 attention
 * kernel also takes FP8 inputs); the pages give no format, so this library's reading is:
 *  - every CLOSED 128-token block of a group's keys, and of its values, is stored as e4m3
 *    codes ("E4M3FN": 4 exponent bits, bias 7, 3 mantissa bits, largest finite 448) with one
 *    fp32 scale per (sequence, group, block): scale = amax / 448 (1 for an all-zero block),
 *    code = e4m3(x / scale), the division in fp32, nearest with ties to the even mantissa,
 *    saturating at +-448; a stored value is code x scale;
 *  - the open block -- always the newest query's own block -- stays in the bf16 cache until it
 *    fills (a per-block scale would otherwise change with every append).
 *   k_codes, v_codes  uint8 [B, G, l_cap, d]   the bf16 cache's layout with one byte per value
 *   k_scale, v_scale  fp32 [B, G, nb_cap]      one scale per block
 * These entry points validate and launch like the others; codes and scales of blocks that are
 * not (yet) closed are not read.
 */

/* Quantise blocks j < n_tokens / Bk of every sequence and group from the bf16 caches
 * k_cache, v_cache [B, G, l_cap, d] (after a prefill of n_tokens tokens; n_tokens <= l_cap,
 * n_tokens / Bk <= nb_cap). */
msa_status_t msa_fp8_quantize_blocks(const msa_shape_t *shape, const void *k_cache, const void *v_cache,
                                     int64_t l_cap, int64_t n_tokens, void *k_codes, void *v_codes,
                                     float *k_scale, float *v_scale, int64_t nb_cap, msa_stream_t stream);

/* Decode step, after msa_pooled_keys_append: for every sequence whose new token (at position
 * ctx_len[b], device int32 [B]) completes block j = ctx_len[b] / Bk, quantise that block from
 * the bf16 caches. A position outside [0, l_cap) or a block j >= nb_cap is a device bounds
 * error recorded in `workspace` (>= 256 bytes, zeroed before first use). */
msa_status_t msa_fp8_close_blocks(const msa_shape_t *shape, const int32_t *ctx_len, const void *k_cache,
                                  const void *v_cache, int64_t l_cap, void *k_codes, void *v_codes,
                                  float *k_scale, float *v_scale, int64_t nb_cap, void *workspace,
                                  size_t workspace_bytes, msa_stream_t stream);

/* Main Branch, decode, over the FP8 cache: as msa_sparse_attn_decode, but every selected
 * block below the query's own one is read as e4m3 codes and scales (half the bytes of bf16);
 * the query's own block is read from the bf16 caches k_cache, v_cache. Scores are
 * scale_k * (q . code) and the values code x scale_v, accumulated in fp32; on the e4m3 blocks
 * the products run in f16, which holds every code exactly and every bf16 query value in its
 * normal range, so query values must stay below 65504 in magnitude.
 *   nb_cap  blocks per (sequence, group) in k_scale / v_scale; must be >= max_pos / Bk
 *   workspace of msa_workspace_size(MSA_OP_ATTN_DECODE, max_pos) */
msa_status_t msa_sparse_attn_decode_fp8(const msa_shape_t *shape, const void *q, const void *k_codes,
                                        const void *v_codes, const float *k_scale, const float *v_scale,
                                        int64_t nb_cap, const void *k_cache, const void *v_cache,
                                        int64_t l_cap, const int32_t *q_pos, int64_t max_pos,
                                        const int32_t *sel, void *out, float *lse, void *workspace,
                                        size_t workspace_bytes, msa_stream_t stream);

/*
 * Synchronises `stream`, returns the status recorded in the workspace's error word by the
 * device (MSA_OK, MSA_ERR_DEVICE_BOUNDS or MSA_ERR_TIMEOUT) and clears it. `info` (nullable,
 * 4 int32) receives the recorded detail: kernel id, block, index, value.
 */
msa_status_t msa_get_device_status(void *workspace, int32_t *info, msa_stream_t stream);

/*
 * Exp-free top-k of every row of a score matrix: the Index Branch's selection step on its
 * own, for block scores computed elsewhere. Sources: KuCoin flash "MiniMax launches MSA
 * sparse attention method and MiniMax-M3 model", "ME AI News" paragraph (the top-k is
 * exp-free and is compared with torch.topk at 128K context); youmind article "MiniMax M3
 * sparse attention agents", bullet "Fast in production".
 *   scores  device fp32 [rows, n], row-major; rows of n >= k values, n <= 2^30
 *   k       1..16
 *   idx     device int32 [rows, k]: the k best columns of each row, best first, under the
 *           total order (score descending, column ascending); every NaN ranks above +inf
 *           (NaNs tie with each other) and -0 ties with +0
 *   val     device fp32 [rows, k] or NULL: the scores at idx (the stored values, bit for bit)
 * Only integer compares of order-preserving codes are used (no exponential, no float
 * arithmetic), so the result is exact. No workspace; rows == 0 launches nothing.
 * Returns MSA_ERR_INVALID_ARGUMENT (nothing launched) for rows < 0, k outside 1..16, n < k,
 * n > 2^30, or a null or non-16-byte-aligned scores/idx/val pointer.
 */
msa_status_t msa_topk_rows(const float *scores, int64_t rows, int64_t n, int32_t k, int32_t *idx, float *val,
                           msa_stream_t stream);

/*
 * Self-test of the device failure path. The paper has no counterpart: it lets a caller, and
 * the tests, check that an expired wait is reported rather than hung. One CTA of 32 threads
 * is launched on `stream`; lane 0 waits on a shared-memory barrier that nothing completes,
 * with the same bounded wait every kernel of the library uses (about 2 s of SM clocks), then
 * records MSA_ERR_TIMEOUT with kernel id 9 in the workspace's error word and the kernel ends;
 * the context stays usable. Read the result with msa_get_device_status.
 *   workspace  device, >= 256 bytes, zero before the call (its error word is written)
 * Returns MSA_ERR_WORKSPACE for a null or short workspace (nothing launched).
 */
msa_status_t msa_selftest_wait_timeout(void *workspace, size_t workspace_bytes, msa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H */
