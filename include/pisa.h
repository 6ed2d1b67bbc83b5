/*
 * pisa.h - C ABI of the B200 (sm_100a) PISA pyramid block-sparse attention library.
 *
 * The method, as described in "Attention clairsemee PISA : noyaux Triton sans
 * matrice de scores" (irisproject.cloud):
 *   1. keys are mean-pooled into blocks, then into coarser and coarser levels
 *      (sections "Une pyramide de cles plutot qu'un tapis uniforme" and
 *      "Le pooling comme premiere reduction");
 *   2. each query block descends that pyramid, keeping its top-K blocks
 *      (section "La selection top-K guidee par la pyramide");
 *   3. exact softmax attention runs over the selected key/value blocks only,
 *      fused so that no score matrix is written to memory (section
 *      "Des noyaux Triton qui ne materialisent rien").
 *
 * Conventions shared by every call:
 *   - Q, K, V, O are bf16, contiguous [batch, heads, tokens, head_dim] with
 *     head_dim innermost. Device pointers, 16-byte aligned.
 *   - The caller owns and allocates every buffer, the workspace included.
 *     The library never allocates or frees memory and never synchronises,
 *     except pisa_check_status, which synchronises the given stream.
 *   - Every compute call only enqueues work on `stream` and returns.
 *   - Argument errors are detected on the host, before anything is enqueued,
 *     and returned synchronously. A failed kernel launch returns
 *     PISA_ERR_CUDA. Errors a kernel detects on the device (an index outside
 *     the eligible blocks, a pipeline wait that ran out of time) are recorded
 *     in the status word at the start of the workspace and reported by
 *     pisa_check_status; the kernel skips the offending work and returns.
 *   - Argument checks never touch the GPU, so they can be exercised on a host
 *     without one.
 */
#ifndef PISA_H
#define PISA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PISA_API __attribute__((visibility("default")))
#else
#define PISA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t / CUstream). NULL is the legacy default stream. */
typedef struct CUstream_st *pisa_stream_t;

/* Problem description shared by every call.
 *   batch, heads_q, heads_kv : heads_q % heads_kv == 0 (g = heads_q / heads_kv query
 *                              heads share one KV head; g = 1 is multi-head attention).
 *   seq_kv                   : keys per sequence, a multiple of `block`.
 *   seq_q                    : == seq_kv for prefill (query t sits at position t);
 *                              == 1 for decode (the query sits at position seq_kv - 1).
 *   head_dim                 : 64 or 128.
 *   block                    : key-block size b (and query-block size for prefill): 64 or 128.
 *   factor                   : pooling factor f >= 2 between pyramid levels.
 *   topk                     : K, key blocks kept per query block, 1 <= K; factor * K <= 4096,
 *                              and K <= 256 for prefill (seq_q == seq_kv).
 *   causal                   : 0/1. Prefill only: query block i may use key blocks j <= i
 *                              and, inside block i, keys at or before the query.
 *   select_per_qhead         : 0 = one selection per (batch, KV head, query block) from the
 *                              mean over the g query heads (default); 1 = one selection per
 *                              query head.
 *   scale                    : softmax scale; <= 0 selects 1/sqrt(head_dim).
 *   forced_blocks            : selection variant (PISA page, section "Ce que cela change pour
 *                              vous": top-K variants per domain; Pulsar Attention page, section
 *                              "Phase 1 : Encodage statistique du contexte": a fixed
 *                              attention-sink prefix). Bit mask of
 *                              PISA_FORCE_SINK (key block 0) and PISA_FORCE_LOCAL (the query's own
 *                              block: block i for prefill, the last block for decode). A forced
 *                              block is always selected; the descent fills the other
 *                              K - (forced blocks) slots at level 0 from the remaining candidates
 *                              (coarser levels keep their budgets). At most K forced blocks are
 *                              kept, the sink first. 0 = plain top-K (default).
 *   kv_capacity              : decode over a growing KV cache: K and V are [B, Hkv, kv_capacity,
 *                              D] of which the first seq_kv positions hold keys; the pyramid
 *                              layout (levels, offsets, size) is that of kv_capacity, so it does
 *                              not move as the cache grows (pisa_append_pyramid). A multiple of
 *                              block, >= seq_kv. 0 means seq_kv. Prefill requires 0 or seq_kv. */
typedef struct {
    int32_t batch, heads_q, heads_kv, seq_q, seq_kv, head_dim;
    int32_t block, factor, topk, causal;
    int32_t select_per_qhead;
    float scale;
    int32_t forced_blocks;
    int32_t kv_capacity;
} pisa_shape;

#define PISA_FORCE_SINK 1
#define PISA_FORCE_LOCAL 2

typedef enum {
    PISA_OK = 0,
    PISA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, inconsistent shape                */
    PISA_ERR_UNSUPPORTED = 2,  /* a valid shape this build has no kernel for                 */
    PISA_ERR_WORKSPACE = 3,    /* workspace smaller than pisa_workspace_size                 */
    PISA_ERR_CUDA = 4,         /* a CUDA call or kernel launch failed                        */
    PISA_ERR_TIMEOUT = 5,      /* device: a pipeline wait ran out of time                    */
    PISA_ERR_BAD_INDEX = 6     /* device: a selected block outside [0, n0) or after the query */
} pisa_status;

#define PISA_MAX_LEVELS 24
/* Largest candidate set one pyramid level may score: factor * max level budget. */
#define PISA_MAX_CANDIDATES 4096

/* Number of pyramid levels L (n_0 = seq_kv / block, n_{l+1} = ceil(n_l / factor),
 * built while n_l > factor), or -1 if the shape is invalid. Host only. */
PISA_API int32_t pisa_num_levels(const pisa_shape *shape);

/* Node count n_l and row offset of every level inside one (batch, KV head) plane
 * of the pyramid buffer. `sizes` and `offsets` hold at least PISA_MAX_LEVELS
 * entries; unused entries are set to 0. Host only. */
PISA_API pisa_status pisa_level_layout(const pisa_shape *shape, int32_t *sizes, int32_t *offsets);

/* Bytes of the pyramid buffer: fp32 [batch, heads_kv, sum_l n_l, head_dim].
 * Level l of plane (b, h) starts at row offsets[l] of that plane. Host only. */
PISA_API pisa_status pisa_pyramid_size(const pisa_shape *shape, size_t *bytes);

/* Bytes of workspace that pisa_forward, pisa_select_blocks and
 * pisa_sparse_attention need for this shape (one size serves all three).
 * The first 256 bytes are the device status word; zero them once when the
 * workspace is allocated (pisa_check_status clears them after each read).
 * Prefill with 16 or more query blocks and more than 592 selection rows
 * (batch * Hsel * nQB), while scoring every eligible node is cheaper than the
 * sparse descent (up to about 1M tokens at block 128), also
 * holds an fp32 score plane of B * Hsel * qc * total_nodes values (Hsel =
 * heads_kv, or heads_q with select_per_qhead): the selection scores and
 * descends qc query blocks at a time, qc a multiple of 128 chosen so the plane
 * stays within 192 MiB (128 query blocks if even those need more), and a copy
 * of the query summaries and of the pyramid split into tf32 head and remainder
 * (2 * 4 * D * (B * Hsel * nQB + B * heads_kv * total_nodes) bytes) for the
 * tensor-core scoring. Host only. */
PISA_API pisa_status pisa_workspace_size(const pisa_shape *shape, size_t *bytes);

/* Step 1, the key pyramid ("Le pooling comme premiere reduction"): level 0 is
 * the fp32 mean of every key block of `block` keys; a node of level l+1 is the
 * mean of its children weighted by the level-0 blocks each covers (so every
 * node is the mean of all keys under it). With spare capacity (kv_capacity >
 * seq_kv) only the first seq_kv / block blocks hold keys: the weights count
 * those alone, and a node over none of them is 0.
 *   K        : bf16 [batch, heads_kv, kv_capacity (or seq_kv), head_dim], device.
 *   pyramid  : fp32 output, pisa_pyramid_size bytes, device. */
PISA_API pisa_status pisa_build_pyramid(const pisa_shape *shape, const void *K, float *pyramid,
                               pisa_stream_t stream);

/* Keeps a pyramid current as a KV cache grows, without rebuilding it (incremental pyramid
 * maintenance for decode; PISA page, section "Le pooling comme premiere reduction": each level
 * summarises the one below). `pyramid` must hold the pyramid of the cache at length
 * `seq_kv_old` (from pisa_build_pyramid or an earlier append with the same kv_capacity; a
 * zero-filled buffer is the pyramid of an empty cache). The call computes the level-0 means of
 * the blocks completed since, [seq_kv_old / block, seq_kv / block), and every coarser node over
 * them, with the arithmetic of pisa_build_pyramid: the result equals a build at seq_kv bit for
 * bit. Work is O((new blocks) * block * D + L * f * D) per plane, not O(seq_kv * D).
 *   shape      : the cache after the append (seq_kv = new length, kv_capacity as before).
 *   K          : bf16 [B, Hkv, kv_capacity, D], device.
 *   pyramid    : fp32, device, pisa_pyramid_size bytes, updated in place.
 *   seq_kv_old : 0 <= seq_kv_old <= seq_kv, a multiple of block.
 * Errors: PISA_ERR_INVALID_ARG for a bad shape, null or misaligned pointers or a bad
 * seq_kv_old; PISA_ERR_CUDA if a launch fails. Asynchronous on `stream`. */
PISA_API pisa_status pisa_append_pyramid(const pisa_shape *shape, const void *K, float *pyramid,
                                         int32_t seq_kv_old, pisa_stream_t stream);

/* Step 2, pyramid-guided top-K ("La selection top-K guidee par la pyramide").
 * For every query block: its summary q = mean of its queries (over the g query
 * heads of the KV head unless select_per_qhead; decode: the single token);
 * start from every eligible node of the top level; at each level score the
 * candidates by the fp32 dot product q . node, keep the best K_l (higher score
 * first, lower node index on equal scores; all of them if there are no more
 * than K_l) and descend to their children. Causal: only blocks j <= i are
 * eligible and a node that straddles block i is scored with the mean of its
 * eligible blocks.
 *   Q            : bf16 queries (layout above), device.
 *   pyramid      : fp32 pyramid from pisa_build_pyramid, device.
 *   level_budget : HOST array of L budgets K_l (level 0 first, K_0 == topk), or
 *                  NULL for K at every level.
 *   idx          : int32 output [batch, Hsel, nQB, topk], device; Hsel = heads_kv
 *                  (shared) or heads_q (per query head); nQB = seq_q / block
 *                  (prefill) or 1 (decode). Each row lists the kept blocks in
 *                  ascending order, padded with -1.
 *   margin       : optional fp32 output [batch, Hsel, nQB], device: smallest
 *                  relative gap (s_K - s_K+1) / max(|s_K|, |s_K+1|) met at a
 *                  pruning level (+inf if no level was pruned). NULL to skip.
 *   ws, ws_bytes : workspace (pisa_workspace_size), device. */
PISA_API pisa_status pisa_select_blocks(const pisa_shape *shape, const void *Q, const float *pyramid,
                               const int32_t *level_budget, int32_t *idx, float *margin,
                               void *ws, size_t ws_bytes, pisa_stream_t stream);

/* Step 3, fused block-sparse attention ("Des noyaux Triton qui ne
 * materialisent rien"): for every query row, S = scale * q . k over the keys
 * of the blocks listed in its idx row (keys after the query masked when
 * causal), O = softmax(S) V and LSE = log sum exp S, computed tile by tile
 * with an online softmax; scores never leave on-chip memory.
 *   idx   : int32 [batch, Hsel, nQB, topk] as produced by pisa_select_blocks;
 *           entries < 0 are skipped; an entry >= n0, or > i when causal,
 *           is skipped and recorded as PISA_ERR_BAD_INDEX. Entries must be
 *           distinct (a repeated block is attended twice).
 *   O     : bf16 output, same layout as Q, device.
 *   lse   : optional fp32 output [batch, heads_q, seq_q] (natural log), or NULL.
 * A query row whose idx row holds no valid block gets O = 0 and LSE = -inf. */
PISA_API pisa_status pisa_sparse_attention(const pisa_shape *shape, const void *Q, const void *K,
                                  const void *V, const int32_t *idx, void *O, float *lse,
                                  void *ws, size_t ws_bytes, pisa_stream_t stream);

/* Workspace bytes pisa_sparse_attention_backward needs for `shape` (prefill shapes only;
 * PISA_ERR_UNSUPPORTED for decode). Host only. */
PISA_API pisa_status pisa_backward_workspace_size(const pisa_shape *shape, size_t *bytes);

/* Backward of step 3 through a fixed selection (PISA page, section "Ce que cela change pour
 * vous": the sparse kernels also serve training; the block selection is a discrete choice and
 * passes no gradient). With S = scale Q K^T over the selected keys, P = exp(S - LSE):
 *   dV = P^T dO,  dS = P * (dO V^T - rowsum(dO * O)),  dQ = scale dS K,  dK = scale dS^T Q,
 * a KV head's dK and dV summing over all query rows (of all its query heads) that use each key.
 *   Q, K, V, O : bf16 as in pisa_sparse_attention (O its output), device.
 *   lse        : fp32 [batch, heads_q, seq_q], the forward's LSE, device.
 *   dO         : bf16, same layout as O, device.
 *   idx        : the selection the forward used. Entries < 0, >= n0, or > i when causal are
 *                skipped (not recorded: the forward call that produced or checked idx records
 *                them).
 *   dQ, dK, dV : bf16 outputs, the layouts of Q, K, V, device. Every element is written (keys
 *                no query uses get 0).
 *   ws         : >= pisa_backward_workspace_size bytes, 16-byte aligned, device.
 * Prefill only (seq_q == seq_kv, no spare capacity); PISA_ERR_UNSUPPORTED otherwise.
 * Deterministic: no atomics; every sum runs in a fixed order. Asynchronous on `stream`. */
PISA_API pisa_status pisa_sparse_attention_backward(const pisa_shape *shape, const void *Q, const void *K,
                                                    const void *V, const void *O, const float *lse,
                                                    const void *dO, const int32_t *idx, void *dQ, void *dK,
                                                    void *dV, void *ws, size_t ws_bytes, pisa_stream_t stream);

/* Steps 1-3 in one call on one stream: pyramid and query summaries into the
 * workspace, selection, attention.
 *   idx_out : optional int32 [batch, Hsel, nQB, topk] copy of the selection
 *             (NULL keeps it in the workspace). */
PISA_API pisa_status pisa_forward(const pisa_shape *shape, const void *Q, const void *K, const void *V,
                         void *O, float *lse, int32_t *idx_out, void *ws, size_t ws_bytes,
                         pisa_stream_t stream);

/* Decode attention that allocates nothing. The paper has no counterpart: this
 * is a convenience for callers that may not call cudaMalloc, such as code
 * running inside another framework's memory pool, a plugin without an
 * allocator of its own, or a serving loop that must not allocate once running.
 * It computes exactly what pisa_sparse_attention computes for a decode shape
 * (seq_q == 1), with the same kernels, but keeps the split-KV partials and the
 * status word in a fixed 8 MiB device array built into the library instead of
 * a caller workspace. The caller still passes Q, K, V, idx, O and lse (lse may
 * be NULL), laid out as for pisa_sparse_attention.
 *   - Every GPU that loads the library holds the 8 MiB array until exit.
 *   - Every call looks up the array's device address (cudaGetSymbolAddress,
 *     which allocates nothing) with the calling device current. The first
 *     call on a device may load the library's device code there: make it
 *     before any stream capture.
 *   - Size limit: with rows = batch * Hsel (Hsel = heads_kv, or heads_q with
 *     select_per_qhead), gsel = heads_q / heads_kv (1 with select_per_qhead),
 *     per_split = clamp(ceil(topk / ceil(592 / rows)), 2, 16) and
 *     splits = ceil(topk / per_split), the call needs
 *     256 + rows * splits * gsel * (head_dim + 2) * 4 bytes <= 8 MiB; a larger
 *     shape returns PISA_ERR_WORKSPACE. (64 sequences, 8 KV heads, 32 query
 *     heads, head_dim 128, topk 64: 4 splits, 4.26 MB.) Non-decode shapes
 *     return PISA_ERR_INVALID_ARG.
 *   - Calls share the array: calls whose kernels overlap on the GPU race on it.
 *     Each call clears the status word when it starts; errors its kernels
 *     record there (an idx entry outside [0, n0), a pipeline wait that ran out
 *     of time) are read by pisa_decode_noalloc_check_status.
 *     pisa_last_launch_count does not count this call.
 *   - No cudaMalloc, cudaFree or allocating library routine is called. */
PISA_API pisa_status pisa_decode_attention_noalloc(const pisa_shape *shape, const void *Q, const void *K,
                                                   const void *V, const int32_t *idx, void *O, float *lse,
                                                   pisa_stream_t stream);

/* Companion of pisa_decode_attention_noalloc (no counterpart in the paper either):
 * synchronises `stream`, returns the device-side error the most recent
 * pisa_decode_attention_noalloc call on the current device recorded in the
 * library's array (PISA_OK if none) and clears it. `detail`, if not NULL,
 * receives the code locating the error. Allocates nothing. */
PISA_API pisa_status pisa_decode_noalloc_check_status(uint32_t *detail, pisa_stream_t stream);

/* Self-test of the bounded waits (no counterpart in the paper): enqueues one kernel whose single
 * mbarrier wait can never complete (nothing arrives on the barrier and no copy or MMA is issued).
 * The wait gives up after `limit_us` microseconds (1 .. 1,000,000), records PISA_ERR_TIMEOUT in
 * the status word at the start of `ws` (detail 0x501) and the kernel returns, which is what any
 * pipeline wait of the library does when its limit (2 s) runs out. Read the result with
 * pisa_check_status. `ws`: device, 16-byte aligned, at least 256 bytes. Asynchronous on `stream`.
 *
 * Fault injection: when the environment variable PISA_FAULT is "launch", every call of this
 * header that enqueues work returns PISA_ERR_CUDA after its argument checks, as if its first
 * kernel launch had failed, and enqueues nothing. */
PISA_API pisa_status pisa_selftest_wait_timeout(void *ws, uint32_t limit_us, pisa_stream_t stream);

/* Synchronises `stream`, returns the first device-side error recorded in the
 * workspace status word since the last call (PISA_OK if none) and clears it.
 * `detail`, if not NULL, receives a code locating the error (kernel and wait site). */
PISA_API pisa_status pisa_check_status(void *ws, uint32_t *detail, pisa_stream_t stream);

/* Static, human-readable name of a status code. */
PISA_API const char *pisa_status_string(pisa_status status);

/* Kernel launches the last compute call on this host thread enqueued. */
PISA_API int32_t pisa_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* PISA_H */
