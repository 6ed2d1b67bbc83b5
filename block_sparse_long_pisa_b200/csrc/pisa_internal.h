// Internal definitions shared by the host-side API and the kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include <cuda.h>

#include "pisa.h"

namespace pisa {

// Upper bound on any single pipeline wait inside a kernel (ns).
constexpr uint64_t kWaitLimitNs = 2000000000ull;
// Suspend-time hint of one mbarrier wait attempt (ns); the bound above still applies.
constexpr uint32_t kTryWaitHintNs = 1000000u;

// First pass: every row keeps the maximum of its first key group as the
// reference for all later groups, so the two warps of a row need not agree on
// a new maximum per group. Probabilities then stay below 2^kFirstPassLimit;
// a row whose scores exceed that (in log2 units) marks the CTA, which redoes
// its unit in a second pass with the exact lazy rescale below.
constexpr float kFirstPassLimit = 16.0f;
// Second pass: the running max is kept until a new row max exceeds it by this
// much (log2 units), so probabilities stay below 2^8.
constexpr float kRescaleThreshold = 8.0f;
// Named barrier at which all roles learn whether a second pass runs (1..8
// are the softmax warp pairs' barriers).
constexpr uint32_t kPassBarrier = 15;

// Selected blocks per query block the prefill attention kernel holds on chip.
constexpr int kMaxPrefillTopk = 256;
// Largest number of selected blocks one decode CTA streams (its block list lives in shared memory).
constexpr int kDecMaxBps = 16;
// Prefill with at least this many query blocks per selection row scores every
// eligible node densely (the tiles are shared by 128 query blocks); fewer
// query blocks (and decode) score only the descent's candidates.
constexpr int kDenseSelectMinQBlocks = 16;
// Prefill selections of at most this many rows (batch x selection heads x query blocks: one wave
// of the per-row descent, four 128-thread CTAs on each of 148 SMs) run the per-row descent: its
// one launch beats the dense path's three there (measured: 128 rows 0.048 -> 0.038 ms, 512 rows
// 0.065 -> 0.056 ms; at 600 rows the dense path takes 0.070 ms, the per-row descent a second wave).
constexpr int64_t kSparseSelectMaxRows = 592;
// The dense scoring is used while it scores at most this many times the
// candidates the sparse descent scores (it is ~5x cheaper per candidate);
// past that (very long contexts) the sparse descent's O(N log N) work wins.
constexpr int kDenseSelectMaxWorkRatio = 4;
// Bytes of score plane one dense-selection pass may hold: the query blocks
// are scored and descended in chunks whose plane fits this (the 128K GQA
// prefill fits in one chunk; every chunk costs two more launches).
constexpr size_t kSelectPlaneBudget = size_t(192) << 20;

// Bytes reserved for the status word at the start of the workspace.
constexpr size_t kStatusBytes = 256;

// Wait-site codes reported through the status word's detail field:
// (kernel id << 8) | site.
enum : uint32_t {
    kKernAttnPrefill = 1,
    kKernAttnDecode = 2,
    kKernSelect = 3,
    kKernAttnBackward = 4,
    kKernSelftest = 5,
};

// Fault injection on the host: true when the environment variable PISA_FAULT
// is "launch". Every enqueuing entry point then returns PISA_ERR_CUDA after
// its argument checks, as if its first kernel launch had failed, and enqueues
// nothing (no GPU fault is involved).
bool injected_launch_failure();

// Derived sizes of one problem (host side).
struct Plan {
    int32_t B, Hq, Hkv, g, Nq, N, D, blk, f, topk, causal, per_qhead, decode;
    int32_t forced;      // PISA_FORCE_* bit mask
    float scale;
    int32_t n0;          // key blocks that hold keys (seq_kv / block)
    int32_t n0_cap;      // key blocks of the capacity (kv_capacity / block); the pyramid layout's n_0
    int32_t L;           // pyramid levels
    int32_t lsize[PISA_MAX_LEVELS];
    int32_t loff[PISA_MAX_LEVELS];
    int32_t total_nodes; // sum of level sizes (rows of one pyramid plane)
    int32_t Hsel;        // selection rows per batch: Hkv (shared) or Hq (per query head)
    int32_t nqb;         // query blocks: Nq / blk (prefill) or 1 (decode)
    int32_t gsel;        // query heads averaged into one selection summary
    // decode split-KV
    int32_t dec_bps;     // selected blocks per split
    int32_t dec_splits;
    // workspace layout (byte offsets)
    size_t ws_pyramid, ws_qbar, ws_idx, ws_part, ws_scores, ws_total;
    int32_t dense_select;       // prefill selection scores densely (score plane in the workspace)
    int32_t dense_qc;           // query blocks per dense-selection chunk (a multiple of 128, or nqb)
    size_t ws_split;            // dense selection: tf32 head and remainder of the summaries and nodes
    size_t pyramid_bytes;
};

// Validates a shape and fills the plan. Host only, never touches the GPU.
pisa_status make_plan(const pisa_shape* s, Plan* p);

// ---------------------------------------------------------------- kernel parameter blocks

struct MeanParams {
    const __nv_bfloat16* src;   // bf16 [.., Hsrc, Nsrc, D]
    float* dst;                 // fp32 rows
    int32_t Hsrc, Nsrc, D;
    int32_t Hout;               // output planes per batch
    int32_t rows_out;           // output rows per plane computed by this launch
    int32_t row0;               // first output row (rows row0 .. row0 + rows_out - 1)
    int32_t rows_valid;         // rows at or past this index have no data: written as zeros
    int32_t dst_plane_rows;     // row stride between output planes
    int32_t rows_per_group;     // source rows averaged per output row (block, or 1)
    int32_t planes_per_group;   // consecutive source heads averaged (g or 1)
    int32_t batch;
};

struct LevelParams {
    float* pyr;                 // pyramid base
    int32_t planes;             // batch * heads_kv
    int32_t plane_rows;         // total_nodes
    int32_t off_below, off_cur; // row offsets of the two levels inside a plane
    int32_t n_below, n_cur;     // n_cur: nodes computed by this launch, from node c0 on
    int32_t c0;
    int32_t n0, factor, D;      // n0: level-0 blocks that hold keys (the weights count only these)
    int64_t width_below;        // level-0 blocks under one node of the level below (f^(l-1))
};

// Two-launch pyramid build: subtrees of S = factor^m key blocks, then the levels above them.
struct SubtreeParams {
    const __nv_bfloat16* K;     // bf16 [planes, N, D]
    float* pyr;                 // fp32 [planes, plane_rows, D]
    int64_t planes;             // batch * heads_kv
    int32_t subtrees;           // ceil(lsize[0] / S) per plane
    int32_t S, m;               // key blocks per subtree (factor^m) and the levels formed inside it
    int32_t N, D, blk, factor, L, plane_rows;
    int32_t n0;                 // level-0 blocks that hold keys (the rest of the capacity is zero)
    int32_t lsize[PISA_MAX_LEVELS];
    int32_t loff[PISA_MAX_LEVELS];
};

struct SelectParams {
    const float* qbar;          // fp32 [B, Hsel, nqb, D] (prefill)
    const __nv_bfloat16* qtok;  // decode: the query tokens [B, Hq, 1, D], summarised by the kernel
    int32_t Hq, qheads;         // decode: query heads, and heads averaged per selection row
    const float* pyr;           // fp32 [B, Hkv, total_nodes, D]
    int32_t* idx;               // int32 [B, Hsel, nqb, topk]
    float* margin;              // optional fp32 [B, Hsel, nqb]
    uint32_t* status;
    int32_t Hsel, Hkv, gsel_div, nqb, D, factor, topk, causal, decode, L, total_nodes;
    int32_t n0;                 // level-0 blocks of the pyramid layout (node spans)
    int32_t n0_valid;           // level-0 blocks that hold keys (decode: the last one is the query's)
    int32_t forced;             // PISA_FORCE_* bit mask
    int32_t lsize[PISA_MAX_LEVELS];
    int32_t loff[PISA_MAX_LEVELS];
    int32_t budget[PISA_MAX_LEVELS];
    int64_t width[PISA_MAX_LEVELS];  // f^l (saturated)
    int32_t fshift;                  // log2 f when f is a power of two, else -1
    float* scores;                   // dense prefill scoring: fp32 [B, Hsel, qc, total_nodes], or null
    int32_t qc;                      // query blocks per dense chunk (plane rows per selection row)
    const float* qsplit;             // dense scoring: [2, B * Hsel * nqb, D] tf32 head, then remainder
    const float* nsplit;             // dense scoring: [2, B * Hkv * total_nodes, D] likewise
    int32_t i_lo, nqc;               // the chunk being scored: query blocks [i_lo, i_lo + nqc)
    int32_t tile_off[PISA_MAX_LEVELS + 1];  // score tiles before level l (set by the launcher)
    int32_t tiles_c[PISA_MAX_LEVELS];       // node tiles of level l (set by the launcher)
};

struct AttnParams {
    const int32_t* idx;         // [B, Hsel, nqb, topk]
    __nv_bfloat16* O;           // [B, Hq, N, D]
    float* lse;                 // optional [B, Hq, N]
    uint32_t* status;
    int32_t Hq, Hkv, g, N, n0, topk, causal, per_qhead, Hsel, nqb;
    int32_t gh;                 // query heads in one CTA
    int32_t chunks;             // CTAs per (batch, selection row, query block) = heads / gh
    float scale_log2;           // softmax scale * log2(e)
};

struct DecodeParams {
    const __nv_bfloat16* Q;     // [B, Hq, 1, D]
    const __nv_bfloat16* K;     // [B, Hkv, N, D]
    const __nv_bfloat16* V;
    const int32_t* idx;         // [B, Hsel, 1, topk]
    float* part;                // [B, Hsel, splits, gh, D + 2]
    __nv_bfloat16* O;           // [B, Hq, 1, D]
    float* lse;                 // optional [B, Hq, 1]
    uint32_t* status;
    int32_t Hq, Hkv, g, N, n0, D, blk, topk, per_qhead, Hsel, gh, bps, splits;
    float scale_log2;
};

struct BwdParams {
    const __nv_bfloat16* Q;     // [B, Hq, N, D]
    const __nv_bfloat16* K;     // [B, Hkv, N, D]
    const __nv_bfloat16* V;
    const __nv_bfloat16* O;     // forward output [B, Hq, N, D]
    const __nv_bfloat16* dO;    // gradient of O
    const float* lse;           // forward LSE [B, Hq, N] (natural log)
    const int32_t* idx;         // [B, Hsel, nqb, topk]
    __nv_bfloat16* dQ;          // [B, Hq, N, D]
    __nv_bfloat16* dK;          // [B, Hkv, N, D]
    __nv_bfloat16* dV;
    float* delta;               // workspace [B, Hq, N]
    int32_t* counts;            // workspace [B, Hkv, n0 + 1]: list offsets of every key block
    int32_t* entries;           // workspace [B, Hkv, max_entries]: (query block * g + head in group)
    int32_t* rcounts;           // workspace [B, Hkv, nranges, n0]: per query-block range, then its list cursors
    uint32_t* status;
    int32_t Hq, Hkv, g, N, n0, nqb, topk, causal, per_qhead, Hsel, D, blk;
    int32_t max_entries;        // nqb * topk * g
    int32_t nranges, rsize;     // the inverse lists are filled by ranges of rsize query blocks
    float scale, scale_log2;
};

// ---------------------------------------------------------------- launchers (return false on launch error)

bool launch_block_mean(const MeanParams& p, cudaStream_t st);
bool launch_pyramid_level(const LevelParams& p, cudaStream_t st);
// Whole pyramid in two launches (adds them to *launches).
bool launch_pyramid_two_pass(const SubtreeParams& p, cudaStream_t st, int32_t* launches);
// Launches the selection; adds the kernels it launched to *launches. Prefill
// with a score plane and candidate sets of at most 1024 runs the dense scoring
// kernel and the warp descent; otherwise the one-CTA-per-row sparse descent.
bool launch_select(const SelectParams& p, int32_t batch, cudaStream_t st, int32_t* launches);
int dense_select_cap(int cap);
bool launch_select_dense(SelectParams p, int32_t batch, int cap, cudaStream_t st, int32_t* launches);
// Prefill attention: builds the tensor maps and picks the kernel variant.
pisa_status launch_attn_prefill(const Plan& pl, const void* Q, const void* K, const void* V, const AttnParams& p,
                                cudaStream_t st, int32_t* launches);
// Prefill attention with two units (neighbouring query blocks) per CTA, one per tensor-core tile,
// for units of at most 128 rows; grid as for one unit per CTA (x = query blocks).
bool launch_attn_prefill_dual(int D, int blk, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                              const AttnParams& p, dim3 grid, cudaStream_t st);
bool launch_attn_decode(const Plan& pl, const DecodeParams& p, cudaStream_t st, int32_t* launches);
bool launch_attn_backward(const BwdParams& p, int32_t batch, cudaStream_t st, int32_t* launches);
// Backward column pass (dK, dV) on the tensor cores (head dim 64 or 128, 64- or 128-key blocks:
// every shape the library accepts); false when the shape is another one or on a launch error.
bool bwd_dkdv_tc_supported(const BwdParams& p);
bool launch_bwd_dkdv_tc(const BwdParams& p, int32_t batch, cudaStream_t st);
// Backward row pass (dQ) on the tensor cores, same shapes (and K up to the prefill limit).
bool bwd_dq_tc_supported(const BwdParams& p);
bool launch_bwd_dq_tc(const BwdParams& p, int32_t batch, cudaStream_t st);
// 2-D TMA view [rows, D] of a bf16 tensor, boxes of 64 columns x box_rows rows, 128-byte swizzle.
// Raises a kernel's dynamic shared-memory limit to `bytes` on the current device, once per
// device: the attribute belongs to each device's copy of the kernel, so a process that drives
// several GPUs sets it on each. `done` holds one bit per device (devices 64 and up set it on
// every call).
bool configure_smem_once(const void* func, int bytes, std::atomic<uint64_t>& done);
bool make_tmap_2d(CUtensorMap* m, const void* ptr, int64_t rows, int D, int box_rows);
// 2-D TMA view [rows, D] of an fp32 tensor, boxes of 32 columns x 128 rows, 128-byte swizzle.
bool make_tmap_2d_f32(CUtensorMap* m, const void* ptr, int64_t rows, int D);
// Dense prefill scoring of one chunk on the tensor cores (grid: tiles, Hsel, batch).
bool launch_score_tc(const SelectParams& p, dim3 grid, cudaStream_t st);
// Splits n fp32 values (n % 4 == 0, 16-byte aligned) into a tf32 head (the 13 low mantissa bits
// cleared) and the exact fp32 remainder, for the two arrays src0 (n0 values) and src1 (n1).
bool launch_split_tf32(const float* src0, float* hi0, float* lo0, int64_t n0, const float* src1, float* hi1,
                       float* lo1, int64_t n1, cudaStream_t st);

}  // namespace pisa
