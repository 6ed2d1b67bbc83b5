// Host side of the C ABI declared in include/pisa.h: argument checks (which
// never touch the GPU), workspace layout and the launch sequence of every call.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "pisa.h"
#include "pisa_internal.h"

namespace pisa {

bool configure_smem_once(const void* func, int bytes, std::atomic<uint64_t>& done) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const uint64_t bit = dev >= 0 && dev < 64 ? (uint64_t(1) << dev) : 0;
    if (bit != 0 && (done.load(std::memory_order_acquire) & bit) != 0) return true;
    if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    done.fetch_or(bit, std::memory_order_release);
    return true;
}

static thread_local int32_t g_launches = 0;

static size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pisa_status make_plan(const pisa_shape* s, Plan* p) {
    if (s == nullptr || p == nullptr) return PISA_ERR_INVALID_ARG;
    memset(p, 0, sizeof(*p));
    if (s->batch < 1 || s->heads_q < 1 || s->heads_kv < 1 || s->seq_q < 1 || s->seq_kv < 1 || s->head_dim < 1 ||
        s->block < 1 || s->factor < 2 || s->topk < 1 || (s->causal != 0 && s->causal != 1) ||
        (s->select_per_qhead != 0 && s->select_per_qhead != 1) || !(s->scale == s->scale) ||
        (s->forced_blocks & ~(PISA_FORCE_SINK | PISA_FORCE_LOCAL)) != 0)
        return PISA_ERR_INVALID_ARG;
    if (s->heads_q % s->heads_kv != 0) return PISA_ERR_INVALID_ARG;
    if (s->seq_kv % s->block != 0) return PISA_ERR_INVALID_ARG;
    if (s->seq_q != s->seq_kv && s->seq_q != 1) return PISA_ERR_INVALID_ARG;
    const int32_t cap = s->kv_capacity == 0 ? s->seq_kv : s->kv_capacity;
    if (cap < s->seq_kv || cap % s->block != 0) return PISA_ERR_INVALID_ARG;
    if (s->seq_q != 1 && cap != s->seq_kv) return PISA_ERR_INVALID_ARG;  // capacity: decode only
    if (s->head_dim != 64 && s->head_dim != 128) return PISA_ERR_UNSUPPORTED;
    if (s->block != 64 && s->block != 128) return PISA_ERR_UNSUPPORTED;
    // every row index must fit the 32-bit TMA coordinate and grid limits
    const int64_t qrows = static_cast<int64_t>(s->batch) * s->heads_q * s->seq_q;
    const int64_t krows = static_cast<int64_t>(s->batch) * s->heads_kv * cap;
    if (qrows >= (int64_t(1) << 31) || krows >= (int64_t(1) << 31)) return PISA_ERR_UNSUPPORTED;
    if (s->batch > 65535) return PISA_ERR_UNSUPPORTED;

    p->B = s->batch;
    p->Hq = s->heads_q;
    p->Hkv = s->heads_kv;
    p->g = s->heads_q / s->heads_kv;
    p->Nq = s->seq_q;
    p->N = cap;
    p->D = s->head_dim;
    p->blk = s->block;
    p->f = s->factor;
    p->topk = s->topk;
    p->decode = s->seq_q == 1 ? 1 : 0;
    p->causal = p->decode ? 0 : s->causal;
    p->per_qhead = s->select_per_qhead;
    p->forced = s->forced_blocks;
    p->scale = s->scale > 0.f ? s->scale : 1.0f / sqrtf(static_cast<float>(s->head_dim));
    p->n0 = s->seq_kv / s->block;
    p->n0_cap = cap / s->block;

    int n = p->n0_cap, L = 0, off = 0;
    while (true) {
        if (L >= PISA_MAX_LEVELS) return PISA_ERR_UNSUPPORTED;
        p->lsize[L] = n;
        p->loff[L] = off;
        off += n;
        ++L;
        if (n <= p->f) break;
        n = (n + p->f - 1) / p->f;
    }
    p->L = L;
    p->total_nodes = off;
    if (static_cast<int64_t>(p->f) * p->topk > PISA_MAX_CANDIDATES) return PISA_ERR_UNSUPPORTED;

    p->Hsel = p->per_qhead ? p->Hq : p->Hkv;
    p->gsel = p->per_qhead ? 1 : p->g;
    p->nqb = p->decode ? 1 : p->Nq / p->blk;
    if (p->Hsel > 65535 / 16) return PISA_ERR_UNSUPPORTED;
    if (p->decode && p->gsel > 8) return PISA_ERR_UNSUPPORTED;
    if (!p->decode && p->topk > kMaxPrefillTopk) return PISA_ERR_UNSUPPORTED;

    // decode split: enough CTAs to fill the 148 SMs about four times over, at most kDecMaxBps
    // blocks per CTA (longer splits keep the copy ring streaming), at least 2
    {
        const int64_t rows = static_cast<int64_t>(p->B) * p->Hsel;
        const int64_t want = (4 * 148 + rows - 1) / rows;  // splits per row wanted
        const int64_t bps = (p->topk + want - 1) / want;
        p->dec_bps = static_cast<int32_t>(bps < 2 ? 2 : (bps > kDecMaxBps ? kDecMaxBps : bps));
    }
    p->dec_splits = p->decode ? (p->topk + p->dec_bps - 1) / p->dec_bps : 0;

    p->pyramid_bytes = static_cast<size_t>(p->B) * p->Hkv * p->total_nodes * p->D * sizeof(float);
    size_t o = kStatusBytes;
    p->ws_pyramid = o;
    o = align256(o + p->pyramid_bytes);
    p->ws_qbar = o;
    o = align256(o + static_cast<size_t>(p->B) * p->Hsel * p->nqb * p->D * sizeof(float));
    p->ws_idx = o;
    o = align256(o + static_cast<size_t>(p->B) * p->Hsel * p->nqb * p->topk * sizeof(int32_t));
    p->ws_part = o;
    if (p->decode)
        o = align256(o + static_cast<size_t>(p->B) * p->Hsel * p->dec_splits * p->gsel * (p->D + 2) * sizeof(float));
    // dense prefill scoring while its candidate count stays within a few times the sparse
    // descent's (causal rows see half the nodes on average), in chunks of query blocks whose
    // score plane fits kSelectPlaneBudget
    {
        const int64_t dense = static_cast<int64_t>(p->total_nodes) / (p->causal ? 2 : 1);
        const int64_t sparse = p->lsize[p->L - 1] + static_cast<int64_t>(p->L - 1) * p->topk * p->f;
        p->dense_select = !p->decode && p->nqb >= kDenseSelectMinQBlocks &&
                          static_cast<int64_t>(p->B) * p->Hsel * p->nqb > kSparseSelectMaxRows &&
                          dense <= static_cast<int64_t>(kDenseSelectMaxWorkRatio) * sparse;
    }
    p->ws_scores = o;
    if (p->dense_select) {
        const size_t per128 = size_t(128) * p->B * p->Hsel * p->total_nodes * sizeof(float);
        const int64_t max_qc = 128 * static_cast<int64_t>(kSelectPlaneBudget / per128 > 0 ? kSelectPlaneBudget / per128 : 1);
        const int64_t chunks = (p->nqb + max_qc - 1) / max_qc;
        const int64_t qc = chunks <= 1 ? p->nqb : ((p->nqb + chunks - 1) / chunks + 127) / 128 * 128;
        p->dense_qc = static_cast<int32_t>(qc);
        o = align256(o + static_cast<size_t>(p->B) * p->Hsel * p->dense_qc * p->total_nodes * sizeof(float));
        p->ws_split = o;
        o = align256(o + 2 * (static_cast<size_t>(p->B) * p->Hsel * p->nqb + static_cast<size_t>(p->B) * p->Hkv *
                                                                               p->total_nodes) *
                             p->D * sizeof(float));
    }
    p->ws_total = o;
    return PISA_OK;
}

// Heads of one attention CTA: the largest divisor of the shared group whose
// rows fit two 128-row tensor-core tiles (one tile for 128-key blocks, whose
// score tiles double the TMEM need).
static int heads_per_cta(const Plan& pl) {
    if (pl.per_qhead) return 1;
    const int max_rows = pl.blk == 128 ? 128 : 256;
    int best = 1;
    for (int d = 1; d <= pl.g; ++d)
        if (pl.g % d == 0 && d * pl.blk <= max_rows) best = d;
    return best;
}

// Pyramid nodes over level-0 blocks [b_lo, b_hi) (and over no block when the range is empty at
// a level), bottom-up: level-0 means of those blocks, then at every coarser level the nodes
// whose span meets the range. A full build is the range [0, n0_cap): blocks past n0 (spare
// capacity) come out as zeros.
static pisa_status pyramid_range(const Plan& pl, const void* K, float* pyr, int32_t b_lo, int32_t b_hi,
                                 cudaStream_t st) {
    if (b_hi <= b_lo) return PISA_OK;
    MeanParams m{};
    m.src = static_cast<const __nv_bfloat16*>(K);
    m.dst = pyr;
    m.Hsrc = pl.Hkv;
    m.Nsrc = pl.N;
    m.D = pl.D;
    m.Hout = pl.Hkv;
    m.row0 = b_lo;
    m.rows_out = b_hi - b_lo;
    m.rows_valid = pl.n0;
    m.dst_plane_rows = pl.total_nodes;
    m.rows_per_group = pl.blk;
    m.planes_per_group = 1;
    m.batch = pl.B;
    if (!launch_block_mean(m, st)) return PISA_ERR_CUDA;
    ++g_launches;
    int64_t width = 1;
    for (int l = 1; l < pl.L; ++l) {
        const int64_t wl = width * pl.f;
        const int32_t c_lo = static_cast<int32_t>(b_lo / wl);
        const int32_t c_hi = static_cast<int32_t>(min(static_cast<int64_t>(pl.lsize[l]), (b_hi - 1) / wl + 1));
        LevelParams lp{};
        lp.pyr = pyr;
        lp.planes = pl.B * pl.Hkv;
        lp.plane_rows = pl.total_nodes;
        lp.off_below = pl.loff[l - 1];
        lp.off_cur = pl.loff[l];
        lp.n_below = pl.lsize[l - 1];
        lp.c0 = c_lo;
        lp.n_cur = c_hi - c_lo;
        lp.n0 = pl.n0;
        lp.factor = pl.f;
        lp.D = pl.D;
        lp.width_below = width;
        if (!launch_pyramid_level(lp, st)) return PISA_ERR_CUDA;
        ++g_launches;
        width = wl;
    }
    return PISA_OK;
}

// Whole pyramid: subtrees of S = f^m key blocks (f^m <= max(64, f), m <= L - 1) formed in one
// launch, the levels above them in a second; a single-level pyramid or a factor above 64 takes
// the per-level path. Both give the same values bit for bit. (Subtrees of 16 blocks at the 128K
// workload, 1024 CTAs instead of 256, measured slower: 0.068 vs 0.062 ms for the stage.)
static pisa_status build_pyramid(const Plan& pl, const void* K, float* pyr, cudaStream_t st) {
    if (pl.L < 2 || pl.f > 64) return pyramid_range(pl, K, pyr, 0, pl.n0_cap, st);
    SubtreeParams p{};
    p.m = 1;
    p.S = pl.f;
    while (p.m + 1 <= pl.L - 1 && static_cast<int64_t>(p.S) * pl.f <= 64) {
        p.S *= pl.f;
        ++p.m;
    }
    p.K = static_cast<const __nv_bfloat16*>(K);
    p.pyr = pyr;
    p.planes = static_cast<int64_t>(pl.B) * pl.Hkv;
    p.subtrees = (pl.lsize[0] + p.S - 1) / p.S;
    if (p.planes * p.subtrees >= (int64_t(1) << 31) || p.planes >= (int64_t(1) << 31))
        return pyramid_range(pl, K, pyr, 0, pl.n0_cap, st);
    p.N = pl.N;
    p.D = pl.D;
    p.blk = pl.blk;
    p.factor = pl.f;
    p.L = pl.L;
    p.plane_rows = pl.total_nodes;
    p.n0 = pl.n0;
    for (int l = 0; l < pl.L; ++l) {
        p.lsize[l] = pl.lsize[l];
        p.loff[l] = pl.loff[l];
    }
    return launch_pyramid_two_pass(p, st, &g_launches) ? PISA_OK : PISA_ERR_CUDA;
}

static pisa_status query_summary(const Plan& pl, const void* Q, float* qbar, cudaStream_t st) {
    MeanParams m{};
    m.src = static_cast<const __nv_bfloat16*>(Q);
    m.dst = qbar;
    m.Hsrc = pl.Hq;
    m.Nsrc = pl.Nq;
    m.D = pl.D;
    m.Hout = pl.Hsel;
    m.rows_out = pl.nqb;
    m.row0 = 0;
    m.rows_valid = pl.nqb;
    m.dst_plane_rows = pl.nqb;
    m.rows_per_group = pl.decode ? 1 : pl.blk;
    m.planes_per_group = pl.gsel;
    m.batch = pl.B;
    if (!launch_block_mean(m, st)) return PISA_ERR_CUDA;
    ++g_launches;
    return PISA_OK;
}

// Decode passes the query tokens (Q) and no summaries: the descent kernel forms each row's
// summary itself. Prefill passes the summaries of query_summary.
static pisa_status select(const Plan& pl, const float* qbar, const void* Q, const float* pyr, const int32_t* budget,
                          int32_t* idx, float* margin, uint8_t* ws, cudaStream_t st) {
    uint32_t* status = reinterpret_cast<uint32_t*>(ws);
    SelectParams sp{};
    sp.qbar = qbar;
    sp.qtok = pl.decode ? static_cast<const __nv_bfloat16*>(Q) : nullptr;
    sp.Hq = pl.Hq;
    sp.qheads = pl.gsel;
    sp.pyr = pyr;
    sp.idx = idx;
    sp.margin = margin;
    sp.status = status;
    sp.Hsel = pl.Hsel;
    sp.Hkv = pl.Hkv;
    sp.gsel_div = pl.per_qhead ? pl.g : 1;
    sp.nqb = pl.nqb;
    sp.D = pl.D;
    sp.n0 = pl.n0_cap;
    sp.n0_valid = pl.n0;
    sp.factor = pl.f;
    sp.topk = pl.topk;
    sp.causal = pl.causal;
    sp.decode = pl.decode;
    sp.forced = pl.forced;
    sp.L = pl.L;
    sp.total_nodes = pl.total_nodes;
    int64_t w = 1;
    for (int l = 0; l < pl.L; ++l) {
        sp.lsize[l] = pl.lsize[l];
        sp.loff[l] = pl.loff[l];
        sp.budget[l] = budget ? budget[l] : pl.topk;
        sp.width[l] = w;
        w = w > (int64_t(1) << 40) ? w : w * pl.f;
    }
    sp.fshift = (pl.f & (pl.f - 1)) == 0 ? __builtin_ctz(static_cast<unsigned>(pl.f)) : -1;
    sp.scores = pl.dense_select ? reinterpret_cast<float*>(ws + pl.ws_scores) : nullptr;
    sp.qc = pl.dense_qc;
    if (pl.dense_select) {
        // tf32 head and remainder of the summaries and of the pyramid for the tensor-core scoring
        const int64_t nq = static_cast<int64_t>(pl.B) * pl.Hsel * pl.nqb * pl.D;
        const int64_t nn = static_cast<int64_t>(pl.B) * pl.Hkv * pl.total_nodes * pl.D;
        float* qs = reinterpret_cast<float*>(ws + pl.ws_split);
        float* ns = qs + 2 * nq;
        if (!launch_split_tf32(qbar, qs, qs + nq, nq, pyr, ns, ns + nn, nn, st)) return PISA_ERR_CUDA;
        ++g_launches;
        sp.qsplit = qs;
        sp.nsplit = ns;
    }
    if (!launch_select(sp, pl.B, st, &g_launches)) return PISA_ERR_CUDA;
    return PISA_OK;
}

static pisa_status attention(const Plan& pl, const void* Q, const void* K, const void* V, const int32_t* idx,
                             void* O, float* lse, uint8_t* ws, cudaStream_t st) {
    uint32_t* status = reinterpret_cast<uint32_t*>(ws);
    const float scale_log2 = pl.scale * 1.4426950408889634f;
    if (pl.decode) {
        DecodeParams d{};
        d.Q = static_cast<const __nv_bfloat16*>(Q);
        d.K = static_cast<const __nv_bfloat16*>(K);
        d.V = static_cast<const __nv_bfloat16*>(V);
        d.idx = idx;
        d.part = reinterpret_cast<float*>(ws + pl.ws_part);
        d.O = static_cast<__nv_bfloat16*>(O);
        d.lse = lse;
        d.status = status;
        d.Hq = pl.Hq;
        d.Hkv = pl.Hkv;
        d.g = pl.g;
        d.N = pl.N;
        d.n0 = pl.n0;
        d.D = pl.D;
        d.blk = pl.blk;
        d.topk = pl.topk;
        d.per_qhead = pl.per_qhead;
        d.Hsel = pl.Hsel;
        d.gh = pl.gsel;
        d.bps = pl.dec_bps;
        d.splits = pl.dec_splits;
        d.scale_log2 = scale_log2;
        return launch_attn_decode(pl, d, st, &g_launches) ? PISA_OK : PISA_ERR_CUDA;
    }
    AttnParams a{};
    a.idx = idx;
    a.O = static_cast<__nv_bfloat16*>(O);
    a.lse = lse;
    a.status = status;
    a.Hq = pl.Hq;
    a.Hkv = pl.Hkv;
    a.g = pl.g;
    a.N = pl.N;
    a.n0 = pl.n0;
    a.topk = pl.topk;
    a.causal = pl.causal;
    a.per_qhead = pl.per_qhead;
    a.Hsel = pl.Hsel;
    a.nqb = pl.nqb;
    a.gh = heads_per_cta(pl);
    a.chunks = pl.per_qhead ? 1 : pl.g / a.gh;
    a.scale_log2 = scale_log2;
    return launch_attn_prefill(pl, Q, K, V, a, st, &g_launches);
}

static pisa_status check_ws(const Plan& pl, const void* ws, size_t ws_bytes) {
    if (ws == nullptr || !aligned16(ws)) return PISA_ERR_INVALID_ARG;
    if (ws_bytes < pl.ws_total) return PISA_ERR_WORKSPACE;
    return PISA_OK;
}

}  // namespace pisa

bool pisa::injected_launch_failure() {
    const char* f = getenv("PISA_FAULT");
    return f != nullptr && strcmp(f, "launch") == 0;
}

using namespace pisa;

extern "C" {

int32_t pisa_num_levels(const pisa_shape* shape) {
    Plan pl;
    return make_plan(shape, &pl) == PISA_OK ? pl.L : -1;
}

pisa_status pisa_level_layout(const pisa_shape* shape, int32_t* sizes, int32_t* offsets) {
    Plan pl;
    if (sizes == nullptr || offsets == nullptr) return PISA_ERR_INVALID_ARG;
    const pisa_status s = make_plan(shape, &pl);
    if (s != PISA_OK) return s;
    for (int l = 0; l < PISA_MAX_LEVELS; ++l) {
        sizes[l] = l < pl.L ? pl.lsize[l] : 0;
        offsets[l] = l < pl.L ? pl.loff[l] : 0;
    }
    return PISA_OK;
}

pisa_status pisa_pyramid_size(const pisa_shape* shape, size_t* bytes) {
    Plan pl;
    if (bytes == nullptr) return PISA_ERR_INVALID_ARG;
    const pisa_status s = make_plan(shape, &pl);
    if (s == PISA_OK) *bytes = pl.pyramid_bytes;
    return s;
}

pisa_status pisa_workspace_size(const pisa_shape* shape, size_t* bytes) {
    Plan pl;
    if (bytes == nullptr) return PISA_ERR_INVALID_ARG;
    const pisa_status s = make_plan(shape, &pl);
    if (s == PISA_OK) *bytes = pl.ws_total;
    return s;
}

pisa_status pisa_build_pyramid(const pisa_shape* shape, const void* K, float* pyramid, pisa_stream_t stream) {
    g_launches = 0;
    Plan pl;
    const pisa_status s = make_plan(shape, &pl);
    if (s != PISA_OK) return s;
    if (K == nullptr || pyramid == nullptr || !aligned16(K) || !aligned16(pyramid)) return PISA_ERR_INVALID_ARG;
    if (injected_launch_failure()) return PISA_ERR_CUDA;
    return build_pyramid(pl, K, pyramid, reinterpret_cast<cudaStream_t>(stream));
}

pisa_status pisa_append_pyramid(const pisa_shape* shape, const void* K, float* pyramid, int32_t seq_kv_old,
                                pisa_stream_t stream) {
    g_launches = 0;
    Plan pl;
    const pisa_status s = make_plan(shape, &pl);
    if (s != PISA_OK) return s;
    if (K == nullptr || pyramid == nullptr || !aligned16(K) || !aligned16(pyramid)) return PISA_ERR_INVALID_ARG;
    if (seq_kv_old < 0 || seq_kv_old > shape->seq_kv || seq_kv_old % pl.blk != 0) return PISA_ERR_INVALID_ARG;
    if (injected_launch_failure()) return PISA_ERR_CUDA;
    return pyramid_range(pl, K, pyramid, seq_kv_old / pl.blk, pl.n0, reinterpret_cast<cudaStream_t>(stream));
}

// Backward workspace: status word, Delta [B, Hq, N] fp32, list offsets [B, Hkv, n0 + 1] int32,
// list entries [B, Hkv, nqb * topk * g] int32 and per-range counts / cursors [B, Hkv, R, n0] int32
// (the inverse lists are filled by R ranges of query blocks in parallel).
constexpr int32_t kFillRanges = 32;
struct BwdLayout {
    size_t delta, counts, entries, rcounts, total;
    int32_t max_entries, nranges, rsize;
};

static pisa_status bwd_layout(const Plan& pl, BwdLayout* w) {
    if (pl.decode) return PISA_ERR_UNSUPPORTED;
    if (pl.n0_cap != pl.n0) return PISA_ERR_INVALID_ARG;
    if (pl.n0 + 1 > (227 * 1024) / 4) return PISA_ERR_UNSUPPORTED;  // list cursors of one plane in shared memory
    const int64_t me = static_cast<int64_t>(pl.nqb) * pl.topk * pl.g;
    if (me >= (int64_t(1) << 31)) return PISA_ERR_UNSUPPORTED;
    w->max_entries = static_cast<int32_t>(me);
    size_t o = kStatusBytes;
    w->delta = o;
    o = align256(o + static_cast<size_t>(pl.B) * pl.Hq * pl.N * sizeof(float));
    w->counts = o;
    o = align256(o + static_cast<size_t>(pl.B) * pl.Hkv * (pl.n0 + 1) * sizeof(int32_t));
    w->entries = o;
    o = align256(o + static_cast<size_t>(pl.B) * pl.Hkv * me * sizeof(int32_t));
    w->rsize = (pl.nqb + kFillRanges - 1) / kFillRanges;
    w->nranges = (pl.nqb + w->rsize - 1) / w->rsize;
    w->rcounts = o;
    o = align256(o + static_cast<size_t>(pl.B) * pl.Hkv * w->nranges * pl.n0 * sizeof(int32_t));
    w->total = o;
    return PISA_OK;
}

pisa_status pisa_backward_workspace_size(const pisa_shape* shape, size_t* bytes) {
    Plan pl;
    pisa_status s = make_plan(shape, &pl);
    if (s != PISA_OK) return s;
    if (bytes == nullptr) return PISA_ERR_INVALID_ARG;
    BwdLayout w;
    if ((s = bwd_layout(pl, &w)) != PISA_OK) return s;
    *bytes = w.total;
    return PISA_OK;
}

pisa_status pisa_sparse_attention_backward(const pisa_shape* shape, const void* Q, const void* K, const void* V,
                                           const void* O, const float* lse, const void* dO, const int32_t* idx,
                                           void* dQ, void* dK, void* dV, void* ws, size_t ws_bytes,
                                           pisa_stream_t stream) {
    g_launches = 0;
    Plan pl;
    pisa_status s = make_plan(shape, &pl);
    if (s != PISA_OK) return s;
    BwdLayout w;
    if ((s = bwd_layout(pl, &w)) != PISA_OK) return s;
    const void* ptrs[] = {Q, K, V, O, lse, dO, idx, dQ, dK, dV};
    for (const void* q : ptrs)
        if (q == nullptr || !aligned16(q)) return PISA_ERR_INVALID_ARG;
    if (ws == nullptr || !aligned16(ws)) return PISA_ERR_INVALID_ARG;
    if (ws_bytes < w.total) return PISA_ERR_WORKSPACE;
    if (injected_launch_failure()) return PISA_ERR_CUDA;
    uint8_t* wb = static_cast<uint8_t*>(ws);
    BwdParams p{};
    p.Q = static_cast<const __nv_bfloat16*>(Q);
    p.K = static_cast<const __nv_bfloat16*>(K);
    p.V = static_cast<const __nv_bfloat16*>(V);
    p.O = static_cast<const __nv_bfloat16*>(O);
    p.dO = static_cast<const __nv_bfloat16*>(dO);
    p.lse = lse;
    p.idx = idx;
    p.dQ = static_cast<__nv_bfloat16*>(dQ);
    p.dK = static_cast<__nv_bfloat16*>(dK);
    p.dV = static_cast<__nv_bfloat16*>(dV);
    p.delta = reinterpret_cast<float*>(wb + w.delta);
    p.counts = reinterpret_cast<int32_t*>(wb + w.counts);
    p.entries = reinterpret_cast<int32_t*>(wb + w.entries);
    p.rcounts = reinterpret_cast<int32_t*>(wb + w.rcounts);
    p.nranges = w.nranges;
    p.rsize = w.rsize;
    p.status = reinterpret_cast<uint32_t*>(wb);
    p.Hq = pl.Hq;
    p.Hkv = pl.Hkv;
    p.g = pl.g;
    p.N = pl.N;
    p.n0 = pl.n0;
    p.nqb = pl.nqb;
    p.topk = pl.topk;
    p.causal = pl.causal;
    p.per_qhead = pl.per_qhead;
    p.Hsel = pl.Hsel;
    p.D = pl.D;
    p.blk = pl.blk;
    p.max_entries = w.max_entries;
    p.scale = pl.scale;
    p.scale_log2 = pl.scale * 1.4426950408889634f;
    if (!launch_attn_backward(p, pl.B, reinterpret_cast<cudaStream_t>(stream), &g_launches)) return PISA_ERR_CUDA;
    return PISA_OK;
}

static pisa_status check_budget(const Plan& pl, const int32_t* level_budget) {
    if (level_budget == nullptr) return PISA_OK;
    if (level_budget[0] != pl.topk) return PISA_ERR_INVALID_ARG;
    for (int l = 0; l < pl.L; ++l) {
        if (level_budget[l] < 1) return PISA_ERR_INVALID_ARG;
        if (static_cast<int64_t>(level_budget[l]) * pl.f > PISA_MAX_CANDIDATES) return PISA_ERR_UNSUPPORTED;
    }
    return PISA_OK;
}

pisa_status pisa_select_blocks(const pisa_shape* shape, const void* Q, const float* pyramid,
                               const int32_t* level_budget, int32_t* idx, float* margin, void* ws, size_t ws_bytes,
                               pisa_stream_t stream) {
    g_launches = 0;
    Plan pl;
    pisa_status s = make_plan(shape, &pl);
    if (s != PISA_OK) return s;
    if (Q == nullptr || pyramid == nullptr || idx == nullptr || !aligned16(Q) || !aligned16(pyramid) ||
        !aligned16(idx))
        return PISA_ERR_INVALID_ARG;
    if ((s = check_budget(pl, level_budget)) != PISA_OK) return s;
    if ((s = check_ws(pl, ws, ws_bytes)) != PISA_OK) return s;
    if (injected_launch_failure()) return PISA_ERR_CUDA;
    uint8_t* w = static_cast<uint8_t*>(ws);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float* qbar = reinterpret_cast<float*>(w + pl.ws_qbar);
    if (!pl.decode && (s = query_summary(pl, Q, qbar, st)) != PISA_OK) return s;
    return select(pl, qbar, Q, pyramid, level_budget, idx, margin, w, st);
}

pisa_status pisa_sparse_attention(const pisa_shape* shape, const void* Q, const void* K, const void* V,
                                  const int32_t* idx, void* O, float* lse, void* ws, size_t ws_bytes,
                                  pisa_stream_t stream) {
    g_launches = 0;
    Plan pl;
    pisa_status s = make_plan(shape, &pl);
    if (s != PISA_OK) return s;
    if (Q == nullptr || K == nullptr || V == nullptr || idx == nullptr || O == nullptr || !aligned16(Q) ||
        !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(idx))
        return PISA_ERR_INVALID_ARG;
    if ((s = check_ws(pl, ws, ws_bytes)) != PISA_OK) return s;
    if (injected_launch_failure()) return PISA_ERR_CUDA;
    return attention(pl, Q, K, V, idx, O, lse, static_cast<uint8_t*>(ws), reinterpret_cast<cudaStream_t>(stream));
}

pisa_status pisa_forward(const pisa_shape* shape, const void* Q, const void* K, const void* V, void* O, float* lse,
                         int32_t* idx_out, void* ws, size_t ws_bytes, pisa_stream_t stream) {
    g_launches = 0;
    Plan pl;
    pisa_status s = make_plan(shape, &pl);
    if (s != PISA_OK) return s;
    if (Q == nullptr || K == nullptr || V == nullptr || O == nullptr || !aligned16(Q) || !aligned16(K) ||
        !aligned16(V) || !aligned16(O) || (idx_out != nullptr && !aligned16(idx_out)))
        return PISA_ERR_INVALID_ARG;
    if ((s = check_ws(pl, ws, ws_bytes)) != PISA_OK) return s;
    if (injected_launch_failure()) return PISA_ERR_CUDA;
    uint8_t* w = static_cast<uint8_t*>(ws);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    float* pyr = reinterpret_cast<float*>(w + pl.ws_pyramid);
    float* qbar = reinterpret_cast<float*>(w + pl.ws_qbar);
    int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(w + pl.ws_idx);
    if ((s = build_pyramid(pl, K, pyr, st)) != PISA_OK) return s;
    if (!pl.decode && (s = query_summary(pl, Q, qbar, st)) != PISA_OK) return s;
    if ((s = select(pl, qbar, Q, pyr, nullptr, idx, nullptr, w, st)) != PISA_OK) return s;
    return attention(pl, Q, K, V, idx, O, lse, w, st);
}

pisa_status pisa_check_status(void* ws, uint32_t* detail, pisa_stream_t stream) {
    if (ws == nullptr) return PISA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t host[2] = {0, 0};
    if (cudaMemcpyAsync(host, ws, sizeof(host), cudaMemcpyDeviceToHost, st) != cudaSuccess) return PISA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return PISA_ERR_CUDA;
    if (host[0] != 0) {
        if (cudaMemsetAsync(ws, 0, sizeof(host), st) != cudaSuccess) return PISA_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return PISA_ERR_CUDA;
    }
    if (detail) *detail = host[1];
    return static_cast<pisa_status>(host[0]);
}

const char* pisa_status_string(pisa_status status) {
    switch (status) {
        case PISA_OK: return "ok";
        case PISA_ERR_INVALID_ARG: return "invalid argument";
        case PISA_ERR_UNSUPPORTED: return "unsupported shape";
        case PISA_ERR_WORKSPACE: return "workspace too small";
        case PISA_ERR_CUDA: return "CUDA error";
        case PISA_ERR_TIMEOUT: return "device wait timed out";
        case PISA_ERR_BAD_INDEX: return "selected block index out of range";
    }
    return "unknown status";
}

int32_t pisa_last_launch_count(void) { return g_launches; }

}  // extern "C"
