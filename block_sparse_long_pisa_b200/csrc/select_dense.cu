// Pyramid-guided top-K selection for prefill ("La selection top-K guidee par la
// pyramide", PISA page), in two kernels per chunk of query blocks.
//
// score_tc_kernel (score_tc.cu): every query-block summary of one selection
// row against every eligible node of every level the descent can visit, as
// fp32-accurate dot products on the tensor cores, 128 query blocks x 128 nodes
// per CTA. A query block at level l needs nodes c <= last / f^l, and only when
// the descent starts at l or above, so tiles entirely outside that region exit
// at once. The scores go to an fp32 plane [rows, total_nodes] in the workspace.
//
// descent_kernel: one warp per query block. It walks down from the start level
// (the coarsest whose eligible nodes outnumber its budget), reads the scores of
// its candidates, and keeps the K_l best by the same 64-bit order as the
// sparse kernel (score, then lower node index): the K_l-th largest key is found
// by bisection over the score bits with warp-wide counts (a second bisection
// over the index bits settles equal scores at the cut), then the kept nodes are
// compacted in order. Candidates are produced in ascending node order at every
// level (children of kept parents, parents ascending), so the final level-0
// list is already ascending. The node that straddles the query block is
// scored with the mean of its eligible level-0 blocks, built bottom-up.
#include <cuda_bf16.h>

#include "pisa_device.cuh"

namespace pisa {

constexpr int kScTile = 128;      // query blocks and nodes per score tile
constexpr int kDescWarps = 8;

__device__ __forceinline__ uint32_t dorder_bits(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float dorder_bits_inv(uint32_t e) {
    const uint32_t u = (e & 0x80000000u) ? (e & 0x7FFFFFFFu) : ~e;
    return __uint_as_float(u);
}

// Coarsest level whose eligible nodes outnumber its budget; -1 when every
// eligible block fits the level-0 budget.
__device__ __forceinline__ int start_level(const SelectParams& p, int64_t last) {
    for (int l = p.L - 1; l >= 0; --l)
        if (div_width(p, last, l) + 1 > p.budget[l]) return l;
    return -1;
}

template <int D, int J>
__global__ void __launch_bounds__(32 * kDescWarps) descent_kernel(const SelectParams p, int64_t rows) {
    extern __shared__ __align__(16) int32_t dsm[];
    constexpr int DL = D / 32;  // query-summary dims per lane
    constexpr uint32_t FULL = 0xFFFFFFFFu;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t prow = static_cast<int64_t>(blockIdx.x) * kDescWarps + warp;  // row of the chunk's plane
    if (prow >= rows) return;
    int32_t* kl = dsm + warp * (32 * J + PISA_MAX_LEVELS);          // kept nodes of the current level
    float* pscore = reinterpret_cast<float*>(kl + 32 * J);           // straddling-node score per level

    const int i = p.i_lo + static_cast<int>(prow % p.nqc);
    const int hs = static_cast<int>((prow / p.nqc) % p.Hsel);
    const int b = static_cast<int>(prow / (static_cast<int64_t>(p.nqc) * p.Hsel));
    const int64_t row = (static_cast<int64_t>(b) * p.Hsel + hs) * p.nqb + i;  // selection row
    const int kvh = hs / p.gsel_div;
    const int64_t last = p.causal ? i : p.n0_valid - 1;
    int32_t* dst = p.idx + row * p.topk;
    const int l0 = start_level(p, last);
    if (l0 < 0) {  // every eligible block fits the budget
        for (int t = lane; t < p.topk; t += 32) dst[t] = t <= last ? t : -1;
        if (p.margin != nullptr && lane == 0) p.margin[row] = __int_as_float(0x7F800000);
        return;
    }

    // scores of the straddling nodes, levels 1..l0 (level 0 never straddles)
    if (l0 >= 1) {
        const float* plane = p.pyr + (static_cast<int64_t>(b) * p.Hkv + kvh) * p.total_nodes * D;
        float q[DL], sum[DL];
#pragma unroll
        for (int e = 0; e < DL; ++e) {
            q[e] = p.qbar[row * D + lane * DL + e];
            sum[e] = plane[(p.loff[0] + last) * D + lane * DL + e];
        }
        for (int l = 1; l <= l0; ++l) {
            const int64_t wl = p.width[l], wb = p.width[l - 1];
            const int64_t c_l = div_width(p, last, l), c_b = div_width(p, last, l - 1);
            for (int64_t c = c_l * p.factor; c < c_b; ++c) {
                const float* v = plane + (p.loff[l - 1] + c) * D + lane * DL;
#pragma unroll
                for (int e = 0; e < DL; ++e) sum[e] += static_cast<float>(wb) * v[e];
            }
            const float cnt = static_cast<float>(last - c_l * wl + 1);
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < DL; ++e) s = fmaf(q[e], sum[e] / cnt, s);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
            if (lane == 0) pscore[l] = s;
        }
        __syncwarp();
    }

    const float* srow = p.scores + ((static_cast<int64_t>(b) * p.Hsel + hs) * p.qc + (i - p.i_lo)) * p.total_nodes;
    const uint32_t lt_mask = (1u << lane) - 1u;
    // forced blocks (sink, local): not candidates at level 0, added to the output at the end
    int32_t f0, f1;
    const int nf = forced_blocks(p.forced, i, p.budget[0], f0, f1);
    float margin = __int_as_float(0x7F800000);
    int32_t node[J];
    {
        const int64_t cnt0 = div_width(p, last, l0) + 1;
#pragma unroll
        for (int j = 0; j < J; ++j) node[j] = 32 * j + lane < cnt0 ? 32 * j + lane : -1;
    }
    for (int l = l0;; --l) {
        if (l == 0 && nf > 0) {
#pragma unroll
            for (int j = 0; j < J; ++j)
                if (node[j] == f0 || node[j] == f1) node[j] = -1;
        }
        const int64_t c_part = div_width(p, last, l);
        const bool has_part = min((c_part + 1) * p.width[l], static_cast<int64_t>(p.n0)) - 1 > last;
        const float ps = has_part ? pscore[l] : 0.f;
        uint32_t hi[J];
        int nv = 0;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const bool v = node[j] >= 0;
            const float s = v ? ((has_part && node[j] == c_part) ? ps : srow[p.loff[l] + node[j]]) : 0.f;
            hi[j] = v ? dorder_bits(s) : 0u;
            nv += v;
        }
        const int nvalid = __reduce_add_sync(FULL, nv);
        const int K = l == 0 ? p.budget[0] - nf : p.budget[l];
        // kept: hi > t_hi, or hi == t_hi and ~node >= t_lo; invalid candidates have hi == 0
        uint32_t t_hi = 1u, t_lo = 0u;
        if (K > 0 && nvalid > K) {
            // MSB-first bisection for the K-th largest score bits; it stops as soon as a
            // tested threshold keeps exactly K candidates (the cut then falls between
            // two distinct scores), which takes about log2(candidates) + a few steps
            uint32_t T = 0u;
            bool exact = false;
            for (int bit = 31; bit >= 0; --bit) {
                const uint32_t cand = T | (1u << bit);
                int c = 0;
#pragma unroll
                for (int j = 0; j < J; ++j) c += hi[j] >= cand;
                const int tot = __reduce_add_sync(FULL, c);
                if (tot >= K) {
                    T = cand;
                    if (tot == K) {
                        exact = true;
                        break;
                    }
                }
            }
            t_hi = T;
            float rel;
            if (exact) {
                uint32_t kmin = 0xFFFFFFFFu, below = 0u;
#pragma unroll
                for (int j = 0; j < J; ++j) {
                    if (hi[j] >= T) kmin = min(kmin, hi[j]);
                    else below = max(below, hi[j]);
                }
                const float a = dorder_bits_inv(__reduce_min_sync(FULL, kmin));
                const float c = dorder_bits_inv(__reduce_max_sync(FULL, below));
                rel = (a - c) / fmaxf(fmaxf(fabsf(a), fabsf(c)), 1e-30f);
            } else {
                // T is the K-th largest score and equal scores straddle the cut:
                // lower node indices (larger inverted index) win
                int gt = 0;
#pragma unroll
                for (int j = 0; j < J; ++j) gt += hi[j] > T;
                const int need = K - __reduce_add_sync(FULL, gt);
                uint32_t U = 0u;
                for (int bit = 31; bit >= 0; --bit) {
                    const uint32_t cand = U | (1u << bit);
                    int c = 0;
#pragma unroll
                    for (int j = 0; j < J; ++j) c += (hi[j] == T) && (~static_cast<uint32_t>(node[j]) >= cand);
                    const int tot = __reduce_add_sync(FULL, c);
                    if (tot >= need) {
                        U = cand;
                        if (tot == need) break;
                    }
                }
                t_lo = U;
                rel = 0.f;
            }
            margin = fminf(margin, rel);
        }
        // order-preserving compaction of the kept nodes
        int nkeep = 0;
#pragma unroll
        for (int j = 0; j < J; ++j) {
            // (K == 0: every slot of the level is taken by forced blocks, no candidate is kept)
            const bool keep = K > 0 && (hi[j] > t_hi || (hi[j] == t_hi && ~static_cast<uint32_t>(node[j]) >= t_lo));
            const uint32_t bal = __ballot_sync(FULL, keep);
            if (keep) kl[nkeep + __popc(bal & lt_mask)] = node[j];
            nkeep += __popc(bal);
        }
        __syncwarp();
        if (l == 0) {
            // merge the forced blocks into the ascending list of kept blocks (none of them is kept)
            int below0 = 0, below1 = 0;
            for (int t = lane; t < nkeep; t += 32) {
                const int32_t v = kl[t];
                dst[t + (nf >= 1 && f0 < v) + (nf >= 2 && f1 < v)] = v;
                below0 += v < f0;
                below1 += v < f1;
            }
            below0 = __reduce_add_sync(FULL, below0);
            below1 = __reduce_add_sync(FULL, below1);
            if (lane == 0) {
                if (nf >= 1) dst[below0] = f0;
                if (nf >= 2) dst[below1 + 1] = f1;
            }
            for (int t = nkeep + nf + lane; t < p.topk; t += 32) dst[t] = -1;
            if (p.margin != nullptr && lane == 0) p.margin[row] = margin;
            return;
        }
        const int64_t last_below = div_width(p, last, l - 1);
        const int n_below = p.lsize[l - 1];
#pragma unroll
        for (int j = 0; j < J; ++j) {
            const int t = 32 * j + lane;
            const int r = div_factor(p, t);
            int32_t ch = -1;
            if (r < nkeep) {
                const int64_t c = static_cast<int64_t>(kl[r]) * p.factor + (t - r * p.factor);
                if (c <= last_below && c < n_below) ch = static_cast<int32_t>(c);
            }
            node[j] = ch;
        }
        __syncwarp();  // kl is rewritten at the next level
    }
}

template <int D, int J>
static bool launch_descent(const SelectParams& p, int64_t rows, cudaStream_t st) {
    const size_t smem = static_cast<size_t>(kDescWarps) * (32 * J + PISA_MAX_LEVELS) * sizeof(int32_t);
    const unsigned grid = static_cast<unsigned>((rows + kDescWarps - 1) / kDescWarps);
    descent_kernel<D, J><<<grid, 32 * kDescWarps, smem, st>>>(p, rows);
    return cudaGetLastError() == cudaSuccess;
}

int dense_select_cap(int cap) { return cap <= 32 * 8 ? 256 : cap <= 32 * 16 ? 512 : cap <= 32 * 32 ? 1024 : 0; }

bool launch_select_dense(SelectParams p, int32_t batch, int cap, cudaStream_t st, int32_t* launches) {
    const int J = dense_select_cap(cap) / 32;
    // query blocks in chunks of qc: each chunk is scored into the plane, then descended
    for (p.i_lo = 0; p.i_lo < p.nqb; p.i_lo += p.qc) {
        p.nqc = min(p.qc, p.nqb - p.i_lo);
        int tiles = 0;
        for (int l = 0; l < p.L; ++l) {
            p.tile_off[l] = tiles;
            p.tiles_c[l] = (p.lsize[l] + kScTile - 1) / kScTile;
            tiles += ((p.nqc + kScTile - 1) / kScTile) * p.tiles_c[l];
        }
        p.tile_off[p.L] = tiles;
        dim3 grid(tiles, p.Hsel, batch);
        if (!launch_score_tc(p, grid, st)) return false;
        const int64_t rows = static_cast<int64_t>(batch) * p.Hsel * p.nqc;
        bool ok;
        if (p.D == 64)
            ok = J == 8 ? launch_descent<64, 8>(p, rows, st)
                        : (J == 16 ? launch_descent<64, 16>(p, rows, st) : launch_descent<64, 32>(p, rows, st));
        else
            ok = J == 8 ? launch_descent<128, 8>(p, rows, st)
                        : (J == 16 ? launch_descent<128, 16>(p, rows, st) : launch_descent<128, 32>(p, rows, st));
        if (!ok) return false;
        *launches += 2;
    }
    return true;
}

}  // namespace pisa
