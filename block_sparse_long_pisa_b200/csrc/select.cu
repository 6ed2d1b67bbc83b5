// Pyramid-guided top-K selection ("La selection top-K guidee par la pyramide",
// PISA page). One CTA of 128 threads per (batch, selection row, query block).
//
// 1. Each lane holds its slice of the query summary, loaded from global memory
//    alongside the first nodes: for prefill the fp32 summary the pooling kernel
//    computed; for decode the kernel forms it from the row's query tokens (the
//    same fp32 arithmetic, so no separate summary launch).
// 2. Causal: the node that straddles the query block at each level is
//    summarised by the mean of its eligible level-0 blocks, built bottom-up
//    from the pyramid (full children left of the straddling child, plus the
//    straddling child's own partial sum), so no future key enters a score.
//    When no level has such a node (decode over a whole cache whose length is
//    a multiple of every level's width, for one) the step is skipped.
// 3. The descent starts at the coarsest level whose eligible nodes outnumber
//    that level's budget: every level above it keeps all its nodes, so its
//    children are exactly the eligible nodes of this level, and skipping the
//    coarser scores changes nothing.
// 4. At each level every candidate gets an fp32 dot product with the query
//    summary (eight lanes per candidate, so each warp load covers four whole
//    128-byte lines of node vectors; a three-step shuffle adds the lanes). The
//    16 groups of eight lanes issue the loads of four candidates each before
//    any arithmetic. (Measured at 64 sequences x 8 KV heads over 128K keys:
//    CTAs of 256 or 512 threads, which score a level in fewer rounds, take
//    1.3x and 2x as long, since fewer of them are resident per SM.) Candidates are ranked by
//    a 64-bit key (order-preserving score bits, then inverted node index): higher score first
//    and, on equal scores, lower index. One warp finds the K_l-th largest key by bisection with
//    warp-wide counts, stopping as soon as a threshold keeps exactly K_l candidates (the score
//    word first, the index word only when scores tie at the cut;
//    a CTA barrier per step costs several hundred cycles here) and compacts the kept
//    candidates in candidate order. Candidates are produced in
//    ascending node order at every level (the first scored level's eligible nodes, then the
//    children of the kept parents, parents ascending), so every kept list is ascending; holes
//    (ineligible children) carry key 0 and are never kept.
// 5. The kept level-0 blocks are written in ascending order, padded with -1.
//    Forced blocks (sink, local) are left out of the level-0 candidates, which
//    then keep K minus their count, and are merged into the ascending output.
#include <cuda_bf16.h>

#include "pisa_device.cuh"

namespace pisa {

constexpr int kSelThreads = 128;
// Candidates one group of eight lanes scores per loop trip (all their loads are issued first).
constexpr int kSelBatch = 4;

__device__ __forceinline__ uint32_t order_bits(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float order_bits_inv(uint32_t e) {
    const uint32_t u = (e & 0x80000000u) ? (e & 0x7FFFFFFFu) : ~e;
    return __uint_as_float(u);
}

__device__ __forceinline__ uint64_t rank_key(float s, int32_t node) {
    return (static_cast<uint64_t>(order_bits(s + 0.0f)) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(node));
}

__device__ __forceinline__ int32_t key_node(uint64_t k) {
    return static_cast<int32_t>(~static_cast<uint32_t>(k & 0xFFFFFFFFull));
}

__device__ __forceinline__ int next_pow2(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

template <int D>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const SelectParams p, int cap) {
    extern __shared__ __align__(16) uint8_t sm[];
    uint64_t* keys = reinterpret_cast<uint64_t*>(sm);                         // [cap]
    int32_t* cand = reinterpret_cast<int32_t*>(keys + cap);                    // [cap]
    int32_t* kept = cand + cap;                                                // [cap]
    float* part = reinterpret_cast<float*>(kept + cap);                        // [L][D]
    __shared__ int s_nvalid;
    __shared__ float s_margin;
    __shared__ int s_scan[1];   // kept count of the level

    const int i = blockIdx.x, hs = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x;
    const int kvh = hs / p.gsel_div;
    const int last = (p.causal && !p.decode) ? i : p.n0_valid - 1;
    const float* plane = p.pyr + (static_cast<int64_t>(b) * p.Hkv + kvh) * p.total_nodes * D;
    const int64_t row = (static_cast<int64_t>(b) * p.Hsel + hs) * p.nqb + i;

    // this lane's slice of the query summary: dims 32k + 4*sub .. +3 (its loads overlap the rest
    // of the set-up and the first level's node loads)
    const int sub = tid & 7;
    float4 qv[D / 32];
    if (p.qtok != nullptr) {
        // decode: the summary is the mean of the row's heads' tokens, formed here in the fp32 order
        // of block_mean_kernel (a running sum over the heads from zero, the +0 its lane reduction
        // adds, one multiply by the reciprocal of the head count), so it is the same bit for bit
        const float inv = 1.0f / static_cast<float>(p.qheads);
        const __nv_bfloat16* q0 =
            p.qtok + (static_cast<int64_t>(b) * p.Hq + static_cast<int64_t>(hs) * p.qheads) * D + 4 * sub;
#pragma unroll
        for (int k = 0; k < D / 32; ++k) {
            float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
            for (int h = 0; h < p.qheads; ++h) {
                const uint2 w = *reinterpret_cast<const uint2*>(q0 + static_cast<int64_t>(h) * D + 32 * k);
                a0 += __uint_as_float(w.x << 16);
                a1 += __uint_as_float(w.x & 0xFFFF0000u);
                a2 += __uint_as_float(w.y << 16);
                a3 += __uint_as_float(w.y & 0xFFFF0000u);
            }
            qv[k] = make_float4((a0 + 0.0f) * inv, (a1 + 0.0f) * inv, (a2 + 0.0f) * inv, (a3 + 0.0f) * inv);
        }
    } else {
#pragma unroll
        for (int k = 0; k < D / 32; ++k) qv[k] = *reinterpret_cast<const float4*>(p.qbar + row * D + 32 * k + 4 * sub);
    }
    // partial (straddling) node summaries, bottom-up, where some level has a partial node
    bool any_part = false;
    for (int l = 1; l < p.L; ++l) {
        const int64_t c_part = div_width(p, last, l);
        any_part |= min((c_part + 1) * p.width[l], static_cast<int64_t>(p.n0)) - 1 > last;
    }
    for (int d = tid; any_part && d < D; d += kSelThreads) {
        float sum = plane[static_cast<int64_t>(p.loff[0] + last) * D + d];
        for (int l = 1; l < p.L; ++l) {
            const int64_t wl = p.width[l], wb = p.width[l - 1];
            const int64_t c_l = div_width(p, last, l), c_b = div_width(p, last, l - 1);
            // at most f-1 full children precede the straddling one; load them together
            float ch[8];
            const int nch = static_cast<int>(c_b - c_l * p.factor);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                ch[u] = u < nch ? plane[(p.loff[l - 1] + c_l * p.factor + u) * D + d] : 0.f;
            for (int u = 8; u < nch; ++u)
                sum += static_cast<float>(wb) * plane[(p.loff[l - 1] + c_l * p.factor + u) * D + d];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (u < nch) sum += static_cast<float>(wb) * ch[u];
            part[l * D + d] = sum / static_cast<float>(last - c_l * wl + 1);
        }
    }
    if (tid == 0) s_margin = __int_as_float(0x7F800000);  // +inf
    __syncthreads();

    // coarsest level whose eligible nodes exceed its budget
    int l0 = -1;
    for (int l = p.L - 1; l >= 0; --l) {
        if (div_width(p, last, l) + 1 > p.budget[l]) {
            l0 = l;
            break;
        }
    }
    int32_t f0, f1;
    const int nf = forced_blocks(p.forced, p.decode ? p.n0_valid - 1 : i, p.budget[0], f0, f1);
    int32_t* dst = p.idx + row * p.topk;
    const int warp = tid >> 5, lane = tid & 31;
    if (l0 < 0) {
        // every eligible block fits the budget (the forced ones among them)
        const int nkeep = last + 1;
        for (int t = tid; t < p.topk; t += kSelThreads) dst[t] = t < nkeep ? t : -1;
    } else {
        int ncand = static_cast<int>(div_width(p, last, l0) + 1);
        // at level 0 the forced blocks (all eligible) are not candidates
        for (int t = tid; t < ncand; t += kSelThreads) cand[t] = (l0 == 0 && (t == f0 || t == f1)) ? -1 : t;
        if (tid == 0) s_nvalid = l0 == 0 ? ncand - nf : ncand;
        __syncthreads();
        for (int l = l0; l >= 0; --l) {
            const int n = next_pow2(ncand);
            const int64_t c_part = div_width(p, last, l);
            const bool has_part = min((c_part + 1) * p.width[l], static_cast<int64_t>(p.n0)) - 1 > last;
            // 8 lanes per candidate: each warp load instruction covers four whole 128-byte lines;
            // each group issues the loads of kSelBatch candidates before any arithmetic
            constexpr int GROUPS = kSelThreads / 8;
            for (int t0 = 0; t0 < n; t0 += GROUPS * kSelBatch) {
                float4 x[kSelBatch][D / 32];
                int32_t cb[kSelBatch];
                bool live[kSelBatch];
#pragma unroll
                for (int j = 0; j < kSelBatch; ++j) {
                    const int t = t0 + j * GROUPS + (tid >> 3);
                    live[j] = t < ncand && cand[t] >= 0;
                    cb[j] = live[j] ? cand[t] : 0;
                    const float* v = (has_part && cb[j] == c_part) ? part + l * D
                                                                  : plane + static_cast<int64_t>(p.loff[l] + cb[j]) * D;
#pragma unroll
                    for (int k = 0; k < D / 32; ++k)
                        x[j][k] = live[j] ? *reinterpret_cast<const float4*>(v + 32 * k + 4 * sub)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int j = 0; j < kSelBatch; ++j) {
                    float acc = 0.f;
#pragma unroll
                    for (int k = 0; k < D / 32; ++k) {
                        acc = fmaf(qv[k].x, x[j][k].x, acc);
                        acc = fmaf(qv[k].y, x[j][k].y, acc);
                        acc = fmaf(qv[k].z, x[j][k].z, acc);
                        acc = fmaf(qv[k].w, x[j][k].w, acc);
                    }
                    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 4);
                    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 2);
                    acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 1);
                    const int t = t0 + j * GROUPS + (tid >> 3);
                    if (sub == 0 && t < n) keys[t] = live[j] ? rank_key(acc, cb[j]) : 0ull;
                }
            }
            __syncthreads();
            const int nvalid = s_nvalid;
            const int k_l = l == 0 ? p.budget[0] - nf : p.budget[l];
            // warp 0 selects: counts by warp reductions, no CTA barrier per bisection step
            if (warp == 0) {
                // this lane's candidates form one contiguous run, so the compaction keeps their order
                const int per = (ncand + 31) / 32;
                const int s0 = min(ncand, lane * per), s1 = min(ncand, s0 + per);
                // kept: key >= (th_hi, th_lo) as (score word, index word); (0, 1) keeps every valid
                // key (a valid key's score word is never 0; a hole's key is 0)
                uint32_t th_hi = 0, th_lo = 1;
                if (nvalid > k_l && k_l <= 0) {
                    th_hi = 0xFFFFFFFFu;  // nothing is kept (finite scores never reach this word)
                    th_lo = 0xFFFFFFFFu;
                } else if (nvalid > k_l) {
                    // score-word threshold of the K_l-th largest key by MSB-first bisection: the
                    // largest h with at least K_l words >= h, or, as soon as a tested h keeps
                    // exactly K_l words, that h (the cut then falls between two distinct scores)
                    th_hi = 0;
                    for (int bit = 31; bit >= 0; --bit) {
                        const uint32_t c = th_hi | (1u << bit);
                        int cnt = 0;
                        for (int t = s0; t < s1; ++t) cnt += static_cast<uint32_t>(keys[t] >> 32) >= c;
                        const int tot = static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, cnt));
                        if (tot >= k_l) {
                            th_hi = c;
                            if (tot == k_l) break;
                        }
                    }
                    int gt = 0, eq = 0;
                    uint32_t below = 0;            // largest score word under th_hi: the (K_l+1)-th score if no tie
                    uint32_t kept_min = 0xFFFFFFFFu;  // smallest score word at or above th_hi: the K_l-th score
                    for (int t = s0; t < s1; ++t) {
                        const uint32_t h = static_cast<uint32_t>(keys[t] >> 32);
                        gt += h > th_hi;
                        eq += h == th_hi;
                        if (h < th_hi)
                            below = max(below, h);
                        else
                            kept_min = min(kept_min, h);
                    }
                    gt = static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, gt));
                    eq = static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, eq));
                    below = __reduce_max_sync(0xFFFFFFFFu, below);
                    kept_min = __reduce_min_sync(0xFFFFFFFFu, kept_min);
                    const int need = k_l - gt;  // kept among the keys whose score word is th_hi
                    th_lo = 0;
                    if (eq > need) {
                        // equal scores at the cut: the `need` largest index words (lower nodes)
                        for (int bit = 31; bit >= 0; --bit) {
                            const uint32_t c = th_lo | (1u << bit);
                            int cnt = 0;
                            for (int t = s0; t < s1; ++t) {
                                const uint64_t key = keys[t];
                                cnt += static_cast<uint32_t>(key >> 32) == th_hi && static_cast<uint32_t>(key) >= c;
                            }
                            if (static_cast<int>(__reduce_add_sync(0xFFFFFFFFu, cnt)) >= need) th_lo = c;
                        }
                        below = th_hi;  // the (K_l+1)-th score equals the K_l-th
                    }
                    if (lane == 0) {
                        const float a = order_bits_inv(kept_min);
                        const float c = order_bits_inv(below);
                        const float rel = (a - c) / fmaxf(fmaxf(fabsf(a), fabsf(c)), 1e-30f);
                        s_margin = fminf(s_margin, rel);
                    }
                }
                const uint64_t th = (static_cast<uint64_t>(th_hi) << 32) | th_lo;
                // stable compaction of the kept candidates
                int mine = 0;
                for (int t = s0; t < s1; ++t) mine += keys[t] >= th;
                int incl = mine;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                    if (lane >= o) incl += y;
                }
                int pos = incl - mine;
                for (int t = s0; t < s1; ++t)
                    if (keys[t] >= th) kept[pos++] = cand[t];
                if (lane == 31) s_scan[0] = incl;  // how many are kept
            }
            __syncthreads();  // kept[] complete; s_nvalid read by every thread
            const int nkeep = s_scan[0];
            if (l > 0) {
                // the next candidates: children of the kept parents, parents ascending
                const int64_t last_below = div_width(p, last, l - 1);
                const int n_below = p.lsize[l - 1];
                const int slots = nkeep * p.factor;
                if (tid == 0) s_nvalid = 0;
                __syncthreads();
                int valid_here = 0;
                for (int t = tid; t < slots; t += kSelThreads) {
                    const int r = div_factor(p, t);
                    const int32_t c = kept[r];
                    const int64_t ch = static_cast<int64_t>(c) * p.factor + (t - r * p.factor);
                    const bool ok = ch <= last_below && ch < n_below && (l > 1 || (ch != f0 && ch != f1));
                    cand[t] = ok ? static_cast<int32_t>(ch) : -1;
                    valid_here += ok;
                }
                if (valid_here) atomicAdd(&s_nvalid, valid_here);
                ncand = slots;
                __syncthreads();
            } else {
                // the ascending kept blocks with the forced ones merged in, padded with -1
                for (int t = tid; t < nkeep; t += kSelThreads) {
                    const int32_t v = kept[t];
                    dst[t + (f0 >= 0 && f0 < v) + (f1 >= 0 && f1 < v)] = v;
                }
                if (tid < 2) {
                    const int32_t f = tid == 0 ? f0 : f1, other = tid == 0 ? f1 : f0;
                    if (f >= 0) {
                        int lo = 0, hi = nkeep;  // kept blocks below f
                        while (lo < hi) {
                            const int mid = (lo + hi) >> 1;
                            if (kept[mid] < f)
                                lo = mid + 1;
                            else
                                hi = mid;
                        }
                        dst[lo + (other >= 0 && other < f)] = f;
                    }
                }
                for (int t = nkeep + nf + tid; t < p.topk; t += kSelThreads) dst[t] = -1;
            }
        }
    }
    if (p.margin != nullptr && tid == 0) p.margin[row] = s_margin;
}

bool launch_select(const SelectParams& p, int32_t batch, cudaStream_t st, int32_t* launches) {
    int maxb = 1;
    for (int l = 0; l < p.L; ++l) maxb = max(maxb, p.budget[l]);
    int cap = 1;
    while (cap < max(p.factor * maxb, p.lsize[p.L - 1])) cap <<= 1;
    if (cap < 4) cap = 4;  // keeps the fp32 partial-node rows 16-byte aligned
    if (p.scores != nullptr && !p.decode && dense_select_cap(cap) > 0) return launch_select_dense(p, batch, cap, st, launches);
    *launches += 1;
    const size_t smem = static_cast<size_t>(cap) * (sizeof(uint64_t) + 2 * sizeof(int32_t)) +
                        static_cast<size_t>(p.D) * p.L * sizeof(float);
    dim3 grid(p.nqb, p.Hsel, batch);
    if (p.D == 64) {
        cudaFuncSetAttribute(select_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        select_kernel<64><<<grid, kSelThreads, smem, st>>>(p, cap);
    } else {
        cudaFuncSetAttribute(select_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        select_kernel<128><<<grid, kSelThreads, smem, st>>>(p, cap);
    }
    return cudaGetLastError() == cudaSuccess;
}

}  // namespace pisa
