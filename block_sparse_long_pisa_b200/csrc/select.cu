// Pyramid-guided top-K selection ("La selection top-K guidee par la pyramide",
// PISA page). One CTA of 128 threads per (batch, selection row, query block).
//
// 1. The query summary (fp32, computed by the pooling kernel) goes to shared
//    memory.
// 2. Causal: the node that straddles the query block at each level is
//    summarised by the mean of its eligible level-0 blocks, built bottom-up
//    from the pyramid (full children left of the straddling child, plus the
//    straddling child's own partial sum), so no future key enters a score.
// 3. The descent starts at the coarsest level whose eligible nodes outnumber
//    that level's budget: every level above it keeps all its nodes, so its
//    children are exactly the eligible nodes of this level, and skipping the
//    coarser scores changes nothing.
// 4. At each level every candidate gets an fp32 dot product with the query
//    summary (eight lanes per candidate, so each warp load covers four whole
//    128-byte lines of node vectors; a three-step shuffle adds the lanes). Candidates are ranked by
//    a 64-bit key (order-preserving score bits, then inverted node index), so
//    that a bitonic sort in shared memory orders by higher score and, on equal
//    scores, lower index. The kept nodes' eligible children become the next
//    candidates; holes (ineligible children) carry key 0 and sort last.
// 5. The kept level-0 blocks are written in ascending order, padded with -1.
//    Forced blocks (sink, local) are left out of the level-0 candidates, which
//    then keep K minus their count, and join the output before the final sort.
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

// Sorts keys[0, n) in descending order; n is a power of two.
__device__ void bitonic_desc(uint64_t* keys, int n) {
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int t = threadIdx.x; t < n; t += kSelThreads) {
                const int u = t ^ j;
                if (u > t) {
                    const uint64_t a = keys[t], b = keys[u];
                    const bool desc = (t & k) == 0;
                    if (desc ? (a < b) : (a > b)) {
                        keys[t] = b;
                        keys[u] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
}

// Sorts ints[0, n) ascending; n is a power of two.
__device__ void bitonic_asc(int32_t* v, int n) {
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int t = threadIdx.x; t < n; t += kSelThreads) {
                const int u = t ^ j;
                if (u > t) {
                    const int32_t a = v[t], b = v[u];
                    const bool asc = (t & k) == 0;
                    if (asc ? (a > b) : (a < b)) {
                        v[t] = b;
                        v[u] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
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
    float* qs = reinterpret_cast<float*>(cand + cap);                          // [D]
    float* part = qs + D;                                                      // [L][D]
    __shared__ int s_nvalid;
    __shared__ float s_margin;

    const int i = blockIdx.x, hs = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x;
    const int kvh = hs / p.gsel_div;
    const int last = (p.causal && !p.decode) ? i : p.n0_valid - 1;
    const float* plane = p.pyr + (static_cast<int64_t>(b) * p.Hkv + kvh) * p.total_nodes * D;
    const int64_t row = (static_cast<int64_t>(b) * p.Hsel + hs) * p.nqb + i;

    for (int d = tid; d < D; d += kSelThreads) qs[d] = p.qbar[row * D + d];
    // partial (straddling) node summaries, bottom-up
    for (int d = tid; d < D; d += kSelThreads) {
        float sum = plane[static_cast<int64_t>(p.loff[0] + last) * D + d];
        for (int l = 1; l < p.L; ++l) {
            const int64_t wl = p.width[l], wb = p.width[l - 1];
            const int64_t c_l = last / wl, c_b = last / wb;
            // at most f-1 full children precede the straddling one; load them together
            float ch[8];
            const int nch = static_cast<int>(c_b - c_l * p.factor);
#pragma unroll
            for (int u = 0; u < 8; ++u)
                ch[u] = u < nch ? plane[(p.loff[l - 1] + c_l * p.factor + u) * D + d] : 0.f;
            for (int u = 8; u < nch; ++u) sum += static_cast<float>(wb) * plane[(p.loff[l - 1] + c_l * p.factor + u) * D + d];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (u < nch) sum += static_cast<float>(wb) * ch[u];
            part[l * D + d] = sum / static_cast<float>(last - c_l * wl + 1);
        }
    }
    if (tid == 0) s_margin = __int_as_float(0x7F800000);  // +inf
    __syncthreads();
    // this lane's slice of the query summary: dims 32k + 4*sub .. +3
    const int sub = tid & 7;
    float4 qv[D / 32];
#pragma unroll
    for (int k = 0; k < D / 32; ++k) qv[k] = *reinterpret_cast<const float4*>(qs + 32 * k + 4 * sub);

    // coarsest level whose eligible nodes exceed its budget
    int l0 = -1;
    for (int l = p.L - 1; l >= 0; --l) {
        if (last / p.width[l] + 1 > p.budget[l]) {
            l0 = l;
            break;
        }
    }
    int nkeep;
    int32_t* out_ids = cand;  // reused for the final ascending sort
    int32_t f0, f1;
    const int nf = forced_blocks(p.forced, p.decode ? p.n0_valid - 1 : i, p.budget[0], f0, f1);
    if (l0 < 0) {
        nkeep = last + 1;  // every eligible block fits the budget
        const int n = next_pow2(nkeep);
        for (int t = tid; t < n; t += kSelThreads) out_ids[t] = t < nkeep ? t : 0x7FFFFFFF;
        __syncthreads();
    } else {
        int ncand = static_cast<int>(last / p.width[l0] + 1);
        // at level 0 the forced blocks (all eligible) are not candidates
        for (int t = tid; t < ncand; t += kSelThreads) cand[t] = (l0 == 0 && (t == f0 || t == f1)) ? -1 : t;
        if (tid == 0) s_nvalid = l0 == 0 ? ncand - nf : ncand;
        __syncthreads();
        nkeep = 0;
        for (int l = l0; l >= 0; --l) {
            const int n = next_pow2(ncand);
            const int64_t c_part = last / p.width[l];
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
            bitonic_desc(keys, n);
            const int k_l = l == 0 ? p.budget[0] - nf : p.budget[l];
            nkeep = min(k_l, nvalid);
            if (tid == 0 && nvalid > k_l && k_l > 0) {
                const float a = order_bits_inv(static_cast<uint32_t>(keys[k_l - 1] >> 32));
                const float c = order_bits_inv(static_cast<uint32_t>(keys[k_l] >> 32));
                const float rel = (a - c) / fmaxf(fmaxf(fabsf(a), fabsf(c)), 1e-30f);
                s_margin = fminf(s_margin, rel);
            }
            if (l > 0) {
                const int64_t last_below = last / p.width[l - 1];
                const int n_below = p.lsize[l - 1];
                const int slots = nkeep * p.factor;
                __syncthreads();  // every thread has read s_nvalid
                if (tid == 0) s_nvalid = 0;
                __syncthreads();
                int mine = 0;
                for (int t = tid; t < slots; t += kSelThreads) {
                    const int32_t c = key_node(keys[t / p.factor]);
                    const int64_t ch = static_cast<int64_t>(c) * p.factor + (t % p.factor);
                    const bool ok = ch <= last_below && ch < n_below && (l > 1 || (ch != f0 && ch != f1));
                    cand[t] = ok ? static_cast<int32_t>(ch) : -1;
                    mine += ok;
                }
                if (mine) atomicAdd(&s_nvalid, mine);
                ncand = slots;
                __syncthreads();
            } else {
                const int nn = next_pow2(nkeep + nf);
                __syncthreads();
                for (int t = tid; t < nn; t += kSelThreads)
                    out_ids[t] = t < nkeep ? key_node(keys[t]) : t < nkeep + nf ? (t == nkeep ? f0 : f1) : 0x7FFFFFFF;
                nkeep += nf;
                __syncthreads();
            }
        }
    }
    bitonic_asc(out_ids, next_pow2(nkeep));
    int32_t* dst = p.idx + row * p.topk;
    for (int t = tid; t < p.topk; t += kSelThreads) dst[t] = t < nkeep ? out_ids[t] : -1;
    if (p.margin != nullptr && tid == 0) p.margin[row] = s_margin;
}

bool launch_select(const SelectParams& p, int32_t batch, cudaStream_t st, int32_t* launches) {
    int maxb = 1;
    for (int l = 0; l < p.L; ++l) maxb = max(maxb, p.budget[l]);
    int cap = 1;
    while (cap < max(p.factor * maxb, p.lsize[p.L - 1])) cap <<= 1;
    if (cap < 4) cap = 4;  // keeps the fp32 query row 16-byte aligned
    if (p.scores != nullptr && !p.decode && dense_select_cap(cap) > 0) {
        *launches += 2;
        return launch_select_dense(p, batch, cap, st);
    }
    *launches += 1;
    const size_t smem = static_cast<size_t>(cap) * (sizeof(uint64_t) + sizeof(int32_t)) +
                        static_cast<size_t>(p.D) * (1 + p.L) * sizeof(float);
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
