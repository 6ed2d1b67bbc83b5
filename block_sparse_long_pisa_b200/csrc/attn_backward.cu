// Backward of the sparse attention step through a fixed selection (PISA page,
// section "Ce que cela change pour vous": the same sparse kernels serve
// training; the selection is a discrete choice and has no gradient).
//
// With S = scale Q K^T over the selected keys (causal mask on the diagonal
// block), P = exp(S - LSE) (the forward's row log-sum-exp), O = P V:
//   Delta = rowsum(dO * O)
//   dP = dO V^T,  dS = P * (dP - Delta)
//   dQ = scale dS K,  dK = scale dS^T Q,  dV = P^T dO
// A KV head's dK and dV sum over all query rows (of all its query heads) whose
// selection holds the key.
//
// Launches:
//   bwd_delta_kernel   Delta per query row (fp32, workspace).
//   bwd_index_*        the inverse of the selection: for every (batch, KV head,
//                      key block) the (query block, query head) pairs that
//                      use it, in ascending order (counts per range of query
//                      blocks, scan, ordered fill of the ranges in parallel),
//                      so the column pass sums in a fixed order.
//   row pass (dQ) and column pass (dK, dV): the tcgen05/TMEM kernels of
//   attn_backward_tc.cu, for both head dims (64, 128) and both block sizes
//   (64, 128 keys).
// No atomics on any gradient: results are deterministic.
#include <cuda_bf16.h>

#include "pisa_device.cuh"

namespace pisa {

namespace {

// A selected block the attention used: inside the keys and, causal, not after the query block.
__device__ __forceinline__ bool valid_block(const BwdParams& p, int32_t j, int i) {
    return j >= 0 && j < p.n0 && (!p.causal || j <= i);
}

}  // namespace

// ---------------------------------------------------------------- Delta

template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const BwdParams p, int64_t rows) {
    constexpr int TPR = D / 8;  // threads per row, 8 elements each
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t row = t / TPR;
    const int part = static_cast<int>(t % TPR);
    float acc = 0.f;
    if (row < rows) {
        const uint4 a = *reinterpret_cast<const uint4*>(p.dO + row * D + part * 8);
        const uint4 b = *reinterpret_cast<const uint4*>(p.O + row * D + part * 8);
        const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            acc = fmaf(__uint_as_float(wa[k] << 16), __uint_as_float(wb[k] << 16), acc);
            acc = fmaf(__uint_as_float(wa[k] & 0xFFFF0000u), __uint_as_float(wb[k] & 0xFFFF0000u), acc);
        }
    }
#pragma unroll
    for (int o = TPR / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
    if (row < rows && part == 0) p.delta[row] = acc;
}

// ---------------------------------------------------------------- inverse of the selection

// counts[(b * Hkv + kvh) * (n0 + 1) + j] += pairs (query block, query head) that use key block j
__global__ void __launch_bounds__(256) bwd_index_count_kernel(const BwdParams p, int64_t entries) {
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= entries) return;
    const int i = static_cast<int>((t / p.topk) % p.nqb);
    const int hs = static_cast<int>((t / (static_cast<int64_t>(p.topk) * p.nqb)) % p.Hsel);
    const int b = static_cast<int>(t / (static_cast<int64_t>(p.topk) * p.nqb * p.Hsel));
    const int32_t j = p.idx[t];
    if (!valid_block(p, j, i)) return;
    const int kvh = p.per_qhead ? hs / p.g : hs;
    const int64_t plane = static_cast<int64_t>(b) * p.Hkv + kvh;
    atomicAdd(p.rcounts + (plane * p.nranges + i / p.rsize) * p.n0 + j, p.per_qhead ? 1 : p.g);
}

// One CTA per (batch, KV head) plane. Per key block j: the counts of the query-block ranges
// become running sums (where each range's entries start inside j's list), the list lengths are
// scanned into offsets (counts), and every range cursor is moved to its absolute position.
__global__ void __launch_bounds__(256) bwd_index_scan_kernel(const BwdParams p) {
    __shared__ int32_t part[256];
    const int plane = blockIdx.x;
    int32_t* rc = p.rcounts + static_cast<int64_t>(plane) * p.nranges * p.n0;
    int32_t* offs = p.counts + static_cast<int64_t>(plane) * (p.n0 + 1);
    const int n = p.n0 + 1;  // list lengths and the total
    for (int j = threadIdx.x; j < p.n0; j += blockDim.x) {
        int acc = 0;
        for (int r = 0; r < p.nranges; ++r) {
            const int c = rc[static_cast<int64_t>(r) * p.n0 + j];
            rc[static_cast<int64_t>(r) * p.n0 + j] = acc;
            acc += c;
        }
        offs[j] = acc;
    }
    __syncthreads();
    // exclusive scan of offs[0 .. n0] (offs[n0] taken as 0): each thread a contiguous segment
    const int seg = (n + blockDim.x - 1) / blockDim.x;
    const int lo = threadIdx.x * seg, hi = min(n, lo + seg);
    int sum = 0;
    for (int j = lo; j < hi; ++j) sum += j < p.n0 ? offs[j] : 0;
    part[threadIdx.x] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {
        int run = 0;
        for (int k = 0; k < static_cast<int>(blockDim.x); ++k) {
            const int v = part[k];
            part[k] = run;
            run += v;
        }
    }
    __syncthreads();
    int run = part[threadIdx.x];
    for (int j = lo; j < hi; ++j) {
        const int v = j < p.n0 ? offs[j] : 0;
        offs[j] = run;
        run += v;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < p.n0; j += blockDim.x) {
        const int off = offs[j];
        for (int r = 0; r < p.nranges; ++r) rc[static_cast<int64_t>(r) * p.n0 + j] += off;
    }
}

// One warp per (range of query blocks, plane): the range's entries in ascending (query block,
// query head) order, starting at the cursors the scan left. Equal key blocks within a chunk of 32
// candidates are ranked by lane (match.any), so the order is fixed.
__global__ void __launch_bounds__(32) bwd_index_fill_kernel(const BwdParams p) {
    extern __shared__ int32_t cursor[];  // [n0]
    const int lane = threadIdx.x;
    const int r = blockIdx.x, plane = blockIdx.y;  // plane = b * Hkv + kvh
    const int b = plane / p.Hkv, kvh = plane % p.Hkv;
    const int32_t* rc = p.rcounts + (static_cast<int64_t>(plane) * p.nranges + r) * p.n0;
    int32_t* out = p.entries + static_cast<int64_t>(plane) * p.max_entries;
    for (int j = lane; j < p.n0; j += 32) cursor[j] = rc[j];
    __syncwarp();
    const int hper = p.per_qhead ? p.g : 1;                 // selection rows of this plane per query block
    const int mult = p.per_qhead ? 1 : p.g;                  // entries per selected block
    const int i_lo = r * p.rsize, i_hi = min(p.nqb, i_lo + p.rsize);
    const int64_t c_lo = static_cast<int64_t>(i_lo) * hper * p.topk;
    const int64_t c_hi = static_cast<int64_t>(i_hi) * hper * p.topk;
    constexpr int BATCH = 8;  // candidate loads in flight per lane
    for (int64_t cb = c_lo; cb < c_hi; cb += 32 * BATCH) {
        int32_t jb[BATCH];
#pragma unroll
        for (int q = 0; q < BATCH; ++q) {
            const int64_t c = cb + q * 32 + lane;
            jb[q] = -1;
            if (c < c_hi) {
                const int slot = static_cast<int>(c % p.topk);
                const int hsub = static_cast<int>((c / p.topk) % hper);
                const int i = static_cast<int>(c / (static_cast<int64_t>(p.topk) * hper));
                const int hs = p.per_qhead ? kvh * p.g + hsub : kvh;
                jb[q] = p.idx[((static_cast<int64_t>(b) * p.Hsel + hs) * p.nqb + i) * p.topk + slot];
            }
        }
        for (int q = 0; q < BATCH; ++q) {
            const int64_t c = cb + q * 32 + lane;
            int32_t j = -1;
            int i = 0, hsub = 0;
            if (c < c_hi) {
                hsub = static_cast<int>((c / p.topk) % hper);
                i = static_cast<int>(c / (static_cast<int64_t>(p.topk) * hper));
                j = valid_block(p, jb[q], i) ? jb[q] : -1;
            }
            const uint32_t peers = __match_any_sync(0xFFFFFFFFu, j);
            const int rank = __popc(peers & ((1u << lane) - 1u));
            if (j >= 0) {
                const int pos = cursor[j] + rank * mult;
                if (p.per_qhead) {
                    out[pos] = i * p.g + hsub;
                } else {
                    for (int e = 0; e < p.g; ++e) out[pos + e] = i * p.g + e;
                }
            }
            __syncwarp();
            // the highest-ranked lane of each key block moves its cursor past the chunk's entries
            if (j >= 0 && (peers >> lane) == 1u) cursor[j] += (rank + 1) * mult;
            __syncwarp();
        }
    }
}

// ---------------------------------------------------------------- launcher

bool launch_attn_backward(const BwdParams& p, int32_t batch, cudaStream_t st, int32_t* launches) {
    // Delta
    const int64_t rows = static_cast<int64_t>(batch) * p.Hq * p.N;
    {
        const int64_t threads = rows * (p.D / 8);
        const unsigned grid = static_cast<unsigned>((threads + 255) / 256);
        if (p.D == 64)
            bwd_delta_kernel<64><<<grid, 256, 0, st>>>(p, rows);
        else
            bwd_delta_kernel<128><<<grid, 256, 0, st>>>(p, rows);
        if (cudaGetLastError() != cudaSuccess) return false;
    }
    // inverse of the selection: counts per (plane, query-block range, key block), scan, ordered fill
    if (cudaMemsetAsync(p.rcounts, 0,
                        static_cast<size_t>(batch) * p.Hkv * p.nranges * p.n0 * sizeof(int32_t), st) != cudaSuccess)
        return false;
    const int64_t cand = static_cast<int64_t>(batch) * p.Hsel * p.nqb * p.topk;
    bwd_index_count_kernel<<<static_cast<unsigned>((cand + 255) / 256), 256, 0, st>>>(p, cand);
    if (cudaGetLastError() != cudaSuccess) return false;
    bwd_index_scan_kernel<<<static_cast<unsigned>(batch * p.Hkv), 256, 0, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return false;
    const size_t smem_fill = static_cast<size_t>(p.n0) * sizeof(int32_t);
    if (cudaFuncSetAttribute(bwd_index_fill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_fill)) != cudaSuccess)
        return false;
    bwd_index_fill_kernel<<<dim3(static_cast<unsigned>(p.nranges), static_cast<unsigned>(batch * p.Hkv)), 32,
                            smem_fill, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return false;
    *launches += 4;
    const bool ok = launch_bwd_dq_tc(p, batch, st) && launch_bwd_dkdv_tc(p, batch, st);
    if (ok) *launches += 2;
    return ok;
}

}  // namespace pisa
