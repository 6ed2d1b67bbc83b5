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
//   row pass (dQ) and column pass (dK, dV): for head dim 128 with 64-key
//   blocks, the tcgen05/TMEM kernels of attn_backward_tc.cu; for the other
//   shapes the two kernels below, on the warp-level mma.sync path:
//   bwd_dq_kernel      row-parallel: one CTA per (batch, query head, query
//                      block), one warp per 16 rows; S and dP recomputed per
//                      selected block (m16n8k16, bf16 in, fp32 accumulate),
//                      dQ kept in registers and written once. The next
//                      block's K and V copy overlaps this block's MMAs.
//   bwd_dkdv_kernel    column-parallel: one CTA per (batch, KV head, key
//                      block), one warp per 16 keys; S^T and dP^T recomputed
//                      for every pair of the list (the next pair's Q, dO copy
//                      overlapping), dK and dV kept in registers and written
//                      once.
// No atomics on any gradient: results are deterministic.
// Operand tiles of the mma.sync kernels sit in shared memory as [rows][D]
// bf16 with the 16-byte chunks of a row XOR-swizzled by the row index, so
// ldmatrix reads are conflict-free.
#include <cuda_bf16.h>

#include "pisa_device.cuh"

namespace pisa {

namespace {

constexpr int kKC = 64;  // keys (dQ pass) or queries (dK/dV pass) per inner chunk

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void cp_async16(uint32_t saddr, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Byte offset of element (row, col) in a swizzled [rows][D] bf16 tile.
template <int D>
__device__ __forceinline__ uint32_t tile_off(int row, int col) {
    return static_cast<uint32_t>(row * D * 2 + ((((col >> 3) ^ (row & 7))) << 4) + (col & 7) * 2);
}

// Copies `rows` consecutive rows of a [.., D] bf16 global tensor into a swizzled tile.
template <int D, int THREADS>
__device__ __forceinline__ void load_tile(uint32_t tile, const __nv_bfloat16* src, int rows) {
    constexpr int CH = D / 8;
    for (int t = threadIdx.x; t < rows * CH; t += THREADS) {
        const int r = t / CH, c = t % CH;
        cp_async16(tile + tile_off<D>(r, c * 8), src + static_cast<int64_t>(r) * D + c * 8);
    }
}

// A fragment (16 x 16 at rows r0.., cols k0..) of a swizzled tile.
template <int D>
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], uint32_t tile, int r0, int k0) {
    const int l = threadIdx.x & 31;
    ldsm_x4(a, tile + tile_off<D>(r0 + (l & 7) + ((l >> 3) & 1) * 8, k0 + (l >> 4) * 8));
}

// B fragments of two n-tiles (rows n0..n0+15 of the tile are the n index, cols k0..k0+15 the k
// index): {b0, b1} of n-tile 0 in r[0], r[1], of n-tile 1 in r[2], r[3].
template <int D>
__device__ __forceinline__ void frag_b(uint32_t (&r)[4], uint32_t tile, int n0, int k0) {
    const int l = threadIdx.x & 31;
    ldsm_x4(r, tile + tile_off<D>(n0 + (l & 7) + (l >> 4) * 8, k0 + ((l >> 3) & 1) * 8));
}

// B fragments of two n-tiles where the tile's rows are the k index (k0..k0+15) and its columns
// the n index (n0..n0+15): {b0, b1} of n-tile 0 in r[0], r[1], of n-tile 1 in r[2], r[3].
template <int D>
__device__ __forceinline__ void frag_b_t(uint32_t (&r)[4], uint32_t tile, int k0, int n0) {
    const int l = threadIdx.x & 31;
    ldsm_x4_t(r, tile + tile_off<D>(k0 + (l & 7) + ((l >> 3) & 1) * 8, n0 + (l >> 4) * 8));
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) { return pack_bf16x2(lo, hi); }

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

// ---------------------------------------------------------------- dQ

template <int D, int BLK>
__global__ void __launch_bounds__(BLK * 2) bwd_dq_kernel(const BwdParams p) {
    constexpr int THREADS = BLK * 2;  // BLK / 16 warps
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr uint32_t TILE = BLK * D * 2;
    // Q, dO, then two stages of (K, V): the next selected block's copy overlaps this one's MMAs
    const uint32_t sQ = smem_u32(smem), sO = sQ + TILE, sKV = sO + TILE;
    int32_t* list = reinterpret_cast<int32_t*>(smem + 6 * TILE);
    __shared__ int s_n;

    const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g4 = lane >> 2, t4 = lane & 3;
    const int hs = p.per_qhead ? h : h / p.g;
    const int kvh = h / p.g;
    const int64_t qbase = (static_cast<int64_t>(b) * p.Hq + h) * p.N + static_cast<int64_t>(i) * BLK;
    const int64_t kbase = (static_cast<int64_t>(b) * p.Hkv + kvh) * p.N;

    if (warp == 0) {
        const int32_t* row = p.idx + ((static_cast<int64_t>(b) * p.Hsel + hs) * p.nqb + i) * p.topk;
        int cnt = 0;
        for (int t0 = 0; t0 < p.topk; t0 += 32) {
            const int t = t0 + lane;
            const int32_t j = t < p.topk ? row[t] : -1;
            const bool ok = t < p.topk && valid_block(p, j, i);
            const uint32_t m = __ballot_sync(0xFFFFFFFFu, ok);
            if (ok) list[cnt + __popc(m & ((1u << lane) - 1u))] = j;
            cnt += __popc(m);
        }
        if (lane == 0) s_n = cnt;
    }
    load_tile<D, THREADS>(sQ, p.Q + qbase * D, BLK);
    load_tile<D, THREADS>(sO, p.dO + qbase * D, BLK);
    cp_async_commit();
    __syncthreads();  // the block list is written
    const int nsel = s_n;
    auto load_kv = [&](int u) {
        const int64_t row = kbase + static_cast<int64_t>(list[u]) * BLK;
        load_tile<D, THREADS>(sKV + (u & 1) * 2 * TILE, p.K + row * D, BLK);
        load_tile<D, THREADS>(sKV + (u & 1) * 2 * TILE + TILE, p.V + row * D, BLK);
        cp_async_commit();
    };
    if (nsel > 0) load_kv(0);

    const int r0 = warp * 16;
    const float c2 = p.scale_log2;
    const float lse2[2] = {p.lse[qbase + r0 + g4] * 1.4426950408889634f, p.lse[qbase + r0 + g4 + 8] * 1.4426950408889634f};
    const float dlt[2] = {p.delta[qbase + r0 + g4], p.delta[qbase + r0 + g4 + 8]};
    float dq[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n) dq[n][0] = dq[n][1] = dq[n][2] = dq[n][3] = 0.f;

    for (int u = 0; u < nsel; ++u) {
        const int j = list[u];
        const uint32_t sK = sKV + (u & 1) * 2 * TILE, sV = sK + TILE;
        if (u + 1 < nsel) {
            load_kv(u + 1);  // its stage was last read in iteration u - 1, closed by the barrier below
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();  // this block's K, V (and, the first time, Q and dO) are in shared memory
        for (int kc = 0; kc < BLK; kc += kKC) {
            float s[kKC / 8][4], dp[kKC / 8][4];
#pragma unroll
            for (int n = 0; n < kKC / 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[n][e] = dp[n][e] = 0.f;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t aq[4], ao[4];
                frag_a<D>(aq, sQ, r0, ks * 16);
                frag_a<D>(ao, sO, r0, ks * 16);
#pragma unroll
                for (int n = 0; n < kKC / 8; n += 2) {
                    uint32_t bk[4], bv[4];
                    frag_b<D>(bk, sK, kc + n * 8, ks * 16);
                    frag_b<D>(bv, sV, kc + n * 8, ks * 16);
                    mma16816(s[n], aq, bk[0], bk[1]);
                    mma16816(s[n + 1], aq, bk[2], bk[3]);
                    mma16816(dp[n], ao, bv[0], bv[1]);
                    mma16816(dp[n + 1], ao, bv[2], bv[3]);
                }
            }
            // P and dS, in place of S
#pragma unroll
            for (int n = 0; n < kKC / 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int rr = r0 + g4 + (e >> 1) * 8;  // query row in the block
                    const int cc = kc + n * 8 + 2 * t4 + (e & 1);  // key in the block
                    float pv = fast_exp2(s[n][e] * c2 - lse2[e >> 1]);
                    if (p.causal && j == i && cc > rr) pv = 0.f;
                    s[n][e] = pv * (dp[n][e] - dlt[e >> 1]);
                }
            // dQ += dS K (keys are the k index)
#pragma unroll
            for (int ks = 0; ks < kKC / 16; ++ks) {
                uint32_t a[4];
                a[0] = pack2(s[2 * ks][0], s[2 * ks][1]);
                a[1] = pack2(s[2 * ks][2], s[2 * ks][3]);
                a[2] = pack2(s[2 * ks + 1][0], s[2 * ks + 1][1]);
                a[3] = pack2(s[2 * ks + 1][2], s[2 * ks + 1][3]);
#pragma unroll
                for (int n = 0; n < D / 8; n += 2) {
                    uint32_t bk[4];
                    frag_b_t<D>(bk, sK, kc + ks * 16, n * 8);
                    mma16816(dq[n], a, bk[0], bk[1]);
                    mma16816(dq[n + 1], a, bk[2], bk[3]);
                }
            }
        }
        __syncthreads();  // every warp is done with this stage before it is refilled
    }
    cp_async_wait<0>();  // (no selected block: the Q and dO copies)
    // dQ = scale * (dS K), bf16
    const float sc = p.scale;
    __nv_bfloat16* dst = p.dQ + (qbase + r0) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
        const int col = n * 8 + 2 * t4;
        *reinterpret_cast<uint32_t*>(dst + g4 * D + col) = pack2(dq[n][0] * sc, dq[n][1] * sc);
        *reinterpret_cast<uint32_t*>(dst + (g4 + 8) * D + col) = pack2(dq[n][2] * sc, dq[n][3] * sc);
    }
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

// ---------------------------------------------------------------- dK, dV

template <int D, int BLK>
__global__ void __launch_bounds__(BLK * 2) bwd_dkdv_kernel(const BwdParams p) {
    constexpr int THREADS = BLK * 2;
    extern __shared__ __align__(1024) uint8_t smem[];
    constexpr uint32_t TILE = BLK * D * 2;
    // K, V, then two stages of (Q, dO, LSE, Delta): the next pair's copy overlaps this one's MMAs
    constexpr uint32_t STAGE = 2 * TILE + 2 * BLK * 4;
    const uint32_t sK = smem_u32(smem), sV = sK + TILE, sStage = sV + TILE;

    const int j = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g4 = lane >> 2, t4 = lane & 3;
    const int plane = b * p.Hkv + kvh;
    const int64_t kbase = (static_cast<int64_t>(b) * p.Hkv + kvh) * p.N + static_cast<int64_t>(j) * BLK;
    const int32_t* offs = p.counts + static_cast<int64_t>(plane) * (p.n0 + 1);
    const int32_t* ent = p.entries + static_cast<int64_t>(plane) * p.max_entries;
    const int e_lo = offs[j], e_hi = offs[j + 1];

    load_tile<D, THREADS>(sK, p.K + kbase * D, BLK);
    load_tile<D, THREADS>(sV, p.V + kbase * D, BLK);
    cp_async_commit();
    auto load_pair = [&](int e) {
        const int code = ent[e];
        const int i = code / p.g, h = kvh * p.g + code % p.g;
        const int64_t qbase = (static_cast<int64_t>(b) * p.Hq + h) * p.N + static_cast<int64_t>(i) * BLK;
        const uint32_t st = sStage + ((e - e_lo) & 1) * STAGE;
        load_tile<D, THREADS>(st, p.Q + qbase * D, BLK);
        load_tile<D, THREADS>(st + TILE, p.dO + qbase * D, BLK);
        for (int t = threadIdx.x; t < BLK / 4; t += THREADS) {  // 16-byte pieces of the row statistics
            cp_async16(st + 2 * TILE + t * 16, p.lse + qbase + t * 4);
            cp_async16(st + 2 * TILE + BLK * 4 + t * 16, p.delta + qbase + t * 4);
        }
        cp_async_commit();
    };
    if (e_hi > e_lo) load_pair(e_lo);

    const int r0 = warp * 16;  // this warp's keys in the block
    const float c2 = p.scale_log2;
    float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
    for (int n = 0; n < D / 8; ++n)
#pragma unroll
        for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.f;

    for (int e = e_lo; e < e_hi; ++e) {
        const int i = ent[e] / p.g;
        const uint32_t sQ = sStage + ((e - e_lo) & 1) * STAGE, sO = sQ + TILE;
        const float* s_lse = reinterpret_cast<const float*>(smem + (sQ - sK) + 2 * TILE);
        const float* s_dlt = s_lse + BLK;
        if (e + 1 < e_hi) {
            load_pair(e + 1);  // its stage was last read in iteration e - 1, closed by the barrier below
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();  // this pair's tiles (and, the first time, K and V) are in shared memory
        for (int qc = 0; qc < BLK; qc += kKC) {
            float s[kKC / 8][4], dp[kKC / 8][4];
#pragma unroll
            for (int n = 0; n < kKC / 8; ++n)
#pragma unroll
                for (int x = 0; x < 4; ++x) s[n][x] = dp[n][x] = 0.f;
            // S^T = K Q^T and dP^T = V dO^T (keys are the rows, queries the columns)
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                uint32_t ak[4], av[4];
                frag_a<D>(ak, sK, r0, ks * 16);
                frag_a<D>(av, sV, r0, ks * 16);
#pragma unroll
                for (int n = 0; n < kKC / 8; n += 2) {
                    uint32_t bq[4], bo[4];
                    frag_b<D>(bq, sQ, qc + n * 8, ks * 16);
                    frag_b<D>(bo, sO, qc + n * 8, ks * 16);
                    mma16816(s[n], ak, bq[0], bq[1]);
                    mma16816(s[n + 1], ak, bq[2], bq[3]);
                    mma16816(dp[n], av, bo[0], bo[1]);
                    mma16816(dp[n + 1], av, bo[2], bo[3]);
                }
            }
            // P^T (kept in s) and dS^T (kept in dp)
#pragma unroll
            for (int n = 0; n < kKC / 8; ++n)
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int kr = r0 + g4 + (x >> 1) * 8;        // key in the block
                    const int qq = qc + n * 8 + 2 * t4 + (x & 1);  // query in its block
                    float pv = fast_exp2(s[n][x] * c2 - s_lse[qq] * 1.4426950408889634f);
                    if (p.causal && j == i && kr > qq) pv = 0.f;
                    s[n][x] = pv;
                    dp[n][x] = pv * (dp[n][x] - s_dlt[qq]);
                }
            // dV += P^T dO, dK += dS^T Q (queries are the k index)
#pragma unroll
            for (int ks = 0; ks < kKC / 16; ++ks) {
                uint32_t ap[4], as[4];
                ap[0] = pack2(s[2 * ks][0], s[2 * ks][1]);
                ap[1] = pack2(s[2 * ks][2], s[2 * ks][3]);
                ap[2] = pack2(s[2 * ks + 1][0], s[2 * ks + 1][1]);
                ap[3] = pack2(s[2 * ks + 1][2], s[2 * ks + 1][3]);
                as[0] = pack2(dp[2 * ks][0], dp[2 * ks][1]);
                as[1] = pack2(dp[2 * ks][2], dp[2 * ks][3]);
                as[2] = pack2(dp[2 * ks + 1][0], dp[2 * ks + 1][1]);
                as[3] = pack2(dp[2 * ks + 1][2], dp[2 * ks + 1][3]);
#pragma unroll
                for (int n = 0; n < D / 8; n += 2) {
                    uint32_t bo[4], bq[4];
                    frag_b_t<D>(bo, sO, qc + ks * 16, n * 8);
                    frag_b_t<D>(bq, sQ, qc + ks * 16, n * 8);
                    mma16816(dv[n], ap, bo[0], bo[1]);
                    mma16816(dv[n + 1], ap, bo[2], bo[3]);
                    mma16816(dk[n], as, bq[0], bq[1]);
                    mma16816(dk[n + 1], as, bq[2], bq[3]);
                }
            }
        }
        __syncthreads();  // every warp is done with this stage before it is refilled
    }
    cp_async_wait<0>();  // (no pair: the K and V copies)
    const float sc = p.scale;
    __nv_bfloat16* dK = p.dK + (kbase + r0) * D;
    __nv_bfloat16* dV = p.dV + (kbase + r0) * D;
#pragma unroll
    for (int n = 0; n < D / 8; ++n) {
        const int col = n * 8 + 2 * t4;
        *reinterpret_cast<uint32_t*>(dK + g4 * D + col) = pack2(dk[n][0] * sc, dk[n][1] * sc);
        *reinterpret_cast<uint32_t*>(dK + (g4 + 8) * D + col) = pack2(dk[n][2] * sc, dk[n][3] * sc);
        *reinterpret_cast<uint32_t*>(dV + g4 * D + col) = pack2(dv[n][0], dv[n][1]);
        *reinterpret_cast<uint32_t*>(dV + (g4 + 8) * D + col) = pack2(dv[n][2], dv[n][3]);
    }
}

// ---------------------------------------------------------------- launcher

template <int D, int BLK>
static bool launch_bwd_variant(const BwdParams& p, int32_t batch, cudaStream_t st) {
    const int threads = BLK * 2;
    const size_t smem_dq = 6 * BLK * D * 2 + static_cast<size_t>(p.topk) * 4;
    const size_t smem_kv = 6 * BLK * D * 2 + 4 * BLK * sizeof(float);
    if (cudaFuncSetAttribute(bwd_dq_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_dq)) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_dkdv_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_kv)) != cudaSuccess)
        return false;
    if (bwd_dq_tc_supported(p)) {
        if (!launch_bwd_dq_tc(p, batch, st)) return false;
    } else {
        bwd_dq_kernel<D, BLK><<<dim3(p.nqb, p.Hq, batch), threads, smem_dq, st>>>(p);
        if (cudaGetLastError() != cudaSuccess) return false;
    }
    if (bwd_dkdv_tc_supported(p)) return launch_bwd_dkdv_tc(p, batch, st);
    bwd_dkdv_kernel<D, BLK><<<dim3(p.n0, p.Hkv, batch), threads, smem_kv, st>>>(p);
    return cudaGetLastError() == cudaSuccess;
}

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
    bool ok;
    if (p.D == 128)
        ok = p.blk == 64 ? launch_bwd_variant<128, 64>(p, batch, st) : launch_bwd_variant<128, 128>(p, batch, st);
    else
        ok = p.blk == 64 ? launch_bwd_variant<64, 64>(p, batch, st) : launch_bwd_variant<64, 128>(p, batch, st);
    if (ok) *launches += 2;
    return ok;
}

}  // namespace pisa
