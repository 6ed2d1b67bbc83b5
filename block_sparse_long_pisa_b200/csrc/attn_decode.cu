// Decode: one query token per sequence at position N-1 attends to the K/V
// blocks its pyramid descent selected. The work is bound by the bytes of the
// selected K/V blocks; the arithmetic only has to stay out of the way:
//
//   attn_decode_kernel: one CTA of four warps per (batch, selection row,
//     split); a split is up to `bps` consecutive entries of the compacted
//     block list. K and V blocks arrive by 2-D TMA (128-byte swizzle) in a
//     ring of NSTG stages. The gh <= 8 query heads of the selection row are
//     the rows of a 16-row bf16 tensor-core tile (rows gh.. are zero): each
//     warp takes a quarter of every block's keys and computes its scores and
//     its share of P.V with mma.sync m16n8k16 (fragments by ldmatrix from the
//     swizzled tiles), with its own online softmax. At the end the four warps'
//     (o, m, l) combine into one unnormalised partial per head.
//   attn_merge_kernel: combines the partials of all splits with the
//     online-softmax merge of the Pulsar Attention page ("Phase 2"):
//     m = max m_s, l = sum exp2(m_s - m) l_s, o = sum exp2(m_s - m) o_s / l.
#include <cuda.h>
#include <cuda_bf16.h>

#include "pisa_device.cuh"

namespace pisa {

constexpr int kDecThreads = 128;

template <int D, int BLK>
struct DecodeCfg {
    static constexpr int DS = D / 64;                      // 128-byte column tiles of a row
    static constexpr int SUBT = BLK * 128;                 // one [BLK rows x 128 B] swizzled tile
    static constexpr int TILE = DS * SUBT;                 // one K (or V) block
    static constexpr int STAGE = 2 * TILE;                 // K and V
    static constexpr int NSTG = STAGE <= 16384 ? 4 : (STAGE <= 32768 ? 3 : 2);
    static constexpr int KW = BLK / 4;                     // keys of a block per warp
    static constexpr int NT = KW / 8;                      // score n-tiles per warp
    static constexpr int COMBINE = 4 * 8 * (D + 2) * 4;    // per-warp (o, m, l) of 8 heads
    static constexpr int SMEM = 1024 + NSTG * STAGE;
    static_assert(COMBINE <= NSTG * STAGE, "combine area reuses the ring");
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// D += A B for one m16n8k16 bf16 tile with fp32 accumulators; a1 = a3 = 0 (rows 8-15 unused)
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
// byte offset of row `row`, 16-byte chunk `chunk` (of the 8 in a 128-byte row) inside a swizzled tile
__device__ __forceinline__ uint32_t sw128(int row, int chunk) {
    return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int D, int BLK>
__global__ void __launch_bounds__(kDecThreads) attn_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                  const __grid_constant__ CUtensorMap tmV,
                                                                  const DecodeParams p) {
    using C = DecodeCfg<D, BLK>;
    extern __shared__ uint8_t dsm_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t full[C::NSTG], empty[C::NSTG];
    __shared__ int32_t list[kDecMaxBps];
    __shared__ int s_cnt;

    const int split = blockIdx.x, hs = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gh = p.gh;
    const int kvh = p.per_qhead ? hs / p.g : hs;
    const int head0 = p.per_qhead ? hs : kvh * p.g;
    const uint32_t detail_base = kKernAttnDecode << 8;

    // this split's slice of the compacted block list
    if (warp == 0) {
        const int32_t* row = p.idx + (static_cast<int64_t>(b) * p.Hsel + hs) * p.topk;
        const int lo = split * p.bps, hi = lo + p.bps;
        int cnt = 0;
        for (int t0 = 0; t0 < p.topk; t0 += 32) {
            const int t = t0 + lane;
            const int32_t j = t < p.topk ? row[t] : -1;
            const bool ok = j >= 0 && j < p.n0;
            if (t < p.topk && j >= 0 && !ok && split == 0)
                record_error(p.status, PISA_ERR_BAD_INDEX, detail_base | 0xB0u);
            const uint32_t m = __ballot_sync(0xFFFFFFFFu, ok);
            const int pos = cnt + __popc(m & ((1u << lane) - 1u));
            if (ok && pos >= lo && pos < hi) list[pos - lo] = j;
            cnt += __popc(m);
        }
        if (lane == 0) {
            s_cnt = min(max(cnt - lo, 0), p.bps);
            for (int s = 0; s < C::NSTG; ++s) {
                mbar_init(&full[s], 1);
                mbar_init(&empty[s], 4);
            }
            fence_barrier_init();
        }
    }
    __syncthreads();
    const int cnt = s_cnt;
    const int64_t row0 = (static_cast<int64_t>(b) * p.Hkv + kvh) * p.N;  // first K/V row of this plane
    auto issue = [&](int n) {
        const int s = n % C::NSTG;
        uint8_t* kt = ring + s * C::STAGE;
        mbar_arrive_expect_tx(&full[s], C::STAGE);
        const int y = static_cast<int>(row0 + static_cast<int64_t>(list[n]) * BLK);
#pragma unroll
        for (int c = 0; c < C::DS; ++c) {
            tma_load_2d(kt + c * C::SUBT, &tmK, c * 64, y, &full[s]);
            tma_load_2d(kt + C::TILE + c * C::SUBT, &tmV, c * 64, y, &full[s]);
        }
    };
    int issued = 0;  // thread 0: blocks whose copies were started
    if (tid == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        for (; issued < C::NSTG && issued < cnt; ++issued) issue(issued);
    }

    // query fragments: row hh = lane / 4 (zero past gh), dims 16 ks + 2 (lane % 4) (+8)
    const int hh = lane >> 2, q4 = lane & 3;
    uint32_t qa[D / 16][2];
    {
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(p.Q + (static_cast<int64_t>(b) * p.Hq + head0 + hh) * D);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            qa[ks][0] = hh < gh ? qrow[ks * 8 + q4] : 0u;
            qa[ks][1] = hh < gh ? qrow[ks * 8 + 4 + q4] : 0u;
        }
    }
    const float cs = p.scale_log2;
    float o[D / 8][4];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m_run = -INFINITY, l_thr = 0.f;  // this thread's row hh: running max, partial sum
    const int kw0 = warp * C::KW;          // this warp's keys of every block
    const int mi = lane >> 3, mr = lane & 7;  // ldmatrix: matrix and row this lane addresses
    bool ok = true;
    int n = 0;
    for (; n < cnt; ++n) {
        const int s = n % C::NSTG;
        ok = mbar_wait(&full[s], (n / C::NSTG) & 1, p.status, detail_base | 0x01u);
        if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
        const uint32_t kbase = smem_u32(ring + s * C::STAGE), vbase = kbase + C::TILE;
        // scores of this warp's keys: S[hh][key] for key = kw0 + 8 nt + 2 (lane % 4) (+1)
        float sc[C::NT][4];
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
            sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
            const int key = kw0 + 8 * nt + mr;
#pragma unroll
            for (int j = 0; j < D / 32; ++j) {  // two k-steps (32 dims) per ldmatrix.x4
                const int dim = 32 * j + 8 * mi;
                uint32_t kb[4];
                ldsm_x4(kbase + (dim / 64) * C::SUBT + sw128(key, (dim % 64) / 8), kb);
                mma_16816(sc[nt], qa[2 * j][0], qa[2 * j][1], kb[0], kb[1]);
                mma_16816(sc[nt], qa[2 * j + 1][0], qa[2 * j + 1][1], kb[2], kb[3]);
            }
        }
        // online softmax of row hh over this warp's keys (the four lanes of a quad share the row)
        float mx = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
            sc[nt][0] *= cs;
            sc[nt][1] *= cs;
            mx = fmax3(mx, sc[nt][0], sc[nt][1]);
        }
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        const float alpha = fast_exp2(m_run - m_new);
        m_run = m_new;
        l_thr *= alpha;
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
            o[j][0] *= alpha;
            o[j][1] *= alpha;
        }
        uint32_t pa[C::NT];  // P as bf16 pairs, A-fragment halves
#pragma unroll
        for (int nt = 0; nt < C::NT; ++nt) {
            const float e0 = fast_exp2(sc[nt][0] - m_new), e1 = fast_exp2(sc[nt][1] - m_new);
            l_thr += e0 + e1;
            pa[nt] = pack_bf16x2(e0, e1);
        }
        // O[hh][:] += P V over this warp's keys: k-steps of 16 keys, two n-tiles per ldmatrix.x4
#pragma unroll
        for (int kk = 0; kk < C::KW / 16; ++kk) {
            const int key = kw0 + 16 * kk + mr + 8 * (mi & 1);
#pragma unroll
            for (int jj = 0; jj < D / 16; ++jj) {
                const int dim = 16 * jj + 8 * (mi >> 1);
                uint32_t vb[4];
                ldsm_x4_t(vbase + (dim / 64) * C::SUBT + sw128(key, (dim % 64) / 8), vb);
                mma_16816(o[2 * jj], pa[2 * kk], pa[2 * kk + 1], vb[0], vb[1]);
                mma_16816(o[2 * jj + 1], pa[2 * kk], pa[2 * kk + 1], vb[2], vb[3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        // refill this stage with block n + NSTG once all four warps are done with it
        if (tid == 0 && n + C::NSTG < cnt) {
            if (!mbar_wait(&empty[s], (n / C::NSTG) & 1, p.status, detail_base | 0x03u)) ok = false;
            else {
                issue(n + C::NSTG);
                ++issued;
            }
        }
        if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
    }
    // in-flight copies land before the ring is reused (only after a failed wait can any be pending)
    if (tid == 0 && !ok) {
        for (int u = n; u < issued; ++u) mbar_wait(&full[u % C::NSTG], (u / C::NSTG) & 1, p.status, detail_base | 0x02u);
    }
    const bool all_ok = __syncthreads_and(ok);
    // the four warps' (o, m, l) of heads 0..gh-1 meet in the ring, then one partial per head
    float* cw = reinterpret_cast<float*>(ring);  // [warp][head][D + 2]
    l_thr += __shfl_xor_sync(0xFFFFFFFFu, l_thr, 1);
    l_thr += __shfl_xor_sync(0xFFFFFFFFu, l_thr, 2);
    if (hh < gh) {
        float* dst = cw + (warp * 8 + hh) * (D + 2);
#pragma unroll
        for (int j = 0; j < D / 8; ++j) {
            dst[8 * j + 2 * q4] = o[j][0];
            dst[8 * j + 2 * q4 + 1] = o[j][1];
        }
        if (q4 == 0) {
            dst[D] = (all_ok && cnt > 0) ? m_run : -INFINITY;
            dst[D + 1] = l_thr;
        }
    }
    __syncthreads();
    float* part = p.part + ((static_cast<int64_t>(b) * p.Hsel + hs) * p.splits + split) * gh * (D + 2);
    for (int e = tid; e < gh * (D + 2); e += kDecThreads) {
        const int h2 = e / (D + 2), d = e % (D + 2);
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, cw[(w * 8 + h2) * (D + 2) + D]);
        float v = 0.f;
        if (d == D) {
            v = M;
        } else if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const float* src = cw + (w * 8 + h2) * (D + 2);
                v += fast_exp2(src[D] - M) * src[d == D + 1 ? D + 1 : d];
            }
        }
        part[h2 * (D + 2) + d] = v;
    }
}

template <int D>
__global__ void __launch_bounds__(128) attn_merge_kernel(const DecodeParams p) {
    const int hs = blockIdx.x, b = blockIdx.y;
    const float* part = p.part + (static_cast<int64_t>(b) * p.Hsel + hs) * p.splits * p.gh * (D + 2);
    const int head0 = p.per_qhead ? hs : hs * p.g;
    for (int e = threadIdx.x; e < p.gh * D; e += blockDim.x) {
        const int hh = e / D, d = e % D;
        float m = -INFINITY;
        for (int s = 0; s < p.splits; ++s) m = fmaxf(m, part[(s * p.gh + hh) * (D + 2) + D]);
        float l = 0.f, o = 0.f;
        if (m != -INFINITY) {
            for (int s = 0; s < p.splits; ++s) {
                const float* ps = part + (s * p.gh + hh) * (D + 2);
                const float w = fast_exp2(ps[D] - m);
                l += w * ps[D + 1];
                o += w * ps[d];
            }
        }
        const int64_t orow = static_cast<int64_t>(b) * p.Hq + head0 + hh;
        p.O[orow * D + d] = __float2bfloat16_rn(l > 0.f ? o / l : 0.f);
        if (d == 0 && p.lse != nullptr) p.lse[orow] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
    }
}

bool launch_attn_decode(const Plan& pl, const DecodeParams& p, cudaStream_t st, int32_t* launches) {
    const int D = pl.D, BLK = pl.blk;
    const int64_t krows = static_cast<int64_t>(pl.B) * pl.Hkv * pl.N;
    if (krows > INT32_MAX) return false;
    CUtensorMap tk, tv;
    if (!make_tmap_2d(&tk, p.K, krows, D, BLK) || !make_tmap_2d(&tv, p.V, krows, D, BLK)) return false;
    dim3 grid(p.splits, p.Hsel, pl.B);
    cudaError_t e = cudaSuccess;
#define PISA_DECODE_CASE(DD, BB)                                                                              \
    if (D == DD && BLK == BB) {                                                                               \
        e = cudaFuncSetAttribute(attn_decode_kernel<DD, BB>, cudaFuncAttributeMaxDynamicSharedMemorySize,    \
                                 DecodeCfg<DD, BB>::SMEM);                                                    \
        if (e == cudaSuccess)                                                                                 \
            attn_decode_kernel<DD, BB><<<grid, kDecThreads, DecodeCfg<DD, BB>::SMEM, st>>>(tk, tv, p);        \
    }
    PISA_DECODE_CASE(64, 64)
    PISA_DECODE_CASE(64, 128)
    PISA_DECODE_CASE(128, 64)
    PISA_DECODE_CASE(128, 128)
#undef PISA_DECODE_CASE
    if (e != cudaSuccess || cudaGetLastError() != cudaSuccess) return false;
    ++*launches;
    dim3 mgrid(pl.Hsel, pl.B);
    if (D == 64)
        attn_merge_kernel<64><<<mgrid, 128, 0, st>>>(p);
    else
        attn_merge_kernel<128><<<mgrid, 128, 0, st>>>(p);
    if (cudaGetLastError() != cudaSuccess) return false;
    ++*launches;
    return true;
}

}  // namespace pisa
