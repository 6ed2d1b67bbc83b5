// Decode: one query token per sequence at position N-1 attends to the K/V
// blocks its pyramid descent selected. The work is bound by the bytes of the
// selected K/V blocks, so the kernel is built for HBM streaming, not the
// tensor core:
//
//   attn_decode_kernel: one CTA per (batch, selection row, split). A split is
//     up to `bps` consecutive entries of the selected-block list. Each K or V
//     block (b rows x D, contiguous in memory) is fetched by one bulk copy
//     into a double-buffered shared-memory ring. The CTA's gh query heads run
//     an online softmax over the split's keys with fp32 FMA and leave an
//     unnormalised partial (o, running max m, sum l) in the workspace.
//   attn_merge_kernel: combines the partials of all splits with the
//     online-softmax merge of the Pulsar Attention page ("Phase 2"):
//     m = max m_s, l = sum exp2(m_s - m) l_s, o = sum exp2(m_s - m) o_s / l.
#include <cuda_bf16.h>

#include "pisa_device.cuh"

namespace pisa {

constexpr int kDecThreads = 128;

template <int D, int BLK>
__global__ void __launch_bounds__(kDecThreads) attn_decode_kernel(const DecodeParams p) {
    constexpr int TILE = BLK * D * 2;  // bytes of one K (or V) block
    extern __shared__ __align__(1024) uint8_t sm[];
    uint8_t* kbuf = sm;                          // [2][TILE]
    uint8_t* vbuf = sm + 2 * TILE;               // [2][TILE]
    float* qs = reinterpret_cast<float*>(sm + 4 * TILE);  // [gh][D], pre-scaled by scale*log2(e)
    float* ss = qs + 8 * D;                      // [gh][BLK] scores, then probabilities
    float* m_run = ss + 8 * BLK;                 // [gh]
    float* l_run = m_run + 8;                    // [gh]
    float* alpha = l_run + 8;                    // [gh]
    int32_t* list = reinterpret_cast<int32_t*>(alpha + 8);  // this split's blocks
    __shared__ __align__(8) uint64_t full[2];
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
        int cnt = 0, taken = 0;
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
        taken = min(max(cnt - lo, 0), p.bps);
        if (lane == 0) {
            s_cnt = taken;
            mbar_init(&full[0], 1);
            mbar_init(&full[1], 1);
            fence_barrier_init();
        }
    }
    const float cs = p.scale_log2;
    for (int e = tid; e < gh * D; e += kDecThreads) {
        const int hh = e / D, d = e % D;
        qs[hh * D + d] = __bfloat162float(p.Q[(static_cast<int64_t>(b) * p.Hq + head0 + hh) * D + d]) * cs;
    }
    if (tid < gh) {
        m_run[tid] = -INFINITY;
        l_run[tid] = 0.f;
    }
    __syncthreads();
    const int cnt = s_cnt;
    const __nv_bfloat16* kplane = p.K + (static_cast<int64_t>(b) * p.Hkv + kvh) * p.N * D;
    const __nv_bfloat16* vplane = p.V + (static_cast<int64_t>(b) * p.Hkv + kvh) * p.N * D;
    int issued = 0;  // thread 0: blocks whose copies were started
    if (tid == 0) {
        for (int u = 0; u < 2 && u < cnt; ++u, ++issued) {
            mbar_arrive_expect_tx(&full[u], 2 * TILE);
            bulk_load(kbuf + u * TILE, kplane + static_cast<int64_t>(list[u]) * BLK * D, TILE, &full[u]);
            bulk_load(vbuf + u * TILE, vplane + static_cast<int64_t>(list[u]) * BLK * D, TILE, &full[u]);
        }
    }
    // output accumulators: this thread owns (head, 4 dims) chunks e = tid + 128 * u
    constexpr int CHUNKS = D / 4;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    bool ok = true;
    int n = 0;
    for (; n < cnt; ++n) {
        const int buf = n & 1;
        ok = mbar_wait(&full[buf], (n >> 1) & 1, p.status, detail_base | 0x01u);
        if (!__syncthreads_and(ok)) {
            ok = false;
            break;
        }
        const __nv_bfloat16* kt = reinterpret_cast<const __nv_bfloat16*>(kbuf + buf * TILE);
        const __nv_bfloat16* vt = reinterpret_cast<const __nv_bfloat16*>(vbuf + buf * TILE);
        // scores: pair e -> (head e / BLK, key e % BLK); rotate the 16-byte chunk order per key
        for (int e = tid; e < gh * BLK; e += kDecThreads) {
            const int hh = e / BLK, key = e % BLK;
            const uint4* krow = reinterpret_cast<const uint4*>(kt + key * D);
            const float* q = qs + hh * D;
            float a = 0.f;
#pragma unroll 4
            for (int cc = 0; cc < D / 8; ++cc) {
                const int c = (cc + key) & (D / 8 - 1);
                const uint4 v = krow[c];
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    a = fmaf(q[c * 8 + 2 * k], __uint_as_float(w[k] << 16), a);
                    a = fmaf(q[c * 8 + 2 * k + 1], __uint_as_float(w[k] & 0xFFFF0000u), a);
                }
            }
            ss[hh * BLK + key] = a;
        }
        __syncthreads();
        // online softmax statistics, one warp per head
        for (int hh = warp; hh < gh; hh += kDecThreads / 32) {
            float mx = -INFINITY;
            for (int key = lane; key < BLK; key += 32) mx = fmaxf(mx, ss[hh * BLK + key]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
            const float m_old = m_run[hh];
            const float m_new = fmaxf(m_old, mx);
            float sum = 0.f;
            for (int key = lane; key < BLK; key += 32) {
                const float e2 = fast_exp2(ss[hh * BLK + key] - m_new);
                ss[hh * BLK + key] = e2;
                sum += e2;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, off);
            __syncwarp();
            if (lane == 0) {
                const float a = fast_exp2(m_old - m_new);
                alpha[hh] = a;
                l_run[hh] = l_run[hh] * a + sum;
                m_run[hh] = m_new;
            }
        }
        __syncthreads();
        // o = o * alpha + P V
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int e = tid + kDecThreads * u;
            if (e < gh * CHUNKS) {
                const int hh = e / CHUNKS, dq = e % CHUNKS;
                const float a = alpha[hh];
                float o0 = acc[u][0] * a, o1 = acc[u][1] * a, o2 = acc[u][2] * a, o3 = acc[u][3] * a;
                const float* pr = ss + hh * BLK;
#pragma unroll 4
                for (int key = 0; key < BLK; ++key) {
                    const uint2 v = *reinterpret_cast<const uint2*>(vt + key * D + dq * 4);
                    const float pk = pr[key];
                    o0 = fmaf(pk, __uint_as_float(v.x << 16), o0);
                    o1 = fmaf(pk, __uint_as_float(v.x & 0xFFFF0000u), o1);
                    o2 = fmaf(pk, __uint_as_float(v.y << 16), o2);
                    o3 = fmaf(pk, __uint_as_float(v.y & 0xFFFF0000u), o3);
                }
                acc[u][0] = o0;
                acc[u][1] = o1;
                acc[u][2] = o2;
                acc[u][3] = o3;
            }
        }
        __syncthreads();
        // refill this buffer with block n + 2
        if (tid == 0 && n + 2 < cnt) {
            ++issued;
            mbar_arrive_expect_tx(&full[buf], 2 * TILE);
            bulk_load(kbuf + buf * TILE, kplane + static_cast<int64_t>(list[n + 2]) * BLK * D, TILE, &full[buf]);
            bulk_load(vbuf + buf * TILE, vplane + static_cast<int64_t>(list[n + 2]) * BLK * D, TILE, &full[buf]);
        }
    }
    // partial: [gh][D] o, then m, l
    float* part = p.part + ((static_cast<int64_t>(b) * p.Hsel + hs) * p.splits + split) * gh * (D + 2);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int e = tid + kDecThreads * u;
        if (e < gh * CHUNKS) {
            const int hh = e / CHUNKS, dq = e % CHUNKS;
            float* dst = part + hh * (D + 2) + dq * 4;
            dst[0] = acc[u][0];
            dst[1] = acc[u][1];
            dst[2] = acc[u][2];
            dst[3] = acc[u][3];
        }
    }
    if (tid < gh) {
        part[tid * (D + 2) + D] = (ok && cnt > 0) ? m_run[tid] : -INFINITY;
        part[tid * (D + 2) + D + 1] = (ok && cnt > 0) ? l_run[tid] : 0.f;
    }
    // in-flight copies land before the CTA exits (only after a failed wait can any be pending)
    if (tid == 0 && !ok) {
        for (int u = n; u < issued; ++u) mbar_wait(&full[u & 1], (u >> 1) & 1, p.status, detail_base | 0x02u);
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
    const size_t tile = static_cast<size_t>(BLK) * D * 2;
    const size_t smem = 4 * tile + (8 * D + 8 * BLK + 24) * sizeof(float) + static_cast<size_t>(p.bps) * 4;
    dim3 grid(p.splits, p.Hsel, pl.B);
    cudaError_t e = cudaSuccess;
#define PISA_DECODE_CASE(DD, BB)                                                                              \
    if (D == DD && BLK == BB) {                                                                               \
        e = cudaFuncSetAttribute(attn_decode_kernel<DD, BB>, cudaFuncAttributeMaxDynamicSharedMemorySize,    \
                                 static_cast<int>(smem));                                                    \
        if (e == cudaSuccess) attn_decode_kernel<DD, BB><<<grid, kDecThreads, smem, st>>>(p);                \
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
