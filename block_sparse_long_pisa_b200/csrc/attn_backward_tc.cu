// Backward column pass on the tensor cores (sm_100a): dK and dV of one 64-key
// block through a fixed selection (PISA page, section "Ce que cela change pour
// vous": the sparse kernels serve training; the selection has no gradient).
//
// One CTA per (batch, KV head, key block j). Its inverse list (the query blocks
// and query heads whose selection holds j, ascending) is taken two entries at a
// time: a tile of 128 query rows. Per tile, with the forward's LSE and
// Delta = rowsum(dO * O):
//   S  = Q K_j^T,  dP = dO V_j^T            tcgen05, M = 128 rows, N = 64 keys, fp32 in TMEM
//   P  = exp(scale S - LSE),  dS = P (dP - Delta)   (elementwise warps, bf16 into shared memory)
//   dV_j^T += dO^T P,  dK_j^T += Q^T dS     tcgen05, M = 128 (head dim), N = 64 keys, K = 128 rows
// dK = scale dK_j. The two accumulators stay in TMEM for the whole list and are written once, so
// the result does not depend on timing (no atomics).
//
// A 64-wide operand costs a tcgen05 MMA as much as a 128-wide one on this part (measured: M128
// N64 and M64 N128 both take the cycles of M128 N128), so these MMAs run at half the peak rate;
// a 64-key block leaves no 128-wide dimension here except the rows and the head dim.
//
// Roles: warps 0-7 elementwise (thread = query row = TMEM lane of quadrant w % 4, keys 32 (w / 4)
// onwards; in the epilogue, head-dim lane), warp 8 TMA producer (K_j and V_j once, then Q and dO
// rows of every tile into a 2-stage ring), warp 9 MMA issue (one lane) and TMEM allocation.
// S/dP and P/dS are double-buffered. The MMAs go in rounds of two tiles: S and dP of both, then
// dV, dK of both, so the copy that refills a stage (which waits for that stage's dV, dK MMAs)
// overlaps the other tile's MMAs. Every wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>

#include "pisa_device.cuh"

namespace pisa {

namespace {

constexpr int kTD = 128;                        // head dim
constexpr int kTB = 64;                         // keys per block
constexpr int kDS = kTD / 64;                   // 128-byte column tiles along the head dim
constexpr uint32_t kSub = 128 * 128;            // [128 rows x 128 B] tile
constexpr uint32_t kKSub = kTB * 128;           // [64 keys x 128 B] tile
constexpr uint32_t kKVBytes = kDS * kKSub;      // K_j or V_j
constexpr uint32_t kQOBytes = kDS * kSub;       // the Q or the dO rows of one tile
constexpr uint32_t kPDBytes = 128 * 128;        // P or dS of one tile: [128 rows x 64 keys] bf16
constexpr int kNst = 2;
constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kKVBytes;
constexpr uint32_t kOffQ = 2 * kKVBytes;                  // stage s: Q, then dO
constexpr uint32_t kOffP = kOffQ + kNst * 2 * kQOBytes;   // stage s: P, then dS
constexpr uint32_t kOffAux = kOffP + kNst * 2 * kPDBytes;
constexpr uint32_t kSmem = 1024 + kOffAux + 256;
constexpr uint32_t kColS = 0;     // S of buffer s at kColS + 64 s
constexpr uint32_t kColDP = 128;  // dP of buffer s at kColDP + 64 s
constexpr uint32_t kColDV = 256;  // dV_j^T: lane = head dim, column = key
constexpr uint32_t kColDK = 320;  // dK_j^T
constexpr int kEwThreads = 256;  // elementwise threads: two per query row
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kThreads = 320;
static_assert(kSmem <= 232448, "shared memory budget");
static_assert(kSmem < (1 << 18), "descriptor start addresses below 2^18");

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                       const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + kOffAux);
    uint64_t* kv_full = bars;                 // 1    K_j and V_j landed
    uint64_t* qo_full = kv_full + 1;          // kNst Q and dO rows of the tile landed
    uint64_t* qo_empty = qo_full + kNst;      // kNst dV, dK MMAs of the tile done: Q/dO stage and P/dS free
    uint64_t* sdp_full = qo_empty + kNst;     // kNst S and dP of the tile in TMEM
    uint64_t* sdp_read = sdp_full + kNst;     // kNst the elementwise warps read S and dP (256 arrivals)
    uint64_t* p_ready = sdp_read + kNst;      // kNst P and dS in shared memory (256 arrivals)
    uint64_t* mma_final = p_ready + kNst;     // 1
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_final + 1);

    const int j = static_cast<int>(blockIdx.x), kvh = static_cast<int>(blockIdx.y), b = static_cast<int>(blockIdx.z);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int plane = b * p.Hkv + kvh;
    const int32_t* offs = p.counts + static_cast<int64_t>(plane) * (p.n0 + 1);
    const int32_t* ent = p.entries + static_cast<int64_t>(plane) * p.max_entries;
    const int e_lo = offs[j], e_hi = offs[j + 1];
    const int ntiles = (e_hi - e_lo + 1) / 2;
    const int64_t kbase = static_cast<int64_t>(plane) * p.N + static_cast<int64_t>(j) * kTB;
    const uint32_t detail_base = kKernAttnBackward << 8;
    // list entry of half `half` of tile t; a missing second entry repeats the last one (its rows
    // get P = dS = 0, and repeating real rows keeps every operand finite)
    auto entry_of = [&](int t, int half) -> int {
        const int e = e_lo + 2 * t + half;
        return e < e_hi ? e : e_hi - 1;
    };

    if (warp == kProducerWarp && lane == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < kNst; ++s) {
            mbar_init(qo_full + s, 1);
            mbar_init(qo_empty + s, 1);
            mbar_init(sdp_full + s, 1);
            mbar_init(sdp_read + s, kEwThreads);
            mbar_init(p_ready + s, kEwThreads);
        }
        mbar_init(mma_final, 1);
        fence_barrier_init();
    }
    if (warp == kMmaWarp) tmem_alloc(tmem_slot, 512);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;

    int issued_last = -1;  // producer lane 0: last tile whose copies it started
    if (warp == kProducerWarp) {
        if (lane == 0 && ntiles > 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmdO);
            mbar_arrive_expect_tx(kv_full, 2 * kKVBytes);
#pragma unroll
            for (int s = 0; s < kDS; ++s) {
                tma_load_2d(base + kOffK + s * kKSub, &tmK, s * 64, static_cast<int32_t>(kbase), kv_full);
                tma_load_2d(base + kOffV + s * kKSub, &tmV, s * 64, static_cast<int32_t>(kbase), kv_full);
            }
            for (int t = 0; t < ntiles; ++t) {
                const int st = t % kNst, use = t / kNst;
                if (!mbar_wait(qo_empty + st, (use & 1) ^ 1, p.status, detail_base | 0x01u)) break;
                mbar_arrive_expect_tx(qo_full + st, 2 * kQOBytes);
                uint8_t* sq = base + kOffQ + st * 2 * kQOBytes;
                for (int half = 0; half < 2; ++half) {
                    const int code = ent[entry_of(t, half)];
                    const int i = code / p.g, head = kvh * p.g + code % p.g;
                    const int32_t qrow = static_cast<int32_t>((static_cast<int64_t>(b) * p.Hq + head) * p.N +
                                                              static_cast<int64_t>(i) * kTB);
#pragma unroll
                    for (int s = 0; s < kDS; ++s) {
                        tma_load_2d(sq + s * kSub + half * kTB * 128, &tmQ, s * 64, qrow, qo_full + st);
                        tma_load_2d(sq + kQOBytes + s * kSub + half * kTB * 128, &tmdO, s * 64, qrow, qo_full + st);
                    }
                }
                issued_last = t;
            }
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        if (lane == 0 && ntiles > 0) {
            constexpr uint32_t idesc_s = idesc_bf16_f32(128, kTB, 0, 0);  // S, dP: A and B K-major
            constexpr uint32_t idesc_g = idesc_bf16_f32(128, kTB, 1, 1);  // dV^T, dK^T: A and B MN-major
            const uint32_t sK = smem_u32(base + kOffK), sV = smem_u32(base + kOffV);
            bool ok = mbar_wait(kv_full, 0, p.status, detail_base | 0x10u);
            for (int r0 = 0; ok && r0 < ntiles; r0 += kNst) {
                const int r1 = min(r0 + kNst, ntiles);
                for (int t = r0; ok && t < r1; ++t) {
                    const int st = t % kNst;
                    const uint32_t ph = (t / kNst) & 1;
                    if (!(ok = mbar_wait(qo_full + st, ph, p.status, detail_base | 0x11u))) break;
                    if (!(ok = mbar_wait(sdp_read + st, ph ^ 1, p.status, detail_base | 0x12u))) break;
                    tc_fence_after();
                    const uint32_t sQ = smem_u32(base + kOffQ + st * 2 * kQOBytes), sO = sQ + kQOBytes;
#pragma unroll
                    for (int ks = 0; ks < kTD / 16; ++ks) {
                        const uint32_t oa = (ks / 4) * kSub + (ks % 4) * 32, ob = (ks / 4) * kKSub + (ks % 4) * 32;
                        mma_bf16_ss(tm + kColS + 64 * st, smem_desc_sw128(sQ + oa, 16, 1024),
                                    smem_desc_sw128(sK + ob, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
                    }
#pragma unroll
                    for (int ks = 0; ks < kTD / 16; ++ks) {
                        const uint32_t oa = (ks / 4) * kSub + (ks % 4) * 32, ob = (ks / 4) * kKSub + (ks % 4) * 32;
                        mma_bf16_ss(tm + kColDP + 64 * st, smem_desc_sw128(sO + oa, 16, 1024),
                                    smem_desc_sw128(sV + ob, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(sdp_full + st);
                }
                // dV^T += dO^T P and dK^T += Q^T dS: the head dim is M (two 64-column tiles LBO
                // apart), the 128 rows are K (16 per MMA), the keys N
                for (int u = r0; ok && u < r1; ++u) {
                    const int su = u % kNst;
                    if (!(ok = mbar_wait(p_ready + su, (u / kNst) & 1, p.status, detail_base | 0x13u))) break;
                    tc_fence_after();
                    const uint32_t sQ = smem_u32(base + kOffQ + su * 2 * kQOBytes), sO = sQ + kQOBytes;
                    const uint32_t sP = smem_u32(base + kOffP + su * 2 * kPDBytes), sdS = sP + kPDBytes;
#pragma unroll
                    for (int ks = 0; ks < 128 / 16; ++ks) {
                        const uint32_t ro = ks * 16 * 128;
                        mma_bf16_ss(tm + kColDV, smem_desc_sw128(sO + ro, kSub, 1024),
                                    smem_desc_sw128(sP + ro, kPDBytes, 1024), idesc_g, (u > 0 || ks > 0) ? 1u : 0u);
                    }
#pragma unroll
                    for (int ks = 0; ks < 128 / 16; ++ks) {
                        const uint32_t ro = ks * 16 * 128;
                        mma_bf16_ss(tm + kColDK, smem_desc_sw128(sQ + ro, kSub, 1024),
                                    smem_desc_sw128(sdS + ro, kPDBytes, 1024), idesc_g, (u > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(qo_empty + su);
                }
            }
            // every MMA issued so far completes before the epilogue reads dV^T and dK^T
            mma_commit(mma_final);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- elementwise warps
        const int r = (warp % 4) * 32 + lane;  // row of the tile (TMEM lane)
        const int ch = warp / 4;               // this thread's 32 keys: 32 ch ..
        const int half = r / kTB, tr = r % kTB;
        const uint32_t lane_base = static_cast<uint32_t>((warp % 4) * 32) << 16;
        const float c2 = p.scale_log2;
        bool ok = true;
        for (int t = 0; t < ntiles; ++t) {
            const int st = t % kNst;
            const uint32_t ph = (t / kNst) & 1;
            const int e = e_lo + 2 * t + half;
            const bool valid = e < e_hi;
            const int code = ent[entry_of(t, half)];
            const int i = code / p.g, head = kvh * p.g + code % p.g;
            const int64_t row = (static_cast<int64_t>(b) * p.Hq + head) * p.N + static_cast<int64_t>(i) * kTB + tr;
            const float lse2 = p.lse[row] * 1.4426950408889634f;
            const float dlt = p.delta[row];
            // keys from mask_from on are masked (causal diagonal block), all of them for a padding row
            const int mask_from = !valid ? 0 : ((p.causal && i == j) ? tr + 1 : kTB);
            if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(sdp_full + st, ph, p.status, detail_base | 0x20u));
            tc_fence_after();
            uint32_t pk[16], dk[16];  // P and dS of this thread's 32 keys, bf16 pairs
            {
                uint32_t sv[32], dv[32];
                tmem_ld32(tm + lane_base + kColS + 64 * st + 32 * ch, sv);
                tmem_ld32(tm + lane_base + kColDP + 64 * st + 32 * ch, dv);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int u0 = 32 * ch + 2 * k;
                    float p0 = fast_exp2(__uint_as_float(sv[2 * k]) * c2 - lse2);
                    float p1 = fast_exp2(__uint_as_float(sv[2 * k + 1]) * c2 - lse2);
                    if (u0 >= mask_from) p0 = 0.f;
                    if (u0 + 1 >= mask_from) p1 = 0.f;
                    const float d0 = p0 * (__uint_as_float(dv[2 * k]) - dlt);
                    const float d1 = p1 * (__uint_as_float(dv[2 * k + 1]) - dlt);
                    pk[k] = pack_bf16x2(p0, p1);
                    dk[k] = pack_bf16x2(d0, d1);
                }
            }
            tc_fence_before();
            mbar_arrive(sdp_read + st);  // the MMA warp may refill this S/dP buffer
            // this P/dS buffer was last read by the dV, dK MMAs of tile t - 2
            if (ok && t >= kNst)
                ok = __all_sync(0xFFFFFFFFu,
                                mbar_wait(qo_empty + st, ((t / kNst) - 1) & 1, p.status, detail_base | 0x21u));
            const uint32_t sP = smem_u32(base + kOffP + st * 2 * kPDBytes), sdS = sP + kPDBytes;
#pragma unroll
            for (int q = 0; q < 4; ++q) {  // 16-byte chunks 4 ch + q of the row, 128-byte swizzle
                const int c8 = 4 * ch + q;
                const uint32_t off = r * 128 + ((c8 ^ (r & 7)) << 4);
                st_shared_v4(sP + off, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                st_shared_v4(sdS + off, dk[4 * q], dk[4 * q + 1], dk[4 * q + 2], dk[4 * q + 3]);
            }
            fence_proxy_async_smem();
            mbar_arrive(p_ready + st);
        }
        // ---------------------------------------------------------------- epilogue
        // TMEM lane = head dim d; this warp writes the block's keys 32 ch .. 32 ch + 31
        if (ok && ntiles > 0) ok = __all_sync(0xFFFFFFFFu, mbar_wait(mma_final, 0, p.status, detail_base | 0x22u));
        tc_fence_after();
        const int d = r;
        __nv_bfloat16* dv_col = p.dV + kbase * kTD + d;
        __nv_bfloat16* dk_col = p.dK + kbase * kTD + d;
        const float sc = p.scale;
        uint32_t v[32], k[32];
        if (ntiles > 0) {
            tmem_ld32(tm + lane_base + kColDV + 32 * ch, v);
            tmem_ld32(tm + lane_base + kColDK + 32 * ch, k);
            tmem_wait_ld();
        } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) v[x] = k[x] = 0u;
        }
        if (ok) {
#pragma unroll
            for (int x = 0; x < 32; ++x) {
                const int64_t key = 32 * ch + x;
                dv_col[key * kTD] = __float2bfloat16_rn(__uint_as_float(v[x]));
                dk_col[key * kTD] = __float2bfloat16_rn(__uint_as_float(k[x]) * sc);
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncthreads();
    if (warp == kProducerWarp && lane == 0 && ntiles > 0) {
        // every TMA copy this CTA started has landed before shared memory is released
        mbar_wait(kv_full, 0, p.status, detail_base | 0x30u);
        for (int t = issued_last - kNst + 1; t <= issued_last; ++t)
            if (t >= 0) mbar_wait(qo_full + t % kNst, (t / kNst) & 1, p.status, detail_base | 0x31u);
    }
    if (warp == kMmaWarp && lane == 0 && ntiles > 0) mbar_wait(mma_final, 0, p.status, detail_base | 0x32u);
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

bool bwd_dkdv_tc_supported(const BwdParams& p) { return p.D == kTD && p.blk == kTB; }

bool launch_bwd_dkdv_tc(const BwdParams& p, int32_t batch, cudaStream_t st) {
    if (!bwd_dkdv_tc_supported(p)) return false;
    CUtensorMap tq, tdo, tk, tv;
    const int64_t qrows = static_cast<int64_t>(batch) * p.Hq * p.N;
    const int64_t krows = static_cast<int64_t>(batch) * p.Hkv * p.N;
    if (!make_tmap_2d(&tq, p.Q, qrows, kTD, kTB) || !make_tmap_2d(&tdo, p.dO, qrows, kTD, kTB) ||
        !make_tmap_2d(&tk, p.K, krows, kTD, kTB) || !make_tmap_2d(&tv, p.V, krows, kTD, kTB))
        return false;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kSmem)) != cudaSuccess)
            return false;
        configured = true;
    }
    bwd_dkdv_tc_kernel<<<dim3(p.n0, p.Hkv, batch), kThreads, kSmem, st>>>(tq, tdo, tk, tv, p);
    return cudaGetLastError() == cudaSuccess;
}

}  // namespace pisa
