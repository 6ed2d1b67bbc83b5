// Backward on the tensor cores (sm_100a), both passes, through a fixed selection
// (PISA page, section "Ce que cela change pour vous": the sparse kernels serve
// training; the selection has no gradient). Head dim 64 or 128; 64- or 128-key
// blocks.
//
// Column pass: dK and dV of 64 keys. One CTA per (batch, KV head, key block j)
// for 64-key blocks, per (batch, KV head, half of key block j) for 128-key
// blocks. Its inverse list (the query blocks and query heads whose selection
// holds j, ascending) makes tiles of 128 query rows: two entries of 64-row query
// blocks, or one 128-row query block. Per tile, with the forward's LSE and
// Delta = rowsum(dO * O):
//   S  = Q K_j^T,  dP = dO V_j^T            tcgen05, M = 128 rows, N = 64 keys, fp32 in TMEM
//                                           (separate barriers: P is computed while dP forms)
//   P  = exp(scale S - LSE),  dS = P (dP - Delta)   (elementwise warps, bf16 into shared memory)
//   dV_j^T += dO^T P,  dK_j^T += Q^T dS     tcgen05, M = 128 (head dim), N = 64 keys, K = 128 rows
// dK = scale dK_j. The two accumulators stay in TMEM for the whole list and are written once, so
// the result does not depend on timing (no atomics).
//
// A 64-wide operand costs a tcgen05 MMA as much as a 128-wide one on this part (measured: M128
// N64 and M64 N128 both take the cycles of M128 N128), so these MMAs run at half the peak rate;
// a 64-key block leaves no 128-wide dimension here except the rows and the head dim. Per tile
// the MMAs read 192 KB of shared memory (6 KB each), the copies write 64 KB and P, dS 32 KB:
// shared-memory bandwidth (128 B per clock) bounds the pass near 2,250 cycles per tile.
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

constexpr int kTD = 128;                        // largest head dim (the shared-memory layout's)
constexpr int kTB = 64;                         // keys per CTA
constexpr int kDS = kTD / 64;                   // 128-byte column tiles along the head dim
constexpr uint32_t kSub = 128 * 128;            // [128 rows x 128 B] tile
constexpr uint32_t kKSub = kTB * 128;           // [64 keys x 128 B] tile
constexpr uint32_t kKVBytes = kDS * kKSub;      // K_j or V_j
constexpr uint32_t kQOBytes = kDS * kSub;       // the Q or the dO rows of one tile
constexpr uint32_t kPDBytes = 128 * 128;        // P or dS of one tile: [128 rows x 64 keys] bf16
// A descriptor moved by `bytes` (a multiple of 16): the start-address field holds address / 16
// in 14 bits and shared memory ends below 2^18 bytes, so the add never carries out of it. The
// MMA lane forms each operand's descriptor once and only adds offsets, which keeps its
// instruction count per MMA small beside the busy elementwise warps on its sub-partition.
__device__ __forceinline__ uint64_t dmove(uint64_t desc, uint32_t bytes) { return desc + (bytes >> 4); }

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

template <int D, int BLK>
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
    uint64_t* s_full = qo_empty + kNst;       // kNst S of the tile in TMEM
    uint64_t* dp_full = s_full + kNst;        // kNst dP of the tile in TMEM
    uint64_t* sdp_read = dp_full + kNst;      // kNst the elementwise warps read S and dP (256 arrivals)
    uint64_t* p_ready = sdp_read + kNst;      // kNst P and dS in shared memory (256 arrivals)
    uint64_t* mma_final = p_ready + kNst;     // 1
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_final + 1);

    // 64 keys per CTA: key block j, or half jh of a 128-key block
    constexpr int HB = BLK / kTB;
    constexpr int DS = D / 64;  // 128-byte column tiles loaded per row
    const int j = static_cast<int>(blockIdx.x) / HB, jh = static_cast<int>(blockIdx.x) % HB;
    const int kvh = static_cast<int>(blockIdx.y), b = static_cast<int>(blockIdx.z);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int plane = b * p.Hkv + kvh;
    const int32_t* offs = p.counts + static_cast<int64_t>(plane) * (p.n0 + 1);
    const int32_t* ent = p.entries + static_cast<int64_t>(plane) * p.max_entries;
    const int e_lo = offs[j], e_hi = offs[j + 1];
    // a tile is 128 query rows: two entries of 64-row query blocks, or one 128-row query block
    // (its rows 0-63 as the first half, 64-127 as the second)
    const int ntiles = HB == 1 ? (e_hi - e_lo + 1) / 2 : e_hi - e_lo;
    const int64_t kbase = static_cast<int64_t>(plane) * p.N + static_cast<int64_t>(j) * BLK + jh * kTB;
    const uint32_t detail_base = kKernAttnBackward << 8;
    // list entry of half `half` of tile t; a missing second entry repeats the last one (its rows
    // get P = dS = 0, and repeating real rows keeps every operand finite)
    auto entry_of = [&](int t, int half) -> int {
        if (HB == 2) return e_lo + t;
        const int e = e_lo + 2 * t + half;
        return e < e_hi ? e : e_hi - 1;
    };

    if (warp == kProducerWarp && lane == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < kNst; ++s) {
            mbar_init(qo_full + s, 1);
            mbar_init(qo_empty + s, 1);
            mbar_init(s_full + s, 1);
            mbar_init(dp_full + s, 1);
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
            mbar_arrive_expect_tx(kv_full, 2 * DS * kKSub);
#pragma unroll
            for (int s = 0; s < DS; ++s) {
                tma_load_2d(base + kOffK + s * kKSub, &tmK, s * 64, static_cast<int32_t>(kbase), kv_full);
                tma_load_2d(base + kOffV + s * kKSub, &tmV, s * 64, static_cast<int32_t>(kbase), kv_full);
            }
            for (int t = 0; t < ntiles; ++t) {
                const int st = t % kNst, use = t / kNst;
                if (!mbar_wait(qo_empty + st, (use & 1) ^ 1, p.status, detail_base | 0x01u)) break;
                mbar_arrive_expect_tx(qo_full + st, 2 * 2 * DS * kTB * 128);
                uint8_t* sq = base + kOffQ + st * 2 * kQOBytes;
                for (int half = 0; half < 2; ++half) {
                    const int code = ent[entry_of(t, half)];
                    const int i = code / p.g, head = kvh * p.g + code % p.g;
                    const int32_t qrow = static_cast<int32_t>((static_cast<int64_t>(b) * p.Hq + head) * p.N +
                                                              static_cast<int64_t>(i) * BLK + (HB == 2 ? half * kTB : 0));
#pragma unroll
                    for (int s = 0; s < DS; ++s) {
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
            const uint32_t s0 = smem_u32(base);
            const uint64_t dK = smem_desc_sw128(s0 + kOffK, 16, 1024), dV = smem_desc_sw128(s0 + kOffV, 16, 1024);
            const uint64_t dQk = smem_desc_sw128(s0 + kOffQ, 16, 1024);         // Q / dO, K-major
            const uint64_t dQm = smem_desc_sw128(s0 + kOffQ, kSub, 1024);       // Q / dO, MN-major
            const uint64_t dPm = smem_desc_sw128(s0 + kOffP, kPDBytes, 1024);   // P / dS, MN-major
            bool ok = mbar_wait(kv_full, 0, p.status, detail_base | 0x10u);
            for (int r0 = 0; ok && r0 < ntiles; r0 += kNst) {
                const int r1 = min(r0 + kNst, ntiles);
                for (int t = r0; ok && t < r1; ++t) {
                    const int st = t % kNst;
                    const uint32_t ph = (t / kNst) & 1;
                    if (!(ok = mbar_wait(qo_full + st, ph, p.status, detail_base | 0x11u))) break;
                    if (!(ok = mbar_wait(sdp_read + st, ph ^ 1, p.status, detail_base | 0x12u))) break;
                    tc_fence_after();
                    const uint64_t dq = dmove(dQk, st * 2 * kQOBytes), dout = dmove(dq, kQOBytes);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t oa = (ks / 4) * kSub + (ks % 4) * 32, ob = (ks / 4) * kKSub + (ks % 4) * 32;
                        mma_bf16_ss(tm + kColS + 64 * st, dmove(dq, oa), dmove(dK, ob), idesc_s, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(s_full + st);  // the exponentials start while dP is formed
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t oa = (ks / 4) * kSub + (ks % 4) * 32, ob = (ks / 4) * kKSub + (ks % 4) * 32;
                        mma_bf16_ss(tm + kColDP + 64 * st, dmove(dout, oa), dmove(dV, ob), idesc_s, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(dp_full + st);
                }
                // dV^T += dO^T P and dK^T += Q^T dS: the head dim is M (two 64-column tiles LBO
                // apart), the 128 rows are K (16 per MMA), the keys N. At head dim 64 the second
                // tile is never loaded: M stays 128 (an M = 64 MMA takes as long), TMEM lanes
                // 64-127 receive products of whatever that shared memory holds, and are not read
                for (int u = r0; ok && u < r1; ++u) {
                    const int su = u % kNst;
                    if (!(ok = mbar_wait(p_ready + su, (u / kNst) & 1, p.status, detail_base | 0x13u))) break;
                    tc_fence_after();
                    const uint64_t dq = dmove(dQm, su * 2 * kQOBytes), dout = dmove(dq, kQOBytes);
                    const uint64_t dp = dmove(dPm, su * 2 * kPDBytes), dds = dmove(dp, kPDBytes);
#pragma unroll
                    for (int ks = 0; ks < 128 / 16; ++ks) {
                        const uint32_t ro = ks * 16 * 128;
                        mma_bf16_ss(tm + kColDV, dmove(dout, ro), dmove(dp, ro), idesc_g, (u > 0 || ks > 0) ? 1u : 0u);
                    }
#pragma unroll
                    for (int ks = 0; ks < 128 / 16; ++ks) {
                        const uint32_t ro = ks * 16 * 128;
                        mma_bf16_ss(tm + kColDK, dmove(dq, ro), dmove(dds, ro), idesc_g, (u > 0 || ks > 0) ? 1u : 0u);
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
            const bool valid = HB == 2 || e_lo + 2 * t + half < e_hi;
            const int code = ent[entry_of(t, half)];
            const int i = code / p.g, head = kvh * p.g + code % p.g;
            const int qt = (HB == 2 ? half * kTB : 0) + tr;  // query position in its block
            const int64_t row = (static_cast<int64_t>(b) * p.Hq + head) * p.N + static_cast<int64_t>(i) * BLK + qt;
            const float lse2 = p.lse[row] * 1.4426950408889634f;
            const float dlt = p.delta[row];
            // keys from mask_from on are masked (causal diagonal block: key jh * 64 + u is visible
            // from query position qt when jh * 64 + u <= qt), all of them for a padding row
            const int mask_from = !valid ? 0 : ((p.causal && i == j) ? max(0, min(kTB, qt - jh * kTB + 1)) : kTB);
            if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(s_full + st, ph, p.status, detail_base | 0x20u));
            tc_fence_after();
            uint32_t pk[16], dk[16];  // P and dS of this thread's 32 keys, bf16 pairs
            {
                float pv[32];
                uint32_t sv[32];
                tmem_ld32(tm + lane_base + kColS + 64 * st + 32 * ch, sv);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) {
                    const float e = fast_exp2(__uint_as_float(sv[k]) * c2 - lse2);
                    pv[k] = 32 * ch + k >= mask_from ? 0.f : e;
                }
#pragma unroll
                for (int k = 0; k < 16; ++k) pk[k] = pack_bf16x2(pv[2 * k], pv[2 * k + 1]);
                uint32_t dv[32];
                if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(dp_full + st, ph, p.status, detail_base | 0x23u));
                tc_fence_after();
                tmem_ld32(tm + lane_base + kColDP + 64 * st + 32 * ch, dv);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    dk[k] = pack_bf16x2(pv[2 * k] * (__uint_as_float(dv[2 * k]) - dlt),
                                        pv[2 * k + 1] * (__uint_as_float(dv[2 * k + 1]) - dlt));
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
        __nv_bfloat16* dv_col = p.dV + kbase * D + d;
        __nv_bfloat16* dk_col = p.dK + kbase * D + d;
        const float sc = p.scale;
        uint32_t v[32], k[32];
        if (ntiles > 0 && (warp % 4) * 32 < D) {
            tmem_ld32(tm + lane_base + kColDV + 32 * ch, v);
            tmem_ld32(tm + lane_base + kColDK + 32 * ch, k);
            tmem_wait_ld();
        } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) v[x] = k[x] = 0u;
        }
        if (ok && d < D) {
#pragma unroll
            for (int x = 0; x < 32; ++x) {
                const int64_t key = 32 * ch + x;
                dv_col[key * D] = __float2bfloat16_rn(__uint_as_float(v[x]));
                dk_col[key * D] = __float2bfloat16_rn(__uint_as_float(k[x]) * sc);
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

// ---------------------------------------------------------------- row pass: dQ
//
// One CTA per (batch, selection row, query block, pair of query heads): 128 query rows (two
// heads x 64 tokens; one head and 64 valid rows under per-query-head selection) that share the
// block list. The selected blocks are taken in groups of 128 keys (two blocks), as in the
// forward. Per group g:
//   S = Q K_g^T, dP = dO V_g^T        tcgen05 SS, M = 128 rows, N = 128 keys, fp32 in TMEM
//   dS = P (dP - Delta), P = exp(scale S - LSE)   (elementwise warps, written as bf16 over the
//                                      S columns already read: keys 32 c .. 32 c + 31 into
//                                      columns 32 c .. 32 c + 15)
//   dQ += dS K_g                       tcgen05 with A = dS from TMEM, B = K_g (MN-major)
// dQ = scale dQ at the end. S is double-buffered in TMEM (S 2 x 128, dP 128, dQ 128 columns), so
// group g+1's S and dP are formed while group g's dS is computed and used; the K ring has three
// stages (K is read by S(g) and by dQ(g)), the V ring two.
// Roles: warps 0-15 elementwise (four per row: keys 32 (w / 4) .. of each group, whose dS goes
// into the first 16 of the 32 S columns the warp read; in the epilogue, head-dim columns
// 32 (w / 4) ..), warp 16 producer (block list, Q and dO once, K lane 0, V lane 1), warp 17 MMA
// issue and TMEM allocation.
namespace {

constexpr int kRD = 128;                       // largest head dim (the shared-memory layout's)
constexpr int kRDS = kRD / 64;
constexpr uint32_t kRSub = 128 * 128;          // [128 rows x 128 B]
constexpr uint32_t kRTile = kRDS * kRSub;      // Q, dO, or one 128-key K / V group: 32 KB
constexpr int kRNstK = 3;
constexpr int kRNstV = 2;
constexpr uint32_t kROffQ = 0;
constexpr uint32_t kROffO = kRTile;
constexpr uint32_t kROffK = 2 * kRTile;
constexpr uint32_t kROffV = kROffK + kRNstK * kRTile;
constexpr uint32_t kROffAux = kROffV + kRNstV * kRTile;
constexpr int kRMaxList = kMaxPrefillTopk;
constexpr uint32_t kRAux = 256 + kRMaxList * 4;
constexpr uint32_t kRSmem = 1024 + kROffAux + kRAux;
constexpr uint32_t kRColS = 0;     // S / dS of buffer s at 128 s
constexpr uint32_t kRColDP = 256;
constexpr uint32_t kRColDQ = 384;
constexpr int kREwThreads = 512;
constexpr int kRProducerWarp = 16;
constexpr int kRMmaWarp = 17;
constexpr int kRThreads = 576;
static_assert(kRSmem <= 232448, "shared memory budget");
static_assert(kRSmem < (1 << 18), "descriptor start addresses below 2^18");

}  // namespace

template <int D, int BLK>
__global__ void __launch_bounds__(kRThreads, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                     const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const BwdParams p, const int gh, const int chunks) {
    constexpr int GB = 128 / BLK;  // selected blocks per 128-key group
    constexpr int DS = D / 64;     // 128-byte column tiles loaded per row
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* aux = base + kROffAux;
    uint64_t* bars = reinterpret_cast<uint64_t*>(aux);
    uint64_t* q_full = bars;                   // 1     Q and dO rows landed
    uint64_t* k_full = q_full + 1;             // NstK
    uint64_t* k_empty = k_full + kRNstK;       // NstK  S and dQ MMAs of the group done
    uint64_t* v_full = k_empty + kRNstK;       // NstV
    uint64_t* v_empty = v_full + kRNstV;       // NstV  dP MMAs of the group done
    uint64_t* sdp_full = v_empty + kRNstV;     // 1     S and dP of the group in TMEM
    uint64_t* dp_read = sdp_full + 1;          // 1     elementwise warps read S and dP (512 arrivals)
    uint64_t* ds_ready = dp_read + 1;          // 2     dS of S buffer s in TMEM (512 arrivals)
    uint64_t* dq_done = ds_ready + 2;          // 1     dQ MMAs of the group done
    uint64_t* mma_final = dq_done + 1;         // 1     teardown: every MMA issued has completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_final + 1);
    int32_t* s_nsel = reinterpret_cast<int32_t*>(tmem_slot + 1);
    int32_t* s_diag = s_nsel + 1;
    int32_t* list = reinterpret_cast<int32_t*>(aux + 256);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = p.nqb - 1 - static_cast<int>(blockIdx.x);  // longest rows first
    const int hs = static_cast<int>(blockIdx.y) / chunks;
    const int chunk = static_cast<int>(blockIdx.y) % chunks;
    const int b = static_cast<int>(blockIdx.z);
    const int kvh = p.per_qhead ? hs / p.g : hs;
    const int head0 = p.per_qhead ? hs : kvh * p.g + chunk * gh;
    const uint32_t detail_base = (kKernAttnBackward << 8) | 0x80u;

    if (warp == kRProducerWarp && lane == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < kRNstK; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(k_empty + s, 1);
        }
        for (int s = 0; s < kRNstV; ++s) {
            mbar_init(v_full + s, 1);
            mbar_init(v_empty + s, 1);
        }
        mbar_init(sdp_full, 1);
        mbar_init(dp_read, kREwThreads);
        mbar_init(ds_ready, kREwThreads);
        mbar_init(ds_ready + 1, kREwThreads);
        mbar_init(dq_done, 1);
        mbar_init(mma_final, 1);
        fence_barrier_init();
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmdO);
        mbar_arrive_expect_tx(q_full, static_cast<uint32_t>(2 * gh * BLK * D * 2));
        for (int hh = 0; hh < gh; ++hh) {
            const int32_t qrow = static_cast<int32_t>((static_cast<int64_t>(b) * p.Hq + head0 + hh) * p.N +
                                                      static_cast<int64_t>(i) * BLK);
#pragma unroll
            for (int s = 0; s < DS; ++s) {
                tma_load_2d(base + kROffQ + s * kRSub + hh * BLK * 128, &tmQ, s * 64, qrow, q_full);
                tma_load_2d(base + kROffO + s * kRSub + hh * BLK * 128, &tmdO, s * 64, qrow, q_full);
            }
        }
    }
    if (warp == kRMmaWarp) tmem_alloc(tmem_slot, 512);
    if (warp == kRProducerWarp) {
        // compact the block row: eligible entries in order; the diagonal block's position
        const int32_t* row = p.idx + ((static_cast<int64_t>(b) * p.Hsel + hs) * p.nqb + i) * p.topk;
        int cnt = 0, diag = -1;
        for (int t0 = 0; t0 < p.topk; t0 += 32) {
            const int t = t0 + lane;
            const int32_t jj = t < p.topk ? row[t] : -1;
            const bool ok = jj >= 0 && jj < p.n0 && (!p.causal || jj <= i);
            const uint32_t m = __ballot_sync(0xFFFFFFFFu, ok);
            const int pos = cnt + __popc(m & ((1u << lane) - 1u));
            if (ok && pos < kRMaxList) list[pos] = jj;
            const uint32_t md = __ballot_sync(0xFFFFFFFFu, p.causal && ok && jj == i && pos < kRMaxList);
            if (diag < 0 && md != 0u) diag = __shfl_sync(0xFFFFFFFFu, pos, __ffs(md) - 1);
            cnt += __popc(m);
        }
        if (lane == 0) {
            *s_nsel = cnt < kRMaxList ? cnt : kRMaxList;
            *s_diag = diag;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    const int nsel = *s_nsel;
    const int ngroups = (nsel + GB - 1) / GB;
    const int diag_pos = *s_diag;

    int issued_last = -1;
    if (warp == kRProducerWarp) {
        if (lane < 2 && ngroups > 0) {
            const bool is_k = lane == 0;
            const void* tmap = is_k ? static_cast<const void*>(&tmK) : static_cast<const void*>(&tmV);
            uint8_t* ring = base + (is_k ? kROffK : kROffV);
            uint64_t* full = is_k ? k_full : v_full;
            uint64_t* empty = is_k ? k_empty : v_empty;
            const int nst = is_k ? kRNstK : kRNstV;
            prefetch_tmap(tmap);
            for (int g = 0; g < ngroups; ++g) {
                const int st = g % nst, use = g / nst;
                if (!mbar_wait(empty + st, (use & 1) ^ 1, p.status, detail_base | (is_k ? 0x01u : 0x02u))) break;
                const int nb = min(GB, nsel - GB * g);
                mbar_arrive_expect_tx(full + st, static_cast<uint32_t>(nb * BLK * D * 2));
                for (int u = 0; u < nb; ++u) {
                    const int32_t krow = static_cast<int32_t>((static_cast<int64_t>(b) * p.Hkv + kvh) * p.N +
                                                              static_cast<int64_t>(list[GB * g + u]) * BLK);
#pragma unroll
                    for (int s = 0; s < DS; ++s)
                        tma_load_2d(ring + st * kRTile + s * kRSub + u * BLK * 128, tmap, s * 64, krow, full + st);
                }
                issued_last = g;
            }
        }
        __syncwarp();
    } else if (warp == kRMmaWarp) {
        if (lane == 0 && ngroups > 0) {
            const uint32_t s0 = smem_u32(base);
            const uint64_t dQk = smem_desc_sw128(s0 + kROffQ, 16, 1024), dOk = smem_desc_sw128(s0 + kROffO, 16, 1024);
            const uint64_t dKk = smem_desc_sw128(s0 + kROffK, 16, 1024), dVk = smem_desc_sw128(s0 + kROffV, 16, 1024);
            const uint64_t dKm = smem_desc_sw128(s0 + kROffK, kRSub, 1024);  // K as the MN-major B of dS.K
            constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, 0, 1);
            bool ok = mbar_wait(q_full, 0, p.status, detail_base | 0x10u);
            auto ncols_of = [&](int g) { return min(GB, nsel - GB * g) * BLK; };
            // dP(g) = dO V_g^T into the dP columns (after the elementwise warps read dP(g-1)) and
            // S(g) = Q K_g^T into S buffer g % 2 (after dQ(g-2) read the dS it held); the two chains
            // alternate so the tensor pipe runs them at its independent-MMA rate
            auto issue_sdp = [&](int g) -> bool {
                const int sv = g % kRNstV, sk = g % kRNstK;
                if (!mbar_wait(v_full + sv, (g / kRNstV) & 1, p.status, detail_base | 0x11u)) return false;
                if (g > 0 && !mbar_wait(dp_read, (g - 1) & 1, p.status, detail_base | 0x12u)) return false;
                if (!mbar_wait(k_full + sk, (g / kRNstK) & 1, p.status, detail_base | 0x13u)) return false;
                if (g > 1 && !mbar_wait(dq_done, (g - 2) & 1, p.status, detail_base | 0x14u)) return false;
                tc_fence_after();
                const uint32_t id = idesc_bf16_f32(128, ncols_of(g), 0, 0);
                const uint64_t dv = dmove(dVk, sv * kRTile), dk = dmove(dKk, sk * kRTile);
                const uint32_t s_col = tm + kRColS + 128 * (g % 2);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks / 4) * kRSub + (ks % 4) * 32;
                    mma_bf16_ss(tm + kRColDP, dmove(dOk, off), dmove(dv, off), id, ks > 0 ? 1u : 0u);
                    mma_bf16_ss(s_col, dmove(dQk, off), dmove(dk, off), id, ks > 0 ? 1u : 0u);
                }
                mma_commit(v_empty + sv);
                mma_commit(sdp_full);
                return true;
            };
            // dQ += dS(g) K_g (dS in TMEM: keys 32 c .. 32 c + 31 in columns 32 c .. 32 c + 15)
            auto issue_dq = [&](int g) -> bool {
                const int st = g % kRNstK;
                if (!mbar_wait(ds_ready + g % 2, (g / 2) & 1, p.status, detail_base | 0x15u)) return false;
                tc_fence_after();
                const int nks = ncols_of(g) / 16;
                const uint32_t a_tmem = tm + kRColS + 128 * (g % 2);
                const uint64_t b0 = dmove(dKm, st * kRTile);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    if (ks < nks) {
                        const uint32_t acol = (ks / 2) * 32 + (ks % 2) * 8;
                        const uint32_t boff = static_cast<uint32_t>((ks * 16 * 128) >> 4);
                        mma_bf16_ts(tm + kRColDQ, a_tmem + acol, b0 + boff, idesc_dq, (g > 0 || ks > 0) ? 1u : 0u);
                    }
                }
                mma_commit(dq_done);
                mma_commit(k_empty + st);
                return true;
            };
            // dP(g+1) and S(g+1) go ahead of dQ(g), so the tensor pipe forms the next group's
            // scores while the elementwise warps work on this one
            if (ok) ok = issue_sdp(0);
            for (int g = 0; ok && g < ngroups; ++g) {
                if (g + 1 < ngroups && !(ok = issue_sdp(g + 1))) break;
                ok = issue_dq(g);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- elementwise warps
        const int q = warp % 4, c4 = warp / 4;  // TMEM lane quadrant; keys 32 c4 .. of each group
        const int r = q * 32 + lane;             // row of the tile
        const bool valid = r < gh * BLK;
        const int hh = valid ? r / BLK : 0, t = r % BLK;
        const int64_t grow = (static_cast<int64_t>(b) * p.Hq + head0 + hh) * p.N + static_cast<int64_t>(i) * BLK + t;
        const float lse2 = p.lse[grow] * 1.4426950408889634f;
        const float dlt = p.delta[grow];
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const float c2 = p.scale_log2;
        bool ok = true;
        for (int g = 0; g < ngroups; ++g) {
            const int ncols = min(GB, nsel - GB * g) * BLK;
            const bool mine = c4 * 32 < ncols;  // this quarter of the group holds keys
            // first column of the diagonal block in this group (128: not here)
            const int diag_lo = (diag_pos >= 0 && diag_pos / GB == g) ? (diag_pos % GB) * BLK : 128;
            if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(sdp_full, g & 1, p.status, detail_base | 0x20u));
            tc_fence_after();
            const uint32_t s_col = tm + lane_base + kRColS + 128 * (g % 2) + 32 * c4;
            if (mine) {
                uint32_t sv[32], dv[32], pk[16];
                tmem_ld32(s_col, sv);
                tmem_ld32(tm + lane_base + kRColDP + 32 * c4, dv);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(dp_read);  // the dP columns may be overwritten
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const int c0 = c4 * 32 + 2 * k;  // key column in the group
                    const bool m0 = !valid || (c0 >= diag_lo && c0 - diag_lo > t);
                    const bool m1 = !valid || (c0 + 1 >= diag_lo && c0 + 1 - diag_lo > t);
                    const float p0 = fast_exp2(__uint_as_float(sv[2 * k]) * c2 - lse2);
                    const float p1 = fast_exp2(__uint_as_float(sv[2 * k + 1]) * c2 - lse2);
                    const float d0 = m0 ? 0.f : p0 * (__uint_as_float(dv[2 * k]) - dlt);
                    const float d1 = m1 ? 0.f : p1 * (__uint_as_float(dv[2 * k + 1]) - dlt);
                    pk[k] = pack_bf16x2(d0, d1);
                }
                tmem_st16(s_col, pk);
                tmem_wait_st();
            } else {
                mbar_arrive(dp_read);
            }
            tc_fence_before();
            mbar_arrive(ds_ready + g % 2);
        }
        // ---------------------------------------------------------------- epilogue
        // dQ(ngroups - 1) done; phase by phase, since dq_done may still be one group behind
        for (int g = max(0, ngroups - 2); ok && g < ngroups; ++g)
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(dq_done, g & 1, p.status, detail_base | 0x22u));
        tc_fence_after();
        if (ok && valid && c4 * 32 < D) {
            const float sc = p.scale;
            uint4* dst = reinterpret_cast<uint4*>(p.dQ + grow * D + c4 * 32);
            uint32_t o[32];
            if (ngroups > 0) {
                tmem_ld32(tm + lane_base + kRColDQ + c4 * 32, o);
                tmem_wait_ld();
            } else {
#pragma unroll
                for (int x = 0; x < 32; ++x) o[x] = 0u;
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint32_t v[4];
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    v[e] = pack_bf16x2(__uint_as_float(o[8 * k + 2 * e]) * sc,
                                       __uint_as_float(o[8 * k + 2 * e + 1]) * sc);
                dst[k] = make_uint4(v[0], v[1], v[2], v[3]);
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncthreads();
    if (warp == kRProducerWarp && lane < 2) {
        uint64_t* full = lane == 0 ? k_full : v_full;
        const int nst = lane == 0 ? kRNstK : kRNstV;
        for (int g = max(0, issued_last - nst + 1); g <= issued_last; ++g)
            mbar_wait(full + g % nst, (g / nst) & 1, p.status, detail_base | 0x30u);
        if (lane == 0) mbar_wait(q_full, 0, p.status, detail_base | 0x31u);
    }
    if (warp == kRMmaWarp && lane == 0 && ngroups > 0) {
        // every MMA issued (all of them, or what an error left) completes before TMEM is freed
        mma_commit(mma_final);
        mbar_wait(mma_final, 0, p.status, detail_base | 0x32u);
    }
    __syncthreads();
    if (warp == kRMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tm, 512);
    }
}

bool bwd_dq_tc_supported(const BwdParams& p) {
    return (p.D == 64 || p.D == 128) && (p.blk == 64 || p.blk == 128) && p.topk <= kRMaxList;
}

template <int D, int BLK>
static bool launch_dq(const BwdParams& p, int32_t batch, cudaStream_t st) {
    CUtensorMap tq, tdo, tk, tv;
    const int64_t qrows = static_cast<int64_t>(batch) * p.Hq * p.N;
    const int64_t krows = static_cast<int64_t>(batch) * p.Hkv * p.N;
    if (!make_tmap_2d(&tq, p.Q, qrows, D, BLK) || !make_tmap_2d(&tdo, p.dO, qrows, D, BLK) ||
        !make_tmap_2d(&tk, p.K, krows, D, BLK) || !make_tmap_2d(&tv, p.V, krows, D, BLK))
        return false;
    static std::atomic<uint64_t> configured{0};
    if (!configure_smem_once(reinterpret_cast<const void*>(bwd_dq_tc_kernel<D, BLK>), static_cast<int>(kRSmem),
                             configured))
        return false;
    // 128 rows: two heads of 64-token blocks (one head, 64 rows, when the group is odd), or one head
    // of 128-token blocks
    const int gsel = p.per_qhead ? 1 : p.g;
    const int gh = BLK == 128 ? 1 : (gsel % 2 == 0 ? 2 : 1);
    const int chunks = gsel / gh;
    bwd_dq_tc_kernel<D, BLK><<<dim3(p.nqb, p.Hsel * chunks, batch), kRThreads, kRSmem, st>>>(tq, tdo, tk, tv, p,
                                                                                             gh, chunks);
    return cudaGetLastError() == cudaSuccess;
}

bool launch_bwd_dq_tc(const BwdParams& p, int32_t batch, cudaStream_t st) {
    if (!bwd_dq_tc_supported(p)) return false;
    if (p.D == 128) return p.blk == 128 ? launch_dq<128, 128>(p, batch, st) : launch_dq<128, 64>(p, batch, st);
    return p.blk == 128 ? launch_dq<64, 128>(p, batch, st) : launch_dq<64, 64>(p, batch, st);
}

bool bwd_dkdv_tc_supported(const BwdParams& p) { return (p.D == 64 || p.D == 128) && (p.blk == 64 || p.blk == 128); }

template <int D, int BLK>
static bool launch_dkdv(const BwdParams& p, int32_t batch, cudaStream_t st) {
    CUtensorMap tq, tdo, tk, tv;
    const int64_t qrows = static_cast<int64_t>(batch) * p.Hq * p.N;
    const int64_t krows = static_cast<int64_t>(batch) * p.Hkv * p.N;
    if (!make_tmap_2d(&tq, p.Q, qrows, D, kTB) || !make_tmap_2d(&tdo, p.dO, qrows, D, kTB) ||
        !make_tmap_2d(&tk, p.K, krows, D, kTB) || !make_tmap_2d(&tv, p.V, krows, D, kTB))
        return false;
    static std::atomic<uint64_t> configured{0};
    if (!configure_smem_once(reinterpret_cast<const void*>(bwd_dkdv_tc_kernel<D, BLK>), static_cast<int>(kSmem),
                             configured))
        return false;
    // one CTA per 64 keys: a 128-key block is taken as its two halves
    bwd_dkdv_tc_kernel<D, BLK><<<dim3(p.n0 * (BLK / kTB), p.Hkv, batch), kThreads, kSmem, st>>>(tq, tdo, tk, tv, p);
    return cudaGetLastError() == cudaSuccess;
}

bool launch_bwd_dkdv_tc(const BwdParams& p, int32_t batch, cudaStream_t st) {
    if (!bwd_dkdv_tc_supported(p)) return false;
    if (p.D == 128) return p.blk == 128 ? launch_dkdv<128, 128>(p, batch, st) : launch_dkdv<128, 64>(p, batch, st);
    return p.blk == 128 ? launch_dkdv<64, 128>(p, batch, st) : launch_dkdv<64, 64>(p, batch, st);
}

}  // namespace pisa
