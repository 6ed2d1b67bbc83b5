// Fused block-sparse attention for prefill on sm_100a, two units per CTA
// ("Des noyaux Triton qui ne materialisent rien", PISA page; online softmax as
// in the merge of the Pulsar Attention page, section "Phase 2").
//
// attn_prefill_kernel (attn_prefill.cu) gives a CTA one unit - the rows of one
// selection row's query block, gh heads x b tokens - and splits more than 128
// rows over two 128-row tensor-core tiles whose softmax and MMAs alternate. A
// unit of at most 128 rows (multi-head attention, 128-key blocks, per-query-head
// selection, small groups) fills one tile, and one tile per CTA leaves the
// tensor cores idle while the tile's softmax runs. This kernel gives such a CTA
// two units instead: two neighbouring query blocks of the same heads, one per
// tile, each with its own block list and its own K/V ring. The MMA lane runs the
// same alternation as the one-unit kernel, Q.K^T(0, g), P.V(1, g-1), Q.K^T(1, g),
// P.V(0, g), over the two units' group sequences, and every other step (128-key
// groups, P in TMEM over the S columns, two softmax warps per row, first pass
// against the first group's row max, exact second pass, bounded waits, teardown
// drains) is that kernel's.
#include <cuda.h>
#include <cuda_bf16.h>

#include <type_traits>

#include "pisa_device.cuh"

namespace pisa {

template <int D, int BLK>
struct DualCfg {
    static constexpr int NM = 2;                       // two tiles, one unit each
    static constexpr bool DU = true;
    static constexpr int DS = D / 64;                  // 128-byte column tiles along the head dim
    static constexpr int GB = 128 / BLK;               // selected blocks per 128-key group
    static constexpr int SUB = 128 * 128;              // one [128 rows x 128 B] operand tile
    static constexpr int Q_BYTES = NM * DS * SUB;
    static constexpr int KG_BYTES = DS * SUB;          // a 128-key K (or V) group
    static constexpr int NU = DU ? 2 : 1;              // units (block lists) per CTA: one per tile when DU
    static constexpr int MAX_LIST = kMaxPrefillTopk;   // selected blocks per query block
    static constexpr int AUX = 512 + NU * MAX_LIST * 4;    // barriers, TMEM slot, block lists
    static constexpr int SMEM_LIMIT = 232448;          // 227 KB opt-in maximum
    static constexpr int NST_FIT = (SMEM_LIMIT - 1024 - Q_BYTES - AUX) / (NU * 2 * KG_BYTES);
    static constexpr int NST = NST_FIT > 4 ? 4 : NST_FIT;   // K and V ring stages per unit
    static constexpr int SMEM = 1024 + Q_BYTES + NU * NST * 2 * KG_BYTES + AUX;
    static constexpr int O_COL = 0;
    static constexpr int S_COL = NM * D;               // S/P of tile h at S_COL + 128 h
    static constexpr int TMEM_NEED = NM * D + NM * 128;
    static constexpr int TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
    static constexpr int SOFTMAX_WARPS = 8 * NM;          // two warps per query row
    static constexpr int PRODUCER_WARP = SOFTMAX_WARPS;
    static constexpr int MMA_WARP = SOFTMAX_WARPS + 1;
    static constexpr int THREADS = 32 * (SOFTMAX_WARPS + 2);
    static_assert(NST >= (DU ? 1 : 2), "shared memory too small for the K/V rings");
    static_assert(!DU || NM == 2, "two units need two tiles");
    static_assert(TMEM_NEED <= 512, "TMEM budget exceeded");
    static_assert(BLK == 64 || BLK == 128, "key block of 64 or 128");
    static_assert(SMEM < (1 << 18), "descriptor offsets assume shared addresses below 2^18");
};

template <int D, int BLK>
__global__ void __launch_bounds__(DualCfg<D, BLK>::THREADS, 1)
    attn_prefill_dual_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using C = DualCfg<D, BLK>;
    constexpr int NM = C::NM;
    constexpr bool DU = C::DU;
    constexpr int NU = C::NU;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Qs = base;
    uint8_t* Ks = Qs + C::Q_BYTES;                     // unit u's K ring at Ks + u * NST * KG_BYTES
    uint8_t* Vs = Ks + NU * C::NST * C::KG_BYTES;      // unit u's V ring at Vs + u * NST * KG_BYTES
    uint8_t* aux = Vs + NU * C::NST * C::KG_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(aux);
    uint64_t* q_full = bars;                      // 1
    uint64_t* k_full = q_full + 1;                // NU * NST (unit u, stage s at u * NST + s)
    uint64_t* v_full = k_full + NU * C::NST;      // NU * NST
    uint64_t* k_empty = v_full + NU * C::NST;     // NU * NST  (Q.K^T of the group completed)
    uint64_t* v_empty = k_empty + NU * C::NST;    // NU * NST  (P.V of the group completed)
    uint64_t* s_full = v_empty + NU * C::NST;     // NM   (S of tile h in TMEM)
    uint64_t* p_full = s_full + NM;               // NM   (P of tile h in TMEM, O rescaled)
    uint64_t* pv_done = p_full + NM;              // NM   (P.V of tile h completed)
    uint64_t* mma_final = pv_done + NM;           // 1
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_final + 1);
    int32_t* s_nsel = reinterpret_cast<int32_t*>(tmem_slot + 1);  // NU
    int32_t* s_diag = s_nsel + NU;            // NU: list position of the diagonal block, -1 if absent
    int32_t* s_retry = s_diag + NU;           // set when a row outgrew the first pass's reference
    int32_t* lists = reinterpret_cast<int32_t*>(aux + 512);  // unit u's list at lists + u * MAX_LIST

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    // query block of unit u, longest rows first; with two units a CTA takes two neighbouring query
    // blocks (one per tile), the second absent (-1) when the count is odd
    auto unit_block = [&](int u) -> int {
        return DU ? p.nqb - 1 - 2 * static_cast<int>(blockIdx.x) - u : p.nqb - 1 - static_cast<int>(blockIdx.x);
    };
    const int hs = static_cast<int>(blockIdx.y) / p.chunks;
    const int chunk = static_cast<int>(blockIdx.y) % p.chunks;
    const int b = static_cast<int>(blockIdx.z);
    const int kvh = p.per_qhead ? hs / p.g : hs;
    const int head0 = p.per_qhead ? hs : kvh * p.g + chunk * p.gh;
    const uint32_t detail_base = kKernAttnPrefill << 8;

    if (warp == C::PRODUCER_WARP && lane == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < NU * C::NST; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(v_full + s, 1);
            mbar_init(k_empty + s, 1);
            mbar_init(v_empty + s, 1);
        }
        for (int h = 0; h < NM; ++h) {
            mbar_init(s_full + h, 1);
            mbar_init(p_full + h, 256);
            mbar_init(pv_done + h, 1);
        }
        mbar_init(mma_final, 1);
        fence_barrier_init();
        // Q does not depend on the selection: its copy starts before the block rows are read
        prefetch_tmap(&tmQ);
        int units = 0;
        for (int u = 0; u < NU; ++u) units += unit_block(u) >= 0;
        mbar_arrive_expect_tx(q_full, static_cast<uint32_t>(units * p.gh * BLK * D * 2));
        for (int u = 0; u < NU; ++u) {
            const int iu = unit_block(u);
            if (iu < 0) continue;
            for (int hh = 0; hh < p.gh; ++hh) {
                const int r0 = u * 128 + hh * BLK;  // DU: tile u holds unit u's rows
                const int qrow = static_cast<int>((static_cast<int64_t>(b) * p.Hq + head0 + hh) * p.N +
                                                  static_cast<int64_t>(iu) * BLK);
#pragma unroll
                for (int s = 0; s < C::DS; ++s)
                    tma_load_2d(Qs + ((r0 / 128) * C::DS + s) * C::SUB + (r0 % 128) * 128, &tmQ, s * 64, qrow,
                                q_full);
            }
        }
    }
    if (warp == C::MMA_WARP) tmem_alloc(tmem_slot, C::TMEM_COLS);
    if (warp == C::PRODUCER_WARP) {
        // compact each unit's selected-block row: valid entries in order, bad ones recorded
        for (int u = 0; u < NU; ++u) {
            const int iu = unit_block(u);
            int32_t* list = lists + u * C::MAX_LIST;
            int cnt = 0, diag = -1;
            if (iu >= 0) {
                const int32_t* row = p.idx + ((static_cast<int64_t>(b) * p.Hsel + hs) * p.nqb + iu) * p.topk;
                for (int t0 = 0; t0 < p.topk; t0 += 32) {
                    const int t = t0 + lane;
                    const int32_t j = t < p.topk ? row[t] : -1;
                    const bool ok = j >= 0 && j < p.n0 && (!p.causal || j <= iu);
                    if (t < p.topk && j >= 0 && !ok) record_error(p.status, PISA_ERR_BAD_INDEX, detail_base | 0xB0u);
                    const uint32_t m = __ballot_sync(0xFFFFFFFFu, ok);
                    const int pos = cnt + __popc(m & ((1u << lane) - 1u));
                    if (ok && pos < C::MAX_LIST) list[pos] = j;
                    // the diagonal block needs the per-token causal mask; its list position is found
                    // here once, so the softmax warps need no shared-memory read per key group
                    const uint32_t md = __ballot_sync(0xFFFFFFFFu, p.causal && ok && j == iu && pos < C::MAX_LIST);
                    if (diag < 0 && md != 0u) diag = __shfl_sync(0xFFFFFFFFu, pos, __ffs(md) - 1);
                    cnt += __popc(m);
                }
            }
            if (lane == 0) {
                s_nsel[u] = cnt < C::MAX_LIST ? cnt : C::MAX_LIST;
                s_diag[u] = diag;
            }
        }
        if (lane == 0) *s_retry = 0;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    // per unit: selected blocks, key groups, list position of the diagonal block
    int nsel_u[NU], ngroups_u[NU], diag_u[NU];
#pragma unroll
    for (int u = 0; u < NU; ++u) {
        nsel_u[u] = s_nsel[u];
        ngroups_u[u] = (nsel_u[u] + C::GB - 1) / C::GB;
        diag_u[u] = s_diag[u];
    }

    int issued_last = -1;  // producer lanes: last group whose copies they started
    bool issued_any_mma = false;
    // Every role runs its loop over the key groups once, then all meet at kPassBarrier; if a
    // softmax row marked the CTA, every role runs it once more (second pass, exact rescale).
    // Ring slots and barrier phases follow the running group count gg = pass * ngroups + g of the
    // unit (ring) or tile (S, P, O barriers) they belong to.
    auto second_pass = [&]() -> bool {
        named_bar_sync(kPassBarrier, C::THREADS);
        return *reinterpret_cast<volatile int32_t*>(s_retry) != 0;
    };

    if (warp == C::PRODUCER_WARP) {
        // lane 2u streams unit u's K groups, lane 2u + 1 its V groups
        const int u = min(lane >> 1, NU - 1);
        const bool active = lane < 2 * NU;
        const bool is_k = (lane & 1) == 0;
        const void* tmap = is_k ? static_cast<const void*>(&tmK) : static_cast<const void*>(&tmV);
        uint8_t* ring = (is_k ? Ks : Vs) + u * C::NST * C::KG_BYTES;
        uint64_t* full = (is_k ? k_full : v_full) + u * C::NST;
        uint64_t* empty = (is_k ? k_empty : v_empty) + u * C::NST;
        const int32_t* list = lists + u * C::MAX_LIST;
        const int ng = ngroups_u[u], ns = nsel_u[u];
        bool ok = true;
        if (active && ng > 0) prefetch_tmap(tmap);
        for (int pass = 0; pass < 2; ++pass) {
            for (int g = 0; ok && active && g < ng; ++g) {
                const int gg = pass * ng + g;
                const int st = gg % C::NST, use = gg / C::NST;
                if (!(ok = mbar_wait(empty + st, (use & 1) ^ 1, p.status, detail_base | (is_k ? 0x01u : 0x02u))))
                    break;
                const int nb = min(C::GB, ns - g * C::GB);
                mbar_arrive_expect_tx(full + st, static_cast<uint32_t>(nb * BLK * D * 2));
                for (int v = 0; v < nb; ++v) {
                    const int krow = static_cast<int>((static_cast<int64_t>(b) * p.Hkv + kvh) * p.N +
                                                      static_cast<int64_t>(list[g * C::GB + v]) * BLK);
#pragma unroll
                    for (int s = 0; s < C::DS; ++s)
                        tma_load_2d(ring + st * C::KG_BYTES + s * C::SUB + v * BLK * 128, tmap, s * 64, krow,
                                    full + st);
                }
                issued_last = gg;
            }
            __syncwarp();
            if (pass == 0 && !second_pass()) break;
        }
    } else if (warp == C::MMA_WARP) {
        bool ok = true;
        for (int pass = 0; pass < 2; ++pass) {
            const int ng_max = DU ? max(ngroups_u[0], ngroups_u[NU - 1]) : ngroups_u[0];
            if (lane == 0 && ng_max > 0 && ok) {
                // Operand descriptors are formed once; every tile the MMAs read lies at a fixed offset
                // from these bases. The start-address field holds address / 16 in 14 bits, and shared
                // memory ends below 2^18 bytes, so adding offset / 16 never carries out of the field.
                const uint64_t dq0 = smem_desc_sw128(smem_u32(Qs), 16, 1024);
                const uint64_t dk0 = smem_desc_sw128(smem_u32(Ks), 16, 1024);
                const uint64_t dv0 = smem_desc_sw128(smem_u32(Vs), C::SUB, 1024);
                constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
                if (pass == 0) ok = mbar_wait(q_full, 0, p.status, detail_base | 0x10u);
                tc_fence_after();
                // unit (ring) of tile h, its group count and the running count of group g
                auto unit_of = [&](int h) { return DU ? h : 0; };
                auto ring_slot = [&](int h, int g) {
                    const int u = unit_of(h);
                    return u * C::NST + (pass * ngroups_u[u] + g) % C::NST;
                };
                // S[h] = Q_h K_g^T (after P.V of group g-1 on tile h has released the TMEM columns)
                auto qk = [&](int g, int h) -> bool {
                    const int u = unit_of(h);
                    const int gg = pass * ngroups_u[u] + g;
                    const int rs = ring_slot(h, g);
                    if (!mbar_wait(k_full + rs, (gg / C::NST) & 1, p.status, detail_base | 0x11u)) return false;
                    if (gg > 0 && !mbar_wait(pv_done + h, (gg - 1) & 1, p.status, detail_base | 0x12u)) return false;
                    tc_fence_after();
                    const int ncols = min(C::GB, nsel_u[u] - g * C::GB) * BLK;
                    const uint32_t idesc_qk = idesc_bf16_f32(128, ncols, 0, 0);
                    const uint32_t d_tmem = tm + C::S_COL + h * 128;
                    const uint64_t a0 = dq0 + static_cast<uint32_t>((h * C::DS * C::SUB) >> 4);
                    const uint64_t b0 = dk0 + static_cast<uint32_t>((rs * C::KG_BYTES) >> 4);
#pragma unroll
                    for (int ks = 0; ks < D / 16; ++ks) {
                        const uint32_t off = static_cast<uint32_t>(((ks / 4) * C::SUB + (ks % 4) * 32) >> 4);
                        mma_bf16_ss(d_tmem, a0 + off, b0 + off, idesc_qk, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(s_full + h);
                    issued_any_mma = true;
                    return true;
                };
                // O[h] += P_h V_g (P in TMEM: keys 0-63 in columns 0-31, keys 64-127 in columns 64-95)
                auto pv = [&](int g, int h) -> bool {
                    const int u = unit_of(h);
                    const int gg = pass * ngroups_u[u] + g;
                    const int rs = ring_slot(h, g);
                    if (!mbar_wait(v_full + rs, (gg / C::NST) & 1, p.status, detail_base | 0x13u)) return false;
                    if (!mbar_wait(p_full + h, gg & 1, p.status, detail_base | 0x14u)) return false;
                    tc_fence_after();
                    const int nks = min(C::GB, nsel_u[u] - g * C::GB) * BLK / 16;
                    const uint32_t d_tmem = tm + C::O_COL + h * D;
                    const uint32_t a_tmem = tm + C::S_COL + h * 128;
                    const uint64_t b0 = dv0 + static_cast<uint32_t>((rs * C::KG_BYTES) >> 4);
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        if (ks < nks) {
                            const uint32_t acol = ks < 4 ? ks * 8 : 64 + (ks - 4) * 8;
                            const uint32_t boff = static_cast<uint32_t>((ks * 16 * 128) >> 4);
                            mma_bf16_ts(d_tmem, a_tmem + acol, b0 + boff, idesc_pv, (g > 0 || ks > 0) ? 1u : 0u);
                        }
                    }
                    mma_commit(pv_done + h);
                    return true;
                };
                // Order per group g: Q.K^T(0, g), P.V(1, g-1), Q.K^T(1, g), P.V(0, g): each tile's
                // softmax overlaps two MMAs of the other tile. A ring slot is released after the last
                // MMA that reads it: K after Q.K^T of the unit's last tile, V after its P.V.
                const int ng0 = ngroups_u[0], ng1 = ngroups_u[NU - 1];
                for (int g = 0; ok && g < ng_max; ++g) {
                    if (g < ng0) {
                        if (!(ok = qk(g, 0))) break;
                        if (DU || NM == 1) mma_commit(k_empty + ring_slot(0, g));
                    }
                    if (NM == 2) {
                        if (g > 0 && g - 1 < ng1) {
                            if (!(ok = pv(g - 1, 1))) break;
                            mma_commit(v_empty + ring_slot(1, g - 1));
                        }
                        if (g < ng1) {
                            if (!(ok = qk(g, 1))) break;
                            mma_commit(k_empty + ring_slot(1, g));
                        }
                    }
                    if (g < ng0) {
                        if (!(ok = pv(g, 0))) break;
                        if (DU || NM == 1) mma_commit(v_empty + ring_slot(0, g));
                    }
                }
                // the last P.V of tile 1 (issued in the loop already when tile 1 has fewer groups)
                if (ok && NM == 2 && ng1 > 0 && ng1 == ng_max) {
                    if ((ok = pv(ng1 - 1, 1))) mma_commit(v_empty + ring_slot(1, ng1 - 1));
                }
            }
            __syncwarp();
            if (pass == 0 && !second_pass()) break;
        }
    } else {
        // ---------------------------------------------------------------- softmax warps
        const int h = (warp / 4) % NM;
        const int qd = warp % 4;
        const int ch = warp / (4 * NM);   // column half: keys [64 ch, 64 ch + 64) of every group
        const int r = qd * 32 + lane;     // row inside tile h
        // tile h's unit: its own query block with two units, else the CTA's one unit over both tiles
        const int u = DU ? h : 0;
        const int R = DU ? r : h * 128 + r;  // row inside the unit
        const int iu = unit_block(u);
        const bool valid = R < p.gh * BLK && iu >= 0;
        const int hh = R / BLK, t = R % BLK;
        const int nsel = nsel_u[u], ngroups = ngroups_u[u], diag_pos = diag_u[u];
        const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
        const uint32_t s_tmem = tm + lane_base + C::S_COL + h * 128 + ch * 64;
        // Row statistics of the two warps of a row quadrant meet in TMEM: each warp writes its
        // value into the last column of its own half of S (already read into registers), the
        // pair meets at a named barrier, and each reads the partner's column. Shared memory is
        // kept off this path: the tensor cores' operand reads keep it busy, and a shared access
        // there waits hundreds of cycles. The barrier has no time limit, so the loop below never
        // leaves early: after a failed wait a warp records the error, skips the remaining waits
        // and keeps meeting its partner, once per key group and once in the epilogue.
        const uint32_t xbar_id = 1u + static_cast<uint32_t>(h * 4 + qd);
        const uint32_t slot_mine = s_tmem + 63;
        const uint32_t slot_other = tm + lane_base + C::S_COL + h * 128 + (ch ^ 1) * 64 + 63;
        auto exchange = [&](float mine_v) -> float {
            tmem_st1(slot_mine, __float_as_uint(mine_v));
            tmem_wait_st();
            tc_fence_before();
            named_bar_sync(xbar_id, 64);
            tc_fence_after();
            const uint32_t o = tmem_ld1(slot_other);
            tmem_wait_ld();
            return __uint_as_float(o);
        };
        const float cs = p.scale_log2;
        const uint64_t cs2 = f2_pack(cs, cs);
        float m_used = -INFINITY, l_part = 0.f;
        bool ok = true;
        int g_last = ngroups - 1;  // running index of the last group of the final pass
        for (int pass = 0; pass < 2; ++pass) {
            const bool exact = pass > 0;
            const int g0 = pass * ngroups;
            m_used = -INFINITY;
            l_part = 0.f;
            for (int g = 0; g < ngroups; ++g) {
                const int gg = g0 + g;
                const int nb = min(C::GB, nsel - g * C::GB);
                const int ncols = nb * BLK;
                const int mine = max(0, min(64, ncols - ch * 64));  // columns of this half that hold keys
                if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(s_full + h, gg & 1, p.status, detail_base | 0x20u));
                tc_fence_after();
                // first column of the diagonal block, 128 if this group does not hold it
                const int diag_lo = (diag_pos >= 0 && diag_pos / C::GB == g) ? (diag_pos % C::GB) * BLK : 128;
                const bool any_mask = ncols < 128 || diag_lo < 128;  // uniform across the CTA
                uint32_t pk[32];                                     // this half's P, bf16 pairs
                uint64_t sum2[2] = {0ull, 0ull};
                float s_last = 0.f;  // raw score of this half's last column, whose TMEM cell the exchange reuses
                // exp2 of one 32-column chunk against the reference max; returns the chunk's max x.
                // TRACK, MASKED and PATCH are compile-time, so the unrolled pair loop has no branches
                // and the compiler can interleave the sixteen independent pair chains. PATCH puts the
                // saved last score back after an exchange has overwritten its cell.
                auto chunk_exp = [&](int c, float m_ref, auto track_c, auto masked_c, auto patch_c) -> float {
                    constexpr bool TRACK = decltype(track_c)::value;
                    constexpr bool MASKED = decltype(masked_c)::value;
                    constexpr bool PATCH = decltype(patch_c)::value;
                    float sv[32];
                    tmem_ld32(s_tmem + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sv));
                    tmem_wait_ld();
                    if (c == 1) {
                        if (PATCH)
                            sv[31] = s_last;
                        else
                            s_last = sv[31];
                    }
                    if (MASKED) {
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            const int col = ch * 64 + c * 32 + k;
                            if (col >= ncols || (col >= diag_lo && col - diag_lo > t)) sv[k] = -INFINITY;
                        }
                    }
                    const uint64_t negm2 = f2_pack(-m_ref, -m_ref);
                    float xm = -INFINITY;
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const int kk = c * 16 + k;
                        float x0, x1;
                        f2_unpack(f2_fma(f2_pack(sv[2 * k], sv[2 * k + 1]), cs2, negm2), x0, x1);
                        if (TRACK) xm = fmax3(xm, x0, x1);
                        const uint64_t e2 = f2_pack(fast_exp2(x0), fast_exp2(x1));
                        sum2[k & 1] = f2_add(sum2[k & 1], e2);
                        float e0, e1;
                        f2_unpack(e2, e0, e1);
                        pk[kk] = pack_bf16x2(e0, e1);
                    }
                    return xm;
                };
                // exponentials of this half against m_ref, after the exchange (saved last score restored)
                auto exps_patched = [&](float m_ref) {
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        if (c * 32 < mine) {
                            if (any_mask)
                                chunk_exp(c, m_ref, std::false_type{}, std::true_type{}, std::true_type{});
                            else
                                chunk_exp(c, m_ref, std::false_type{}, std::false_type{}, std::true_type{});
                        }
                };
                float alpha = 1.0f, m_new = m_used;
                if (g > 0) {
                    // fast path: probabilities against the running max m, kept while no score of the
                    // row (in either half) exceeds m by more than the rescale threshold
                    float xmax = -INFINITY;
#pragma unroll
                    for (int c = 0; c < 2; ++c)
                        if (c * 32 < mine)
                            xmax = fmaxf(xmax, any_mask ? chunk_exp(c, m_used, std::true_type{}, std::true_type{},
                                                                    std::false_type{})
                                                        : chunk_exp(c, m_used, std::true_type{}, std::false_type{},
                                                                    std::false_type{}));
                    if (!exact) {
                        // first pass: m stays the first group's row max; a row that outgrew it by more
                        // than the limit sends the CTA to the second pass (this pass's P is discarded)
                        if (valid && xmax > kFirstPassLimit) *reinterpret_cast<volatile int32_t*>(s_retry) = 1;
                    } else {
                        const float xall = fmaxf(xmax, exchange(xmax));  // row max of s*c - m over both halves
                        if (__any_sync(0xFFFFFFFFu, xall > kRescaleThreshold)) {
                            // the row max grew past the threshold: m moves up to it, O is rescaled, and the
                            // exponentials are redone from S
                            const bool resc = xall > kRescaleThreshold;
                            m_new = resc ? m_used + xall : m_used;
                            alpha = resc ? fast_exp2(-xall) : 1.0f;
                            if (ok && __any_sync(0xFFFFFFFFu, resc)) {
                                // O holds P.V of every earlier group (its completion preceded this S); this
                                // warp rescales its half of the columns
                                ok = __all_sync(0xFFFFFFFFu,
                                                mbar_wait(pv_done + h, (gg - 1) & 1, p.status, detail_base | 0x21u));
                                if (ok) {
                                    tc_fence_after();
#pragma unroll
                                    for (int c = 0; c < D / 32; ++c) {
                                        uint32_t o[16];
                                        const uint32_t addr =
                                            tm + lane_base + C::O_COL + h * D + ch * (D / 2) + c * 16;
                                        tmem_ld16(addr, o);
                                        tmem_wait_ld();
#pragma unroll
                                        for (int k = 0; k < 16; ++k)
                                            o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                                        tmem_st16(addr, o);
                                    }
                                }
                            }
#pragma unroll
                            for (int k = 0; k < 2; ++k) sum2[k] = 0ull;
                            exps_patched(m_new);
                        }
                    }
                } else {
                    // first group: the true row max, then the exponentials
                    float mq[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) mq[q] = -INFINITY;
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        if (c * 32 < mine) {
                            float sv[32];
                            tmem_ld32(s_tmem + c * 32, *reinterpret_cast<uint32_t(*)[32]>(sv));
                            tmem_wait_ld();
                            if (c == 1) s_last = sv[31];
                            if (any_mask) {
#pragma unroll
                                for (int k = 0; k < 32; ++k) {
                                    const int col = ch * 64 + c * 32 + k;
                                    if (col >= ncols || (col >= diag_lo && col - diag_lo > t)) sv[k] = -INFINITY;
                                }
                            }
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                mq[q] = fmax3(mq[q], sv[q], fmaxf(sv[8 + q], fmaxf(sv[16 + q], sv[24 + q])));
                        }
                    }
                    const float mxs =
                        fmaxf(fmax3(mq[0], mq[1], mq[2]), fmax3(mq[3], mq[4], fmax3(mq[5], mq[6], mq[7]))) * cs;
                    m_new = fmaxf(mxs, exchange(mxs));
                    exps_patched(m_new);
                }
                // P overwrites this half's S columns, already read: 64 scores -> 32 columns
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    if (c * 32 < mine) tmem_st16(s_tmem + c * 16, *reinterpret_cast<uint32_t(*)[16]>(pk + c * 16));
                float r0, r1;
                f2_unpack(f2_add(sum2[0], sum2[1]), r0, r1);
                l_part = l_part * alpha + (r0 + r1);
                m_used = m_new;
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(p_full + h);
            }
            g_last = g0 + ngroups - 1;
            if (pass == 0 && !second_pass()) break;
        }
        // ---------------------------------------------------------------- epilogue
        if (ok && ngroups > 0)
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(pv_done + h, g_last & 1, p.status, detail_base | 0x22u));
        const float l_sum = l_part + exchange(l_part);
        if (ok) {
            const int head = head0 + hh;
            const int64_t orow = (static_cast<int64_t>(b) * p.Hq + head) * p.N + static_cast<int64_t>(iu) * BLK + t;
            tc_fence_after();
            const float inv = ngroups > 0 ? 1.0f / l_sum : 0.f;
            uint4* dst = reinterpret_cast<uint4*>(p.O + orow * D + ch * (D / 2));
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                uint32_t o[32];
                if (ngroups > 0) {
                    tmem_ld32(tm + lane_base + C::O_COL + h * D + ch * (D / 2) + c * 32, o);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int k = 0; k < 32; ++k) o[k] = 0u;
                }
                if (valid) {
                    // whole 32-byte sectors: each thread writes its row's columns 16 at a time
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        uint32_t v[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            v[e] = pack_bf16x2(__uint_as_float(o[16 * k + 2 * e]) * inv,
                                               __uint_as_float(o[16 * k + 2 * e + 1]) * inv);
                        st_global_v8(dst + c * 4 + 2 * k, v);
                    }
                }
            }
            if (valid && ch == 0 && p.lse != nullptr)
                p.lse[orow] = ngroups > 0 ? (m_used + __log2f(l_sum)) * 0.69314718055994531f : -INFINITY;
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncthreads();
    if (warp == C::PRODUCER_WARP && lane < 2 * NU) {
        // every TMA load this CTA issued has landed before shared memory is released
        uint64_t* full = ((lane & 1) == 0 ? k_full : v_full) + (lane >> 1) * C::NST;
        for (int g = max(0, issued_last - C::NST + 1); g <= issued_last; ++g)
            mbar_wait(full + g % C::NST, (g / C::NST) & 1, p.status, detail_base | 0x30u);
        if (lane == 0) mbar_wait(q_full, 0, p.status, detail_base | 0x32u);
    }
    if (warp == C::MMA_WARP && lane == 0 && issued_any_mma) {
        mma_commit(mma_final);
        mbar_wait(mma_final, 0, p.status, detail_base | 0x33u);
    }
    __syncthreads();
    if (warp == C::MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tm, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side

template <int D, int BLK>
static bool launch_dual(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const AttnParams& p,
                        dim3 grid, cudaStream_t st) {
    using C = DualCfg<D, BLK>;
    static std::atomic<uint64_t> configured{0};
    if (!configure_smem_once(reinterpret_cast<const void*>(attn_prefill_dual_kernel<D, BLK>), C::SMEM, configured))
        return false;
    grid.x = (grid.x + 1) / 2;  // two query blocks per CTA
    attn_prefill_dual_kernel<D, BLK><<<grid, C::THREADS, C::SMEM, st>>>(q, k, v, p);
    return cudaGetLastError() == cudaSuccess;
}

bool launch_attn_prefill_dual(int D, int blk, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                              const AttnParams& p, dim3 grid, cudaStream_t st) {
    if (D == 128 && blk == 64) return launch_dual<128, 64>(q, k, v, p, grid, st);
    if (D == 128 && blk == 128) return launch_dual<128, 128>(q, k, v, p, grid, st);
    if (D == 64 && blk == 64) return launch_dual<64, 64>(q, k, v, p, grid, st);
    if (D == 64 && blk == 128) return launch_dual<64, 128>(q, k, v, p, grid, st);
    return false;
}

}  // namespace pisa
