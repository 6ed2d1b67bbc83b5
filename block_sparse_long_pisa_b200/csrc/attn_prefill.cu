// Fused block-sparse attention for prefill on sm_100a ("Des noyaux Triton qui
// ne materialisent rien", PISA page; online softmax as in the merge of the
// Pulsar Attention page, section "Phase 2").
//
// One CTA per (batch, query-head group, query block). The CTA's query rows are
// gh heads x b tokens that share one list of selected key blocks (gh*b <= 256
// rows = NM tensor-core tiles of 128 rows). Every selected K/V block is loaded
// once by TMA and used by all rows, so GQA groups reuse each gathered byte gh
// times.
//
// The selected blocks are taken in key groups of 128 keys (two 64-key blocks,
// or one 128-key block). A tcgen05 MMA with M = 128 costs the same for N = 64
// as for N = 128, so grouping doubles the useful work of every Q.K^T
// instruction; P.V gets K = 128 per group.
//
// Warp roles (warp-specialised pipeline, all hand-off through mbarriers):
//   warps 0 .. 8*NM-1  softmax: two warps per query row. Warp w reads TMEM
//                      lanes 32*(w%4).. of tile (w/4)%NM and owns the 64
//                      score columns of its half (w/(4*NM)); the partner warp
//                      of the other half shares the rows. They exchange row
//                      maxima and sums through a TMEM column and a 64-thread
//                      named barrier, and each writes half of O at the end.
//   warp 8*NM          producer: lane 0 streams K groups, lane 1 V groups, by
//                      2-D TMA into NST-deep rings (each with its own empty
//                      barrier, so K can run ahead of V)
//   warp 8*NM+1        MMA: allocates TMEM and one lane issues tcgen05.mma
//
// Per key group g and tile h:
//   S[h] = Q_h K_g^T     tcgen05 (A = Q and B = K from shared memory), fp32 in TMEM
//   softmax: P = exp2(S*c - m) against a reference row max m, written as bf16
//            back into the TMEM columns of S already read (keys 0-63 into
//            columns 0-31, keys 64-127 into columns 64-95). m is the row max of
//            the first group; it does not move, so the two warps of a row meet
//            only in the first group and the epilogue. A row whose later
//            scores exceed m by more than 2^16 marks the CTA, and the whole
//            unit runs again in a second pass where m moves whenever a score
//            exceeds it by more than 2^8 (that group is redone from the intact
//            S with the new max, O and the row sums are rescaled)
//   O[h] += P_h V_g      tcgen05 with A = P read from TMEM, B = V (MN-major)
// Because P overwrites S, a tile's next Q.K^T waits for its P.V. With two
// tiles the MMA lane issues Q.K^T(0, g), P.V(1, g-1), Q.K^T(1, g), P.V(0, g):
// each tile's softmax overlaps two MMAs of the other tile. No score ever
// leaves TMEM.
//
// Softmax arithmetic: packed fp32 pair instructions (f32x2) for the
// scale-and-subtract and the row sum, exponentials on the MUFU unit. (Moving a
// share of them to a polynomial on the FMA pipes measured slower here: the
// softmax is bound by instruction issue and latency, not by MUFU throughput.)
#include <cuda.h>
#include <cuda_bf16.h>

#include <type_traits>

#include "pisa_device.cuh"

namespace pisa {

template <int D, int BLK, int NM>
struct PrefillCfg {
    static constexpr int DS = D / 64;                  // 128-byte column tiles along the head dim
    static constexpr int GB = 128 / BLK;               // selected blocks per 128-key group
    static constexpr int SUB = 128 * 128;              // one [128 rows x 128 B] operand tile
    static constexpr int Q_BYTES = NM * DS * SUB;
    static constexpr int KG_BYTES = DS * SUB;          // a 128-key K (or V) group
    static constexpr int MAX_LIST = kMaxPrefillTopk;   // selected blocks per query block
    static constexpr int AUX = 512 + MAX_LIST * 4;         // barriers, TMEM slot, block list
    static constexpr int SMEM_LIMIT = 232448;          // 227 KB opt-in maximum
    static constexpr int NST_FIT = (SMEM_LIMIT - 1024 - Q_BYTES - AUX) / (2 * KG_BYTES);
    static constexpr int NST = NST_FIT > 4 ? 4 : NST_FIT;
    static constexpr int SMEM = 1024 + Q_BYTES + NST * 2 * KG_BYTES + AUX;
    static constexpr int O_COL = 0;
    static constexpr int S_COL = NM * D;               // S/P of tile h at S_COL + 128 h
    static constexpr int TMEM_NEED = NM * D + NM * 128;
    static constexpr int TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
    static constexpr int SOFTMAX_WARPS = 8 * NM;          // two warps per query row
    static constexpr int PRODUCER_WARP = SOFTMAX_WARPS;
    static constexpr int MMA_WARP = SOFTMAX_WARPS + 1;
    static constexpr int THREADS = 32 * (SOFTMAX_WARPS + 2);
    static_assert(NST >= 2, "shared memory too small for double-buffered K/V rings");
    static_assert(TMEM_NEED <= 512, "TMEM budget exceeded");
    static_assert(BLK == 64 || BLK == 128, "key block of 64 or 128");
    static_assert(SMEM < (1 << 18), "descriptor offsets assume shared addresses below 2^18");
};

template <int D, int BLK, int NM>
__global__ void __launch_bounds__(PrefillCfg<D, BLK, NM>::THREADS, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using C = PrefillCfg<D, BLK, NM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Qs = base;
    uint8_t* Ks = Qs + C::Q_BYTES;
    uint8_t* Vs = Ks + C::NST * C::KG_BYTES;
    uint8_t* aux = Vs + C::NST * C::KG_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(aux);
    uint64_t* q_full = bars;                  // 1
    uint64_t* k_full = q_full + 1;            // NST
    uint64_t* v_full = k_full + C::NST;       // NST
    uint64_t* k_empty = v_full + C::NST;      // NST  (Q.K^T of the group completed)
    uint64_t* v_empty = k_empty + C::NST;     // NST  (P.V of the group completed)
    uint64_t* s_full = v_empty + C::NST;      // NM   (S of tile h in TMEM)
    uint64_t* p_full = s_full + NM;           // NM   (P of tile h in TMEM, O rescaled)
    uint64_t* pv_done = p_full + NM;          // NM   (P.V of tile h completed)
    uint64_t* mma_final = pv_done + NM;       // 1
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_final + 1);
    int32_t* s_nsel = reinterpret_cast<int32_t*>(tmem_slot + 1);
    int32_t* s_diag = s_nsel + 1;             // list position of the diagonal block i, -1 if absent
    int32_t* s_retry = s_diag + 1;            // set when a row outgrew the first pass's reference
    int32_t* list = reinterpret_cast<int32_t*>(aux + 512);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int i = p.nqb - 1 - static_cast<int>(blockIdx.x);  // longest rows first
    const int hs = static_cast<int>(blockIdx.y) / p.chunks;
    const int chunk = static_cast<int>(blockIdx.y) % p.chunks;
    const int b = static_cast<int>(blockIdx.z);
    const int kvh = p.per_qhead ? hs / p.g : hs;
    const int head0 = p.per_qhead ? hs : kvh * p.g + chunk * p.gh;
    const uint32_t detail_base = kKernAttnPrefill << 8;

    if (warp == C::PRODUCER_WARP && lane == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::NST; ++s) {
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
        // Q does not depend on the selection: its copy starts before the block row is read
        prefetch_tmap(&tmQ);
        mbar_arrive_expect_tx(q_full, static_cast<uint32_t>(p.gh * BLK * D * 2));
        for (int hh = 0; hh < p.gh; ++hh) {
            const int r0 = hh * BLK;
            const int qrow = static_cast<int>((static_cast<int64_t>(b) * p.Hq + head0 + hh) * p.N +
                                              static_cast<int64_t>(i) * BLK);
#pragma unroll
            for (int s = 0; s < C::DS; ++s)
                tma_load_2d(Qs + ((r0 / 128) * C::DS + s) * C::SUB + (r0 % 128) * 128, &tmQ, s * 64, qrow, q_full);
        }
    }
    if (warp == C::MMA_WARP) tmem_alloc(tmem_slot, C::TMEM_COLS);
    if (warp == C::PRODUCER_WARP) {
        // compact the selected-block row: valid entries in order, bad ones recorded
        const int32_t* row = p.idx + ((static_cast<int64_t>(b) * p.Hsel + hs) * p.nqb + i) * p.topk;
        int cnt = 0, diag = -1;
        for (int t0 = 0; t0 < p.topk; t0 += 32) {
            const int t = t0 + lane;
            const int32_t j = t < p.topk ? row[t] : -1;
            const bool ok = j >= 0 && j < p.n0 && (!p.causal || j <= i);
            if (t < p.topk && j >= 0 && !ok) record_error(p.status, PISA_ERR_BAD_INDEX, detail_base | 0xB0u);
            const uint32_t m = __ballot_sync(0xFFFFFFFFu, ok);
            const int pos = cnt + __popc(m & ((1u << lane) - 1u));
            if (ok && pos < C::MAX_LIST) list[pos] = j;
            // the diagonal block needs the per-token causal mask; its list position is found here
            // once, so the softmax warps need no shared-memory read per key group
            const uint32_t md = __ballot_sync(0xFFFFFFFFu, p.causal && ok && j == i && pos < C::MAX_LIST);
            if (diag < 0 && md != 0u) diag = __shfl_sync(0xFFFFFFFFu, pos, __ffs(md) - 1);
            cnt += __popc(m);
        }
        if (lane == 0) {
            *s_nsel = cnt < C::MAX_LIST ? cnt : C::MAX_LIST;
            *s_diag = diag;
            *s_retry = 0;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    const int nsel = *s_nsel;
    const int ngroups = (nsel + C::GB - 1) / C::GB;
    const int diag_pos = *s_diag;

    int issued_last = -1;  // producer lanes: last group whose copies they started
    bool issued_any_mma = false;
    // Every role runs its loop over the key groups once, then all meet at kPassBarrier; if a
    // softmax row marked the CTA, every role runs it once more (second pass, exact rescale).
    // Ring slots and barrier phases follow the running group count gg = pass * ngroups + g.
    auto second_pass = [&]() -> bool {
        named_bar_sync(kPassBarrier, C::THREADS);
        return *reinterpret_cast<volatile int32_t*>(s_retry) != 0;
    };

    if (warp == C::PRODUCER_WARP) {
        const bool is_k = lane == 0;
        const void* tmap = is_k ? static_cast<const void*>(&tmK) : static_cast<const void*>(&tmV);
        uint8_t* ring = is_k ? Ks : Vs;
        uint64_t* full = is_k ? k_full : v_full;
        uint64_t* empty = is_k ? k_empty : v_empty;
        bool ok = true;
        if (lane < 2 && ngroups > 0) prefetch_tmap(tmap);
        for (int pass = 0; pass < 2; ++pass) {
            for (int g = 0; ok && lane < 2 && g < ngroups; ++g) {
                const int gg = pass * ngroups + g;
                const int st = gg % C::NST, use = gg / C::NST;
                if (!(ok = mbar_wait(empty + st, (use & 1) ^ 1, p.status, detail_base | (is_k ? 0x01u : 0x02u))))
                    break;
                const int nb = min(C::GB, nsel - g * C::GB);
                mbar_arrive_expect_tx(full + st, static_cast<uint32_t>(nb * BLK * D * 2));
                for (int u = 0; u < nb; ++u) {
                    const int krow = static_cast<int>((static_cast<int64_t>(b) * p.Hkv + kvh) * p.N +
                                                      static_cast<int64_t>(list[g * C::GB + u]) * BLK);
#pragma unroll
                    for (int s = 0; s < C::DS; ++s)
                        tma_load_2d(ring + st * C::KG_BYTES + s * C::SUB + u * BLK * 128, tmap, s * 64, krow,
                                    full + st);
                }
                issued_last = gg;
            }
            __syncwarp();
            if (pass == 0 && !second_pass()) break;
        }
    } else if (warp == C::MMA_WARP) {
        bool ok = true;
        int g0 = 0;  // groups of earlier passes
        for (int pass = 0; pass < 2; ++pass) {
            g0 = pass * ngroups;
            if (lane == 0 && ngroups > 0 && ok) {
                // Operand descriptors are formed once; every tile the MMAs read lies at a fixed offset
                // from these bases. The start-address field holds address / 16 in 14 bits, and shared
                // memory ends below 2^18 bytes, so adding offset / 16 never carries out of the field.
                const uint64_t dq0 = smem_desc_sw128(smem_u32(Qs), 16, 1024);
                const uint64_t dk0 = smem_desc_sw128(smem_u32(Ks), 16, 1024);
                const uint64_t dv0 = smem_desc_sw128(smem_u32(Vs), C::SUB, 1024);
                constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
                if (pass == 0) ok = mbar_wait(q_full, 0, p.status, detail_base | 0x10u);
                tc_fence_after();
                // S[h] = Q_h K_g^T (after P.V of group g-1 on tile h has released the TMEM columns)
                auto qk = [&](int g, int h) -> bool {
                    const int gg = g0 + g;
                    const int st = gg % C::NST;
                    if (gg > 0 && !mbar_wait(pv_done + h, (gg - 1) & 1, p.status, detail_base | 0x12u)) return false;
                    tc_fence_after();
                    const int ncols = min(C::GB, nsel - g * C::GB) * BLK;
                    const uint32_t idesc_qk = idesc_bf16_f32(128, ncols, 0, 0);
                    const uint32_t d_tmem = tm + C::S_COL + h * 128;
                    const uint64_t a0 = dq0 + static_cast<uint32_t>((h * C::DS * C::SUB) >> 4);
                    const uint64_t b0 = dk0 + static_cast<uint32_t>((st * C::KG_BYTES) >> 4);
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
                    const int gg = g0 + g;
                    const int st = gg % C::NST;
                    if (!mbar_wait(p_full + h, gg & 1, p.status, detail_base | 0x14u)) return false;
                    tc_fence_after();
                    const int nks = min(C::GB, nsel - g * C::GB) * BLK / 16;
                    const uint32_t d_tmem = tm + C::O_COL + h * D;
                    const uint32_t a_tmem = tm + C::S_COL + h * 128;
                    const uint64_t b0 = dv0 + static_cast<uint32_t>((st * C::KG_BYTES) >> 4);
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
                for (int g = 0; ok && g < ngroups; ++g) {
                    const int gg = g0 + g;
                    const int st = gg % C::NST, ph = (gg / C::NST) & 1;
                    if (!(ok = mbar_wait(k_full + st, ph, p.status, detail_base | 0x11u))) break;
                    if (!(ok = qk(g, 0))) break;
                    if (NM == 2) {
                        if (g > 0) {
                            // P.V(1, g-1) goes between the two Q.K^T of group g
                            if (!(ok = pv(g - 1, 1))) break;
                            mma_commit(v_empty + (gg - 1) % C::NST);
                        }
                        if (!(ok = qk(g, 1))) break;
                    }
                    mma_commit(k_empty + st);
                    if (!(ok = mbar_wait(v_full + st, ph, p.status, detail_base | 0x13u))) break;
                    if (!(ok = pv(g, 0))) break;
                    if (NM == 1) mma_commit(v_empty + st);
                }
                if (ok && NM == 2) {
                    if ((ok = pv(ngroups - 1, 1))) mma_commit(v_empty + (g0 + ngroups - 1) % C::NST);
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
        const int R = h * 128 + r;        // row inside the CTA
        const bool valid = R < p.gh * BLK;
        const int hh = R / BLK, t = R % BLK;
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
            const int64_t orow = (static_cast<int64_t>(b) * p.Hq + head) * p.N + static_cast<int64_t>(i) * BLK + t;
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
    if (warp == C::PRODUCER_WARP && lane < 2) {
        // every TMA load this CTA issued has landed before shared memory is released
        uint64_t* full = lane == 0 ? k_full : v_full;
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

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// 2-D view [rows, D] of a bf16 [.., tokens, D] tensor; boxes of 64 columns x box_rows rows, 128-byte swizzle.
bool make_tmap_2d(CUtensorMap* m, const void* ptr, int64_t rows, int D, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D view [rows, D] of an fp32 tensor; boxes of 32 columns (128 bytes) x 128 rows, 128-byte swizzle.
bool make_tmap_2d_f32(CUtensorMap* m, const void* ptr, int64_t rows, int D) {
    EncodeTiledFn enc = encode_fn();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 4};
    const cuuint32_t box[2] = {32, 128};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int BLK, int NM>
static bool launch_variant(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const AttnParams& p,
                           dim3 grid, cudaStream_t st) {
    using C = PrefillCfg<D, BLK, NM>;
    static std::atomic<uint64_t> configured{0};
    if (!configure_smem_once(reinterpret_cast<const void*>(attn_prefill_kernel<D, BLK, NM>), C::SMEM, configured))
        return false;
    attn_prefill_kernel<D, BLK, NM><<<grid, C::THREADS, C::SMEM, st>>>(q, k, v, p);
    return cudaGetLastError() == cudaSuccess;
}

pisa_status launch_attn_prefill(const Plan& pl, const void* Q, const void* K, const void* V, const AttnParams& p,
                                cudaStream_t st, int32_t* launches) {
    CUtensorMap tq, tk, tv;
    const int64_t qrows = static_cast<int64_t>(pl.B) * pl.Hq * pl.N;
    const int64_t krows = static_cast<int64_t>(pl.B) * pl.Hkv * pl.N;
    if (!make_tmap_2d(&tq, Q, qrows, pl.D, pl.blk) || !make_tmap_2d(&tk, K, krows, pl.D, pl.blk) ||
        !make_tmap_2d(&tv, V, krows, pl.D, pl.blk))
        return PISA_ERR_CUDA;
    const int nm = p.gh * pl.blk > 128 ? 2 : 1;
    dim3 grid(pl.nqb, pl.Hsel * p.chunks, pl.B);
    if (nm == 1 && pl.nqb >= 2) {
        // units of at most 128 rows: two query blocks per CTA, one per tile
        if (!launch_attn_prefill_dual(pl.D, pl.blk, tq, tk, tv, p, grid, st)) return PISA_ERR_CUDA;
        ++*launches;
        return PISA_OK;
    }
    bool ok = false;
    if (pl.D == 128 && pl.blk == 64)
        ok = nm == 2 ? launch_variant<128, 64, 2>(tq, tk, tv, p, grid, st)
                     : launch_variant<128, 64, 1>(tq, tk, tv, p, grid, st);
    else if (pl.D == 128 && pl.blk == 128)
        ok = launch_variant<128, 128, 1>(tq, tk, tv, p, grid, st);
    else if (pl.D == 64 && pl.blk == 64)
        ok = nm == 2 ? launch_variant<64, 64, 2>(tq, tk, tv, p, grid, st)
                     : launch_variant<64, 64, 1>(tq, tk, tv, p, grid, st);
    else if (pl.D == 64 && pl.blk == 128)
        ok = launch_variant<64, 128, 1>(tq, tk, tv, p, grid, st);
    else
        return PISA_ERR_UNSUPPORTED;
    if (!ok) return PISA_ERR_CUDA;
    ++*launches;
    return PISA_OK;
}

}  // namespace pisa
