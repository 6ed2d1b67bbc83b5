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
// Warp roles (warp-specialised pipeline, all hand-off through mbarriers):
//   warps 0 .. 4*NM-1  softmax: warp w owns TMEM lanes 32*(w%4).. of tile w/4,
//                      one query row per thread
//   warp 4*NM          producer: one lane issues the TMA loads (Q once, then
//                      K and V of every selected block into an NST-deep ring)
//   warp 4*NM+1        MMA: allocates TMEM and one lane issues tcgen05.mma
//
// Per selected block j and tile h:
//   S[h][j&1] = Q_h K_j^T           (tcgen05, M=128, N=b, K=D, fp32 in TMEM)
//   softmax reads S, finds the row max, keeps a running max that only moves
//   when the new max exceeds it by more than 2^8 (the output and the row sum
//   are rescaled then), writes P = exp2(S*c - m) as bf16 into shared memory
//   (two P buffers per tile, so P for block j+1 can be written while P.V of
//   block j still reads the other one)
//   O[h] += P_h V_j                 (tcgen05, M=128, N=D, K=b, fp32 in TMEM)
// The MMA lane issues S for block j+1 before O for block j, so the tensor
// core works on one tile while the softmax warps work on the other. No score
// ever leaves TMEM/shared memory; O is normalised once at the end.
//
// Softmax arithmetic per row and block: a three-input max tree, packed fp32
// pair instructions (f32x2) for the scale-and-subtract and the row sum, and
// the exponentials split between the MUFU unit (two thirds) and a polynomial
// on the FMA pipes (one third), which balances the two.
//
// Shared memory operands use the 128-byte swizzle: Q, K and P are K-major
// (head dim / key index contiguous), V is read MN-major straight from its
// [key, dim] layout.
#include <cuda.h>
#include <cuda_bf16.h>

#include "pisa_device.cuh"

namespace pisa {

template <int D, int BLK, int NM>
struct PrefillCfg {
    static constexpr int DS = D / 64;                  // 128-byte column tiles along the head dim
    static constexpr int BS = BLK / 64;                // 128-byte column tiles along the key block
    static constexpr int SUB = 128 * 128;              // one [128 rows x 128 B] operand tile
    static constexpr int Q_BYTES = NM * DS * SUB;
    static constexpr int P_BUF = NM * BS * SUB;         // one P buffer (all tiles)
    static constexpr int P_BYTES = 2 * P_BUF;
    static constexpr int KV_SUB = BLK * 128;           // one [BLK rows x 128 B] tile
    static constexpr int KV_BYTES = DS * KV_SUB;       // a whole K (or V) block
    static constexpr int MAX_LIST = kMaxPrefillTopk;   // selected blocks per query block
    static constexpr int AUX = 256 + MAX_LIST * 4;     // barriers, TMEM slot, block list
    static constexpr int SMEM_LIMIT = 232448;          // 227 KB opt-in maximum
    static constexpr int NST_FIT = (SMEM_LIMIT - 1024 - Q_BYTES - P_BYTES - AUX) / (2 * KV_BYTES);
    static constexpr int NST = NST_FIT > 4 ? 4 : NST_FIT;
    static constexpr int SMEM = 1024 + Q_BYTES + P_BYTES + NST * 2 * KV_BYTES + AUX;
    static constexpr int O_COL = 0;
    static constexpr int S_COL = NM * D;
    static constexpr int TMEM_NEED = NM * D + 2 * NM * BLK;
    static constexpr int TMEM_COLS = TMEM_NEED <= 32    ? 32
                                     : TMEM_NEED <= 64  ? 64
                                     : TMEM_NEED <= 128 ? 128
                                     : TMEM_NEED <= 256 ? 256
                                                        : 512;
    static constexpr int SOFTMAX_WARPS = 4 * NM;
    static constexpr int PRODUCER_WARP = SOFTMAX_WARPS;
    static constexpr int MMA_WARP = SOFTMAX_WARPS + 1;
    static constexpr int THREADS = 32 * (SOFTMAX_WARPS + 2);
    static_assert(NST >= 2, "shared memory too small for a double-buffered K/V ring");
    static_assert(TMEM_NEED <= 512, "TMEM budget exceeded");
};

// Lazy rescale threshold (log2 units): the running max is kept until a new
// row max exceeds it by this much, so probabilities stay below 2^8.
constexpr float kRescaleThreshold = 8.0f;
// Pairs of scores k with k % kPolyMod == kPolyMod - 1 take the FMA-pipe exp2.
constexpr int kPolyMod = 3;

template <int D, int BLK, int NM>
__global__ void __launch_bounds__(PrefillCfg<D, BLK, NM>::THREADS, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
    using C = PrefillCfg<D, BLK, NM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* Qs = base;
    uint8_t* Ps = Qs + C::Q_BYTES;
    uint8_t* Ks = Ps + C::P_BYTES;
    uint8_t* Vs = Ks + C::NST * C::KV_BYTES;
    uint8_t* aux = Vs + C::NST * C::KV_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(aux);
    uint64_t* q_full = bars;                        // 1
    uint64_t* k_full = q_full + 1;                  // NST
    uint64_t* v_full = k_full + C::NST;             // NST
    uint64_t* kv_empty = v_full + C::NST;           // NST
    uint64_t* s_full = kv_empty + C::NST;           // NM*2
    uint64_t* s_empty = s_full + NM * 2;            // NM*2
    uint64_t* p_full = s_empty + NM * 2;            // NM*2: P buffer written by the softmax
    uint64_t* p_empty = p_full + NM * 2;            // NM*2: P.V that read the buffer completed
    uint64_t* mma_final = p_empty + NM * 2;         // 1
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_final + 1);
    int32_t* s_nsel = reinterpret_cast<int32_t*>(tmem_slot + 1);
    int32_t* list = reinterpret_cast<int32_t*>(aux + 256);

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

    if (tid == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(k_full + s, 1);
            mbar_init(v_full + s, 1);
            mbar_init(kv_empty + s, 1);
        }
        for (int h = 0; h < NM; ++h) {
            mbar_init(s_full + 2 * h, 1);
            mbar_init(s_full + 2 * h + 1, 1);
            mbar_init(s_empty + 2 * h, 128);
            mbar_init(s_empty + 2 * h + 1, 128);
            mbar_init(p_full + 2 * h, 128);
            mbar_init(p_full + 2 * h + 1, 128);
            mbar_init(p_empty + 2 * h, 1);
            mbar_init(p_empty + 2 * h + 1, 1);
        }
        mbar_init(mma_final, 1);
        fence_barrier_init();
    }
    if (warp == C::MMA_WARP) tmem_alloc(tmem_slot, C::TMEM_COLS);
    if (warp == C::PRODUCER_WARP) {
        // compact the selected-block row: valid entries in order, bad ones recorded
        const int32_t* row = p.idx + ((static_cast<int64_t>(b) * p.Hsel + hs) * p.nqb + i) * p.topk;
        int cnt = 0;
        for (int t0 = 0; t0 < p.topk; t0 += 32) {
            const int t = t0 + lane;
            const int32_t j = t < p.topk ? row[t] : -1;
            const bool ok = j >= 0 && j < p.n0 && (!p.causal || j <= i);
            if (t < p.topk && j >= 0 && !ok) record_error(p.status, PISA_ERR_BAD_INDEX, detail_base | 0xB0u);
            const uint32_t m = __ballot_sync(0xFFFFFFFFu, ok);
            if (ok && cnt + __popc(m & ((1u << lane) - 1u)) < C::MAX_LIST) list[cnt + __popc(m & ((1u << lane) - 1u))] = j;
            cnt += __popc(m);
        }
        if (lane == 0) *s_nsel = cnt < C::MAX_LIST ? cnt : C::MAX_LIST;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;
    const int nsel = *s_nsel;

    int issued_last[C::NST];  // producer: last ring use issued per stage (-1 = none)
#pragma unroll
    for (int s = 0; s < C::NST; ++s) issued_last[s] = -1;
    bool issued_any_mma = false;

    if (warp == C::PRODUCER_WARP) {
        if (lane == 0 && nsel > 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            mbar_arrive_expect_tx(q_full, static_cast<uint32_t>(p.gh * BLK * D * 2));
            for (int hh = 0; hh < p.gh; ++hh) {
                const int r0 = hh * BLK;
                const int qrow = static_cast<int>((static_cast<int64_t>(b) * p.Hq + head0 + hh) * p.N +
                                                  static_cast<int64_t>(i) * BLK);
#pragma unroll
                for (int s = 0; s < C::DS; ++s)
                    tma_load_2d(Qs + ((r0 / 128) * C::DS + s) * C::SUB + (r0 % 128) * 128, &tmQ, s * 64, qrow,
                                q_full);
            }
            for (int j = 0; j < nsel; ++j) {
                const int st = j % C::NST, use = j / C::NST;
                if (!mbar_wait(kv_empty + st, (use & 1) ^ 1, p.status, detail_base | 0x01u)) break;
                const int krow = static_cast<int>((static_cast<int64_t>(b) * p.Hkv + kvh) * p.N +
                                                  static_cast<int64_t>(list[j]) * BLK);
                mbar_arrive_expect_tx(k_full + st, C::KV_BYTES);
#pragma unroll
                for (int s = 0; s < C::DS; ++s)
                    tma_load_2d(Ks + st * C::KV_BYTES + s * C::KV_SUB, &tmK, s * 64, krow, k_full + st);
                mbar_arrive_expect_tx(v_full + st, C::KV_BYTES);
#pragma unroll
                for (int s = 0; s < C::DS; ++s)
                    tma_load_2d(Vs + st * C::KV_BYTES + s * C::KV_SUB, &tmV, s * 64, krow, v_full + st);
                issued_last[st] = use;
            }
        }
        __syncwarp();
    } else if (warp == C::MMA_WARP) {
        if (lane == 0 && nsel > 0) {
            constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BLK, 0, 0);
            constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
            const uint32_t q_addr = smem_u32(Qs), k_addr = smem_u32(Ks), v_addr = smem_u32(Vs),
                           p_addr = smem_u32(Ps);
            bool ok = mbar_wait(q_full, 0, p.status, detail_base | 0x10u);
            tc_fence_after();
            for (int j = 0; ok && j <= nsel; ++j) {
                if (j < nsel) {
                    const int st = j % C::NST;
                    if (!(ok = mbar_wait(k_full + st, (j / C::NST) & 1, p.status, detail_base | 0x11u))) break;
                    const int buf = j & 1;
                    for (int h = 0; h < NM; ++h) {
                        if (!(ok = mbar_wait(s_empty + 2 * h + buf, ((j >> 1) & 1) ^ 1, p.status,
                                             detail_base | 0x12u)))
                            break;
                        tc_fence_after();
                        const uint32_t d_tmem = tm + C::S_COL + (buf * NM + h) * BLK;
#pragma unroll
                        for (int ks = 0; ks < D / 16; ++ks) {
                            const uint32_t koff = (ks % 4) * 32;
                            const uint64_t a = smem_desc_sw128(q_addr + (h * C::DS + ks / 4) * C::SUB + koff, 16, 1024);
                            const uint64_t bd = smem_desc_sw128(
                                k_addr + st * C::KV_BYTES + (ks / 4) * C::KV_SUB + koff, 16, 1024);
                            mma_bf16_ss(d_tmem, a, bd, idesc_qk, ks > 0 ? 1u : 0u);
                        }
                        mma_commit(s_full + 2 * h + buf);
                        issued_any_mma = true;
                    }
                    if (!ok) break;
                }
                if (j >= 1) {
                    const int jj = j - 1, st = jj % C::NST;
                    if (!(ok = mbar_wait(v_full + st, (jj / C::NST) & 1, p.status, detail_base | 0x13u))) break;
                    const int pb = jj & 1;
                    for (int h = 0; h < NM; ++h) {
                        if (!(ok = mbar_wait(p_full + 2 * h + pb, (jj >> 1) & 1, p.status, detail_base | 0x14u)))
                            break;
                        tc_fence_after();
                        const uint32_t d_tmem = tm + C::O_COL + h * D;
#pragma unroll
                        for (int ks = 0; ks < BLK / 16; ++ks) {
                            const uint32_t koff = (ks % 4) * 32;
                            const uint64_t a = smem_desc_sw128(
                                p_addr + pb * C::P_BUF + (h * C::BS + ks / 4) * C::SUB + koff, 16, 1024);
                            const uint64_t bd = smem_desc_sw128(v_addr + st * C::KV_BYTES + ks * 16 * 128,
                                                                C::KV_SUB, 1024);
                            mma_bf16_ss(d_tmem, a, bd, idesc_pv, (jj > 0 || ks > 0) ? 1u : 0u);
                        }
                        mma_commit(p_empty + 2 * h + pb);
                        issued_any_mma = true;
                    }
                    if (!ok) break;
                    mma_commit(kv_empty + st);
                }
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- softmax warps
        const int h = warp / 4;
        const int qd = warp % 4;
        const int r = qd * 32 + lane;     // row inside tile h
        const int R = h * 128 + r;        // row inside the CTA
        const bool valid = R < p.gh * BLK;
        const int hh = R / BLK, t = R % BLK;
        const uint32_t lane_base = static_cast<uint32_t>(qd * 32) << 16;
        const float cs = p.scale_log2;
        const uint64_t cs2 = f2_pack(cs, cs);
        float m_used = -INFINITY, l_sum = 0.f;
        bool ok = true;
        for (int j = 0; j < nsel; ++j) {
            const int buf = j & 1;
            ok = mbar_wait(s_full + 2 * h + buf, (j >> 1) & 1, p.status, detail_base | 0x20u);
            if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
            tc_fence_after();
            float sv[BLK];
#pragma unroll
            for (int c = 0; c < BLK / 32; ++c)
                tmem_ld32(tm + lane_base + C::S_COL + (buf * NM + h) * BLK + c * 32,
                          *reinterpret_cast<uint32_t(*)[32]>(sv + c * 32));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(s_empty + 2 * h + buf);

            const bool diag = p.causal && list[j] == i;  // uniform across the CTA
            if (diag) {
#pragma unroll
                for (int c = 0; c < BLK; ++c) sv[c] = c > t ? -INFINITY : sv[c];
            }
            // row max: eight independent three-input max chains
            float mq[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) mq[q] = sv[q];
#pragma unroll
            for (int c = 8; c + 16 <= BLK; c += 16) {
#pragma unroll
                for (int q = 0; q < 8; ++q) mq[q] = fmax3(mq[q], sv[c + q], sv[c + 8 + q]);
            }
            if ((BLK - 8) % 16 != 0) {
#pragma unroll
                for (int q = 0; q < 8; ++q) mq[q] = fmaxf(mq[q], sv[BLK - 8 + q]);
            }
            const float mx = fmaxf(fmax3(mq[0], mq[1], mq[2]), fmax3(mq[3], mq[4], fmax3(mq[5], mq[6], mq[7])));
            const float mxs = mx * cs;
            bool resc = false;
            float m_new = m_used;
            if (j == 0) {
                m_new = mxs;
            } else if (mxs > m_used + kRescaleThreshold) {
                resc = true;
                m_new = mxs;
            }
            const float alpha = resc ? fast_exp2(m_used - m_new) : 1.0f;
            const uint64_t negm2 = f2_pack(-m_new, -m_new);
            uint32_t pk[BLK / 2];
            uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int k = 0; k < BLK / 2; ++k) {
                float x0, x1;
                f2_unpack(f2_fma(f2_pack(sv[2 * k], sv[2 * k + 1]), cs2, negm2), x0, x1);
                uint64_t e2;
                if (!diag && (k % kPolyMod) == kPolyMod - 1) {
                    e2 = exp2_poly_x2(x0, x1);
                } else {
                    e2 = f2_pack(fast_exp2(x0), fast_exp2(x1));
                }
                sum2[k & 3] = f2_add(sum2[k & 3], e2);
                float e0, e1;
                f2_unpack(e2, e0, e1);
                pk[k] = pack_bf16x2(e0, e1);
            }
            float r0, r1, r2, r3;
            f2_unpack(f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3])), r0, r1);
            const float rs = r0 + r1;
            (void)r2;
            (void)r3;
            if (j > 0 && __any_sync(0xFFFFFFFFu, resc)) {
                // O must hold P.V of block j-1 before it is rescaled
                const int pj = j - 1;
                ok = mbar_wait(p_empty + 2 * h + (pj & 1), (pj >> 1) & 1, p.status, detail_base | 0x21u);
                if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    const uint32_t addr = tm + lane_base + C::O_COL + h * D + c * 32;
                    tmem_ld32(addr, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
                    tmem_st32(addr, o);
                }
                tmem_wait_st();
            }
            l_sum = l_sum * alpha + rs;
            m_used = m_new;
            // this P buffer was last read by P.V of block j-2
            ok = mbar_wait(p_empty + 2 * h + buf, ((j >> 1) & 1) ^ 1, p.status, detail_base | 0x23u);
            if (!__all_sync(0xFFFFFFFFu, ok)) { ok = false; break; }
            if (valid) {
#pragma unroll
                for (int ps = 0; ps < C::BS; ++ps) {
                    const uint32_t rowaddr = smem_u32(Ps + buf * C::P_BUF + (h * C::BS + ps) * C::SUB) + r * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t* q4 = pk + ps * 32 + c * 4;
                        st_shared_v4(rowaddr + ((c ^ (r & 7)) << 4), q4[0], q4[1], q4[2], q4[3]);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(p_full + 2 * h + buf);
        }
        // ---------------------------------------------------------------- epilogue
        if (ok) {
            const int head = head0 + hh;
            const int64_t orow = (static_cast<int64_t>(b) * p.Hq + head) * p.N + static_cast<int64_t>(i) * BLK + t;
            if (nsel > 0) {
                const int pj = nsel - 1;
                ok = mbar_wait(p_empty + 2 * h + (pj & 1), (pj >> 1) & 1, p.status, detail_base | 0x22u);
                ok = __all_sync(0xFFFFFFFFu, ok);
            }
            if (ok) {
                tc_fence_after();
                const float inv = nsel > 0 ? 1.0f / l_sum : 0.f;
                uint4* dst = reinterpret_cast<uint4*>(p.O + orow * D);
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    if (nsel > 0) {
                        tmem_ld32(tm + lane_base + C::O_COL + h * D + c * 32, o);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] = 0u;
                    }
                    if (valid) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            uint4 v;
                            v.x = pack_bf16x2(__uint_as_float(o[8 * k + 0]) * inv, __uint_as_float(o[8 * k + 1]) * inv);
                            v.y = pack_bf16x2(__uint_as_float(o[8 * k + 2]) * inv, __uint_as_float(o[8 * k + 3]) * inv);
                            v.z = pack_bf16x2(__uint_as_float(o[8 * k + 4]) * inv, __uint_as_float(o[8 * k + 5]) * inv);
                            v.w = pack_bf16x2(__uint_as_float(o[8 * k + 6]) * inv, __uint_as_float(o[8 * k + 7]) * inv);
                            dst[c * 4 + k] = v;
                        }
                    }
                }
                if (valid && p.lse != nullptr)
                    p.lse[orow] = nsel > 0 ? (m_used + __log2f(l_sum)) * 0.69314718055994531f : -INFINITY;
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncthreads();
    if (warp == C::PRODUCER_WARP && lane == 0) {
        // every TMA load this CTA issued has landed before shared memory is released
        for (int s = 0; s < C::NST; ++s) {
            if (issued_last[s] < 0) continue;
            mbar_wait(k_full + s, issued_last[s] & 1, p.status, detail_base | 0x30u);
            mbar_wait(v_full + s, issued_last[s] & 1, p.status, detail_base | 0x31u);
        }
        if (nsel > 0) mbar_wait(q_full, 0, p.status, detail_base | 0x32u);
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
static bool make_tmap(CUtensorMap* m, const void* ptr, int64_t rows, int D, int box_rows) {
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

template <int D, int BLK, int NM>
static bool launch_variant(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const AttnParams& p,
                           dim3 grid, cudaStream_t st) {
    using C = PrefillCfg<D, BLK, NM>;
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(attn_prefill_kernel<D, BLK, NM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::SMEM) != cudaSuccess)
            return false;
        configured = true;
    }
    attn_prefill_kernel<D, BLK, NM><<<grid, C::THREADS, C::SMEM, st>>>(q, k, v, p);
    return cudaGetLastError() == cudaSuccess;
}

pisa_status launch_attn_prefill(const Plan& pl, const void* Q, const void* K, const void* V, const AttnParams& p,
                                cudaStream_t st, int32_t* launches) {
    CUtensorMap tq, tk, tv;
    const int64_t qrows = static_cast<int64_t>(pl.B) * pl.Hq * pl.N;
    const int64_t krows = static_cast<int64_t>(pl.B) * pl.Hkv * pl.N;
    if (!make_tmap(&tq, Q, qrows, pl.D, pl.blk) || !make_tmap(&tk, K, krows, pl.D, pl.blk) ||
        !make_tmap(&tv, V, krows, pl.D, pl.blk))
        return PISA_ERR_CUDA;
    const int nm = p.gh * pl.blk > 128 ? 2 : 1;
    dim3 grid(pl.nqb, pl.Hsel * p.chunks, pl.B);
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
