// Dense prefill scoring on the tensor cores ("La selection top-K guidee par la
// pyramide", PISA page): every query-block summary of one selection row
// against every eligible pyramid node of the levels the descent can visit, as
// fp32 dot products q . node, written to the score plane that descent_kernel
// reads. A tile is skipped when none of its nodes is eligible for any of its
// query blocks at its level (a query block needs level l only when its descent
// starts at l or above, and only nodes up to its last eligible one).
//
// One CTA per 128 query blocks x 128 nodes. Every fp32 operand value x enters
// as a tf32 head h (x with its 13 low mantissa bits cleared) and the exact fp32
// remainder r = x - h, written by split_tf32_kernel into the workspace before
// the tiles run; tcgen05 MMAs of kind tf32 accumulate h*h + h*r + r*h in TMEM.
// The dropped r*r term and the remainders' own tf32 rounding are below 2^-21
// of |q||node| per product, the size of fp32 rounding over the dot product, so
// the ranking the descent draws from these scores differs from an fp32 dot
// product only where two scores agree to about six digits (a near-tie).
//
// The four operand chunks of 32 columns (heads and remainders of both sides)
// arrive by 2-D TMA (32 columns x 128 rows per box, 128-byte swizzle) into one
// 64 KB stage; thread 0 runs the copy-MMA loop over D, and three CTAs share an
// SM so that one CTA's copies overlap the others' MMAs and stores. The eight
// warps then read the 128 x 128 accumulator out of TMEM (warp w: query blocks
// 32 (w % 4).., nodes 64 (w / 4)..) and store it through a padded shared tile,
// 32 consecutive nodes of one row per store instruction.
#include <cuda.h>

#include "pisa_device.cuh"

namespace pisa {

constexpr int kStTile = 128;                 // query blocks and nodes per tile
constexpr int kStChunk = 32;                 // D per stage (one 128-byte swizzle atom of fp32)
constexpr int kStThreads = 256;
constexpr int kStOp = kStTile * kStChunk * 4;  // one operand chunk: 16 KB
constexpr int kStStage = 4 * kStOp;            // A head, A remainder, B head, B remainder
constexpr int kStSmem = 1024 + kStStage + 256;  // three CTAs share an SM

// kind::tf32 instruction descriptor: fp32 accumulator, A and B tf32, both K-major.
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int m, int n) {
    return (1u << 4) | (2u << 7) | (2u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(m >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// head and remainder of n4 float4 values (grid-stride)
__global__ void __launch_bounds__(256) split_tf32_kernel(const float4* src0, float4* hi0, float4* lo0, int64_t n0,
                                                         const float4* src1, float4* hi1, float4* lo1, int64_t n1) {
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < n0 + n1; e += stride) {
        const bool first = e < n0;
        const int64_t k = first ? e : e - n0;
        const float4 x = first ? src0[k] : src1[k];
        float4 h, r;
        h.x = __uint_as_float(__float_as_uint(x.x) & 0xFFFFE000u);
        h.y = __uint_as_float(__float_as_uint(x.y) & 0xFFFFE000u);
        h.z = __uint_as_float(__float_as_uint(x.z) & 0xFFFFE000u);
        h.w = __uint_as_float(__float_as_uint(x.w) & 0xFFFFE000u);
        r.x = x.x - h.x;
        r.y = x.y - h.y;
        r.z = x.z - h.z;
        r.w = x.w - h.w;
        (first ? hi0 : hi1)[k] = h;
        (first ? lo0 : lo1)[k] = r;
    }
}

bool launch_split_tf32(const float* src0, float* hi0, float* lo0, int64_t n0, const float* src1, float* hi1,
                       float* lo1, int64_t n1, cudaStream_t st) {
    const int64_t n4 = (n0 + n1) / 4;
    const int64_t want = (n4 + 255) / 256;
    const int64_t blocks = want < 148 * 8 ? want : 148 * 8;
    if (blocks <= 0) return true;
    split_tf32_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        reinterpret_cast<const float4*>(src0), reinterpret_cast<float4*>(hi0), reinterpret_cast<float4*>(lo0),
        n0 / 4, reinterpret_cast<const float4*>(src1), reinterpret_cast<float4*>(hi1), reinterpret_cast<float4*>(lo1),
        n1 / 4);
    return cudaGetLastError() == cudaSuccess;
}

template <int D>
__global__ void __launch_bounds__(kStThreads, 3)
    score_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmN,
                    const SelectParams p) {
    constexpr int NC = D / kStChunk;
    extern __shared__ uint8_t st_raw[];
    uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(st_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(base + kStStage);  // the stage's copies landed
    uint64_t* done = full + 1;                                       // the MMAs of the stage completed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

    const int hs = blockIdx.y, b = blockIdx.z;
    int tile = blockIdx.x, l = 0;
    while (l + 1 < p.L && tile >= p.tile_off[l + 1]) ++l;
    tile -= p.tile_off[l];
    const int i_end = p.i_lo + p.nqc;
    const int i0 = p.i_lo + (tile / p.tiles_c[l]) * kStTile;
    const int c0 = (tile % p.tiles_c[l]) * kStTile;
    const int i_hi = min(i0 + kStTile, i_end) - 1;
    const int64_t last_hi = p.causal ? i_hi : p.n0_valid - 1;
    // the descent's start level and the eligible nodes only grow with the query block
    int start = -1;
    for (int ll = p.L - 1; ll >= 0; --ll)
        if (div_width(p, last_hi, ll) + 1 > p.budget[ll]) {
            start = ll;
            break;
        }
    if (start < l || c0 > div_width(p, last_hi, l)) return;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int kvh = hs / p.gsel_div;
    // head rows of the tile; the remainder rows follow the whole head array
    const int qrows = static_cast<int>(gridDim.z) * p.Hsel * p.nqb;
    const int nrows = static_cast<int>(gridDim.z) * p.Hkv * p.total_nodes;
    const int qrow = static_cast<int>((static_cast<int64_t>(b) * p.Hsel + hs) * p.nqb + i0);
    const int nrow = static_cast<int>((static_cast<int64_t>(b) * p.Hkv + kvh) * p.total_nodes + p.loff[l] + c0);
    const uint32_t detail_base = kKernSelect << 8;

    if (tid == 0) {
        mbar_init(full, 1);
        mbar_init(done, 1);
        fence_barrier_init();
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmN);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 128);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tm = *tmem_slot;

    auto op_ptr = [&](int op) { return base + op * kStOp; };  // op: 0 A head, 1 A rest, 2 B head, 3 B rest
    // thread 0 runs the copies and the MMAs: chunk c's copies land, its MMAs run, and once they
    // have read the stage the next chunk's copies start
    bool ok = true;
    if (tid == 0) {
        constexpr uint32_t idesc = idesc_tf32_f32(128, 128);
        const uint64_t ah = smem_desc_sw128(smem_u32(op_ptr(0)), 16, 1024);
        const uint64_t ar = smem_desc_sw128(smem_u32(op_ptr(1)), 16, 1024);
        const uint64_t bh = smem_desc_sw128(smem_u32(op_ptr(2)), 16, 1024);
        const uint64_t br = smem_desc_sw128(smem_u32(op_ptr(3)), 16, 1024);
        int loaded = 0, committed = 0;
        for (int c = 0; c < NC; ++c) {
            if (c > 0 && !(ok = mbar_wait(done, (c - 1) & 1, p.status, detail_base | 0x42u))) break;
            mbar_arrive_expect_tx(full, 4 * kStOp);
            tma_load_2d(op_ptr(0), &tmQ, c * kStChunk, qrow, full);
            tma_load_2d(op_ptr(1), &tmQ, c * kStChunk, qrow + qrows, full);
            tma_load_2d(op_ptr(2), &tmN, c * kStChunk, nrow, full);
            tma_load_2d(op_ptr(3), &tmN, c * kStChunk, nrow + nrows, full);
            ++loaded;
            if (!(ok = mbar_wait(full, c & 1, p.status, detail_base | 0x41u))) break;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < kStChunk / 8; ++ks) {
                const uint32_t off = static_cast<uint32_t>((ks * 32) >> 4);  // 8 tf32 = 32 bytes per K step
                mma_tf32_ss(tm, ah + off, bh + off, idesc, (c > 0 || ks > 0) ? 1u : 0u);
                mma_tf32_ss(tm, ah + off, br + off, idesc, 1u);
                mma_tf32_ss(tm, ar + off, bh + off, idesc, 1u);
            }
            mma_commit(done);
            ++committed;
        }
        // every MMA issued has completed (the last commit covers all), and every copy started has
        // landed (only the last can be pending), before the epilogue and before memory is released
        if (committed > 0) mbar_wait(done, (committed - 1) & 1, p.status, detail_base | 0x43u);
        if (loaded > committed) mbar_wait(full, (loaded - 1) & 1, p.status, detail_base | 0x44u);
    }
    ok = __syncthreads_and(ok);
    tc_fence_after();
    if (ok) {
        // warp w reads TMEM lanes 32 (w % 4).. (query blocks) and node columns 64 (w / 4).. in two
        // 32-column pieces; each piece goes through a padded shared tile so that the stores cover
        // 32 consecutive nodes of one row per instruction (the stages are free: every MMA is done)
        float* stile = reinterpret_cast<float*>(base) + warp * 32 * 33;
        const int q4 = warp & 3, half = warp >> 2;
        const int ncols = min(kStTile, p.lsize[l] - c0);
        const int64_t prow0 = (static_cast<int64_t>(b) * p.Hsel + hs) * p.qc - p.i_lo;  // plane row of block 0
#pragma unroll 1
        for (int q = 0; q < 2; ++q) {
            const int col0 = half * 64 + q * 32;
            uint32_t v[32];
            tmem_ld32(tm + (static_cast<uint32_t>(q4 * 32) << 16) + col0, v);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) stile[lane * 33 + k] = __uint_as_float(v[k]);
            __syncwarp();
            const int col = col0 + lane;
#pragma unroll 4
            for (int r = 0; r < 32; ++r) {
                const int i = i0 + q4 * 32 + r;
                if (i < i_end && col < ncols) p.scores[(prow0 + i) * p.total_nodes + p.loff[l] + c0 + col] = stile[r * 33 + lane];
            }
            __syncwarp();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tm, 128);
    }
}

bool launch_score_tc(const SelectParams& p, dim3 grid, cudaStream_t st) {
    const int64_t qrows = static_cast<int64_t>(grid.z) * p.Hsel * p.nqb;
    const int64_t nrows = static_cast<int64_t>(grid.z) * p.Hkv * p.total_nodes;
    if (2 * qrows >= (int64_t(1) << 31) || 2 * nrows >= (int64_t(1) << 31)) return false;
    CUtensorMap tq, tn;
    if (!make_tmap_2d_f32(&tq, p.qsplit, 2 * qrows, p.D) || !make_tmap_2d_f32(&tn, p.nsplit, 2 * nrows, p.D))
        return false;
    static std::atomic<uint64_t> configured[2] = {};
    const int k = p.D == 64 ? 0 : 1;
    if (!configure_smem_once(k == 0 ? reinterpret_cast<const void*>(score_tc_kernel<64>)
                                    : reinterpret_cast<const void*>(score_tc_kernel<128>),
                             kStSmem, configured[k]))
        return false;
    if (k == 0)
        score_tc_kernel<64><<<grid, kStThreads, kStSmem, st>>>(tq, tn, p);
    else
        score_tc_kernel<128><<<grid, kStThreads, kStSmem, st>>>(tq, tn, p);
    return cudaGetLastError() == cudaSuccess;
}

}  // namespace pisa
