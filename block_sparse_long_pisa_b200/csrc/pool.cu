// Pyramid pooling and query-block summaries ("Le pooling comme premiere
// reduction", PISA page): HBM-streaming means of bf16 rows into fp32.
//
// block_mean_kernel: one warp per output row. The warp reads the rows it
// averages as 16-byte vectors; with D = 128 one warp load instruction covers
// two consecutive 256-byte rows (fully coalesced). Every input byte is read
// once, so the kernel is bound by HBM bandwidth.
//
// pyramid_level_kernel: one thread per (plane, node, 4 floats); a node of
// level l is the mean of its children weighted by the level-0 blocks holding
// keys that each child covers (the last node of a level may have fewer than f
// children; in a cache with spare capacity, nodes past the keys weigh 0, and a
// node over no key at all is 0).
//
// pyramid_subtree_kernel + pyramid_top_kernel: the whole pyramid in two
// launches. A subtree CTA streams the keys of S = f^m consecutive key blocks
// (one warp per block, the block_mean_kernel arithmetic), keeps their means in
// shared memory and forms the m levels above them inside the subtree; one CTA
// per plane then forms the levels above the subtree roots. Compared with one
// launch per level, the small levels no longer cost a launch each; the second
// kernel is a programmatic dependent of the first (it is launched while the
// subtrees stream and waits for their completion), so its launch is hidden.
//
// Every path computes a row mean and a node mean with the same device
// functions in the same order, so a build, an append (which recomputes a
// range with block_mean_kernel and pyramid_level_kernel) and the two-launch
// build agree bit for bit.
#include <cuda_bf16.h>

#include "pisa_device.cuh"

namespace pisa {

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void acc_bf16x8(float (&a)[8], const uint4& v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        a[2 * k] += __uint_as_float(w[k] << 16);
        a[2 * k + 1] += __uint_as_float(w[k] & 0xFFFF0000u);
    }
}

// One lane's share of the sum of `rows` consecutive rows of D bf16 starting at `base` (already
// offset to the lane's 8-column chunk); lane row offset `rsub`, eight loads in flight.
template <int D>
__device__ __forceinline__ void accumulate_rows(const __nv_bfloat16* base, int rows, int rsub, float (&acc)[8]) {
    constexpr int RPI = 32 / (D / 8);  // rows one warp covers per load instruction
    int r = rsub;
    for (; r + 7 * RPI < rows; r += 8 * RPI) {
        uint4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = ldg_stream(base + static_cast<int64_t>(r + u * RPI) * D);
#pragma unroll
        for (int u = 0; u < 8; ++u) acc_bf16x8(acc, v[u]);
    }
    for (; r < rows; r += RPI) acc_bf16x8(acc, ldg_stream(base + static_cast<int64_t>(r) * D));
}

// Sum of the lanes that share a chunk (lanes chunk, chunk + D/8, ...): afterwards every lane
// holds its chunk's total.
template <int D>
__device__ __forceinline__ void reduce_row_lanes(float (&acc)[8]) {
#pragma unroll
    for (int off = D / 8; off < 32; off <<= 1) {
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] += __shfl_xor_sync(0xFFFFFFFFu, acc[k], off);
    }
}

// Mean of the children of node c (in the level below, whose row j sits at rows[(j - first) *
// stride]) weighted by the level-0 blocks holding keys that each child covers; 4 floats at the
// caller's column offset. n0: level-0 blocks that hold keys; width_below: f^(l-1).
__device__ __forceinline__ float4 node_mean4(const float* rows, int64_t first, int stride, int64_t c, int factor,
                                             int64_t n_below, int64_t width_below, int64_t n0) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int64_t wsum = 0;
    for (int u = 0; u < factor; ++u) {
        const int64_t ch = c * factor + u;
        if (ch >= n_below) break;
        const int64_t lo = ch * width_below;
        const int64_t hi = min((ch + 1) * width_below, n0);
        if (hi <= lo) break;  // this child and the ones after it hold no key
        const float w = static_cast<float>(hi - lo);
        const float4 v = *reinterpret_cast<const float4*>(rows + (ch - first) * stride);
        acc.x = __fmaf_rn(w, v.x, acc.x);
        acc.y = __fmaf_rn(w, v.y, acc.y);
        acc.z = __fmaf_rn(w, v.z, acc.z);
        acc.w = __fmaf_rn(w, v.w, acc.w);
        wsum += hi - lo;
    }
    const float inv = wsum > 0 ? 1.0f / static_cast<float>(wsum) : 0.f;
    return make_float4(__fmul_rn(acc.x, inv), __fmul_rn(acc.y, inv), __fmul_rn(acc.z, inv), __fmul_rn(acc.w, inv));
}

template <int D>
__global__ void __launch_bounds__(256) block_mean_kernel(const MeanParams p) {
    constexpr int CH = D / 8;     // 16-byte chunks per row
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t total = static_cast<int64_t>(p.batch) * p.Hout * p.rows_out;
    if (warp >= total) return;
    const int i = p.row0 + static_cast<int>(warp % p.rows_out);
    const int hs = static_cast<int>((warp / p.rows_out) % p.Hout);
    const int b = static_cast<int>(warp / (static_cast<int64_t>(p.rows_out) * p.Hout));
    const int chunk = lane % CH;
    const int rsub = lane / CH;

    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;

    for (int pp = 0; pp < (i < p.rows_valid ? p.planes_per_group : 0); ++pp) {
        const int64_t head = static_cast<int64_t>(hs) * p.planes_per_group + pp;
        const __nv_bfloat16* base = p.src + ((static_cast<int64_t>(b) * p.Hsrc + head) * p.Nsrc +
                                             static_cast<int64_t>(i) * p.rows_per_group) * D + chunk * 8;
        accumulate_rows<D>(base, p.rows_per_group, rsub, acc);
    }
    reduce_row_lanes<D>(acc);
    if (rsub == 0) {
        const float inv = 1.0f / static_cast<float>(p.rows_per_group * p.planes_per_group);
        float* dst = p.dst + ((static_cast<int64_t>(b) * p.Hout + hs) * p.dst_plane_rows + i) * D + chunk * 8;
        float4 lo = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
        float4 hi = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
        reinterpret_cast<float4*>(dst)[0] = lo;
        reinterpret_cast<float4*>(dst)[1] = hi;
    }
}

__global__ void __launch_bounds__(256) pyramid_level_kernel(const LevelParams p) {
    const int q4 = p.D / 4;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t total = static_cast<int64_t>(p.planes) * p.n_cur * q4;
    if (t >= total) return;
    const int q = static_cast<int>(t % q4);
    const int c = p.c0 + static_cast<int>((t / q4) % p.n_cur);
    const int64_t plane = t / (static_cast<int64_t>(q4) * p.n_cur);
    const float* below = p.pyr + (plane * p.plane_rows + p.off_below) * p.D + 4 * q;
    float* dst = p.pyr + (plane * p.plane_rows + p.off_cur + c) * p.D + 4 * q;
    *reinterpret_cast<float4*>(dst) = node_mean4(below, 0, p.D, c, p.factor, p.n_below, p.width_below, p.n0);
}

// The pyramid of S = f^m consecutive key blocks (a subtree) per CTA: level-0 means (one warp per
// block, blocks w, w + warps, ...), then levels 1..m of the subtree from shared memory. Grid:
// planes x subtrees, flattened (subtree fastest). Dynamic shared memory: the subtree's rows of
// levels 0..m, level after level.
template <int D>
__global__ void __launch_bounds__(512) pyramid_subtree_kernel(const SubtreeParams p) {
    extern __shared__ __align__(16) float tree[];
    constexpr int CH = D / 8;
    // the top-level kernel may be launched now (it waits for this grid's completion before it
    // reads anything), so its launch overlaps this grid's work
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t plane = blockIdx.x / p.subtrees;
    const int sub = static_cast<int>(blockIdx.x % p.subtrees);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const int chunk = lane % CH, rsub = lane / CH;
    const int64_t j0 = static_cast<int64_t>(sub) * p.S;
    float* out_plane = p.pyr + plane * p.plane_rows * D;
    // level 0
    for (int r = warp; r < p.S; r += nwarps) {
        const int64_t j = j0 + r;
        if (j >= p.lsize[0]) break;
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.f;
        if (j < p.n0) {
            const __nv_bfloat16* base = p.K + (plane * p.N + j * p.blk) * D + chunk * 8;
            accumulate_rows<D>(base, p.blk, rsub, acc);
        }
        reduce_row_lanes<D>(acc);
        if (rsub == 0) {
            const float inv = 1.0f / static_cast<float>(p.blk);
            const float4 lo = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
            const float4 hi = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
            float4* g = reinterpret_cast<float4*>(out_plane + j * D + chunk * 8);
            float4* t = reinterpret_cast<float4*>(tree + r * D + chunk * 8);
            g[0] = lo;
            g[1] = hi;
            t[0] = lo;
            t[1] = hi;
        }
    }
    // levels 1..m inside the subtree
    int64_t width_below = 1;
    int span_below = p.S;          // rows of the level below held in shared memory
    float* below = tree;
    for (int l = 1; l <= p.m; ++l) {
        __syncthreads();
        const int span = span_below / p.factor;
        float* cur = below + span_below * D;
        const int64_t c0 = j0 / (width_below * p.factor);
        const int64_t first_below = j0 / width_below;
        for (int e = threadIdx.x; e < span * (D / 4); e += blockDim.x) {
            const int cl = e / (D / 4), q = e % (D / 4);
            const int64_t c = c0 + cl;
            if (c >= p.lsize[l]) continue;
            const float4 v = node_mean4(below + 4 * q, first_below, D, c, p.factor, p.lsize[l - 1], width_below, p.n0);
            *reinterpret_cast<float4*>(cur + cl * D + 4 * q) = v;
            *reinterpret_cast<float4*>(out_plane + (p.loff[l] + c) * D + 4 * q) = v;
        }
        below = cur;
        span_below = span;
        width_below *= p.factor;
    }
}

// Levels m+1 .. L-1 of one plane per CTA, level after level. With `in_smem`, the subtree roots
// (level m) are read into shared memory once and every level above is formed there (and written
// out), so the chain after the subtree grid is one round of global loads; otherwise each level
// reads the one below from global memory (planes whose top levels exceed the shared memory).
__global__ void __launch_bounds__(512) pyramid_top_kernel(const SubtreeParams p, const bool in_smem) {
    extern __shared__ __align__(16) float top[];  // [rows of levels m .. L-1][D] when in_smem
    // launched as a programmatic dependent of the subtree kernel: wait until that grid has
    // completed and its writes are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int64_t plane = blockIdx.x;
    float* out_plane = p.pyr + plane * p.plane_rows * p.D;
    int64_t width_below = 1;
    for (int l = 1; l <= p.m; ++l) width_below *= p.factor;
    const int q4 = p.D / 4;
    const float* below = out_plane + static_cast<int64_t>(p.loff[p.m]) * p.D;
    if (in_smem) {
        const float4* src = reinterpret_cast<const float4*>(below);
        for (int e = threadIdx.x; e < p.lsize[p.m] * q4; e += blockDim.x) reinterpret_cast<float4*>(top)[e] = src[e];
        __syncthreads();
        below = top;
    }
    for (int l = p.m + 1; l < p.L; ++l) {
        float* cur = in_smem ? const_cast<float*>(below) + static_cast<int64_t>(p.lsize[l - 1]) * p.D : nullptr;
        float* dst = out_plane + static_cast<int64_t>(p.loff[l]) * p.D;
        for (int e = threadIdx.x; e < p.lsize[l] * q4; e += blockDim.x) {
            const int c = e / q4, q = e % q4;
            const float4 v = node_mean4(below + 4 * q, 0, p.D, c, p.factor, p.lsize[l - 1], width_below, p.n0);
            *reinterpret_cast<float4*>(dst + static_cast<int64_t>(c) * p.D + 4 * q) = v;
            if (in_smem) *reinterpret_cast<float4*>(cur + static_cast<int64_t>(c) * p.D + 4 * q) = v;
        }
        width_below *= p.factor;
        below = in_smem ? cur : dst;
        __syncthreads();
    }
}

bool launch_block_mean(const MeanParams& p, cudaStream_t st) {
    const int64_t warps = static_cast<int64_t>(p.batch) * p.Hout * p.rows_out;
    const int64_t blocks = (warps * 32 + 255) / 256;
    if (blocks <= 0) return true;
    if (p.D == 64)
        block_mean_kernel<64><<<static_cast<unsigned>(blocks), 256, 0, st>>>(p);
    else
        block_mean_kernel<128><<<static_cast<unsigned>(blocks), 256, 0, st>>>(p);
    return cudaGetLastError() == cudaSuccess;
}

// Shared memory the top-level kernel may take for a plane's levels m .. L-1 (beyond it, each level
// reads the one below from global memory).
constexpr size_t kTopSmemLimit = 160 * 1024;

bool launch_pyramid_two_pass(const SubtreeParams& p, cudaStream_t st, int32_t* launches) {
    const int warps = p.S < 16 ? p.S : 16;
    int rows = 0, span = p.S;
    for (int l = 0; l <= p.m; ++l, span /= p.factor) rows += span;
    const size_t smem = static_cast<size_t>(rows) * p.D * sizeof(float);
    const int64_t blocks = static_cast<int64_t>(p.planes) * p.subtrees;
    if (blocks <= 0) return true;
    if (p.D == 64) {
        if (smem > 48 * 1024 && cudaFuncSetAttribute(pyramid_subtree_kernel<64>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     static_cast<int>(smem)) != cudaSuccess)
            return false;
        pyramid_subtree_kernel<64><<<static_cast<unsigned>(blocks), 32 * warps, smem, st>>>(p);
    } else {
        if (smem > 48 * 1024 && cudaFuncSetAttribute(pyramid_subtree_kernel<128>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     static_cast<int>(smem)) != cudaSuccess)
            return false;
        pyramid_subtree_kernel<128><<<static_cast<unsigned>(blocks), 32 * warps, smem, st>>>(p);
    }
    ++*launches;
    if (cudaGetLastError() != cudaSuccess) return false;
    if (p.m + 1 < p.L) {
        size_t top_rows = 0;
        for (int l = p.m; l < p.L; ++l) top_rows += static_cast<size_t>(p.lsize[l]);
        const size_t top_smem = top_rows * p.D * sizeof(float);
        const bool in_smem = top_smem <= kTopSmemLimit;
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(static_cast<unsigned>(p.planes));
        cfg.blockDim = dim3(512);
        cfg.dynamicSmemBytes = in_smem ? top_smem : 0;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (in_smem && top_smem > 48 * 1024 &&
            cudaFuncSetAttribute(pyramid_top_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(kTopSmemLimit)) != cudaSuccess)
            return false;
        if (cudaLaunchKernelEx(&cfg, pyramid_top_kernel, p, in_smem) != cudaSuccess) return false;
        ++*launches;
    }
    return cudaGetLastError() == cudaSuccess;
}

bool launch_pyramid_level(const LevelParams& p, cudaStream_t st) {
    const int64_t threads = static_cast<int64_t>(p.planes) * p.n_cur * (p.D / 4);
    const int64_t blocks = (threads + 255) / 256;
    pyramid_level_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(p);
    return cudaGetLastError() == cudaSuccess;
}

}  // namespace pisa
