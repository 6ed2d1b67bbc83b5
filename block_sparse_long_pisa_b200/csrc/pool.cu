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
// Both kernels compute a contiguous range of rows or nodes, so that appending
// blocks to a KV cache recomputes only what changed, with the same arithmetic.
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

template <int D>
__global__ void __launch_bounds__(256) block_mean_kernel(const MeanParams p) {
    constexpr int CH = D / 8;     // 16-byte chunks per row
    constexpr int RPI = 32 / CH;  // rows one warp covers per load instruction
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
        int r = rsub;
        // eight loads in flight per lane before the first add
        for (; r + 7 * RPI < p.rows_per_group; r += 8 * RPI) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = ldg_stream(base + static_cast<int64_t>(r + u * RPI) * D);
#pragma unroll
            for (int u = 0; u < 8; ++u) acc_bf16x8(acc, v[u]);
        }
        for (; r < p.rows_per_group; r += RPI) acc_bf16x8(acc, ldg_stream(base + static_cast<int64_t>(r) * D));
    }
#pragma unroll
    for (int off = CH; off < 32; off <<= 1) {
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] += __shfl_xor_sync(0xFFFFFFFFu, acc[k], off);
    }
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
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int64_t wsum = 0;
    for (int u = 0; u < p.factor; ++u) {
        const int64_t ch = static_cast<int64_t>(c) * p.factor + u;
        if (ch >= p.n_below) break;
        const int64_t lo = ch * p.width_below;
        const int64_t hi = min((ch + 1) * p.width_below, static_cast<int64_t>(p.n0));
        if (hi <= lo) break;  // this child and the ones after it hold no key
        const float w = static_cast<float>(hi - lo);
        const float4 v = *reinterpret_cast<const float4*>(below + ch * p.D);
        acc.x += w * v.x;
        acc.y += w * v.y;
        acc.z += w * v.z;
        acc.w += w * v.w;
        wsum += hi - lo;
    }
    const float inv = wsum > 0 ? 1.0f / static_cast<float>(wsum) : 0.f;
    float* dst = p.pyr + (plane * p.plane_rows + p.off_cur + c) * p.D + 4 * q;
    *reinterpret_cast<float4*>(dst) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
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

bool launch_pyramid_level(const LevelParams& p, cudaStream_t st) {
    const int64_t threads = static_cast<int64_t>(p.planes) * p.n_cur * (p.D / 4);
    const int64_t blocks = (threads + 255) / 256;
    pyramid_level_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(p);
    return cudaGetLastError() == cudaSuccess;
}

}  // namespace pisa
