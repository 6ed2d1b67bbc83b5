// Decode attention for callers that cannot allocate device memory.
//
// Some callers may not call cudaMalloc at all: code that runs inside another
// framework's memory pool, a plugin that owns no allocator, or a serving loop
// that must not allocate once it is running. For them,
// pisa_decode_attention_noalloc runs the same split-KV decode kernels as
// pisa_sparse_attention, with the split partials and the status word in a
// fixed array that is part of this library (kNoAllocScratchBytes, 8 MiB).
// Every GPU that loads the library holds that array until the process exits.
//
// Host code cannot pass the array's name to a kernel (on the host it only
// stands in for the symbol), so every call looks up its device address with
// cudaGetSymbolAddress, with the calling device current. The lookup allocates
// nothing; doing it per call (rather than caching the address) keeps it right
// after the device's context is torn down and created again. The first call on
// a device may load the library's device code there, so it should come before
// any stream capture. Every call on a
// device shares the one array: two calls whose kernels overlap on the GPU
// (different streams, no ordering between them) race on it.
//
// Each call clears the array's status word before its kernels run; the
// kernels record an out-of-range block index or a pipeline wait that ran out
// of time there, and pisa_decode_noalloc_check_status reads and clears it.
#include <cuda_runtime.h>

#include "pisa.h"
#include "pisa_internal.h"

namespace pisa {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device.
static cudaError_t noalloc_scratch(void** out) {
    return cudaGetSymbolAddress(out, g_noalloc_scratch);
}

}  // namespace pisa

using namespace pisa;

extern "C" pisa_status pisa_decode_attention_noalloc(const pisa_shape* shape, const void* Q, const void* K,
                                                     const void* V, const int32_t* idx, void* O, float* lse,
                                                     pisa_stream_t stream) {
    Plan pl;
    const pisa_status s = make_plan(shape, &pl);
    if (s != PISA_OK) return s;
    if (!pl.decode) return PISA_ERR_INVALID_ARG;
    const auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
    if (Q == nullptr || K == nullptr || V == nullptr || idx == nullptr || O == nullptr || misaligned(Q) ||
        misaligned(K) || misaligned(V) || misaligned(O) || misaligned(idx))
        return PISA_ERR_INVALID_ARG;
    const size_t part_bytes =
        static_cast<size_t>(pl.B) * pl.Hsel * pl.dec_splits * pl.gsel * (pl.D + 2) * sizeof(float);
    if (kStatusBytes + part_bytes > kNoAllocScratchBytes) return PISA_ERR_WORKSPACE;
    if (injected_launch_failure()) return PISA_ERR_CUDA;

    void* scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return PISA_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // the array keeps the previous call's contents: the status word must start at zero (the
    // partials need no clearing: every split writes its partial before the merge reads it)
    if (cudaMemsetAsync(scratch, 0, kStatusBytes, st) != cudaSuccess) return PISA_ERR_CUDA;

    DecodeParams d{};
    d.Q = static_cast<const __nv_bfloat16*>(Q);
    d.K = static_cast<const __nv_bfloat16*>(K);
    d.V = static_cast<const __nv_bfloat16*>(V);
    d.idx = idx;
    d.part = reinterpret_cast<float*>(static_cast<unsigned char*>(scratch) + kStatusBytes);
    d.O = static_cast<__nv_bfloat16*>(O);
    d.lse = lse;
    d.status = static_cast<uint32_t*>(scratch);
    d.Hq = pl.Hq;
    d.Hkv = pl.Hkv;
    d.g = pl.g;
    d.N = pl.N;
    d.n0 = pl.n0;
    d.D = pl.D;
    d.blk = pl.blk;
    d.topk = pl.topk;
    d.per_qhead = pl.per_qhead;
    d.Hsel = pl.Hsel;
    d.gh = pl.gsel;
    d.bps = pl.dec_bps;
    d.splits = pl.dec_splits;
    d.scale_log2 = pl.scale * 1.4426950408889634f;
    int32_t launches = 0;
    return launch_attn_decode(pl, d, st, &launches) ? PISA_OK : PISA_ERR_CUDA;
}

extern "C" pisa_status pisa_decode_noalloc_check_status(uint32_t* detail, pisa_stream_t stream) {
    void* scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return PISA_ERR_CUDA;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint32_t host[2] = {0, 0};
    if (cudaMemcpyAsync(host, scratch, sizeof(host), cudaMemcpyDeviceToHost, st) != cudaSuccess) return PISA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return PISA_ERR_CUDA;
    if (host[0] != 0) {
        if (cudaMemsetAsync(scratch, 0, sizeof(host), st) != cudaSuccess) return PISA_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return PISA_ERR_CUDA;
    }
    if (detail) *detail = host[1];
    return static_cast<pisa_status>(host[0]);
}
