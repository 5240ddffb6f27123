// noalloc.cu -- ulysses_attn_fwd_noalloc: the attention forward for callers
// that cannot allocate device memory.
//
// Some callers only ever receive their input and output buffers: a plugin
// running inside a host framework whose device memory all belongs to the
// framework's own pool, or a latency-critical path that must not call
// cudaMalloc (which can synchronise the whole device). They have nowhere to
// put the forward's workspace (per-token document starts, per-tile key ranges,
// the tile schedule and the status word). This entry point keeps that scratch
// in a file-scope device array instead, so the caller passes only inputs and
// outputs and nothing is allocated.
//
// Limits and sharing rules:
//  - the array holds the workspace of up to kNoAllocMaxTokens = 131072 tokens
//    (544 KiB); longer sequences are rejected with ULYSSES_ERR_UNSUPPORTED;
//  - every GPU that loads the library holds the array until the process exits;
//  - all calls on a device share the one array and it keeps the last call's
//    contents; the kernels overwrite or clear everything they read, but calls
//    that overlap on the GPU (different streams, or unordered host threads)
//    race on it and give wrong results;
//  - the first call on each device looks up the array's device address with
//    cudaGetSymbolAddress, with that device current; make that first call
//    before any stream capture;
//  - a bounded device wait that runs out is recorded in the array's status
//    word, which this entry point cannot report (it returns before the
//    kernels run).
#include "ulysses.h"
#include "ulysses_internal.cuh"

#include <cuda_runtime.h>

#include <mutex>

namespace uly {
namespace {

constexpr int64_t kNoAllocMaxTokens = 131072;
constexpr size_t kNoAllocScratchBytes = 544 * 1024;

// The forward's workspace for up to kNoAllocMaxTokens tokens. In host code
// this name is only a host-side stand-in; the kernels get the device address
// obtained below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once
// per device). Returns null and sets *err on failure.
void *scratch_address(cudaError_t *err)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) { *err = e; return nullptr; }
    if (dev < 0 || dev >= kMaxDevices) { *err = cudaErrorInvalidDevice; return nullptr; }
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) { *err = e != cudaSuccess ? e : cudaErrorInvalidSymbol; return nullptr; }
        g_scratch_addr[dev] = p;
    }
    *err = cudaSuccess;
    return g_scratch_addr[dev];
}

}  // namespace
}  // namespace uly

extern "C" int ulysses_attn_fwd_noalloc(const void *q, const void *k, const void *v, const int32_t *position_ids,
                                        int64_t N, int Hl, int Hkvl, int d, float scale, void *o, float *lse,
                                        void *stream)
{
    using namespace uly;
    clear_last_error();
    if (N > kNoAllocMaxTokens)
        return set_last_error(ULYSSES_ERR_UNSUPPORTED,
                              "ulysses_attn_fwd_noalloc: N exceeds the static scratch limit of 131072 tokens");
    if (N >= 0 && Hl >= 1 && ws_layout(N, Hl, false).total > kNoAllocScratchBytes)
        return set_last_error(ULYSSES_ERR_UNSUPPORTED, "ulysses_attn_fwd_noalloc: workspace exceeds the static scratch");
    cudaError_t e = cudaSuccess;
    void *ws = scratch_address(&e);
    if (!ws) return set_last_error(ULYSSES_ERR_CUDA, "ulysses_attn_fwd_noalloc: cudaGetSymbolAddress failed");
    return ulysses_attn_fwd(q, k, v, position_ids, N, Hl, Hkvl, d, scale, o, lse, ws, kNoAllocScratchBytes, stream);
}
