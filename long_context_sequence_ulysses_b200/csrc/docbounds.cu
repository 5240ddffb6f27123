// docbounds.cu -- per-token document starts and per-tile key ranges from
// position_ids, plus the longest-first tile schedule.
//
// Packed documents are masked through position ids rather than a 4-D mask
// (page "Ulysses verteilt Millionen-Token-Kontexte auf mehrere GPUs", section
// "Integration in den Hugging-Face-Stack"): a document starts wherever the id
// is 0 (and at token 0), so
//     doc_start[i] = max{ j <= i : pos[j] == 0 }   (0 if there is none),
// an inclusive max-scan of (pos[j] == 0 ? j : 0). Row i attends to keys
// [doc_start[i], i]; since doc_start never decreases, a 128-row query tile
// starting at r0 needs key tiles doc_start[r0]/128 .. r0/128 and nothing else.
//
// Kernels: a block-local scan, a fix-up with the carry of earlier blocks
// (which also writes each query tile's first key), for the backward the last
// query row of each key tile (a binary search over doc_start), and a counting
// sort of the scheduling units by work, heaviest first: query tiles (the
// backward, and a forward whose items pair two heads of one KV group), pairs
// of consecutive query tiles (a forward with an odd group size), and key
// tiles (the backward).
#include "ulysses_internal.cuh"

namespace uly {

namespace {

__device__ __forceinline__ int warp_incl_max(int v)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if ((threadIdx.x & 31) >= o) v = max(v, u);
    }
    return v;
}

// Block-local inclusive max-scan over kScanBlock tokens (one per thread).
__global__ void __launch_bounds__(kScanBlock) doc_scan_kernel(const int32_t *__restrict__ pos, int64_t N,
                                                             int32_t *__restrict__ doc_start,
                                                             int32_t *__restrict__ block_agg,
                                                             uint32_t *__restrict__ status)
{
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        status[0] = 0u;   // fresh status for this call
        status[1] = 0u;   // work counter of the persistent forward kernel
    }
    __shared__ int warp_max[kScanBlock / 32];
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kScanBlock + threadIdx.x;
    int v = (i < N && pos[i] == 0) ? static_cast<int>(i) : 0;
    v = warp_incl_max(v);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 31) warp_max[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = warp_max[lane];
        w = warp_incl_max(w);
        warp_max[lane] = w;
    }
    __syncthreads();
    if (warp > 0) v = max(v, warp_max[warp - 1]);
    if (i < N) doc_start[i] = v;
    if (threadIdx.x == kScanBlock - 1) block_agg[blockIdx.x] = v;
}

// Adds the carry of all earlier blocks and records each query tile's first key.
__global__ void __launch_bounds__(kScanBlock) doc_fixup_kernel(int64_t N, int32_t *__restrict__ doc_start,
                                                              const int32_t *__restrict__ block_agg,
                                                              int32_t *__restrict__ tile_lo)
{
    __shared__ int red[kScanBlock / 32];
    int c = 0;
    for (int b = threadIdx.x; b < static_cast<int>(blockIdx.x); b += kScanBlock) c = max(c, block_agg[b]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c = max(c, __shfl_xor_sync(0xffffffffu, c, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = c;
    __syncthreads();
    if (threadIdx.x < 32) {
        int w = red[threadIdx.x];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) w = max(w, __shfl_xor_sync(0xffffffffu, w, o));
        if (threadIdx.x == 0) red[0] = w;
    }
    __syncthreads();
    const int carry = red[0];
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kScanBlock + threadIdx.x;
    if (i < N) {
        const int v = max(doc_start[i], carry);
        doc_start[i] = v;
        if ((i % kTileM) == 0) tile_lo[i / kTileM] = v;
    }
}

// For key tile t: one past the last query row whose document reaches a key of
// the tile, i.e. the number of rows i with doc_start[i] <= min(t*128+127, N-1).
__global__ void kv_qend_kernel(int64_t N, int T, const int32_t *__restrict__ doc_start, int32_t *__restrict__ kv_qend)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    const int64_t last_key = min(static_cast<int64_t>(t) * kTileN + kTileN - 1, N - 1);
    int64_t lo = last_key, hi = N;   // doc_start[last_key] <= last_key always holds
    while (hi - lo > 1) {            // invariant: doc_start[lo] <= last_key, doc_start[hi] > last_key (or hi == N)
        const int64_t mid = (lo + hi) >> 1;
        if (doc_start[mid] <= last_key) lo = mid; else hi = mid;
    }
    kv_qend[t] = static_cast<int32_t>(hi);
}

// Work of one scheduling unit. kQueryPairs: unit u is the pair of query
// tiles (2u, 2u+1), work = key tiles visited by both (src = tile_lo, each
// query tile's first key). kQueryTiles: unit t is query tile t, work = key
// tiles it visits. kKeyTiles: unit t is key tile t, work = query tiles that
// visit it (src = kv_qend).
enum class Unit { kQueryPairs, kQueryTiles, kKeyTiles };

template <Unit kUnit>
__device__ __forceinline__ int unit_work(int t, int T, const int32_t *__restrict__ src)
{
    if (kUnit == Unit::kKeyTiles) return static_cast<int>((src[t] + kTileM - 1) / kTileM) - t;
    if (kUnit == Unit::kQueryTiles) return t - src[t] / kTileN + 1;
    const int ta = 2 * t, tb = 2 * t + 1;
    int w = ta - src[ta] / kTileN + 1;
    if (tb < T) w += tb - src[tb] / kTileN + 1;
    return w;
}

// Exclusive prefix sum over the 1024 threads of a block (warp shuffles, then
// the 32 warp totals in warp 0). warp_tot: 32 ints of shared memory.
__device__ __forceinline__ int block_excl_sum_1024(int v, int *warp_tot)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += u;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += u;
        }
        warp_tot[lane] = w;
    }
    __syncthreads();
    const int r = (warp > 0 ? warp_tot[warp - 1] : 0) + x - v;
    __syncthreads();   // warp_tot may be reused after this
    return r;
}

// Largest work value whose histogram is kept in shared memory.
constexpr int kOrderSmemWork = 11999;   // 48 KB of static shared memory with warp_tot

// Counting sort of `units` scheduling units by work (in [0, max_work]),
// heaviest first. One CTA of 1024 threads; the histogram lives in shared
// memory up to kOrderSmemWork, else in global scratch [max_work + 1]. Units
// of equal work are placed in arrival order of the atomics (any order is a
// valid schedule).
template <Unit kUnit>
__global__ void __launch_bounds__(1024) unit_order_kernel(int units, int T, int max_work,
                                                         const int32_t *__restrict__ src,
                                                         int32_t *__restrict__ ghist, int32_t *__restrict__ order)
{
    __shared__ int shist[kOrderSmemWork + 1];
    __shared__ int warp_tot[32];
    int *hist = max_work <= kOrderSmemWork ? shist : ghist;
    const int tid = threadIdx.x;
    for (int w = tid; w <= max_work; w += 1024) hist[w] = 0;
    __syncthreads();
    for (int t = tid; t < units; t += 1024) atomicAdd(&hist[unit_work<kUnit>(t, T, src)], 1);
    __syncthreads();
    // Exclusive prefix over work values in DESCENDING order: the slot of the
    // first unit with work w is the number of units with work > w. Thread tid
    // owns a contiguous segment of work values counted from the top.
    const int per = (max_work + 1 + 1023) / 1024;
    const int hi = max_work - tid * per;     // segment covers work values hi, hi-1, ..., hi-per+1
    int sum = 0;
    for (int k = 0; k < per; ++k) {
        const int w = hi - k;
        if (w >= 0) sum += hist[w];
    }
    int run = block_excl_sum_1024(sum, warp_tot);   // units with work above this segment
    for (int k = 0; k < per; ++k) {
        const int w = hi - k;
        if (w >= 0) {
            const int c = hist[w];
            hist[w] = run;
            run += c;
        }
    }
    __syncthreads();
    for (int t = tid; t < units; t += 1024) {
        const int p = atomicAdd(&hist[unit_work<kUnit>(t, T, src)], 1);
        order[p] = t;
    }
}

}  // namespace

cudaError_t launch_docbounds(const int32_t *pos, int64_t N, char *ws, const WsLayout &L, bool backward,
                             bool fwd_tile_pairs, cudaStream_t stream)
{
    const int64_t T = ceil_div(N, kTileM);
    const int nb = static_cast<int>(ceil_div(N, kScanBlock));
    int32_t *doc_start = reinterpret_cast<int32_t *>(ws + L.doc_start);
    int32_t *tile_lo = reinterpret_cast<int32_t *>(ws + L.tile_lo);
    int32_t *block_agg = reinterpret_cast<int32_t *>(ws + L.block_agg);
    int32_t *scratch = reinterpret_cast<int32_t *>(ws + L.scratch);
    doc_scan_kernel<<<nb, kScanBlock, 0, stream>>>(pos, N, doc_start, block_agg,
                                                   reinterpret_cast<uint32_t *>(ws + L.status));
    doc_fixup_kernel<<<nb, kScanBlock, 0, stream>>>(N, doc_start, block_agg, tile_lo);
    if (!backward && fwd_tile_pairs) {
        const int pairs = static_cast<int>(ceil_div(T, 2));
        unit_order_kernel<Unit::kQueryPairs><<<1, 1024, 0, stream>>>(pairs, static_cast<int>(T),
                                                                     static_cast<int>(2 * T), tile_lo, scratch,
                                                                     reinterpret_cast<int32_t *>(ws + L.q_order));
    } else {
        unit_order_kernel<Unit::kQueryTiles><<<1, 1024, 0, stream>>>(static_cast<int>(T), static_cast<int>(T),
                                                                     static_cast<int>(T), tile_lo, scratch,
                                                                     reinterpret_cast<int32_t *>(ws + L.q_order));
    }
    if (backward) {
        int32_t *kv_qend = reinterpret_cast<int32_t *>(ws + L.kv_qend);
        kv_qend_kernel<<<static_cast<int>(ceil_div(T, 256)), 256, 0, stream>>>(N, static_cast<int>(T), doc_start,
                                                                               kv_qend);
        unit_order_kernel<Unit::kKeyTiles><<<1, 1024, 0, stream>>>(static_cast<int>(T), static_cast<int>(T),
                                                                   static_cast<int>(T), kv_qend, scratch,
                                                                   reinterpret_cast<int32_t *>(ws + L.kv_order));
    }
    return cudaGetLastError();
}

}  // namespace uly
