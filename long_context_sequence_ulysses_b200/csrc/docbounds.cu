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
// Kernels (all short; measured faster than one CTA doing everything, whose
// serial passes over the ids sit on the attention's critical path):
//   1. doc_scan: block-local scan of 1024 tokens per block, block maxima;
//   2. (more than 1024 blocks only) carry_prefix: one CTA turns the block maxima
//      into each block's carry, so that the total work stays O(N);
//   3. doc_fixup: adds the carry of earlier blocks, writes each query tile's
//      first key;
//   4. backward only: the last query row of each key tile (binary search);
//   5. unit_order: a counting sort of the scheduling units by work, heaviest
//      first -- query tiles (the backward, and a forward whose items pair two
//      heads of one KV group), pairs of consecutive query tiles (a forward with
//      an odd group size), key tiles (the backward) -- counting only key tiles
//      inside the forward's key window. The forward's attention kernel is
//      launched as a programmatic dependent of the last sort, which lets it
//      start its prologue while the sort runs. For the forward (up to 2^20
//      tokens) steps 3 and 5 share one launch: the last fix-up block to finish
//      runs the sort (one launch fewer: 1.1 % faster on a 0.19 ms forward).
#include "ulysses_internal.cuh"

namespace uly {

namespace {

constexpr int kDbThreads = 1024;

__device__ __forceinline__ int warp_incl_max(int v)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if ((threadIdx.x & 31) >= o) v = max(v, u);
    }
    return v;
}

// Inclusive max-scan of v over the 1024 threads of the block. wmax: 32 ints of shared memory.
__device__ __forceinline__ int block_incl_max_1024(int v, int *wmax)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_incl_max(v);
    if (lane == 31) wmax[warp] = v;
    __syncthreads();
    if (warp == 0) wmax[lane] = warp_incl_max(wmax[lane]);
    __syncthreads();
    if (warp > 0) v = max(v, wmax[warp - 1]);
    __syncthreads();   // wmax may be reused after this
    return v;
}

// 1. Block-local inclusive max-scan over kScanBlock tokens (one per thread).
__global__ void __launch_bounds__(kScanBlock) doc_scan_kernel(const int32_t *__restrict__ pos, int64_t N,
                                                             int32_t *__restrict__ doc_start,
                                                             int32_t *__restrict__ block_agg,
                                                             uint32_t *__restrict__ status)
{
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        status[0] = 0u;   // fresh status for this call
        status[1] = 0u;   // work counter of the persistent forward kernel
        status[2] = 0u;   // fix-up blocks finished (the forward's fused fix-up and sort)
    }
    __shared__ int wmax[32];
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kScanBlock + threadIdx.x;
    const int v = block_incl_max_1024((i < N && pos[i] == 0) ? static_cast<int>(i) : 0, wmax);
    if (i < N) doc_start[i] = v;
    if (threadIdx.x == kScanBlock - 1) block_agg[blockIdx.x] = v;
}

// 2. More than kScanBlock blocks: block b's carry = max of block_agg[0..b), by
// one CTA walking the maxima 1024 at a time (O(nb) in all).
__global__ void __launch_bounds__(kScanBlock) carry_prefix_kernel(const int32_t *__restrict__ block_agg, int nb,
                                                                 int32_t *__restrict__ block_carry)
{
    __shared__ int wmax[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int run = 0;   // maximum of the blocks of earlier passes
    for (int base = 0; base < nb; base += kScanBlock) {
        const int b = base + threadIdx.x;
        const int incl = block_incl_max_1024(b < nb ? block_agg[b] : 0, wmax);   // wmax: prefix over warps
        const int prev = __shfl_up_sync(0xffffffffu, incl, 1);
        const int excl = lane ? prev : (warp ? wmax[warp - 1] : 0);
        if (b < nb) block_carry[b] = max(run, excl);
        run = max(run, wmax[31]);
        __syncthreads();   // wmax is rewritten by the next pass
    }
}

// 3. Adds the carry of all earlier blocks and records each query tile's first
// key. With at most kScanBlock blocks every block reduces the maxima before it
// (one load per thread); beyond that it reads the carry computed in step 2.
__device__ __forceinline__ void fixup_block(int64_t N, int nb, int32_t *__restrict__ doc_start,
                                            const int32_t *__restrict__ block_agg,
                                            const int32_t *__restrict__ block_carry, int32_t *__restrict__ tile_lo,
                                            int *red)
{
    int carry;
    if (nb <= kScanBlock) {
        int c = threadIdx.x < static_cast<int>(blockIdx.x) ? block_agg[threadIdx.x] : 0;
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
        carry = red[0];
    } else {
        carry = block_carry[blockIdx.x];
    }
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kScanBlock + threadIdx.x;
    if (i < N) {
        const int v = max(doc_start[i], carry);
        doc_start[i] = v;
        if ((i % kTileM) == 0) tile_lo[i / kTileM] = v;
    }
}

__global__ void __launch_bounds__(kScanBlock) doc_fixup_kernel(int64_t N, int nb, int32_t *__restrict__ doc_start,
                                                              const int32_t *__restrict__ block_agg,
                                                              const int32_t *__restrict__ block_carry,
                                                              int32_t *__restrict__ tile_lo)
{
    __shared__ int red[32];
    fixup_block(N, nb, doc_start, block_agg, block_carry, tile_lo, red);
}

// For key tile t: one past the last query row whose document reaches a key of
// the tile, i.e. the number of rows i with doc_start[i] <= min(t*128+127, N-1).
__device__ __forceinline__ int key_tile_qend(int64_t N, int t, const int32_t *doc_start)
{
    const int64_t last_key = min(static_cast<int64_t>(t) * kTileN + kTileN - 1, N - 1);
    int64_t lo = last_key, hi = N;   // doc_start[last_key] <= last_key always holds
    while (hi - lo > 1) {            // invariant: doc_start[lo] <= last_key, doc_start[hi] > last_key (or hi == N)
        const int64_t mid = (lo + hi) >> 1;
        if (doc_start[mid] <= last_key) lo = mid; else hi = mid;
    }
    return static_cast<int>(hi);
}

// Work of one scheduling unit, in key tiles inside the key window.
// kQueryPairs: unit u is the pair of query tiles (q_tile0 + 2u, q_tile0 + 2u + 1),
// work = key tiles visited by both (src = tile_lo, each query tile's first
// key); the order lists u. kQueryTiles: unit u is query tile q_tile0 + u, work
// = key tiles it visits; the order lists the tile itself. kKeyTiles: unit t is
// key tile t, work = query tiles that visit it (src = kv_qend).
enum class Unit { kQueryPairs, kQueryTiles, kKeyTiles };

// (L2 loads: in the fused fix-up and sort, other blocks wrote these values.)
__device__ __forceinline__ int query_tile_work(int t, const int32_t *tile_lo, const DbWindow &w)
{
    return max(0, min(t, w.kvhi_t) - max(__ldcg(tile_lo + t) / kTileN, w.kvlo_t) + 1);
}

template <Unit kUnit>
__device__ __forceinline__ int unit_work(int u, const int32_t *src, const DbWindow &w)
{
    if (kUnit == Unit::kKeyTiles) return static_cast<int>((__ldcg(src + u) + kTileM - 1) / kTileM) - u;
    if (kUnit == Unit::kQueryTiles) return query_tile_work(w.q_tile0 + u, src, w);
    const int ta = w.q_tile0 + 2 * u, tb = ta + 1;
    int work = query_tile_work(ta, src, w);
    if (tb < w.q_tile0 + w.q_tiles) work += query_tile_work(tb, src, w);
    return work;
}

template <Unit kUnit>
__device__ __forceinline__ int unit_label(int u, const DbWindow &w)
{
    return kUnit == Unit::kQueryTiles ? w.q_tile0 + u : u;
}

// Exclusive prefix sum over the 1024 threads of the block (warp shuffles, then
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
constexpr int kOrderSmemWork = 11999;

// Counting sort of `units` scheduling units by work (in [0, max_work]),
// heaviest first, by the whole block. The histogram lives in shared memory up
// to kOrderSmemWork, else in global scratch [max_work + 1]. Units of equal
// work are placed in arrival order of the atomics (any order is a valid
// schedule).
template <Unit kUnit>
__device__ void unit_order(int units, const DbWindow &win, int max_work, const int32_t *src, int *shist,
                           int32_t *ghist, int *warp_tot, int32_t *order)
{
    int *hist = max_work <= kOrderSmemWork ? shist : ghist;
    const int tid = threadIdx.x;
    for (int w = tid; w <= max_work; w += kDbThreads) hist[w] = 0;
    __syncthreads();
    for (int t = tid; t < units; t += kDbThreads) atomicAdd(&hist[unit_work<kUnit>(t, src, win)], 1);
    __syncthreads();
    // Exclusive prefix over work values in DESCENDING order: the slot of the
    // first unit with work w is the number of units with work > w. Thread tid
    // owns a contiguous segment of work values counted from the top.
    const int per = (max_work + 1 + kDbThreads - 1) / kDbThreads;
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
    for (int t = tid; t < units; t += kDbThreads) {
        const int p = atomicAdd(&hist[unit_work<kUnit>(t, src, win)], 1);
        order[p] = unit_label<kUnit>(t, win);
    }
    __syncthreads();
}

// 4. For each key tile: one past the last query row that reaches it.
__global__ void kv_qend_kernel(int64_t N, int T, const int32_t *__restrict__ doc_start, int32_t *__restrict__ kv_qend)
{
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t < T) kv_qend[t] = key_tile_qend(N, t, doc_start);
}

// 5. One schedule. `trigger`: the kernel after this one (the forward's
// attention kernel) may start its prologue right away; it reads this kernel's
// results only after its grid-dependency wait.
template <Unit kUnit>
__global__ void __launch_bounds__(kDbThreads, 1) unit_order_kernel(int units, DbWindow win, int max_work,
                                                                  const int32_t *__restrict__ src,
                                                                  int32_t *__restrict__ ghist,
                                                                  int32_t *__restrict__ order, int trigger)
{
    if (trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ int shist[kOrderSmemWork + 1];
    __shared__ int wtot[32];
    unit_order<kUnit>(units, win, max_work, src, shist, ghist, wtot, order);
}

// 3 + 5 for the forward (at most kScanBlock scan blocks): the fix-up, then
// the last block to finish it (counted in status[2], which the scan zeroed)
// sorts the schedule. One launch fewer on the attention's critical path; no
// block waits for another. Every block lets the attention kernel start its
// prologue right away.
template <Unit kUnit>
__global__ void __launch_bounds__(kScanBlock, 1)
    doc_fixup_order_kernel(int64_t N, int nb, int32_t *__restrict__ doc_start, const int32_t *__restrict__ block_agg,
                           int32_t *__restrict__ tile_lo, uint32_t *__restrict__ done, int units, DbWindow win,
                           int max_work, int32_t *__restrict__ ghist, int32_t *__restrict__ order)
{
    static_assert(kDbThreads == kScanBlock, "the sort runs on one fix-up block");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ int red[32];
    __shared__ int shist[kOrderSmemWork + 1];
    __shared__ int wtot[32];
    __shared__ int last;
    fixup_block(N, nb, doc_start, block_agg, nullptr, tile_lo, red);
    __threadfence();   // this block's tile_lo before its count
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(done, 1u) == static_cast<unsigned>(gridDim.x - 1);
    __syncthreads();
    if (!last) return;
    __threadfence();   // every block's tile_lo is visible from here on
    unit_order<kUnit>(units, win, max_work, tile_lo, shist, ghist, wtot, order);
}

}  // namespace

cudaError_t launch_docbounds(const int32_t *pos, int64_t N, char *ws, const WsLayout &L, bool backward,
                             bool fwd_tile_pairs, const DbWindow &win, cudaStream_t stream)
{
    const int T = static_cast<int>(ceil_div(N, kTileM));
    const int nb = static_cast<int>(ceil_div(N, kScanBlock));
    int32_t *doc_start = reinterpret_cast<int32_t *>(ws + L.doc_start);
    int32_t *tile_lo = reinterpret_cast<int32_t *>(ws + L.tile_lo);
    int32_t *q_order = reinterpret_cast<int32_t *>(ws + L.q_order);
    int32_t *block_agg = reinterpret_cast<int32_t *>(ws + L.block_agg);
    int32_t *block_carry = reinterpret_cast<int32_t *>(ws + L.block_carry);
    int32_t *ghist = reinterpret_cast<int32_t *>(ws + L.scratch);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws + L.status);
    doc_scan_kernel<<<nb, kScanBlock, 0, stream>>>(pos, N, doc_start, block_agg, status);
    if (!backward && nb <= kScanBlock) {
        if (fwd_tile_pairs)
            doc_fixup_order_kernel<Unit::kQueryPairs><<<nb, kScanBlock, 0, stream>>>(
                N, nb, doc_start, block_agg, tile_lo, status + 2, (win.q_tiles + 1) / 2, win, 2 * T, ghist, q_order);
        else
            doc_fixup_order_kernel<Unit::kQueryTiles><<<nb, kScanBlock, 0, stream>>>(
                N, nb, doc_start, block_agg, tile_lo, status + 2, win.q_tiles, win, T, ghist, q_order);
        return cudaGetLastError();
    }
    if (nb > kScanBlock) carry_prefix_kernel<<<1, kScanBlock, 0, stream>>>(block_agg, nb, block_carry);
    doc_fixup_kernel<<<nb, kScanBlock, 0, stream>>>(N, nb, doc_start, block_agg, block_carry, tile_lo);
    if (backward) {
        int32_t *kv_qend = reinterpret_cast<int32_t *>(ws + L.kv_qend);
        kv_qend_kernel<<<static_cast<int>(ceil_div(T, 256)), 256, 0, stream>>>(N, T, doc_start, kv_qend);
        unit_order_kernel<Unit::kQueryTiles><<<1, kDbThreads, 0, stream>>>(win.q_tiles, win, T, tile_lo, ghist,
                                                                            q_order, 0);
        unit_order_kernel<Unit::kKeyTiles><<<1, kDbThreads, 0, stream>>>(T, win, T, kv_qend, ghist,
                                                                          reinterpret_cast<int32_t *>(ws + L.kv_order), 0);
    } else if (fwd_tile_pairs) {
        unit_order_kernel<Unit::kQueryPairs><<<1, kDbThreads, 0, stream>>>((win.q_tiles + 1) / 2, win, 2 * T,
                                                                            tile_lo, ghist, q_order, 1);
    } else {
        unit_order_kernel<Unit::kQueryTiles><<<1, kDbThreads, 0, stream>>>(win.q_tiles, win, T, tile_lo, ghist,
                                                                            q_order, 1);
    }
    return cudaGetLastError();
}

}  // namespace uly
