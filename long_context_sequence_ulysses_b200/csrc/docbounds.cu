// docbounds.cu -- per-token document starts and per-tile key ranges from
// position_ids, plus the longest-first tile schedule, in one launch.
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
// One CTA of 1024 threads does all of it, so an attention call costs a single
// small launch before its main kernel (which is launched as a programmatic
// dependent of this one and runs its prologue meanwhile):
//   1. the scan, 16384 tokens per pass: each warp scans 512 consecutive tokens
//      (16 coalesced rows of 32), warp totals are scanned by warp 0, and the
//      running maximum carries from pass to pass; every token costs O(1);
//   2. for the backward, the last query row of each key tile (a binary search
//      over doc_start);
//   3. a counting sort of the scheduling units by work, heaviest first: query
//      tiles (the backward, and a forward whose items pair two heads of one KV
//      group), pairs of consecutive query tiles (a forward with an odd group
//      size), and key tiles (the backward).
#include "ulysses_internal.cuh"

namespace uly {

namespace {

constexpr int kDbThreads = 1024;
constexpr int kDbWarps = kDbThreads / 32;
constexpr int kDbRows = 16;                              // rows of 32 tokens per warp and pass
constexpr int kDbPass = kDbThreads * kDbRows;            // tokens per pass

__device__ __forceinline__ int warp_incl_max(int v)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if ((threadIdx.x & 31) >= o) v = max(v, u);
    }
    return v;
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

__device__ __forceinline__ int query_tile_work(int t, const int32_t *tile_lo, const DbWindow &w)
{
    return max(0, min(t, w.kvhi_t) - max(tile_lo[t] / kTileN, w.kvlo_t) + 1);
}

template <Unit kUnit>
__device__ __forceinline__ int unit_work(int u, const int32_t *src, const DbWindow &w)
{
    if (kUnit == Unit::kKeyTiles) return static_cast<int>((src[u] + kTileM - 1) / kTileM) - u;
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

struct DbArgs {
    const int32_t *pos;
    int64_t N;
    int T;
    int32_t *doc_start, *tile_lo, *q_order, *kv_qend, *kv_order, *ghist;
    uint32_t *status;
    int backward, fwd_tile_pairs;
    DbWindow win;
};

__global__ void __launch_bounds__(kDbThreads, 1) docbounds_kernel(const DbArgs a)
{
    // The attention kernel that follows may start its prologue now; it reads
    // nothing this kernel writes before its grid-dependency wait.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ int shist[kOrderSmemWork + 1];
    __shared__ int wtot[kDbWarps];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        a.status[0] = 0u;   // fresh status for this call
        a.status[1] = 0u;   // work counter of the persistent forward kernel
    }

    // ---- 1. doc_start scan and each query tile's first key
    int carry = 0;   // largest index of a 0 id in earlier passes (0 if none)
    for (int64_t base = 0; base < a.N; base += kDbPass) {
        const int64_t wbase = base + static_cast<int64_t>(warp) * (32 * kDbRows) + lane;
        int v[kDbRows];
#pragma unroll
        for (int k = 0; k < kDbRows; ++k) {
            const int64_t j = wbase + 32 * k;
            v[k] = (j < a.N && a.pos[j] == 0) ? static_cast<int>(j) : 0;
        }
        int run = 0;   // maximum over this warp's earlier rows
#pragma unroll
        for (int k = 0; k < kDbRows; ++k) {
            const int x = max(warp_incl_max(v[k]), run);
            v[k] = x;
            run = __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0) wtot[warp] = run;
        __syncthreads();
        if (warp == 0) wtot[lane] = warp_incl_max(wtot[lane]);
        __syncthreads();
        const int pre = max(carry, warp > 0 ? wtot[warp - 1] : 0);
#pragma unroll
        for (int k = 0; k < kDbRows; ++k) {
            const int64_t j = wbase + 32 * k;
            if (j < a.N) {
                const int ds = max(v[k], pre);
                a.doc_start[j] = ds;
                if ((j & (kTileM - 1)) == 0) a.tile_lo[j / kTileM] = ds;
            }
        }
        carry = max(carry, wtot[kDbWarps - 1]);
        __syncthreads();   // wtot is rewritten by the next pass
    }
    // (the block's global writes above are visible to all its threads after a barrier)
    __syncthreads();

    // ---- 2. backward: last query row of each key tile
    if (a.backward) {
        for (int t = threadIdx.x; t < a.T; t += kDbThreads) a.kv_qend[t] = key_tile_qend(a.N, t, a.doc_start);
        __syncthreads();
    }

    // ---- 3. schedules, heaviest first
    const int qt = a.win.q_tiles;
    if (!a.backward && a.fwd_tile_pairs)
        unit_order<Unit::kQueryPairs>((qt + 1) / 2, a.win, 2 * a.T, a.tile_lo, shist, a.ghist, wtot, a.q_order);
    else
        unit_order<Unit::kQueryTiles>(qt, a.win, a.T, a.tile_lo, shist, a.ghist, wtot, a.q_order);
    if (a.backward)
        unit_order<Unit::kKeyTiles>(a.T, a.win, a.T, a.kv_qend, shist, a.ghist, wtot, a.kv_order);
}

}  // namespace

cudaError_t launch_docbounds(const int32_t *pos, int64_t N, char *ws, const WsLayout &L, bool backward,
                             bool fwd_tile_pairs, const DbWindow &win, cudaStream_t stream)
{
    DbArgs a;
    a.pos = pos;
    a.N = N;
    a.T = static_cast<int>(ceil_div(N, kTileM));
    a.doc_start = reinterpret_cast<int32_t *>(ws + L.doc_start);
    a.tile_lo = reinterpret_cast<int32_t *>(ws + L.tile_lo);
    a.q_order = reinterpret_cast<int32_t *>(ws + L.q_order);
    a.kv_qend = backward ? reinterpret_cast<int32_t *>(ws + L.kv_qend) : nullptr;
    a.kv_order = backward ? reinterpret_cast<int32_t *>(ws + L.kv_order) : nullptr;
    a.ghist = reinterpret_cast<int32_t *>(ws + L.scratch);
    a.status = reinterpret_cast<uint32_t *>(ws + L.status);
    a.backward = backward ? 1 : 0;
    a.fwd_tile_pairs = fwd_tile_pairs ? 1 : 0;
    a.win = win;
    docbounds_kernel<<<1, kDbThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace uly
