// attn_fwd.cu -- causal, document-masked, grouped-KV attention forward for one
// rank's head slice, on the sm_100a tensor cores.
//
// This is the "本地注意力计算" step of Ulysses (page "Hugging Face并行加速：10倍提升
// 超长序列训练效率", section "Ulysses的工作原理"): after the exchange every GPU runs
// ordinary attention over the whole sequence for its own heads, with no further
// communication, because heads are independent. Work stays O(n^2) but memory is
// O(n) by tiling with an online softmax (section "超长序列训练的挑战").
//
// The kernel is persistent: one CTA per SM takes work items from a global
// counter, heaviest first. An item is two 128-row query tiles A and B that
// share every K/V tile load. When the query heads of a KV group come in pairs
// (G = Hl/Hkvl even) they are the same query tile t of heads 2g and 2g+1 of
// one group: identical key ranges, so both tiles run the same steps.
// Otherwise (G odd) they are consecutive tiles 2u and 2u+1 of one head; B
// then has one key tile more than A, and where a document starts inside the
// pair B's range is much shorter than A's.
//   warps 0..3   softmax warpgroup of tile A (thread t owns row t = TMEM lane t)
//   warps 4..7   softmax warpgroup of tile B
//   warp 8       takes the items, decodes them and hands them to the other
//                roles through a two-slot ring in shared memory; TMA producer
//                of Q_A, K_0, Q_B, K_1, ... (K in a KST-stage ring)
//   warp 9       allocates tensor memory; issues every tcgen05.mma (one elected lane)
//   warp 10      TMA producer of the V tiles (VST-stage ring; a V tile is held one
//                step longer than its K tile, so it gets the extra stage)
// Tensor memory (512 columns): S_A at 0, S_B at 128 (fp32 128x128 each; the
// bf16 probabilities P overwrite the first 64 columns of their own S), O_A at
// 256, O_B at 256 + d.
// The issue order ping-pongs the two tiles so that one warpgroup's softmax runs
// while the tensor core works on the other tile:
//     ... PV_A(j-1), S_A(j), PV_B(j-1), S_B(j), PV_A(j), S_A(j+1) ...
// and runs on into the next item without a break: the K/V rings, the barrier
// phases and the tensor memory carry over, the next item's Q tiles load as
// soon as the last S of the current item has read them, and the step at an
// item boundary is itself ping-ponged -- PV_A(last), S_A'(0), PV_B(last),
// S_B'(0) -- so a tile that is done starts its next item without waiting for
// the other tile's last step, and its first S overlaps its epilogue.
// Waits before a .sync.aligned tensor-memory load are warp-uniform.
// S = Q K^T is an SS MMA (both operands K-major in 128B-swizzled shared memory);
// O += P V is a TS MMA (P from tensor memory, V MN-major from its TMA tile).
// The softmax reads its S row, masks only diagonal / document-boundary tiles,
// keeps a running max with lazy rescaling (O and l are rescaled only when the
// max grows by more than 2^8), and writes P = exp2(...) back as bf16. The
// row arithmetic uses the packed fp32x2 FMA / add and the 3-input max; a
// quarter of the exponentials (every fourth column pair) are evaluated on the
// FMA pipe (ex2_poly2) so that the special-function unit is not the limit.
// Key tiles outside [doc_start(first row), last row] of a tile are never
// visited by that tile.
#include "ptx.cuh"
#include "ulysses_internal.cuh"

#include <cuda_bf16.h>
#include <math_constants.h>

namespace uly {

namespace {

constexpr int kFwdThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kVProducerWarp = 10;
constexpr uint32_t kTmemCols = 512;
// One column pair in every kEmuEvery has its exponentials on the FMA pipe:
// the SFU needs 8 cycles per warp instruction, so with only SFU exponentials
// a 128-column row costs 1024 SFU cycles per warp against ~400 issue slots of
// other work; moving part of them to packed polynomials balances the two
// (a quarter measured fastest: 2 % over 3 of 8, 6 % over 4 of 8; spreading
// them one pair in four rather than two adjacent pairs in eight, 0.6-1.3 %).
constexpr int kEmuEvery = 4;
// Register split: launched at 168 per thread (384 x 168 = 64512); the two
// softmax warpgroups take 216, the producer / MMA warpgroup keeps 72:
// 256 x 216 + 128 x 72 = 64512.
constexpr uint32_t kLaunchRegs = 168;
constexpr uint32_t kSoftmaxRegs = 216;
constexpr uint32_t kControlRegs = 72;
static_assert(256 * kSoftmaxRegs + 128 * kControlRegs <= kFwdThreads * kLaunchRegs, "register split");

struct FwdParams {
    const int32_t *doc_start;
    const int32_t *tile_lo;
    const int32_t *q_order;
    __nv_bfloat16 *o;
    int64_t o_row_elems;   // elements between consecutive token rows of O
    int o_head0;
    float *lse;            // [Hl][lse_ld]
    int N, Hl, Hkvl;
    int q_head0, kv_head0;
    // Query window: rows [q_lo, q_end) in query tiles q_tile0 .. q_tile0+T-1;
    // O row i goes to o + (i - q_lo) * o_row_elems, its LSE to lse[h][i - q_lo].
    int q_tile0, T, q_lo, q_end, lse_ld;
    // Key window [kv_lo, kv_hi), key tiles kvlo_t .. kvhi_t (a ring step's
    // chunk of keys; the whole sequence otherwise).
    int kv_lo, kv_hi, kvlo_t, kvhi_t;
    float scale_log2;      // softmax scale * log2(e)
    int pair_heads;        // 1: items pair heads (T x Hl/2 items); 0: items pair tiles (ceil(T/2) x Hl)
    int items;
    uint32_t *status;      // [0] status word, [1] work counter (both zeroed before the launch)
    // 1: each tile's O is staged in its Q buffer (free once the item's last S
    // has run) and written by TMA bulk stores of whole rows; the Q buffer is
    // released to the producer by the epilogue, after the store has read it.
    // 0 (a query window that does not start on a tile): per-thread row stores.
    int o_tma;
    uint64_t wait_limit_ns;
    uint32_t debug_flags;   // bit 0: CTA 0 waits on a barrier nobody arrives on (tests the timeout path)
};

constexpr int kItemInts = 12;   // ints of one FwdItem

// One work item. Head pairs: tile q_order[idx / (Hl/2)] of heads 2g, 2g+1,
// g = idx % (Hl/2). Tile pairs: the pair q_order[idx / Hl] of head idx % Hl.
// A tile's key tiles are those of its rows' documents inside the key window;
// a tile with none (nA or nB == 0) only writes O = 0, LSE = -inf.
struct FwdItem {
    int idx;       // work item index, -1: no more work
    int hA, hB, kvh, tA, tB;
    int hasB;
    int j0;        // first key tile of the union of both tiles' ranges
    int nA;        // key tiles of A: union steps [0, nA)
    int bstart;    // key tiles of B: union steps [bstart, n_union)
    int nB;
    int n_union;
};
static_assert(sizeof(FwdItem) == kItemInts * sizeof(int), "the item ring copies a FwdItem as kItemInts ints");

__device__ __forceinline__ FwdItem decode_item(const FwdParams &p, int idx)
{
    FwdItem it;
    it.idx = idx;
    if (p.pair_heads) {
        const int groups2 = p.Hl >> 1;
        const int t = p.q_order[idx / groups2];
        it.hA = 2 * (idx % groups2);
        it.hB = it.hA + 1;
        it.kvh = it.hA / (p.Hl / p.Hkvl);
        it.tA = it.tB = t;
        it.hasB = 1;
        it.j0 = max(p.tile_lo[t] / kTileN, p.kvlo_t);
        it.nA = it.nB = it.n_union = max(0, min(t, p.kvhi_t) - it.j0 + 1);
        it.bstart = 0;
        return it;
    }
    const int pair = p.q_order[idx / p.Hl];
    it.hA = it.hB = idx % p.Hl;
    it.kvh = it.hA / (p.Hl / p.Hkvl);
    it.tA = p.q_tile0 + 2 * pair;
    it.tB = it.tA + 1;
    it.hasB = it.tB < p.q_tile0 + p.T ? 1 : 0;
    const int loA = max(p.tile_lo[it.tA] / kTileN, p.kvlo_t);
    const int hiA = min(it.tA, p.kvhi_t);
    it.nA = max(0, hiA - loA + 1);
    const int loB = it.hasB ? max(p.tile_lo[it.tB] / kTileN, p.kvlo_t) : 0;
    const int hiB = min(it.tB, p.kvhi_t);
    it.nB = it.hasB ? max(0, hiB - loB + 1) : 0;
    // B's range starts no earlier than A's and ends no earlier, with no gap
    if (it.nA > 0) {
        it.j0 = loA;
        it.bstart = it.nB > 0 ? loB - loA : 0;
        it.n_union = it.nB > 0 ? hiB - loA + 1 : it.nA;
    } else {
        it.j0 = it.nB > 0 ? loB : 0;
        it.bstart = 0;
        it.n_union = it.nB;
    }
    return it;
}

template <int D>
struct FwdCfg {
    static constexpr int SW = (D * 2 >= 128) ? 128 : D * 2;   // swizzle span in bytes (row of one atom)
    static constexpr int AW = SW / 2;                         // bf16 elements per atom row
    static constexpr int NA = D / AW;                         // atoms along d
    static constexpr int ATOM_BYTES = kTileM * SW;            // one 128-row atom block
    static constexpr int TILE_BYTES = kTileM * D * 2;         // a Q, K or V tile
    static constexpr int KST = (D == 128) ? 2 : 4;            // K pipeline stages
    static constexpr int VST = (D == 128) ? 3 : 4;            // V pipeline stages
    static constexpr uint32_t SWZ = (SW == 128) ? kSwizzle128 : kSwizzle64;
    static constexpr int OFF_Q = 0;                           // Q_A, Q_B
    static constexpr int OFF_K = 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + KST * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + VST * TILE_BYTES;
    static constexpr int NBAR = 2 + 2 + 2 * KST + 2 * VST + 2 + 2 + 2 + 2 + 2 + 1 + 1 + 2;
    static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 2 * kItemInts * 4 + 1024;   // + item ring, alignment slack
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(kTileM, kTileN, false, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(kTileM, D, false, true);
    // tensor-memory columns: S / P of tile x at ts_col(x), O of tile x at to_col(x)
    __host__ __device__ static constexpr uint32_t ts_col(int x) { return static_cast<uint32_t>(x) * 128u; }
    __host__ __device__ static constexpr uint32_t to_col(int x) { return 256u + static_cast<uint32_t>(x * D); }
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const FwdParams p)
{
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars;                 // [2]
    uint64_t *q_empty = bars + 2;            // [2] Q_x is free: its item's last S has read it (or,
                                             // with o_tma, its epilogue's store has read the O staged there)
    uint64_t *k_full = bars + 4;             // [KST]
    uint64_t *k_empty = k_full + C::KST;
    uint64_t *v_full = k_empty + C::KST;     // [VST]
    uint64_t *v_empty = v_full + C::VST;
    uint64_t *s_full = v_empty + C::VST;     // [2] per tile
    uint64_t *p_full = s_full + 2;           // [2] per tile
    uint64_t *o_done = p_full + 2;           // [2] per tile
    uint64_t *item_full = o_done + 2;        // [2] item ring slot written
    uint64_t *item_empty = item_full + 2;    // [2] item ring slot read by every consumer
    uint64_t *mma_done = item_empty + 2;
    uint64_t *never = mma_done + 1;          // never arrived on (timeout test only)
    uint64_t *o_staged = never + 1;          // [2] every row of tile x's O is staged (o_tma)
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(o_staged + 2);
    // two decoded FwdItems, written by the producer, read by every other role
    volatile int *item_ring = reinterpret_cast<volatile int *>(tmem_holder + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // consumers of every ring slot: MMA warp (1), V producer (1), both softmax warpgroups (256)
    constexpr uint32_t kItemConsumers = 2 + 256;

    if (threadIdx.x == 0) {
        for (int x = 0; x < 2; ++x) {
            mbar_init(&q_full[x], 1);
            mbar_init(&q_empty[x], 1);
            mbar_init(&s_full[x], 1);
            mbar_init(&p_full[x], 128);
            mbar_init(&o_done[x], 1);
            mbar_init(&item_full[x], 1);
            mbar_init(&item_empty[x], kItemConsumers);
            mbar_init(&o_staged[x], 128);
        }
        for (int s = 0; s < C::KST; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < C::VST; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(mma_done, 1);
        mbar_init(never, 1);
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;
    // Launched as a programmatic dependent of the doc-bounds kernel: everything
    // above overlapped it; the schedule, the document starts and the status
    // word it writes are read only from here on.
    griddep_wait();

    // A CTA that starts after another one has timed out skips its work.
    WaitCtx wc{p.wait_limit_ns, p.status, *reinterpret_cast<volatile uint32_t *>(p.status) != 0u};

    // Consumer side of the item ring: the n-th item of this CTA, decoded by the
    // producer (idx -1: no more work).
    auto take_item = [&](int n, bool warp_wide) -> FwdItem {
        const int slot = n & 1;
        const bool ok = warp_wide ? mbar_wait_warp(&item_full[slot], (n >> 1) & 1, wc)
                                  : mbar_wait(&item_full[slot], (n >> 1) & 1, wc);
        FwdItem w;
        int *wi = reinterpret_cast<int *>(&w);
#pragma unroll
        for (int f = 0; f < kItemInts; ++f) wi[f] = item_ring[slot * kItemInts + f];
        if (!ok) w.idx = -1;
        return w;
    };

    if (warp >= 8) {
    setmaxnreg_dec<kControlRegs>();
    if (warp == kProducerWarp) {
        // ================================================================ items, Q and K producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            int kcount = 0;                  // K tiles loaded so far (ring position)
            int qcount[2] = {0, 0};          // Q_x tiles loaded so far
            int last_use[C::KST];
#pragma unroll
            for (int s = 0; s < C::KST; ++s) last_use[s] = -1;
            for (int n = 0;; ++n) {
                const int slot = n & 1;
                if (n >= 2 && !mbar_wait(&item_empty[slot], ((n >> 1) - 1) & 1, wc)) break;
                const int idx = static_cast<int>(atomicAdd(p.status + 1, 1u));
                FwdItem w{};
                w.idx = -1;
                if (idx < p.items) w = decode_item(p, idx);
                const int *wi = reinterpret_cast<const int *>(&w);
#pragma unroll
                for (int f = 0; f < kItemInts; ++f) item_ring[slot * kItemInts + f] = wi[f];
                mbar_arrive(&item_full[slot]);   // release: the fields are visible to every waiter
                if (w.idx < 0) break;
                // The item is known about two key steps before the current one ends,
                // but its Q tiles and first K/V tiles can only be loaded into shared
                // memory as the current item frees them: bring them into L2 now,
                // so that those loads do not wait for HBM at the item boundary.
#pragma unroll
                for (int a = 0; a < C::NA; ++a) {
                    if (w.nA > 0) tma_prefetch_3d(&tmQ, a * C::AW, p.q_head0 + w.hA, w.tA * kTileM);
                    if (w.hasB && w.nB > 0) tma_prefetch_3d(&tmQ, a * C::AW, p.q_head0 + w.hB, w.tB * kTileM);
                    for (int j = 0; j < 2 && j < w.n_union; ++j) {
                        tma_prefetch_3d(&tmK, a * C::AW, p.kv_head0 + w.kvh, (w.j0 + j) * kTileN);
                        tma_prefetch_3d(&tmV, a * C::AW, p.kv_head0 + w.kvh, (w.j0 + j) * kTileN);
                    }
                }
                // Q_A, K_0, Q_B, K_1, K_2, ...: the next item's first S (tile A) needs
                // only Q_A and K_0, and Q_B's buffer is freed last (by B's final S).
                auto load_q = [&](int x) -> bool {
                    if (qcount[x] > 0 && !mbar_wait(&q_empty[x], (qcount[x] - 1) & 1, wc)) return false;
                    mbar_arrive_expect_tx(&q_full[x], C::TILE_BYTES);
#pragma unroll
                    for (int a = 0; a < C::NA; ++a)
                        tma_load_3d(sQ + x * C::TILE_BYTES + a * C::ATOM_BYTES, &tmQ, &q_full[x], a * C::AW,
                                    p.q_head0 + (x == 0 ? w.hA : w.hB), (x == 0 ? w.tA : w.tB) * kTileM);
                    ++qcount[x];
                    return true;
                };
                bool ok = w.nA > 0 ? load_q(0) : true;
                for (int j = 0; ok && j < w.n_union; ++j, ++kcount) {
                    const int s = kcount % C::KST, u = kcount / C::KST;
                    if (u > 0 && !mbar_wait(&k_empty[s], (u - 1) & 1, wc)) { ok = false; break; }
                    mbar_arrive_expect_tx(&k_full[s], C::TILE_BYTES);
#pragma unroll
                    for (int a = 0; a < C::NA; ++a)
                        tma_load_3d(sK + s * C::TILE_BYTES + a * C::ATOM_BYTES, &tmK, &k_full[s], a * C::AW,
                                    p.kv_head0 + w.kvh, (w.j0 + j) * kTileN);
                    last_use[s] = u;
                    if (j == 0 && w.hasB && w.nB > 0 && !load_q(1)) { ok = false; break; }
                }
                if (!ok) break;
            }
            // Never leave the CTA with bulk copies still landing in its shared memory.
            WaitCtx drain{p.wait_limit_ns, p.status, false};
            for (int x = 0; x < 2; ++x)
                if (qcount[x] > 0) mbar_wait(&q_full[x], (qcount[x] - 1) & 1, drain);
            for (int s = 0; s < C::KST; ++s)
                if (last_use[s] >= 0) mbar_wait(&k_full[s], last_use[s] & 1, drain);
        }
    } else if (warp == kVProducerWarp) {
        // ================================================================ V producer
        if (lane == 0) {
            prefetch_tmap(&tmV);
            int vcount = 0;
            int last_use[C::VST];
#pragma unroll
            for (int s = 0; s < C::VST; ++s) last_use[s] = -1;
            for (int n = 0;; ++n) {
                const FwdItem w = take_item(n, false);
                mbar_arrive(&item_empty[n & 1]);
                if (w.idx < 0) break;
                bool ok = true;
                for (int j = 0; j < w.n_union; ++j, ++vcount) {
                    const int s = vcount % C::VST, u = vcount / C::VST;
                    if (u > 0 && !mbar_wait(&v_empty[s], (u - 1) & 1, wc)) { ok = false; break; }
                    mbar_arrive_expect_tx(&v_full[s], C::TILE_BYTES);
#pragma unroll
                    for (int a = 0; a < C::NA; ++a)
                        tma_load_3d(sV + s * C::TILE_BYTES + a * C::ATOM_BYTES, &tmV, &v_full[s], a * C::AW,
                                    p.kv_head0 + w.kvh, (w.j0 + j) * kTileN);
                    last_use[s] = u;
                }
                if (!ok) break;
            }
            WaitCtx drain{p.wait_limit_ns, p.status, false};
            for (int s = 0; s < C::VST; ++s)
                if (last_use[s] >= 0) mbar_wait(&v_full[s], last_use[s] & 1, drain);
        }
    } else if (warp == kMmaWarp) {
        // ================================================================ MMA issuer
        // The whole warp runs the loop; one elected lane issues each tcgen05
        // instruction (faster than issuing from a one-lane branch).
        const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
        // S_x = Q_x K^T, K-major operands, 16-element K steps
        // (descriptor of step kk = descriptor of step 0 + the step's byte offset >> 4)
        auto issue_s = [&](int x, int s) {
            constexpr int steps = C::SW / 32;
            const uint64_t ad = smem_desc(aQ + x * C::TILE_BYTES, 16, 8 * C::SW, C::SWZ);
            const uint64_t bd = smem_desc(aK + s * C::TILE_BYTES, 16, 8 * C::SW, C::SWZ);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const uint32_t koff = ((kk / steps) * C::ATOM_BYTES + (kk % steps) * 32) >> 4;
                umma_ss_elect_off(tbase + C::ts_col(x), ad, koff, bd, koff, C::IDESC_QK, kk > 0 ? 1u : 0u);
            }
            umma_commit_elect(&s_full[x]);
        };
        // O_x += P_x V, P from tensor memory (8 columns per 16 keys)
        auto issue_pv = [&](int x, int s, bool first) {
            const uint64_t bd = smem_desc(aV + s * C::TILE_BYTES, C::ATOM_BYTES, 8 * C::SW, C::SWZ);
#pragma unroll
            for (int kk = 0; kk < kTileN / 16; ++kk)
                umma_ts_elect_off(tbase + C::to_col(x), tbase + C::ts_col(x) + kk * 8, bd, (kk * 16 * C::SW) >> 4,
                                  C::IDESC_PV, (!first || kk > 0) ? 1u : 0u);
        };
        int kbase = 0, vbase = 0;            // K / V ring positions of the current item's first tile
        int pbase[2] = {0, 0};               // P tiles of each tile slot consumed by earlier items
        int qcount[2] = {0, 0};
        bool ok = true;
        FwdItem cur{};
        bool have_cur = false;
        for (int n = 0; ok; ++n) {
            // ---- boundary step: the last PVs of the current item, interleaved per
            // tile with the first S of item n, so that a tile that has finished
            // starts its next item without waiting for the other tile's last step:
            //     PV_A(cur, last), S_A(next, 0), PV_B(cur, last), S_B(next, 0)
            const FwdItem nxt = take_item(n, true);
            if (lane == 0) mbar_arrive(&item_empty[n & 1]);
            __syncwarp();
            const bool have_nxt = nxt.idx >= 0;
            const int nu = have_cur ? cur.n_union : 0;
            const int gv = vbase + nu - 1;                     // V position of the current item's last PV
            const int sp = (gv + C::VST) % C::VST, up = gv / C::VST;
            const int gk = kbase + nu;                         // K position of the next item's first S
            const int s = gk % C::KST, u = gk / C::KST;
            // A tile's last PV falls on the boundary when its key range ends the
            // union; B's always does (its range ends at its own diagonal tile).
            const bool pvA = have_cur && cur.nA > 0 && cur.nA == nu;
            const bool pvB = have_cur && cur.hasB && cur.nB > 0;
            const bool sA = have_nxt && nxt.nA > 0;
            const bool sB = have_nxt && nxt.hasB && nxt.nB > 0 && nxt.bstart == 0;
            // With O staged in the Q buffers (o_tma) the next item's Q tiles arrive only
            // after this item's epilogues, so both last PVs go first.
            const bool late_q = p.o_tma != 0;
            if (pvA || pvB) ok = mbar_wait_warp(&v_full[sp], up & 1, wc);
            if (ok && sA && !late_q) ok = mbar_wait_warp(&k_full[s], u & 1, wc);
            if (ok && pvA) {
                ok = mbar_wait_warp(&p_full[0], (pbase[0] + cur.nA - 1) & 1, wc);
                if (ok) {
                    tc_fence_after();
                    issue_pv(0, sp, cur.nA == 1);
                    umma_commit_elect(&o_done[0]);
                }
            }
            if (ok && sA && !late_q) {
                ok = mbar_wait_warp(&q_full[0], qcount[0] & 1, wc);
                ++qcount[0];
                if (ok) {
                    tc_fence_after();
                    issue_s(0, s);
                    if (nxt.nA == 1) umma_commit_elect(&q_empty[0]);
                }
            }
            if (ok && pvB) {
                ok = mbar_wait_warp(&p_full[1], (pbase[1] + cur.nB - 1) & 1, wc);
                if (ok) {
                    tc_fence_after();
                    issue_pv(1, sp, cur.nB == 1);
                    umma_commit_elect(&o_done[1]);
                }
            }
            if (ok && sA && late_q) {
                ok = mbar_wait_warp(&k_full[s], u & 1, wc);
                if (ok) ok = mbar_wait_warp(&q_full[0], qcount[0] & 1, wc);
                ++qcount[0];
                if (ok) {
                    tc_fence_after();
                    issue_s(0, s);
                }
            }
            if (ok && have_nxt && nxt.hasB && nxt.nB > 0) {
                ok = mbar_wait_warp(&q_full[1], qcount[1] & 1, wc);
                ++qcount[1];
            }
            if (ok && sB) {
                tc_fence_after();
                issue_s(1, s);
                if (!late_q && nxt.nB == 1) umma_commit_elect(&q_empty[1]);
            }
            if (!ok) break;
            if (sA) umma_commit_elect(&k_empty[s]);
            if (pvA || pvB) umma_commit_elect(&v_empty[sp]);
            if (have_cur) {
                kbase += cur.n_union;
                vbase += cur.n_union;
                pbase[0] += cur.nA;
                pbase[1] += cur.nB;
            }
            if (!have_nxt) break;
            cur = nxt;
            have_cur = true;
            // ---- steps 1 .. n_union-1 of the item: PV_A(j-1), S_A(j), PV_B(j-1), S_B(j)
            for (int j = 1; ok && j < cur.n_union; ++j) {
                const int gkj = kbase + j, gvj = vbase + j - 1;   // ring positions of K_j and V_(j-1)
                const int sj = gkj % C::KST, uj = gkj / C::KST;
                const int spj = gvj % C::VST, upj = gvj / C::VST;
                const bool pvAj = j - 1 < cur.nA;
                const bool sAj = j < cur.nA;
                const int jb = j - cur.bstart;
                const bool pvBj = cur.hasB && jb - 1 >= 0 && jb - 1 < cur.nB;
                const bool sBj = cur.hasB && jb >= 0 && jb < cur.nB;
                if ((pvAj || pvBj) && !mbar_wait_warp(&v_full[spj], upj & 1, wc)) { ok = false; break; }
                if ((sAj || sBj) && !mbar_wait_warp(&k_full[sj], uj & 1, wc)) { ok = false; break; }
                // tile A
                if (pvAj) {
                    if (!mbar_wait_warp(&p_full[0], (pbase[0] + j - 1) & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv(0, spj, j - 1 == 0);
                    if (j - 1 == cur.nA - 1) umma_commit_elect(&o_done[0]);
                }
                if (sAj) {
                    tc_fence_after();
                    issue_s(0, sj);
                    if (!p.o_tma && j == cur.nA - 1) umma_commit_elect(&q_empty[0]);
                }
                // tile B
                if (pvBj) {
                    if (!mbar_wait_warp(&p_full[1], (pbase[1] + jb - 1) & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv(1, spj, jb - 1 == 0);
                    if (jb - 1 == cur.nB - 1) umma_commit_elect(&o_done[1]);
                }
                if (sBj) {
                    tc_fence_after();
                    issue_s(1, sj);
                    if (!p.o_tma && jb == cur.nB - 1) umma_commit_elect(&q_empty[1]);
                }
                if (sAj || sBj) umma_commit_elect(&k_empty[sj]);
                if (pvAj || pvBj) umma_commit_elect(&v_empty[spj]);
            }
        }
        umma_commit_elect(mma_done);
        WaitCtx drain{p.wait_limit_ns, p.status, false};
        mbar_wait(mma_done, 0, drain);
    }
    } else {
        setmaxnreg_inc<kSoftmaxRegs>();
        // ================================================================ softmax warpgroups
        const int x = warp >> 2;                                   // 0: tile A, 1: tile B
        const int r = threadIdx.x & 127;                           // row within the tile == TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tbase + C::ts_col(x) + lane_off;
        const uint32_t tO = tbase + C::to_col(x) + lane_off;
        const float sl2 = p.scale_log2;
        int sbase = 0;      // S tiles of this slot consumed by earlier items
        int ocount = 0;     // items finished by this slot
        int scount = 0;     // O tiles of this slot staged for a TMA store
        bool ok = true;
        if ((p.debug_flags & 1u) && blockIdx.x == 0 && x == 0) ok = mbar_wait_warp(never, 0, wc);   // runs out
        for (int n = 0; ok; ++n) {
            const FwdItem w = take_item(n, false);
            mbar_arrive(&item_empty[n & 1]);
            if (w.idx < 0) break;
            const int n_it = x == 0 ? w.nA : w.nB;
            const int hx = x == 0 ? w.hA : w.hB;
            const int i = (x == 0 ? w.tA : w.tB) * kTileM + r;
            const bool valid = i >= p.q_lo && i < p.q_end && (x == 0 || w.hasB);
            if (n_it == 0) {
                // no key of the window for this tile: O = 0, LSE = -inf
                if (valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(p.o + static_cast<int64_t>(i - p.q_lo) * p.o_row_elems +
                                                           static_cast<int64_t>(p.o_head0 + hx) * D);
#pragma unroll
                    for (int e = 0; e < D / 8; ++e) dst[e] = make_uint4(0u, 0u, 0u, 0u);
                    p.lse[static_cast<int64_t>(hx) * p.lse_ld + (i - p.q_lo)] = -CUDART_INF_F;
                }
                continue;
            }
            const int first_union = x == 0 ? 0 : w.bstart;
            // keys this row may see: its document's, up to itself, inside the key window
            const int lo = valid ? max(p.doc_start[i], p.kv_lo) : i;
            const int hi = min(i, p.kv_hi - 1);
            float ms = -CUDART_INF_F;   // exponent offset in use (scaled log2 units)
            float l = 0.f;
            for (int it = 0; it < n_it; ++it) {
                // warp-uniform wait: the tcgen05.ld below needs the whole warp converged
                if (!mbar_wait_warp(&s_full[x], (sbase + it) & 1, wc)) { ok = false; break; }
                tc_fence_after();
                float s[kTileN];
                {
                    uint32_t raw0[64], raw1[64];
                    tmem_ld64(tS, raw0);
                    tmem_ld64(tS + 64, raw1);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        s[e] = __uint_as_float(raw0[e]);
                        s[64 + e] = __uint_as_float(raw1[e]);
                    }
                }
                const int c0 = (w.j0 + first_union + it) * kTileN;
                // This row may see key columns [cl, ch) of the tile. A row that sees
                // none (its document starts in a later key tile: a tile straddling
                // a document boundary) is zeroed through its exponent offset below;
                // only rows cut inside the tile need a per-column mask.
                const int cl = lo - c0, ch = hi - c0 + 1;
                const bool row_out = cl >= kTileN;
                if (__any_sync(0xffffffffu, !row_out && (cl > 0 || ch < kTileN))) {
                    // 32-column chunks valid for the whole warp are skipped; the
                    // others select column by column, branch-free.
#pragma unroll
                    for (int k = 0; k < kTileN / 32; ++k) {
                        if (!__all_sync(0xffffffffu, cl <= 32 * k && ch >= 32 * k + 32)) {
#pragma unroll
                            for (int e = 0; e < 32; ++e) {
                                const int c = 32 * k + e;
                                s[c] = (c >= cl && c < ch) ? s[c] : -CUDART_INF_F;
                            }
                        }
                    }
                }
                // row max: 4 independent chains of 3-input max, column groups of 8
                static_assert(kTileN % 8 == 0, "row max works on groups of 8 columns");
                float mx[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) mx[e] = fmaxf(s[e], s[4 + e]);
#pragma unroll
                for (int c = 8; c < kTileN; c += 8)
#pragma unroll
                    for (int e = 0; e < 4; ++e) mx[e] = max3f(mx[e], s[c + e], s[c + 4 + e]);
                const float mt = row_out ? -CUDART_INF_F : max3f(mx[0], mx[1], fmaxf(mx[2], mx[3]));
                const float mt_s = mt * sl2;
                const bool resc = mt_s > ms + 8.0f;
                float alpha = 1.f;
                if (resc) {
                    alpha = ex2_approx(ms - mt_s);
                    ms = mt_s;
                    l *= alpha;
                }
                if (it > 0 && __any_sync(0xffffffffu, resc)) {
                    // O holds the previous tiles' sum in the old units. PV_x(it-1)
                    // was issued before S_x(it), so it has completed.
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t raw[32];
                        tmem_ld32(tO + c * 32, raw);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
                        tmem_st32(tO + c * 32, raw);
                    }
                }
                // offset +inf turns every exponent of an all-masked row into exp2(-inf)
                const float moff = row_out ? CUDART_INF_F : ((ms == -CUDART_INF_F) ? 0.f : ms);
                // P = exp2(s * scale*log2(e) - offset): the argument two columns at a
                // time (packed FMA), the exponential on the SFU, the row sum two
                // columns at a time (packed add, 4 independent accumulator pairs).
                float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                uint32_t pk[64];
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    float x0, x1;
                    fma2_bcast(x0, x1, s[2 * e], s[2 * e + 1], sl2, -moff);
                    // one column pair in kEmuEvery takes the FMA-pipe exponential, the rest the SFU
                    float e0, e1;
                    if (e % kEmuEvery == 0) {
                        ex2_poly2(e0, e1, x0, x1);
                    } else {
                        e0 = ex2_approx(x0);
                        e1 = ex2_approx(x1);
                    }
                    add2_acc(ls[2 * (e & 3)], ls[2 * (e & 3) + 1], e0, e1);
                    pk[e] = pack_bf16x2(e0, e1);
                }
                tmem_st64(tS, pk);   // P overwrites the first 64 columns of S
                l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&p_full[x]);
            }
            sbase += n_it;
            // ---- epilogue: O / l -> bf16, LSE. The next item's first PV into O_x
            // waits for this slot's next P, which comes after these reads.
            if (!ok || !mbar_wait_warp(&o_done[x], ocount & 1, wc)) { ok = false; break; }
            ++ocount;
            tc_fence_after();
            // A row that saw no key (possible only with a key window) never raised its
            // running max above -inf: O = 0, LSE = -inf. (Its l need not be 0: the
            // FMA-pipe exponential gives 2^-125 rather than 0 for masked columns.)
            const bool seen = ms != -CUDART_INF_F;
            const float inv_l = seen ? 1.f / l : 0.f;
            __nv_bfloat16 *orow = p.o + static_cast<int64_t>(i - p.q_lo) * p.o_row_elems +
                                  static_cast<int64_t>(p.o_head0 + hx) * D;
            // the whole O row in one round trip (up to two x64 loads, one wait)
            uint32_t orw[D];
            if constexpr (D >= 64) {
#pragma unroll
                for (int c = 0; c < D / 64; ++c)
                    tmem_ld64(tO + c * 64, *reinterpret_cast<uint32_t(*)[64]>(orw + c * 64));
            } else {
                tmem_ld32(tO, *reinterpret_cast<uint32_t(*)[32]>(orw));
            }
            tmem_ld_wait();
            if (p.o_tma) {
                // Stage the bf16 row in this tile's Q buffer in the TMA box layout (atoms of
                // AW columns x 128 rows, 16-byte chunks swizzled by the row), then one thread
                // stores the tile with whole-row writes and hands the buffer back.
                uint8_t *stage = sQ + x * C::TILE_BYTES;
                constexpr int kChunks = C::SW / 16;   // 16-byte chunks per row of an atom
                const int swz = C::SW == 128 ? (r & 7) : ((r >> 1) & 3);
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t wv[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        wv[e] = pack_bf16x2(__uint_as_float(orw[c * 32 + 2 * e]) * inv_l,
                                            __uint_as_float(orw[c * 32 + 2 * e + 1]) * inv_l);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int col = c * 32 + e * 8;                 // first of these 8 columns
                        const int atom = col / C::AW, chunk = (col % C::AW) / 8;
                        uint4 *dst = reinterpret_cast<uint4 *>(stage + atom * C::ATOM_BYTES + r * C::SW +
                                                               ((chunk ^ swz) % kChunks) * 16);
                        *dst = make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
                    }
                }
                fence_async_smem();             // the staged row is visible to the TMA store
                mbar_arrive(&o_staged[x]);
                if (r == 0) {
                    // bounded: if a thread of the tile gave up on a wait, this gives up too
                    if (mbar_wait(&o_staged[x], scount & 1, wc)) {
                        const int row0 = (x == 0 ? w.tA : w.tB) * kTileM - p.q_lo;
#pragma unroll
                        for (int a = 0; a < C::NA; ++a)
                            tma_store_3d(&tmO, stage + a * C::ATOM_BYTES, a * C::AW, p.o_head0 + hx, row0);
                        bulk_commit_group();
                        bulk_wait_read_all();
                        mbar_arrive(&q_empty[x]);   // the producer may load the next Q_x
                    }
                }
                ++scount;
            } else {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t wv[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        wv[e] = pack_bf16x2(__uint_as_float(orw[c * 32 + 2 * e]) * inv_l,
                                            __uint_as_float(orw[c * 32 + 2 * e + 1]) * inv_l);
                    if (valid) {
                        uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            dst[e] = make_uint4(wv[4 * e], wv[4 * e + 1], wv[4 * e + 2], wv[4 * e + 3]);
                    }
                }
            }
            if (valid)
                p.lse[static_cast<int64_t>(hx) * p.lse_ld + (i - p.q_lo)] =
                    seen ? (ms + __log2f(l)) * 0.69314718055994530942f : -CUDART_INF_F;
            tc_fence_before();
        }
    }

    // the softmax threads that issued bulk stores see them complete before the CTA exits
    if (warp < 8 && (threadIdx.x & 127) == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kMmaWarp) tmem_dealloc(tbase, kTmemCols);
}

template <int D>
cudaError_t launch_fwd_d(const FwdLaunch &a, cudaStream_t stream)
{
    using C = FwdCfg<D>;
    static_assert(C::SMEM_BYTES <= 232448, "shared memory budget");
    alignas(64) CUtensorMap tq, tk, tv, to;
    const int box = C::AW;
    if (!encode_tmap_3d(&tq, a.q, D, a.Hq_total, a.N, int64_t(D) * 2, int64_t(a.Hq_total) * D * 2, box, kTileM,
                        C::SW) ||
        !encode_tmap_3d(&tk, a.k, D, a.Hkv_total, a.N, int64_t(D) * 2, int64_t(a.Hkv_total) * D * 2, box, kTileN,
                        C::SW) ||
        !encode_tmap_3d(&tv, a.v, D, a.Hkv_total, a.N, int64_t(D) * 2, int64_t(a.Hkv_total) * D * 2, box, kTileN,
                        C::SW))
        return cudaErrorInvalidValue;
    // O through TMA stores when the query window starts on a tile (coordinates
    // of a store must not be negative): the map's rows are the window's
    const bool o_tma = (a.q_lo % kTileM) == 0;
    if (o_tma && !encode_tmap_3d(&to, a.o, D, a.Ho_total, a.q_hi - a.q_lo, int64_t(D) * 2,
                                 int64_t(a.Ho_total) * D * 2, box, kTileM, C::SW))
        return cudaErrorInvalidValue;
    if (!o_tma) to = tq;   // not read
    FwdParams p;
    p.doc_start = reinterpret_cast<const int32_t *>(a.ws + a.L.doc_start);
    p.tile_lo = reinterpret_cast<const int32_t *>(a.ws + a.L.tile_lo);
    p.q_order = reinterpret_cast<const int32_t *>(a.ws + a.L.q_order);
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.o_row_elems = int64_t(a.Ho_total) * D;
    p.o_head0 = a.o_head0;
    p.lse = a.lse;
    p.N = static_cast<int>(a.N);
    p.q_tile0 = static_cast<int>(a.q_lo / kTileM);
    p.T = static_cast<int>(ceil_div(a.q_hi, kTileM)) - p.q_tile0;
    p.q_lo = static_cast<int>(a.q_lo);
    p.q_end = static_cast<int>(a.q_hi);
    p.lse_ld = static_cast<int>(a.lse_ld);
    p.kv_lo = static_cast<int>(a.kv_lo);
    p.kv_hi = static_cast<int>(a.kv_hi);
    p.kvlo_t = static_cast<int>(a.kv_lo / kTileN);
    p.kvhi_t = a.kv_hi > 0 ? static_cast<int>((a.kv_hi - 1) / kTileN) : -1;
    p.Hl = a.Hl;
    p.Hkvl = a.Hkvl;
    p.q_head0 = a.q_head0;
    p.kv_head0 = a.kv_head0;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.status = reinterpret_cast<uint32_t *>(const_cast<char *>(a.ws) + a.L.status);
    p.pair_heads = fwd_pairs_heads(a.Hl, a.Hkvl) ? 1 : 0;
    const int64_t items = p.pair_heads ? int64_t(p.T) * (a.Hl / 2) : ceil_div(p.T, 2) * a.Hl;
    // the work counter and item indices are 32-bit; check_attn_shapes rejects larger problems
    if (items > INT32_MAX) return cudaErrorInvalidValue;
    p.items = static_cast<int>(items);
    p.wait_limit_ns = a.wait_limit_ns;
    p.debug_flags = a.debug_flags;
    p.o_tma = o_tma ? 1 : 0;
    static bool attr_set[64] = {};
    static int sm_count[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&sm_count[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    // persistent: one CTA per SM (each needs a whole SM's tensor memory)
    const int sms = (dev < 64 && sm_count[dev] > 0) ? sm_count[dev] : 148;
    const int grid = p.items < sms ? p.items : sms;
    // programmatic dependent launch: the prologue (barriers, tensor memory,
    // descriptor prefetch) overlaps the doc-bounds kernel before it
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kFwdThreads);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, attn_fwd_kernel<D>, tq, tk, tv, to, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd(const FwdLaunch &a, cudaStream_t stream)
{
    switch (a.d) {
    case 32: return launch_fwd_d<32>(a, stream);
    case 64: return launch_fwd_d<64>(a, stream);
    case 128: return launch_fwd_d<128>(a, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace uly
