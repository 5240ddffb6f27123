// attn_fwd.cu -- causal, document-masked, grouped-KV attention forward for one
// rank's head slice, on the sm_100a tensor cores.
//
// This is the "本地注意力计算" step of Ulysses (page "Hugging Face并行加速：10倍提升
// 超长序列训练效率", section "Ulysses的工作原理"): after the exchange every GPU runs
// ordinary attention over the whole sequence for its own heads, with no further
// communication, because heads are independent. Work stays O(n^2) but memory is
// O(n) by tiling with an online softmax (section "超长序列训练的挑战").
//
// One CTA computes one 128-row query tile of one head:
//   warp 0      TMA producer: Q once, then K and V tiles into an NST-stage ring
//   warp 1      allocates tensor memory; lane 0 issues every tcgen05.mma
//   warps 4..7  softmax warpgroup: thread t owns query row t (TMEM lane t)
// Tensor memory (512 columns): S double buffer at columns 0 and 128 (fp32
// 128x128), O accumulator at column 256 (fp32 128 x d).
// Per key tile j:  S_j = Q K_j^T (SS MMA, both K-major) -> softmax reads S_j,
// masks diagonal / document-boundary tiles only, updates the running max with
// lazy rescaling (O and l are rescaled only when the max grows by more than
// 2^8), writes P_j = exp2(...) as bf16 into a 128B-swizzled shared buffer ->
// O += P_j V_j (SS MMA, V read MN-major straight from its TMA tile).
// Key tiles outside [doc_start(first row), last row] are never visited.
#include "ptx.cuh"
#include "ulysses_internal.cuh"

#include <cuda_bf16.h>
#include <math_constants.h>

namespace uly {

namespace {

constexpr int kFwdThreads = 256;
constexpr int kSoftmaxWarp0 = 4;   // first warp of the softmax warpgroup
constexpr uint32_t kTmemCols = 512;

struct FwdParams {
    const int32_t *doc_start;
    const int32_t *tile_lo;
    const int32_t *q_order;
    __nv_bfloat16 *o;
    int64_t o_row_elems;   // elements between consecutive token rows of O
    int o_head0;
    float *lse;
    int N, Hl, Hkvl;
    int q_head0, kv_head0;
    float scale_log2;      // softmax scale * log2(e)
    uint32_t *status;
    uint64_t wait_limit_ns;
};

template <int D>
struct FwdCfg {
    static constexpr int SW = (D * 2 >= 128) ? 128 : D * 2;   // swizzle span in bytes (row of one atom)
    static constexpr int AW = SW / 2;                         // bf16 elements per atom row
    static constexpr int NA = D / AW;                         // atoms along d
    static constexpr int ATOM_BYTES = kTileM * SW;            // one 128-row atom block
    static constexpr int TILE_BYTES = kTileM * D * 2;         // a Q, K or V tile
    static constexpr int NST = (D == 128) ? 2 : 4;            // K/V pipeline stages
    static constexpr int P_BYTES = kTileM * kTileN * 2;       // one P buffer (two 128B atoms)
    static constexpr uint32_t SWZ = (SW == 128) ? kSwizzle128 : kSwizzle64;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = TILE_BYTES;
    static constexpr int OFF_V = OFF_K + NST * TILE_BYTES;
    static constexpr int OFF_P = OFF_V + NST * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_P + 2 * P_BYTES;
    static constexpr int NBAR = 1 + 4 * NST + 8 + 1;
    static constexpr int SMEM_BYTES = OFF_BAR + NBAR * 8 + 16 + 1024;   // + alignment slack
    static constexpr uint32_t IDESC_QK = idesc_bf16_f32(kTileM, kTileN, false, false);
    static constexpr uint32_t IDESC_PV = idesc_bf16_f32(kTileM, D, false, true);
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p)
{
    using C = FwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    uint8_t *sP = smem + C::OFF_P;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars;
    uint64_t *k_full = bars + 1;
    uint64_t *k_empty = k_full + C::NST;
    uint64_t *v_full = k_empty + C::NST;
    uint64_t *v_empty = v_full + C::NST;
    uint64_t *s_full = v_empty + C::NST;   // [2]
    uint64_t *s_free = s_full + 2;         // [2]
    uint64_t *p_full = s_free + 2;         // [2]
    uint64_t *pv_done = p_full + 2;        // [2]
    uint64_t *mma_done = pv_done + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work item: heaviest query tiles first
    const int item = blockIdx.x;
    const int tile = p.q_order[item / p.Hl];
    const int h = item % p.Hl;
    const int kvh = h / (p.Hl / p.Hkvl);
    const int row0 = tile * kTileM;
    const int kv_t0 = p.tile_lo[tile] / kTileN;
    const int n_kv = tile - kv_t0 + 1;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], 128);
            mbar_init(&p_full[b], 128);
            mbar_init(&pv_done[b], 1);
        }
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;
    const uint32_t tS = tbase;          // + b*128
    const uint32_t tO = tbase + 256;

    // A CTA that starts after another one has timed out skips its work.
    WaitCtx wc{p.wait_limit_ns, p.status, *reinterpret_cast<volatile uint32_t *>(p.status) != 0u};

    if (warp == 0) {
        // ================================================================ producer
        if (lane == 0) {
            prefetch_tmap(&tmQ);
            prefetch_tmap(&tmK);
            prefetch_tmap(&tmV);
            mbar_arrive_expect_tx(q_full, C::TILE_BYTES);
#pragma unroll
            for (int a = 0; a < C::NA; ++a)
                tma_load_3d(sQ + a * C::ATOM_BYTES, &tmQ, q_full, a * C::AW, p.q_head0 + h, row0);
            int last_k_use[C::NST], last_v_use[C::NST];
#pragma unroll
            for (int s = 0; s < C::NST; ++s) last_k_use[s] = last_v_use[s] = -1;
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % C::NST, u = j / C::NST;
                const int key0 = (kv_t0 + j) * kTileN;
                if (u > 0 && !mbar_wait(&k_empty[s], (u - 1) & 1, wc)) break;
                mbar_arrive_expect_tx(&k_full[s], C::TILE_BYTES);
#pragma unroll
                for (int a = 0; a < C::NA; ++a)
                    tma_load_3d(sK + s * C::TILE_BYTES + a * C::ATOM_BYTES, &tmK, &k_full[s], a * C::AW,
                                p.kv_head0 + kvh, key0);
                last_k_use[s] = u;
                if (u > 0 && !mbar_wait(&v_empty[s], (u - 1) & 1, wc)) break;
                mbar_arrive_expect_tx(&v_full[s], C::TILE_BYTES);
#pragma unroll
                for (int a = 0; a < C::NA; ++a)
                    tma_load_3d(sV + s * C::TILE_BYTES + a * C::ATOM_BYTES, &tmV, &v_full[s], a * C::AW,
                                p.kv_head0 + kvh, key0);
                last_v_use[s] = u;
            }
            // Never leave the CTA with bulk copies still landing in its shared memory.
            WaitCtx drain{p.wait_limit_ns, p.status, false};
            mbar_wait(q_full, 0, drain);
            for (int s = 0; s < C::NST; ++s) {
                if (last_k_use[s] >= 0) mbar_wait(&k_full[s], last_k_use[s] & 1, drain);
                if (last_v_use[s] >= 0) mbar_wait(&v_full[s], last_v_use[s] & 1, drain);
            }
        }
    } else if (warp == 1) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
            auto issue_pv = [&](int jj) -> bool {
                const int s = jj % C::NST, u = jj / C::NST, pb = jj & 1;
                if (!mbar_wait(&v_full[s], u & 1, wc)) return false;
                if (!mbar_wait(&p_full[pb], (jj >> 1) & 1, wc)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kTileN / 16; ++kk) {
                    // A = P (128 rows x 128 keys, K-major, two 128B atoms of 64 keys)
                    const uint64_t ad = smem_desc(aP + pb * C::P_BYTES + (kk >> 2) * (kTileM * 128) + (kk & 3) * 32,
                                                  16, 1024, kSwizzle128);
                    // B = V tile (keys x d), d contiguous: MN-major; 16 keys = 16 atom rows
                    const uint64_t bd = smem_desc(aV + s * C::TILE_BYTES + kk * 16 * C::SW, C::ATOM_BYTES,
                                                  8 * C::SW, C::SWZ);
                    umma_ss(tO, ad, bd, C::IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&pv_done[pb]);
                umma_commit(&v_empty[s]);
                return true;
            };
            bool ok = mbar_wait(q_full, 0, wc);
            int j = 0;
            for (; ok && j < n_kv; ++j) {
                const int s = j % C::NST, u = j / C::NST, b = j & 1;
                if (!mbar_wait(&k_full[s], u & 1, wc)) { ok = false; break; }
                if (j >= 2 && !mbar_wait(&s_free[b], ((j >> 1) - 1) & 1, wc)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    constexpr int steps = C::SW / 32;   // 16-element K steps per atom row
                    const uint32_t koff = (kk / steps) * C::ATOM_BYTES + (kk % steps) * 32;
                    const uint64_t ad = smem_desc(aQ + koff, 16, 8 * C::SW, C::SWZ);
                    const uint64_t bd = smem_desc(aK + s * C::TILE_BYTES + koff, 16, 8 * C::SW, C::SWZ);
                    umma_ss(tS + b * 128, ad, bd, C::IDESC_QK, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[b]);
                umma_commit(&k_empty[s]);
                if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
            }
            if (ok) issue_pv(n_kv - 1);
            umma_commit(mma_done);
            WaitCtx drain{p.wait_limit_ns, p.status, false};
            mbar_wait(mma_done, 0, drain);
        }
    } else if (warp >= kSoftmaxWarp0) {
        // ================================================================ softmax warpgroup
        const int r = threadIdx.x - kSoftmaxWarp0 * 32;           // query row within the tile == TMEM lane
        const uint32_t lane_off = static_cast<uint32_t>((warp - kSoftmaxWarp0) * 32) << 16;
        const int i = row0 + r;
        const bool valid = i < p.N;
        const int lo = valid ? p.doc_start[i] : i;
        const int hi = i;
        const float sl2 = p.scale_log2;
        float ms = -CUDART_INF_F;   // running max actually used as exponent offset (scaled log2 units)
        float l = 0.f;
        const uint32_t aP = smem_u32(sP);
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            const int b = j & 1;
            if (!mbar_wait(&s_full[b], (j >> 1) & 1, wc)) { ok = false; break; }
            tc_fence_after();
            float s[kTileN];
            {
                uint32_t raw[32];
#pragma unroll
                for (int c = 0; c < kTileN / 32; ++c) {
                    tmem_ld32(tS + b * 128 + lane_off + c * 32, raw);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(raw[e]);
                }
            }
            tc_fence_before();
            mbar_arrive(&s_free[b]);

            const int c0 = (kv_t0 + j) * kTileN;
            const bool need_mask = (c0 < lo) || (c0 + kTileN - 1 > hi);
            if (__any_sync(0xffffffffu, need_mask)) {
#pragma unroll
                for (int c = 0; c < kTileN; ++c) {
                    const int key = c0 + c;
                    if (key < lo || key > hi) s[c] = -CUDART_INF_F;
                }
            }
            float mt = s[0];
#pragma unroll
            for (int c = 1; c < kTileN; ++c) mt = fmaxf(mt, s[c]);
            const float mt_s = mt * sl2;
            const bool resc = mt_s > ms + 8.0f;
            float alpha = 1.f;
            if (resc) {
                alpha = ex2_approx(ms - mt_s);
                ms = mt_s;
                l *= alpha;
            }
            const float moff = (ms == -CUDART_INF_F) ? 0.f : ms;
            uint32_t pk[kTileN / 2];
            float lsum = 0.f;
#pragma unroll
            for (int c = 0; c < kTileN; c += 2) {
                const float e0 = ex2_approx(fmaf(s[c], sl2, -moff));
                const float e1 = ex2_approx(fmaf(s[c + 1], sl2, -moff));
                lsum += e0 + e1;
                pk[c / 2] = pack_bf16x2(e0, e1);
            }
            l += lsum;
            // P buffer b was last read by PV_{j-2}
            if (j >= 2 && !mbar_wait(&pv_done[b], ((j >> 1) - 1) & 1, wc)) { ok = false; break; }
#pragma unroll
            for (int q = 0; q < kTileN / 8; ++q) {
                const uint32_t addr = aP + b * C::P_BYTES + (q >> 3) * (kTileM * 128) + r * 128 +
                                      (((q & 7) ^ (r & 7)) << 4);
                st_shared_v4(addr, pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
            fence_proxy_async_smem();
            if (j > 0 && __any_sync(0xffffffffu, resc)) {
                // O holds sum_{j' < j} P_j' V_j' in the old units: rescale after PV_{j-1} lands
                if (!mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, wc)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t raw[32];
                    tmem_ld32(tO + lane_off + c * 32, raw);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 32; ++e) raw[e] = __float_as_uint(__uint_as_float(raw[e]) * alpha);
                    tmem_st32(tO + lane_off + c * 32, raw);
                }
                tmem_st_wait();
            }
            tc_fence_before();
            mbar_arrive(&p_full[b]);
        }
        // ---- epilogue: O / l -> bf16, LSE
        const int last = n_kv - 1;
        if (ok && mbar_wait(&pv_done[last & 1], (last >> 1) & 1, wc)) {
            tc_fence_after();
            const float inv_l = 1.f / l;
            __nv_bfloat16 *orow = p.o + static_cast<int64_t>(i) * p.o_row_elems +
                                  static_cast<int64_t>(p.o_head0 + h) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t raw[32];
                tmem_ld32(tO + lane_off + c * 32, raw);
                tmem_ld_wait();
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    w[e] = pack_bf16x2(__uint_as_float(raw[2 * e]) * inv_l, __uint_as_float(raw[2 * e + 1]) * inv_l);
                if (valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
                }
            }
            if (valid) p.lse[static_cast<int64_t>(h) * p.N + i] = (ms + __log2f(l)) * 0.69314718055994530942f;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

template <int D>
cudaError_t launch_fwd_d(const FwdLaunch &a, cudaStream_t stream)
{
    using C = FwdCfg<D>;
    static_assert(C::SMEM_BYTES <= 232448, "shared memory budget");
    alignas(64) CUtensorMap tq, tk, tv;
    const int box = C::AW;
    if (!encode_tmap_3d(&tq, a.q, D, a.Hq_total, a.N, int64_t(D) * 2, int64_t(a.Hq_total) * D * 2, box, kTileM,
                        C::SW) ||
        !encode_tmap_3d(&tk, a.k, D, a.Hkv_total, a.N, int64_t(D) * 2, int64_t(a.Hkv_total) * D * 2, box, kTileN,
                        C::SW) ||
        !encode_tmap_3d(&tv, a.v, D, a.Hkv_total, a.N, int64_t(D) * 2, int64_t(a.Hkv_total) * D * 2, box, kTileN,
                        C::SW))
        return cudaErrorInvalidValue;
    FwdParams p;
    p.doc_start = reinterpret_cast<const int32_t *>(a.ws + a.L.doc_start);
    p.tile_lo = reinterpret_cast<const int32_t *>(a.ws + a.L.tile_lo);
    p.q_order = reinterpret_cast<const int32_t *>(a.ws + a.L.q_order);
    p.o = static_cast<__nv_bfloat16 *>(a.o);
    p.o_row_elems = int64_t(a.Ho_total) * D;
    p.o_head0 = a.o_head0;
    p.lse = a.lse;
    p.N = static_cast<int>(a.N);
    p.Hl = a.Hl;
    p.Hkvl = a.Hkvl;
    p.q_head0 = a.q_head0;
    p.kv_head0 = a.kv_head0;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.status = reinterpret_cast<uint32_t *>(const_cast<char *>(a.ws) + a.L.status);
    p.wait_limit_ns = a.wait_limit_ns;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const int64_t T = ceil_div(a.N, kTileM);
    const int64_t items = T * a.Hl;
    attn_fwd_kernel<D><<<static_cast<unsigned>(items), kFwdThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
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
