// attn_bwd.cu -- attention backward for one rank's head slice on the sm_100a
// tensor cores: the gradients of sum(dO * O) with respect to Q, K and V.
//
// With s_ij = scale q_i.k_j, P_ij = exp(s_ij - LSE_i) (recomputed from the
// forward's logsumexp), D_i = sum_c dO_ic O_ic:
//   dV_j = sum_{h in group} sum_i P_ij dO_i          dP_ij = dO_i . v_j
//   dS_ij = P_ij (dP_ij - D_i)
//   dK_j = scale sum_{h in group} sum_i dS_ij q_i     dQ_i = scale sum_j dS_ij k_j
// over the unmasked pairs (doc_start(i) <= j <= i). Training through the
// attention step of Ulysses needs these (every page speaks of training; the
// attention itself is the "本地注意力计算" step of the page "Hugging Face并行加速：
// 10倍提升超长序列训练效率", section "Ulysses的工作原理").
//
// Three kernels, all deterministic (no atomics):
//  1. prep: D_i and -LSE_i*log2(e) per (head, row) into a 128-padded layout.
//  2. dK/dV: one CTA per (key tile, KV head) loops over the query tiles that
//     see the key tile and, for each, the query heads of the GQA group (heads
//     inner: CTAs of neighbouring key tiles then read the same Q / dO tiles a
//     few steps apart, while they are still in L2):
//       S^T = K Q^T - LSE / scale, dP^T = V dO^T - D
//                                         (SS MMA, M = keys, N = queries)
//       P^T, dS^T -> bf16 into the first 64 columns of S^T / dP^T in TMEM
//       dV += P^T dO, dK += dS^T Q      (TS MMA, dO / Q read MN-major)
//     so the group reduction happens in the accumulator. The per-query terms
//     enter S^T and dP^T as one extra 16-wide K step (a column of ones
//     against each query's term split into hi and lo bf16 halves, exact to
//     about 2^-17 relative; the producer warp builds those operand tiles from
//     4 bytes per query): the element-wise threads then read no per-query
//     values at all (as broadcast shared-memory loads, those took 41 % of the
//     shared-memory load bandwidth).
//     The element-wise step runs in two phases so that the tensor core always
//     has work: once P^T(i) is stored, dV(i) and S^T(i+1) run while dS^T(i)
//     is computed (from the fp32 P^T kept in registers); once dS^T(i) is
//     stored, dK(i) and dP^T(i+1) run while P^T(i+1) is computed.
//  3. dQ: one CTA per (query tile, head) loops over its key tiles:
//       S = Q K^T, dP = dO V^T -> dS (bf16, into S's columns) -> dQ += dS K.
//     S has two buffers (the second in the columns the dQ accumulator leaves
//     free) and runs two key tiles ahead: P is formed while dP is computed,
//     and the next dP, dQ and the S after next run while the element-wise
//     step of the following tile proceeds.
#include "ptx.cuh"
#include "ulysses_internal.cuh"

#include <cuda_bf16.h>
#include <math_constants.h>

namespace uly {

namespace {

// Warps 0..3: producers and the MMA issuer; warps 4..19: the element-wise
// step. Compute warp w handles the 32 TMEM lanes (rows) of quarter w % 4 and
// part (w - 4) / 4 of the 128 columns (kPartCols each): four warps per SM
// sub-partition hide each other's latency in the exponential and product
// phases. Each part writes its bf16 results to the first half of its own
// columns, so no part overwrites columns another still has to read; the TS
// MMAs find K step kk (16 rows, 8 packed columns) at pcol(kk).
// All exponentials go to the SFU here: moving 1 or 2 of every 8 pairs to the
// FMA-pipe polynomial (as the forward does) measured no faster in either
// kernel (the special-function unit is not what bounds them).
constexpr int kParts = 4;
constexpr int kPartCols = kTileN / kParts;
constexpr int kBwdThreads = 128 + kParts * 128;
constexpr int kComputeWarp0 = 4;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

struct BwdParams {
    const int32_t *doc_start;
    const int32_t *tile_lo;
    const int32_t *q_order;
    const int32_t *kv_qend;
    const int32_t *kv_order;
    const float *delta;   // [Hl][Npad]
    const float *lse2;    // [Hl][Npad]: -LSE * log2(e) (-inf on padding rows)
    const uint32_t *qx;   // [Hl][Npad]: -LSE / scale as a hi/lo bf16 pair (the dK/dV kernel's extra K step)
    const uint32_t *dx;   // [Hl][Npad]: -D as a hi/lo bf16 pair
    __nv_bfloat16 *dq, *dk, *dv;
    int N, Npad, T, Hl, Hkvl;
    int Hq_total, Hkv_total;   // heads per token row of the q / kv-side buffers
    int q_head0, kv_head0;     // this slice's first head in those rows
    float scale_log2, scale;
    uint32_t *status;
    uint64_t wait_limit_ns;
    uint32_t debug_flags;   // bit 1: the first dK/dV CTA's element-wise warps wait on a barrier nobody arrives on
};

template <int D>
struct BwdCfg {
    static constexpr int SW = (D * 2 >= 128) ? 128 : D * 2;
    static constexpr int AW = SW / 2;
    static constexpr int NA = D / AW;
    static constexpr int ATOM_BYTES = kTileM * SW;
    static constexpr int TILE_BYTES = kTileM * D * 2;
    static constexpr int NST = 2;
    static constexpr uint32_t SWZ = (SW == 128) ? kSwizzle128 : kSwizzle64;
    static constexpr uint32_t IDESC_SS = idesc_bf16_f32(128, 128, false, false);
    static constexpr uint32_t IDESC_TS = idesc_bf16_f32(128, D, false, true);
    static constexpr uint32_t T_S = 0, T_DP = 128, T_ACC0 = 256, T_ACC1 = 256 + D;
    // dK/dV kernel shared memory: K, V, then NST stages of {Q, dO}, then NST
    // stages of the extra K-step blocks {QB, DB} (128 rows x 16 bf16, 32-byte
    // swizzle), the constant block of ones, then barriers.
    static constexpr int XB_BYTES = kTileM * kXStepBytes;
    static constexpr int KV_OFF_K = 0;
    static constexpr int KV_OFF_V = TILE_BYTES;
    static constexpr int KV_OFF_Q = 2 * TILE_BYTES;
    static constexpr int KV_OFF_DO = KV_OFF_Q + NST * TILE_BYTES;
    static constexpr int KV_OFF_QB = KV_OFF_DO + NST * TILE_BYTES;
    static constexpr int KV_OFF_DB = KV_OFF_QB + NST * XB_BYTES;
    static constexpr int KV_OFF_ONES = KV_OFF_DB + NST * XB_BYTES;
    static constexpr int KV_OFF_BAR = KV_OFF_ONES + XB_BYTES;
    static constexpr int KV_SMEM = KV_OFF_BAR + 16 * 8 + 16 + 1024;
    // dQ kernel shared memory: Q, dO, then QKST stages of K and QVST of V,
    // then barriers. S runs two key tiles ahead of dQ, so a K tile is needed
    // about two steps after its slot frees only with a third K stage; a V
    // tile is read once, one step ahead.
    static constexpr int QKST = (D == 128) ? 3 : 4;
    static constexpr int QVST = (D == 128) ? 2 : 4;
    static constexpr int Q_OFF_Q = 0;
    static constexpr int Q_OFF_DO = TILE_BYTES;
    static constexpr int Q_OFF_K = 2 * TILE_BYTES;
    static constexpr int Q_OFF_V = Q_OFF_K + QKST * TILE_BYTES;
    static constexpr int Q_OFF_BAR = Q_OFF_V + QVST * TILE_BYTES;
    static constexpr int Q_SMEM = Q_OFF_BAR + 24 * 8 + 16 + 1024;
    static constexpr uint32_t T_S2 = 384;   // dQ kernel: second S buffer
};

__device__ __forceinline__ float dot8_bf16(const uint4 &a, const uint4 &b)
{
    const __nv_bfloat162 *x = reinterpret_cast<const __nv_bfloat162 *>(&a);
    const __nv_bfloat162 *y = reinterpret_cast<const __nv_bfloat162 *>(&b);
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 fx = __bfloat1622float2(x[k]);
        const float2 fy = __bfloat1622float2(y[k]);
        acc = fmaf(fx.x, fy.x, acc);
        acc = fmaf(fx.y, fy.y, acc);
    }
    return acc;
}

// Two bf16 values whose sum is v to about 2^-17 relative: v's rounding and
// the rounding of what it left over.
__device__ __forceinline__ uint32_t bf16_hi_lo(float v)
{
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const float rest = isinf(v) ? 0.f : v - __bfloat162float(hi);
    return pack_bf16x2(__bfloat162float(hi), rest);
}

// D_i = sum_c dO_ic O_ic and -LSE_i * log2(e), D/8 lanes per (head, padded
// row): each lane one 16-byte chunk of O and dO, so a warp takes 32/(D/8) rows.
// For the dK/dV kernel the same two terms also go, as hi/lo bf16 pairs, into
// an extra K step of its products: qx[h][i] holds -LSE_i / scale (S^T + that,
// times scale*log2(e), is the exponent of P^T), dx[h][i] holds -D_i (dP^T +
// that is dP^T - D); a padding row gets -inf and 0. The first 128 threads
// also write the block of ones the key side multiplies them with.
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16 *__restrict__ o,
                                                      const __nv_bfloat16 *__restrict__ dout,
                                                      const float *__restrict__ lse, float *__restrict__ delta,
                                                      float *__restrict__ lse2, uint32_t *__restrict__ qx,
                                                      uint32_t *__restrict__ dx, uint4 *__restrict__ ones,
                                                      float inv_scale, int N, int Npad, int Hl, int Hq_total,
                                                      int q_head0)
{
    if (blockIdx.x == 0 && threadIdx.x < kTileM) {
        const uint32_t one2 = pack_bf16x2(1.f, 1.f);
        ones[2 * threadIdx.x] = make_uint4(one2, 0u, 0u, 0u);
        ones[2 * threadIdx.x + 1] = make_uint4(0u, 0u, 0u, 0u);
    }
    constexpr int kLanesPerRow = D / 8;
    static_assert(kLanesPerRow >= 1 && kLanesPerRow <= 32 && 32 % kLanesPerRow == 0, "lanes per row");
    const int lane = threadIdx.x & 31;
    const int64_t w = ((static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5) * (32 / kLanesPerRow) +
                      lane / kLanesPerRow;
    const int sl = lane % kLanesPerRow;
    const bool in_range = w < static_cast<int64_t>(Hl) * Npad;
    const int h = in_range ? static_cast<int>(w / Npad) : 0;
    const int i = in_range ? static_cast<int>(w % Npad) : N;
    float acc = 0.f;
    if (i < N) {
        const int64_t off = (static_cast<int64_t>(i) * Hq_total + q_head0 + h) * D;
        acc = dot8_bf16(reinterpret_cast<const uint4 *>(o + off)[sl], reinterpret_cast<const uint4 *>(dout + off)[sl]);
    }
    // the row's lanes in a fixed tree (every lane of the warp takes part)
#pragma unroll
    for (int off = kLanesPerRow / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (in_range && sl == 0) {
        const float lse_i = i < N ? lse[static_cast<int64_t>(h) * N + i] : CUDART_INF_F;
        delta[w] = i < N ? acc : 0.f;
        lse2[w] = i < N ? -lse_i * kLog2e : -CUDART_INF_F;
        qx[w] = bf16_hi_lo(i < N ? -lse_i * inv_scale : -CUDART_INF_F);
        dx[w] = bf16_hi_lo(i < N ? -acc : 0.f);
    }
}

// Column of the bf16 operand packed in tensor memory for K step kk (16 rows
// of the 128, two per column): part q wrote the 16-row steps of its columns
// into columns q * kPartCols + 0 .. kPartCols / 2 - 1.
__device__ __forceinline__ uint32_t pcol(int kk)
{
    constexpr int steps = kPartCols / 16;   // K steps per part
    return static_cast<uint32_t>((kk / steps) * kPartCols + (kk % steps) * 8);
}

// K-major SS descriptors for a 16-element K step kk of a 128-row tile.
template <int D>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_addr, int kk)
{
    using C = BwdCfg<D>;
    constexpr int steps = C::SW / 32;
    const uint32_t koff = (kk / steps) * C::ATOM_BYTES + (kk % steps) * 32;
    return smem_desc(tile_addr + koff, 16, 8 * C::SW, C::SWZ);
}

// MN-major descriptor of a [rows][d] tile used as B with N = d, K = rows:
// 16 rows per K step.
template <int D>
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile_addr, int kk)
{
    using C = BwdCfg<D>;
    return smem_desc(tile_addr + kk * 16 * C::SW, C::ATOM_BYTES, 8 * C::SW, C::SWZ);
}

template <int D>
__device__ __forceinline__ void tma_tile(const CUtensorMap *m, uint8_t *dst, uint64_t *bar, int head, int row0)
{
    using C = BwdCfg<D>;
#pragma unroll
    for (int a = 0; a < C::NA; ++a) tma_load_3d(dst + a * C::ATOM_BYTES, m, bar, a * C::AW, head, row0);
}

// ============================================================== dK / dV
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                         const __grid_constant__ CUtensorMap tmOnes, const BwdParams p)
{
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sK = smem + C::KV_OFF_K;
    uint8_t *sV = smem + C::KV_OFF_V;
    uint8_t *sQ = smem + C::KV_OFF_Q;
    uint8_t *sDO = smem + C::KV_OFF_DO;
    uint8_t *sQB = smem + C::KV_OFF_QB;
    uint8_t *sDB = smem + C::KV_OFF_DB;
    uint8_t *sOnes = smem + C::KV_OFF_ONES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::KV_OFF_BAR);
    uint64_t *kv_full = bars;
    uint64_t *qdo_full = bars + 1;            // [NST]
    uint64_t *qdo_empty = qdo_full + C::NST;  // [NST]
    uint64_t *s_full = qdo_empty + C::NST;   // S^T(i) computed
    uint64_t *ds_full = s_full + 1;           // dS^T(i) stored (all compute threads)
    uint64_t *dp_full = ds_full + 1;          // dP^T(i) computed
    uint64_t *p_ready = dp_full + 1;          // P^T(i) stored (all compute threads)
    uint64_t *acc_done = p_ready + 1;
    uint64_t *mma_done = acc_done + 1;
    uint64_t *never = mma_done + 1;           // never arrived on (timeout test only)
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(never + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int item = blockIdx.x;
    const int t = p.kv_order[item / p.Hkvl];
    const int kvh = item % p.Hkvl;
    const int G = p.Hl / p.Hkvl;
    const int qt0 = t;
    const int n_q = static_cast<int>((p.kv_qend[t] + kTileM - 1) / kTileM) - qt0;
    const int n_it = G * n_q;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < C::NST; ++s) {
            mbar_init(&qdo_full[s], 2);   // the copies' bytes and the producer warp's extra-step tiles
            mbar_init(&qdo_empty[s], 1);
        }
        mbar_init(s_full, 1);
        mbar_init(ds_full, kParts * 128);
        mbar_init(dp_full, 1);
        mbar_init(p_ready, kParts * 128);
        mbar_init(acc_done, 1);
        mbar_init(mma_done, 1);
        mbar_init(never, 1);
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
    WaitCtx wc{p.wait_limit_ns, p.status, *reinterpret_cast<volatile uint32_t *>(p.status) != 0u};

    if (warp == 0) {
        // ------------------------------------------------ producer: lane 0 issues the copies; the
        // whole warp builds each stage's extra K-step tiles (128 rows x 16 bf16, 32-byte
        // swizzle: a row's first 16 bytes sit in chunk (row >> 2) & 1) from the compact
        // per-query terms. Only the first 16 bytes of a row change; the rest stay zero.
        if (lane == 0) {
            mbar_arrive_expect_tx(kv_full, 2 * C::TILE_BYTES + C::XB_BYTES);
            tma_tile<D>(&tmK, sK, kv_full, p.kv_head0 + kvh, t * kTileN);
            tma_tile<D>(&tmV, sV, kv_full, p.kv_head0 + kvh, t * kTileN);
            tma_load_3d(sOnes, &tmOnes, kv_full, 0, 0, 0);
        }
        const int xchunk = (lane >> 2) & 1;   // chunk of rows lane + 32k holding the term
        for (int b = 0; b < 2 * C::NST; ++b) {
            uint8_t *blk = (b < C::NST ? sQB : sDB) + (b % C::NST) * C::XB_BYTES;
#pragma unroll
            for (int k = 0; k < kTileM / 32; ++k)
                reinterpret_cast<uint4 *>(blk + (lane + 32 * k) * kXStepBytes)[xchunk ^ 1] = make_uint4(0u, 0u, 0u, 0u);
        }
        int last_use[C::NST];
#pragma unroll
        for (int s = 0; s < C::NST; ++s) last_use[s] = -1;
        // the terms of iteration it, loaded one iteration ahead (while the stage is still busy)
        uint32_t qv[kTileM / 32], dv[kTileM / 32];
        auto load_terms = [&](int it) {
            const int h = kvh * G + it % G;
            const int64_t xo = static_cast<int64_t>(h) * p.Npad + static_cast<int64_t>(qt0 + it / G) * kTileM + lane;
#pragma unroll
            for (int k = 0; k < kTileM / 32; ++k) {
                qv[k] = p.qx[xo + 32 * k];
                dv[k] = p.dx[xo + 32 * k];
            }
        };
        if (n_it > 0) load_terms(0);
        for (int it = 0; it < n_it; ++it) {
            const int s = it % C::NST, u = it / C::NST;
            const int h = kvh * G + it % G;
            const int qt = qt0 + it / G;
            if (u > 0 && !mbar_wait_warp(&qdo_empty[s], (u - 1) & 1, wc)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&qdo_full[s], 2 * C::TILE_BYTES);
                tma_tile<D>(&tmQ, sQ + s * C::TILE_BYTES, &qdo_full[s], p.q_head0 + h, qt * kTileM);
                tma_tile<D>(&tmDO, sDO + s * C::TILE_BYTES, &qdo_full[s], p.q_head0 + h, qt * kTileM);
            }
            uint8_t *qb = sQB + s * C::XB_BYTES, *db = sDB + s * C::XB_BYTES;
#pragma unroll
            for (int k = 0; k < kTileM / 32; ++k) {
                const int r = lane + 32 * k;
                reinterpret_cast<uint4 *>(qb + r * kXStepBytes)[xchunk] = make_uint4(qv[k], 0u, 0u, 0u);
                reinterpret_cast<uint4 *>(db + r * kXStepBytes)[xchunk] = make_uint4(dv[k], 0u, 0u, 0u);
            }
            fence_async_smem();   // visible to the tensor core's operand reads
            __syncwarp();
            if (lane == 0) mbar_arrive(&qdo_full[s]);
            last_use[s] = u;
            if (it + 1 < n_it) load_terms(it + 1);
        }
        if (lane == 0) {
            WaitCtx drain{p.wait_limit_ns, p.status, false};
            mbar_wait(kv_full, 0, drain);
            for (int s = 0; s < C::NST; ++s)
                if (last_use[s] >= 0) mbar_wait(&qdo_full[s], last_use[s] & 1, drain);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        {   // the whole warp runs the loop; elect.sync picks the issuing lane
            const uint32_t aK = smem_u32(sK), aV = smem_u32(sV), aQ = smem_u32(sQ), aDO = smem_u32(sDO);
            // the extra K step: a column of ones (in pairs) against each query's hi/lo terms
            const uint64_t d_ones = smem_desc(smem_u32(sOnes), 16, 8 * kXStepBytes, kSwizzle32);
            bool ok = mbar_wait_warp(kv_full, 0, wc);
            auto issue_s = [&](int st) {   // S^T = K Q^T - LSE / scale for the query tile in stage st
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    umma_ss_elect(tbase + C::T_S, kmajor_desc<D>(aK, kk), kmajor_desc<D>(aQ + st * C::TILE_BYTES, kk),
                                  C::IDESC_SS, kk > 0 ? 1u : 0u);
                umma_ss_elect(tbase + C::T_S, d_ones,
                              smem_desc(smem_u32(sQB + st * C::XB_BYTES), 16, 8 * kXStepBytes, kSwizzle32),
                              C::IDESC_SS, 1u);
                umma_commit_elect(s_full);
            };
            auto issue_dp = [&](int st) {   // dP^T = V dO^T - D
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    umma_ss_elect(tbase + C::T_DP, kmajor_desc<D>(aV, kk), kmajor_desc<D>(aDO + st * C::TILE_BYTES, kk),
                                  C::IDESC_SS, kk > 0 ? 1u : 0u);
                umma_ss_elect(tbase + C::T_DP, d_ones,
                              smem_desc(smem_u32(sDB + st * C::XB_BYTES), 16, 8 * kXStepBytes, kSwizzle32),
                              C::IDESC_SS, 1u);
                umma_commit_elect(dp_full);
            };
            if (ok && n_it > 0) {
                ok = mbar_wait_warp(&qdo_full[0], 0, wc);
                if (ok) {
                    tc_fence_after();
                    issue_s(0);
                    issue_dp(0);
                }
            }
            for (int it = 0; ok && it < n_it; ++it) {
                const int s = it % C::NST;
                const int s1 = (it + 1) % C::NST, u1 = (it + 1) / C::NST;
                const bool more = it + 1 < n_it;
                if (!mbar_wait_warp(p_ready, it & 1, wc)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kTileM / 16; ++kk)   // dV += P^T dO
                    umma_ts_elect(tbase + C::T_ACC0, tbase + C::T_S + pcol(kk), mnmajor_desc<D>(aDO + s * C::TILE_BYTES, kk),
                                  C::IDESC_TS, (it > 0 || kk > 0) ? 1u : 0u);
                // the next S^T overwrites P^T(it), which the dV products above read first
                if (more) {
                    if (!mbar_wait_warp(&qdo_full[s1], u1 & 1, wc)) { ok = false; break; }
                    tc_fence_after();
                    issue_s(s1);
                }
                if (!mbar_wait_warp(ds_full, it & 1, wc)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < kTileM / 16; ++kk)   // dK += dS^T Q
                    umma_ts_elect(tbase + C::T_ACC1, tbase + C::T_DP + pcol(kk), mnmajor_desc<D>(aQ + s * C::TILE_BYTES, kk),
                                  C::IDESC_TS, (it > 0 || kk > 0) ? 1u : 0u);
                umma_commit_elect(&qdo_empty[s]);
                if (more) issue_dp(s1);
            }
            if (ok) umma_commit_elect(acc_done);
            umma_commit_elect(mma_done);
            WaitCtx drain{p.wait_limit_ns, p.status, false};
            mbar_wait(mma_done, 0, drain);
        }
    } else if (warp >= kComputeWarp0) {
        // ------------------------------------------------ element-wise: thread = key row r, kPartCols query columns
        const int quad = warp & 3, part = (warp - kComputeWarp0) >> 2;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const int j = t * kTileN + r;
        // keys past N see no query; otherwise the queries of key j are [j, dend)
        int dend = j;
        if (j < p.N) {
            int lo = j, hi = p.N;   // doc_start[lo] <= j; find the first index with doc_start > j
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (p.doc_start[mid] <= j) lo = mid; else hi = mid;
            }
            dend = hi;
        }
        const float sl2 = p.scale_log2;
        const uint32_t col = static_cast<uint32_t>(part * kPartCols);   // this part's columns in S^T / dP^T
        bool ok = true;
        if ((p.debug_flags & 2u) && blockIdx.x == 0) ok = mbar_wait_warp(never, 0, wc);   // runs out
        for (int it = 0; ok && it < n_it; ++it) {
            const int q0 = (qt0 + it / G) * kTileM + part * kPartCols;   // first query of this part
            // warp-uniform wait: the tcgen05.ld below needs the whole warp converged
            if (!mbar_wait_warp(s_full, it & 1, wc)) { ok = false; break; }
            tc_fence_after();
            const bool any_mask = __any_sync(0xffffffffu, (q0 < j) || (q0 + kPartCols - 1 >= dend));
            // phase 1: P^T = exp2((S^T - LSE / scale) * scale*log2(e)), bf16 into S^T's
            // columns (the products' extra K step has already subtracted LSE / scale)
            float pf[kPartCols];   // P^T in fp32: dS is formed from it, rounded once
            {
                uint32_t pp[kPartCols / 2];
                uint32_t sr[kPartCols];
                tmem_ld32(tbase + C::T_S + lane_off + col, sr);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < kPartCols / 2; ++e) {
                    float x0, x1;
                    mul2(x0, x1, __uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]), sl2, sl2);
                    if (any_mask) {
                        const int qi = q0 + 2 * e;
                        if (qi < j || qi >= dend) x0 = -CUDART_INF_F;
                        if (qi + 1 < j || qi + 1 >= dend) x1 = -CUDART_INF_F;
                    }
                    pf[2 * e] = ex2_approx(x0);
                    pf[2 * e + 1] = ex2_approx(x1);
                    pp[e] = pack_bf16x2(pf[2 * e], pf[2 * e + 1]);
                }
                tmem_st16(tbase + C::T_S + lane_off + col, pp);   // P^T (queries packed in pairs)
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(p_ready);
            // phase 2: dS^T = P^T (dP^T - D) from the fp32 P^T (the products' extra K step
            // has already subtracted D), bf16 into dP^T's columns
            if (!mbar_wait_warp(dp_full, it & 1, wc)) { ok = false; break; }
            tc_fence_after();
            {
                uint32_t dr[kPartCols];
                tmem_ld32(tbase + C::T_DP + lane_off + col, dr);
                tmem_ld_wait();
                uint32_t dd[kPartCols / 2];
#pragma unroll
                for (int e = 0; e < kPartCols / 2; ++e) {
                    float d0, d1;
                    mul2(d0, d1, pf[2 * e], pf[2 * e + 1], __uint_as_float(dr[2 * e]), __uint_as_float(dr[2 * e + 1]));
                    dd[e] = pack_bf16x2(d0, d1);
                }
                tmem_st16(tbase + C::T_DP + lane_off + col, dd);   // dS^T
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(ds_full);
        }
        // ---- epilogue: part p writes d columns [p * E, (p + 1) * E) of dV and dK, E = max(16, D / kParts)
        constexpr int E = (D / kParts) >= 16 ? D / kParts : 16;
        if (ok && part * E < D && mbar_wait_warp(acc_done, 0, wc)) {
            tc_fence_after();
            const bool valid = j < p.N;
            const int64_t kv_off = (static_cast<int64_t>(j) * p.Hkv_total + p.kv_head0 + kvh) * D + part * E;
            __nv_bfloat16 *dv_row = p.dv + kv_off;
            __nv_bfloat16 *dk_row = p.dk + kv_off;
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const float mul = which == 0 ? 1.f : p.scale;
                __nv_bfloat16 *row = which == 0 ? dv_row : dk_row;
                const uint32_t tacc = tbase + (which == 0 ? C::T_ACC0 : C::T_ACC1) + lane_off + part * E;
#pragma unroll
                for (int c = 0; c < E / 16; ++c) {
                    uint32_t raw[16];
                    tmem_ld16(tacc + c * 16, raw);
                    tmem_ld_wait();
                    uint32_t w[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        w[e] = pack_bf16x2(__uint_as_float(raw[2 * e]) * mul, __uint_as_float(raw[2 * e + 1]) * mul);
                    if (valid) {
                        uint4 *dst = reinterpret_cast<uint4 *>(row + c * 16);
                        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

// ============================================================== dQ
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       const BwdParams p)
{
    using C = BwdCfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + C::Q_OFF_Q;
    uint8_t *sDO = smem + C::Q_OFF_DO;
    uint8_t *sK = smem + C::Q_OFF_K;
    uint8_t *sV = smem + C::Q_OFF_V;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::Q_OFF_BAR);
    uint64_t *qdo_full = bars;
    uint64_t *k_full = bars + 1;             // [QKST]
    uint64_t *k_empty = k_full + C::QKST;    // [QKST] S(j) and dQ(j) have read K_j
    uint64_t *v_full = k_empty + C::QKST;    // [QVST]
    uint64_t *v_empty = v_full + C::QVST;    // [QVST] dP(j) has read V_j
    uint64_t *s_full = v_empty + C::QVST;    // [2] S(j) computed into buffer j % 2
    uint64_t *dp_full = s_full + 2;          // dP(j) computed
    uint64_t *ds_full = dp_full + 1;         // dS(j) stored (all compute threads)
    uint64_t *acc_done = ds_full + 1;
    uint64_t *mma_done = acc_done + 1;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int item = blockIdx.x;
    const int qt = p.q_order[item / p.Hl];
    const int h = item % p.Hl;
    const int kvh = h / (p.Hl / p.Hkvl);
    const int kt0 = p.tile_lo[qt] / kTileN;
    const int n_kv = qt - kt0 + 1;

    if (threadIdx.x == 0) {
        mbar_init(qdo_full, 1);
        for (int s = 0; s < C::QKST; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
        }
        for (int s = 0; s < C::QVST; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
        }
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(dp_full, 1);
        mbar_init(ds_full, kParts * 128);
        mbar_init(acc_done, 1);
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
    WaitCtx wc{p.wait_limit_ns, p.status, *reinterpret_cast<volatile uint32_t *>(p.status) != 0u};

    if (warp == 0) {
        // ------------------------------------------------ Q, dO and K producer
        if (lane == 0) {
            mbar_arrive_expect_tx(qdo_full, 2 * C::TILE_BYTES);
            tma_tile<D>(&tmQ, sQ, qdo_full, p.q_head0 + h, qt * kTileM);
            tma_tile<D>(&tmDO, sDO, qdo_full, p.q_head0 + h, qt * kTileM);
            int last_use[C::QKST];
#pragma unroll
            for (int s = 0; s < C::QKST; ++s) last_use[s] = -1;
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % C::QKST, u = j / C::QKST;
                if (u > 0 && !mbar_wait(&k_empty[s], (u - 1) & 1, wc)) break;
                mbar_arrive_expect_tx(&k_full[s], C::TILE_BYTES);
                tma_tile<D>(&tmK, sK + s * C::TILE_BYTES, &k_full[s], p.kv_head0 + kvh, (kt0 + j) * kTileN);
                last_use[s] = u;
            }
            WaitCtx drain{p.wait_limit_ns, p.status, false};
            mbar_wait(qdo_full, 0, drain);
            for (int s = 0; s < C::QKST; ++s)
                if (last_use[s] >= 0) mbar_wait(&k_full[s], last_use[s] & 1, drain);
        }
    } else if (warp == 2) {
        // ------------------------------------------------ V producer
        if (lane == 0) {
            int last_use[C::QVST];
#pragma unroll
            for (int s = 0; s < C::QVST; ++s) last_use[s] = -1;
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % C::QVST, u = j / C::QVST;
                if (u > 0 && !mbar_wait(&v_empty[s], (u - 1) & 1, wc)) break;
                mbar_arrive_expect_tx(&v_full[s], C::TILE_BYTES);
                tma_tile<D>(&tmV, sV + s * C::TILE_BYTES, &v_full[s], p.kv_head0 + kvh, (kt0 + j) * kTileN);
                last_use[s] = u;
            }
            WaitCtx drain{p.wait_limit_ns, p.status, false};
            for (int s = 0; s < C::QVST; ++s)
                if (last_use[s] >= 0) mbar_wait(&v_full[s], last_use[s] & 1, drain);
        }
    } else if (warp == 1) {
        {   // the whole warp runs the loop; elect.sync picks the issuing lane
            const uint32_t aQ = smem_u32(sQ), aDO = smem_u32(sDO), aK = smem_u32(sK), aV = smem_u32(sV);
            bool ok = mbar_wait_warp(qdo_full, 0, wc);
            auto sbuf = [&](int jj) { return tbase + ((jj & 1) ? C::T_S2 : C::T_S); };
            auto issue_s = [&](int jj) -> bool {   // S(jj) = Q K_jj^T into buffer jj % 2
                const int s = jj % C::QKST;
                if (!mbar_wait_warp(&k_full[s], (jj / C::QKST) & 1, wc)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    umma_ss_elect(sbuf(jj), kmajor_desc<D>(aQ, kk), kmajor_desc<D>(aK + s * C::TILE_BYTES, kk),
                                  C::IDESC_SS, kk > 0 ? 1u : 0u);
                umma_commit_elect(&s_full[jj & 1]);
                return true;
            };
            auto issue_dp = [&](int jj) -> bool {   // dP(jj) = dO V_jj^T
                const int s = jj % C::QVST;
                if (!mbar_wait_warp(&v_full[s], (jj / C::QVST) & 1, wc)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    umma_ss_elect(tbase + C::T_DP, kmajor_desc<D>(aDO, kk), kmajor_desc<D>(aV + s * C::TILE_BYTES, kk),
                                  C::IDESC_SS, kk > 0 ? 1u : 0u);
                umma_commit_elect(dp_full);
                umma_commit_elect(&v_empty[s]);
                return true;
            };
            if (ok && n_kv > 0) ok = issue_s(0) && issue_dp(0);
            if (ok && n_kv > 1) ok = issue_s(1);
            for (int j = 0; ok && j < n_kv; ++j) {
                const int s = j % C::QKST;
                if (!mbar_wait_warp(ds_full, j & 1, wc)) { ok = false; break; }
                tc_fence_after();
                // dP(j+1) first: it overwrites only dP(j), which the element-wise step
                // of j has read, and the next step's phase 1 then finds it done
                if (j + 1 < n_kv && !issue_dp(j + 1)) { ok = false; break; }
#pragma unroll
                for (int kk = 0; kk < kTileN / 16; ++kk)
                    umma_ts_elect(tbase + C::T_ACC0, sbuf(j) + pcol(kk), mnmajor_desc<D>(aK + s * C::TILE_BYTES, kk),
                                  C::IDESC_TS, (j > 0 || kk > 0) ? 1u : 0u);   // dQ += dS K
                umma_commit_elect(&k_empty[s]);
                // S(j+2) overwrites dS(j), read by the products just issued
                if (j + 2 < n_kv && !issue_s(j + 2)) { ok = false; break; }
            }
            if (ok) umma_commit_elect(acc_done);
            umma_commit_elect(mma_done);
            WaitCtx drain{p.wait_limit_ns, p.status, false};
            mbar_wait(mma_done, 0, drain);
        }
    } else if (warp >= kComputeWarp0) {
        // ------------------------------------------------ element-wise: thread = query row r, kPartCols key columns
        const int quad = warp & 3, part = (warp - kComputeWarp0) >> 2;
        const int r = quad * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
        const int i = qt * kTileM + r;
        const bool valid = i < p.N;
        const int lo = valid ? p.doc_start[i] : i;
        const float nl2 = p.lse2[static_cast<int64_t>(h) * p.Npad + i];   // -LSE * log2(e)
        const float di = p.delta[static_cast<int64_t>(h) * p.Npad + i];
        const float sl2 = p.scale_log2;
        const uint32_t col = static_cast<uint32_t>(part * kPartCols);
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            const int c0 = (kt0 + j) * kTileN + part * kPartCols;   // first key of this part
            const uint32_t tS = tbase + ((j & 1) ? C::T_S2 : C::T_S) + lane_off + col;
            if (!mbar_wait_warp(&s_full[j & 1], (j >> 1) & 1, wc)) { ok = false; break; }
            tc_fence_after();
            const bool any_mask = __any_sync(0xffffffffu, (c0 < lo) || (c0 + kPartCols - 1 > i));
            // phase 1 (while dP(j) may still be computing): P = exp2(S * scale*log2(e)
            // - LSE*log2(e)), kept in fp32 so that dS is rounded only once
            float pf[kPartCols];
            {
                uint32_t sr[kPartCols];
                tmem_ld32(tS, sr);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < kPartCols / 2; ++e) {
                    float x0, x1;
                    fma2_bcast(x0, x1, __uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1]), sl2, nl2);
                    if (any_mask) {
                        const int key = c0 + 2 * e;
                        if (key < lo || key > i) x0 = -CUDART_INF_F;
                        if (key + 1 < lo || key + 1 > i) x1 = -CUDART_INF_F;
                    }
                    pf[2 * e] = ex2_approx(x0);
                    pf[2 * e + 1] = ex2_approx(x1);
                }
            }
            // phase 2: dS = P (dP - D) from the fp32 P, bf16 into S's columns
            if (!mbar_wait_warp(dp_full, j & 1, wc)) { ok = false; break; }
            tc_fence_after();
            {
                uint32_t dr[kPartCols];
                tmem_ld32(tbase + C::T_DP + lane_off + col, dr);
                tmem_ld_wait();
                uint32_t dd[kPartCols / 2];
#pragma unroll
                for (int e = 0; e < kPartCols / 2; ++e) {
                    float t0, t1, d0, d1;
                    sub2(t0, t1, __uint_as_float(dr[2 * e]), __uint_as_float(dr[2 * e + 1]), di, di);
                    mul2(d0, d1, pf[2 * e], pf[2 * e + 1], t0, t1);
                    dd[e] = pack_bf16x2(d0, d1);
                }
                tmem_st16(tS, dd);   // dS (keys packed in pairs)
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(ds_full);
        }
        // ---- epilogue: part p writes d columns [p * E, (p + 1) * E) of dQ, E = max(16, D / kParts)
        constexpr int E = (D / kParts) >= 16 ? D / kParts : 16;
        if (ok && part * E < D && mbar_wait_warp(acc_done, 0, wc)) {
            tc_fence_after();
            __nv_bfloat16 *row = p.dq + (static_cast<int64_t>(i) * p.Hq_total + p.q_head0 + h) * D + part * E;
            const uint32_t tacc = tbase + C::T_ACC0 + lane_off + part * E;
#pragma unroll
            for (int c = 0; c < E / 16; ++c) {
                uint32_t raw[16];
                tmem_ld16(tacc + c * 16, raw);
                tmem_ld_wait();
                uint32_t w[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    w[e] = pack_bf16x2(__uint_as_float(raw[2 * e]) * p.scale, __uint_as_float(raw[2 * e + 1]) * p.scale);
                if (valid) {
                    uint4 *dst = reinterpret_cast<uint4 *>(row + c * 16);
                    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes, bool *done)
{
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) return e;
        done[dev] = true;
    }
    return cudaSuccess;
}

template <int D>
cudaError_t launch_bwd_d(const BwdLaunch &a, cudaStream_t stream)
{
    using C = BwdCfg<D>;
    static_assert(C::KV_SMEM <= 232448 && C::Q_SMEM <= 232448, "shared memory budget");
    const int T = static_cast<int>(ceil_div(a.N, kTileM));
    const int Npad = T * kTileM;
    alignas(64) CUtensorMap tq, tk, tv, tdo;
    const int64_t qs = int64_t(a.Hq_total) * D * 2, ks = int64_t(a.Hkv_total) * D * 2;
    if (!encode_tmap_3d(&tq, a.q, D, a.Hq_total, a.N, int64_t(D) * 2, qs, C::AW, kTileM, C::SW) ||
        !encode_tmap_3d(&tdo, a.dout, D, a.Hq_total, a.N, int64_t(D) * 2, qs, C::AW, kTileM, C::SW) ||
        !encode_tmap_3d(&tk, a.k, D, a.Hkv_total, a.N, int64_t(D) * 2, ks, C::AW, kTileN, C::SW) ||
        !encode_tmap_3d(&tv, a.v, D, a.Hkv_total, a.N, int64_t(D) * 2, ks, C::AW, kTileN, C::SW))
        return cudaErrorInvalidValue;
    // the dK/dV kernel's block of ones for its extra K step (128 rows x 16 bf16)
    alignas(64) CUtensorMap tones;
    if (!encode_tmap_3d(&tones, a.ws + a.L.ones, 16, 1, kTileM, kXStepBytes, kXStepBytes, 16, kTileM, kXStepBytes))
        return cudaErrorInvalidValue;
    BwdParams p;
    p.doc_start = reinterpret_cast<const int32_t *>(a.ws + a.L.doc_start);
    p.tile_lo = reinterpret_cast<const int32_t *>(a.ws + a.L.tile_lo);
    p.q_order = reinterpret_cast<const int32_t *>(a.ws + a.L.q_order);
    p.kv_qend = reinterpret_cast<const int32_t *>(a.ws + a.L.kv_qend);
    p.kv_order = reinterpret_cast<const int32_t *>(a.ws + a.L.kv_order);
    float *delta = reinterpret_cast<float *>(a.ws + a.L.delta);
    float *lse2 = reinterpret_cast<float *>(a.ws + a.L.lse2);
    p.delta = delta;
    p.lse2 = lse2;
    p.qx = reinterpret_cast<const uint32_t *>(a.ws + a.L.qb);
    p.dx = reinterpret_cast<const uint32_t *>(a.ws + a.L.db);
    p.dq = static_cast<__nv_bfloat16 *>(a.dq);
    p.dk = static_cast<__nv_bfloat16 *>(a.dk);
    p.dv = static_cast<__nv_bfloat16 *>(a.dv);
    p.N = static_cast<int>(a.N);
    p.Npad = Npad;
    p.T = T;
    p.Hl = a.Hl;
    p.Hkvl = a.Hkvl;
    p.Hq_total = a.Hq_total;
    p.Hkv_total = a.Hkv_total;
    p.q_head0 = a.q_head0;
    p.kv_head0 = a.kv_head0;
    p.scale = a.scale;
    p.scale_log2 = a.scale * kLog2e;
    p.status = reinterpret_cast<uint32_t *>(a.ws + a.L.status);
    p.wait_limit_ns = a.wait_limit_ns;
    p.debug_flags = a.debug_flags;

    const int64_t prep_threads = int64_t(a.Hl) * Npad * (D / 8);   // D/8 lanes per (head, row)
    bwd_prep_kernel<D><<<static_cast<unsigned>(ceil_div(prep_threads, 256)), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(a.o), static_cast<const __nv_bfloat16 *>(a.dout), a.lse, delta, lse2,
        reinterpret_cast<uint32_t *>(a.ws + a.L.qb), reinterpret_cast<uint32_t *>(a.ws + a.L.db),
        reinterpret_cast<uint4 *>(a.ws + a.L.ones), 1.f / a.scale, p.N, Npad, a.Hl, a.Hq_total, a.q_head0);
    static bool kv_attr[64] = {}, q_attr[64] = {};
    cudaError_t e = set_smem(attn_bwd_dkdv_kernel<D>, C::KV_SMEM, kv_attr);
    if (e != cudaSuccess) return e;
    e = set_smem(attn_bwd_dq_kernel<D>, C::Q_SMEM, q_attr);
    if (e != cudaSuccess) return e;
    attn_bwd_dkdv_kernel<D><<<static_cast<unsigned>(int64_t(T) * a.Hkvl), kBwdThreads, C::KV_SMEM, stream>>>(
        tq, tk, tv, tdo, tones, p);
    attn_bwd_dq_kernel<D><<<static_cast<unsigned>(int64_t(T) * a.Hl), kBwdThreads, C::Q_SMEM, stream>>>(
        tq, tk, tv, tdo, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd(const BwdLaunch &a, cudaStream_t stream)
{
    switch (a.d) {
    case 32: return launch_bwd_d<32>(a, stream);
    case 64: return launch_bwd_d<64>(a, stream);
    case 128: return launch_bwd_d<128>(a, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace uly
