// proj.cu -- the projections on either side of the Ulysses exchange, on the
// sm_100a tensor cores, with the exchange's relayout fused into them.
//
// Page "Hugging Face并行加速：10倍提升超长序列训练效率", section "Ulysses的工作原理":
// each GPU projects its own tokens to Q, K, V (step QKV投影) before the first
// all-to-all, and applies the output projection (step 输出投影) after the
// second; page "DeepSpeed Ulysses 详解", section "DeepSpeed-Ulysses 的核心机制",
// items 2 and 6. Both are plain GEMMs, C[M][Nc] = A[M][K] B[Nc][K]^T with the
// token rows as M, computed here for the tokens of all P emulated ranks at
// once, with the layout change done by the GEMM itself:
//   - QKV projection: x [N][hidden] times w_qkv [(H+2Hkv)d][hidden]^T; the
//     epilogue writes each 32-column chunk of a row (part of one head) straight
//     into that head's rank slice, q [P][N][H/P][d] and k, v [P][N][Hkv/P][d],
//     the layout the exchange delivers, so the projection and the first
//     exchange are one pass over HBM;
//   - output projection: the A operand is loaded straight from the head
//     slices o [P][N][H/P][d] by a 4-D TMA map (K block kb covers head
//     kb*64/d of the sequence layout, i.e. rank and local head), so the second
//     exchange and the projection are one pass; y [N][hidden] row-major.
//
// Kernel: persistent, one CTA per SM, 128 x BN output tiles (BN = 256, or 128
// when Nc is not a multiple of 256), K in 64-column blocks through a
// kStages-deep TMA ring (128-byte swizzle, K-major A and B), tcgen05 SS MMAs
// 128 x BN x 16 issued by one elected lane into one of two tensor-memory
// accumulators, so that the epilogue of tile i (four warps: tensor-memory
// load, bf16 rounding, global stores) overlaps the main loop of tile i+1.
// Tiles go out in row-block-major order (all column blocks of a row block
// before the next), so the CTAs in flight share A rows and the weights in L2.
// Warps: 0 TMA producer, 1 tensor-memory allocation and MMA issue, 4..7
// epilogue. Every wait is bounded (a timeout is recorded in the workspace
// status word, and the kernel drains and returns).
#include "ptx.cuh"
#include "ulysses_internal.cuh"

#include <cuda_bf16.h>

namespace uly {

namespace {

constexpr int kGemmThreads = 256;
constexpr int kBM = 128;
constexpr int kBK = 64;           // one 128-byte swizzle atom of bf16
constexpr int kStages = 4;
constexpr int kEpiWarp0 = 4;

template <int BN>
struct GemmCfg {
    static constexpr int A_BYTES = kBM * kBK * 2;
    static constexpr int B_BYTES = BN * kBK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int OFF_BAR = kStages * STAGE;
    static constexpr int NBAR = 2 * kStages + 2 + 2 + 1;
    static constexpr int SMEM = OFF_BAR + NBAR * 8 + 16 + 1024;
    static constexpr uint32_t IDESC = idesc_bf16_f32(kBM, BN, false, false);
    static constexpr uint32_t TMEM_COLS = 2 * BN;
};

struct GemmParams {
    int M, Nc, K;                 // C[M][Nc] = A[M][K] B[Nc][K]^T
    int n_blocks, k_blocks, tiles;
    int a_heads;                  // 1: A is read from head slices [P][M][Hl][d] (4-D map)
    int d, Hl, a_aw;              // head dim, heads per rank, A box width along d
    int epi_qkv;                  // 1: scatter C into Q, K, V head slices; 0: plain row-major C
    __nv_bfloat16 *out0, *out1, *out2;
    int H, Hkv, P;
    uint32_t *status;
    uint64_t wait_limit_ns;
};

// Destination of the 32 output columns starting at `col` of token row `row`.
__device__ __forceinline__ __nv_bfloat16 *out_ptr(const GemmParams &p, int row, int col)
{
    if (!p.epi_qkv) return p.out0 + static_cast<int64_t>(row) * p.Nc + col;
    __nv_bfloat16 *base;
    int Hx;
    if (col < p.H * p.d) {
        base = p.out0; Hx = p.H;
    } else if (col < (p.H + p.Hkv) * p.d) {
        base = p.out1; Hx = p.Hkv; col -= p.H * p.d;
    } else {
        base = p.out2; Hx = p.Hkv; col -= (p.H + p.Hkv) * p.d;
    }
    const int g = col / p.d, cc = col - g * p.d;   // global head, column within it
    const int hxl = Hx / p.P;
    const int r = g / hxl, h = g - r * hxl;        // rank, head within the rank's slice
    return base + ((static_cast<int64_t>(r) * p.M + row) * hxl + h) * p.d + cc;
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const GemmParams p)
{
    using C = GemmCfg<BN>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *full = bars;                   // [kStages]
    uint64_t *empty = bars + kStages;        // [kStages]
    uint64_t *acc_full = empty + kStages;    // [2]
    uint64_t *acc_empty = acc_full + 2;      // [2]
    uint64_t *mma_done = acc_empty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(mma_done + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 128);
        }
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;
    WaitCtx wc{p.wait_limit_ns, p.status, *reinterpret_cast<volatile uint32_t *>(p.status) != 0u};

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            prefetch_tmap(&tmA);
            prefetch_tmap(&tmB);
            int it = 0;
            int last_use[kStages];
#pragma unroll
            for (int s = 0; s < kStages; ++s) last_use[s] = -1;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
                const int m0 = (t / p.n_blocks) * kBM, n0 = (t % p.n_blocks) * BN;
                for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                    const int s = it % kStages, u = it / kStages;
                    if (u > 0 && !mbar_wait(&empty[s], (u - 1) & 1, wc)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[s], C::STAGE);
                    uint8_t *sa = smem + s * C::STAGE;
                    if (p.a_heads) {
                        // K columns [kb*64, kb*64+64) of the sequence layout: global head
                        // g = kb*64/d (and the next 64/d - 1 heads when d < 64), column c0 within it
                        const int k0 = kb * kBK;
                        const int g = k0 / p.d, c0 = k0 - g * p.d;
                        tma_load_4d(sa, &tmA, &full[s], c0, g % p.Hl, m0, g / p.Hl);
                    } else {
                        tma_load_3d(sa, &tmA, &full[s], kb * kBK, 0, m0);
                    }
                    tma_load_3d(sa + C::A_BYTES, &tmB, &full[s], kb * kBK, 0, n0);
                    last_use[s] = u;
                }
            }
            WaitCtx drain{p.wait_limit_ns, p.status, false};
            for (int s = 0; s < kStages; ++s)
                if (last_use[s] >= 0) mbar_wait(&full[s], last_use[s] & 1, drain);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (whole warp, elected lane)
        const uint32_t a0 = smem_u32(smem);
        int it = 0, tc = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++tc) {
            const int b = tc & 1, ub = tc >> 1;
            if (ub > 0 && !mbar_wait_warp(&acc_empty[b], (ub - 1) & 1, wc)) { ok = false; break; }
            tc_fence_after();
            const uint32_t dacc = tbase + static_cast<uint32_t>(b * BN);
            for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
                const int s = it % kStages, u = it / kStages;
                if (!mbar_wait_warp(&full[s], u & 1, wc)) { ok = false; break; }
                tc_fence_after();
                const uint32_t sa = a0 + s * C::STAGE, sb = sa + C::A_BYTES;
#pragma unroll
                for (int kk = 0; kk < kBK / 16; ++kk)
                    umma_ss_elect(dacc, smem_desc(sa + kk * 32, 16, 1024, kSwizzle128),
                                  smem_desc(sb + kk * 32, 16, 1024, kSwizzle128), C::IDESC,
                                  (kb > 0 || kk > 0) ? 1u : 0u);
                umma_commit_elect(&empty[s]);
            }
            if (ok) umma_commit_elect(&acc_full[b]);
        }
        umma_commit_elect(mma_done);
        WaitCtx drain{p.wait_limit_ns, p.status, false};
        mbar_wait(mma_done, 0, drain);
    } else if (warp >= kEpiWarp0) {
        // ------------------------------------------------------------ epilogue: thread = output row
        const int e = threadIdx.x - kEpiWarp0 * 32;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        int tc = 0;
        for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++tc) {
            const int b = tc & 1, ub = tc >> 1;
            if (!mbar_wait_warp(&acc_full[b], ub & 1, wc)) break;
            tc_fence_after();
            const int row = (t / p.n_blocks) * kBM + e, n0 = (t % p.n_blocks) * BN;
            const uint32_t tacc = tbase + static_cast<uint32_t>(b * BN) + lane_off;
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t raw[32];
                tmem_ld32(tacc + c * 32, raw);
                tmem_ld_wait();
                uint32_t pk[16];
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    pk[k] = pack_bf16x2(__uint_as_float(raw[2 * k]), __uint_as_float(raw[2 * k + 1]));
                if (row < p.M) {
                    uint4 *dst = reinterpret_cast<uint4 *>(out_ptr(p, row, n0 + c * 32));
#pragma unroll
                    for (int k = 0; k < 4; ++k) dst[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[b]);
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, C::TMEM_COLS);
}

template <int BN>
cudaError_t launch_gemm_bn(const ProjLaunch &a, cudaStream_t stream)
{
    using C = GemmCfg<BN>;
    static_assert(C::SMEM <= 232448, "shared memory budget");
    alignas(64) CUtensorMap ta, tb;
    bool ok;
    if (a.a_heads) {
        // A: head slices [P][M][Hl][d], box {aw, 64/aw heads, 128 tokens, 1 rank}
        const int aw = a.d < kBK ? a.d : kBK;
        const int64_t dims[4] = {a.d, a.Hl, a.M, a.P};
        const int64_t strides[3] = {int64_t(a.d) * 2, int64_t(a.Hl) * a.d * 2, int64_t(a.M) * a.Hl * a.d * 2};
        const int box[4] = {aw, kBK / aw, kBM, 1};
        ok = encode_tmap(&ta, a.A, 4, dims, strides, box, 128);
    } else {
        const int64_t dims[3] = {a.K, 1, a.M};
        const int64_t strides[2] = {int64_t(a.K) * 2, int64_t(a.K) * 2};
        const int box[3] = {kBK, 1, kBM};
        ok = encode_tmap(&ta, a.A, 3, dims, strides, box, 128);
    }
    {
        const int64_t dims[3] = {a.K, 1, a.Nc};
        const int64_t strides[2] = {int64_t(a.K) * 2, int64_t(a.K) * 2};
        const int box[3] = {kBK, 1, BN};
        ok = ok && encode_tmap(&tb, a.B, 3, dims, strides, box, 128);
    }
    if (!ok) return cudaErrorInvalidValue;
    GemmParams p;
    p.M = static_cast<int>(a.M);
    p.Nc = a.Nc;
    p.K = a.K;
    p.n_blocks = a.Nc / BN;
    p.k_blocks = a.K / kBK;
    const int64_t tiles = ceil_div(a.M, kBM) * p.n_blocks;
    if (tiles > INT32_MAX) return cudaErrorInvalidValue;
    p.tiles = static_cast<int>(tiles);
    p.a_heads = a.a_heads;
    p.d = a.d;
    p.Hl = a.Hl;
    p.a_aw = a.d < kBK ? a.d : kBK;
    p.epi_qkv = a.epi_qkv;
    p.out0 = static_cast<__nv_bfloat16 *>(a.out0);
    p.out1 = static_cast<__nv_bfloat16 *>(a.out1);
    p.out2 = static_cast<__nv_bfloat16 *>(a.out2);
    p.H = a.H;
    p.Hkv = a.Hkv;
    p.P = a.P;
    p.status = a.status;
    p.wait_limit_ns = a.wait_limit_ns;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(proj_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const int sms = num_sms_current_device();
    const int grid = p.tiles < sms ? p.tiles : sms;
    proj_gemm_kernel<BN><<<static_cast<unsigned>(grid), kGemmThreads, C::SMEM, stream>>>(ta, tb, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_proj_gemm(const ProjLaunch &a, cudaStream_t stream)
{
    if (a.Nc % 256 == 0) return launch_gemm_bn<256>(a, stream);
    return launch_gemm_bn<128>(a, stream);
}

}  // namespace uly
