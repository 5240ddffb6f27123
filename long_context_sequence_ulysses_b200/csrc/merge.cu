// merge.cu -- the merge of partial attention results over disjoint key sets.
//
// Ring attention (set against Ulysses on the page "Ulysses 序列並行：百萬 Token
// 上下文訓練", section "競品分析", and on the page "Ulysses verteilt
// Millionen-Token-Kontexte auf mehrere GPUs", section "Wann Ulysses sinnvoll
// ist") passes chunks of keys and values around the ranks; each step gives a
// partial result (o_s, lse_s) of the local queries over one chunk. Because each
// o_s is normalised by its own sum exp(lse_s), the result over the union is
//     L = log sum_s exp(lse_s),   o = sum_s exp(lse_s - L) o_s,   lse = L,
// evaluated here with the largest lse_s subtracted first. Partials with
// lse_s = -inf (no key) weigh 0; a row with none gets o = 0, lse = -inf.
//
// HBM-bound (R reads of o per output written): one thread per 16-byte vector
// of an output row, 8 bf16 values, the R weights of its row computed from the
// fp32 LSEs (read through L1, shared by the threads of a row), accumulation in
// fp32, result rounded to bf16 once.
#include "ulysses_internal.cuh"

#include <cuda_bf16.h>
#include <math_constants.h>

namespace uly {

namespace {

constexpr int kMergeThreads = 256;
constexpr int kMergeMaxParts = 64;

template <int D>
__global__ void __launch_bounds__(kMergeThreads) attn_merge_kernel(const uint4 *__restrict__ o_parts,
                                                                  const float *__restrict__ lse_parts, int R,
                                                                  int64_t M, int Hl, uint4 *__restrict__ o,
                                                                  float *__restrict__ lse, int64_t lse_ld)
{
    constexpr int V = D / 8;   // 16-byte vectors per row of one head
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kMergeThreads + threadIdx.x;
    const int64_t rows = M * Hl;
    if (t >= rows * V) return;
    const int64_t row = t / V;            // (m, h) in the [M][Hl] order of o
    const int e = static_cast<int>(t - row * V);
    const int64_t m = row / Hl;
    const int h = static_cast<int>(row - m * Hl);
    float mx = -CUDART_INF_F;
    for (int s = 0; s < R; ++s) mx = fmaxf(mx, lse_parts[(static_cast<int64_t>(s) * Hl + h) * M + m]);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float L = -CUDART_INF_F;
    if (mx != -CUDART_INF_F) {
        float sum = 0.f;
        for (int s = 0; s < R; ++s) sum += __expf(lse_parts[(static_cast<int64_t>(s) * Hl + h) * M + m] - mx);
        L = mx + __logf(sum);
        for (int s = 0; s < R; ++s) {
            const float ls = lse_parts[(static_cast<int64_t>(s) * Hl + h) * M + m];
            if (ls == -CUDART_INF_F) continue;
            const float w = __expf(ls - L);
            const uint4 v = o_parts[(static_cast<int64_t>(s) * rows + row) * V + e];
            const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 f = __bfloat1622float2(b[k]);
                acc[2 * k] = fmaf(w, f.x, acc[2 * k]);
                acc[2 * k + 1] = fmaf(w, f.y, acc[2 * k + 1]);
            }
        }
    }
    uint4 out;
    __nv_bfloat162 *ob = reinterpret_cast<__nv_bfloat162 *>(&out);
#pragma unroll
    for (int k = 0; k < 4; ++k) ob[k] = __floats2bfloat162_rn(acc[2 * k], acc[2 * k + 1]);
    o[row * V + e] = out;
    if (e == 0) lse[static_cast<int64_t>(h) * lse_ld + m] = L;
}

}  // namespace

cudaError_t launch_attn_merge(const void *o_parts, const float *lse_parts, int R, int64_t M, int Hl, int d,
                              void *o, float *lse, int64_t lse_ld, cudaStream_t stream)
{
    if (R < 1 || R > kMergeMaxParts) return cudaErrorInvalidValue;
    const int64_t threads = M * Hl * (d / 8);
    const int64_t blocks = (threads + kMergeThreads - 1) / kMergeThreads;
    if (blocks == 0) return cudaSuccess;
    const uint4 *src = static_cast<const uint4 *>(o_parts);
    uint4 *dst = static_cast<uint4 *>(o);
    switch (d) {
    case 32: attn_merge_kernel<32><<<static_cast<unsigned>(blocks), kMergeThreads, 0, stream>>>(src, lse_parts, R, M, Hl, dst, lse, lse_ld); break;
    case 64: attn_merge_kernel<64><<<static_cast<unsigned>(blocks), kMergeThreads, 0, stream>>>(src, lse_parts, R, M, Hl, dst, lse, lse_ld); break;
    case 128: attn_merge_kernel<128><<<static_cast<unsigned>(blocks), kMergeThreads, 0, stream>>>(src, lse_parts, R, M, Hl, dst, lse, lse_ld); break;
    default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace uly
