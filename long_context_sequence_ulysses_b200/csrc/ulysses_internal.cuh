// ulysses_internal.cuh -- declarations shared by the library's .cu files:
// workspace layout and kernel launchers. Not part of the public ABI.
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace uly {

constexpr int kTileM = 128;   // query rows per tile
constexpr int kTileN = 128;   // keys per tile
constexpr int kScanBlock = 1024;   // tokens per block of the doc-start scan
constexpr uint32_t kStatusTimeoutHost = 1u;   // same bit as the device-side timeout flag

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace layout (every section 256-byte aligned):
//   status     uint32 [64]        [0] status word (bit 0: a bounded wait ran out),
//                                 [1] work counter of the persistent forward kernel
//   doc_start  int32  [N]         first token of the row's document
//   tile_lo    int32  [T]         doc_start of the first row of each 128-row tile
//   q_order    int32  [T]         query tiles heaviest first (backward, and the
//                                 forward when its items pair heads); forward with
//                                 tile-pair items: pairs (2u, 2u+1), heaviest first
//   block_agg  int32  [nb]        per-block maxima of the doc-start scan (nb = ceil(N/1024))
//   block_carry int32 [nb]        each block's carry (used when nb > 1024)
//   scratch    int32  [2T + 2]    histogram for the tile sort (when it does not
//                                 fit in the sorting CTA's shared memory)
// backward only (Npad = T * 128):
//   kv_qend    int32  [T]         one past the last row that attends to key tile t
//   kv_order   int32  [T]         key tiles, heaviest first
//   delta      fp32   [Hl][Npad]  D_i = sum_c dO_ic O_ic (0 on padding rows)
//   lse2       fp32   [Hl][Npad]  LSE_i * log2(e) (+inf on padding rows)
// Bytes of one row of an extra 16-element (bf16) K step of the backward's
// S^T and dP^T products.
constexpr int kXStepBytes = 32;

struct WsLayout {
    size_t status, doc_start, tile_lo, q_order, block_agg, block_carry, scratch;
    size_t kv_qend, kv_order, delta, lse2;
    size_t qb, db, ones;   // backward: per-query terms as an extra K step (see attn_bwd.cu)
    size_t total;
};

inline WsLayout ws_layout(int64_t N, int Hl, bool backward)
{
    WsLayout L{};
    const int64_t T = ceil_div(N, kTileM);
    size_t off = 0;
    L.status = off;    off += align256(64 * 4);
    L.doc_start = off; off += align256(static_cast<size_t>(N) * 4);
    L.tile_lo = off;   off += align256(static_cast<size_t>(T) * 4);
    L.q_order = off;   off += align256(static_cast<size_t>(T) * 4);
    L.block_agg = off;   off += align256(static_cast<size_t>(ceil_div(N, kScanBlock)) * 4);
    L.block_carry = off; off += align256(static_cast<size_t>(ceil_div(N, kScanBlock)) * 4);
    L.scratch = off;   off += align256(static_cast<size_t>(2 * T + 2) * 4);
    if (backward) {
        L.kv_qend = off;  off += align256(static_cast<size_t>(T) * 4);
        L.kv_order = off; off += align256(static_cast<size_t>(T) * 4);
        L.delta = off;    off += align256(static_cast<size_t>(T) * kTileM * Hl * 4);
        L.lse2 = off;     off += align256(static_cast<size_t>(T) * kTileM * Hl * 4);
        L.qb = off;       off += align256(static_cast<size_t>(T) * kTileM * Hl * 4);
        L.db = off;       off += align256(static_cast<size_t>(T) * kTileM * Hl * 4);
        L.ones = off;     off += align256(static_cast<size_t>(kTileM) * kXStepBytes);
    } else {
        L.kv_qend = L.kv_order = L.delta = L.lse2 = L.qb = L.db = L.ones = 0;
    }
    L.total = off;
    return L;
}

// relayout.cu
// The sequence side's rows hold row_heads heads, of which [head0, head0 + Hx)
// are exchanged (row_heads = Hx, head0 = 0 for whole rows).
cudaError_t launch_relayout(bool to_head, const void *src, void *dst, int64_t N, int P, int Hx, int d, int rank,
                            int row_heads, int head0, cudaStream_t stream, int num_sms);

// The forward pairs two query heads of one KV group in a work item when the
// group size Hl/Hkvl is even, else two consecutive query tiles of one head.
inline bool fwd_pairs_heads(int Hl, int Hkvl) { return Hkvl > 0 && (Hl / Hkvl) % 2 == 0; }

// docbounds.cu: doc_start, tile_lo and the query order (single tiles, or
// pairs of tiles for a forward with tile-pair items; for the backward also
// kv_qend and the key-tile order); the forward's last sort lets the attention
// kernel start early (programmatic dependent launch).
// The forward's schedule covers query tiles [q_tile0, q_tile0 + q_tiles) and
// counts only the key tiles kvlo_t .. kvhi_t (the key window); the backward
// passes the whole sequence (0, T, 0, T - 1).
struct DbWindow {
    int q_tile0, q_tiles, kvlo_t, kvhi_t;
};
cudaError_t launch_docbounds(const int32_t *pos, int64_t N, char *ws, const WsLayout &L, bool backward,
                             bool fwd_tile_pairs, const DbWindow &win,
                             cudaStream_t stream);   // also clears the status word

// Forward attention launch description.
struct FwdLaunch {
    const void *q, *k, *v;       // base pointers of [N][Hq_total][d] / [N][Hkv_total][d]
    int Hq_total, Hkv_total;     // heads per token row in the q / kv buffers
    int q_head0, kv_head0;       // first head of this rank's slice in those rows
    void *o;                     // base of [N][Ho_total][d]
    int Ho_total, o_head0;
    float *lse;                  // [Hl][lse_ld]
    int64_t N;
    int Hl, Hkvl, d;
    // rows [q_lo, q_hi) are computed (O row i at row i - q_lo of o, LSE at
    // column i - q_lo of lse), over the keys [kv_lo, kv_hi) only; a
    // whole-sequence call has q_lo = kv_lo = 0, q_hi = kv_hi = lse_ld = N
    int64_t q_lo, q_hi, kv_lo, kv_hi, lse_ld;
    float scale;
    const char *ws;
    WsLayout L;
    uint64_t wait_limit_ns;
    uint32_t debug_flags;
};
cudaError_t launch_attn_fwd(const FwdLaunch &a, cudaStream_t stream);

// Merge of R partial attention results over disjoint key sets (merge.cu).
cudaError_t launch_attn_merge(const void *o_parts, const float *lse_parts, int R, int64_t M, int Hl, int d,
                              void *o, float *lse, int64_t lse_ld, cudaStream_t stream);

// Backward attention launch description (no fused layout: slice buffers).
struct BwdLaunch {
    const void *q, *k, *v, *o, *dout;   // [N][Hq_total][d] (q, o, dout) / [N][Hkv_total][d] (k, v)
    const float *lse;
    void *dq, *dk, *dv;                 // same row layouts as q / k / v
    int64_t N;
    int Hl, Hkvl, d;
    int Hq_total, Hkv_total;            // heads per token row (Hl / Hkvl for slice buffers)
    int q_head0, kv_head0;              // first head of this rank's slice in those rows
    float scale;
    char *ws;
    WsLayout L;
    uint64_t wait_limit_ns;
    uint32_t debug_flags = 0;
};
cudaError_t launch_attn_bwd(const BwdLaunch &a, cudaStream_t stream);

// Projection GEMM launch description (proj.cu): C[M][Nc] = A[M][K] B[Nc][K]^T.
struct ProjLaunch {
    const void *A, *B;
    int64_t M;
    int Nc, K;
    int a_heads;                 // 1: A is the head slices [P][M][Hl][d] (K = P*Hl*d), else [M][K]
    int d, Hl, P;
    int epi_qkv;                 // 1: C goes to the Q, K, V head slices (out0..2); 0: row-major C in out0
    int H, Hkv;
    void *out0, *out1, *out2;
    uint32_t *status;
    uint64_t wait_limit_ns;
};
cudaError_t launch_proj_gemm(const ProjLaunch &a, cudaStream_t stream);

// api.cu
int num_sms_current_device();
int set_last_error(int code, const char *msg);   // records msg for ulysses_last_error(); returns code
void clear_last_error();
bool encode_tmap_3d(void *tmap /*CUtensorMap*/, const void *base, int64_t inner, int64_t mid, int64_t outer,
                    int64_t mid_stride_bytes, int64_t outer_stride_bytes, int box_inner, int box_outer,
                    int swizzle_bytes);
// bf16 tensor map of `rank` (<= 5) dimensions, dims innermost first, byte
// strides of dimensions 1..rank-1, box extents per dimension.
bool encode_tmap(void *tmap /*CUtensorMap*/, const void *base, int rank, const int64_t *dims,
                 const int64_t *strides_bytes, const int *box, int swizzle_bytes);

}  // namespace uly
