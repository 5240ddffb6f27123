// api.cu -- the C ABI declared in include/ulysses.h: argument validation,
// workspace sizing, tensor-map encoding and kernel launches. Every argument
// error is reported before anything is launched.
#include "ulysses.h"
#include "ulysses_internal.cuh"

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

namespace uly {

namespace {

thread_local char g_err[512] = "";
int64_t g_wait_limit_ns = 1000000000LL;
uint32_t g_debug_flags = 0;

int fail(int code, const char *fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(cudaError_t e, const char *what)
{
    return fail(ULYSSES_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool head_dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

}  // namespace

int set_last_error(int code, const char *msg) { return fail(code, "%s", msg); }

void clear_last_error() { g_err[0] = 0; }

int num_sms_current_device()
{
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64) {
        if (cache[dev] == 0) {
            int n = 0;
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
            cache[dev] = n > 0 ? n : 148;
        }
        return cache[dev];
    }
    return 148;
}

bool encode_tmap_3d(void *tmap, const void *base, int64_t inner, int64_t mid, int64_t outer, int64_t mid_stride_bytes,
                    int64_t outer_stride_bytes, int box_inner, int box_outer, int swizzle_bytes)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(mid),
                          static_cast<cuuint64_t>(outer)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(mid_stride_bytes), static_cast<cuuint64_t>(outer_stride_bytes)};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), 1u, static_cast<cuuint32_t>(box_outer)};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                            : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                            : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                  : CU_TENSOR_MAP_SWIZZLE_NONE;
    CUresult r = fn(static_cast<CUtensorMap *>(tmap), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base),
                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool encode_tmap(void *tmap, const void *base, int rank, const int64_t *dims, const int64_t *strides_bytes,
                 const int *box, int swizzle_bytes)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn || rank < 1 || rank > 5) return false;
    cuuint64_t d[5], st[4];
    cuuint32_t bx[5], es[5];
    for (int i = 0; i < rank; ++i) {
        d[i] = static_cast<cuuint64_t>(dims[i]);
        bx[i] = static_cast<cuuint32_t>(box[i]);
        es[i] = 1u;
    }
    for (int i = 0; i + 1 < rank; ++i) st[i] = static_cast<cuuint64_t>(strides_bytes[i]);
    CUtensorMapSwizzle sw = swizzle_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                            : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                  : CU_TENSOR_MAP_SWIZZLE_NONE;
    CUresult r = fn(static_cast<CUtensorMap *>(tmap), CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
                    const_cast<void *>(base), d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace uly

using namespace uly;

extern "C" {

const char *ulysses_last_error(void) { return g_err; }

const char *ulysses_version(void) { return "ulysses-b200 0.1 (sm_100a)"; }

void ulysses_set_wait_limit_ns(int64_t ns) { g_wait_limit_ns = ns > 0 ? ns : 1000000000LL; }

void ulysses_set_debug_flags(uint32_t flags) { g_debug_flags = flags; }

static int relayout_common(bool to_head, const void *src, void *dst, int64_t N, int P, int Hx, int d, int rank,
                           int row_heads, int head0, void *stream, const char *name)
{
    g_err[0] = 0;
    if (head0 < 0 || row_heads < head0 + Hx)
        return fail(ULYSSES_ERR_INVALID, "%s: heads [%d, %d) do not fit rows of %d heads", name, head0, head0 + Hx,
                    row_heads);
    if (N < 0) return fail(ULYSSES_ERR_INVALID, "%s: N=%lld < 0", name, (long long)N);
    if (P < 1) return fail(ULYSSES_ERR_INVALID, "%s: P=%d < 1", name, P);
    if (Hx < 1) return fail(ULYSSES_ERR_INVALID, "%s: head count %d < 1", name, Hx);
    if (!head_dim_ok(d)) return fail(ULYSSES_ERR_INVALID, "%s: d=%d not in {32,64,128}", name, d);
    if (Hx % P) return fail(ULYSSES_ERR_INVALID, "%s: heads %d not divisible by P=%d", name, Hx, P);
    if (N % P) return fail(ULYSSES_ERR_INVALID, "%s: N=%lld not divisible by P=%d", name, (long long)N, P);
    if (rank >= P) return fail(ULYSSES_ERR_INVALID, "%s: rank=%d >= P=%d", name, rank, P);
    if (N == 0) return ULYSSES_OK;
    if (!src || !dst) return fail(ULYSSES_ERR_INVALID, "%s: null pointer", name);
    if (!aligned16(src) || !aligned16(dst)) return fail(ULYSSES_ERR_INVALID, "%s: pointers must be 16-byte aligned", name);
    cudaError_t e = launch_relayout(to_head, src, dst, N, P, Hx, d, rank, row_heads, head0,
                                    static_cast<cudaStream_t>(stream), num_sms_current_device());
    if (e != cudaSuccess) return cuda_fail(e, name);
    return ULYSSES_OK;
}

int ulysses_seq_to_head(const void *src, void *dst, int64_t N, int P, int Hx, int d, int rank, void *stream)
{
    return relayout_common(true, src, dst, N, P, Hx, d, rank, Hx, 0, stream, "ulysses_seq_to_head");
}

int ulysses_head_to_seq(const void *src, void *dst, int64_t N, int P, int Hx, int d, int rank, void *stream)
{
    return relayout_common(false, src, dst, N, P, Hx, d, rank, Hx, 0, stream, "ulysses_head_to_seq");
}

int ulysses_seq_to_head_heads(const void *src, void *dst, int64_t N, int P, int Hx, int d, int rank, int row_heads,
                              int head0, void *stream)
{
    return relayout_common(true, src, dst, N, P, Hx, d, rank, row_heads, head0, stream, "ulysses_seq_to_head_heads");
}

int ulysses_head_to_seq_heads(const void *src, void *dst, int64_t N, int P, int Hx, int d, int rank, int row_heads,
                              int head0, void *stream)
{
    return relayout_common(false, src, dst, N, P, Hx, d, rank, row_heads, head0, stream, "ulysses_head_to_seq_heads");
}

size_t ulysses_attn_workspace_bytes(int64_t N, int Hl, int Hkvl, int d, int backward)
{
    (void)Hkvl;
    (void)d;
    if (N < 0 || Hl < 1) return 0;
    return ws_layout(N, Hl, backward != 0).total;
}

static int check_attn_shapes(const char *name, int64_t N, int Hl, int Hkvl, int d)
{
    if (N < 0) return fail(ULYSSES_ERR_INVALID, "%s: N=%lld < 0", name, (long long)N);
    if (N > (int64_t(1) << 31) - 256) return fail(ULYSSES_ERR_UNSUPPORTED, "%s: N=%lld too large", name, (long long)N);
    if (Hl < 1 || Hkvl < 1) return fail(ULYSSES_ERR_INVALID, "%s: head counts must be >= 1", name);
    if (Hl % Hkvl) return fail(ULYSSES_ERR_INVALID, "%s: Hl=%d not divisible by Hkvl=%d", name, Hl, Hkvl);
    if (!head_dim_ok(d)) return fail(ULYSSES_ERR_INVALID, "%s: d=%d not in {32,64,128}", name, d);
    // Work items, CTA counts and the backward's per-row launch are 32-bit: at
    // most Hl * ceil(N/128) * 16 of them (the backward's per-row grid, the
    // largest) may be launched.
    const int64_t T = (N + kTileM - 1) / kTileM;
    if (int64_t(Hl) * T * 16 > INT32_MAX)
        return fail(ULYSSES_ERR_UNSUPPORTED, "%s: Hl * ceil(N/128) = %lld exceeds the 32-bit launch limit of %d",
                    name, (long long)(int64_t(Hl) * T), INT32_MAX / 16);
    return ULYSSES_OK;
}

static int check_ws(const char *name, void *ws, size_t ws_bytes, const WsLayout &L)
{
    if (!ws) return fail(ULYSSES_ERR_WORKSPACE, "%s: workspace is null", name);
    if (!aligned16(ws)) return fail(ULYSSES_ERR_INVALID, "%s: workspace must be 16-byte aligned", name);
    if (ws_bytes < L.total)
        return fail(ULYSSES_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", name, ws_bytes, L.total);
    return ULYSSES_OK;
}

static int attn_fwd_common(const char *name, const void *q, const void *k, const void *v, const int32_t *pos,
                           int64_t N, int Hl, int Hkvl, int d, float scale, void *o, float *lse, void *ws,
                           size_t ws_bytes, void *stream, int Hq_total, int Hkv_total, int q_head0, int kv_head0,
                           int64_t q_lo, int64_t q_hi, int64_t kv_lo, int64_t kv_hi)
{
    WsLayout L = ws_layout(N, Hl, false);
    int rc = check_ws(name, ws, ws_bytes, L);
    if (rc) return rc;
    if (N == 0 || q_hi == q_lo) return ULYSSES_OK;
    if (!q || !k || !v || !pos || !o || !lse) return fail(ULYSSES_ERR_INVALID, "%s: null pointer", name);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
        return fail(ULYSSES_ERR_INVALID, "%s: q, k, v, o must be 16-byte aligned", name);
    if (!aligned4(pos) || !aligned4(lse)) return fail(ULYSSES_ERR_INVALID, "%s: position_ids/lse misaligned", name);
    if (!(scale > 0.f) || !std::isfinite(scale)) scale = 1.0f / std::sqrt(static_cast<float>(d));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    DbWindow win;
    win.q_tile0 = static_cast<int>(q_lo / kTileM);
    win.q_tiles = static_cast<int>(ceil_div(q_hi, kTileM)) - win.q_tile0;
    win.kvlo_t = static_cast<int>(kv_lo / kTileN);
    win.kvhi_t = kv_hi > 0 ? static_cast<int>((kv_hi - 1) / kTileN) : -1;
    cudaError_t e = launch_docbounds(pos, N, static_cast<char *>(ws), L, false, !fwd_pairs_heads(Hl, Hkvl), win, s);
    if (e != cudaSuccess) return cuda_fail(e, name);
    FwdLaunch a;
    a.q = q; a.k = k; a.v = v;
    a.Hq_total = Hq_total; a.Hkv_total = Hkv_total;
    a.q_head0 = q_head0; a.kv_head0 = kv_head0;
    a.o = o; a.Ho_total = Hq_total; a.o_head0 = q_head0;
    a.lse = lse;
    a.N = N; a.Hl = Hl; a.Hkvl = Hkvl; a.d = d;
    a.q_lo = q_lo; a.q_hi = q_hi; a.kv_lo = kv_lo; a.kv_hi = kv_hi;
    a.lse_ld = q_hi - q_lo;
    a.scale = scale;
    a.ws = static_cast<const char *>(ws);
    a.L = L;
    a.wait_limit_ns = static_cast<uint64_t>(g_wait_limit_ns);
    a.debug_flags = g_debug_flags;
    e = launch_attn_fwd(a, s);
    if (e != cudaSuccess) return cuda_fail(e, name);
    return ULYSSES_OK;
}

int ulysses_attn_fwd(const void *q, const void *k, const void *v, const int32_t *position_ids, int64_t N, int Hl,
                     int Hkvl, int d, float scale, void *o, float *lse, void *ws, size_t ws_bytes, void *stream)
{
    g_err[0] = 0;
    int rc = check_attn_shapes("ulysses_attn_fwd", N, Hl, Hkvl, d);
    if (rc) return rc;
    return attn_fwd_common("ulysses_attn_fwd", q, k, v, position_ids, N, Hl, Hkvl, d, scale, o, lse, ws, ws_bytes,
                           stream, Hl, Hkvl, 0, 0, 0, N, 0, N);
}

int ulysses_attn_fwd_window(const void *q, const void *k, const void *v, const int32_t *position_ids, int64_t N,
                            int Hl, int Hkvl, int d, int64_t q_lo, int64_t q_hi, int64_t kv_lo, int64_t kv_hi,
                            float scale, void *o, float *lse, void *ws, size_t ws_bytes, void *stream)
{
    const char *name = "ulysses_attn_fwd_window";
    g_err[0] = 0;
    int rc = check_attn_shapes(name, N, Hl, Hkvl, d);
    if (rc) return rc;
    if (q_lo < 0 || q_hi < q_lo || q_hi > N)
        return fail(ULYSSES_ERR_INVALID, "%s: query window [%lld, %lld) outside [0, %lld]", name, (long long)q_lo,
                    (long long)q_hi, (long long)N);
    if (kv_lo < 0 || kv_hi < kv_lo || kv_hi > N)
        return fail(ULYSSES_ERR_INVALID, "%s: key window [%lld, %lld) outside [0, %lld]", name, (long long)kv_lo,
                    (long long)kv_hi, (long long)N);
    return attn_fwd_common(name, q, k, v, position_ids, N, Hl, Hkvl, d, scale, o, lse, ws, ws_bytes, stream, Hl,
                           Hkvl, 0, 0, q_lo, q_hi, kv_lo, kv_hi);
}

int ulysses_attn_merge(const void *o_parts, const float *lse_parts, int R, int64_t M, int Hl, int d, void *o,
                       float *lse, int64_t lse_ld, void *stream)
{
    const char *name = "ulysses_attn_merge";
    g_err[0] = 0;
    if (R < 1 || R > 64) return fail(ULYSSES_ERR_INVALID, "%s: R=%d outside [1, 64]", name, R);
    if (M < 0 || Hl < 1) return fail(ULYSSES_ERR_INVALID, "%s: M=%lld, Hl=%d", name, (long long)M, Hl);
    if (!head_dim_ok(d)) return fail(ULYSSES_ERR_INVALID, "%s: d=%d not in {32,64,128}", name, d);
    if (lse_ld < M) return fail(ULYSSES_ERR_INVALID, "%s: lse_ld=%lld < M=%lld", name, (long long)lse_ld, (long long)M);
    if (M == 0) return ULYSSES_OK;
    if (!o_parts || !lse_parts || !o || !lse) return fail(ULYSSES_ERR_INVALID, "%s: null pointer", name);
    if (!aligned16(o_parts) || !aligned16(o)) return fail(ULYSSES_ERR_INVALID, "%s: o_parts, o must be 16-byte aligned", name);
    if (!aligned4(lse_parts) || !aligned4(lse)) return fail(ULYSSES_ERR_INVALID, "%s: lse misaligned", name);
    cudaError_t e = launch_attn_merge(o_parts, lse_parts, R, M, Hl, d, o, lse, lse_ld, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, name);
    return ULYSSES_OK;
}

int ulysses_attn_fwd_fused(const void *q_seq, const void *k_seq, const void *v_seq, const int32_t *position_ids,
                           int64_t N, int P, int H, int Hkv, int d, int rank, float scale, void *o_seq, float *lse,
                           void *ws, size_t ws_bytes, void *stream)
{
    const char *name = "ulysses_attn_fwd_fused";
    g_err[0] = 0;
    if (P < 1) return fail(ULYSSES_ERR_INVALID, "%s: P=%d < 1", name, P);
    if (H < 1 || Hkv < 1) return fail(ULYSSES_ERR_INVALID, "%s: head counts must be >= 1", name);
    if (H % P || Hkv % P)
        return fail(ULYSSES_ERR_INVALID, "%s: H=%d and Hkv=%d must be divisible by P=%d", name, H, Hkv, P);
    if (N % P) return fail(ULYSSES_ERR_INVALID, "%s: N=%lld not divisible by P=%d", name, (long long)N, P);
    if (rank < 0 || rank >= P) return fail(ULYSSES_ERR_INVALID, "%s: rank=%d outside [0,%d)", name, rank, P);
    const int Hl = H / P, Hkvl = Hkv / P;
    int rc = check_attn_shapes(name, N, Hl, Hkvl, d);
    if (rc) return rc;
    return attn_fwd_common(name, q_seq, k_seq, v_seq, position_ids, N, Hl, Hkvl, d, scale, o_seq, lse, ws, ws_bytes,
                           stream, H, Hkv, rank * Hl, rank * Hkvl, 0, N, 0, N);
}

// Shared by the slice and the fused (sequence-layout) backward entry points.
static int attn_bwd_common(const char *name, const void *q, const void *k, const void *v, const void *o,
                           const void *dout, const float *lse, const int32_t *position_ids, int64_t N, int Hl,
                           int Hkvl, int d, float scale, void *dq, void *dk, void *dv, void *ws, size_t ws_bytes,
                           void *stream, int Hq_total, int Hkv_total, int q_head0, int kv_head0)
{
    WsLayout L = ws_layout(N, Hl, true);
    int rc = check_ws(name, ws, ws_bytes, L);
    if (rc) return rc;
    if (N == 0) return ULYSSES_OK;
    if (!q || !k || !v || !o || !dout || !lse || !position_ids || !dq || !dk || !dv)
        return fail(ULYSSES_ERR_INVALID, "%s: null pointer", name);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv))
        return fail(ULYSSES_ERR_INVALID, "%s: bf16 tensors must be 16-byte aligned", name);
    if (!aligned4(position_ids) || !aligned4(lse)) return fail(ULYSSES_ERR_INVALID, "%s: position_ids/lse misaligned", name);
    if (!(scale > 0.f) || !std::isfinite(scale)) scale = 1.0f / std::sqrt(static_cast<float>(d));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int T = static_cast<int>(ceil_div(N, kTileM));
    cudaError_t e = launch_docbounds(position_ids, N, static_cast<char *>(ws), L, true, false, DbWindow{0, T, 0, T - 1}, s);
    if (e != cudaSuccess) return cuda_fail(e, name);
    BwdLaunch a;
    a.q = q; a.k = k; a.v = v; a.o = o; a.dout = dout; a.lse = lse;
    a.dq = dq; a.dk = dk; a.dv = dv;
    a.N = N; a.Hl = Hl; a.Hkvl = Hkvl; a.d = d;
    a.Hq_total = Hq_total; a.Hkv_total = Hkv_total;
    a.q_head0 = q_head0; a.kv_head0 = kv_head0;
    a.scale = scale;
    a.ws = static_cast<char *>(ws);
    a.L = L;
    a.wait_limit_ns = static_cast<uint64_t>(g_wait_limit_ns);
    a.debug_flags = g_debug_flags;
    e = launch_attn_bwd(a, s);
    if (e == cudaErrorNotSupported) return fail(ULYSSES_ERR_UNSUPPORTED, "%s: not built", name);
    if (e != cudaSuccess) return cuda_fail(e, name);
    return ULYSSES_OK;
}

int ulysses_attn_bwd(const void *q, const void *k, const void *v, const void *o, const void *dout, const float *lse,
                     const int32_t *position_ids, int64_t N, int Hl, int Hkvl, int d, float scale, void *dq, void *dk,
                     void *dv, void *ws, size_t ws_bytes, void *stream)
{
    const char *name = "ulysses_attn_bwd";
    g_err[0] = 0;
    int rc = check_attn_shapes(name, N, Hl, Hkvl, d);
    if (rc) return rc;
    return attn_bwd_common(name, q, k, v, o, dout, lse, position_ids, N, Hl, Hkvl, d, scale, dq, dk, dv, ws, ws_bytes,
                           stream, Hl, Hkvl, 0, 0);
}

int ulysses_attn_bwd_fused(const void *q_seq, const void *k_seq, const void *v_seq, const void *o_seq,
                           const void *dout_seq, const float *lse, const int32_t *position_ids, int64_t N, int P,
                           int H, int Hkv, int d, int rank, float scale, void *dq_seq, void *dk_seq, void *dv_seq,
                           void *ws, size_t ws_bytes, void *stream)
{
    const char *name = "ulysses_attn_bwd_fused";
    g_err[0] = 0;
    if (P < 1) return fail(ULYSSES_ERR_INVALID, "%s: P=%d < 1", name, P);
    if (H < 1 || Hkv < 1) return fail(ULYSSES_ERR_INVALID, "%s: head counts must be >= 1", name);
    if (H % P || Hkv % P)
        return fail(ULYSSES_ERR_INVALID, "%s: H=%d and Hkv=%d must be divisible by P=%d", name, H, Hkv, P);
    if (N % P) return fail(ULYSSES_ERR_INVALID, "%s: N=%lld not divisible by P=%d", name, (long long)N, P);
    if (rank < 0 || rank >= P) return fail(ULYSSES_ERR_INVALID, "%s: rank=%d outside [0,%d)", name, rank, P);
    const int Hl = H / P, Hkvl = Hkv / P;
    int rc = check_attn_shapes(name, N, Hl, Hkvl, d);
    if (rc) return rc;
    return attn_bwd_common(name, q_seq, k_seq, v_seq, o_seq, dout_seq, lse, position_ids, N, Hl, Hkvl, d, scale,
                           dq_seq, dk_seq, dv_seq, ws, ws_bytes, stream, H, Hkv, rank * Hl, rank * Hkvl);
}

size_t ulysses_proj_workspace_bytes(void) { return 256; }

static int proj_common(const char *name, ProjLaunch &a, void *ws, size_t ws_bytes, void *stream)
{
    if (!ws) return fail(ULYSSES_ERR_WORKSPACE, "%s: workspace is null", name);
    if (!aligned16(ws)) return fail(ULYSSES_ERR_INVALID, "%s: workspace must be 16-byte aligned", name);
    if (ws_bytes < ulysses_proj_workspace_bytes())
        return fail(ULYSSES_ERR_WORKSPACE, "%s: workspace %zu bytes < required %zu", name, ws_bytes,
                    ulysses_proj_workspace_bytes());
    if (a.M == 0) return ULYSSES_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    a.status = static_cast<uint32_t *>(ws);
    a.wait_limit_ns = static_cast<uint64_t>(g_wait_limit_ns);
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(uint32_t), s);   // fresh status word for this call
    if (e != cudaSuccess) return cuda_fail(e, name);
    e = launch_proj_gemm(a, s);
    if (e != cudaSuccess) return cuda_fail(e, name);
    return ULYSSES_OK;
}

static int proj_check_heads(const char *name, int64_t N, int hidden, int P, int H, int Hkv, int d)
{
    if (N < 0 || N > (int64_t(1) << 31) - 256) return fail(ULYSSES_ERR_INVALID, "%s: N=%lld", name, (long long)N);
    if (P < 1 || H < 1 || Hkv < 1) return fail(ULYSSES_ERR_INVALID, "%s: P, H, Hkv must be >= 1", name);
    if (H % P || Hkv % P)
        return fail(ULYSSES_ERR_INVALID, "%s: H=%d and Hkv=%d must be divisible by P=%d", name, H, Hkv, P);
    if (N % P) return fail(ULYSSES_ERR_INVALID, "%s: N=%lld not divisible by P=%d", name, (long long)N, P);
    if (!head_dim_ok(d)) return fail(ULYSSES_ERR_INVALID, "%s: d=%d not in {32,64,128}", name, d);
    if (hidden < 64 || hidden % 64)
        return fail(ULYSSES_ERR_UNSUPPORTED, "%s: hidden=%d must be a positive multiple of 64", name, hidden);
    return ULYSSES_OK;
}

int ulysses_qkv_proj(const void *x, const void *w_qkv, int64_t N, int hidden, int P, int H, int Hkv, int d,
                     void *q_heads, void *k_heads, void *v_heads, void *ws, size_t ws_bytes, void *stream)
{
    const char *name = "ulysses_qkv_proj";
    g_err[0] = 0;
    int rc = proj_check_heads(name, N, hidden, P, H, Hkv, d);
    if (rc) return rc;
    const int64_t nc = int64_t(H + 2 * Hkv) * d;
    if (nc % 128) return fail(ULYSSES_ERR_UNSUPPORTED, "%s: (H+2Hkv)*d=%lld must be a multiple of 128", name, (long long)nc);
    if (N > 0 && (!x || !w_qkv || !q_heads || !k_heads || !v_heads))
        return fail(ULYSSES_ERR_INVALID, "%s: null pointer", name);
    if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q_heads) || !aligned16(k_heads) || !aligned16(v_heads))
        return fail(ULYSSES_ERR_INVALID, "%s: pointers must be 16-byte aligned", name);
    ProjLaunch a{};
    a.A = x; a.B = w_qkv; a.M = N; a.Nc = static_cast<int>(nc); a.K = hidden;
    a.a_heads = 0; a.d = d; a.Hl = H / P; a.P = P;
    a.epi_qkv = 1; a.H = H; a.Hkv = Hkv;
    a.out0 = q_heads; a.out1 = k_heads; a.out2 = v_heads;
    return proj_common(name, a, ws, ws_bytes, stream);
}

int ulysses_out_proj(const void *o_heads, const void *w_o, int64_t N, int hidden, int P, int H, int d, void *y,
                     void *ws, size_t ws_bytes, void *stream)
{
    const char *name = "ulysses_out_proj";
    g_err[0] = 0;
    int rc = proj_check_heads(name, N, hidden, P, H, P, d);
    if (rc) return rc;
    if (d < 64) return fail(ULYSSES_ERR_UNSUPPORTED, "%s: d=%d: the head-slice operand needs d >= 64", name, d);
    if (hidden % 128) return fail(ULYSSES_ERR_UNSUPPORTED, "%s: hidden=%d must be a multiple of 128", name, hidden);
    if (N > 0 && (!o_heads || !w_o || !y)) return fail(ULYSSES_ERR_INVALID, "%s: null pointer", name);
    if (!aligned16(o_heads) || !aligned16(w_o) || !aligned16(y))
        return fail(ULYSSES_ERR_INVALID, "%s: pointers must be 16-byte aligned", name);
    ProjLaunch a{};
    a.A = o_heads; a.B = w_o; a.M = N; a.Nc = hidden; a.K = H * d;
    a.a_heads = 1; a.d = d; a.Hl = H / P; a.P = P;
    a.epi_qkv = 0; a.H = H; a.Hkv = H;
    a.out0 = y;
    return proj_common(name, a, ws, ws_bytes, stream);
}

int ulysses_sync_status(void *ws, void *stream)
{
    g_err[0] = 0;
    if (!ws) return fail(ULYSSES_ERR_WORKSPACE, "ulysses_sync_status: workspace is null");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "ulysses_sync_status");
    uint32_t st = 0;
    e = cudaMemcpy(&st, ws, sizeof st, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "ulysses_sync_status");
    if (st & kStatusTimeoutHost) {
        const uint32_t zero = 0;
        cudaMemcpy(ws, &zero, sizeof zero, cudaMemcpyHostToDevice);
        return fail(ULYSSES_ERR_TIMEOUT, "a bounded device-side wait ran out");
    }
    return ULYSSES_OK;
}

}  // extern "C"
