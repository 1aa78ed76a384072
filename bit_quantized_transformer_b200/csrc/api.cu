// C ABI of libvox: argument validation (before any launch) and dispatch to
// the kernels.  See include/vox.h for the contract of every entry point.
#include <string.h>

#include "vox_internal.cuh"

namespace vox {
const char* last_error_text();
vox_status launch_q4_pack(const uint8_t*, int64_t, int64_t, int, uint8_t*, cudaStream_t);
vox_status launch_q4_dequant(const uint8_t*, int64_t, int64_t, int64_t, const int32_t*, int64_t, void*, int,
                             int64_t, cudaStream_t, int gather = 0);
vox_status launch_q4_gemv(const uint8_t*, int64_t, int64_t, const float*, int64_t, int64_t, float*, int64_t,
                          const vox_epilogue*, void*, cudaStream_t);
size_t gemv_workspace_bytes(int64_t n, int64_t k, int op);
vox_status launch_q4_gemm(const uint8_t*, int64_t, int64_t, const void*, int64_t, int64_t, void*, int, int64_t,
                          const vox_epilogue*, cudaStream_t);
vox_status launch_kv_append(void*, void*, const void*, const void*, int, int, int, int, int64_t, const int64_t*,
                            cudaStream_t);
vox_status launch_gqa_decode_attn(const float*, const void*, const void*, float*, int, int, int, int, int64_t,
                                  const int64_t*, float, void*, cudaStream_t);
size_t attn_workspace_bytes(int n_kv, int hd, int window, int n_seq = 1);
vox_status launch_gqa_decode_attn_seqs(const float*, const void*, const void*, float*, int, int, int, int, int64_t,
                                       const int64_t*, float, void*, cudaStream_t, int, const int32_t*, int64_t,
                                       int64_t);
vox_status launch_window_attn(const void*, int64_t, const void*, const void*, int64_t, int64_t, const void*,
                              const void*, int64_t, int64_t, void*, int, int64_t, int, int, int, float,
                              cudaStream_t);
vox_status launch_rmsnorm(const float*, int64_t, int64_t, int64_t, float, const float*, void*, int, int64_t,
                          cudaStream_t);
vox_status launch_cast_rows(const float*, int64_t, int64_t, int64_t, void*, int, int64_t, cudaStream_t);
}  // namespace vox

using namespace vox;

namespace {
inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t S(void* s) { return static_cast<cudaStream_t>(s); }
constexpr int kGemvMaxM = 8;
constexpr int64_t kGemvMaxMK = 81920;
}  // namespace

extern "C" {

const char* vox_status_str(vox_status s)
{
    switch (s) {
    case VOX_OK: return "VOX_OK";
    case VOX_ERR_NULL: return "VOX_ERR_NULL";
    case VOX_ERR_SHAPE: return "VOX_ERR_SHAPE";
    case VOX_ERR_ALIGN: return "VOX_ERR_ALIGN";
    case VOX_ERR_DTYPE: return "VOX_ERR_DTYPE";
    case VOX_ERR_RANGE: return "VOX_ERR_RANGE";
    case VOX_ERR_WORKSPACE: return "VOX_ERR_WORKSPACE";
    case VOX_ERR_TIMEOUT: return "VOX_ERR_TIMEOUT";
    case VOX_ERR_CUDA: return "VOX_ERR_CUDA";
    default: return "VOX_ERR_UNKNOWN";
    }
}

const char* vox_last_error(void) { return last_error_text(); }

int64_t vox_q4_packed_bytes(int64_t n, int64_t k)
{
    if (n < 1 || k < 32 || k % 32) return -1;
    return ceil_div(n, 16) * ceil_div(k, 64) * kChunkBytes;
}

vox_status vox_q4_pack(const void* gguf, int64_t n, int64_t k, int32_t flags, void* packed, void* stream)
{
    if (!gguf || !packed) return VOX_ERR_NULL;
    if (n < 1 || k < 32 || k % 32) return VOX_ERR_SHAPE;
    if (flags != VOX_PACK_PLAIN && flags != VOX_PACK_GATE_UP) return VOX_ERR_RANGE;
    if (flags == VOX_PACK_GATE_UP && (n % 16)) return VOX_ERR_SHAPE;   // n = 2F, F % 8 == 0
    if (!al16(packed)) return VOX_ERR_ALIGN;
    return launch_q4_pack(static_cast<const uint8_t*>(gguf), n, k, flags == VOX_PACK_GATE_UP,
                          static_cast<uint8_t*>(packed), S(stream));
}

static vox_status check_weight(const vox_q4_weight* w)
{
    if (!w || !w->data) return VOX_ERR_NULL;
    if (w->n < 1 || w->k < 32 || w->k % 32) return VOX_ERR_SHAPE;
    if (!al16(w->data)) return VOX_ERR_ALIGN;
    return VOX_OK;
}

vox_status vox_q4_dequant(const vox_q4_weight* w, int64_t row0, int64_t nrows, void* out, int32_t out_dtype,
                          int64_t ldo, void* stream)
{
    vox_status st = check_weight(w);
    if (st) return st;
    if (!out) return VOX_ERR_NULL;
    if (out_dtype != VOX_F32 && out_dtype != VOX_BF16) return VOX_ERR_DTYPE;
    if (nrows < 1 || row0 < 0 || row0 + nrows > w->n) return VOX_ERR_RANGE;
    if (ldo < w->k) return VOX_ERR_SHAPE;
    return launch_q4_dequant(static_cast<const uint8_t*>(w->data), w->n, w->k, row0, nullptr, nrows, out,
                             out_dtype, ldo, S(stream));
}

static vox_status check_epilogue(const vox_epilogue* ep, int64_t n, int64_t k, int64_t m, int64_t ldy,
                                 bool allow_rms, bool gemm)
{
    int op = ep ? ep->op : VOX_EP_NONE;
    if (op < VOX_EP_NONE || op > VOX_EP_KV_APPEND_PAGED) return VOX_ERR_RANGE;
    if (ep && ep->rmsnorm && !allow_rms) return VOX_ERR_RANGE;
    if (ep && ep->rmsnorm && !(ep->eps >= 0.f)) return VOX_ERR_RANGE;
    if (ep && ep->rope_theta != 0.f) {
        if (op != VOX_EP_KV_APPEND && op != VOX_EP_KV_APPEND_PAGED) return VOX_ERR_RANGE;
        if (!(ep->rope_theta > 0.f) || ep->rope_theta > 3.0e38f) return VOX_ERR_RANGE;
        if (ep->head_dim % 16 || ep->head_dim < 16 || ep->q_rows % ep->head_dim) return VOX_ERR_RANGE;
    }
    int64_t ncols = op == VOX_EP_SILU_MUL ? n / 2 : n;
    if (ldy < ncols) return VOX_ERR_SHAPE;
    (void)k;
    switch (op) {
    case VOX_EP_RESIDUAL:
        if (!ep->residual) return VOX_ERR_NULL;
        if (ep->ldr < n) return VOX_ERR_SHAPE;
        break;
    case VOX_EP_SILU_MUL:
        if (n % 16) return VOX_ERR_SHAPE;
        break;
    case VOX_EP_KV_APPEND:
        if (gemm) return VOX_ERR_RANGE;
        if (!ep->k_cache || !ep->v_cache) return VOX_ERR_NULL;
        if (ep->n_kv_heads < 1 || ep->head_dim < 1 || ep->q_rows < 0) return VOX_ERR_SHAPE;
        if ((int64_t)ep->q_rows + 2LL * ep->n_kv_heads * ep->head_dim > n) return VOX_ERR_SHAPE;
        if (ep->window < 1 || (!ep->pos_dev && ep->pos < 0)) return VOX_ERR_RANGE;
        break;
    case VOX_EP_KV_APPEND_PAGED:
        if (gemm) return VOX_ERR_RANGE;
        if (!ep->k_cache || !ep->v_cache || !ep->page_table || !ep->pos_dev) return VOX_ERR_NULL;
        if (ep->n_kv_heads < 1 || ep->head_dim < 1 || ep->q_rows < 0) return VOX_ERR_SHAPE;
        if ((int64_t)ep->q_rows + 2LL * ep->n_kv_heads * ep->head_dim > n) return VOX_ERR_SHAPE;
        if (ep->window < 64 || ep->window % 64 || ep->n_pages < 1) return VOX_ERR_RANGE;
        break;
    case VOX_EP_ARGMAX:
        if (gemm) return VOX_ERR_RANGE;
        if (!ep->argmax) return VOX_ERR_NULL;
        if (n > 0x7ffffff0LL) return VOX_ERR_SHAPE;
        break;
    default:
        break;
    }
    (void)m;
    return VOX_OK;
}

size_t vox_q4_gemv_workspace(const vox_q4_weight* w, int64_t m, const vox_epilogue* ep)
{
    (void)m;
    if (!w || w->n < 1) return 0;
    return gemv_workspace_bytes(w->n, w->k, ep ? ep->op : VOX_EP_NONE);
}

vox_status vox_q4_gemv(const vox_q4_weight* w, const float* x, int64_t m, int64_t ldx, float* y, int64_t ldy,
                       const vox_epilogue* ep, void* workspace, size_t ws_bytes, void* stream)
{
    vox_status st = check_weight(w);
    if (st) return st;
    if (!x || !y) return VOX_ERR_NULL;
    if (m < 1 || m > kGemvMaxM) return VOX_ERR_SHAPE;
    if (ldx < w->k) return VOX_ERR_SHAPE;
    if (m * ceil_div(w->k, 64) * 64 > kGemvMaxMK) return VOX_ERR_SHAPE;
    if ((st = check_epilogue(ep, w->n, w->k, m, ldy, true, false))) return st;
    if (!workspace) return VOX_ERR_WORKSPACE;
    if (ws_bytes < vox_q4_gemv_workspace(w, m, ep)) return VOX_ERR_WORKSPACE;
    if (!al16(workspace)) return VOX_ERR_ALIGN;
    return launch_q4_gemv(static_cast<const uint8_t*>(w->data), w->n, w->k, x, m, ldx, y, ldy, ep, workspace,
                          S(stream));
}

vox_status vox_q4_gemm(const vox_q4_weight* w, const void* x, int32_t x_dtype, int64_t m, int64_t ldx, void* y,
                       int32_t y_dtype, int64_t ldy, const vox_epilogue* ep, void* stream)
{
    vox_status st = check_weight(w);
    if (st) return st;
    if (!x || !y) return VOX_ERR_NULL;
    if (x_dtype != VOX_BF16) return VOX_ERR_DTYPE;
    if (y_dtype != VOX_F32 && y_dtype != VOX_BF16) return VOX_ERR_DTYPE;
    if (m < 1 || m > (1LL << 30) || w->k % 64) return VOX_ERR_SHAPE;
    if (ldx < w->k || ldx % 8) return VOX_ERR_SHAPE;
    if (!al16(x)) return VOX_ERR_ALIGN;
    if ((st = check_epilogue(ep, w->n, w->k, m, ldy, false, true))) return st;
    if (ep && ep->op == VOX_EP_SILU_MUL) return VOX_ERR_RANGE;
    if (ep && ep->op == VOX_EP_RESIDUAL && y_dtype != VOX_F32) return VOX_ERR_DTYPE;
    return launch_q4_gemm(static_cast<const uint8_t*>(w->data), w->n, w->k, x, m, ldx, y, y_dtype, ldy, ep,
                          S(stream));
}

// Largest m that vox_q4_matmul runs on the GEMV: on B200 the tcgen05 GEMM at
// m = 16 beat two m = 8 GEMV launches on four of the decoder's five shapes.
constexpr int64_t kMatmulGemvMaxM = 8;

size_t vox_q4_matmul_workspace(const vox_q4_weight* w, int64_t m, const vox_epilogue* ep)
{
    if (!w || w->n < 1 || w->k < 32 || m < 1) return 0;
    const size_t g = (vox_q4_gemv_workspace(w, m < kMatmulGemvMaxM ? m : kMatmulGemvMaxM, ep) + 255) & ~(size_t)255;
    if (m <= kMatmulGemvMaxM) return g;
    return g + (((size_t)m * (size_t)w->k * 2 + 255) & ~(size_t)255);
}

vox_status vox_q4_matmul(const vox_q4_weight* w, const float* x, int64_t m, int64_t ldx, float* y, int64_t ldy,
                         const vox_epilogue* ep, void* workspace, size_t ws_bytes, void* stream)
{
    if (m >= 1 && m <= kMatmulGemvMaxM) return vox_q4_gemv(w, x, m, ldx, y, ldy, ep, workspace, ws_bytes, stream);
    vox_status st = check_weight(w);
    if (st) return st;
    if (!x || !y) return VOX_ERR_NULL;
    if (m < 1 || m > (1LL << 30) || w->k % 64 || ldx < w->k) return VOX_ERR_SHAPE;
    const int op = ep ? ep->op : VOX_EP_NONE;
    if (op != VOX_EP_NONE && op != VOX_EP_RESIDUAL && op != VOX_EP_GELU) return VOX_ERR_RANGE;
    if (ep && ep->rmsnorm && !(ep->eps >= 0.f)) return VOX_ERR_RANGE;
    if (!workspace) return VOX_ERR_WORKSPACE;
    if (ws_bytes < vox_q4_matmul_workspace(w, m, ep)) return VOX_ERR_WORKSPACE;
    if (!al16(workspace)) return VOX_ERR_ALIGN;
    if ((st = check_epilogue(ep, w->n, w->k, m, ldy, true, true))) return st;
    // x (normalised first if asked) -> bf16 rows in the workspace, then the GEMM
    uint8_t* xb = static_cast<uint8_t*>(workspace) + ((vox_q4_gemv_workspace(w, kMatmulGemvMaxM, ep) + 255) & ~(size_t)255);
    st = (ep && ep->rmsnorm) ? launch_rmsnorm(x, m, w->k, ldx, ep->eps, ep->norm_weight, xb, VOX_BF16, w->k, S(stream))
                             : launch_cast_rows(x, m, w->k, ldx, xb, VOX_BF16, w->k, S(stream));
    if (st) return st;
    vox_epilogue e2 = {};
    if (ep) {
        e2 = *ep;
        e2.rmsnorm = 0;
    }
    return launch_q4_gemm(static_cast<const uint8_t*>(w->data), w->n, w->k, xb, m, w->k, y, VOX_F32, ldy,
                          ep ? &e2 : nullptr, S(stream));
}

vox_status vox_kv_append_rolling(void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                                 int32_t new_dtype, int32_t n_kv_heads, int32_t head_dim, int32_t window, int64_t pos,
                                 void* stream)
{
    if (!k_cache || !v_cache || !k_new || !v_new) return VOX_ERR_NULL;
    if (new_dtype != VOX_F32 && new_dtype != VOX_BF16) return VOX_ERR_DTYPE;
    if (n_kv_heads < 1 || head_dim < 1 || head_dim > 1024) return VOX_ERR_SHAPE;
    if (window < 1 || pos < 0) return VOX_ERR_RANGE;
    return launch_kv_append(k_cache, v_cache, k_new, v_new, new_dtype, n_kv_heads, head_dim, window, pos, nullptr,
                            S(stream));
}

size_t vox_gqa_decode_attn_workspace(int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int32_t window)
{
    if (n_q_heads < 1 || n_kv_heads < 1 || head_dim < 1 || window < 1) return 0;
    return attn_workspace_bytes(n_kv_heads, head_dim, window);
}

vox_status vox_gqa_decode_attn(const float* q, const void* k_cache, const void* v_cache, float* out,
                               int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int32_t window, int64_t pos,
                               float scale, void* workspace, size_t ws_bytes, void* stream)
{
    if (!q || !k_cache || !v_cache || !out) return VOX_ERR_NULL;
    if (n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return VOX_ERR_RANGE;
    if (n_q_heads / n_kv_heads > 8 || n_kv_heads > 512) return VOX_ERR_RANGE;
    if (window < 1 || pos < 0) return VOX_ERR_RANGE;
    if (head_dim != 128) return VOX_ERR_SHAPE;
    if ((int64_t)n_kv_heads * window > 0x7fffff00LL) return VOX_ERR_SHAPE;
    if (!workspace) return VOX_ERR_WORKSPACE;
    if (ws_bytes < vox_gqa_decode_attn_workspace(n_q_heads, n_kv_heads, head_dim, window)) return VOX_ERR_WORKSPACE;
    if (!al16(k_cache) || !al16(v_cache) || !al16(workspace) || !al16(out)) return VOX_ERR_ALIGN;
    return launch_gqa_decode_attn(q, k_cache, v_cache, out, n_q_heads, n_kv_heads, head_dim, window, pos, nullptr,
                                  scale, workspace, S(stream));
}

size_t vox_gqa_decode_attn_paged_workspace(int32_t n_seq, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                           int32_t window)
{
    if (n_seq < 1 || n_q_heads < 1 || n_kv_heads < 1 || head_dim < 1 || window < 1) return 0;
    return attn_workspace_bytes(n_kv_heads, head_dim, window, n_seq);
}

vox_status vox_gqa_decode_attn_paged(const float* q, const void* k_pool, const void* v_pool, int64_t n_pages,
                                     const int32_t* page_table, const int64_t* pos, int32_t n_seq, float* out,
                                     int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int32_t window,
                                     float scale, void* workspace, size_t ws_bytes, void* stream)
{
    if (!q || !k_pool || !v_pool || !page_table || !pos || !out) return VOX_ERR_NULL;
    if (n_seq < 1 || n_seq > 64) return VOX_ERR_RANGE;
    if (n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return VOX_ERR_RANGE;
    if (n_q_heads / n_kv_heads > 8 || n_kv_heads > 512) return VOX_ERR_RANGE;
    if (window < 64 || window % 64 || n_pages < 1) return VOX_ERR_RANGE;
    if (head_dim != 128) return VOX_ERR_SHAPE;
    if (n_pages > 0x7fffff00LL / (64LL * n_kv_heads)) return VOX_ERR_SHAPE;
    if (!workspace) return VOX_ERR_WORKSPACE;
    if (ws_bytes < vox_gqa_decode_attn_paged_workspace(n_seq, n_q_heads, n_kv_heads, head_dim, window))
        return VOX_ERR_WORKSPACE;
    if (!al16(k_pool) || !al16(v_pool) || !al16(workspace) || !al16(out)) return VOX_ERR_ALIGN;
    return launch_gqa_decode_attn_seqs(q, k_pool, v_pool, out, n_q_heads, n_kv_heads, head_dim, window, 0, pos, scale,
                                       workspace, S(stream), n_seq, page_table, n_pages, 0);
}

vox_status vox_window_attn(const void* q, int64_t ldq, const void* k_hist, const void* v_hist, int64_t ld_hist,
                           int64_t n_hist, const void* k_new, const void* v_new, int64_t ld_new, int64_t n_q,
                           void* out, int32_t out_dtype, int64_t ldo, int32_t n_heads, int32_t head_dim,
                           int32_t window, float scale, void* stream)
{
    if (!q || !k_new || !v_new || !out) return VOX_ERR_NULL;
    if (n_hist > 0 && (!k_hist || !v_hist)) return VOX_ERR_NULL;
    if (out_dtype != VOX_F32 && out_dtype != VOX_BF16) return VOX_ERR_DTYPE;
    if (window < 1 || n_hist < 0) return VOX_ERR_RANGE;
    if (n_q < 1 || n_heads < 1 || head_dim < 1 || head_dim > 64) return VOX_ERR_SHAPE;
    const int64_t D = (int64_t)n_heads * head_dim;
    if (ldq < D || ld_new < D || ldo < D || (n_hist > 0 && ld_hist < D)) return VOX_ERR_SHAPE;
    return launch_window_attn(q, ldq, k_hist, v_hist, ld_hist, n_hist, k_new, v_new, ld_new, n_q, out, out_dtype,
                              ldo, n_heads, head_dim, window, scale, S(stream));
}

vox_status vox_rmsnorm(const float* x, int64_t m, int64_t n, int64_t ldx, float eps, const float* g, void* out,
                       int32_t out_dtype, int64_t ldo, void* stream)
{
    if (!x || !out) return VOX_ERR_NULL;
    if (out_dtype != VOX_F32 && out_dtype != VOX_BF16) return VOX_ERR_DTYPE;
    if (m < 1 || n < 1 || ldx < n || ldo < n || m > 0x7fffffffLL) return VOX_ERR_SHAPE;
    if (!(eps >= 0.f)) return VOX_ERR_RANGE;
    return launch_rmsnorm(x, m, n, ldx, eps, g, out, out_dtype, ldo, S(stream));
}

int32_t vox_device_status(int32_t clear)
{
    int32_t v = 0;
    if (cudaMemcpyFromSymbol(&v, g_vox_device_status, sizeof(v)) != cudaSuccess) return -1;
    if (clear) {
        int32_t z = 0;
        cudaMemcpyToSymbol(g_vox_device_status, &z, sizeof(z));
    }
    return v;
}

}  // extern "C"
