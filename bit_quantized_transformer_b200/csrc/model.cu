// Composed hot path: the greedy decoder token step and the encoder chunk,
// each a fixed sequence of launches on one stream (capturable as one CUDA
// graph: the pages' "one submission per token step", voxtral.c page,
// "성능 벤치마크").
//
// Decoder layer (voxtral.c page, "모델 아키텍처": 26 layers, dim 3072, GQA
// 32/8; readings: pre-norm RMSNorm, SwiGLU FFN, no RoPE):
//   x -> [RMSNorm + QKV GEMV + rolling append] -> q
//     -> GQA decode attention -> o
//     -> [Wo GEMV + residual x] -> h
//     -> [RMSNorm + W1||W3 GEMV + SiLU*mul] -> a
//     -> [W2 GEMV + residual h] -> x
// Step: x = embedding[token]; 26 layers; [RMSNorm + LM head GEMV + argmax]
// -> token; pos += 1.  The token and position live in device memory so a
// captured step can be replayed for consecutive tokens.
//
// Encoder layer (same page: 32 causal layers, dim 1280, 32 heads, window
// 750; readings: RMSNorm pre-norm, ungated GELU FFN):
//   xn = RMSNorm(x) (bf16) -> QKV GEMM -> window attention -> O GEMM + x
//   -> RMSNorm -> up GEMM + GELU -> down GEMM + x.  Then the 4x downsample
//   (rows 4r..4r+3 side by side = a [rows/4][4 dim] view) and the adapter:
//   GEMM 5120 -> 3072 + GELU (bf16), GEMM 3072 -> 3072.
#include "vox_internal.cuh"

namespace vox {
vox_status launch_q4_dequant(const uint8_t*, int64_t, int64_t, int64_t, const int32_t*, int64_t, void*, int,
                             int64_t, cudaStream_t, int gather = 0);
vox_status launch_q4_gemv(const uint8_t*, int64_t, int64_t, const float*, int64_t, int64_t, float*, int64_t,
                          const vox_epilogue*, void*, cudaStream_t);
size_t gemv_workspace_bytes(int64_t n, int64_t k, int op);
vox_status launch_gqa_decode_attn(const float*, const void*, const void*, float*, int, int, int, int, int64_t,
                                  const int64_t*, float, void*, cudaStream_t);
size_t attn_workspace_bytes(int n_kv, int hd, int window, int n_seq = 1);
vox_status launch_gqa_decode_attn_seqs(const float*, const void*, const void*, float*, int, int, int, int, int64_t,
                                       const int64_t*, float, void*, cudaStream_t, int, const int32_t*, int64_t,
                                       int64_t);
vox_status launch_advance_pos(int64_t*, cudaStream_t, int n = 1);
vox_status launch_hist_roll(const void*, int64_t, const void*, int64_t, int64_t, int64_t, int64_t, void*, int64_t,
                            cudaStream_t);
vox_status launch_rmsnorm(const float*, int64_t, int64_t, int64_t, float, const float*, void*, int, int64_t,
                          cudaStream_t);
vox_status launch_cast_rows(const float*, int64_t, int64_t, int64_t, void*, int, int64_t, cudaStream_t);
vox_status launch_q4_gemm(const uint8_t*, int64_t, int64_t, const void*, int64_t, int64_t, void*, int, int64_t,
                          const vox_epilogue*, cudaStream_t);
vox_status launch_window_attn(const void*, int64_t, const void*, const void*, int64_t, int64_t, const void*,
                              const void*, int64_t, int64_t, void*, int, int64_t, int, int, int, float,
                              cudaStream_t);
size_t decoder_step_ws_bytes(int n_layers, int n_kv, int group);
const char* decoder_step_unsupported(const vox_decoder* d);
bool decoder_step_fits(const vox_decoder* d);
vox_status launch_decoder_step(const vox_decoder* d, uint8_t* ws, cudaStream_t s, int ph_begin = 0, int ph_end = -1);
void set_error_text(const char* text);
}  // namespace vox

using namespace vox;

extern "C" size_t vox_decoder_workspace(const vox_decoder* d);

namespace {
inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t dec_gemv_ws(const vox_decoder* d)
{
    return gemv_workspace_bytes(d->vocab, d->dim, VOX_EP_ARGMAX) > gemv_workspace_bytes(2 * (int64_t)d->ffn, d->dim, 0)
               ? gemv_workspace_bytes(d->vocab, d->dim, VOX_EP_ARGMAX)
               : gemv_workspace_bytes(2 * (int64_t)d->ffn, d->dim, 0);
}

vox_status check_w(const vox_q4_weight& w, int64_t n, int64_t k)
{
    if (!w.data) return VOX_ERR_NULL;
    if (w.n != n || w.k != k) return VOX_ERR_SHAPE;
    if (!al16(w.data)) return VOX_ERR_ALIGN;
    return VOX_OK;
}

// Offset of the persistent step's part of the decoder workspace (after the
// per-kernel sequence's GEMV and attention parts).
size_t dec_ps_offset(const vox_decoder* d)
{
    const size_t g = (dec_gemv_ws(d) + 255) & ~(size_t)255;
    return g + ((attn_workspace_bytes(d->n_kv_heads, d->head_dim, d->window) + 255) & ~(size_t)255);
}

// Host-side checks shared by both forms of the decoder step (and, without
// the workspace size, by the batched step).
vox_status check_decoder(const vox_decoder* d, bool check_ws = true)
{
    if (!d) return VOX_ERR_NULL;
    if (!d->wqkv || !d->wo || !d->w13 || !d->w2 || !d->k_cache || !d->v_cache || !d->token || !d->pos || !d->x ||
        !d->h || !d->qkv || !d->attn || !d->act || !d->logits || !d->workspace)
        return VOX_ERR_NULL;
    if (d->n_layers < 1 || d->head_dim != 128 || d->n_kv_heads < 1 || d->n_q_heads % d->n_kv_heads ||
        d->n_q_heads / d->n_kv_heads > 8 || d->dim % 32 || d->ffn % 32 || d->ffn % 8)
        return VOX_ERR_SHAPE;
    if (d->window < 1) return VOX_ERR_RANGE;
    if (!(d->rope_theta >= 0.f) || d->rope_theta > 3.0e38f) return VOX_ERR_RANGE;
    if (check_ws && d->ws_bytes < vox_decoder_workspace(d)) return VOX_ERR_WORKSPACE;
    if (!al16(d->workspace)) return VOX_ERR_ALIGN;
    const int64_t D = d->dim, QD = (int64_t)d->n_q_heads * d->head_dim, KVD = (int64_t)d->n_kv_heads * d->head_dim;
    const int64_t F = d->ffn;
    if (QD > 81920 || F > 81920) return VOX_ERR_SHAPE;
    if ((int64_t)d->n_kv_heads * d->window > 0x7fffff00LL) return VOX_ERR_SHAPE;
    if (!al16(d->x) || !al16(d->h) || !al16(d->qkv) || !al16(d->attn) || !al16(d->act) || !al16(d->logits))
        return VOX_ERR_ALIGN;
    vox_status st;
    for (int l = 0; l < d->n_layers; ++l) {
        if ((st = check_w(d->wqkv[l], QD + 2 * KVD, D))) return st;
        if ((st = check_w(d->wo[l], D, QD))) return st;
        if ((st = check_w(d->w13[l], 2 * F, D))) return st;
        if ((st = check_w(d->w2[l], D, F))) return st;
        if (!d->k_cache[l] || !d->v_cache[l]) return VOX_ERR_NULL;
        if (!al16(d->k_cache[l]) || !al16(d->v_cache[l])) return VOX_ERR_ALIGN;
    }
    if ((st = check_w(d->embedding, d->vocab, D))) return st;
    if ((st = check_w(d->lm_head, d->vocab, D))) return st;
    return VOX_OK;
}
}  // namespace

extern "C" {

size_t vox_decoder_workspace(const vox_decoder* d)
{
    if (!d || d->dim < 32 || d->vocab < 1 || d->n_kv_heads < 1 || d->window < 1 || d->n_layers < 1 ||
        d->n_q_heads < d->n_kv_heads)
        return 0;
    return dec_ps_offset(d) + decoder_step_ws_bytes(d->n_layers, d->n_kv_heads, d->n_q_heads / d->n_kv_heads);
}

vox_status vox_decoder_step(const vox_decoder* d, void* stream)
{
    vox_status st = check_decoder(d);
    if (st) return st;
    if (const char* why = decoder_step_unsupported(d)) {
        set_error_text(why);
        return VOX_ERR_SHAPE;
    }
    if (!decoder_step_fits(d)) {
        set_error_text("the activations of the widest projection do not fit shared memory");
        return VOX_ERR_SHAPE;
    }
    return launch_decoder_step(d, static_cast<uint8_t*>(d->workspace) + dec_ps_offset(d),
                               static_cast<cudaStream_t>(stream));
}

vox_status vox_decoder_step_fused(const vox_decoder* d, void* stream)
{
    vox_status st = check_decoder(d);
    if (st) return st;
    if (const char* why = decoder_step_unsupported(d)) {
        set_error_text(why);
        return VOX_ERR_SHAPE;
    }
    if (!decoder_step_fits(d)) {
        set_error_text("the activations of the widest projection do not fit shared memory");
        return VOX_ERR_SHAPE;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws_g = static_cast<uint8_t*>(d->workspace);
    uint8_t* ws_a = ws_g + ((dec_gemv_ws(d) + 255) & ~(size_t)255);
    uint8_t* ws_p = ws_g + dec_ps_offset(d);
    const float scale = 1.0f / sqrtf((float)d->head_dim);
    const int L = d->n_layers;
    // layer 0's QKV (from the embedding row), then per layer the attention and
    // one persistent launch for Wo, W1||W3, W2 and the next QKV (the LM head
    // and the position advance after the last layer)
    if ((st = launch_decoder_step(d, ws_p, s, 0, 1))) return st;
    for (int l = 0; l < L; ++l) {
        if ((st = launch_gqa_decode_attn(d->qkv, d->k_cache[l], d->v_cache[l], d->attn, d->n_q_heads, d->n_kv_heads,
                                         d->head_dim, d->window, 0, d->pos, scale, ws_a, s)))
            return st;
        if ((st = launch_decoder_step(d, ws_p, s, 5 * l + 2, l == L - 1 ? 5 * L + 1 : 5 * l + 6))) return st;
    }
    return VOX_OK;
}

vox_status vox_decoder_step_kernels(const vox_decoder* d, void* stream)
{
    vox_status st = check_decoder(d);
    if (st) return st;
    const int64_t D = d->dim, QD = (int64_t)d->n_q_heads * d->head_dim, KVD = (int64_t)d->n_kv_heads * d->head_dim;
    const int64_t F = d->ffn;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws_g = static_cast<uint8_t*>(d->workspace);
    uint8_t* ws_a = ws_g + ((dec_gemv_ws(d) + 255) & ~(size_t)255);
    const float scale = 1.0f / sqrtf((float)d->head_dim);


    // x = embedding row of the token (exact fp32 weights)
    if ((st = launch_q4_dequant(static_cast<const uint8_t*>(d->embedding.data), d->vocab, D, 0, d->token, 1, d->x,
                                VOX_F32, D, s)))
        return st;
    for (int l = 0; l < d->n_layers; ++l) {
        vox_epilogue e = {};
        e.op = VOX_EP_KV_APPEND;
        e.rmsnorm = 1;
        e.eps = d->eps;
        e.k_cache = d->k_cache[l];
        e.v_cache = d->v_cache[l];
        e.n_kv_heads = d->n_kv_heads;
        e.head_dim = d->head_dim;
        e.window = d->window;
        e.q_rows = (int32_t)QD;
        e.pos_dev = d->pos;
        e.rope_theta = d->rope_theta;
        if ((st = launch_q4_gemv(static_cast<const uint8_t*>(d->wqkv[l].data), QD + 2 * KVD, D, d->x, 1, D, d->qkv,
                                 QD + 2 * KVD, &e, ws_g, s)))
            return st;
        if ((st = launch_gqa_decode_attn(d->qkv, d->k_cache[l], d->v_cache[l], d->attn, d->n_q_heads, d->n_kv_heads,
                                         d->head_dim, d->window, 0, d->pos, scale, ws_a, s)))
            return st;
        vox_epilogue r = {};
        r.op = VOX_EP_RESIDUAL;
        r.residual = d->x;
        r.ldr = D;
        if ((st = launch_q4_gemv(static_cast<const uint8_t*>(d->wo[l].data), D, QD, d->attn, 1, QD, d->h, D, &r, ws_g,
                                 s)))
            return st;
        vox_epilogue f = {};
        f.op = VOX_EP_SILU_MUL;
        f.rmsnorm = 1;
        f.eps = d->eps;
        if ((st = launch_q4_gemv(static_cast<const uint8_t*>(d->w13[l].data), 2 * F, D, d->h, 1, D, d->act, F, &f,
                                 ws_g, s)))
            return st;
        vox_epilogue r2 = {};
        r2.op = VOX_EP_RESIDUAL;
        r2.residual = d->h;
        r2.ldr = D;
        if ((st = launch_q4_gemv(static_cast<const uint8_t*>(d->w2[l].data), D, F, d->act, 1, F, d->x, D, &r2, ws_g,
                                 s)))
            return st;
    }
    vox_epilogue am = {};
    am.op = VOX_EP_ARGMAX;
    am.rmsnorm = 1;
    am.eps = d->eps;
    am.argmax = d->token;
    if ((st = launch_q4_gemv(static_cast<const uint8_t*>(d->lm_head.data), d->vocab, D, d->x, 1, D, d->logits,
                             d->vocab, &am, ws_g, s)))
        return st;
    return launch_advance_pos(d->pos, s);
}

// ------------------------------------------------------------ batched step
static size_t batch_gemv_ws(const vox_decoder_batch* b) { return (dec_gemv_ws(&b->d) + 255) & ~(size_t)255; }

size_t vox_decoder_batch_workspace(const vox_decoder_batch* b)
{
    if (!b || b->n_seq < 1 || b->n_seq > 8 || b->d.dim < 32 || b->d.vocab < 1 || b->d.n_kv_heads < 1 ||
        b->d.window < 1 || b->d.n_layers < 1 || b->d.n_q_heads < b->d.n_kv_heads)
        return 0;
    const size_t QD = (size_t)b->d.n_q_heads * (size_t)b->d.head_dim, F = (size_t)b->d.ffn;
    return batch_gemv_ws(b) +
           ((attn_workspace_bytes(b->d.n_kv_heads, b->d.head_dim, b->d.window, b->n_seq) + 255) & ~(size_t)255) +
           ((b->n_seq * QD * 2 + 255) & ~(size_t)255) + ((b->n_seq * F * 2 + 255) & ~(size_t)255);
}

vox_status vox_decoder_batch_step(const vox_decoder_batch* b, void* stream)
{
    if (!b) return VOX_ERR_NULL;
    const vox_decoder* d = &b->d;
    vox_status st = check_decoder(d, false);
    if (st) return st;
    if (b->n_seq < 1 || b->n_seq > 8) return VOX_ERR_RANGE;
    if (!b->page_table) return VOX_ERR_NULL;
    if (d->window < 64 || d->window % 64 || b->n_pages < 1) return VOX_ERR_RANGE;
    if (b->n_pages > 0x7fffff00LL / (64LL * d->n_kv_heads)) return VOX_ERR_SHAPE;
    if (d->ws_bytes < vox_decoder_batch_workspace(b)) return VOX_ERR_WORKSPACE;
    const int64_t m = b->n_seq;
    const int64_t D = d->dim, QD = (int64_t)d->n_q_heads * d->head_dim, KVD = (int64_t)d->n_kv_heads * d->head_dim;
    const int64_t F = d->ffn;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* ws_g = static_cast<uint8_t*>(d->workspace);
    uint8_t* ws_a = ws_g + batch_gemv_ws(b);
    // bf16 copies of the Wo and W2 inputs for the tcgen05 GEMM (after the attention workspace)
    uint8_t* attn16 = ws_a + ((attn_workspace_bytes(d->n_kv_heads, d->head_dim, d->window, (int)m) + 255) & ~(size_t)255);
    uint8_t* act16 = attn16 + ((m * QD * 2 + 255) & ~(int64_t)255);
    const float scale = 1.0f / sqrtf((float)d->head_dim);
    // From 4 sequences on, the Wo and W2 projections (the long-K ones) run on
    // the tcgen05 GEMM over bf16 copies of their inputs: there one GEMM beats
    // the multi-row GEMV (about 11 against 19 us on 3072 x 4096, 19 against 32
    // on 3072 x 9216 at 8 rows; 11 against 13 and 19 against 21 at 4 rows), the
    // copy costing one short launch.  At 3 rows the GEMV is still faster.
    const char* e2 = getenv("VOX_BATCH_GEMM");
    const bool gemm_wo_w2 = m > 3 && !(e2 && e2[0] == '0') && QD % 64 == 0 && F % 64 == 0;

    // x[i] = embedding row of sequence i's token (exact fp32 weights)
    if ((st = launch_q4_dequant(static_cast<const uint8_t*>(d->embedding.data), d->vocab, D, 0, d->token, m, d->x,
                                VOX_F32, D, s, 1)))
        return st;
    for (int l = 0; l < d->n_layers; ++l) {
        vox_epilogue e = {};
        e.op = VOX_EP_KV_APPEND_PAGED;
        e.rmsnorm = 1;
        e.eps = d->eps;
        e.k_cache = d->k_cache[l];
        e.v_cache = d->v_cache[l];
        e.n_kv_heads = d->n_kv_heads;
        e.head_dim = d->head_dim;
        e.window = d->window;
        e.q_rows = (int32_t)QD;
        e.pos_dev = d->pos;
        e.rope_theta = d->rope_theta;
        e.page_table = b->page_table;
        e.n_pages = b->n_pages;
        if ((st = launch_q4_gemv(static_cast<const uint8_t*>(d->wqkv[l].data), QD + 2 * KVD, D, d->x, m, D, d->qkv,
                                 QD + 2 * KVD, &e, ws_g, s)))
            return st;
        if ((st = launch_gqa_decode_attn_seqs(d->qkv, d->k_cache[l], d->v_cache[l], d->attn, d->n_q_heads,
                                              d->n_kv_heads, d->head_dim, d->window, 0, d->pos, scale, ws_a, s,
                                              (int)m, b->page_table, b->n_pages, QD + 2 * KVD)))
            return st;
        vox_epilogue r = {};
        r.op = VOX_EP_RESIDUAL;
        r.residual = d->x;
        r.ldr = D;
        if (gemm_wo_w2) {
            if ((st = launch_cast_rows(d->attn, m, QD, QD, attn16, VOX_BF16, QD, s)) ||
                (st = launch_q4_gemm(static_cast<const uint8_t*>(d->wo[l].data), D, QD, attn16, m, QD, d->h, VOX_F32,
                                     D, &r, s)))
                return st;
        } else if ((st = launch_q4_gemv(static_cast<const uint8_t*>(d->wo[l].data), D, QD, d->attn, m, QD, d->h, D, &r,
                                        ws_g, s))) {
            return st;
        }
        vox_epilogue f = {};
        f.op = VOX_EP_SILU_MUL;
        f.rmsnorm = 1;
        f.eps = d->eps;
        if ((st = launch_q4_gemv(static_cast<const uint8_t*>(d->w13[l].data), 2 * F, D, d->h, m, D, d->act, F, &f,
                                 ws_g, s)))
            return st;
        vox_epilogue r2 = {};
        r2.op = VOX_EP_RESIDUAL;
        r2.residual = d->h;
        r2.ldr = D;
        if (gemm_wo_w2) {
            if ((st = launch_cast_rows(d->act, m, F, F, act16, VOX_BF16, F, s)) ||
                (st = launch_q4_gemm(static_cast<const uint8_t*>(d->w2[l].data), D, F, act16, m, F, d->x, VOX_F32, D,
                                     &r2, s)))
                return st;
        } else if ((st = launch_q4_gemv(static_cast<const uint8_t*>(d->w2[l].data), D, F, d->act, m, F, d->x, D, &r2,
                                        ws_g, s))) {
            return st;
        }
    }
    vox_epilogue am = {};
    am.op = VOX_EP_ARGMAX;
    am.rmsnorm = 1;
    am.eps = d->eps;
    am.argmax = d->token;
    if ((st = launch_q4_gemv(static_cast<const uint8_t*>(d->lm_head.data), d->vocab, D, d->x, m, D, d->logits,
                             d->vocab, &am, ws_g, s)))
        return st;
    return launch_advance_pos(d->pos, s, (int)m);
}

vox_status vox_encoder_chunk(const vox_encoder* e, void* stream)
{
    if (!e) return VOX_ERR_NULL;
    if (!e->wqkv || !e->wo || !e->wup || !e->wdown || !e->k_hist || !e->v_hist || !e->x || !e->xn || !e->qkv ||
        !e->att || !e->up || !e->adapter_mid || !e->adapter_out_buf)
        return VOX_ERR_NULL;
    if (e->n_layers < 1 || e->n_heads < 1 || e->head_dim < 1 || e->head_dim > 64 || e->rows < 4 || e->rows % 4 ||
        e->dim != e->n_heads * e->head_dim || e->dim % 64 || e->ffn % 64)
        return VOX_ERR_SHAPE;
    if (e->window < 1) return VOX_ERR_RANGE;
    if (!al16(e->xn) || !al16(e->qkv) || !al16(e->att) || !al16(e->up) || !al16(e->adapter_mid))
        return VOX_ERR_ALIGN;
    if (e->adapter_out % 64) return VOX_ERR_SHAPE;
    const int64_t D = e->dim, F = e->ffn, R = e->rows;
    vox_status st;
    for (int l = 0; l < e->n_layers; ++l) {
        if ((st = check_w(e->wqkv[l], 3 * D, D))) return st;
        if ((st = check_w(e->wo[l], D, D))) return st;
        if ((st = check_w(e->wup[l], F, D))) return st;
        if ((st = check_w(e->wdown[l], D, F))) return st;
        if (!e->k_hist[l] || !e->v_hist[l]) return VOX_ERR_NULL;
        if (e->k_hist_next || e->v_hist_next) {
            if (!e->k_hist_next || !e->v_hist_next || !e->k_hist_next[l] || !e->v_hist_next[l]) return VOX_ERR_NULL;
            const void* outs[2] = {e->k_hist_next[l], e->v_hist_next[l]};
            for (const void* o : outs) {
                if (!al16(o)) return VOX_ERR_ALIGN;
                if (o == e->k_hist[l] || o == e->v_hist[l]) return VOX_ERR_ALIGN;
            }
        }
    }
    if ((st = check_w(e->adapter, e->adapter_out, 4 * D))) return st;
    if ((st = check_w(e->adapter2, e->adapter_out, e->adapter_out))) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const float scale = 1.0f / sqrtf((float)e->head_dim);
    for (int l = 0; l < e->n_layers; ++l) {
        const bool tap = e->tap && l == e->n_layers - 1;
        if (tap && (st = launch_cast_rows(e->x, R, D, D, e->tap, VOX_F32, D, s))) return st;
        if ((st = launch_rmsnorm(e->x, R, D, D, e->eps, nullptr, e->xn, VOX_BF16, D, s))) return st;
        if ((st = launch_q4_gemm(static_cast<const uint8_t*>(e->wqkv[l].data), 3 * D, D, e->xn, R, D, e->qkv,
                                 VOX_BF16, 3 * D, nullptr, s)))
            return st;
        const uint16_t* qkv = static_cast<const uint16_t*>(e->qkv);
        if ((st = launch_window_attn(qkv, 3 * D, e->k_hist[l], e->v_hist[l], D, e->window, qkv + D, qkv + 2 * D,
                                     3 * D, R, e->att, VOX_BF16, D, e->n_heads, e->head_dim, e->window, scale, s)))
            return st;
        if (e->k_hist_next) {
            if ((st = launch_hist_roll(e->k_hist[l], D, qkv + D, 3 * D, R, e->window, D, e->k_hist_next[l], D, s)))
                return st;
            if ((st = launch_hist_roll(e->v_hist[l], D, qkv + 2 * D, 3 * D, R, e->window, D, e->v_hist_next[l], D, s)))
                return st;
        }
        vox_epilogue r = {};
        r.op = VOX_EP_RESIDUAL;
        r.residual = e->x;
        r.ldr = D;
        if ((st = launch_q4_gemm(static_cast<const uint8_t*>(e->wo[l].data), D, D, e->att, R, D, e->x, VOX_F32, D, &r,
                                 s)))
            return st;
        if (tap && (st = launch_cast_rows(e->x, R, D, D, e->tap + R * D, VOX_F32, D, s))) return st;
        if ((st = launch_rmsnorm(e->x, R, D, D, e->eps, nullptr, e->xn, VOX_BF16, D, s))) return st;
        vox_epilogue gl = {};
        gl.op = VOX_EP_GELU;
        if ((st = launch_q4_gemm(static_cast<const uint8_t*>(e->wup[l].data), F, D, e->xn, R, D, e->up, VOX_BF16, F,
                                 &gl, s)))
            return st;
        if ((st = launch_q4_gemm(static_cast<const uint8_t*>(e->wdown[l].data), D, F, e->up, R, F, e->x, VOX_F32, D,
                                 &r, s)))
            return st;
    }
    // 4x downsample: bf16 copy of the rows, read as [R/4][4D]
    if ((st = launch_cast_rows(e->x, R, D, D, e->xn, VOX_BF16, D, s))) return st;
    vox_epilogue gl = {};
    gl.op = VOX_EP_GELU;
    if ((st = launch_q4_gemm(static_cast<const uint8_t*>(e->adapter.data), e->adapter_out, 4 * D, e->xn, R / 4,
                             4 * D, e->adapter_mid, VOX_BF16, e->adapter_out, &gl, s)))
        return st;
    return launch_q4_gemm(static_cast<const uint8_t*>(e->adapter2.data), e->adapter_out, e->adapter_out,
                          e->adapter_mid, R / 4, e->adapter_out, e->adapter_out_buf, VOX_F32, e->adapter_out, nullptr,
                          s);
}

}  // extern "C"
