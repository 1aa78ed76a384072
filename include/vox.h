/*
 * vox.h -- C ABI of the B200 (sm_100a) Q4_0 decode/encode hot path of
 * Voxtral Mini 4B Realtime.
 *
 * Plain C: every pointer is a raw address, every size an integer, and the
 * stream is a cudaStream_t passed as void* (NULL = the legacy default stream).
 * "device" pointers are CUDA device memory owned by the caller; the library
 * never allocates, never frees and never synchronises.  All calls are
 * asynchronous on the given stream.  Arguments are validated on the host
 * before anything is launched; a call that returns an error has launched
 * nothing (except VOX_ERR_CUDA, which reports a failed launch).
 *
 * Sources of the operations (page titles and sections as on the pages):
 *  [Q4]   "Voxtral Mini 4B Realtime (Rust)", page 5, "Arquitetura": the Q4
 *         GGUF path quantises with GGUF Q4_0 and runs custom shaders.
 *         Q4_0 block: fp16 scale d + 16 bytes holding 32 4-bit codes q,
 *         weight w = (q - 8) * d; element j < 16 is the low nibble of byte j,
 *         element j + 16 the high nibble (GGUF order).
 *  [FUSE] "브라우저에서 도는 4B 음성인식: Voxtral Rust+WASM 구현 해부", section
 *         "F32(9GB) vs Q4 GGUF(2.5GB)": dequantisation fused into the matmul.
 *  [EMB]  same page, and "Voxtral Mini 4B Realtime (Rust)" page 5 "Soluções
 *         técnicas": the 1.5 GiB embedding table kept as Q4 on the GPU with
 *         single-row lookups.
 *  [ARCH] "Mistral Voxtral Realtime 4B ... 순수 C 기반 CPU 전용 추론 구현",
 *         "모델 아키텍처": decoder 26 layers, dim 3072, GQA 32 query / 8 KV
 *         heads; encoder 32 causal layers, dim 1280, 32 heads, window 750;
 *         adapter Linear(5120->3072) -> GELU -> Linear; vocabulary 131072.
 *  [ROLL] same page, "주요 기능": rolling KV cache, an 8192-position sliding
 *         window that keeps memory constant for unbounded audio.
 *  [BATCH] same page, "주요 기능": fused GPU ops and batched attention; and
 *         "성능 벤치마크": the decoder runs a whole token step as one GPU
 *         submission.
 */
#ifndef VOX_H
#define VOX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------ status codes */
typedef int32_t vox_status;
enum {
    VOX_OK = 0,
    VOX_ERR_NULL = 1,       /* a required pointer is NULL                          */
    VOX_ERR_SHAPE = 2,      /* a size is out of the supported set (k % 32 != 0 ...) */
    VOX_ERR_ALIGN = 3,      /* a pointer or leading dimension breaks an alignment rule */
    VOX_ERR_DTYPE = 4,      /* unsupported element type for this argument          */
    VOX_ERR_RANGE = 5,      /* pos < 0, window <= 0, n_q % n_kv != 0, row out of range */
    VOX_ERR_WORKSPACE = 6,  /* workspace NULL or smaller than the query call says   */
    VOX_ERR_TIMEOUT = 7,    /* reserved: a bounded device-side wait gave up         */
    VOX_ERR_CUDA = 8        /* a CUDA launch or query failed; see vox_last_error()   */
};

/* element types */
enum { VOX_F32 = 0, VOX_BF16 = 1, VOX_F16 = 2 };

/* Human-readable name of a status code (static string, never NULL). */
const char *vox_status_str(vox_status s);
/* Text of the last CUDA error seen by this thread in a vox_* call ("" if none). */
const char *vox_last_error(void);
/* Device status word of the calling thread's current device: 0 when every
 * bounded device-side wait completed, else a code naming the wait that gave
 * up (the kernel then returned early and its outputs are not valid).  This
 * call synchronises the device; clear != 0 resets the word.  -1 if the word
 * cannot be read. */
int32_t vox_device_status(int32_t clear);

/* ------------------------------------------------------- packed Q4_0 weight
 * The GGUF blocks of an n x k matrix are repacked once ([Q4]: "repacked once
 * for 16-byte vector loads") into a tiled layout of the same total size up to
 * padding: rows are grouped in tiles of 16, columns in chunks of 64 (two
 * blocks); each (tile, chunk) is 576 contiguous bytes -- 512 bytes of codes
 * arranged so that one 16-byte load per lane feeds that lane's tensor-core
 * fragments, then 64 bytes of the 32 fp16 scales.  Tiles are stored
 * row-tile-major, chunks in k order.  Rows past n and columns past k are
 * padding with d = 0 and q = 8 (weight 0).  The layout is internal: only the
 * vox_* calls read it, and vox_q4_dequant returns the logical weights. */
typedef struct {
    const void *data;   /* device, vox_q4_packed_bytes(n, k) bytes, 16-byte aligned */
    int64_t n;          /* output rows (logical)                                     */
    int64_t k;          /* input columns, a multiple of 32                           */
} vox_q4_weight;

/* Bytes of the packed layout: ceil(n/16)*16 * ceil(k/64)*64 * 18/32.  -1 if
 * n < 1 or k < 32 or k % 32 != 0. */
int64_t vox_q4_packed_bytes(int64_t n, int64_t k);

/* pack flags */
enum {
    VOX_PACK_PLAIN = 0,
    /* The input holds [W1; W3] (n = 2F rows: F gate rows then F up rows, F a
     * multiple of 8).  Packed row order interleaves groups of 8: packed rows
     * 16j..16j+7 are W1 rows 8j..8j+7 and packed rows 16j+8..16j+15 are W3
     * rows 8j..8j+7, which is what the VOX_EP_SILU_MUL epilogue expects. */
    VOX_PACK_GATE_UP = 1
};

/* vox_q4_pack -- [Q4].  gguf: device, n * k/32 blocks of 18 bytes in GGUF
 * order (row-major: block b of row r at byte (r*k/32 + b)*18; bytes 0-1 the
 * little-endian fp16 d, bytes 2-17 the codes).  packed: device,
 * vox_q4_packed_bytes(n, k) bytes, 16-byte aligned, fully written (padding
 * included).  Errors: NULL pointers -> VOX_ERR_NULL; k % 32, n < 1 or a
 * GATE_UP n that is not 2F with F % 8 == 0 -> VOX_ERR_SHAPE; packed not 16-byte
 * aligned -> VOX_ERR_ALIGN; unknown flags -> VOX_ERR_RANGE. */
vox_status vox_q4_pack(const void *gguf, int64_t n, int64_t k, int32_t flags, void *packed,
                       void *stream);

/* vox_q4_dequant -- [Q4], [EMB].  Writes w[r][c] = (q - 8) * d for packed
 * rows r in [row0, row0 + nrows) and all k columns to out (device, row-major
 * with leading dimension ldo >= k elements).  out_dtype VOX_F32 gives the
 * exact product (it always fits fp32); VOX_BF16 rounds it to nearest-even
 * (NaN -> 0x7FC0).  Row numbers are packed rows (for VOX_PACK_GATE_UP weights
 * that is the interleaved order).  Errors: NULL -> VOX_ERR_NULL; rows outside
 * [0, n) -> VOX_ERR_RANGE; ldo < k -> VOX_ERR_SHAPE; other dtypes ->
 * VOX_ERR_DTYPE. */
vox_status vox_q4_dequant(const vox_q4_weight *w, int64_t row0, int64_t nrows, void *out,
                          int32_t out_dtype, int64_t ldo, void *stream);

/* --------------------------------------------------------------- epilogues
 * A small POD that fuses the work around a projection into the projection's
 * kernel: an optional RMSNorm of each input row before the product (reading:
 * x / sqrt(mean(x^2) + eps) * g, pre-norm), and one output operation. */
enum {
    VOX_EP_NONE = 0,      /* y = W x                                                  */
    VOX_EP_RESIDUAL = 1,  /* y = residual + W x (residual may alias y)                 */
    VOX_EP_SILU_MUL = 2,  /* W packed with VOX_PACK_GATE_UP: y[j] = silu(g_j) * u_j,
                             y has n/2 columns; silu(a) = a / (1 + exp(-a))            */
    VOX_EP_GELU = 3,      /* y = gelu(W x), exact erf form                             */
    VOX_EP_KV_APPEND = 4, /* rows [0, q_rows) -> y as usual; rows [q_rows, q_rows+kv)
                             are k and [q_rows+kv, q_rows+2kv) are v (kv =
                             n_kv_heads*head_dim): they are also written to y and,
                             rounded to bf16, into slot (pos + i) mod window of the
                             caches for token i ([ROLL])                               */
    VOX_EP_ARGMAX = 5,    /* y = W x, and argmax[i] = index of the largest y[i][:],
                             lowest index on ties, a NaN wins over numbers             */
    VOX_EP_KV_APPEND_PAGED = 6 /* as KV_APPEND, but input row i is sequence i of a batch
                             with its own paged rolling cache: its k and v go, rounded
                             to bf16, to slot p = pos_dev[i] mod window of that
                             sequence, i.e. row p mod 64 of page
                             page_table[i * (window / 64) + p / 64] of the pools
                             k_cache / v_cache, bf16 [n_pages][n_kv_heads][64][head_dim]
                             ([ROLL] per sequence, [BATCH]).  window a multiple of 64;
                             pos_dev required.  A page index outside [0, n_pages) is
                             not written and sets the device status word (0x105)   */
};

typedef struct {
    int32_t op;                /* VOX_EP_*                                            */
    int32_t rmsnorm;           /* 1: normalise each input row first                    */
    float eps;                 /* RMSNorm epsilon (1e-5 in this library's model)       */
    const float *norm_weight;  /* device [k] gain g, or NULL for g = 1                 */
    const float *residual;     /* RESIDUAL: device [m][ldr] fp32                       */
    int64_t ldr;
    void *k_cache;             /* KV_APPEND: device bf16 [n_kv_heads][window][head_dim] */
    void *v_cache;
    int32_t n_kv_heads, head_dim, window, q_rows;
    int64_t pos;               /* KV_APPEND: position of input row 0                   */
    const int64_t *pos_dev;    /* if not NULL, the position is read from device memory  */
    int32_t *argmax;           /* ARGMAX: device int32 [m]                              */
    const int32_t *page_table; /* KV_APPEND_PAGED: device int32 [m][window / 64]        */
    int64_t n_pages;           /* KV_APPEND_PAGED: pages in each pool                   */
    float rope_theta;          /* KV_APPEND(_PAGED): 0 = off (the pages name no positional
                                  encoding); > 0: rotary embedding of the q and k rows
                                  before they are stored: in each head, the pair
                                  (y[2i], y[2i+1]) turns by pos * theta^(-2i/head_dim),
                                  pos the token's position.  Needs head_dim % 16 == 0
                                  and q_rows % head_dim == 0                            */
} vox_epilogue;

/* ----------------------------------------------------------- Q4_0 GEMV (M<=8)
 * vox_q4_gemv -- [Q4], [FUSE].  y[i][j] = sum_c w[j][c] * x[i][c] for
 * i < m (1 <= m <= 8) and packed rows j < n, dequantising in registers with no
 * separate pass, then the epilogue.  x: device fp32 [m][ldx]; y: device fp32
 * [m][ldy] (n columns, or n/2 for SILU_MUL).  The product runs on the tensor
 * cores with each 32-column block of x (times the RMSNorm weight) rounded to
 * fp16 after an exact power-of-two scaling of its own, and fp32
 * accumulation; the result is within 2e-3 of the fp64 product, normalised by
 * |x_i| |w_j|.  workspace: device scratch of vox_q4_gemv_workspace() bytes
 * (256), 16-byte aligned: the argmax keys and arrival counter.  Zero it once
 * before its first use; every call leaves it at zero again.  Calls that
 * share a workspace must not overlap on the GPU.  Limits: m * ceil(k/64)*64
 * <= 81920 (the fp16 activations live in shared memory).
 * Errors: NULL -> VOX_ERR_NULL; m outside 1..8, k % 32, ldx < k, ldy too small,
 * SILU_MUL with n % 16, KV_APPEND rows that do not fit n, or the size limit ->
 * VOX_ERR_SHAPE; weight data not 16-byte aligned -> VOX_ERR_ALIGN; bad
 * epilogue fields -> VOX_ERR_RANGE; short workspace -> VOX_ERR_WORKSPACE. */
vox_status vox_q4_gemv(const vox_q4_weight *w, const float *x, int64_t m, int64_t ldx,
                       float *y, int64_t ldy, const vox_epilogue *ep,
                       void *workspace, size_t ws_bytes, void *stream);
size_t vox_q4_gemv_workspace(const vox_q4_weight *w, int64_t m, const vox_epilogue *ep);

/* ------------------------------------------------------ Q4_0 GEMM (M >= 16)
 * vox_q4_gemm -- [Q4], [FUSE], encoder chunks and batched rows.
 * Y = X W^T: y[i][j] = sum_c x[i][c] w[j][c] for i < m, j < n.  x: device bf16
 * [m][ldx] (ldx a multiple of 8, x 16-byte aligned).  The packed weights are
 * staged by TMA into shared memory, dequantised there to bf16 and fed to the
 * tcgen05 tensor cores with fp32 accumulation in tensor memory.  y: device
 * [m][ldy] of y_dtype VOX_F32 or VOX_BF16.  Epilogues: NONE, RESIDUAL
 * (fp32 y only), GELU; no RMSNorm prologue (use vox_rmsnorm first).  Errors as
 * for vox_q4_gemv; m < 1 or k % 64 -> VOX_ERR_SHAPE. */
vox_status vox_q4_gemm(const vox_q4_weight *w, const void *x, int32_t x_dtype, int64_t m,
                       int64_t ldx, void *y, int32_t y_dtype, int64_t ldy,
                       const vox_epilogue *ep, void *stream);

/* ------------------------------------------------- Q4_0 matmul, any M
 * vox_q4_matmul -- [Q4], [FUSE]: y = x W^T for m rows of fp32 activations,
 * choosing the kernel by m at the crossover measured on B200 (the batched
 * sweep over the decoder's shapes): m <= 8 runs the register-dequantising
 * GEMV (vox_q4_gemv), m > 8 rounds x (after the optional RMSNorm) to bf16
 * into the workspace and runs the tcgen05 GEMM (vox_q4_gemm).  x: device fp32
 * [m][ldx]; y: device fp32 [m][ldy].  Epilogues: every vox_q4_gemv epilogue
 * at m <= 8; NONE, RESIDUAL and GELU (with or without the RMSNorm prologue)
 * at m > 8, other ones -> VOX_ERR_RANGE.  workspace: device,
 * vox_q4_matmul_workspace() bytes, 16-byte aligned; its first 256 bytes
 * must be zero before the first use (the GEMV's argmax state, left zero by
 * every call).  Calls that share a workspace must not overlap on the GPU.
 * Errors as vox_q4_gemv and vox_q4_gemm. */
vox_status vox_q4_matmul(const vox_q4_weight *w, const float *x, int64_t m, int64_t ldx, float *y, int64_t ldy,
                         const vox_epilogue *ep, void *workspace, size_t ws_bytes, void *stream);
size_t vox_q4_matmul_workspace(const vox_q4_weight *w, int64_t m, const vox_epilogue *ep);

/* ------------------------------------------------------------ rolling cache
 * vox_kv_append_rolling -- [ROLL].  Stores one position: k_new and v_new
 * (device [n_kv_heads][head_dim] of new_dtype VOX_F32 or VOX_BF16) are
 * rounded to bf16 (nearest-even) and written to slot pos mod window of
 * k_cache / v_cache (device bf16 [n_kv_heads][window][head_dim]).  After the
 * call the valid slots are the first min(pos + 1, window).  Errors: NULL ->
 * VOX_ERR_NULL; pos < 0 or window <= 0 -> VOX_ERR_RANGE; head_dim outside
 * 1..1024 or n_kv_heads < 1 -> VOX_ERR_SHAPE. */
vox_status vox_kv_append_rolling(void *k_cache, void *v_cache, const void *k_new, const void *v_new,
                                 int32_t new_dtype, int32_t n_kv_heads, int32_t head_dim,
                                 int32_t window, int64_t pos, void *stream);

/* vox_gqa_decode_attn -- [ARCH] GQA, [ROLL], [BATCH].  One decode query per
 * head over the rolling cache after position pos was written: query head h
 * reads kv head h / (n_q_heads / n_kv_heads); s_j = scale * q_h . k_j over the
 * valid slots j < min(pos + 1, window); out_h = softmax(s) . V.  q: device fp32
 * [n_q_heads][head_dim]; caches: device bf16 [n_kv_heads][window][head_dim],
 * 16-byte aligned; out: device fp32 [n_q_heads][head_dim], 16-byte aligned
 * (it is written with 16-byte stores).  Split-KV: slot
 * ranges are reduced independently into the workspace (device, at least
 * vox_gqa_decode_attn_workspace() bytes, 16-byte aligned, no initial contents
 * needed) and merged by a log-sum-exp combine (a second, small kernel).
 * Calls sharing a workspace must not overlap on the GPU.  head_dim must be
 * 128 (the decoder's).
 * Errors: NULL -> VOX_ERR_NULL; pos < 0, window <= 0, n_q % n_kv != 0, a
 * group above 8 or more than 512 kv heads -> VOX_ERR_RANGE; other head_dim
 * -> VOX_ERR_SHAPE; short workspace -> VOX_ERR_WORKSPACE; caches, out or
 * workspace not 16-byte aligned -> VOX_ERR_ALIGN. */
vox_status vox_gqa_decode_attn(const float *q, const void *k_cache, const void *v_cache, float *out,
                               int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                               int32_t window, int64_t pos, float scale,
                               void *workspace, size_t ws_bytes, void *stream);
size_t vox_gqa_decode_attn_workspace(int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                     int32_t window);

/* vox_gqa_decode_attn_static -- an interface of this library with no
 * counterpart in the source pages: vox_gqa_decode_attn without a caller
 * workspace, for callers that cannot hand in device scratch (a host program
 * that links only this library and owns no device allocator; a real-time
 * audio thread that must not call cudaMalloc, which can block and
 * synchronise the device).  Same arguments, result and precision as
 * vox_gqa_decode_attn.  It allocates nothing: the split-KV partial records
 * go to one fixed array in device memory that is part of the loaded library
 * (about 1.2 MiB), sized for at most 8 kv heads with at most 4 query heads
 * per kv head at head_dim 128 (the decoder's 32 / 8 fits); larger shapes
 * return VOX_ERR_RANGE with a message in vox_last_error().  Nothing in the
 * array needs to start at zero: every call writes each record it reads.
 * All calls on one device share the array, so two calls that overlap on the
 * GPU (other streams, concurrent graph replays) corrupt each other's
 * results: order them on one stream.  The first call on each device looks
 * the array's address up (cudaGetSymbolAddress); make that call outside any
 * stream capture.  The address is kept for the life of the process: after
 * cudaDeviceReset on a device, reload the library before calling this entry
 * point on that device again.  Other errors (out not 16-byte aligned ->
 * VOX_ERR_ALIGN included) as vox_gqa_decode_attn. */
vox_status vox_gqa_decode_attn_static(const float *q, const void *k_cache, const void *v_cache,
                                      float *out, int32_t n_q_heads, int32_t n_kv_heads,
                                      int32_t head_dim, int32_t window, int64_t pos, float scale,
                                      void *stream);

/* ------------------------------------------ batched decode attention (paged)
 * vox_gqa_decode_attn_paged -- [ROLL] per sequence, [BATCH].  The attention of
 * vox_gqa_decode_attn for n_seq independent sequences in one call, each with
 * its own rolling cache held in pages of 64 slots.  Pools: k_pool, v_pool
 * device bf16 [n_pages][n_kv_heads][64][head_dim], 16-byte aligned; sequence
 * s's slot p (0 <= p < window) lives in row p mod 64 of page
 * page_table[s * (window / 64) + p / 64] (page_table: device int32
 * [n_seq][window / 64]); pos: device int64 [n_seq], the position each
 * sequence has just written (valid slots: the first min(pos[s] + 1, window)).
 * q: device fp32 [n_seq][n_q_heads][head_dim]; out: device fp32, same shape,
 * 16-byte aligned.  The SMs are shared evenly by the sequences.  workspace:
 * device, vox_gqa_decode_attn_paged_workspace() bytes, 16-byte aligned, no
 * initial contents needed; calls sharing it must not overlap.  A page index
 * outside [0, n_pages) reads zeros and sets the device status word (0x203).
 * Errors: NULL -> VOX_ERR_NULL; n_seq outside 1..64, pos handling as
 * vox_gqa_decode_attn, window not a positive multiple of 64, n_pages < 1 ->
 * VOX_ERR_RANGE; head_dim != 128 or a pool beyond 2^31 rows -> VOX_ERR_SHAPE;
 * misaligned pools, out or workspace -> VOX_ERR_ALIGN; short workspace ->
 * VOX_ERR_WORKSPACE. */
vox_status vox_gqa_decode_attn_paged(const float *q, const void *k_pool, const void *v_pool, int64_t n_pages,
                                     const int32_t *page_table, const int64_t *pos, int32_t n_seq, float *out,
                                     int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim, int32_t window,
                                     float scale, void *workspace, size_t ws_bytes, void *stream);
size_t vox_gqa_decode_attn_paged_workspace(int32_t n_seq, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                           int32_t window);

/* vox_window_attn -- [ARCH] encoder: causal sliding-window multi-head
 * attention for a chunk of n_q query rows.  Query row i sits at absolute
 * position n_hist + i and sees key position p iff pos_i - window < p <= pos_i.
 * Keys/values at positions < n_hist come from k_hist/v_hist rows (device bf16
 * [n_hist][ld_hist]); positions n_hist + i from k_new/v_new rows (device bf16
 * [n_q][ld_new]).  Head h uses columns [h*head_dim, (h+1)*head_dim).  q: device
 * bf16 [n_q][ldq]; out: device [n_q][ldo] of out_dtype VOX_F32 or VOX_BF16.
 * Errors: NULL -> VOX_ERR_NULL; window <= 0 -> VOX_ERR_RANGE; head_dim not in
 * 1..64 or leading dimensions too small -> VOX_ERR_SHAPE. */
vox_status vox_window_attn(const void *q, int64_t ldq, const void *k_hist, const void *v_hist,
                           int64_t ld_hist, int64_t n_hist, const void *k_new, const void *v_new,
                           int64_t ld_new, int64_t n_q, void *out, int32_t out_dtype, int64_t ldo,
                           int32_t n_heads, int32_t head_dim, int32_t window, float scale,
                           void *stream);

/* ---------------------------------------------------------------- glue ops
 * vox_rmsnorm -- pre-norm of the decoder and encoder layers (reading: eps
 * inside the square root, gain g or 1).  x: device fp32 [m][ldx]; out: device
 * [m][ldo] of out_dtype VOX_F32 or VOX_BF16. */
vox_status vox_rmsnorm(const float *x, int64_t m, int64_t n, int64_t ldx, float eps,
                       const float *g, void *out, int32_t out_dtype, int64_t ldo, void *stream);

/* ------------------------------------------------------------ GGUF files
 * [Q4]: the pages' quantised weights ship as a GGUF file with Q4_0 tensors.
 * vox_gguf_open reads a GGUF (version 2 or 3) file into host memory and
 * indexes its metadata and tensors; the handle owns that copy until
 * vox_gguf_close.  Bounds are checked against the file size: a truncated or
 * malformed file -> VOX_ERR_SHAPE (bad magic, version, counts or tensor
 * infos), VOX_ERR_ALIGN (a tensor offset off the file's alignment) or
 * VOX_ERR_RANGE (a tensor past the end, or the file cannot be read).
 * Tensor dims are innermost first: a weight of n rows x k columns has
 * dims = {k, n}.  Element types: 0 f32, 1 f16, 2 Q4_0; tensors of other
 * types are listed with nbytes = 0 and no data pointer. */
typedef struct vox_gguf vox_gguf;
vox_status vox_gguf_open(const char *path, vox_gguf **out);
void vox_gguf_close(vox_gguf *g);
int64_t vox_gguf_tensor_count(const vox_gguf *g);                 /* -1 for NULL          */
int64_t vox_gguf_find_tensor(const vox_gguf *g, const char *name); /* index, or -1         */
/* name, element type, dimension count, dims[4] (unused ones 1) and data bytes
 * of tensor i; any output pointer may be NULL.  i out of range ->
 * VOX_ERR_RANGE. */
vox_status vox_gguf_tensor_info(const vox_gguf *g, int64_t i, const char **name, int32_t *type,
                                int32_t *n_dims, int64_t *dims, uint64_t *nbytes);
/* Host pointer to tensor i's bytes inside the handle, or NULL. */
const void *vox_gguf_tensor_data(const vox_gguf *g, int64_t i);
/* Metadata by key: integers and bools, floats, strings (NULL if absent or
 * not a string).  Missing key -> VOX_ERR_RANGE, other type -> VOX_ERR_DTYPE. */
vox_status vox_gguf_get_int(const vox_gguf *g, const char *key, int64_t *value);
vox_status vox_gguf_get_float(const vox_gguf *g, const char *key, double *value);
const char *vox_gguf_get_string(const vox_gguf *g, const char *key);
/* Upload Q4_0 tensor i (dims {k, n}) and repack it like vox_q4_pack: its
 * GGUF blocks are copied host -> device into scratch (device, at least the
 * tensor's nbytes; the call returns once the host bytes are staged), then
 * packed into `packed` (device, vox_q4_packed_bytes(n, k) bytes, 16-byte
 * aligned) on `stream`.  Not Q4_0 -> VOX_ERR_DTYPE; more than 2 dims ->
 * VOX_ERR_SHAPE; short scratch -> VOX_ERR_WORKSPACE; flags as vox_q4_pack. */
vox_status vox_gguf_upload_q4(const vox_gguf *g, int64_t i, void *scratch, size_t scratch_bytes, int32_t flags,
                              void *packed, void *stream);

/* ------------------------------------------------------------ composed path
 * The decoder token step and the encoder chunk, built from the calls above
 * and launched back to back on one stream (the pages' "one submission per
 * token step"; the caller may capture the call in a CUDA graph). */
typedef struct {
    int32_t n_layers, dim, n_q_heads, n_kv_heads, head_dim, ffn, vocab, window;
    float eps;
    const vox_q4_weight *wqkv;   /* host array [n_layers]: [Wq; Wk; Wv], (q+2kv) x dim */
    const vox_q4_weight *wo;     /* host array [n_layers]: dim x q_dim                  */
    const vox_q4_weight *w13;    /* host array [n_layers]: VOX_PACK_GATE_UP, 2ffn x dim */
    const vox_q4_weight *w2;     /* host array [n_layers]: dim x ffn                    */
    vox_q4_weight embedding;     /* vocab x dim                                         */
    vox_q4_weight lm_head;       /* vocab x dim                                         */
    void *const *k_cache;        /* host array [n_layers] of device bf16 caches         */
    void *const *v_cache;
    int32_t *token;              /* device [1]: input token; receives the argmax          */
    int64_t *pos;                /* device [1]: this step's position; incremented at end   */
    float *x, *h, *qkv, *attn, *act, *logits;  /* device activations: dim, dim,
                                    q+2kv, q_dim, ffn, vocab floats                     */
    void *workspace;             /* device, vox_decoder_workspace() bytes, zero-filled once  */
    size_t ws_bytes;
    float rope_theta;            /* 0: no positional encoding (default); > 0: rotary
                                    embedding of q and k, see vox_epilogue.rope_theta   */
} vox_decoder;

/* Bytes of decoder workspace (device, 16-byte aligned) that both forms of
 * the step below need on the calling thread's current device.  Zero it once
 * before the first step; every successful step leaves it ready for the next.
 * After a step that left a non-zero device status (vox_device_status),
 * zero it again before the next step. */
size_t vox_decoder_workspace(const vox_decoder *dec);

/* vox_decoder_step -- [ARCH], [ROLL], [BATCH]: one greedy decode step as ONE
 * kernel launch (the pages' single GPU submission per token step):
 * x = embedding[token]; n_layers x {RMSNorm + QKV GEMV with rolling append,
 * GQA attention, Wo GEMV + residual, RMSNorm + W1||W3 GEMV + SiLU*mul, W2 GEMV
 * + residual}; RMSNorm + LM head GEMV + argmax -> token; pos += 1.  A
 * persistent cooperative grid of one CTA per SM runs the phases back to back
 * with grid-wide barriers; it occupies the whole device while it runs.  The
 * same arithmetic as the kernels of vox_decoder_step_kernels (register
 * dequantisation, fp16 activations scaled per block, fp32 accumulation;
 * split-KV attention with bf16 hi + lo operands), summed in another fixed
 * order: results agree within the library's tolerance, not bit for bit, and
 * are the same from run to run.  Every device-side wait is bounded (about one
 * second); one that gives up sets the device status word (0x501, 0x502 ring
 * waits, 0x510 grid barrier, 0x520 drain) and the step returns early.
 * Limits: n_layers <= 32, head_dim 128, at most 4 query heads per kv head,
 * dim % 4 == 0, and the widest projection's activations in shared memory
 * (dim, n_q_heads * 128 and ffn up to about 10000); otherwise VOX_ERR_SHAPE
 * with the reason in vox_last_error() (vox_decoder_step_kernels has none of
 * these limits).  Other errors as vox_decoder_step_kernels. */
vox_status vox_decoder_step(const vox_decoder *dec, void *stream);

/* vox_decoder_step_fused -- the same step as 1 + 3 n_layers launches: layer
 * 0's QKV projection, then per layer the split-KV attention (two launches,
 * as vox_gqa_decode_attn) and one persistent cooperative launch that runs the
 * layer's Wo, W1||W3 and W2 projections and the next layer's QKV (after the
 * last layer: the LM head, argmax and position advance) with grid-wide
 * barriers between them, streaming each projection's weights into shared
 * memory while the grid waits at the barrier before it.  Same arithmetic and
 * limits as vox_decoder_step; can be captured in a CUDA graph.  Errors as
 * vox_decoder_step. */
vox_status vox_decoder_step_fused(const vox_decoder *dec, void *stream);

/* vox_decoder_step_kernels -- the same step as a sequence of launches of the
 * library's kernels on one stream (embedding row, per layer the QKV GEMV with
 * rolling append, attention + combine, Wo, W1||W3 and W2 GEMVs, then the LM
 * head with argmax and the position advance), each with programmatic
 * dependent launch; the sequence can be captured in a CUDA graph.  Errors:
 * NULL fields -> VOX_ERR_NULL; shapes that do not match the weights, a group
 * above 8 or head_dim != 128 -> VOX_ERR_SHAPE; window < 1 -> VOX_ERR_RANGE;
 * a short workspace -> VOX_ERR_WORKSPACE; a workspace, cache or activation
 * buffer that is not 16-byte aligned -> VOX_ERR_ALIGN. */
vox_status vox_decoder_step_kernels(const vox_decoder *dec, void *stream);

/* ------------------------------------------------ batched decoder step
 * n_seq independent sequences stepped together ([BATCH]; [ROLL] per
 * sequence): every projection reads its weights once for all sequences (the
 * GEMV at m = n_seq rows), and each sequence keeps its own rolling cache in
 * pages of 64 slots drawn from per-layer pools, so sequences of any
 * positions share one weight stream.  `d` holds the shapes and weights as
 * for one sequence, with these meanings:
 *   d.k_cache[l], d.v_cache[l]: the layer's page pools, device bf16
 *       [n_pages][n_kv_heads][64][head_dim], 16-byte aligned;
 *   d.token: device int32 [n_seq], the input tokens, replaced by the greedy
 *       next tokens; d.pos: device int64 [n_seq], each sequence's position,
 *       advanced by one;
 *   d.x, d.h, d.qkv, d.attn, d.act, d.logits: device fp32 [n_seq][...] of the
 *       one-sequence sizes (rows back to back);
 *   d.workspace: vox_decoder_batch_workspace() bytes, zero-filled once.
 * page_table: device int32 [n_seq][window / 64] (see vox_gqa_decode_attn_paged);
 * the caller assigns pages (a rolling window reuses its own pages in place). */
typedef struct {
    vox_decoder d;
    int32_t n_seq;               /* 1..8 */
    int64_t n_pages;             /* pages in each pool */
    const int32_t *page_table;
} vox_decoder_batch;

size_t vox_decoder_batch_workspace(const vox_decoder_batch *b);

/* One greedy step of every sequence: the launches of vox_decoder_step_kernels
 * with m = n_seq rows (embedding rows gathered by token, the QKV epilogue
 * VOX_EP_KV_APPEND_PAGED, vox_gqa_decode_attn_paged, argmax per row, every
 * position advanced); from 4 sequences on the Wo and W2 projections run as the
 * tcgen05 GEMM (vox_q4_gemm) on bf16 copies of their inputs, kept in the
 * workspace (VOX_BATCH_GEMM=0 in the environment keeps the GEMV); the
 * sequence can be captured in a CUDA graph.  Errors:
 * as vox_decoder_step_kernels; n_seq outside 1..8, window not a multiple of
 * 64 or n_pages < 1 -> VOX_ERR_RANGE; NULL page_table -> VOX_ERR_NULL. */
vox_status vox_decoder_batch_step(const vox_decoder_batch *b, void *stream);

typedef struct {
    int32_t n_layers, dim, n_heads, head_dim, ffn, window, rows, adapter_out;
    float eps;
    const vox_q4_weight *wqkv;   /* host array [n_layers]: 3dim x dim                   */
    const vox_q4_weight *wo;     /* dim x dim                                           */
    const vox_q4_weight *wup;    /* ffn x dim                                           */
    const vox_q4_weight *wdown;  /* dim x ffn                                           */
    vox_q4_weight adapter;       /* adapter_out x 4dim: the adapter's first Linear        */
    vox_q4_weight adapter2;      /* adapter_out x adapter_out: its second Linear          */
    const void *const *k_hist;   /* host array [n_layers] of device bf16 [window][dim]  */
    const void *const *v_hist;
    float *x;                    /* device fp32 [rows][dim]: chunk input, updated in place */
    void *xn;                    /* device bf16 [rows][dim] scratch                     */
    void *qkv;                   /* device bf16 [rows][3dim] scratch                    */
    void *att;                   /* device bf16 [rows][dim] scratch                     */
    void *up;                    /* device bf16 [rows][ffn] scratch                     */
    void *adapter_mid;           /* device bf16 [rows/4][adapter_out] scratch: GELU output */
    float *adapter_out_buf;      /* device fp32 [rows/4][adapter_out]                   */
    float *tap;                  /* device fp32 [2][rows][dim], or NULL: receives the last
                                    layer's input x (tap[0]) and its residual stream h
                                    after attention (tap[1]), so that layer can be checked
                                    on its own inputs                                   */
    void *const *k_hist_next;    /* host array [n_layers] of device bf16 [window][dim], or
                                    NULL: streaming (P4 주요 기능, overlapping chunks):
                                    receives the next chunk's history of each layer, the
                                    last `window` rows of this chunk's history followed by
                                    its own k (v) rows; must not alias k_hist (v_hist).  The
                                    caller swaps the two sets between chunks             */
    void *const *v_hist_next;
} vox_encoder;

/* One encoder chunk: 32 x {RMSNorm, QKV GEMM, window attention, O GEMM +
 * residual, RMSNorm, up GEMM + GELU, down GEMM + residual}, then the 4x
 * downsample (rows 4r..4r+3 concatenated) and the adapter ([ARCH]: Linear
 * 4dim -> adapter_out, exact-erf GELU, Linear adapter_out -> adapter_out;
 * the GELU output is rounded to bf16 in adapter_mid).  With k_hist_next and
 * v_hist_next set, every layer also writes the next chunk's history after its
 * attention, so consecutive chunks see each other through the 750-row window.
 * Errors: NULL fields -> VOX_ERR_NULL; shapes -> VOX_ERR_SHAPE; misaligned
 * buffers or a next history that is one of the inputs -> VOX_ERR_ALIGN. */
vox_status vox_encoder_chunk(const vox_encoder *enc, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* VOX_H */
