// K1: fused Q4_0 dequantise + GEMV for M <= 8 rows of activations.
//
// Computes y[i][j] = sum_c w[j][c] x[i][c] with w = (q - 8) * d (GGUF Q4_0,
// "Voxtral Mini 4B Realtime (Rust)", page 5 "Arquitetura") and dequantises in
// registers inside the matmul, with no separate dequant pass ("브라우저에서 도는
// 4B 음성인식: Voxtral Rust+WASM 구현 해부", section "F32(9GB) vs Q4 GGUF").
//
// Design (B200, HBM-bound at M <= 8):
//  * Work split: every CTA owns a contiguous run of whole 16-row tiles, and
//    inside it every warp owns one contiguous, equal range of the run's
//    (tile, 64-column chunk) records ("stream-K" at warp granularity).  A
//    tile a warp covers completely is finished from its registers; a tile cut
//    between warps is finished by the warp that started it, which adds the
//    pieces of the following warps in warp order from shared memory:
//    deterministic, and no CTA ever waits for another.
//  * Data movement: each warp streams its range through its own ring of
//    shared-memory stages (three by default), one bulk (TMA) copy of four
//    576-byte records per stage, completing on a per-stage mbarrier.  One
//    stage is issued before griddepcontrol.wait (weights never depend on
//    upstream kernels), the others once the activations are in, so the
//    activation loads do not queue behind a full ring; bytes in flight cost
//    no registers.
//  * Dequantisation: each 32-bit word of codes gives four half2 A-fragment
//    registers with one LOP3 each (OR the nibble into the fraction of 1024.0
//    or 64.0, whose ulp is 1 at that nibble position: exact 1024+q / 64+q).
//    The MMAs start from zero; the constant offsets come back as one
//    per-block correction, -(1032 * sum x_lo + 72 * sum x_hi), added to the
//    MMA result before the scale.
//  * Tensor cores: mma.sync m16n8k16 fp16 x fp16 -> fp32, the low- and
//    high-nibble halves of a block chained, and the four records of a stage
//    issued back to back before any bookkeeping, so the MMA latency
//    overlaps.  A stage with no tile end and no range end takes a fast path
//    (pairwise sum of the four records, no per-record checks).
//  * Activations: each 32-column block of x (times the RMSNorm weight) is
//    scaled by its own exact power of two into [2^13, 2^14) before the fp16
//    conversion, and the block's inverse scale is folded into its d in fp32.
//    No row statistic is needed before the main loop: the RMSNorm factor
//    multiplies the finished dot products in the epilogue.  The prologue is
//    one round of loads and one CTA barrier.
//  * Instances: one row (MT = 1) or up to 8 (MT = 8), each with and without
//    the paged KV append and the rotary embedding in its epilogue (EXT).
//    The decode step's projections run the instances without them, which
//    stay inside the 128-register budget with less spilling.
//  * Build knobs (tuning, not semantics): VOX_GEMV_WARPS, VOX_GEMV_RECS,
//    VOX_GEMV_MIN_CTAS, VOX_GEMV_BATCH at compile time; VOX_GEMV_STAGES,
//    VOX_GEMV_PREFETCH and VOX_GEMV_CTAS_PER_SM in the environment.
#include "q4_math.cuh"

#include <stdlib.h>

namespace vox {

#ifndef VOX_GEMV_WARPS
#define VOX_GEMV_WARPS 8
#endif
constexpr int kGemvWarps = VOX_GEMV_WARPS;
constexpr int kGemvThreads = 32 * kGemvWarps;
#ifndef VOX_GEMV_RECS
#define VOX_GEMV_RECS 4
#endif
constexpr int kGemvRecs = VOX_GEMV_RECS;                      // records per ring stage (one bulk copy)
constexpr int kGemvStageBytes = kGemvRecs * kChunkBytes;
constexpr int kGemvMaxStages = 8;
constexpr int kGemvDefaultStages = 3;
#ifndef VOX_GEMV_MIN_CTAS
#define VOX_GEMV_MIN_CTAS 2
#endif
#ifndef VOX_GEMV_BATCH
#define VOX_GEMV_BATCH 9
#endif
constexpr int kGemvBatch = VOX_GEMV_BATCH;                    // prologue float4 loads in flight per thread

struct GemvArgs {
    const uint8_t* w;
    int64_t n, k;
    int32_t tiles, kc;
    const float* x;
    int64_t ldx;
    int32_t m, vec4;
    float* y;
    int64_t ldy;
    int32_t op, rmsnorm;
    float eps;
    const float* g;
    const float* res;
    int64_t ldr;
    uint16_t* kcache;
    uint16_t* vcache;
    int32_t n_kv, hd, window, q_rows;
    int64_t pos;
    const int64_t* pos_dev;
    int32_t* argmax;
    uint8_t* ws;
    int32_t stages;
    int32_t pre;                             // ring stages issued before griddepcontrol.wait
    int32_t evict_first;                     // 1: weight copies marked evict-first in L2
    const int32_t* pages;                    // KV_APPEND_PAGED: page table [m][window / 64]
    int64_t n_pages;
    float rope;                              // KV_APPEND(_PAGED): rotary theta, 0 = off
};

// Shared-memory carve-up, computed identically on host and device.
struct GemvSmem {
    uint32_t ring, bars, bs, cb, part, ptile, sq, best_v, best_i, total;
};

// Entries per block in the constant table: 1 at m = 1, else m rounded up to even.
__host__ __device__ inline int gemv_cb_stride(int m) { return m == 1 ? 1 : (m + 1) & ~1; }

__host__ __device__ inline GemvSmem gemv_smem_layout(int kc, int m, int stages)
{
    GemvSmem L;
    uint32_t off = 0;
    L.ring = off;    off += (uint32_t)kGemvWarps * (uint32_t)stages * kGemvStageBytes;
    L.bars = off;    off += (uint32_t)kGemvWarps * (uint32_t)stages * 8u;
    off = (off + 15u) & ~15u;
    L.bs = off;      off += (uint32_t)kc * (uint32_t)m * 128u;     // fp16 B fragments
    // per (block, token), a block's tokens adjacent and padded to an even
    // count (one 16-byte load covers tokens 2t, 2t + 1): offset constant, 1/scale
    L.cb = off;      off += (uint32_t)kc * (uint32_t)gemv_cb_stride(m) * 16u;
    L.part = off;    off += kGemvWarps * 32 * 16;
    L.ptile = off;   off += kGemvWarps * 4;
    L.sq = off;      off += kGemvWarps * 8 * 4;
    L.best_v = off;  off += kGemvWarps * 8 * 4;
    L.best_i = off;  off += kGemvWarps * 8 * 4;
    L.total = off;
    return L;
}

// Workspace: one 64-bit argmax key per token and the CTA arrival counter of
// the argmax epilogue.  Both are zero between calls.
constexpr size_t kGemvWsKeys = 0, kGemvWsCount = 64, kGemvWsBytes = 256;

size_t gemv_workspace_bytes(int64_t n, int64_t k, int op)
{
    (void)n;
    (void)k;
    (void)op;
    return kGemvWsBytes;
}

// Issue ring batch j of a warp's range [wb, we): up to kGemvRecs records
// in one bulk copy, completing on `bar`.
__device__ __forceinline__ void gemv_issue(const uint8_t* w, int64_t wb, int64_t we, int j, uint8_t* dst,
                                           uint64_t* bar, int evict_first)
{
    const int64_t r0 = wb + (int64_t)j * kGemvRecs;
    const uint32_t bytes = (uint32_t)min64(kGemvRecs, we - r0) * kChunkBytes;
    mbar_arrive_expect_tx(bar, bytes);
    if (evict_first)
        bulk_g2s_stream(dst, w + r0 * kChunkBytes, bytes, bar);
    else
        bulk_g2s(dst, w + r0 * kChunkBytes, bytes, bar);
}

// Running greedy-argmax candidates of one lane, for its tokens 2t and 2t + 1.
struct GemvBest {
    float v0, v1;
    int32_t i0, i1;
};

// Epilogue of one finished 16-row tile from the MMA accumulator layout:
// lane (g, t) holds acc[2h + e] = tile row g + 8h, token 2t + e; rr[e] is the
// RMSNorm factor of token 2t + e (1 without RMSNorm).  `pre` (with use_pre)
// holds the residual values in the same layout, loaded ahead by the caller.
// Not inlined: it runs once per tile and keeps the record loop small.
template <bool EXT>
__device__ __noinline__ GemvBest gemv_epilogue(const GemvArgs& a, int64_t tile, float4 acc4, int g, int t, float r0,
                                               float r1, int64_t pos, GemvBest best, float4 pre, int use_pre)
{
    const float acc[4] = {acc4.x, acc4.y, acc4.z, acc4.w};
    const float prv[4] = {pre.x, pre.y, pre.z, pre.w};
    const float rr[2] = {r0, r1};
    float best_v[2] = {best.v0, best.v1};
    int32_t best_i[2] = {best.i0, best.i1};
    float v[4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 2; ++e) v[2 * h + e] = acc[2 * h + e] * rr[e];
    if (EXT && a.rope > 0.f && tile * 16 < (int64_t)a.q_rows + (int64_t)a.n_kv * a.hd) {
        // q or k rows (a 16-row tile lies in one region): rows 2i and 2i + 1
        // of a head sit in lanes g and g ^ 1, four lanes apart
        const int64_t base = tile * 16 < a.q_rows ? 0 : a.q_rows;
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float partner = __shfl_xor_sync(0xffffffffu, v[2 * h + e], 4);
                const int mt = 2 * t + e;
                if (mt < a.m) {
                    const int64_t col = (tile * 16 + g + 8 * h - base) % a.hd;
                    const int64_t p = a.op == VOX_EP_KV_APPEND_PAGED ? a.pos_dev[mt] : pos + mt;
                    v[2 * h + e] = rope_rotate(v[2 * h + e], partner, col, a.hd, p, a.rope);
                }
            }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int mt = 2 * t + e;
        if (mt >= a.m) continue;
        float* yr = a.y + (int64_t)mt * a.ldy;
        if (a.op == VOX_EP_SILU_MUL) {
            const int64_t row = tile * 16 + g;              // gate row g pairs with up row g + 8
            if (row < a.n) yr[tile * 8 + g] = silu_f(v[e]) * v[2 + e];
            continue;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t row = tile * 16 + g + 8 * h;
            if (row >= a.n) continue;
            const float val = v[2 * h + e];
            switch (a.op) {
            case VOX_EP_RESIDUAL:
                yr[row] = (use_pre ? prv[2 * h + e] : a.res[(int64_t)mt * a.ldr + row]) + val;
                break;
            case VOX_EP_GELU:
                yr[row] = gelu_erf(val);
                break;
            case VOX_EP_KV_APPEND: {
                yr[row] = val;
                const int64_t kvd = (int64_t)a.n_kv * a.hd;
                const int64_t rel = row - a.q_rows;
                if (rel >= 0 && rel < 2 * kvd) {
                    uint16_t* cache = rel < kvd ? a.kcache : a.vcache;
                    const int64_t rw = rel < kvd ? rel : rel - kvd;
                    const int64_t head = rw / a.hd, col = rw - head * a.hd;
                    const int64_t slot_id = (pos + mt) % a.window;
                    cache[(head * a.window + slot_id) * a.hd + col] = f32_to_bf16_bits(val);
                }
                break;
            }
            case VOX_EP_KV_APPEND_PAGED: {
                // token mt is sequence mt: its slot pos[mt] mod window, in the page its table names
                yr[row] = val;
                if (!EXT) break;
                const int64_t kvd = (int64_t)a.n_kv * a.hd;
                const int64_t rel = row - a.q_rows;
                if (rel >= 0 && rel < 2 * kvd) {
                    uint16_t* pool = rel < kvd ? a.kcache : a.vcache;
                    const int64_t rw = rel < kvd ? rel : rel - kvd;
                    const int64_t head = rw / a.hd, col = rw - head * a.hd;
                    const int64_t slot_id = a.pos_dev[mt] % a.window;
                    const int64_t pg = a.pages[(int64_t)mt * (a.window / 64) + slot_id / 64];
                    if (pg >= 0 && pg < a.n_pages)
                        pool[((pg * a.n_kv + head) * 64 + slot_id % 64) * a.hd + col] = f32_to_bf16_bits(val);
                    else
                        atomicCAS(&g_vox_device_status, 0, 0x105);
                }
                break;
            }
            default:
                yr[row] = val;
                break;
            }
        }
    }
    if (a.op == VOX_EP_ARGMAX) {
        // per token 2t + e: rows g and g + 8 here, rows of other g in the lanes of equal t
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float bv = -INFINITY;
            int32_t bi = 0x7fffffff;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t row = tile * 16 + g + 8 * h;
                if (row < a.n && argmax_better(v[2 * h + e], (int32_t)row, bv, bi)) {
                    bv = v[2 * h + e];
                    bi = (int32_t)row;
                }
            }
#pragma unroll
            for (int o = 4; o <= 16; o <<= 1) {
                const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                const int32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (argmax_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
            }
            if (argmax_better(bv, bi, best_v[e], best_i[e])) { best_v[e] = bv; best_i[e] = bi; }
        }
    }
    return GemvBest{best_v[0], best_v[1], best_i[0], best_i[1]};
}

// Prologue for activation row i: x * g -> per-block power-of-two scale ->
// fp16 B fragments and the block's (offset constant, 1/scale), for the float4
// groups f = f0 + u * threads + lane (f0 warp-uniform, so the 8 float4 of one
// 32-column block sit in 8 adjacent lanes).  Columns past k (the padding of
// the last 64-column chunk) become zeros.  sq accumulates sum x^2.
__device__ __forceinline__ void gemv_convert(const GemvArgs& a, const float* xr, int i, int f0, int nf, int nfp,
                                             int lane, uint32_t* s_bs32, float2* s_cb, float& sq)
{
    const int m = a.m, cs = gemv_cb_stride(a.m);
    float4 v[kGemvBatch], gv[kGemvBatch];
#pragma unroll
    for (int u = 0; u < kGemvBatch; ++u) {
        const int f = f0 + u * kGemvThreads + lane;
        v[u] = f < nf ? ld_f4(xr, f, a.vec4) : make_float4(0.f, 0.f, 0.f, 0.f);
        gv[u] = (a.g && f < nf) ? ld_f4(a.g, f, a.vec4) : make_float4(1.f, 1.f, 1.f, 1.f);
    }
#pragma unroll
    for (int u = 0; u < kGemvBatch; ++u) {
        const int fb = f0 + u * kGemvThreads;             // warp-uniform
        if (fb >= nfp) break;
        const int f = fb + lane;
        sq = fmaf(v[u].x, v[u].x, sq);
        sq = fmaf(v[u].y, v[u].y, sq);
        sq = fmaf(v[u].z, v[u].z, sq);
        sq = fmaf(v[u].w, v[u].w, sq);
        const float4 xg = make_float4(v[u].x * gv[u].x, v[u].y * gv[u].y, v[u].z * gv[u].z, v[u].w * gv[u].w);
        float am = fmaxf(fmaxf(fabsf(xg.x), fabsf(xg.y)), fmaxf(fabsf(xg.z), fabsf(xg.w)));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
        am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));     // max over the 32-column block
        // am in [2^(E-127), 2^(E-126)): scale 2^(140-E) puts it in [2^13, 2^14)
        int E = (int)((__float_as_uint(am) >> 23) & 0xFFu);
        E = E < 14 ? 14 : E;
        const float sc = __uint_as_float((uint32_t)(267 - E) << 23);
        const float inv = __uint_as_float((uint32_t)(E - 13) << 23);
        const __half2 h01 = __floats2half2_rn(xg.x * sc, xg.y * sc);
        const __half2 h23 = __floats2half2_rn(xg.z * sc, xg.w * sc);
        const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
        float s = (f01.x + f01.y) + (f23.x + f23.y);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);        // sum over one 16-column half-block
        const float shi = __shfl_down_sync(0xffffffffu, s, 4);
        if (f < nfp) {
            // columns 4q .. 4q+3 of block blk: half q>>2, fragment register (q&3)>>1, pair 2(q&1)
            const int blk = f >> 3, q = f & 7;
            const int word = (blk * m + i) * 16 + 2 * (q & 1) * 4 + (q >> 2) * 2 + ((q & 3) >> 1);
            s_bs32[word] = *reinterpret_cast<const uint32_t*>(&h01);
            s_bs32[word + 4] = *reinterpret_cast<const uint32_t*>(&h23);
            if (q == 0) s_cb[blk * cs + i] = make_float2(-(1032.0f * s + 72.0f * shi), inv);
        }
    }
}

template <int MT, bool EXT>
__global__ void __launch_bounds__(kGemvThreads, VOX_GEMV_MIN_CTAS) q4_gemv_kernel(const __grid_constant__ GemvArgs a)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int m = a.m, kc = a.kc, stages = a.stages;
    const GemvSmem L = gemv_smem_layout(kc, m, stages);
    uint32_t* s_bs32 = reinterpret_cast<uint32_t*>(smem + L.bs);
    float2* s_cb = reinterpret_cast<float2*>(smem + L.cb);
    float* s_part = reinterpret_cast<float*>(smem + L.part);
    int32_t* s_ptile = reinterpret_cast<int32_t*>(smem + L.ptile);
    float* s_sq = reinterpret_cast<float*>(smem + L.sq);
    float* s_best_v = reinterpret_cast<float*>(smem + L.best_v);
    int32_t* s_best_i = reinterpret_cast<int32_t*>(smem + L.best_i);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t G = gridDim.x, b = blockIdx.x;
    const int64_t tile_b = b * a.tiles / G, tile_e = (b + 1) * a.tiles / G;
    const int64_t rb = tile_b * kc, R = (tile_e - tile_b) * kc;                   // this CTA's records
    const int64_t wb = rb + R * warp / kGemvWarps, we = rb + R * (warp + 1) / kGemvWarps;
    const int nbatch = (int)((we - wb + kGemvRecs - 1) / kGemvRecs);

    // this warp's ring; the first stages are in flight before the upstream kernels finish
    uint8_t* ring = smem + L.ring + (uint32_t)warp * (uint32_t)stages * kGemvStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * stages;
    if (lane == 0) {
        for (int s = 0; s < stages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        for (int j = 0; j < a.pre && j < nbatch; ++j)
            gemv_issue(a.w, wb, we, j, ring + j * kGemvStageBytes, &bars[j], a.evict_first);
        s_ptile[warp] = -1;
    }

    pdl_wait();                              // x (and pos) come from upstream kernels
    pdl_launch_dependents();                 // only after our own wait: at most two kernels overlap

    // ---- prologue: fp16 B fragments and block corrections of every row; sum x^2 per row
    const int nf = (int)(a.k >> 2), nfp = kc * 16;
    for (int i = 0; i < m; ++i) {
        const float* xr = a.x + (int64_t)i * a.ldx;
        float sq = 0.f;
        for (int f0 = warp * 32; f0 < nfp; f0 += kGemvBatch * kGemvThreads)
            gemv_convert(a, xr, i, f0, nf, nfp, lane, s_bs32, s_cb, sq);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) s_sq[warp * 8 + i] = sq;
    }
    __syncthreads();
    // the rest of the ring, issued once the activations are in
    if (lane == 0)
        for (int j = a.pre; j < stages && j < nbatch; ++j)
            gemv_issue(a.w, wb, we, j, ring + j * kGemvStageBytes, &bars[j], a.evict_first);

    // RMSNorm factors of this lane's tokens 2t, 2t+1 (zero for tokens past m)
    float rr[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int tk = MT == 1 ? e : 2 * t + e;
        float r = 0.f;
        if (tk < m) {
            r = 1.0f;
            if (a.rmsnorm) {
                float ssq = 0.f;
                for (int w = 0; w < kGemvWarps; ++w) ssq += s_sq[w * 8 + tk];
                r = 1.0f / sqrtf(ssq / (float)a.k + a.eps);
            }
        }
        rr[e] = r;
    }
    if (MT == 1 && t != 0) rr[0] = 0.f;      // token 2t of a lane with t > 0 does not exist at m = 1

    const int64_t pos = a.pos_dev ? *a.pos_dev : a.pos;
    const int cs = gemv_cb_stride(m);
    const uint32_t tk = smem_token();
    const uint32_t bs_a = smem_addr(s_bs32) + tk, cb_a = smem_addr(s_cb) + tk;
    const uint32_t ring_a = smem_addr(ring);
    const int tok = g < m ? g : 0;
    GemvBest best = {-INFINITY, -INFINITY, 0x7fffffff, 0x7fffffff};

    // ---- main loop: this warp's records through its ring
    float tacc[4] = {0.f, 0.f, 0.f, 0.f};    // piece of the tile this warp started and did not finish
    int64_t tail_tile = -1;
    if (nbatch > 0) {
        int64_t tile = wb / kc;
        int cin = (int)(wb - tile * kc);
        bool whole = (cin == 0);             // this warp saw the tile from its first record
        int left = (int)(we - wb);           // records still to add
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t phase = 0;
        int s = 0, fail_j = -1;
        // add one record's contribution; close the tile at its end or at the range end
        auto step = [&](const float (&p)[4]) {
            acc[0] += p[0]; acc[2] += p[2];
            if (MT != 1) { acc[1] += p[1]; acc[3] += p[3]; }
            --left;
            if (++cin == kc || left == 0) {
                if (!whole) {
                    // started by an earlier warp: leave the piece for it
                    *reinterpret_cast<float4*>(s_part + (warp * 32 + lane) * 4) =
                        make_float4(acc[0], acc[1], acc[2], acc[3]);
                    if (lane == 0) s_ptile[warp] = (int32_t)tile;
                } else if (cin == kc) {
                    best = gemv_epilogue<EXT>(a, tile, make_float4(acc[0], acc[1], acc[2], acc[3]), g, t, rr[0], rr[1],
                                         pos, best, make_float4(0.f, 0.f, 0.f, 0.f), 0);
                } else {
                    tacc[0] = acc[0]; tacc[1] = acc[1]; tacc[2] = acc[2]; tacc[3] = acc[3];
                    tail_tile = tile;
                }
                acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
                cin = 0;
                ++tile;
                whole = true;
            }
        };
        for (int j = 0; j < nbatch; ++j) {
            if (!mbar_wait_bounded(&bars[s], (phase >> s) & 1u, 0x101)) {
                fail_j = j;
                break;
            }
            phase ^= 1u << s;
            const uint32_t base = ring_a + (uint32_t)s * kGemvStageBytes + smem_token();
            // every record's MMAs first; the slots past `left` of a short stage are read and discarded
            float p[kGemvRecs][4];
            int ch = cin;
#pragma unroll
            for (int r = 0; r < kGemvRecs; ++r) {
                const uint4 q = lds128(base + r * kChunkBytes + 16 * lane);
                const uint2 e = lds64(base + r * kChunkBytes + kChunkQsBytes + 8 * g);
                p[r][0] = p[r][1] = p[r][2] = p[r][3] = 0.f;
                gemv_record<MT>(q, e, bs_a, cb_a, cs, ch, m, tok, t, p[r]);
                ch = ch + 1 == kc ? 0 : ch + 1;
            }
            if (left > kGemvRecs && cin + kGemvRecs < kc) {
                // no tile end and no range end inside this stage: pairwise sums of the records
#pragma unroll
                for (int w = 1; w < kGemvRecs; w <<= 1)
#pragma unroll
                    for (int r = 0; r + w < kGemvRecs; r += 2 * w) {
                        p[r][0] += p[r + w][0];
                        p[r][2] += p[r + w][2];
                        if (MT != 1) {
                            p[r][1] += p[r + w][1];
                            p[r][3] += p[r + w][3];
                        }
                    }
                acc[0] += p[0][0];
                acc[2] += p[0][2];
                if (MT != 1) {
                    acc[1] += p[0][1];
                    acc[3] += p[0][3];
                }
                cin += kGemvRecs;
                left -= kGemvRecs;
            } else {
#pragma unroll
                for (int r = 0; r < kGemvRecs; ++r)
                    if (left > 0) step(p[r]);
            }
            __syncwarp();
            if (lane == 0 && j + stages < nbatch)
                gemv_issue(a.w, wb, we, j + stages, ring + s * kGemvStageBytes, &bars[s], a.evict_first);
            if (++s == stages) s = 0;
        }
        if (fail_j >= 0 && lane == 0) {
            // a stage never completed: wait (bounded) for the copies still in flight into this ring
            const int jend = fail_j + stages < nbatch ? fail_j + stages : nbatch;
            for (int j = fail_j; j < jend; ++j)
                mbar_wait_bounded(&bars[j % stages], (uint32_t)(j / stages) & 1u, 0x102);
        }
    }

    // ---- tiles cut between warps: the warp that started one adds the later pieces in warp order;
    // its residual values are loaded before the barrier, off the tail's critical path
    float4 tres = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tail_tile >= 0 && a.op == VOX_EP_RESIDUAL) {
        float rv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int64_t row = tail_tile * 16 + g + 8 * h;
                const int mt = 2 * t + e;
                if (row < a.n && mt < m) rv[2 * h + e] = a.res[(int64_t)mt * a.ldr + row];
            }
        tres = make_float4(rv[0], rv[1], rv[2], rv[3]);
    }
    __syncthreads();
    if (tail_tile >= 0) {
        const int64_t last_rec = tail_tile * kc + kc - 1;
        const int wl = (int)(((last_rec - rb + 1) * kGemvWarps - 1) / R);   // warp holding the tile's last record
        const uint32_t tk2 = smem_token();
        for (int w2 = warp + 1; w2 <= wl; ++w2) {
            if (__float_as_int(lds32f(smem_addr(s_ptile) + 4u * w2 + tk2)) != (int32_t)tail_tile) continue;
            const float4 pv = lds128f(smem_addr(s_part) + (uint32_t)(w2 * 32 + lane) * 16u + tk2);
            tacc[0] += pv.x; tacc[1] += pv.y; tacc[2] += pv.z; tacc[3] += pv.w;
        }
        best = gemv_epilogue<EXT>(a, tail_tile, make_float4(tacc[0], tacc[1], tacc[2], tacc[3]), g, t, rr[0], rr[1], pos,
                             best, tres, a.op == VOX_EP_RESIDUAL);
    }

    // ---- greedy argmax: warps -> CTA -> one 64-bit atomic max per token; the
    // last CTA to arrive turns the keys into indices and clears them
    if (a.op == VOX_EP_ARGMAX) {
        if (g == 0) {
            s_best_v[warp * 8 + 2 * t] = best.v0;
            s_best_v[warp * 8 + 2 * t + 1] = best.v1;
            s_best_i[warp * 8 + 2 * t] = best.i0;
            s_best_i[warp * 8 + 2 * t + 1] = best.i1;
        }
        __syncthreads();
        if (tid == 0) {
            unsigned long long* keys = reinterpret_cast<unsigned long long*>(a.ws + kGemvWsKeys);
            uint32_t* count = reinterpret_cast<uint32_t*>(a.ws + kGemvWsCount);
            for (int i = 0; i < m; ++i) {
                float bv = -INFINITY;
                int32_t bi = 0x7fffffff;
                for (int w = 0; w < kGemvWarps; ++w)
                    if (argmax_better(s_best_v[w * 8 + i], s_best_i[w * 8 + i], bv, bi)) {
                        bv = s_best_v[w * 8 + i];
                        bi = s_best_i[w * 8 + i];
                    }
                atomicMax(&keys[i], argmax_key(bv, bi));
            }
            if (atom_add_acq_rel_gpu(count, 1u) == gridDim.x - 1) {
                for (int i = 0; i < m; ++i) {
                    const unsigned long long key = atomicExch(&keys[i], 0ull);
                    a.argmax[i] = (int32_t)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
                }
                *count = 0u;
            }
        }
    }
}

static int env_int(const char* name, int dflt, int lo, int hi)
{
    const char* e = getenv(name);
    int v = e ? atoi(e) : dflt;
    if (v < lo) v = lo;
    if (v > hi) v = hi;
    return v;
}

vox_status launch_q4_gemv(const uint8_t* w, int64_t n, int64_t k, const float* x, int64_t m, int64_t ldx,
                          float* y, int64_t ldy, const vox_epilogue* ep, void* ws, cudaStream_t s)
{
    GemvArgs a = {};
    a.w = w;
    a.n = n;
    a.k = k;
    a.tiles = (int32_t)ceil_div(n, 16);
    a.kc = (int32_t)ceil_div(k, 64);
    a.x = x;
    a.ldx = ldx;
    a.m = (int32_t)m;
    a.y = y;
    a.ldy = ldy;
    a.op = ep ? ep->op : VOX_EP_NONE;
    a.rmsnorm = ep ? ep->rmsnorm : 0;
    a.eps = ep ? ep->eps : 0.f;
    a.g = ep ? ep->norm_weight : nullptr;
    a.res = ep ? ep->residual : nullptr;
    a.ldr = ep ? ep->ldr : 0;
    if (ep && (ep->op == VOX_EP_KV_APPEND || ep->op == VOX_EP_KV_APPEND_PAGED)) {
        a.rope = ep->rope_theta;
        a.pages = ep->page_table;
        a.n_pages = ep->n_pages;
        a.kcache = static_cast<uint16_t*>(ep->k_cache);
        a.vcache = static_cast<uint16_t*>(ep->v_cache);
        a.n_kv = ep->n_kv_heads;
        a.hd = ep->head_dim;
        a.window = ep->window;
        a.q_rows = ep->q_rows;
        a.pos = ep->pos;
        a.pos_dev = ep->pos_dev;
    }
    a.argmax = ep ? ep->argmax : nullptr;
    a.ws = static_cast<uint8_t*>(ws);
    a.vec4 = ((reinterpret_cast<uintptr_t>(x) & 15u) == 0 && (ldx & 3) == 0 &&
              (!a.g || (reinterpret_cast<uintptr_t>(a.g) & 15u) == 0)) ? 1 : 0;

    int stages = env_int("VOX_GEMV_STAGES", kGemvDefaultStages, 2, kGemvMaxStages);
    GemvSmem L = gemv_smem_layout(a.kc, a.m, stages);
    while (stages > 2 && L.total > 227 * 1024) L = gemv_smem_layout(a.kc, a.m, --stages);
    if (L.total > 227 * 1024) return VOX_ERR_SHAPE;            // activations do not fit shared memory
    a.stages = stages;
    a.pre = env_int("VOX_GEMV_PREFETCH", 1, 0, stages);
    a.evict_first = env_int("VOX_GEMV_EVICT_FIRST", 1, 0, 1);

    // The paged append and the rotary embedding live in their own instances,
    // so the instances the decode step runs compile without them.
    const bool ext = ep && (ep->op == VOX_EP_KV_APPEND_PAGED || (ep->op == VOX_EP_KV_APPEND && ep->rope_theta > 0.f));
    void (*const kerns[4])(GemvArgs) = {q4_gemv_kernel<1, false>, q4_gemv_kernel<1, true>, q4_gemv_kernel<8, false>,
                                        q4_gemv_kernel<8, true>};
    static std::atomic<unsigned long long> attr_done[4];
    const int ki = (m == 1 ? 0 : 2) + (ext ? 1 : 0);
    void (*kern)(GemvArgs) = kerns[ki];
    vox_status st = smem_attr_per_device(reinterpret_cast<const void*>(kern), 227 * 1024, attr_done[ki]);
    if (st != VOX_OK) return st;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kGemvThreads, L.total);
    if (e != cudaSuccess || per_sm < 1) {
        set_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
        return VOX_ERR_CUDA;
    }
    const int cap = env_int("VOX_GEMV_CTAS_PER_SM", 2, 1, 4);
    if (per_sm > cap) per_sm = cap;
    int64_t G = (int64_t)device_sm_count() * per_sm;
    if (G > a.tiles) G = a.tiles;
    return launch_pdl(kern, dim3((unsigned)G), dim3(kGemvThreads), L.total, s, a);
}

}  // namespace vox
