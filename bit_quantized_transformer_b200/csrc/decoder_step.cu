// The greedy decoder token step as ONE persistent launch: every projection,
// the rolling-cache append, the split-KV GQA attention and the LM head with
// its argmax run inside a single cooperative grid of one CTA per SM, with
// bounded grid-wide phase barriers in place of kernel boundaries (the
// voxtral.c page, "성능 벤치마크": the decoder submits a whole token step to
// the GPU at once).
//
// Layer ("Mistral Voxtral Realtime 4B ... 순수 C 기반 CPU 전용 추론 구현",
// "모델 아키텍처": 26 layers, dim 3072, GQA 32 query / 8 KV heads; readings:
// pre-norm RMSNorm, SwiGLU FFN, no RoPE; rolling cache from "주요 기능"):
//   QKV  : qkv = Wqkv RMSNorm(x); k, v -> bf16 cache slot pos mod W
//   ATTN : o = softmax(q K^T / sqrt(128)) V over the valid slots
//   WO   : h = x + Wo o
//   W13  : a = silu(W1 n) * (W3 n), n = RMSNorm(h)
//   W2   : x = h + W2 a
// then LM : logits = Wlm RMSNorm(x), token = argmax (lowest index on ties).
// Layer 0's QKV reads the token's embedding row straight from the packed
// Q4_0 table.  Q4_0 (w = (q - 8) d, "Voxtral Mini 4B Realtime (Rust)", page 5,
// "Arquitetura") is dequantised in registers inside the products.
//
// Design (B200, HBM-bound at M = 1):
//  * One CTA per SM, 12 warps.  Every warp owns a ring of 4 shared-memory
//    stages of 4 KB in which its lane 0 keeps bulk (TMA) copies in flight.
//    The ring is one continuous stream across phases: once a warp has
//    consumed its last stage of a phase it immediately issues the first
//    stages of the next phase (weights and old cache rows never depend on
//    this step's activations), so HBM stays busy while the CTA waits at the
//    grid barrier.
//  * GEMV phases: every CTA owns a contiguous run of whole 16-row tiles of
//    the packed matrix (at most one tile more than another), and inside a
//    CTA the run's (tile, 64-column chunk) records are split evenly over the
//    warps (stream-K); a GEMV stage is up to 7 records (4032 bytes).  A tile
//    a warp covers alone is finished from its registers; a tile cut between
//    warps is summed in warp order from shared memory.  Residuals are loaded
//    before the main loop.  All sums have a fixed order: the result does not
//    depend on timing.  The phase's input vector is scaled by one power of
//    two per 128 columns (the columns one warp converts) into [2^13, 2^14)
//    before the fp16 conversion; a record's block MMAs start from the
//    block's offset constant (`gemv_record_m1`), and the records of a stage
//    run in groups of four up to each tile end.
//  * ATTN phases: 16-slot units (kv head, slots) are split evenly over CTAs;
//    inside a CTA the warps take units round robin, each unit two stages
//    (its K rows, then its V rows) of two 2-D TMA boxes each (64 columns x
//    16 rows, 128-byte swizzle).
//    Per unit a warp runs S = K q'^T and O^T += V^T P on mma.sync with an
//    online softmax in the exp2 domain (q' = q * scale * log2 e split into
//    bf16 hi + lo).  At the end of each kv head the warps' states are merged
//    in shared memory; a head that several CTAs share is merged from their
//    per-CTA records by the last CTA to arrive.
//  * Every wait is bounded (about one second): a wait that gives up records
//    a code in the device status word, raises a global abort flag that every
//    other wait also watches, and the kernel returns after its own copies in
//    flight have landed.
#include "q4_math.cuh"
#include "tma.cuh"

#include <stdlib.h>
#include <string.h>

namespace vox {

#ifndef VOX_PS_WARPS
#define VOX_PS_WARPS 12
#endif
#ifndef VOX_PS_STAGES
#define VOX_PS_STAGES 4
#endif
constexpr int kPsWarps = VOX_PS_WARPS;
constexpr int kPsThreads = 32 * kPsWarps;
constexpr int kPsStages = VOX_PS_STAGES;
constexpr int kPsStageBytes = 4096;                          // one K or V half of an attention unit
constexpr int kPsRecs = kPsStageBytes / kChunkBytes;       // 7 records per GEMV stage
constexpr int kPsMaxLayers = 32;
constexpr int kPsUnit = 16;                                  // cache slots per attention unit
constexpr int kPsHd = 128;
constexpr int kPsMaxGroup = 4;
constexpr int kPsBatch = 9;                                  // prologue float4 loads in flight per thread
constexpr int kPsRingBytes = kPsWarps * kPsStages * kPsStageBytes;

enum { PS_QKV = 0, PS_ATTN = 1, PS_WO = 2, PS_W13 = 3, PS_W2 = 4, PS_LM = 5 };

struct PsArgs {
    CUtensorMap kmap[kPsMaxLayers];          // K cache of each layer: [n_kv * W][128] bf16, box 64 x 16
    CUtensorMap vmap[kPsMaxLayers];
    const uint8_t* wqkv[kPsMaxLayers];
    const uint8_t* wo[kPsMaxLayers];
    const uint8_t* w13[kPsMaxLayers];
    const uint8_t* w2[kPsMaxLayers];
    uint16_t* kc[kPsMaxLayers];
    uint16_t* vc[kPsMaxLayers];
    const uint8_t* emb;
    const uint8_t* lm;
    int32_t* token;
    int64_t* pos;
    float *x, *h, *qkv, *attn, *act, *logits;
    uint8_t* ws;
    int32_t n_layers, dim, q_dim, kv_dim, ffn, vocab, n_kv, group, window;
    float eps, qscale;
    float rope;                      // rotary theta of q and k, 0 = off
    int32_t ph_begin, ph_end;        // the phases this launch runs (all: 0 .. 5 n_layers + 1)
    uint32_t act_bytes;                      // shared bytes of the activation / merge region
    int32_t test_withhold;                   // test hook: warp 0 of CTA 0 first waits on a barrier nothing completes
};

// ------------------------------------------------------------ workspace
// All counters are zero between steps (the finisher of each count resets
// it); the barrier counter only grows, by a multiple of the grid per step.
struct PsWs {
    size_t bar, abort, amax_key, amax_cnt, attncnt, recs, total;
    int32_t rmax, rec_floats;
};

__host__ __device__ inline int ps_rec_floats(int group) { return (group * (kPsHd + 2) + 3) & ~3; }

__host__ __device__ inline PsWs ps_ws_layout(int G, int n_layers, int n_kv, int group)
{
    PsWs L;
    L.rmax = (G + n_kv - 1) / n_kv + 2;
    L.rec_floats = ps_rec_floats(group);
    L.bar = 0;
    L.abort = 128;
    L.amax_key = 256;
    L.amax_cnt = 264;
    size_t off = 512;
    L.attncnt = off;
    off += ((size_t)n_layers * n_kv * 4 + 255) & ~(size_t)255;
    L.recs = off;
    off += ((size_t)n_kv * L.rmax * L.rec_floats * 4 + 255) & ~(size_t)255;
    L.total = off;
    return L;
}

// ------------------------------------------------------- shared memory
struct PsSmem {
    uint32_t ring, bars, act, piece, q, sq, best_v, best_i, flags, never, total;
};

__host__ __device__ inline PsSmem ps_smem_layout(uint32_t act_bytes)
{
    PsSmem L;
    uint32_t off = 0;
    L.ring = off;   off += kPsRingBytes;                       // 1024-aligned base
    L.bars = off;   off += kPsWarps * kPsStages * 8;
    L.act = off;    off += (act_bytes + 15u) & ~15u;
    L.piece = off;  off += kPsWarps * 2 * 16 * 4;
    L.q = off;      off += kPsMaxGroup * kPsHd * 4;             // the query heads of the CTA's kv head
    L.sq = off;     off += kPsWarps * 4;
    L.best_v = off; off += kPsWarps * 4;
    L.best_i = off; off += kPsWarps * 4;
    L.flags = off;  off += 16;
    L.never = off;  off += 8;                                   // an mbarrier nothing ever completes
    L.total = off + 1024;                                       // alignment slack
    return L;
}

// ------------------------------------------------------------ helpers
// floor(num / den) for non-negative operands, in 32 bits when they fit
// (64-bit division is a long software sequence on the GPU).
__device__ __forceinline__ int64_t udiv(uint64_t num, uint64_t den)
{
    if (num < (1ull << 32) && den < (1ull << 32)) return (int64_t)((uint32_t)num / (uint32_t)den);
    return (int64_t)(num / den);
}

__device__ __forceinline__ int64_t split_begin(int64_t b, int64_t total, int64_t parts)
{
    return udiv((uint64_t)b * (uint64_t)total, (uint64_t)parts);
}

// Part holding item c when `total` items are split into `parts` ranges
// [split_begin(b), split_begin(b + 1)) (the last non-empty one at or before c).
__device__ __forceinline__ int64_t split_owner(int64_t c, int64_t total, int64_t parts)
{
    return udiv((uint64_t)(c + 1) * (uint64_t)parts - 1, (uint64_t)total);
}

__device__ __forceinline__ uint64_t ld_acquire_u64(const uint64_t* p)
{
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ int32_t ld_relaxed_s32(const int32_t* p)
{
    int32_t v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Record `where` in the status word, then raise the abort flag.  The fence
// orders the two: a CTA that sees the flag and records its own code finds
// this code already there, so the word names the wait that gave up first.
__device__ __forceinline__ void ps_raise(const PsArgs& P, const PsWs& W, int32_t where)
{
    atomicCAS(&g_vox_device_status, 0, where);
    __threadfence();
    atomicExch(reinterpret_cast<int32_t*>(P.ws + W.abort), 1);
}

// A phase of the step: which matrix / layer, and the warp's share of it.
struct PsPhase {
    int kind, layer;
    const uint8_t* w;          // GEMV: packed weight
    int64_t n, k;
    int32_t kc;
    int64_t R;                 // GEMV: records; ATTN: units
    int64_t cb, ce;            // this CTA's range
    int64_t wb, we;            // GEMV: this warp's record range
    int32_t nst;               // this warp's stages in the phase
    int64_t hfirst, hcnt;      // ATTN: the first CTA of this CTA's kv head and the head's CTA count
};

__device__ __forceinline__ PsPhase ps_phase(const PsArgs& P, int ph, int64_t b, int64_t G, int warp, int64_t nch)
{
    PsPhase f;
    f.layer = ph / 5;
    f.kind = ph == 5 * P.n_layers ? PS_LM : ph % 5;
    const int l = f.layer;
    f.w = nullptr;
    f.n = 0;
    f.k = 0;
    switch (f.kind) {
    case PS_QKV: f.w = P.wqkv[l]; f.n = P.q_dim + 2 * P.kv_dim; f.k = P.dim; break;
    case PS_WO:  f.w = P.wo[l];   f.n = P.dim;                  f.k = P.q_dim; break;
    case PS_W13: f.w = P.w13[l];  f.n = 2 * (int64_t)P.ffn;     f.k = P.dim; break;
    case PS_W2:  f.w = P.w2[l];   f.n = P.dim;                  f.k = P.ffn; break;
    case PS_LM:  f.w = P.lm;      f.n = P.vocab;                f.k = P.dim; break;
    default: break;
    }
    if (f.kind == PS_ATTN) {
        // every CTA works on one kv head: head h has CTAs [h G / n_kv, (h + 1) G / n_kv),
        // which split its nch units evenly
        f.kc = 0;
        f.R = (int64_t)P.n_kv * nch;
        const int64_t h = split_owner(b, G, P.n_kv);
        f.hfirst = split_begin(h, G, P.n_kv);
        f.hcnt = split_begin(h + 1, G, P.n_kv) - f.hfirst;
        f.cb = h * nch + split_begin(b - f.hfirst, nch, f.hcnt);
        f.ce = h * nch + split_begin(b - f.hfirst + 1, nch, f.hcnt);
        f.wb = f.we = 0;
        const int64_t mine = f.ce - f.cb - warp;               // units cb + warp + kPsWarps * j
        f.nst = mine > 0 ? 2 * (int32_t)((mine + kPsWarps - 1) / kPsWarps) : 0;   // a K and a V stage each
    } else {
        // whole 16-row tiles per CTA (a tile is never cut between CTAs), the
        // CTA's records split evenly over its warps
        f.hfirst = f.hcnt = 0;
        f.kc = (int32_t)((f.k + 63) / 64);
        const int64_t T = (f.n + 15) / 16;
        f.R = T * f.kc;
        f.cb = split_begin(b, T, G) * f.kc;
        f.ce = split_begin(b + 1, T, G) * f.kc;
        const int64_t Rb = f.ce - f.cb;
        f.wb = f.cb + Rb * warp / kPsWarps;
        f.we = f.cb + Rb * (warp + 1) / kPsWarps;
        f.nst = (int32_t)((f.we - f.wb + kPsRecs - 1) / kPsRecs);
    }
    return f;
}

// The issue side of a warp's ring: walks the stages of the phases in order.
struct PsCursor {
    int ph;
    int idx;
    PsPhase f;
};

__device__ __forceinline__ void ps_cursor_settle(const PsArgs& P, PsCursor& c, int nph, int64_t b, int64_t G,
                                                 int warp, int64_t nch)
{
    while (c.ph < nph && c.idx >= c.f.nst) {
        ++c.ph;
        c.idx = 0;
        if (c.ph < nph) c.f = ps_phase(P, c.ph, b, G, warp, nch);
    }
}

// Issue the cursor's stage into ring slot `slot` (lane 0 only).
__device__ __forceinline__ void ps_issue(const PsArgs& P, const PsCursor& c, int warp, int64_t nch, uint8_t* dst,
                                         uint64_t* bar)
{
    const PsPhase& f = c.f;
    if (f.kind == PS_ATTN) {
        // stage 2u: the K rows of the warp's unit u, stage 2u + 1: its V rows
        const int64_t unit = f.cb + warp + (int64_t)kPsWarps * (c.idx >> 1);
        const int64_t hh = unit / nch, ci = unit - hh * nch;
        const int32_t row = (int32_t)(hh * P.window + ci * kPsUnit);
        const CUtensorMap* map = (c.idx & 1) ? &P.vmap[f.layer] : &P.kmap[f.layer];
        mbar_arrive_expect_tx(bar, kPsStageBytes);
        tma_load_2d(dst + 0, map, 0, row, bar);
        tma_load_2d(dst + 2048, map, 64, row, bar);
    } else {
        const int64_t r0 = f.wb + (int64_t)kPsRecs * c.idx;
        const uint32_t bytes = (uint32_t)min64(kPsRecs, f.we - r0) * kChunkBytes;
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(dst, f.w + r0 * kChunkBytes, bytes, bar);
    }
}

// Per-warp ring state (warp-uniform; lane 0 issues).
struct PsRing {
    uint8_t* base;          // this warp's 3 stages
    uint64_t* bars;
    uint32_t issued, consumed;
    PsCursor cur;
};

#ifndef VOX_PS_PREFETCH
#define VOX_PS_PREFETCH VOX_PS_STAGES
#endif
constexpr int kPsPrefetch = VOX_PS_PREFETCH;                 // stages of a later phase in flight at most

// Top the warp's ring up to kPsStages stages in flight; stages of a phase
// after ph_now count against the smaller kPsPrefetch.
__device__ __forceinline__ void ps_ring_fill(const PsArgs& P, PsRing& r, int nph, int64_t b, int64_t G, int warp,
                                             int lane, int64_t nch, int ph_now)
{
    while (r.issued - r.consumed < (uint32_t)kPsStages) {
        ps_cursor_settle(P, r.cur, nph, b, G, warp, nch);
        if (r.cur.ph >= nph) break;
        if (kPsPrefetch < kPsStages && r.cur.ph > ph_now && r.issued - r.consumed >= (uint32_t)kPsPrefetch) break;
        const uint32_t slot = r.issued % kPsStages;
        if (lane == 0) ps_issue(P, r.cur, warp, nch, r.base + slot * kPsStageBytes, &r.bars[slot]);
        ++r.issued;
        ++r.cur.idx;
    }
}

// Wait for stage consumed + ahead of the ring; false if the wait gave up.
__device__ __forceinline__ bool ps_ring_wait(PsRing& r, int32_t where, uint32_t ahead = 0)
{
    const uint32_t slot = (r.consumed + ahead) % kPsStages;
    const uint32_t parity = ((r.consumed + ahead) / kPsStages) & 1u;
    return mbar_wait_bounded(&r.bars[slot], parity, where);
}

// ------------------------------------------------------------ grid barrier
// One arrival per CTA on a monotonically growing counter; the target is the
// next multiple of the grid size above the arrival's old value.  Bounded:
// gives up after about one second or when another CTA raised the abort flag.
// The arriving thread is lane 1 of warp 0, which issues no bulk copies: a
// fence waits for the memory operations of its own thread only.
constexpr int kPsSyncThread = 1;

__device__ __forceinline__ bool ps_grid_barrier(const PsArgs& P, const PsWs& W, int32_t* s_flag, int32_t where)
{
    __syncthreads();
    if (threadIdx.x == kPsSyncThread) {
        uint64_t* ctr = reinterpret_cast<uint64_t*>(P.ws + W.bar);
        const int32_t* abort = reinterpret_cast<const int32_t*>(P.ws + W.abort);
        const uint64_t G = gridDim.x;
        __threadfence();
        const uint64_t old = atomicAdd(reinterpret_cast<unsigned long long*>(ctr), 1ull);
        const uint64_t target = (old / G + 1) * G;
        int ok = ld_relaxed_s32(abort) ? 0 : 1;               // another CTA already gave up
        if (ok && ld_acquire_u64(ctr) < target) {
            const uint64_t t0 = global_ns();
            for (;;) {
                bool done = false;
                for (int i = 0; i < 32; ++i)
                    if (ld_acquire_u64(ctr) >= target) { done = true; break; }
                if (done) break;
                if (ld_relaxed_s32(abort) || global_ns() - t0 > 1000000000ull) {
                    ok = 0;
                    break;
                }
            }
        }
        if (!ok) ps_raise(P, W, where);
        __threadfence();
        *s_flag = ok;
    }
    __syncthreads();
    return *reinterpret_cast<volatile int32_t*>(s_flag) != 0;
}

// ------------------------------------------------------------ prologue
// Four consecutive weights (4f .. 4f+3) of packed row `row` (exact fp32).
__device__ __forceinline__ float4 ps_emb_f4(const uint8_t* packed, int32_t kc, int64_t row, int f)
{
    const int c = 4 * f, blk = c >> 5, e0 = c & 31;
    const int i = (int)(row & 15), g = i & 7, rowsel = i >> 3;
    const int chunk = blk >> 1, bb = blk & 1;
    const uint8_t* rec = packed + ((row >> 4) * kc + chunk) * kChunkBytes;
    const uint16_t dbits = *reinterpret_cast<const uint16_t*>(rec + kChunkQsBytes + 8 * g + 2 * (bb * 2 + rowsel));
    const float d = __half2float(__ushort_as_half(dbits));
    float w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int e = e0 + u, half = e >> 4, ep = e & 15, wsel = ep >> 3, pp = ep & 7, t = pp >> 1, elem = pp & 1;
        const int s = rowsel * 2 + half + elem * 4;
        const uint32_t word = *reinterpret_cast<const uint32_t*>(rec + 16 * (4 * g + t) + 4 * (2 * bb + wsel));
        w[u] = (float)((int)((word >> (4 * s)) & 15u) - 8) * d;
    }
    return make_float4(w[0], w[1], w[2], w[3]);
}

// Activation row -> per-block power-of-two scaled fp16 B fragments and the
// block's (offset constant, 1/scale), as the GEMV record math expects (M = 1).
// Source: x (fp32, written by other CTAs: read through L2) or, for the first
// layer, the embedding row of `tok`; in that case the groups with
// f % G == b are also stored to x for the later residual.  Returns this
// thread's sum of x^2.
__device__ __forceinline__ float ps_convert(const PsArgs& P, const float* x, bool from_emb, int64_t tok, int64_t k,
                                            int32_t kc, uint32_t* s_bs32, float2* s_cb, int64_t b, int64_t G)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nf = (int)(k >> 2), nfp = kc * 16;
    const int32_t kc_emb = (int32_t)((P.dim + 63) / 64);
    float sq = 0.f;
    for (int f0 = warp * 32; f0 < nfp; f0 += kPsBatch * kPsThreads) {
        float4 v[kPsBatch];
#pragma unroll
        for (int u = 0; u < kPsBatch; ++u) {
            const int f = f0 + u * kPsThreads + lane;
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (f < nf) {
                if (from_emb) {
                    v[u] = ps_emb_f4(P.emb, kc_emb, tok, f);
                    if (f % G == b) reinterpret_cast<float4*>(P.x)[f] = v[u];
                } else {
                    v[u] = __ldcg(reinterpret_cast<const float4*>(x) + f);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kPsBatch; ++u) {
            const int fb = f0 + u * kPsThreads;                  // warp-uniform
            if (fb >= nfp) break;
            const int f = fb + lane;
            const float4 xg = v[u];
            sq = fmaf(xg.x, xg.x, sq);
            sq = fmaf(xg.y, xg.y, sq);
            sq = fmaf(xg.z, xg.z, sq);
            sq = fmaf(xg.w, xg.w, sq);
            float am = fmaxf(fmaxf(fabsf(xg.x), fabsf(xg.y)), fmaxf(fabsf(xg.z), fabsf(xg.w)));
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 8));
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 16));    // max over the warp's 128 columns
            int E = (int)((__float_as_uint(am) >> 23) & 0xFFu);
            E = E < 14 ? 14 : E;
            const float sc = __uint_as_float((uint32_t)(267 - E) << 23);
            const float inv = __uint_as_float((uint32_t)(E - 13) << 23);
            const __half2 h01 = __floats2half2_rn(xg.x * sc, xg.y * sc);
            const __half2 h23 = __floats2half2_rn(xg.z * sc, xg.w * sc);
            const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
            float s = (f01.x + f01.y) + (f23.x + f23.y);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);             // sum over one 16-column half-block
            const float shi = __shfl_down_sync(0xffffffffu, s, 4);
            if (f < nfp) {
                const int blk = f >> 3, q = f & 7;
                const int word = blk * 16 + 2 * (q & 1) * 4 + (q >> 2) * 2 + ((q & 3) >> 1);
                s_bs32[word] = *reinterpret_cast<const uint32_t*>(&h01);
                s_bs32[word + 4] = *reinterpret_cast<const uint32_t*>(&h23);
                if (q == 0) {
                    const float c = -(1032.0f * s + 72.0f * shi);
                    reinterpret_cast<float4*>(s_cb)[blk] = make_float4(c, inv, c, inv);
                }
            }
        }
    }
    return sq;
}

// ------------------------------------------------------------ epilogues
// Values of one finished 16-row tile in the MMA layout (lane (g, t): rows g
// and g + 8; every t holds the same values at M = 1); lanes with t == 0 write.
struct PsBest {
    float v;
    int32_t i;
};

// Rotary embedding of a q or k tile's rows g and g + 8 (base: the region's
// first row); rows 2i and 2i + 1 of a head sit in lanes g and g ^ 1.  Whole
// warp; not inlined, so that only steps with RoPE on pay for it.
__device__ __noinline__ float2 ps_rope(float2 v, int64_t tile, int g, int64_t base, int64_t pos, float theta)
{
    const float p0 = __shfl_xor_sync(0xffffffffu, v.x, 4), p1 = __shfl_xor_sync(0xffffffffu, v.y, 4);
    return make_float2(rope_rotate(v.x, p0, (tile * 16 + g - base) % kPsHd, kPsHd, pos, theta),
                       rope_rotate(v.y, p1, (tile * 16 + g + 8 - base) % kPsHd, kPsHd, pos, theta));
}

// res0 / res1: the residual of rows g and g + 8 (WO, W2), loaded ahead.
__device__ __forceinline__ void ps_epilogue(const PsArgs& P, const PsPhase& f, int64_t tile, float v0, float v1,
                                            float rr, int64_t pos, PsBest& best, float res0, float res1)
{
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    float val[2] = {v0 * rr, v1 * rr};
    if (f.kind == PS_QKV && P.rope > 0.f && tile * 16 < P.q_dim + P.kv_dim) {
        const float2 r = ps_rope(make_float2(val[0], val[1]), tile, g, tile * 16 < P.q_dim ? 0 : P.q_dim, pos, P.rope);
        val[0] = r.x;
        val[1] = r.y;
    }
    if (f.kind == PS_LM) {
        float bv = -INFINITY;
        int32_t bi = 0x7fffffff;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            const int64_t row = tile * 16 + g + 8 * hh;
            if (row < f.n) {
                if (t == 0) P.logits[row] = val[hh];
                if (argmax_better(val[hh], (int32_t)row, bv, bi)) { bv = val[hh]; bi = (int32_t)row; }
            }
        }
#pragma unroll
        for (int o = 4; o <= 16; o <<= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (argmax_better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
        }
        if (argmax_better(bv, bi, best.v, best.i)) { best.v = bv; best.i = bi; }
        return;
    }
    if (t != 0) return;
    if (f.kind == PS_W13) {
        const int64_t row = tile * 16 + g;                   // gate row g pairs with up row g + 8
        if (row < f.n) P.act[tile * 8 + g] = silu_f(val[0]) * val[1];
        return;
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        const int64_t row = tile * 16 + g + 8 * hh;
        if (row >= f.n) continue;
        if (f.kind == PS_QKV) {
            P.qkv[row] = val[hh];
            const int64_t rel = row - P.q_dim;
            if (rel >= 0) {
                const bool is_v = rel >= P.kv_dim;
                const int64_t rw = is_v ? rel - P.kv_dim : rel;
                const int64_t head = rw / kPsHd, col = rw - head * kPsHd;
                uint16_t* cache = is_v ? P.vc[f.layer] : P.kc[f.layer];
                cache[(head * P.window + pos % P.window) * kPsHd + col] = f32_to_bf16_bits(val[hh]);
            }
        } else if (f.kind == PS_WO) {
            P.h[row] = (hh ? res1 : res0) + val[hh];
        } else {                                             // PS_W2
            P.x[row] = (hh ? res1 : res0) + val[hh];
        }
    }
}

// ------------------------------------------------------------ GEMV phase
// The warp's stages of one GEMV phase, then the tiles it shares with other
// warps of the CTA (summed in warp order from shared memory by the warp that
// holds the tile's first record).  A CTA owns whole tiles, so no tile is
// ever split between CTAs.  `ok` turns false when a wait gave up; the warp
// then skips work but still reaches every CTA barrier.
__device__ __forceinline__ void ps_gemv_phase(const PsArgs& P, const PsWs& W, const PsPhase& f, int ph,
                                              PsRing& ring, int nph, int64_t b, int64_t G, int64_t nch, int64_t pos,
                                              uint8_t* smem, const PsSmem& SL, PsBest& best, float rr, bool& ok)
{
    (void)W;
    (void)ph;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int kc = f.kc;
    float* s_piece = reinterpret_cast<float*>(smem + SL.piece);
    const uint32_t tk = smem_token();
    const uint32_t bs_a = smem_addr(smem + SL.act) + tk;
    const uint32_t cb_a = bs_a + (uint32_t)kc * 128u;
    const int64_t wb = f.wb, we = f.we;

    // The residual of the first two tiles that start in this warp's range
    // (the tiles it finishes), loaded before the main loop.
    const float* res_src = f.kind == PS_WO ? P.x : f.kind == PS_W2 ? P.h : nullptr;
    const int64_t t_a = (wb + kc - 1) / kc;
    float res[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    if (res_src && we > wb) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            if ((t_a + i) * kc >= we) break;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const int64_t row = (t_a + i) * 16 + g + 8 * hh;
                if (row < f.n) res[i][hh] = __ldcg(res_src + row);
            }
        }
    }
    auto res_of = [&](int64_t tile, int hh) -> float {
        if (!res_src) return 0.f;
        if (tile == t_a) return res[0][hh];
        if (tile == t_a + 1) return res[1][hh];
        const int64_t row = tile * 16 + g + 8 * hh;
        return row < f.n ? __ldcg(res_src + row) : 0.f;
    };

    // ---- main loop: this warp's records.  A stage is cut at tile ends; each
    // run of records inside one tile goes in groups of four (their MMAs in
    // flight together, chunk addresses as constant offsets) straight into the
    // tile's sums, and the tile is closed once, at its end or the range end.
    if (we > wb && ok) {
        int64_t tile = wb / kc;
        int cin = (int)(wb - tile * kc);
        bool whole = (cin == 0);
        float acc0 = 0.f, acc2 = 0.f;
        int64_t r = wb;
        for (int j = 0; j < f.nst; ++j) {
            if (!ps_ring_wait(ring, 0x501)) {
                ok = false;
                ps_raise(P, W, 0x501);
                break;
            }
            const uint32_t base = smem_addr(ring.base) + (ring.consumed % kPsStages) * kPsStageBytes + smem_token();
            const int nrec = (int)min64(kPsRecs, we - r);
            for (int u = 0; u < nrec;) {
                const int run = nrec - u < kc - cin ? nrec - u : kc - cin;     // records up to the tile end
                const uint32_t rec_a = base + (uint32_t)u * kChunkBytes;
                const uint32_t bsb = bs_a + 128u * (uint32_t)cin + 16u * (uint32_t)t;
                const uint32_t cbc = cb_a + 32u * (uint32_t)cin;
#pragma unroll 1
                for (int v0 = 0; v0 < run; v0 += 4) {
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        if (v0 + v >= run) break;
                        const uint32_t o = (uint32_t)(v0 + v);
                        const uint4 qv = lds128(rec_a + o * kChunkBytes + 16 * lane);
                        const uint2 e = lds64(rec_a + o * kChunkBytes + kChunkQsBytes + 8 * g);
                        gemv_record_m1(qv, e, bsb + 128u * o, cbc + 32u * o, acc0, acc2);
                    }
                }
                u += run;
                r += run;
                cin += run;
                if (cin == kc || r == we) {
                    if (whole && cin == kc) {
                        ps_epilogue(P, f, tile, acc0, acc2, rr, pos, best, res_of(tile, 0), res_of(tile, 1));
                    } else if (t == 0) {
                        // a piece of a tile shared with other warps: slot 0 is the warp's first tile
                        const int slot = (tile == wb / kc) ? 0 : 1;
                        s_piece[(warp * 2 + slot) * 16 + g] = acc0;
                        s_piece[(warp * 2 + slot) * 16 + g + 8] = acc2;
                    }
                    acc0 = acc2 = 0.f;
                    cin = 0;
                    ++tile;
                    whole = true;
                }
            }
            __syncwarp();
            ++ring.consumed;
            ps_ring_fill(P, ring, nph, b, G, warp, lane, nch, ph);
        }
    }
    named_barrier(1, kPsThreads);
    if (!ok || we <= wb) return;

    // ---- tiles cut between warps: the warp holding the tile's first record
    // sums the pieces in warp order and finishes the tile
    const int64_t cb = f.cb, ce = f.ce, Rb = ce - cb;
    const int64_t lt = (we - 1) / kc;
    const int64_t t0 = lt * kc, t1 = t0 + kc;
    if (t0 >= wb && t1 > we) {
        const int wl = (int)(((t1 - cb) * kPsWarps - 1) / Rb);       // warp holding the tile's last record
        float s0 = 0.f, s2 = 0.f;
        for (int w2 = warp; w2 <= wl; ++w2) {
            const int64_t b2 = cb + Rb * w2 / kPsWarps, e2 = cb + Rb * (w2 + 1) / kPsWarps;
            if (e2 <= b2) continue;
            const int slot = (w2 == warp) ? (lt == wb / kc ? 0 : 1) : 0;
            s0 += s_piece[(w2 * 2 + slot) * 16 + g];
            s2 += s_piece[(w2 * 2 + slot) * 16 + g + 8];
        }
        ps_epilogue(P, f, lt, s0, s2, rr, pos, best, res_of(lt, 0), res_of(lt, 1));
    }
}

// ------------------------------------------------------------ ATTN phase
// The CTA's units, head by head; at each head's end the warps' (m, l, O)
// states are merged in shared memory.  A head inside this CTA is finished
// here; a head shared with other CTAs goes out as one record per CTA, and
// the last CTA to arrive combines the records in CTA order.
__device__ __forceinline__ void ps_attn_phase(const PsArgs& P, const PsWs& W, const PsPhase& f, PsRing& ring, int nph, int64_t b,
                              int64_t G, int64_t nch, int64_t pos, int64_t n_valid, uint8_t* smem, const PsSmem& SL,
                              bool& ok)
{
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t = lane & 3;
    const int group = P.group, Wn = P.window, l = f.layer;
    const int64_t new_slot = pos % Wn;
    float* merge = reinterpret_cast<float*>(smem + SL.act);
    const int mstride = group * kPsHd + 2 * group;
    int32_t* s_flag = reinterpret_cast<int32_t*>(smem + SL.flags) + 1;
    float* recs = reinterpret_cast<float*>(P.ws + W.recs);
    if (f.ce <= f.cb) return;
    const int64_t h0 = f.cb / nch, h1 = (f.ce - 1) / nch;
    int j = 0;
    for (int64_t hh = h0; hh <= h1; ++hh) {
        float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
        float o[8][4];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) o[jj][0] = o[jj][1] = o[jj][2] = o[jj][3] = 0.f;
        uint32_t qh[8][2], ql[8][2];
        bool have_q = false;
        // the head's queries, written by the QKV phase of other CTAs: one round
        // of loads for the whole CTA into shared memory
        float* s_q = reinterpret_cast<float*>(smem + SL.q);
        for (int i = tid; i < group * kPsHd; i += kPsThreads) s_q[i] = __ldcg(P.qkv + hh * group * kPsHd + i);
        named_barrier(1, kPsThreads);
        while (ok && j < f.nst / 2) {
            const int64_t unit = f.cb + warp + (int64_t)kPsWarps * j;
            if (unit / nch != hh) break;
            if (!have_q) {
                // q' = q * scale * log2(e), split into bf16 hi + lo B fragments (heads >= group are zero)
                const bool okq = g < group;
                const float* qr = s_q + (okq ? g : 0) * kPsHd;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
                    if (okq) {
                        const float2 a0 = *reinterpret_cast<const float2*>(qr + 16 * kk + 2 * t);
                        const float2 a1 = *reinterpret_cast<const float2*>(qr + 16 * kk + 2 * t + 8);
                        v0 = a0.x * P.qscale;
                        v1 = a0.y * P.qscale;
                        v2 = a1.x * P.qscale;
                        v3 = a1.y * P.qscale;
                    }
                    split_bf16x2(v0, v1, qh[kk][0], ql[kk][0]);
                    split_bf16x2(v2, v3, qh[kk][1], ql[kk][1]);
                }
                have_q = true;
            }
            if (!ps_ring_wait(ring, 0x502) || !ps_ring_wait(ring, 0x502, 1)) {
                ok = false;
                ps_raise(P, W, 0x502);
                break;
            }
            uint8_t* stK = ring.base + (ring.consumed % kPsStages) * kPsStageBytes;
            uint8_t* stV = ring.base + ((ring.consumed + 1) % kPsStages) * kPsStageBytes;
            const uint32_t sK = smem_addr(stK), sV = smem_addr(stV);
            const int64_t slot0 = (unit - hh * nch) * kPsUnit;   // first cache slot of the unit

            // generic-proxy fix-ups of the TMA-written stage
            bool touched = false;
            if (new_slot >= slot0 && new_slot < slot0 + kPsUnit) {
                // the newest row (K and V, 4 x 128 bytes), written this step by the QKV phase
                const uint32_t rr = (uint32_t)(new_slot - slot0);
                const int part = lane >> 3, u8 = lane & 7;             // K lo, K hi, V lo, V hi
                const uint16_t* src = (part < 2 ? P.kc[l] : P.vc[l]) + (hh * Wn + new_slot) * kPsHd + (part & 1) * 64 +
                                      u8 * 8;
                const uint4 v = __ldcg(reinterpret_cast<const uint4*>(src));
                *reinterpret_cast<uint4*>((part < 2 ? stK : stV) + (part & 1) * 2048 + sw128_offset(rr, (uint32_t)u8)) =
                    v;
                touched = true;
            }
            if (slot0 + kPsUnit > n_valid) {
                // slots past the valid range may hold anything (NaN included): zero their V rows
                for (int i = lane; i < 16 * 16; i += 32) {
                    const int rr = i >> 4, half = (i >> 3) & 1, u8 = i & 7;
                    if (slot0 + rr >= n_valid)
                        *reinterpret_cast<uint4*>(stV + half * 2048 + sw128_offset((uint32_t)rr, (uint32_t)u8)) =
                            make_uint4(0u, 0u, 0u, 0u);
                }
                touched = true;
            }
            __syncwarp();

            // ---- S = K q'^T for the 16 slots (four accumulator chains)
            float sa[4][4];
#pragma unroll
            for (int u = 0; u < 4; ++u) sa[u][0] = sa[u][1] = sa[u][2] = sa[u][3] = 0.f;
            {
                const int mi = lane >> 3;
                const uint32_t rr = (uint32_t)(8 * (mi & 1) + (lane & 7));
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t tile = sK + (kk >> 2) * 2048;
                    uint32_t ak[4];
                    ldsm_x4(ak, tile + sw128_offset(rr, (uint32_t)(2 * (kk & 3) + (mi >> 1))));
                    mma_bf16_16816(sa[(kk & 1) * 2 + 0], ak, qh[kk][0], qh[kk][1], sa[(kk & 1) * 2 + 0]);
                    mma_bf16_16816(sa[(kk & 1) * 2 + 1], ak, ql[kk][0], ql[kk][1], sa[(kk & 1) * 2 + 1]);
                }
            }
            float sv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sv[e] = (sa[0][e] + sa[1][e]) + (sa[2][e] + sa[3][e]);
                if (slot0 + g + 8 * (e >> 1) >= n_valid) sv[e] = -INFINITY;
            }
            // ---- online softmax per head (exp2 domain), reduced over the 8 lanes of equal t
            float pr[4], corr[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                float mx = fmaxf(sv[u], sv[u + 2]);
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
                const float m_new = fmaxf(m_run[u], mx);
                if (m_new == -INFINITY) {
                    corr[u] = 1.f;
                    pr[u] = pr[u + 2] = 0.f;
                } else {
                    corr[u] = exp2f(m_run[u] - m_new);
                    pr[u] = exp2f(sv[u] - m_new);
                    pr[u + 2] = exp2f(sv[u + 2] - m_new);
                }
                float ps = pr[u] + pr[u + 2];
                ps += __shfl_xor_sync(0xffffffffu, ps, 4);
                ps += __shfl_xor_sync(0xffffffffu, ps, 8);
                ps += __shfl_xor_sync(0xffffffffu, ps, 16);
                l_run[u] = l_run[u] * corr[u] + ps;
                m_run[u] = m_new;
            }
            // ---- P into B-fragment layout: lane (g, t) needs P[slot 2t (+1) (+8)][head g]
            uint32_t bh[2], bl[2];
            {
                const int src0 = (2 * t) * 4 + (g >> 1), src1 = (2 * t + 1) * 4 + (g >> 1);
                const bool odd = g & 1;
                const float x00 = __shfl_sync(0xffffffffu, pr[0], src0), x01 = __shfl_sync(0xffffffffu, pr[1], src0);
                const float x10 = __shfl_sync(0xffffffffu, pr[0], src1), x11 = __shfl_sync(0xffffffffu, pr[1], src1);
                const float y00 = __shfl_sync(0xffffffffu, pr[2], src0), y01 = __shfl_sync(0xffffffffu, pr[3], src0);
                const float y10 = __shfl_sync(0xffffffffu, pr[2], src1), y11 = __shfl_sync(0xffffffffu, pr[3], src1);
                split_bf16x2(odd ? x01 : x00, odd ? x11 : x10, bh[0], bl[0]);
                split_bf16x2(odd ? y01 : y00, odd ? y11 : y10, bh[1], bl[1]);
            }
            // ---- O^T = O^T * corr + V^T P: 8 dim tiles of 16, A = V^T by ldmatrix.trans
            {
                const int mi = lane >> 3;
                const uint32_t rr = (uint32_t)(8 * (mi >> 1) + (lane & 7));
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const uint32_t tile = sV + (jj >> 2) * 2048;
                    uint32_t av[4];
                    ldsm_x4_trans(av, tile + sw128_offset(rr, (uint32_t)(2 * (jj & 3) + (mi & 1))));
                    float c[4] = {o[jj][0] * corr[0], o[jj][1] * corr[1], o[jj][2] * corr[0], o[jj][3] * corr[1]};
                    mma_bf16_16816(c, av, bh[0], bh[1], c);
                    mma_bf16_16816(c, av, bl[0], bl[1], c);
                    o[jj][0] = c[0];
                    o[jj][1] = c[1];
                    o[jj][2] = c[2];
                    o[jj][3] = c[3];
                }
            }
            // generic writes into a buffer the async proxy refills next: order them first
            if (touched) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            ring.consumed += 2;
            ++j;
            ps_ring_fill(P, ring, nph, b, G, warp, lane, nch, (int)f.layer * 5 + 1);
        }

        // ---- this warp's state for head hh -> merge buffer
        float* mw = merge + warp * mstride;
        if (g == 0) {
#pragma unroll
            for (int u = 0; u < 2; ++u)
                if (2 * t + u < group) {
                    mw[group * kPsHd + (2 * t + u) * 2 + 0] = m_run[u];
                    mw[group * kPsHd + (2 * t + u) * 2 + 1] = l_run[u];
                }
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
            if (2 * t < group) {
                mw[(2 * t) * kPsHd + 16 * jj + g] = o[jj][0];
                mw[(2 * t) * kPsHd + 16 * jj + 8 + g] = o[jj][2];
            }
            if (2 * t + 1 < group) {
                mw[(2 * t + 1) * kPsHd + 16 * jj + g] = o[jj][1];
                mw[(2 * t + 1) * kPsHd + 16 * jj + 8 + g] = o[jj][3];
            }
        }
        named_barrier(1, kPsThreads);

        // ---- merge the warps (warp order), then finish the head or publish the CTA's record
        const bool inside = hh * nch >= f.cb && (hh + 1) * nch <= f.ce;
        const int64_t fc = f.hfirst, lc = f.hfirst + f.hcnt - 1;   // the CTAs of this kv head
        float* rec = recs + ((size_t)hh * W.rmax + (size_t)(b - fc)) * W.rec_floats;
        for (int i = tid; i < group * kPsHd; i += kPsThreads) {
            const int hi = i / kPsHd, cc = i - hi * kPsHd;
            float M = -INFINITY;
            for (int w = 0; w < kPsWarps; ++w) M = fmaxf(M, merge[w * mstride + group * kPsHd + hi * 2]);
            float O = 0.f, L = 0.f;
            for (int w = 0; w < kPsWarps; ++w) {
                const float* m2 = merge + w * mstride;
                const float mv = m2[group * kPsHd + hi * 2];
                const float fct = (mv == -INFINITY) ? 0.f : exp2f(mv - M);
                O += fct * m2[hi * kPsHd + cc];
                L += fct * m2[group * kPsHd + hi * 2 + 1];
            }
            if (inside) {
                P.attn[(hh * group + hi) * kPsHd + cc] = O / L;
            } else {
                __stcg(rec + hi * kPsHd + cc, O);
                if (cc == 0) {
                    __stcg(rec + group * kPsHd + hi * 2 + 0, M);
                    __stcg(rec + group * kPsHd + hi * 2 + 1, L);
                }
            }
        }
        if (!inside) {
            named_barrier(1, kPsThreads);                 // every record store of the CTA is issued
            if (tid == kPsSyncThread) {
                __threadfence();                          // ... and published before the arrival
                uint32_t ncon = 0;
                for (int64_t c = 0; c < f.hcnt; ++c)
                    ncon += split_begin(c, nch, f.hcnt) < split_begin(c + 1, nch, f.hcnt) ? 1u : 0u;
                uint32_t* ctr = reinterpret_cast<uint32_t*>(P.ws + W.attncnt) + (size_t)l * P.n_kv + hh;
                const uint32_t old = atom_add_acq_rel_gpu(ctr, 1u);
                const int last = old + 1u == ncon;
                if (last) atomicExch(ctr, 0u);
                *s_flag = last;
            }
            named_barrier(1, kPsThreads);
            if (*reinterpret_cast<volatile int32_t*>(s_flag)) {
                // last CTA of the head: fold the CTAs' records in CTA order.  Each
                // thread first issues the loads of its outputs' O values of every
                // record (they do not depend on m), then the (m, l) pairs go
                // through shared memory, where the factors exp2(m - M) replace m.
                __threadfence();
                const float* base = recs + (size_t)hh * W.rmax * W.rec_floats;
                const int nrec = (int)(lc - fc + 1);
                float* s_ml = merge;                              // [nrec][group] x (m or factor, l)
                float* s_L = merge + 2 * nrec * group;
                constexpr int kFold = 24;                          // records of one round of O loads
                for (int i0 = 0; i0 < group * kPsHd; i0 += kPsThreads) {
                    const int i = i0 + tid;
                    const int hi = i < group * kPsHd ? i / kPsHd : 0, cc = i - hi * kPsHd;
                    float O = 0.f;
                    for (int r0 = 0; r0 < nrec; r0 += kFold) {
                        float ov[kFold];
#pragma unroll
                        for (int u = 0; u < kFold; ++u)
                            ov[u] = (i < group * kPsHd && r0 + u < nrec)
                                        ? __ldcg(base + (size_t)(r0 + u) * W.rec_floats + hi * kPsHd + cc) : 0.f;
                        if (i0 == 0 && r0 == 0) {
                            for (int q = tid; q < nrec * group; q += kPsThreads) {
                                const int r = q / group, h2 = q - r * group;
                                float2 ml = make_float2(-INFINITY, 0.f);   // a CTA with no units wrote no record
                                if (split_begin(r, nch, f.hcnt) < split_begin(r + 1, nch, f.hcnt))
                                    ml = __ldcg(reinterpret_cast<const float2*>(base + (size_t)r * W.rec_floats +
                                                                               group * kPsHd) + h2);
                                s_ml[2 * q] = ml.x;
                                s_ml[2 * q + 1] = ml.y;
                            }
                            named_barrier(1, kPsThreads);
                            if (tid < group) {
                                float M = -INFINITY, L = 0.f;
                                for (int r = 0; r < nrec; ++r) M = fmaxf(M, s_ml[2 * (r * group + tid)]);
                                for (int r = 0; r < nrec; ++r) {
                                    const float mv = s_ml[2 * (r * group + tid)];
                                    const float fct = (mv == -INFINITY) ? 0.f : exp2f(mv - M);
                                    s_ml[2 * (r * group + tid)] = fct;
                                    L += fct * s_ml[2 * (r * group + tid) + 1];
                                }
                                s_L[tid] = L;
                            }
                            named_barrier(1, kPsThreads);
                        }
#pragma unroll
                        for (int u = 0; u < kFold; ++u) {
                            if (r0 + u >= nrec) break;
                            const float fct = s_ml[2 * ((r0 + u) * group + hi)];
                            O += fct != 0.f ? fct * ov[u] : 0.f;   // an empty CTA's slot may hold anything
                        }
                    }
                    if (i < group * kPsHd) P.attn[(hh * group + hi) * kPsHd + cc] = O / s_L[hi];
                }
            }
        }
        named_barrier(1, kPsThreads);                     // the merge buffer is reused by the next head
    }
}

// ------------------------------------------------------------ the step
__global__ void __launch_bounds__(kPsThreads, 1) decoder_step_kernel(const __grid_constant__ PsArgs P)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const PsSmem SL = ps_smem_layout(P.act_bytes);
    const int64_t G = gridDim.x, b = blockIdx.x;
    const PsWs W = ps_ws_layout((int)G, P.n_layers, P.n_kv, P.group);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int32_t* s_flag = reinterpret_cast<int32_t*>(smem + SL.flags);
    float* s_sq = reinterpret_cast<float*>(smem + SL.sq);
    float* s_best_v = reinterpret_cast<float*>(smem + SL.best_v);
    int32_t* s_best_i = reinterpret_cast<int32_t*>(smem + SL.best_i);
    uint32_t* s_bs32 = reinterpret_cast<uint32_t*>(smem + SL.act);

    // position and token of this step (written by the previous step's kernel)
    const int64_t pos = *P.pos;
    const int64_t n_valid = pos + 1 < P.window ? pos + 1 : P.window;
    const int64_t nch = (n_valid + kPsUnit - 1) / kPsUnit;
    int64_t tok = *P.token;
    if (tok < 0 || tok >= P.vocab) {
        if (tid == 0 && b == 0) atomicCAS(&g_vox_device_status, 0, 0x5D0);
        tok = 0;
    }
    // this launch's phases [ph_begin, nph): the whole step, or one segment of
    // GEMV phases between two attention launches
    const int nph_all = 5 * P.n_layers + 1;
    const int nph = P.ph_end;

    PsRing ring;
    ring.base = smem + SL.ring + (uint32_t)warp * kPsStages * kPsStageBytes;
    ring.bars = reinterpret_cast<uint64_t*>(smem + SL.bars) + warp * kPsStages;
    if (lane == 0) {
        for (int s = 0; s < kPsStages; ++s) mbar_init(&ring.bars[s], 1);
        if (warp == 0) mbar_init(reinterpret_cast<uint64_t*>(smem + SL.never), 1);
        fence_mbar_init();
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncwarp();
    ring.issued = ring.consumed = 0;
    ring.cur.ph = P.ph_begin;
    ring.cur.idx = 0;
    ring.cur.f = ps_phase(P, P.ph_begin, b, G, warp, nch);
    ps_ring_fill(P, ring, nph, b, G, warp, lane, nch, P.ph_begin);

    bool ok = true;
    if (P.test_withhold && b == 0 && warp == 0) {
        // test hook: a wait that can only run out (an mbarrier nothing completes),
        // bounded at 0.2 s so that it gives up before any grid barrier would
        uint64_t* never = reinterpret_cast<uint64_t*>(smem + SL.never);
        const uint64_t t0 = global_ns();
        bool done = false;
        while (!done && global_ns() - t0 < 200000000ull) done = mbar_test_wait(never, 0);
        if (!done) {
            ok = false;
            ps_raise(P, W, 0x530);
        }
    }
    PsBest best = {-INFINITY, 0x7fffffff};
    int ph = P.ph_begin;
    for (; ph < nph; ++ph) {
        if (ph > P.ph_begin && !ps_grid_barrier(P, W, s_flag, 0x510)) break;
        const PsPhase f = ps_phase(P, ph, b, G, warp, nch);
        if (f.kind == PS_ATTN) {
            if (kPsPrefetch < kPsStages) ps_ring_fill(P, ring, nph, b, G, warp, lane, nch, ph);
            ps_attn_phase(P, W, f, ring, nph, b, G, nch, pos, n_valid, smem, SL, ok);
            continue;
        }
        // prologue: the phase's input vector -> fp16 fragments in shared memory
        const float* xin = f.kind == PS_WO ? P.attn : f.kind == PS_W13 ? P.h : f.kind == PS_W2 ? P.act : P.x;
        const bool from_emb = f.kind == PS_QKV && f.layer == 0;
        float sq = ps_convert(P, xin, from_emb, tok, f.k, f.kc, s_bs32,
                              reinterpret_cast<float2*>(smem + SL.act + (uint32_t)f.kc * 128u), b, G);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
        if (lane == 0) s_sq[warp] = sq;
        __syncthreads();
        // the rest of this phase's stages, once the activation loads are done
        if (kPsPrefetch < kPsStages) ps_ring_fill(P, ring, nph, b, G, warp, lane, nch, ph);
        float rr = 1.0f;
        if (f.kind == PS_QKV || f.kind == PS_W13 || f.kind == PS_LM) {
            float ssq = 0.f;
            for (int w = 0; w < kPsWarps; ++w) ssq += s_sq[w];
            rr = 1.0f / sqrtf(ssq / (float)f.k + P.eps);
        }
        ps_gemv_phase(P, W, f, ph, ring, nph, b, G, nch, pos, smem, SL, best, rr, ok);
    }

    // ---- greedy argmax: warps -> CTA -> one 64-bit atomic max; the last CTA
    // to arrive writes the token, clears the key and advances the position
    if (ph == nph && nph == nph_all) {
        if (lane == 0) {
            s_best_v[warp] = best.v;
            s_best_i[warp] = best.i;
        }
        __syncthreads();
        if (tid == kPsSyncThread && !ld_relaxed_s32(reinterpret_cast<const int32_t*>(P.ws + W.abort))) {
            float bv = -INFINITY;
            int32_t bi = 0x7fffffff;
            for (int w = 0; w < kPsWarps; ++w)
                if (argmax_better(s_best_v[w], s_best_i[w], bv, bi)) {
                    bv = s_best_v[w];
                    bi = s_best_i[w];
                }
            unsigned long long* key = reinterpret_cast<unsigned long long*>(P.ws + W.amax_key);
            uint32_t* cnt = reinterpret_cast<uint32_t*>(P.ws + W.amax_cnt);
            if (bi != 0x7fffffff) atomicMax(key, argmax_key(bv, bi));
            __threadfence();
            if (atom_add_acq_rel_gpu(cnt, 1u) == (uint32_t)G - 1) {
                const unsigned long long k = atomicExch(key, 0ull);
                *P.token = (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFull));
                *cnt = 0u;
                *P.pos = pos + 1;
            }
        }
    }

    // ---- copies still in flight (only after a wait gave up): let them land
    if (lane == 0)
        for (uint32_t u = ring.consumed; u < ring.issued; ++u)
            mbar_wait_bounded(&ring.bars[u % kPsStages], (u / kPsStages) & 1u, 0x520);
}

// ------------------------------------------------------------ host side
size_t decoder_step_ws_bytes(int n_layers, int n_kv, int group)
{
    return ps_ws_layout(device_sm_count(), n_layers, n_kv, group).total;
}

// Why the persistent step cannot take a decoder, or NULL.
const char* decoder_step_unsupported(const vox_decoder* d)
{
    if (d->n_layers > kPsMaxLayers) return "more than 32 layers";
    if (d->head_dim != kPsHd) return "head_dim is not 128";
    if (d->n_q_heads / d->n_kv_heads > kPsMaxGroup) return "more than 4 query heads per kv head";
    if (d->n_kv_heads > device_sm_count()) return "more kv heads than SMs";
    if (d->dim % 4 || d->ffn % 8) return "dim not a multiple of 4 or ffn not a multiple of 8";
    return nullptr;
}

static uint32_t ps_act_bytes(const vox_decoder* d)
{
    const int64_t kmax = d->dim > d->ffn ? (d->dim > (int64_t)d->n_q_heads * kPsHd ? d->dim : (int64_t)d->n_q_heads * kPsHd)
                                         : (d->ffn > (int64_t)d->n_q_heads * kPsHd ? d->ffn : (int64_t)d->n_q_heads * kPsHd);
    const int64_t kc = (kmax + 63) / 64;
    const int64_t gemv = kc * 128 + kc * 32;                   // B fragments, two constant quads per chunk
    const int group = d->n_q_heads / d->n_kv_heads;
    const int64_t mrg = (int64_t)kPsWarps * (group * kPsHd + 2 * group) * 4;
    return (uint32_t)(gemv > mrg ? gemv : mrg);
}

bool decoder_step_fits(const vox_decoder* d)
{
    return ps_smem_layout(ps_act_bytes(d)).total <= 227 * 1024;
}

vox_status launch_decoder_step(const vox_decoder* d, uint8_t* ws, cudaStream_t s, int ph_begin, int ph_end)
{
    PsArgs a;
    memset(&a, 0, sizeof(a));
    const int L = d->n_layers;
    for (int l = 0; l < L; ++l) {
        vox_status st = make_tmap_2d(&a.kmap[l], d->k_cache[l], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)kPsHd,
                                     (uint64_t)d->n_kv_heads * d->window, (uint64_t)kPsHd * 2, 64, kPsUnit,
                                     CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != VOX_OK) return st;
        st = make_tmap_2d(&a.vmap[l], d->v_cache[l], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)kPsHd,
                          (uint64_t)d->n_kv_heads * d->window, (uint64_t)kPsHd * 2, 64, kPsUnit,
                          CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != VOX_OK) return st;
        a.wqkv[l] = static_cast<const uint8_t*>(d->wqkv[l].data);
        a.wo[l] = static_cast<const uint8_t*>(d->wo[l].data);
        a.w13[l] = static_cast<const uint8_t*>(d->w13[l].data);
        a.w2[l] = static_cast<const uint8_t*>(d->w2[l].data);
        a.kc[l] = static_cast<uint16_t*>(d->k_cache[l]);
        a.vc[l] = static_cast<uint16_t*>(d->v_cache[l]);
    }
    a.emb = static_cast<const uint8_t*>(d->embedding.data);
    a.lm = static_cast<const uint8_t*>(d->lm_head.data);
    a.token = d->token;
    a.pos = d->pos;
    a.x = d->x;
    a.h = d->h;
    a.qkv = d->qkv;
    a.attn = d->attn;
    a.act = d->act;
    a.logits = d->logits;
    a.ws = ws;
    a.n_layers = L;
    a.dim = d->dim;
    a.q_dim = d->n_q_heads * kPsHd;
    a.kv_dim = d->n_kv_heads * kPsHd;
    a.ffn = d->ffn;
    a.vocab = d->vocab;
    a.n_kv = d->n_kv_heads;
    a.group = d->n_q_heads / d->n_kv_heads;
    a.window = d->window;
    a.eps = d->eps;
    a.qscale = (1.0f / sqrtf((float)kPsHd)) * 1.4426950408889634f;
    a.rope = d->rope_theta;
    a.ph_begin = ph_begin;
    a.ph_end = ph_end < 0 ? 5 * L + 1 : ph_end;
    a.act_bytes = ps_act_bytes(d);
    const char* hook = getenv("VOX_TEST_WITHHOLD_STAGE");      // test of the bounded waits only
    a.test_withhold = hook && hook[0] == '1';
    const PsSmem SL = ps_smem_layout(a.act_bytes);

    static std::atomic<unsigned long long> attr_done{0};
    vox_status st = smem_attr_per_device(reinterpret_cast<const void*>(decoder_step_kernel), 227 * 1024, attr_done);
    if (st != VOX_OK) return st;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decoder_step_kernel, kPsThreads, SL.total);
    if (e != cudaSuccess || per_sm < 1) {
        set_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
        return VOX_ERR_CUDA;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)device_sm_count());
    cfg.blockDim = dim3(kPsThreads);
    cfg.dynamicSmemBytes = SL.total;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, decoder_step_kernel, a);
    if (e != cudaSuccess) {
        set_cuda_error(e);
        return VOX_ERR_CUDA;
    }
    return VOX_OK;
}

}  // namespace vox
