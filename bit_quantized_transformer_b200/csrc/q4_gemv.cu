// K1: fused Q4_0 dequantise + GEMV for M <= 8 rows of activations.
//
// Computes y[i][j] = sum_c w[j][c] x[i][c] with w = (q - 8) * d (GGUF Q4_0,
// "Voxtral Mini 4B Realtime (Rust)", page 5 "Arquitetura") and dequantises in
// registers inside the matmul, with no separate dequant pass ("브라우저에서 도는
// 4B 음성인식: Voxtral Rust+WASM 구현 해부", section "F32(9GB) vs Q4 GGUF").
//
// Design (B200, HBM-bound at M <= 8):
//  * Work split: "stream-K" at warp granularity over the (16-row tile,
//    64-column chunk) records of the packed weight: every warp of the grid
//    owns one contiguous range of records, so every warp streams the same
//    number of bytes whatever n and k are, and no warp waits for another
//    while streaming.  Tiles a warp covers completely are finished from its
//    registers; the few tiles cut at range ends are summed once at the end,
//    in warp order through shared memory and, for tiles cut between CTAs, in
//    CTA order through the workspace by whichever CTA arrives last (atomic
//    count per tile): deterministic, and no CTA ever waits for another.
//  * Data movement: each lane's share of a record is exactly one 16-byte
//    load of codes and one 8-byte load of scales, straight into registers,
//    software-pipelined four records deep.  The first loads are issued before
//    griddepcontrol.wait, as weights never depend on upstream kernels.
//  * Dequantisation: each 32-bit word of codes gives four half2 A-fragment
//    registers with one LOP3 each (OR the nibble into the fraction of 1024.0
//    or 64.0, whose ulp is 1 at that nibble position: exact 1024+q / 64+q).
//    The constant offsets are removed through the MMA's C input, which is
//    preloaded with -(1032 * sum x_lo + 72 * sum x_hi) per block.
//  * Tensor cores: mma.sync m16n8k16 fp16 x fp16 -> fp32.  The activations
//    are scaled per row by an exact power of two into fp16 range first, and
//    the per-block scale d is applied in fp32 after each block's two MMAs.
#include "vox_internal.cuh"

namespace vox {

constexpr int kGemvWarps = 8;
constexpr int kGemvThreads = 32 * kGemvWarps;                 // 256
constexpr int kGemvPrefetch = 4;                              // records in flight per lane
constexpr int kGemvMaxCtas = 1024;

struct GemvArgs {
    const uint8_t* w;
    int64_t n, k;
    int32_t tiles, kc;
    const float* x;
    int64_t ldx;
    int32_t m;
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
};

// Shared-memory carve-up, computed identically on host and device.
struct GemvSmem {
    uint32_t bs, bias, part, part_tile, smul, inv, stats, best_v, best_i, flags, total;
};

__host__ __device__ inline GemvSmem gemv_smem_layout(int kc, int m)
{
    GemvSmem L;
    uint32_t off = 0;
    L.bs = off;        off += (uint32_t)kc * (uint32_t)m * 128u;
    L.bias = off;      off += ((uint32_t)kc * (uint32_t)m * 8u + 15u) & ~15u;
    L.part = off;      off += kGemvWarps * 2 * 32 * 4 * 4;
    L.part_tile = off; off += kGemvWarps * 2 * 8;
    L.smul = off;      off += 8 * 4;
    L.inv = off;       off += 8 * 4;
    L.stats = off;     off += 2 * kGemvWarps * 8 * 4;
    L.best_v = off;    off += kGemvWarps * 8 * 4;
    L.best_i = off;    off += kGemvWarps * 8 * 4;
    L.flags = off;     off += 16;
    L.total = off;
    return L;
}

// Workspace: two partial tiles per CTA, the per-CTA argmax candidates with
// one global arrival counter, then the per-tile arrival counters.  The
// fixed-size regions come first so that calls on matrices with different tile
// counts sharing one workspace only ever overlap counter with counter (all
// counters are back at zero when a call ends).
struct GemvWs {
    size_t partials, best_v, best_i, gcount, counters, total;
};

__host__ __device__ inline GemvWs gemv_ws_layout(int64_t tiles, int with_argmax)
{
    (void)with_argmax;
    GemvWs L;
    size_t off = 0;
    L.partials = off;  off += (size_t)kGemvMaxCtas * 2 * 16 * 8 * 4;
    L.best_v = off;    off += (size_t)kGemvMaxCtas * 8 * 4;
    L.best_i = off;    off += (size_t)kGemvMaxCtas * 8 * 4;
    L.gcount = off;    off += 256;
    L.counters = off;  off += (size_t)tiles * 4;
    L.total = (off + 255) & ~(size_t)255;
    return L;
}

size_t gemv_workspace_bytes(int64_t n, int64_t k, int op)
{
    (void)k;
    return gemv_ws_layout(ceil_div(n, 16), op == VOX_EP_ARGMAX).total;
}

__host__ __device__ __forceinline__ int64_t sk_begin(int64_t b, int64_t total, int64_t G)
{
    return b * total / G;
}

// Owner (CTA or warp) of the contiguous range containing record c.
__host__ __device__ __forceinline__ int64_t sk_owner(int64_t c, int64_t total, int64_t G)
{
    return ((c + 1) * G - 1) / total;
}

// "a beats b" for greedy argmax: NaN wins, then larger value, then lower index.
__device__ __forceinline__ bool argmax_better(float va, int32_t ia, float vb, int32_t ib)
{
    bool na = isnan(va), nb = isnan(vb);
    if (na != nb) return na;
    if (!na && va != vb) return va > vb;
    return ia < ib;
}

__device__ __forceinline__ float gelu_erf(float v)
{
    return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}

__device__ __forceinline__ float silu_f(float v)
{
    return v / (1.0f + expf(-v));
}

// One record's math for one warp: two Q4_0 blocks, each two m16n8k16 MMAs
// (low / high nibbles) started from the block's offset correction, then
// scaled by the block's d in fp32.  q, dd: this lane's code and scale words.
template <int MT>
__device__ __forceinline__ void gemv_record(uint4 q, uint2 dd, uint32_t bs, uint32_t bias, int nblk, int chunk,
                                            int m, int tok, int t, float (&acc)[4])
{
    const uint32_t M_P = 0x000F000Fu, M_Q = 0x00F000F0u, C_P = 0x64006400u, C_Q = 0x54005400u;
    const float2 d0 = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
    const float2 d1 = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
    const int blk0 = chunk * 2;
    float2 bias0, bias1;
    if (MT == 1) {
        const float2 bb = lds64f(bias + 4u * blk0);
        bias0 = make_float2(bb.x, 0.f);
        bias1 = make_float2(bb.y, 0.f);
    } else {
        const int t0 = 2 * t, t1 = 2 * t + 1;
        bias0 = make_float2(t0 < m ? lds32f(bias + 4u * (t0 * nblk + blk0)) : 0.f,
                            t1 < m ? lds32f(bias + 4u * (t1 * nblk + blk0)) : 0.f);
        bias1 = make_float2(t0 < m ? lds32f(bias + 4u * (t0 * nblk + blk0 + 1)) : 0.f,
                            t1 < m ? lds32f(bias + 4u * (t1 * nblk + blk0 + 1)) : 0.f);
    }
    const uint32_t bsb = bs + 4u * ((blk0 * (MT == 1 ? 1 : m) + tok) * 16 + t * 4);
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
        const uint4 B = lds128(bsb + 4u * bb * (MT == 1 ? 1 : m) * 16);
        const float2 bi = bb ? bias1 : bias0;
        const uint32_t w0 = bb ? q.z : q.x;
        const uint32_t w1 = bb ? q.w : q.y;
        const uint32_t w0s = w0 >> 8, w1s = w1 >> 8;
        float cc[4] = {bi.x, bi.y, bi.x, bi.y};
        const uint32_t alo[4] = {lop3_and_or(w0, M_P, C_P), lop3_and_or(w0s, M_P, C_P),
                                 lop3_and_or(w1, M_P, C_P), lop3_and_or(w1s, M_P, C_P)};
        mma_f16_16816(cc, alo, B.x, B.y, cc);
        const uint32_t ahi[4] = {lop3_and_or(w0, M_Q, C_Q), lop3_and_or(w0s, M_Q, C_Q),
                                 lop3_and_or(w1, M_Q, C_Q), lop3_and_or(w1s, M_Q, C_Q)};
        mma_f16_16816(cc, ahi, B.z, B.w, cc);
        const float dg = bb ? d1.x : d0.x, dg8 = bb ? d1.y : d0.y;
        acc[0] = fmaf(dg, cc[0], acc[0]);
        acc[2] = fmaf(dg8, cc[2], acc[2]);
        if (MT != 1) {
            acc[1] = fmaf(dg, cc[1], acc[1]);
            acc[3] = fmaf(dg8, cc[3], acc[3]);
        }
    }
}

// Epilogue of one finished 16-row tile from the MMA accumulator layout:
// lane (g, t) holds acc[2h + e] = tile row g + 8h, token 2t + e.
__device__ __forceinline__ void gemv_epilogue(const GemvArgs& a, int64_t tile, const float (&acc)[4], int g, int t,
                                              const float* s_inv, int64_t pos, float (&best_v)[2],
                                              int32_t (&best_i)[2])
{
    float v[4];
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 2; ++e) v[2 * h + e] = acc[2 * h + e] * s_inv[(2 * t + e) & 7];
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
                yr[row] = a.res[(int64_t)mt * a.ldr + row] + val;
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
                    const int64_t rr = rel < kvd ? rel : rel - kvd;
                    const int64_t head = rr / a.hd, col = rr - head * a.hd;
                    const int64_t slot_id = (pos + mt) % a.window;
                    cache[(head * a.window + slot_id) * a.hd + col] = f32_to_bf16_bits(val);
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
}

template <int MT>
__global__ void __launch_bounds__(kGemvThreads, 2) q4_gemv_kernel(const GemvArgs a)
{
    extern __shared__ __align__(128) uint8_t smem[];
    const int m = a.m;
    const int kc = a.kc;
    const GemvSmem L = gemv_smem_layout(kc, m);
    volatile int32_t* s_flag = reinterpret_cast<volatile int32_t*>(smem + L.flags);
    float* s_smul = reinterpret_cast<float*>(smem + L.smul);
    float* s_inv = reinterpret_cast<float*>(smem + L.inv);
    float* s_stats = reinterpret_cast<float*>(smem + L.stats);
    float* s_bias = reinterpret_cast<float*>(smem + L.bias);
    uint16_t* s_bs16 = reinterpret_cast<uint16_t*>(smem + L.bs);
    float* s_part = reinterpret_cast<float*>(smem + L.part);
    int64_t* s_part_tile = reinterpret_cast<int64_t*>(smem + L.part_tile);
    float* s_best_v = reinterpret_cast<float*>(smem + L.best_v);
    int32_t* s_best_i = reinterpret_cast<int32_t*>(smem + L.best_i);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int64_t G = gridDim.x, b = blockIdx.x;
    const int64_t GW = G * kGemvWarps, gw = b * kGemvWarps + warp;
    const int64_t total = (int64_t)a.tiles * kc;
    const int64_t cb = sk_begin(b, total, G), ce = sk_begin(b + 1, total, G);            // CTA range
    const int64_t wb = sk_begin(gw, total, GW), we = sk_begin(gw + 1, total, GW);        // warp range

    // first records of this warp, issued before the upstream kernels finish
    const uint8_t* wsrc = a.w + 16 * lane;
    const uint8_t* dsrc = a.w + kChunkQsBytes + 8 * g;
    uint4 rq[kGemvPrefetch];
    uint2 rd[kGemvPrefetch];
#pragma unroll
    for (int u = 0; u < kGemvPrefetch; ++u) {
        if (wb + u < we) {
            rq[u] = __ldg(reinterpret_cast<const uint4*>(wsrc + (wb + u) * kChunkBytes));
            rd[u] = __ldg(reinterpret_cast<const uint2*>(dsrc + (wb + u) * kChunkBytes));
        } else {
            rq[u] = make_uint4(0u, 0u, 0u, 0u);
            rd[u] = make_uint2(0u, 0u);
        }
    }

    pdl_wait();                              // x (and pos) come from upstream kernels
    pdl_launch_dependents();                 // only after our own wait: at most two kernels overlap

    // ---- prologue: per-row statistics -> RMSNorm factor and fp16 scaling
    const int64_t K = a.k;
    for (int i = 0; i < m; ++i) {
        const float* xr = a.x + (int64_t)i * a.ldx;
        float ssq[4] = {0.f, 0.f, 0.f, 0.f}, amx[4] = {0.f, 0.f, 0.f, 0.f};
        for (int64_t kk = tid; kk < K; kk += 4 * kGemvThreads) {
            float v[4], gg[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int64_t k = kk + (int64_t)u * kGemvThreads;
                v[u] = k < K ? xr[k] : 0.f;
                gg[u] = (a.g && k < K) ? a.g[k] : 1.f;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                ssq[u] = fmaf(v[u], v[u], ssq[u]);
                amx[u] = fmaxf(amx[u], fabsf(v[u] * gg[u]));
            }
        }
        float sq = (ssq[0] + ssq[1]) + (ssq[2] + ssq[3]);
        float am = fmaxf(fmaxf(amx[0], amx[1]), fmaxf(amx[2], amx[3]));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, o);
            am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
        }
        if (lane == 0) {
            s_stats[warp * 8 + i] = sq;
            s_stats[kGemvWarps * 8 + warp * 8 + i] = am;
        }
    }
    __syncthreads();
    if (tid < m) {
        float ssq = 0.f, amx = 0.f;
        for (int w = 0; w < kGemvWarps; ++w) {
            ssq += s_stats[w * 8 + tid];
            amx = fmaxf(amx, s_stats[kGemvWarps * 8 + w * 8 + tid]);
        }
        const float r = a.rmsnorm ? 1.0f / sqrtf(ssq / (float)K + a.eps) : 1.0f;
        const float an = amx * r;
        int e = 0;
        float sc = 1.0f;
        if (an > 0.f && isfinite(an)) {
            frexpf(an, &e);                  // an < 2^e
            sc = ldexpf(1.0f, 14 - e);       // an * sc < 2^14
        }
        s_smul[tid] = r * sc;
        s_inv[tid] = 1.0f / sc;              // exact power of two
    }
    if (tid >= m && tid < 8) s_inv[tid] = 0.f;
    __syncthreads();

    // ---- prologue: activations -> fp16 B fragments + per-block offsets; one
    // warp per (row, block), lane e converts element e, eight loads in flight
    const int nblk = kc * 2;
    {
        const int e = lane, half = e >> 4, ep = e & 15, rr = ep >> 3, tt = (ep & 7) >> 1, elem = ep & 1;
        const int items = m * nblk;
        for (int base = warp; base < items; base += 8 * kGemvWarps) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int it = base + u * kGemvWarps;
                v[u] = 0.f;
                if (it < items) {
                    const int i = it / nblk, blk = it - i * nblk;
                    const int64_t k0 = (int64_t)blk * 32 + e;
                    if (k0 < K) {
                        const float xv = a.x[(int64_t)i * a.ldx + k0];
                        v[u] = a.g ? xv * a.g[k0] : xv;
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int it = base + u * kGemvWarps;
                if (it >= items) break;
                const int i = it / nblk, blk = it - i * nblk;
                const __half h = __float2half_rn(v[u] * s_smul[i]);
                float hf = __half2float(h);
                s_bs16[((blk * m + i) * 16 + tt * 4 + half * 2 + rr) * 2 + elem] = __half_as_ushort(h);
#pragma unroll
                for (int o = 8; o > 0; o >>= 1) hf += __shfl_xor_sync(0xffffffffu, hf, o);   // per 16-lane half
                const float shi = __shfl_sync(0xffffffffu, hf, 16);
                if (lane == 0) s_bias[i * nblk + blk] = -(1032.0f * hf + 72.0f * shi);
            }
        }
    }
    __syncthreads();

    const int64_t pos = a.pos_dev ? *a.pos_dev : a.pos;
    const uint32_t tk = smem_token();
    const uint32_t bs_a = smem_addr(s_bs16) + tk, bias_a = smem_addr(s_bias) + tk;
    const int tok = g < m ? g : 0;
    float best_v[2] = {-INFINITY, -INFINITY};
    int32_t best_i[2] = {0x7fffffff, 0x7fffffff};

    // ---- main loop: this warp's records, four in flight
    int n_part = 0;
    s_part_tile[warp * 2 + 0] = -1;
    s_part_tile[warp * 2 + 1] = -1;
    if (wb < we) {
        int64_t tile = wb / kc;
        int cin = (int)(wb - tile * kc);
        bool tile_whole = (cin == 0);        // this warp saw the tile from its first record
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int64_t base = wb; base < we; base += kGemvPrefetch) {
#pragma unroll
            for (int u = 0; u < kGemvPrefetch; ++u) {
                const int64_t i = base + u;
                if (i >= we) break;
                const uint4 q = rq[u];
                const uint2 dd = rd[u];
                const int64_t nx = i + kGemvPrefetch;
                if (nx < we) {
                    rq[u] = __ldg(reinterpret_cast<const uint4*>(wsrc + nx * kChunkBytes));
                    rd[u] = __ldg(reinterpret_cast<const uint2*>(dsrc + nx * kChunkBytes));
                }
                gemv_record<MT>(q, dd, bs_a, bias_a, nblk, cin, m, tok, t, acc);
                if (++cin == kc || i + 1 == we) {
                    if (cin == kc && tile_whole) {
                        gemv_epilogue(a, tile, acc, g, t, s_inv, pos, best_v, best_i);
                    } else {
                        // a tile cut at this warp's range end: keep the partial sums
                        *reinterpret_cast<float4*>(s_part + ((warp * 2 + n_part) * 32 + lane) * 4) =
                            make_float4(acc[0], acc[1], acc[2], acc[3]);
                        if (lane == 0) s_part_tile[warp * 2 + n_part] = tile;
                        ++n_part;
                    }
                    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
                    cin = 0;
                    ++tile;
                    tile_whole = true;
                }
            }
        }
    }
    __syncthreads();

    // ---- tiles cut between warps: warp 0 sums the parts in warp order
    const GemvWs W = gemv_ws_layout(a.tiles, a.op == VOX_EP_ARGMAX);
    if (warp == 0) {
        float* parts = reinterpret_cast<float*>(a.ws + W.partials);
        int32_t* counters = reinterpret_cast<int32_t*>(a.ws + W.counters);
        int64_t cur = -1;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        for (int e = 0; e <= 2 * kGemvWarps; ++e) {
            const int64_t tl = e < 2 * kGemvWarps ? s_part_tile[e] : -2;
            if (tl == -1) continue;
            if (tl != cur && cur >= 0) {
                // flush tile `cur`: finish here, or combine with the neighbouring CTAs
                const int64_t b_first = sk_owner(cur * kc, total, G);
                const int64_t b_last = sk_owner(cur * kc + kc - 1, total, G);
                bool finish = true;
                if (b_first != b_last) {
                    const int my_slot = (cur == cb / kc) ? 0 : 1;
                    *reinterpret_cast<float4*>(parts + (((size_t)b * 2 + my_slot) * 32 + lane) * 4) =
                        make_float4(acc[0], acc[1], acc[2], acc[3]);
                    __syncwarp();
                    int32_t last = 0;
                    if (lane == 0) {
                        __threadfence();
                        const int32_t old = atomicAdd(&counters[cur], 1);
                        last = (old == (int32_t)(b_last - b_first)) ? 1 : 0;
                        if (last) {
                            __threadfence();
                            counters[cur] = 0;
                        }
                    }
                    finish = __shfl_sync(0xffffffffu, last, 0) != 0;
                    if (finish) {
                        acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
                        for (int64_t bo = b_first; bo <= b_last; ++bo) {
                            const int sl = (cur == sk_begin(bo, total, G) / kc) ? 0 : 1;
                            const float4 pv = __ldcg(reinterpret_cast<const float4*>(
                                parts + (((size_t)bo * 2 + sl) * 32 + lane) * 4));
                            acc[0] += pv.x; acc[1] += pv.y; acc[2] += pv.z; acc[3] += pv.w;
                        }
                    }
                }
                if (finish) gemv_epilogue(a, cur, acc, g, t, s_inv, pos, best_v, best_i);
                acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
            }
            if (tl < 0) break;
            cur = tl;
            const float4 pv = *reinterpret_cast<const float4*>(s_part + (e * 32 + lane) * 4);
            acc[0] += pv.x; acc[1] += pv.y; acc[2] += pv.z; acc[3] += pv.w;
        }
    }

    // ---- greedy argmax: warps -> CTA -> the last CTA to arrive
    if (a.op == VOX_EP_ARGMAX) {
        if (g == 0) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                s_best_v[warp * 8 + 2 * t + e] = best_v[e];
                s_best_i[warp * 8 + 2 * t + e] = best_i[e];
            }
        }
        __syncthreads();
        if (warp == 0) {
            float* bvs = reinterpret_cast<float*>(a.ws + W.best_v);
            int32_t* bis = reinterpret_cast<int32_t*>(a.ws + W.best_i);
            int32_t* gcount = reinterpret_cast<int32_t*>(a.ws + W.gcount);
            if (lane < m) {
                float bv = -INFINITY;
                int32_t bi = 0x7fffffff;
                for (int w = 0; w < kGemvWarps; ++w)
                    if (argmax_better(s_best_v[w * 8 + lane], s_best_i[w * 8 + lane], bv, bi)) {
                        bv = s_best_v[w * 8 + lane];
                        bi = s_best_i[w * 8 + lane];
                    }
                bvs[b * 8 + lane] = bv;
                bis[b * 8 + lane] = bi;
            }
            __syncwarp();
            int32_t last = 0;
            if (lane == 0) {
                __threadfence();
                const int32_t old = atomicAdd(gcount, 1);
                last = (old == (int32_t)(G - 1)) ? 1 : 0;
                if (last) {
                    __threadfence();
                    *gcount = 0;
                }
            }
            last = __shfl_sync(0xffffffffu, last, 0);
            if (last && lane < m) {
                float bv = -INFINITY;
                int32_t bi = 0x7fffffff;
                for (int64_t bo = 0; bo < G; ++bo) {
                    const float v = __ldcg(bvs + bo * 8 + lane);
                    const int32_t ix = __ldcg(bis + bo * 8 + lane);
                    if (argmax_better(v, ix, bv, bi)) { bv = v; bi = ix; }
                }
                a.argmax[lane] = bi;
            }
        }
    }
    (void)s_flag;
}

static int gemv_ctas_per_sm()
{
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("VOX_GEMV_CTAS_PER_SM");
        v = e ? atoi(e) : 2;
        if (v < 1) v = 1;
        if (v > 4) v = 4;
    }
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
    if (ep && ep->op == VOX_EP_KV_APPEND) {
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

    const GemvSmem L = gemv_smem_layout(a.kc, a.m);
    if (L.total > 227 * 1024) return VOX_ERR_SHAPE;           // activations do not fit shared memory
    static bool attr_set = false;
    if (!attr_set) {
        cudaError_t e = cudaFuncSetAttribute(q4_gemv_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(q4_gemv_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) {
            set_cuda_error(e);
            return VOX_ERR_CUDA;
        }
        attr_set = true;
    }
    const int64_t total = (int64_t)a.tiles * a.kc;
    int64_t G = (int64_t)device_sm_count() * gemv_ctas_per_sm();
    if (L.total > 110 * 1024) G = device_sm_count();       // two such CTAs do not fit one SM
    if (G > total) G = total;
    if (G > kGemvMaxCtas) G = kGemvMaxCtas;
    if (m == 1) return launch_pdl(q4_gemv_kernel<1>, dim3((unsigned)G), dim3(kGemvThreads), L.total, s, a);
    return launch_pdl(q4_gemv_kernel<8>, dim3((unsigned)G), dim3(kGemvThreads), L.total, s, a);
}

}  // namespace vox
