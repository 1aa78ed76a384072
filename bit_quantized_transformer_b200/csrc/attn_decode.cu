// Rolling KV cache append (K3), split-KV GQA decode attention (K4) and the
// log-sum-exp combine of its partials (K5).
//
// Sources: "Mistral Voxtral Realtime 4B ... 순수 C 기반 CPU 전용 추론 구현",
// "주요 기능" (rolling KV cache over an 8192-position sliding window; fused
// GPU ops with batched attention) and "모델 아키텍처" (GQA, 32 query / 8 KV
// heads).  Readings: slot = pos mod W, the valid slots after writing pos are
// the first min(pos + 1, W); query head h reads kv head h / (n_q / n_kv).
//
// K4 design: one 160-thread CTA per SM by default (a TMA producer warp and
// four consumer warps; tuning knobs VOX_ATTN_CTAS_PER_SM and VOX_ATTN_STAGES,
// three ring stages of 32 KB by default).  The valid (kv head, 64-slot chunk)
// pairs are split evenly over the CTAs (stream-K), so every CTA streams the
// same number of cache bytes.
// A producer lane loads each chunk's K and V with 2-D TMA tiles (128-byte
// swizzle, 4 x 8 KB) into a shared-memory ring; four consumer warps each take
// 16 slots of the chunk:
//    S^T[head][slot] = q'[head] . K[slot]      mma m16n8k16, heads padded to 16
//    online softmax in the exp2 domain (q' = q * scale * log2 e)
//    O[head][dim]   += P[head][slot] . V[slot][dim]  (P from the S^T fragments)
// q' and P are split into bf16 hi + lo parts (two MMAs each), so the
// tensor-core inputs carry about 16 significant bits; K and V are the cache's
// own bf16 values.  Each CTA writes one (m, l, O) partial per kv head it
// touched, into that head's contiguous run of records; K5 merges each head's
// run in CTA order (deterministic), one small CTA per query head, all of a
// head's records loaded in one round before the arithmetic.
//
// Programmatic dependent launch: the producer starts streaming before the
// upstream kernel (the QKV projection that appends this step's k, v) has
// finished; after griddepcontrol.wait the warp whose slots include the newly
// written one reloads that row from global memory.
#include "tma.cuh"

#include <mutex>
#include <stdlib.h>

namespace vox {

// ------------------------------------------------------------------ K3
__global__ void kv_append_kernel(uint16_t* __restrict__ kc, uint16_t* __restrict__ vc,
                                 const void* __restrict__ kn, const void* __restrict__ vn, int new_bf16,
                                 int n_kv, int hd, int window, int64_t pos, const int64_t* __restrict__ pos_dev)
{
    pdl_wait();
    pdl_launch_dependents();
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n_kv * hd) return;
    int64_t p = pos_dev ? *pos_dev : pos;
    int64_t slot = p % window;
    int h = i / hd, c = i % hd;
    uint16_t kb, vb;
    if (new_bf16) {
        kb = static_cast<const uint16_t*>(kn)[i];
        vb = static_cast<const uint16_t*>(vn)[i];
    } else {
        kb = f32_to_bf16_bits(static_cast<const float*>(kn)[i]);
        vb = f32_to_bf16_bits(static_cast<const float*>(vn)[i]);
    }
    kc[((int64_t)h * window + slot) * hd + c] = kb;
    vc[((int64_t)h * window + slot) * hd + c] = vb;
}

vox_status launch_kv_append(void* kc, void* vc, const void* kn, const void* vn, int new_dtype, int n_kv, int hd,
                            int window, int64_t pos, const int64_t* pos_dev, cudaStream_t s)
{
    int total = n_kv * hd;
    int threads = 256;
    return launch_pdl(kv_append_kernel, dim3((total + threads - 1) / threads), dim3(threads), 0, s,
                      static_cast<uint16_t*>(kc), static_cast<uint16_t*>(vc), kn, vn, (int)(new_dtype == VOX_BF16),
                      n_kv, hd, window, pos, pos_dev);
}

// ------------------------------------------------------------------ K4
constexpr int kAttnChunk = 64;                 // slots per chunk
constexpr int kAttnHd = 128;
constexpr int kAttnWarps = 4;                  // consumer warps, 16 slots each
constexpr int kAttnThreads = 32 * (1 + kAttnWarps);
constexpr int kAttnMaxStages = 6;
constexpr int kAttnTileBytes = kAttnChunk * 128;            // one 64 x 64 bf16 box
constexpr int kAttnStageBytes = 4 * kAttnTileBytes;         // K lo/hi, V lo/hi
constexpr int kAttnMaxCtas = 592;
constexpr int kCombineBatch = 20;                  // records of a head loaded per round in K5
constexpr int kAttnMaxGroup = 8;

struct AttnArgs {
    const float* q;
    const uint16_t* kcache;
    const uint16_t* vcache;
    float* out;
    int32_t n_q, n_kv, hd, window, group;
    int64_t pos;
    const int64_t* pos_dev;
    float qscale;                              // scale * log2(e)
    float* ws;                                 // partial records
    int32_t stages;
    int32_t rec_floats;                        // record stride (floats, a multiple of 4)
    int32_t rmax;                              // record slots per kv head
    // Several sequences (blockIdx.y = sequence s): q, out, the records and
    // pos_dev advance by one sequence's size.  With a page table the caches
    // are pools of 64-slot pages [page][n_kv][64][hd]; sequence s's slot p
    // lives in page pages[s * pps + p / 64] (null: one contiguous cache
    // [n_kv][window][hd]).
    const int32_t* pages;
    int32_t pps;
    int64_t n_pages;
    int64_t q_ld;                              // floats from one sequence's q to the next
};

// First cache row (in the tensor map's rows) of chunk ci of kv head kh of
// sequence s; -1 for a page index outside the pool.
__device__ __forceinline__ int64_t attn_chunk_row(const AttnArgs& a, int s, int64_t kh, int64_t ci)
{
    if (!a.pages) return kh * a.window + ci * kAttnChunk;
    const int64_t pg = __ldg(a.pages + (int64_t)s * a.pps + ci);
    if (pg < 0 || pg >= a.n_pages) return -1;
    return (pg * a.n_kv + kh) * kAttnChunk;
}

// Partial record of one CTA for one kv head: O[group][hd], then (m, l) per
// query head of the group, padded to 16 bytes.  The records of kv head kh
// are contiguous: slot kh * rmax + (CTA - first CTA of kh).
__host__ __device__ constexpr int attn_rec_floats(int group, int hd) { return (group * (hd + 2) + 3) & ~3; }
__host__ __device__ constexpr int attn_rmax(int n_kv) { return (kAttnMaxCtas + n_kv - 1) / n_kv + 2; }

static int env_int_attn(const char* name, int dflt, int lo, int hi)
{
    const char* e = getenv(name);
    int v = e ? atoi(e) : dflt;
    return v < lo ? lo : (v > hi ? hi : v);
}

// CTAs per sequence: the SMs (times the knob) shared evenly by the sequences.
static int64_t attn_grid(int n_kv, int window, int n_seq)
{
    int64_t chunks = (int64_t)n_kv * ceil_div(window, kAttnChunk);
    int64_t G = (int64_t)env_int_attn("VOX_ATTN_CTAS_PER_SM", 1, 1, 2) * device_sm_count() / n_seq;
    if (G > chunks) G = chunks;
    if (G < n_kv) G = n_kv;                    // then no CTA spans more than two kv heads
    if (G > kAttnMaxCtas) G = kAttnMaxCtas;
    return G;
}

// Workspace: rmax partial records per kv head (room for the largest group),
// per sequence.
size_t attn_workspace_bytes(int n_kv, int hd, int window, int n_seq)
{
    (void)window;
    return ((size_t)n_seq * n_kv * attn_rmax(n_kv) * attn_rec_floats(kAttnMaxGroup, hd) * sizeof(float) + 255) &
           ~(size_t)255;
}

__host__ __device__ inline int64_t attn_begin(int64_t b, int64_t total, int64_t G) { return b * total / G; }
__host__ __device__ inline int64_t attn_owner(int64_t c, int64_t total, int64_t G) { return ((c + 1) * G - 1) / total; }

// Shared-memory carve-up for `stages` ring stages (host and device).
struct AttnSmem {
    uint32_t ring, merge, bars, flags, total;
};

__host__ __device__ inline AttnSmem attn_smem_layout(int stages)
{
    AttnSmem L;
    L.ring = 0;
    L.merge = (uint32_t)stages * kAttnStageBytes;
    L.bars = L.merge + kAttnWarps * kAttnMaxGroup * (kAttnHd + 2) * 4;
    L.flags = L.bars + 2u * (uint32_t)stages * 8u;
    L.total = L.flags + 16 + 1024;             // + alignment slack
    return L;
}

__global__ void __launch_bounds__(kAttnThreads, 2)
gqa_decode_attn_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                       const AttnArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    // TMA 128-byte-swizzled tiles need a 1024-byte aligned destination.
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int stages = a.stages;
    const AttnSmem SL = attn_smem_layout(stages);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + SL.bars);
    uint64_t* empty = full + stages;
    volatile int32_t* s_fail = reinterpret_cast<volatile int32_t*>(smem + SL.flags);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t G = gridDim.x, b = blockIdx.x;
    const int W = a.window;
    const int seq = blockIdx.y;
    const float* q_seq = a.q + (int64_t)seq * a.q_ld;
    float* ws_seq = a.ws + (int64_t)seq * a.n_kv * a.rmax * a.rec_floats;

    if (tid == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kAttnWarps);
        }
        s_fail[0] = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // The position array is written by the last kernel of the previous token
    // step; every kernel here triggers its dependents only after its own
    // griddepcontrol.wait, so when this kernel starts that writer has
    // finished and the early read is safe.
    const int64_t pos = a.pos_dev ? a.pos_dev[seq] : a.pos;
    const int64_t n_valid = pos + 1 < W ? pos + 1 : W;
    const int64_t nch = (n_valid + kAttnChunk - 1) / kAttnChunk;      // chunks per kv head
    const int64_t total = (int64_t)a.n_kv * nch;
    const int64_t c_begin = attn_begin(b, total, G), c_end = attn_begin(b + 1, total, G);

    if (warp == kAttnWarps) {
        // ------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tmap(&kmap);
            prefetch_tmap(&vmap);
            int slot = 0;
            uint32_t ph = 0;
            int64_t kh = c_begin / nch, ci = c_begin - (c_begin / nch) * nch;
            for (int64_t c = c_begin; c < c_end; ++c) {
                if (!s_fail[0] && !mbar_wait_bounded(&empty[slot], ph ^ 1u, 0x201)) s_fail[0] = 1;
                if (s_fail[0]) break;
                // a page outside the pool reads the fill value (zeros): the
                // box starts at the map's row count, wholly past its rows
                const int64_t crow = attn_chunk_row(a, seq, kh, ci);
                if (crow < 0) atomicCAS(&g_vox_device_status, 0, 0x203);
                const int32_t row = (int32_t)(crow < 0 ? a.n_pages * a.n_kv * kAttnChunk : crow);
                uint8_t* st = smem + SL.ring + slot * kAttnStageBytes;
                mbar_arrive_expect_tx(&full[slot], kAttnStageBytes);
                tma_load_2d(st + 0 * kAttnTileBytes, &kmap, 0, row, &full[slot]);
                tma_load_2d(st + 1 * kAttnTileBytes, &kmap, 64, row, &full[slot]);
                tma_load_2d(st + 2 * kAttnTileBytes, &vmap, 0, row, &full[slot]);
                tma_load_2d(st + 3 * kAttnTileBytes, &vmap, 64, row, &full[slot]);
                if (++ci == nch) { ci = 0; ++kh; }
                if (++slot == stages) { slot = 0; ph ^= 1u; }
            }
        }
        return;
    }

    // ------------------------------------------------------------ consumers
    const int g = lane >> 2, t = lane & 3;
    const int group = a.group;
    pdl_wait();                                          // q and the new cache slot come from upstream
    pdl_launch_dependents();
    const int64_t new_slot = pos % W;

    float* merge = reinterpret_cast<float*>(smem + SL.merge);
    const uint32_t ring_a = smem_addr(smem + SL.ring);

    // running softmax state of heads 2t, 2t+1 (replicated over g) and O^T
    // fragments: o[J] = (dim 16J+g | 16J+8+g) x (head 2t | 2t+1)
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float o[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    uint32_t qh[8][2], ql[8][2];                       // B fragments of q'^T (column g = head g)
    int64_t seg_head = -1;
    int seg_idx = 0;

    auto flush = [&](int sidx, int64_t kh_seg) {
        // merge the four warps' (m, l, O) for the finished kv head, write the partial
        float* mw = merge + warp * kAttnMaxGroup * (kAttnHd + 2);
        if (g == 0) {
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                mw[kAttnMaxGroup * kAttnHd + (2 * t + u) * 2 + 0] = m_run[u];
                mw[kAttnMaxGroup * kAttnHd + (2 * t + u) * 2 + 1] = l_run[u];
            }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            mw[(2 * t) * kAttnHd + 16 * j + g] = o[j][0];
            mw[(2 * t + 1) * kAttnHd + 16 * j + g] = o[j][1];
            mw[(2 * t) * kAttnHd + 16 * j + 8 + g] = o[j][2];
            mw[(2 * t + 1) * kAttnHd + 16 * j + 8 + g] = o[j][3];
        }
        named_barrier(1, 32 * kAttnWarps);
        (void)sidx;
        const int64_t bf_seg = attn_owner(kh_seg * nch, total, G);
        float* rec = ws_seq + ((size_t)kh_seg * a.rmax + (size_t)(b - bf_seg)) * a.rec_floats;
        for (int i = tid; i < group * kAttnHd; i += 32 * kAttnWarps) {
            const int hh = i / kAttnHd, cc = i % kAttnHd;
            float M = -INFINITY;
            for (int w = 0; w < kAttnWarps; ++w)
                M = fmaxf(M, merge[w * kAttnMaxGroup * (kAttnHd + 2) + kAttnMaxGroup * kAttnHd + hh * 2]);
            float O = 0.f, Lsum = 0.f;
            for (int w = 0; w < kAttnWarps; ++w) {
                const float* mw2 = merge + w * kAttnMaxGroup * (kAttnHd + 2);
                const float mv = mw2[kAttnMaxGroup * kAttnHd + hh * 2];
                const float f = (mv == -INFINITY) ? 0.f : exp2f(mv - M);
                O += f * mw2[hh * kAttnHd + cc];
                Lsum += f * mw2[kAttnMaxGroup * kAttnHd + hh * 2 + 1];
            }
            rec[hh * kAttnHd + cc] = O;
            if (cc == 0) {
                rec[group * kAttnHd + hh * 2 + 0] = M;
                rec[group * kAttnHd + hh * 2 + 1] = Lsum;
            }
        }
        named_barrier(1, 32 * kAttnWarps);
    };

    int slot = 0;
    uint32_t ph = 0;
    int64_t kh = c_begin / nch, ci = c_begin - (c_begin / nch) * nch;
    for (int64_t c = c_begin; c < c_end; ++c) {
        if (kh != seg_head) {
            if (seg_head >= 0) {
                flush(seg_idx++, seg_head);
                m_run[0] = m_run[1] = -INFINITY;
                l_run[0] = l_run[1] = 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
            }
            seg_head = kh;
            // q' = q * scale * log2(e), split into bf16 hi + lo B fragments (heads >= group are zero)
            const bool ok = g < group;
            const float* qr = q_seq + ((int64_t)kh * group + (ok ? g : 0)) * kAttnHd;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                float v0 = 0.f, v1 = 0.f, v2 = 0.f, v3 = 0.f;
                if (ok) {
                    v0 = qr[16 * kk + 2 * t] * a.qscale;
                    v1 = qr[16 * kk + 2 * t + 1] * a.qscale;
                    v2 = qr[16 * kk + 2 * t + 8] * a.qscale;
                    v3 = qr[16 * kk + 2 * t + 9] * a.qscale;
                }
                split_bf16x2(v0, v1, qh[kk][0], ql[kk][0]);
                split_bf16x2(v2, v3, qh[kk][1], ql[kk][1]);
            }
        }

        if (!s_fail[0] && !mbar_wait_bounded(&full[slot], ph, 0x202)) s_fail[0] = 1;
        uint8_t* stp = smem + SL.ring + slot * kAttnStageBytes;
        const uint32_t st = ring_a + slot * kAttnStageBytes;
        const int64_t slot0 = ci * kAttnChunk + warp * 16;   // first cache slot of this warp's slice

        // Generic-proxy fix-ups of this warp's 16 rows of the TMA-written stage.
        bool touched = false;
        const int64_t crow = (new_slot >= slot0 && new_slot < slot0 + 16) ? attn_chunk_row(a, seq, kh, ci) : -1;
        if (crow >= 0) {
            // reload the newest row (K and V, 4 x 128 bytes) written by the upstream kernel
            const uint32_t r = (uint32_t)(new_slot - ci * kAttnChunk);
            const int part = lane >> 3, unit = lane & 7;       // tiles K lo, K hi, V lo, V hi
            const uint16_t* src = (part < 2 ? a.kcache : a.vcache) +
                                  (crow + r) * kAttnHd + (part & 1) * 64 + unit * 8;
            const uint4 v = *reinterpret_cast<const uint4*>(src);
            *reinterpret_cast<uint4*>(stp + part * kAttnTileBytes + sw128_offset(r, (uint32_t)unit)) = v;
            touched = true;
        }
        if (slot0 + 16 > n_valid) {
            // slots past the valid range may hold anything (NaN included): zero their V rows
            for (int i = lane; i < 16 * 16; i += 32) {
                const int rr = i >> 4, part = 2 + ((i >> 3) & 1), unit = i & 7;
                if (slot0 + rr >= n_valid) {
                    const uint32_t r = (uint32_t)(warp * 16 + rr);
                    *reinterpret_cast<uint4*>(stp + part * kAttnTileBytes + sw128_offset(r, (uint32_t)unit)) =
                        make_uint4(0u, 0u, 0u, 0u);
                }
            }
            touched = true;
        }
        __syncwarp();

        // ---- S = K q'^T for 16 slots: A = K rows (ldmatrix), B = q' (registers).
        // Four accumulator chains (k-step parity x hi/lo) keep the MMA latency short.
        float sa[4][4];
#pragma unroll
        for (int u = 0; u < 4; ++u) sa[u][0] = sa[u][1] = sa[u][2] = sa[u][3] = 0.f;
        {
            const int mi = lane >> 3;
            const uint32_t r = (uint32_t)(warp * 16 + 8 * (mi & 1) + (lane & 7));
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t tile = st + (kk >> 2) * kAttnTileBytes;      // K lo / hi
                uint32_t ak[4];
                ldsm_x4(ak, tile + sw128_offset(r, (uint32_t)(2 * (kk & 3) + (mi >> 1))));
                mma_bf16_16816(sa[(kk & 1) * 2 + 0], ak, qh[kk][0], qh[kk][1], sa[(kk & 1) * 2 + 0]);
                mma_bf16_16816(sa[(kk & 1) * 2 + 1], ak, ql[kk][0], ql[kk][1], sa[(kk & 1) * 2 + 1]);
            }
        }
        // sv: (slot g, head 2t), (slot g, head 2t+1), (slot g+8, head 2t), (slot g+8, head 2t+1)
        float sv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            sv[e] = (sa[0][e] + sa[1][e]) + (sa[2][e] + sa[3][e]);
            if (slot0 + g + 8 * (e >> 1) >= n_valid) sv[e] = -INFINITY;
        }
        // ---- online softmax per head (exp2 domain); reduce over the 8 lanes of equal t
        float p[4], corr[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            float mx = fmaxf(sv[u], sv[u + 2]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float m_new = fmaxf(m_run[u], mx);
            if (m_new == -INFINITY) {
                corr[u] = 1.f;
                p[u] = p[u + 2] = 0.f;
            } else {
                corr[u] = exp2f(m_run[u] - m_new);           // m_run = -inf gives 0
                p[u] = exp2f(sv[u] - m_new);
                p[u + 2] = exp2f(sv[u + 2] - m_new);
            }
            float ps = p[u] + p[u + 2];
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
            const float x00 = __shfl_sync(0xffffffffu, p[0], src0), x01 = __shfl_sync(0xffffffffu, p[1], src0);
            const float x10 = __shfl_sync(0xffffffffu, p[0], src1), x11 = __shfl_sync(0xffffffffu, p[1], src1);
            const float y00 = __shfl_sync(0xffffffffu, p[2], src0), y01 = __shfl_sync(0xffffffffu, p[3], src0);
            const float y10 = __shfl_sync(0xffffffffu, p[2], src1), y11 = __shfl_sync(0xffffffffu, p[3], src1);
            split_bf16x2(odd ? x01 : x00, odd ? x11 : x10, bh[0], bl[0]);   // slots 2t, 2t+1
            split_bf16x2(odd ? y01 : y00, odd ? y11 : y10, bh[1], bl[1]);   // slots 2t+8, 2t+9
        }
        // ---- O^T = O^T * corr + V^T P: 8 dim tiles of 16, A = V^T via ldmatrix.trans
        {
            const int mi = lane >> 3;
            const uint32_t r = (uint32_t)(warp * 16 + 8 * (mi >> 1) + (lane & 7));
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t tile = st + (2 + (j >> 2)) * kAttnTileBytes;   // V lo / hi
                uint32_t av[4];
                ldsm_x4_trans(av, tile + sw128_offset(r, (uint32_t)(2 * (j & 3) + (mi & 1))));
                float c[4] = {o[j][0] * corr[0], o[j][1] * corr[1], o[j][2] * corr[0], o[j][3] * corr[1]};
                mma_bf16_16816(c, av, bh[0], bh[1], c);
                mma_bf16_16816(c, av, bl[0], bl[1], c);
                o[j][0] = c[0];
                o[j][1] = c[1];
                o[j][2] = c[2];
                o[j][3] = c[3];
            }
        }
        // generic writes into a buffer the async proxy refills next: order them first
        if (touched) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        if (++slot == stages) { slot = 0; ph ^= 1u; }
        if (++ci == nch) { ci = 0; ++kh; }
    }
    if (seg_head >= 0) flush(seg_idx, seg_head);
}

// ------------------------------------------------------------------ K5
// One 32-thread CTA per (kv head, query head of its group); lane l covers
// dims 4l .. 4l+3.  The head's records sit in one contiguous run; a CTA in
// the head's range that owned no chunk (possible when the grid outnumbers
// the chunks) wrote nothing and is skipped.  Each round loads up to
// kCombineBatch records, then folds them max-first in CTA order.
__device__ __forceinline__ bool attn_cta_nonempty(int64_t bo, int64_t total, int64_t G)
{
    if (total < (1 << 20) && G < (1 << 11)) {
        const uint32_t t32 = (uint32_t)total, g32 = (uint32_t)G, b32 = (uint32_t)bo;
        return (b32 * t32) / g32 != ((b32 + 1) * t32) / g32;
    }
    return attn_begin(bo, total, G) != attn_begin(bo + 1, total, G);
}

__global__ void __launch_bounds__(32) attn_combine_kernel(const AttnArgs a, int64_t G)
{
    // The dependents (the Wo projection) may launch at once: this grid is
    // small, so their first CTAs fit beside the attention kernel and start
    // their weight copies; they still wait for this grid to complete.
    pdl_launch_dependents();
    pdl_wait();
    const int group = a.group;
    const int kh = blockIdx.x / group, gi = blockIdx.x - kh * group, lane = threadIdx.x;
    const int W = a.window;
    const int seq = blockIdx.y;
    const int64_t pos = a.pos_dev ? a.pos_dev[seq] : a.pos;
    const int64_t n_valid = pos + 1 < W ? pos + 1 : W;
    const int64_t nch = (n_valid + kAttnChunk - 1) / kAttnChunk;
    const int64_t total = (int64_t)a.n_kv * nch;
    const int64_t bf = attn_owner((int64_t)kh * nch, total, G), bl = attn_owner((int64_t)kh * nch + nch - 1, total, G);
    const int nrec = (int)(bl - bf + 1);
    const float* recs = a.ws + ((size_t)seq * a.n_kv + kh) * a.rmax * a.rec_floats;
    float M = -INFINITY, L = 0.f;
    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int r0 = 0; r0 < nrec; r0 += kCombineBatch) {
        // lane i decides whether record r0 + i exists
        const bool mine = r0 + lane < nrec && lane < kCombineBatch && attn_cta_nonempty(bf + r0 + lane, total, G);
        const uint32_t mask = __ballot_sync(0xffffffffu, mine);
        float2 ml[kCombineBatch];
        float4 ov[kCombineBatch];
#pragma unroll
        for (int u = 0; u < kCombineBatch; ++u) {
            ml[u] = make_float2(-INFINITY, 0.f);
            ov[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if ((mask >> u) & 1u) {
                const float* rec = recs + (size_t)(r0 + u) * a.rec_floats;
                ml[u] = __ldcg(reinterpret_cast<const float2*>(rec + group * kAttnHd) + gi);
                ov[u] = __ldcg(reinterpret_cast<const float4*>(rec + gi * kAttnHd) + lane);
            }
        }
        float mb = M;
#pragma unroll
        for (int u = 0; u < kCombineBatch; ++u) mb = fmaxf(mb, ml[u].x);
        const float fo = M == -INFINITY ? 0.f : exp2f(M - mb);
        O = make_float4(O.x * fo, O.y * fo, O.z * fo, O.w * fo);
        L *= fo;
#pragma unroll
        for (int u = 0; u < kCombineBatch; ++u) {
            if (ml[u].x == -INFINITY) continue;
            const float f = exp2f(ml[u].x - mb);
            O.x = fmaf(f, ov[u].x, O.x);
            O.y = fmaf(f, ov[u].y, O.y);
            O.z = fmaf(f, ov[u].z, O.z);
            O.w = fmaf(f, ov[u].w, O.w);
            L = fmaf(f, ml[u].y, L);
        }
        M = mb;
    }
    const float inv = 1.0f / L;
    *reinterpret_cast<float4*>(a.out + ((int64_t)seq * a.n_q + (int64_t)kh * group + gi) * kAttnHd + 4 * lane) =
        make_float4(O.x * inv, O.y * inv, O.z * inv, O.w * inv);
}

// One sequence with one contiguous cache (n_seq = 1, pages = null) or n_seq
// sequences over paged pools of n_pages pages.
vox_status launch_gqa_decode_attn_seqs(const float* q, const void* kc, const void* vc, float* out, int n_q, int n_kv,
                                       int hd, int window, int64_t pos, const int64_t* pos_dev, float scale, void* ws,
                                       cudaStream_t s, int n_seq, const int32_t* pages, int64_t n_pages, int64_t q_ld)
{
    const uint64_t rows = pages ? (uint64_t)n_pages * n_kv * kAttnChunk : (uint64_t)n_kv * window;
    CUtensorMap kmap, vmap;
    vox_status st = make_tmap_2d(&kmap, kc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)hd, rows,
                                 (uint64_t)hd * 2, 64, kAttnChunk, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != VOX_OK) return st;
    st = make_tmap_2d(&vmap, vc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)hd, rows, (uint64_t)hd * 2, 64,
                      kAttnChunk, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != VOX_OK) return st;

    AttnArgs a = {};
    a.q = q;
    a.kcache = static_cast<const uint16_t*>(kc);
    a.vcache = static_cast<const uint16_t*>(vc);
    a.out = out;
    a.n_q = n_q;
    a.n_kv = n_kv;
    a.hd = hd;
    a.window = window;
    a.group = n_q / n_kv;
    a.pos = pos;
    a.pos_dev = pos_dev;
    a.qscale = scale * 1.4426950408889634f;
    a.ws = static_cast<float*>(ws);
    a.rec_floats = attn_rec_floats(a.group, hd);
    a.rmax = attn_rmax(n_kv);
    a.stages = env_int_attn("VOX_ATTN_STAGES", 3, 2, kAttnMaxStages);
    a.pages = pages;
    a.q_ld = q_ld > 0 ? q_ld : (int64_t)n_q * hd;
    a.pps = window / kAttnChunk;
    a.n_pages = n_pages;
    const AttnSmem SL = attn_smem_layout(a.stages);

    static std::atomic<unsigned long long> attr_done{0};
    st = smem_attr_per_device(reinterpret_cast<const void*>(gqa_decode_attn_kernel),
                              (int)attn_smem_layout(kAttnMaxStages).total, attr_done);
    if (st != VOX_OK) return st;
    const int64_t G = attn_grid(n_kv, window, n_seq);
    st = launch_pdl(gqa_decode_attn_kernel, dim3((unsigned)G, (unsigned)n_seq), dim3(kAttnThreads), SL.total, s,
                    kmap, vmap, a);
    if (st != VOX_OK) return st;
    return launch_pdl(attn_combine_kernel, dim3((unsigned)(n_kv * a.group), (unsigned)n_seq), dim3(32), 0, s, a, G);
}

vox_status launch_gqa_decode_attn(const float* q, const void* kc, const void* vc, float* out, int n_q, int n_kv,
                                  int hd, int window, int64_t pos, const int64_t* pos_dev, float scale, void* ws,
                                  cudaStream_t s)
{
    return launch_gqa_decode_attn_seqs(q, kc, vc, out, n_q, n_kv, hd, window, pos, pos_dev, scale, ws, s, 1,
                                       nullptr, 0, 0);
}

// --------------------------------------------- allocation-free entry point
// vox_gqa_decode_attn needs the caller to hand in device scratch for the
// split-KV partial records.  Some callers cannot: a host program that links
// only this C library and owns no device allocator, or a real-time audio
// thread that must not call cudaMalloc (it can block and synchronise the
// device).  vox_gqa_decode_attn_static serves them from one fixed scratch
// array in device memory, sized for at most kStaticMaxKv kv heads with
// groups of at most kStaticMaxGroup query heads at head_dim 128 (the
// decoder's 8 kv heads x 4).  It allocates nothing: the array is part of the
// loaded module, and its address is looked up once per device.
constexpr int kStaticMaxKv = 8;
constexpr int kStaticMaxGroup = 4;

// Records of all heads for the largest n_kv * rmax(n_kv) over n_kv = 1..8
// (the per-head record count rounds up, so 7 heads need one more than 8).
constexpr int attn_static_max_records(int n)
{
    return n == 0 ? 0
                  : (n * attn_rmax(n) > attn_static_max_records(n - 1) ? n * attn_rmax(n)
                                                                        : attn_static_max_records(n - 1));
}
constexpr size_t kStaticScratchBytes =
    (size_t)attn_static_max_records(kStaticMaxKv) * attn_rec_floats(kStaticMaxGroup, kAttnHd) * sizeof(float);

static __device__ __align__(256) uint8_t g_attn_static_scratch[kStaticScratchBytes];

// Device address of the scratch array on the current device, looked up with
// cudaGetSymbolAddress the first time each device is used and kept for the
// life of the process.  Later calls read the kept address with one atomic
// load and take no lock; only a first lookup takes the mutex.  The address
// belongs to the device's primary context: after cudaDeviceReset (or any
// teardown that unloads this module from the device) the kept address is
// stale, so a process that resets a device must not call this entry point
// again on it without reloading the library.
static vox_status attn_static_scratch(void** out)
{
    static std::mutex mu;
    static std::atomic<void*> addr[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_cuda_error(e);
        return VOX_ERR_CUDA;
    }
    if (dev < 0 || dev >= 64) return VOX_ERR_RANGE;
    void* p = addr[dev].load(std::memory_order_acquire);
    if (!p) {
        std::lock_guard<std::mutex> lock(mu);
        p = addr[dev].load(std::memory_order_relaxed);
        if (!p) {
            e = cudaGetSymbolAddress(&p, g_attn_static_scratch);
            if (e != cudaSuccess) {
                set_cuda_error(e);
                return VOX_ERR_CUDA;
            }
            addr[dev].store(p, std::memory_order_release);
        }
    }
    *out = p;
    return VOX_OK;
}

}  // namespace vox

extern "C" vox_status vox_gqa_decode_attn_static(const float* q, const void* k_cache, const void* v_cache, float* out,
                                                 int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                                 int32_t window, int64_t pos, float scale, void* stream)
{
    using namespace vox;
    if (!q || !k_cache || !v_cache || !out) return VOX_ERR_NULL;
    if (n_q_heads < 1 || n_kv_heads < 1 || n_q_heads % n_kv_heads) return VOX_ERR_RANGE;
    if (window < 1 || pos < 0) return VOX_ERR_RANGE;
    if (head_dim != kAttnHd) return VOX_ERR_SHAPE;
    if ((int64_t)n_kv_heads * window > 0x7fffff00LL) return VOX_ERR_SHAPE;
    const int group = n_q_heads / n_kv_heads;
    if (n_kv_heads > kStaticMaxKv || group > kStaticMaxGroup) {
        set_error_text("vox_gqa_decode_attn_static: the static scratch holds at most 8 kv heads with groups of "
                       "at most 4 query heads; use vox_gqa_decode_attn with a workspace");
        return VOX_ERR_RANGE;
    }
    if (((reinterpret_cast<uintptr_t>(k_cache) | reinterpret_cast<uintptr_t>(v_cache) |
          reinterpret_cast<uintptr_t>(out)) & 15u) != 0)
        return VOX_ERR_ALIGN;
    // the records this call writes: n_kv runs of rmax records of the group's size
    const size_t need = (size_t)n_kv_heads * attn_rmax(n_kv_heads) * attn_rec_floats(group, kAttnHd) * sizeof(float);
    if (need > kStaticScratchBytes) {
        set_error_text("vox_gqa_decode_attn_static: shape needs more than the static scratch");
        return VOX_ERR_RANGE;
    }
    void* scratch = nullptr;
    vox_status st = attn_static_scratch(&scratch);
    if (st != VOX_OK) return st;
    return launch_gqa_decode_attn(q, k_cache, v_cache, out, n_q_heads, n_kv_heads, head_dim, window, pos, nullptr,
                                  scale, scratch, static_cast<cudaStream_t>(stream));
}
