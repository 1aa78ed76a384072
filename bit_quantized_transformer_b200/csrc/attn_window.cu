// K6: causal sliding-window multi-head attention of the audio encoder.
//
// voxtral.c page, "모델 아키텍처": 32-layer causal encoder, dim 1280, 32
// heads, window 750 (head_dim 40).  Query row i sits at absolute position
// n_hist + i and sees key position p iff pos_i - window < p <= pos_i; keys
// before n_hist come from the history rows, the rest from the chunk itself.
//
// One CTA of eight warps per (32 query rows, head), so the 256-row chunk x
// 32 heads gives 256 CTAs, two per SM.  The keys a CTA needs (its 32 rows'
// windows, 781 positions at window 750) are cut into 64-key tiles, dealt to
// four key splits in rounds (round r holds tiles 4r .. 4r+3): warp w takes
// query rows 16 (w & 1) .. +15 and the tiles of split w >> 1.  A round's
// four K and V tiles are loaded by the whole CTA with 16-byte cp.async
// copies into one of two buffers, so the next round's loads overlap this
// round's math.  Per tile (80-byte rows, which ldmatrix reads without bank
// conflicts):
//   S = Q K^T        mma m16n8k16 bf16, head_dim padded to 48 with zeros
//   online softmax in the exp2 domain, masked by position
//   O += P V         P split into bf16 hi + lo parts (two MMAs)
// At the end each warp leaves its rows' (m, l, O) in shared memory and the
// CTA merges the four splits of every row max-first in split order.
#include "tma.cuh"

namespace vox {

constexpr int kWinQ = 32;       // query rows per CTA
constexpr int kWinSplits = 4;   // key splits per CTA
constexpr int kWinWarps = (kWinQ / 16) * kWinSplits;
constexpr int kWinThreads = 32 * kWinWarps;
constexpr int kWinK = 64;       // keys per tile
constexpr int kWinHd = 40;
constexpr int kWinRow = kWinHd * 2;   // 80 bytes
constexpr int kWinTile = kWinK * kWinRow;   // one K or V tile
constexpr int kWinRound = 2 * kWinSplits * kWinTile;   // K and V tiles of one round (40 KB)
constexpr int kWinSmem = 2 * kWinRound;                 // two round buffers (80 KB)
// merge area (reuses the round buffers): per warp O[16][40] then (m, l)[16]
constexpr int kWinMergeFloats = 16 * kWinHd + 32;
static_assert(kWinWarps * kWinMergeFloats * 4 <= kWinSmem, "merge area must fit the round buffers");

struct WinArgs {
    const uint16_t* q;
    int64_t ldq;
    const uint16_t* kh;
    const uint16_t* vh;
    int64_t ld_hist, n_hist;
    const uint16_t* kn;
    const uint16_t* vn;
    int64_t ld_new, n_q;
    void* out;
    int32_t out_bf16;
    int64_t ldo;
    int32_t n_heads, window;
    float sl2;                  // scale * log2(e)
};

__device__ __forceinline__ uint32_t ld_pair(const uint16_t* p)
{
    return (uint32_t)p[0] | ((uint32_t)p[1] << 16);
}

__device__ __forceinline__ void ldsm_x2(uint32_t (&r)[2], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x2_trans(uint32_t (&r)[2], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1])
                 : "r"(addr) : "memory");
}

// Copies of round r's tiles (tile 4r + sp for split sp, keys from j_begin)
// into one round buffer: K tiles first, then V tiles; rows at or past j_end
// (and tiles past the last) are zero-filled.
__device__ __forceinline__ void win_load_round(const WinArgs& a, int h, int64_t j_begin, int64_t r, int64_t j_end,
                                               uint8_t* buf, int tid)
{
    for (int i = tid; i < 2 * kWinSplits * kWinK * 5; i += kWinThreads) {
        const int mat = i / (kWinSplits * kWinK * 5), rem = i - mat * (kWinSplits * kWinK * 5);
        const int sp = rem / (kWinK * 5), rem2 = rem - sp * (kWinK * 5), kr = rem2 / 5, u = rem2 - kr * 5;
        const int64_t j = j_begin + (r * kWinSplits + sp) * kWinK + kr;
        const bool in = j < j_end;
        const int64_t jj = in ? j : j_end - 1;                 // a valid address; nothing is read when !in
        const uint16_t* src = jj < a.n_hist ? (mat ? a.vh : a.kh) + jj * a.ld_hist
                                            : (mat ? a.vn : a.kn) + (jj - a.n_hist) * a.ld_new;
        cp_async16(buf + (mat * kWinSplits + sp) * kWinTile + kr * kWinRow + u * 16, src + h * kWinHd + u * 8,
                   in ? 16u : 0u);
    }
}

__global__ void __launch_bounds__(kWinThreads, 2) window_attn_kernel(const WinArgs a)
{
    extern __shared__ __align__(128) uint8_t win_smem[];
    pdl_wait();
    pdl_launch_dependents();

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int rg = warp & 1, sp = warp >> 1;                 // row group, key split
    const int h = blockIdx.y;
    const int64_t q0 = (int64_t)blockIdx.x * kWinQ;
    const int64_t qw = q0 + rg * 16;                          // first query row of this warp
    const int64_t W = a.window;
    const int64_t n_keys = a.n_hist + a.n_q;

    // Q fragments: rows qw+g, qw+g+8; dims 16kk + {2t, 2t+1, 2t+8, 2t+9}
    // (register order a0a1: row g k lo, a2a3: row g+8 k lo, a4a5: row g k hi, a6a7: row g+8 k hi)
    uint32_t A[3][4];
#pragma unroll
    for (int kk = 0; kk < 3; ++kk) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int64_t row = qw + g + 8 * hf;
            const bool ok = row < a.n_q;
            const uint16_t* qr = a.q + (ok ? row : 0) * a.ldq + h * kWinHd;
            const int d0 = 16 * kk + 2 * t, d1 = d0 + 8;
            A[kk][hf] = (ok && d0 < kWinHd) ? ld_pair(qr + d0) : 0u;
            A[kk][2 + hf] = (ok && d1 < kWinHd) ? ld_pair(qr + d1) : 0u;
        }
    }

    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float o[5][4];
#pragma unroll
    for (int n = 0; n < 5; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

    const int64_t p_lo = a.n_hist + q0;
    const int64_t q_last = (q0 + kWinQ < a.n_q ? q0 + kWinQ : a.n_q) - 1;
    const int64_t p_hi = a.n_hist + q_last;
    const int64_t j_begin = p_lo - W + 1 > 0 ? p_lo - W + 1 : 0;
    const int64_t j_end = p_hi + 1 < n_keys ? p_hi + 1 : n_keys;
    const int64_t ntiles = j_end > j_begin ? (j_end - j_begin + kWinK - 1) / kWinK : 0;
    const int64_t nrounds = (ntiles + kWinSplits - 1) / kWinSplits;

    if (nrounds > 0) win_load_round(a, h, j_begin, 0, j_end, win_smem, tid);
    cp_async_commit();
    for (int64_t r = 0; r < nrounds; ++r) {
        cp_async_wait<0>();                                  // round r has landed (this thread's copies)
        __syncthreads();                                     // ... everyone's; and round r-1's buffer is free
        if (r + 1 < nrounds) win_load_round(a, h, j_begin, r + 1, j_end, win_smem + ((r + 1) & 1) * kWinRound, tid);
        cp_async_commit();
        const int64_t tile = r * kWinSplits + sp;
        if (tile >= ntiles) continue;                        // warp-uniform: this split has no tile this round
        const int64_t j0 = j_begin + tile * kWinK;
        uint8_t* buf = win_smem + (r & 1) * kWinRound;
        const uint32_t sKa = smem_addr(buf + sp * kWinTile), sVa = smem_addr(buf + (kWinSplits + sp) * kWinTile);

        // ---- S = Q K^T : 8 n-tiles of 8 keys
        float s[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; nt += 2) {
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                // matrices: (keys nt, dims 16kk..+7), (keys nt, +8..+15), (keys nt+1, ...), (keys nt+1, ...)
                const int mi = lane >> 3;
                const int kr = 8 * (nt + (mi >> 1)) + (lane & 7);
                uint32_t b[4];
                ldsm_x4(b, sKa + kr * kWinRow + (16 * kk + 8 * (mi & 1)) * 2);
                mma_bf16_16816(s[nt], A[kk], b[0], b[1], s[nt]);
                mma_bf16_16816(s[nt + 1], A[kk], b[2], b[3], s[nt + 1]);
            }
            {
                // k-step 2: dims 32..39 only (40..47 are zero in A)
                const int mi = (lane >> 3) & 1;
                const int kr = 8 * (nt + mi) + (lane & 7);
                uint32_t b[2];
                ldsm_x2(b, sKa + kr * kWinRow + 32 * 2);
                mma_bf16_16816(s[nt], A[2], b[0], 0u, s[nt]);
                mma_bf16_16816(s[nt + 1], A[2], b[1], 0u, s[nt + 1]);
            }
        }
        // ---- mask + online softmax; rows g (hf=0) and g+8 (hf=1)
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int hf = e >> 1;
                const int64_t qi = qw + g + 8 * hf;
                const int64_t pq = a.n_hist + qi;
                const int64_t j = j0 + 8 * nt + 2 * t + (e & 1);
                const bool vis = qi < a.n_q && j < j_end && j <= pq && j > pq - W;
                s[nt][e] = vis ? s[nt][e] * a.sl2 : -INFINITY;
                mx[hf] = fmaxf(mx[hf], s[nt][e]);
            }
        }
        float corr[2];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            mx[hf] = fmaxf(mx[hf], __shfl_xor_sync(0xffffffffu, mx[hf], 1));
            mx[hf] = fmaxf(mx[hf], __shfl_xor_sync(0xffffffffu, mx[hf], 2));
            const float mn = fmaxf(m_run[hf], mx[hf]);
            corr[hf] = (mn == -INFINITY) ? 1.f : exp2f(m_run[hf] - mn);
            m_run[hf] = mn;
        }
        float ls[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int hf = e >> 1;
                const float p = (m_run[hf] == -INFINITY) ? 0.f : exp2f(s[nt][e] - m_run[hf]);
                s[nt][e] = p;
                ls[hf] += p;
            }
        }
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            ls[hf] += __shfl_xor_sync(0xffffffffu, ls[hf], 1);
            ls[hf] += __shfl_xor_sync(0xffffffffu, ls[hf], 2);
            l_run[hf] = l_run[hf] * corr[hf] + ls[hf];
        }
#pragma unroll
        for (int n = 0; n < 5; ++n) {
            o[n][0] *= corr[0];
            o[n][1] *= corr[0];
            o[n][2] *= corr[1];
            o[n][3] *= corr[1];
        }
        // ---- O += P V : 4 k-steps of 16 keys, 5 dim tiles of 8
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t ph[4], pl[4];
            split_bf16x2(s[2 * kk][0], s[2 * kk][1], ph[0], pl[0]);
            split_bf16x2(s[2 * kk][2], s[2 * kk][3], ph[1], pl[1]);
            split_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1], ph[2], pl[2]);
            split_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3], ph[3], pl[3]);
#pragma unroll
            for (int n = 0; n < 4; n += 2) {
                // matrices: (keys lo, dims n), (keys hi, dims n), (keys lo, dims n+1), (keys hi, dims n+1)
                const int mi = lane >> 3;
                const int kr = 16 * kk + 8 * (mi & 1) + (lane & 7);
                uint32_t b[4];
                ldsm_x4_trans(b, sVa + kr * kWinRow + (8 * (n + (mi >> 1))) * 2);
                mma_bf16_16816(o[n], ph, b[0], b[1], o[n]);
                mma_bf16_16816(o[n], pl, b[0], b[1], o[n]);
                mma_bf16_16816(o[n + 1], ph, b[2], b[3], o[n + 1]);
                mma_bf16_16816(o[n + 1], pl, b[2], b[3], o[n + 1]);
            }
            {
                const int mi = (lane >> 3) & 1;
                const int kr = 16 * kk + 8 * mi + (lane & 7);
                uint32_t b[2];
                ldsm_x2_trans(b, sVa + kr * kWinRow + 32 * 2);
                mma_bf16_16816(o[4], ph, b[0], b[1], o[4]);
                mma_bf16_16816(o[4], pl, b[0], b[1], o[4]);
            }
        }
    }

    // ---- this warp's (m, l, O) of its 16 rows -> shared memory, then the
    // four splits of every (row, dim) merged max-first in split order
    __syncthreads();                                         // every warp is done with the round buffers
    float* mw = reinterpret_cast<float*>(win_smem) + warp * kWinMergeFloats;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int row = g + 8 * hf;
#pragma unroll
        for (int n = 0; n < 5; ++n) {
            const int d = 8 * n + 2 * t;
            mw[row * kWinHd + d] = o[n][2 * hf];
            mw[row * kWinHd + d + 1] = o[n][2 * hf + 1];
        }
        if (t == 0) {
            mw[16 * kWinHd + 2 * row] = m_run[hf];
            mw[16 * kWinHd + 2 * row + 1] = l_run[hf];
        }
    }
    __syncthreads();
    for (int e = tid; e < kWinQ * kWinHd; e += kWinThreads) {
        const int row = e / kWinHd, d = e - row * kWinHd;
        const int64_t qi = q0 + row;
        if (qi >= a.n_q) continue;
        const int rgi = row >> 4, rl = row & 15;
        float M = -INFINITY;
#pragma unroll
        for (int s2 = 0; s2 < kWinSplits; ++s2)
            M = fmaxf(M, reinterpret_cast<const float*>(win_smem)[(2 * s2 + rgi) * kWinMergeFloats + 16 * kWinHd + 2 * rl]);
        float O = 0.f, L = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < kWinSplits; ++s2) {
            const float* ms = reinterpret_cast<const float*>(win_smem) + (2 * s2 + rgi) * kWinMergeFloats;
            const float mv = ms[16 * kWinHd + 2 * rl];
            if (mv == -INFINITY) continue;
            const float f = exp2f(mv - M);
            O = fmaf(f, ms[rl * kWinHd + d], O);
            L = fmaf(f, ms[16 * kWinHd + 2 * rl + 1], L);
        }
        const float v = O / L;
        const int64_t idx = qi * a.ldo + h * kWinHd + d;
        if (a.out_bf16)
            static_cast<uint16_t*>(a.out)[idx] = f32_to_bf16_bits(v);
        else
            static_cast<float*>(a.out)[idx] = v;
    }
}

vox_status launch_window_attn(const void* q, int64_t ldq, const void* k_hist, const void* v_hist, int64_t ld_hist,
                              int64_t n_hist, const void* k_new, const void* v_new, int64_t ld_new, int64_t n_q,
                              void* out, int out_dtype, int64_t ldo, int n_heads, int head_dim, int window,
                              float scale, cudaStream_t s)
{
    if (head_dim != kWinHd) return VOX_ERR_SHAPE;
    auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if ((n_hist > 0 && (!al(k_hist) || !al(v_hist) || ld_hist % 8)) || !al(k_new) || !al(v_new) || ld_new % 8)
        return VOX_ERR_ALIGN;
    WinArgs a = {};
    a.q = static_cast<const uint16_t*>(q);
    a.ldq = ldq;
    a.kh = static_cast<const uint16_t*>(k_hist);
    a.vh = static_cast<const uint16_t*>(v_hist);
    a.ld_hist = ld_hist;
    a.n_hist = n_hist;
    a.kn = static_cast<const uint16_t*>(k_new);
    a.vn = static_cast<const uint16_t*>(v_new);
    a.ld_new = ld_new;
    a.n_q = n_q;
    a.out = out;
    a.out_bf16 = out_dtype == VOX_BF16;
    a.ldo = ldo;
    a.n_heads = n_heads;
    a.window = window;
    a.sl2 = scale * 1.4426950408889634f;
    static std::atomic<unsigned long long> attr_done{0};
    vox_status st = smem_attr_per_device(reinterpret_cast<const void*>(window_attn_kernel), kWinSmem, attr_done);
    if (st != VOX_OK) return st;
    dim3 grid((unsigned)ceil_div(n_q, kWinQ), (unsigned)n_heads);
    return launch_pdl(window_attn_kernel, grid, dim3(kWinThreads), kWinSmem, s, a);
}

}  // namespace vox
