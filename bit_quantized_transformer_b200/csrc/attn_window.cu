// K6: causal sliding-window multi-head attention of the audio encoder.
//
// voxtral.c page, "모델 아키텍처": 32-layer causal encoder, dim 1280, 32
// heads, window 750 (head_dim 40).  Query row i sits at absolute position
// n_hist + i and sees key position p iff pos_i - window < p <= pos_i; keys
// before n_hist come from the history rows, the rest from the chunk itself.
//
// One CTA per (32 query rows, head): two warps of 16 query rows each, so
// the 256-row chunk x 32 heads gives 256 CTAs.  The keys a CTA needs (its
// 32 rows' windows, 781 positions at window 750) stream through a 3-stage
// ring of 64-key K and V tiles filled with 16-byte cp.async copies, so the
// loads of tile i + 2 overlap the math of tile i.  Per tile (80-byte rows,
// which ldmatrix reads without bank conflicts):
//   S = Q K^T        mma m16n8k16 bf16, head_dim padded to 48 with zeros
//   online softmax in the exp2 domain, masked by position
//   O += P V         P split into bf16 hi + lo parts (two MMAs)
#include "tma.cuh"

namespace vox {

constexpr int kWinQ = 32;       // query rows per CTA
constexpr int kWinWarps = kWinQ / 16;
constexpr int kWinThreads = 32 * kWinWarps;
constexpr int kWinK = 64;       // keys per tile
constexpr int kWinStages = 3;
constexpr int kWinHd = 40;
constexpr int kWinRow = kWinHd * 2;   // 80 bytes
constexpr int kWinTile = kWinK * kWinRow;   // one K or V tile

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

// Copies of key tile [j0, j0 + 64) of head h (K and V) into one ring stage;
// rows at or past j_end are zero-filled.
__device__ __forceinline__ void win_load_tile(const WinArgs& a, int h, int64_t j0, int64_t j_end, uint8_t* sK,
                                              uint8_t* sV, int tid)
{
    for (int i = tid; i < kWinK * 5 * 2; i += kWinThreads) {
        const int mat = i / (kWinK * 5), rem = i - mat * (kWinK * 5), kr = rem / 5, u = rem - kr * 5;
        const int64_t j = j0 + kr;
        const bool in = j < j_end;
        const int64_t jj = in ? j : j_end - 1;                 // a valid address; nothing is read when !in
        const uint16_t* src = jj < a.n_hist ? (mat ? a.vh : a.kh) + jj * a.ld_hist
                                            : (mat ? a.vn : a.kn) + (jj - a.n_hist) * a.ld_new;
        cp_async16((mat ? sV : sK) + kr * kWinRow + u * 16, src + h * kWinHd + u * 8, in ? 16u : 0u);
    }
}

__global__ void __launch_bounds__(kWinThreads) window_attn_kernel(const WinArgs a)
{
    __shared__ __align__(128) uint8_t sKs[kWinStages][kWinTile];
    __shared__ __align__(128) uint8_t sVs[kWinStages][kWinTile];
    pdl_wait();
    pdl_launch_dependents();

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, t = lane & 3;
    const int h = blockIdx.y;
    const int64_t q0 = (int64_t)blockIdx.x * kWinQ;
    const int64_t qw = q0 + warp * 16;                       // first query row of this warp
    const int64_t W = a.window;
    const int64_t n_keys = a.n_hist + a.n_q;

    // Q fragments: rows qw+g, qw+g+8; dims 16kk + {2t, 2t+1, 2t+8, 2t+9}
    uint32_t qa[3][4];
#pragma unroll
    for (int kk = 0; kk < 3; ++kk) {
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            const int64_t row = qw + g + 8 * hf;
            const bool ok = row < a.n_q;
            const uint16_t* qr = a.q + (ok ? row : 0) * a.ldq + h * kWinHd;
            const int d0 = 16 * kk + 2 * t, d1 = d0 + 8;
            qa[kk][hf] = (ok && d0 < kWinHd) ? ld_pair(qr + d0) : 0u;
            qa[kk][2 + hf] = (ok && d1 < kWinHd) ? ld_pair(qr + d1) : 0u;
        }
    }
    // fragment register order: a0a1 (row g, k lo), a2a3 (row g+8, k lo), a4a5 (row g, k hi), a6a7 (row g+8, k hi)
    uint32_t A[3][4];
#pragma unroll
    for (int kk = 0; kk < 3; ++kk) {
        A[kk][0] = qa[kk][0];
        A[kk][1] = qa[kk][1];
        A[kk][2] = qa[kk][2];
        A[kk][3] = qa[kk][3];
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

    // prologue: the first two tiles in flight
#pragma unroll
    for (int st = 0; st < kWinStages - 1; ++st) {
        if (st < ntiles) win_load_tile(a, h, j_begin + (int64_t)st * kWinK, j_end, sKs[st], sVs[st], tid);
        cp_async_commit();
    }
    for (int64_t it = 0; it < ntiles; ++it) {
        const int64_t j0 = j_begin + it * kWinK;
        cp_async_wait<kWinStages - 2>();                     // tile `it` has landed (this thread's copies)
        __syncthreads();                                     // ... everyone's; and stage it-1 is free
        {
            const int64_t nx = it + kWinStages - 1;
            const int sn = (int)(nx % kWinStages);
            if (nx < ntiles) win_load_tile(a, h, j_begin + nx * kWinK, j_end, sKs[sn], sVs[sn], tid);
            cp_async_commit();
        }
        const int sc = (int)(it % kWinStages);
        const uint32_t sKa = smem_addr(sKs[sc]), sVa = smem_addr(sVs[sc]);

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

    // ---- normalise and store rows g, g+8
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int64_t qi = qw + g + 8 * hf;
        if (qi >= a.n_q) continue;
        const float inv = 1.0f / l_run[hf];
#pragma unroll
        for (int n = 0; n < 5; ++n) {
            const int d = 8 * n + 2 * t;
            const float v0 = o[n][2 * hf] * inv, v1 = o[n][2 * hf + 1] * inv;
            const int64_t idx = qi * a.ldo + h * kWinHd + d;
            if (a.out_bf16) {
                static_cast<uint16_t*>(a.out)[idx] = f32_to_bf16_bits(v0);
                static_cast<uint16_t*>(a.out)[idx + 1] = f32_to_bf16_bits(v1);
            } else {
                static_cast<float*>(a.out)[idx] = v0;
                static_cast<float*>(a.out)[idx + 1] = v1;
            }
        }
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
    dim3 grid((unsigned)ceil_div(n_q, kWinQ), (unsigned)n_heads);
    return launch_pdl(window_attn_kernel, grid, dim3(kWinThreads), 0, s, a);
}

}  // namespace vox
