// Device-side arithmetic of the Q4_0 GEMV shared by the per-projection
// kernel (q4_gemv.cu) and the persistent decoder step (decoder_step.cu): the
// register dequantisation + tensor-core product of one packed 576-byte
// record, the greedy-argmax ordering, and the epilogue activations.
//
// Q4_0: w = (q - 8) * d, GGUF blocks of 32 ("Voxtral Mini 4B Realtime
// (Rust)", page 5, "Arquitetura").  The record layout is described in
// q4_pack.cu.
#pragma once

#include "vox_internal.cuh"

namespace vox {

// "a beats b" for greedy argmax: NaN wins, then larger value, then lower index.
__device__ __forceinline__ bool argmax_better(float va, int32_t ia, float vb, int32_t ib)
{
    bool na = isnan(va), nb = isnan(vb);
    if (na != nb) return na;
    if (!na && va != vb) return va > vb;
    return ia < ib;
}

// A 64-bit key whose unsigned order is the argmax order above: NaN above
// every number, numbers by value (-0 == +0), then the lower index.  0 is
// below every key, so a zeroed slot is an empty candidate.
__device__ __forceinline__ unsigned long long argmax_key(float v, int32_t i)
{
    uint32_t u = __float_as_uint(v), ku;
    if (isnan(v)) {
        ku = 0xFFFFFFFFu;
    } else {
        if (u == 0x80000000u) u = 0u;
        ku = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    }
    return ((unsigned long long)ku << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)i);
}

__device__ __forceinline__ uint32_t atom_add_acq_rel_gpu(uint32_t* p, uint32_t v)
{
    uint32_t old;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

__device__ __forceinline__ float4 lds128f(uint32_t addr)
{
    float4 v;
    asm("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ float gelu_erf(float v)
{
    return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f));
}

__device__ __forceinline__ float silu_f(float v)
{
    return v / (1.0f + expf(-v));
}

// Four consecutive floats p[4f .. 4f+3]; one 16-byte load when aligned.
__device__ __forceinline__ float4 ld_f4(const float* p, int f, int vec)
{
    if (vec) return *(reinterpret_cast<const float4*>(p) + f);
    return make_float4(p[4 * f], p[4 * f + 1], p[4 * f + 2], p[4 * f + 3]);
}

// One record's math for one warp: two Q4_0 blocks, each as two chained
// m16n8k16 MMAs (low / high nibbles) from zero, then corrected by the
// block's offset constant and scaled by d / (activation scale) in fp32.
// q, dd: this lane's code and scale words.  p[2h + e] += row g + 8h, token 2t + e.
template <int MT>
__device__ __forceinline__ void gemv_record(uint4 q, uint2 dd, uint32_t bs, uint32_t cb, int cs, int chunk,
                                            int m, int tok, int t, float (&p)[4])
{
    const uint32_t M_P = 0x000F000Fu, M_Q = 0x00F000F0u, C_P = 0x64006400u, C_Q = 0x54005400u;
    const float2 d0 = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
    const float2 d1 = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
    const int blk0 = chunk * 2;
    const int ms = MT == 1 ? 1 : m;
    const uint32_t bsb = bs + 4u * ((blk0 * ms + tok) * 16 + t * 4);
    float4 cm = make_float4(0.f, 0.f, 0.f, 0.f);
    if (MT == 1) cm = lds128f(cb + 8u * blk0);                   // (constant, 1/scale) of both blocks
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
        const uint4 B = lds128(bsb + 4u * bb * ms * 16);
        float2 c0, c1;                                           // tokens 2t, 2t + 1
        if (MT == 1) {
            c0 = bb ? make_float2(cm.z, cm.w) : make_float2(cm.x, cm.y);
            c1 = c0;
        } else {
            // [block][token], cs (even) entries per block: tokens 2t, 2t + 1 in one
            // 16-byte load; a quad's lanes read adjacent words (no bank conflict)
            const int t0 = 2 * t, t1 = 2 * t + 1;
            c0 = t0 < m ? lds64f(cb + 8u * ((blk0 + bb) * cs + t0)) : make_float2(0.f, 0.f);
            c1 = t1 < m ? lds64f(cb + 8u * ((blk0 + bb) * cs + t1)) : make_float2(0.f, 0.f);
        }
        const uint32_t w0 = bb ? q.z : q.x;
        const uint32_t w1 = bb ? q.w : q.y;
        const uint32_t w0s = w0 >> 8, w1s = w1 >> 8;
        const uint32_t alo[4] = {lop3_and_or(w0, M_P, C_P), lop3_and_or(w0s, M_P, C_P),
                                 lop3_and_or(w1, M_P, C_P), lop3_and_or(w1s, M_P, C_P)};
        const uint32_t ahi[4] = {lop3_and_or(w0, M_Q, C_Q), lop3_and_or(w0s, M_Q, C_Q),
                                 lop3_and_or(w1, M_Q, C_Q), lop3_and_or(w1s, M_Q, C_Q)};
        float cc[4] = {0.f, 0.f, 0.f, 0.f};
        mma_f16_16816(cc, alo, B.x, B.y, cc);
        mma_f16_16816(cc, ahi, B.z, B.w, cc);
        const float dg = bb ? d1.x : d0.x, dg8 = bb ? d1.y : d0.y;
        p[0] = fmaf(dg * c0.y, cc[0] + c0.x, p[0]);
        p[2] = fmaf(dg8 * c0.y, cc[2] + c0.x, p[2]);
        if (MT != 1) {
            p[1] = fmaf(dg * c1.y, cc[1] + c1.x, p[1]);
            p[3] = fmaf(dg8 * c1.y, cc[3] + c1.x, p[3]);
        }
    }
}

// One record's math for one warp at M = 1 in the persistent step: each
// block's two chained MMAs start from the block's offset constant instead of
// zero, so they return the block's dot product in scaled units; the two
// blocks' d weight them, and the chunk's inverse activation scale (one value
// for both blocks, the activations being scaled per 128 columns) multiplies
// their sum.  At M = 1 each block keeps (constant, 1/scale, constant,
// 1/scale) in shared memory: one 16-byte load is the MMA's accumulator input
// as it stands (elements 0 and 2, rows g and g + 8 of token 0, start from the
// constant; 1 and 3 belong to the unused token columns).  bsb: this lane's
// B-fragment words of the chunk's first block (the second block's are 64
// bytes on); cbc: the chunk's two constant quads.  p0 += row g, p2 += row g + 8.
__device__ __forceinline__ void gemv_record_m1(uint4 q, uint2 dd, uint32_t bsb, uint32_t cbc, float& p0, float& p2)
{
    const uint32_t M_P = 0x000F000Fu, M_Q = 0x00F000F0u, C_P = 0x64006400u, C_Q = 0x54005400u;
    const float2 d0 = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
    const float2 d1 = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));
    float c[2][4];
    float inv = 0.f;
#pragma unroll
    for (int bb = 0; bb < 2; ++bb) {
        const float4 k4 = lds128f(cbc + 16u * bb);
        const uint4 B = lds128(bsb + 64u * bb);
        const uint32_t w0 = bb ? q.z : q.x;
        const uint32_t w1 = bb ? q.w : q.y;
        const uint32_t w0s = w0 >> 8, w1s = w1 >> 8;
        const uint32_t alo[4] = {lop3_and_or(w0, M_P, C_P), lop3_and_or(w0s, M_P, C_P),
                                 lop3_and_or(w1, M_P, C_P), lop3_and_or(w1s, M_P, C_P)};
        const uint32_t ahi[4] = {lop3_and_or(w0, M_Q, C_Q), lop3_and_or(w0s, M_Q, C_Q),
                                 lop3_and_or(w1, M_Q, C_Q), lop3_and_or(w1s, M_Q, C_Q)};
        const float kin[4] = {k4.x, k4.y, k4.z, k4.w};
        float cc[4];
        mma_f16_16816(cc, alo, B.x, B.y, kin);
        mma_f16_16816(cc, ahi, B.z, B.w, cc);
        c[bb][0] = cc[0];
        c[bb][2] = cc[2];
        inv = k4.y;
    }
    p0 = fmaf(inv, fmaf(d1.x, c[1][0], d0.x * c[0][0]), p0);
    p2 = fmaf(inv, fmaf(d1.y, c[1][2], d0.y * c[0][2]), p2);
}

// Rotary embedding: (cos, sin) of the angle pos * theta^(-2i/hd) of pair
// i = col / 2.  The angle is reduced to turns in double precision, so long
// positions keep it accurate; the sine and cosine of the reduced angle are
// taken in single precision.  Not inlined: only the q and k tiles of a
// projection with RoPE on reach it.
static __device__ __noinline__ float2 rope_cs(int64_t col, int hd, int64_t pos, float theta)
{
    const double inv = exp2(-(2.0 * (double)(col >> 1) / hd) * log2((double)theta));
    double turns = (double)pos * inv * 0.15915494309189535;     // 1 / (2 pi)
    turns -= floor(turns);
    float s, c;
    sincospif(2.0f * (float)turns, &s, &c);
    return make_float2(c, s);
}

// One element of an adjacent pair after the rotation (col even: the pair's
// first element, col odd: its second); v is this element, partner the other.
__device__ __forceinline__ float rope_rotate(float v, float partner, int64_t col, int hd, int64_t pos, float theta)
{
    const float2 cs = rope_cs(col, hd, pos, theta);
    return (col & 1) ? fmaf(partner, cs.y, v * cs.x) : fmaf(-partner, cs.y, v * cs.x);
}

}  // namespace vox
