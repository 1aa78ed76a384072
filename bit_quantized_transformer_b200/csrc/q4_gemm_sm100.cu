// K2: fused Q4_0 dequantise + GEMM on the 5th-generation tensor cores
// (tcgen05), for M >= 16 activation rows: encoder chunks and batched decode.
//
// Y[i][j] = sum_c X[i][c] W[j][c], W = (q - 8) * d (GGUF Q4_0, "Voxtral Mini
// 4B Realtime (Rust)", page 5 "Arquitetura"), with the dequantisation fused
// into the matmul ("브라우저에서 도는 4B 음성인식: Voxtral Rust+WASM 구현 해부",
// "F32(9GB) vs Q4 GGUF(2.5GB)").  Encoder shapes: voxtral.c page, "모델
// 아키텍처" (dim 1280, FFN 5120, adapter 5120 -> 3072).
//
// One CTA computes a 128-weight-row x BN-token tile of Y^T in tensor memory:
//   warp 0      producer: per 64-column chunk, one 2-D TMA load of the 8
//               packed 576-byte records of the 128 rows (the packed weight
//               viewed as [tiles][chunks x 576 B]) and one TMA tile (128-byte
//               swizzle) of BN activation rows x 64 columns;
//   warp 1      allocates BN tensor-memory columns and, from one thread,
//               issues tcgen05.mma kind::f16 (M=128, N=BN, K=16, bf16 in, fp32
//               accumulate) on shared-memory descriptors, committing each
//               stage back to the producer;
//   warps 2-9   dequantise into tensor memory (VOX_GEMM_A_TMEM, the
//               default): warp w converts block (w - 2) >> 2 of the rows of its
//               lane quarter (w & 3), one row per lane, gathering the row's
//               codes from the 4 lanes' slots of its record, and writes the
//               bf16 pairs with tcgen05.st into the stage's 32 columns after
//               the accumulator; the MMA then reads A from tensor memory.
//               With VOX_GEMM_A_TMEM=0 the tile goes to shared memory instead:
//               warp w takes the record of row tile w - 2, lane
//               (g, t) its 16 bytes of codes (rows g and g+8, both 32-column
//               blocks); VOX_GEMM_DQ_WARPS=16 builds two warps per record, one
//               block each (measured slower: per chunk about 600 cycles of
//               conversion and stores, 400 of waiting for the stage and 90 for
//               the proxy fence, and more warps do not shorten it; the chunk's
//               shared-memory traffic, A written then read by the MMA next to
//               the X tile, is the likely bound).  Each 32-bit word gives four bf16 pairs 128 + q by
//               OR-ing the nibble into the fraction of 128.0 (exact), then
//               an exact subtraction of 136 gives q - 8, which is widened to
//               fp32 and multiplied by d in fp32 (exact: 4 x 11 significant
//               bits), and the product is rounded to bf16 once (nearest
//               even) -- the same bits vox_q4_dequant returns -- and stored
//               in the canonical K-major
//               128-byte-swizzled layout the MMA reads (4-byte stores, free of
//               bank conflicts); after the last chunk they read the
//               accumulator with tcgen05.ld and run the epilogue (residual
//               add, GELU, fp32 or bf16 store).
#include "tma.cuh"

namespace vox {

#ifndef VOX_GEMM_DQ_WARPS
#define VOX_GEMM_DQ_WARPS 8
#endif
constexpr int kGemmDqWarps = VOX_GEMM_DQ_WARPS;     // dequantising (and epilogue) warps: 8 or 16
static_assert(kGemmDqWarps == 8 || kGemmDqWarps == 16, "8 or 16 dequantising warps");
constexpr int kGemmThreads = 32 * (2 + kGemmDqWarps);
[[maybe_unused]] constexpr int kGemmRecWarps = kGemmDqWarps / 8;   // warps per 16-row record (shared-memory tile)
constexpr int kGemmEpiParts = kGemmDqWarps / 4;     // accumulator column parts per tensor-memory lane quarter
#ifndef VOX_GEMM_A_TMEM
#define VOX_GEMM_A_TMEM 1
#endif
constexpr bool kATmem = VOX_GEMM_A_TMEM != 0;       // dequantised tile in tensor memory (else shared memory)
// with the tensor-memory tile, the dequantising warps form groups of 8 (2 per
// lane quarter) that take alternate chunks
constexpr int kGemmDqGroups = kATmem ? kGemmDqWarps / 8 : 1;
constexpr int kGemmRows = 128;                      // MMA M (weight rows per CTA)
constexpr int kGemmRawBytes = 8 * kChunkBytes;      // 4608
constexpr int kGemmABytes = kATmem ? 0 : kGemmRows * 128;   // the 16 KB bf16 tile of 64 columns, if in shared memory
constexpr int kGemmACols = 32;                      // tensor-memory columns of one stage's tile (64 bf16 per row)

struct GemmArgs {
    const uint8_t* w;
    int64_t n, k;
    int32_t tiles, kc;
    int64_t m;
    void* y;
    int32_t y_bf16;
    int64_t ldy;
    int32_t op;
    const float* res;
    int64_t ldr;
    int32_t splits;                  // K splits = CTAs of a cluster along z (1: no split)
};

template <int BN>
struct GemmCfg {
    static constexpr int xbytes = BN * 128;
    static constexpr int stage = ((xbytes + kGemmABytes + kGemmRawBytes) + 1023) / 1024 * 1024;
    static constexpr int stages = (200 * 1024 / stage) > 6 ? 6 : (200 * 1024 / stage);
    static constexpr int bars = stages * stage;
    static constexpr int smem = bars + (3 * stages + 2) * 8 + 16 + 1024;
    // accumulator columns [0, BN), then (A in tensor memory) 32 columns per stage; a power of two
    static constexpr int tmem_need = (BN < 32 ? 32 : BN) + (kATmem ? stages * kGemmACols : 0);
    static constexpr int tmem_cols = tmem_need <= 32 ? 32 : tmem_need <= 64 ? 64 : tmem_need <= 128 ? 128
                                   : tmem_need <= 256 ? 256 : 512;
    static_assert(tmem_need <= 512, "tensor memory holds 512 columns");
};

__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr)
{
    // start address >> 4 (bits 0-13), LBO 16 B (unused for swizzled K-major),
    // SBO 1024 B between 8-row groups, version 1, 128-byte swizzle.
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

__device__ __forceinline__ void umma_bf16(uint32_t dtmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(dtmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// The same MMA with A (M x 16, rows on lanes, K pairs along columns) read from tensor memory.
__device__ __forceinline__ void umma_bf16_ta(uint32_t dtmem, uint32_t atmem, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(dtmem), "r"(atmem), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// 16 consecutive 32-bit tensor-memory columns of this warp's 32 lanes (one
// value per lane and column), then wait for the stores.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
                   "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
                 : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8])
{
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// bf16x2 a - b (exact here: both are small integers).
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ float gelu_erf_g(float v) { return 0.5f * v * (1.0f + erff(v * 0.70710678118654752f)); }

// The epilogue of one output element: residual add (the residual value `res`
// loaded by the caller, ahead of the sums; 0 unless op is VOX_EP_RESIDUAL) or
// GELU, then an fp32 or bf16 store.
__device__ __forceinline__ void gemm_store_pre(const GemmArgs& a, int64_t mi, int64_t row, float o, float res)
{
    if (a.op == VOX_EP_RESIDUAL) o += res;
    else if (a.op == VOX_EP_GELU) o = gelu_erf_g(o);
    if (a.y_bf16)
        static_cast<uint16_t*>(a.y)[mi * a.ldy + row] = f32_to_bf16_bits(o);
    else
        static_cast<float*>(a.y)[mi * a.ldy + row] = o;
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_map(uint32_t saddr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

// Distributed-shared-memory load; issued without a memory clobber so that
// several can be in flight before their values are summed.
// 16 bytes of another CTA's shared memory in the cluster (address from mapa).
__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr));
    return v;
}

// SPLIT: K split over the CTAs of a cluster along z (a.splits > 1); the
// instance without it carries none of the reduction code.
template <int BN, bool SPLIT>
__global__ void __launch_bounds__(kGemmThreads, 1)
q4_gemm_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap, const GemmArgs a)
{
    using C = GemmCfg<BN>;
    static_assert(BN * kGemmRows * 4 <= C::bars, "the split-K partial tile must fit the ring");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::bars);
    uint64_t* aready = full + C::stages;
    uint64_t* empty = aready + C::stages;
    uint64_t* accb = empty + C::stages;
    volatile uint32_t* s_tmem = reinterpret_cast<volatile uint32_t*>(accb + 2);
    volatile int32_t* s_fail = reinterpret_cast<volatile int32_t*>(accb + 2) + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t group = blockIdx.x;              // 8 row tiles = 128 weight rows
    const int64_t m0 = (int64_t)blockIdx.y * BN;
    // this CTA's K chunks [kb0, kb0 + nk): split blockIdx.z of a.splits
    const int S = SPLIT ? a.splits : 1;
    const int kb0 = SPLIT ? (int)((int64_t)blockIdx.z * a.kc / S) : 0;
    const int nk = SPLIT ? (int)((int64_t)(blockIdx.z + 1) * a.kc / S) - kb0 : a.kc;

    if (tid == 0) {
        for (int s = 0; s < C::stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&aready[s], kGemmDqWarps / kGemmDqGroups);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&accb[0], 1);
        s_fail[0] = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_addr((const void*)s_tmem)), "r"((uint32_t)C::tmem_cols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *s_tmem;
    pdl_wait();

    if (warp == 0) {
        // ------------------------------------------------------- producer
        if (lane == 0) {
            pdl_launch_dependents();
            prefetch_tmap(&xmap);
            prefetch_tmap(&wmap);
            const uint32_t bytes = (uint32_t)kGemmRawBytes + C::xbytes;   // rows past the matrix read as zeros
            for (int i = 0; i < nk; ++i) {
                const int kb = kb0 + i;
                const int s = i % C::stages;
                const uint32_t ph = (uint32_t)((i / C::stages) & 1);
                if (!s_fail[0] && !mbar_wait_bounded(&empty[s], ph ^ 1u, 0x301)) s_fail[0] = 1;
                if (s_fail[0]) break;
                uint8_t* st = smem + s * C::stage;
                mbar_arrive_expect_tx(&full[s], bytes);
                tma_load_2d(st + C::xbytes + kGemmABytes, &wmap, kb * (kChunkBytes / 4), (int32_t)(group * 8), &full[s]);
                tma_load_2d(st, &xmap, kb * 64, (int32_t)m0, &full[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- MMA issue
        if (lane == 0) {
            const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                                   ((uint32_t)(kGemmRows >> 4) << 24);
            for (int i = 0; i < nk; ++i) {
                const int s = i % C::stages;
                const uint32_t ph = (uint32_t)((i / C::stages) & 1);
                if (!s_fail[0] && !mbar_wait_bounded(&aready[s], ph, 0x302)) s_fail[0] = 1;
                if (s_fail[0]) break;
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t xs = smem_addr(smem + s * C::stage);
                if constexpr (kATmem) {
                    const uint32_t at = tmem + (uint32_t)(BN < 32 ? 32 : BN) + (uint32_t)(s * kGemmACols);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16_ta(tmem, at + 8u * kk, umma_desc_sw128(xs + kk * 32), idesc, (i > 0 || kk > 0) ? 1u : 0u);
                } else {
                    const uint32_t as = xs + C::xbytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_bf16(tmem, umma_desc_sw128(as + kk * 32), umma_desc_sw128(xs + kk * 32), idesc,
                                  (i > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&empty[s]);
            }
            umma_commit(&accb[0]);
        }
    } else {
        // ------------------------------------------------- dequant + epilogue
        const int dw = warp - 2;                    // 0 .. kGemmDqWarps-1
        const int q = warp & 3;                     // tensor-memory lane quarter of this warp
        const int r = 32 * q + lane;                // weight row of the epilogue
        const uint32_t M_L = 0x000F000Fu, C_B = 0x43004300u, B136 = 0x43084308u;   // 128.0, 136.0 (bf16x2)
        if constexpr (kATmem) {
            // lane = weight row 32 q + lane (this warp's tensor-memory lanes); block
            // dw >> 2 (32 columns = 16 tensor-memory columns) of every chunk.  The
            // row's codes sit in the 4 lanes' slots (g, t = 0..3) of its record.
            const int grp = dw >> 3;                // chunks grp, grp + groups, ...
            const int bbk = (dw >> 2) & 1;
            const int rrow = 32 * q + lane;
            const int rtile = rrow >> 4, rg = rrow & 7, rhalf = (rrow >> 3) & 1;
            const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(BN < 32 ? 32 : BN) + 16u * (uint32_t)bbk;
            for (int i = grp; i < nk; i += kGemmDqGroups) {
                const int s = i % C::stages;
                const uint32_t ph = (uint32_t)((i / C::stages) & 1);
                if (!s_fail[0] && !mbar_wait_bounded(&full[s], ph, 0x303)) s_fail[0] = 1;
                const uint8_t* rec = smem + s * C::stage + C::xbytes + rtile * kChunkBytes;
                uint2 wv[4];
#pragma unroll
                for (int t4 = 0; t4 < 4; ++t4) wv[t4] = *reinterpret_cast<const uint2*>(rec + 16 * (4 * rg + t4) + 8 * bbk);
                const uint32_t db = *reinterpret_cast<const uint32_t*>(rec + kChunkQsBytes + 8 * rg + 4 * bbk);
                const float dsc = __half2float(__ushort_as_half((unsigned short)(rhalf ? db >> 16 : db & 0xFFFFu)));
                uint32_t vals[16];
#pragma unroll
                for (int t4 = 0; t4 < 4; ++t4)
#pragma unroll
                    for (int wi = 0; wi < 2; ++wi)
#pragma unroll
                        for (int hh = 0; hh < 2; ++hh) {
                            const uint32_t w = wi ? wv[t4].y : wv[t4].x;
                            // this row's nibble pair of the word: row g (w, w >> 4), row g + 8 (w >> 8, w >> 12)
                            const uint32_t src = rhalf ? (hh ? w >> 12 : w >> 8) : (hh ? w >> 4 : w);
                            const uint32_t raw = lop3_and_or(src, M_L, C_B);          // 128 + q, exact
                            const uint32_t qm = bf16x2_sub(raw, B136);                 // q - 8, exact
                            // K pair 16 hh + 8 wi + 2 t4 of the block: column 8 hh + 4 wi + t4
                            vals[8 * hh + 4 * wi + t4] =
                                pack_bf16x2(__uint_as_float(qm << 16) * dsc, __uint_as_float(qm & 0xFFFF0000u) * dsc);
                        }
                tmem_st16(ta + (uint32_t)(s * kGemmACols), vals);
                asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&aready[s]);
            }
        } else {
            const int rt = dw / kGemmRecWarps;      // the row tile (record) this warp dequantises
            const int g = lane >> 2, t = lane & 3;
            const uint32_t row_g = (uint32_t)(rt * 16 + g), row_g8 = row_g + 8u;
            for (int i = 0; i < nk; ++i) {
                const int s = i % C::stages;
                const uint32_t ph = (uint32_t)((i / C::stages) & 1);
                if (!s_fail[0] && !mbar_wait_bounded(&full[s], ph, 0x303)) s_fail[0] = 1;
                uint8_t* st = smem + s * C::stage;
                uint8_t* A = st + C::xbytes;
                if (rt * 16 < (int)(a.n - group * kGemmRows)) {
                    const uint8_t* rec = st + C::xbytes + kGemmABytes + rt * kChunkBytes;
                    const uint4 qv = *reinterpret_cast<const uint4*>(rec + 16 * lane);
                    const uint2 dd = *reinterpret_cast<const uint2*>(rec + kChunkQsBytes + 8 * g);
                    // scales in fp32 (exact): d(row g, block 0), d(row g+8, block 0), d(g, 1), d(g+8, 1)
                    const float2 d0 = __half22float2(*reinterpret_cast<const __half2*>(&dd.x));
                    const float2 d1 = __half22float2(*reinterpret_cast<const __half2*>(&dd.y));

    #pragma unroll
                    for (int bb = 0; bb < 2; ++bb) {
                        if (kGemmRecWarps == 2 && bb != (dw & 1)) continue;    // two warps share a record: one block each
    #pragma unroll
                        for (int wi = 0; wi < 2; ++wi) {
                            const uint32_t w = wi ? (bb ? qv.w : qv.y) : (bb ? qv.z : qv.x);
                            // nibble pairs: (w, w>>8) low halves, (w>>4, w>>12) high halves; rows g, g+8
                            const uint32_t src[4] = {w, w >> 8, w >> 4, w >> 12};
    #pragma unroll
                            for (int h = 0; h < 4; ++h) {
                                const uint32_t raw = lop3_and_or(src[h], M_L, C_B);            // 128 + q, exact
                                const uint32_t qm = bf16x2_sub(raw, B136);          // q - 8, exact
                                const float dd_ = (h & 1) ? (bb ? d1.y : d0.y) : (bb ? d1.x : d0.x);
                                const uint32_t v = pack_bf16x2(__uint_as_float(qm << 16) * dd_,
                                                               __uint_as_float(qm & 0xFFFF0000u) * dd_);
                                const uint32_t row = (h & 1) ? row_g8 : row_g;
                                // columns 32 bb + 16 (h >> 1) + 8 wi + 2t, +1: unit 4 bb + 2 (h >> 1) + wi
                                const uint32_t unit = (uint32_t)(bb * 4 + (h >> 1) * 2 + wi);
                                *reinterpret_cast<uint32_t*>(A + sw128_offset(row, unit) + 4 * t) = v;
                            }
                        }
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&aready[s]);
            }
        }
        // ---- epilogue
        if (!s_fail[0] && !mbar_wait_bounded(&accb[0], 0, 0x304)) s_fail[0] = 1;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const int64_t row = group * kGemmRows + r;
        const int c0 = (dw >> 2) * (BN / kGemmEpiParts);   // this warp's accumulator columns
        // split K: the partial tile goes to the idle ring as [token][row] fp32
        float* part = reinterpret_cast<float*>(smem);
        for (int cc = 0; cc < BN / kGemmEpiParts; cc += 8) {
            float v[8];
            tmem_ld8(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(c0 + cc), v);
            if constexpr (SPLIT) {
#pragma unroll
                for (int j = 0; j < 8; ++j) part[(c0 + cc + j) * kGemmRows + r] = v[j];
            } else if (row < a.n) {
                float rv[8];                         // residuals of the 8 tokens, loaded together
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int64_t mi = m0 + c0 + cc + j;
                    rv[j] = (a.op == VOX_EP_RESIDUAL && mi < a.m) ? a.res[mi * a.ldr + row] : 0.f;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int64_t mi = m0 + c0 + cc + j;
                    if (mi >= a.m) break;
                    gemm_store_pre(a, mi, row, v[j], rv[j]);
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if constexpr (SPLIT) {
        // Every CTA of the cluster holds its partial tile; CTA `rank` sums
        // tokens [rank BN / S, (rank + 1) BN / S) over the ranks in order
        // 0 .. S-1 (deterministic) through distributed shared memory and
        // runs the epilogue on them.  Every thread of every CTA reaches both
        // cluster barriers, also after a wait that gave up.
        cluster_sync_all();
        uint32_t rank;
        asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
        const uint32_t pl = smem_addr(smem);
        uint32_t rb[8];
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2) rb[s2] = cluster_map(pl, (uint32_t)(s2 < S ? s2 : 0));
        const int cb = (int)(rank * BN / S), ce = (int)((rank + 1) * BN / S);
        // groups of 4 consecutive rows of one token (16 bytes of every rank's
        // partial tile), QPT groups per thread per round: all their loads (the
        // ranks' partials and the residuals) in flight before the sums
        const int nq = (ce - cb) * (kGemmRows / 4);
        constexpr int QPT = kGemmThreads >= 512 ? 1 : 2;          // groups per thread per round
        for (int q0 = tid; q0 < nq; q0 += QPT * kGemmThreads) {
            float4 v[QPT][8];
            float rv[QPT][4];
#pragma unroll
            for (int u = 0; u < QPT; ++u) {
                const int qd = q0 + u * kGemmThreads;
                const int c = cb + qd / (kGemmRows / 4), r4 = 4 * (qd % (kGemmRows / 4));
                const uint32_t off = qd < nq ? (uint32_t)(c * kGemmRows + r4) * 4u : 0u;
#pragma unroll
                for (int s2 = 0; s2 < 8; ++s2)
                    v[u][s2] = (s2 < S && qd < nq) ? ld_cluster_f32x4(rb[s2] + off) : make_float4(0.f, 0.f, 0.f, 0.f);
                const int64_t mi = m0 + c;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int64_t row = group * kGemmRows + r4 + e;
                    rv[u][e] = (a.op == VOX_EP_RESIDUAL && qd < nq && row < a.n && mi < a.m) ? a.res[mi * a.ldr + row]
                                                                                             : 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < QPT; ++u) {
                const int qd = q0 + u * kGemmThreads;
                if (qd >= nq) break;
                float4 o = v[u][0];
#pragma unroll
                for (int s2 = 1; s2 < 8; ++s2)
                    if (s2 < S) {
                        o.x += v[u][s2].x;
                        o.y += v[u][s2].y;
                        o.z += v[u][s2].z;
                        o.w += v[u][s2].w;
                    }
                const int c = cb + qd / (kGemmRows / 4), r4 = 4 * (qd % (kGemmRows / 4));
                const int64_t mi = m0 + c;
                const float ov[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int64_t row = group * kGemmRows + r4 + e;
                    if (row < a.n && mi < a.m) gemm_store_pre(a, mi, row, ov[e], rv[u][e]);
                }
            }
        }
        cluster_sync_all();
    }
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)C::tmem_cols)
                     : "memory");
    }
}

template <int BN>
static vox_status launch_gemm_bn(const GemmArgs& a, const void* x, int64_t ldx, cudaStream_t s)
{
    using C = GemmCfg<BN>;
    CUtensorMap xmap;
    vox_status st = make_tmap_2d(&xmap, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)a.k, (uint64_t)a.m,
                                 (uint64_t)ldx * 2, 64, BN, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != VOX_OK) return st;
    // the packed weight as 32-bit words: [tiles][kc * 144], one box = one chunk of 8 row tiles
    CUtensorMap wmap;
    st = make_tmap_2d(&wmap, a.w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, (uint64_t)a.kc * (kChunkBytes / 4),
                      (uint64_t)a.tiles, (uint64_t)a.kc * kChunkBytes, kChunkBytes / 4, 8, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != VOX_OK) return st;
    static std::atomic<unsigned long long> attr_done{0}, attr_done_split{0};
    dim3 grid((unsigned)ceil_div(a.tiles, 8), (unsigned)ceil_div(a.m, BN), (unsigned)a.splits);
    if (a.splits > 1) {
        st = smem_attr_per_device(reinterpret_cast<const void*>(q4_gemm_kernel<BN, true>), C::smem, attr_done_split);
        if (st != VOX_OK) return st;
        return launch_pdl_cluster(q4_gemm_kernel<BN, true>, grid, dim3(kGemmThreads), (size_t)C::smem, s,
                                  (unsigned)a.splits, xmap, wmap, a);
    }
    st = smem_attr_per_device(reinterpret_cast<const void*>(q4_gemm_kernel<BN, false>), C::smem, attr_done);
    if (st != VOX_OK) return st;
    return launch_pdl(q4_gemm_kernel<BN, false>, grid, dim3(kGemmThreads), (size_t)C::smem, s, xmap, wmap, a);
}

// Clusters of `splits` CTAs of q4_gemm_kernel<BN> that the device runs at
// once (the occupancy query accounts for how the SMs fall into GPCs), cached
// per device; 0 if the query fails.
template <int BN>
static int gemm_max_clusters(int dev, int splits)
{
    static std::atomic<int> cache[64][9];
    if (dev < 0 || dev >= 64 || splits < 1 || splits > 8) return 0;
    int v = cache[dev][splits].load(std::memory_order_relaxed);
    if (v) return v - 1;
    using C = GemmCfg<BN>;
    static std::atomic<unsigned long long> attr_done{0};
    if (smem_attr_per_device(reinterpret_cast<const void*>(q4_gemm_kernel<BN, true>), C::smem, attr_done) != VOX_OK)
        return 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, (unsigned)splits);
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = C::smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = (unsigned)splits;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, q4_gemm_kernel<BN, true>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    cache[dev][splits].store(n + 1, std::memory_order_relaxed);
    return n;
}

static int max_clusters(int dev, int bn, int splits)
{
    switch (bn) {
    case 32: return gemm_max_clusters<32>(dev, splits);
    case 64: return gemm_max_clusters<64>(dev, splits);
    case 128: return gemm_max_clusters<128>(dev, splits);
    default: return gemm_max_clusters<256>(dev, splits);
    }
}

// Tile width BN and K splits by a cost model in microseconds fitted to B200
// measurements of this kernel: a K chunk takes about 0.54, 0.6, 0.6 and
// 0.9 us per CTA for BN 32, 64, 128 and 256; a CTA has about 6 us of fixed
// cost (12 at BN 256, whose epilogue is four times larger), and a split adds
// about 2 us of cluster reduction.  Cost = waves x (chunks per split x chunk
// time + fixed + reduction).  Splits (at most 8, one portable cluster, and
// at least 2 chunks each) are only taken when all clusters run at once.
// VOX_GEMM_BN and VOX_GEMM_SPLITS override the choice.
static void pick_tile(int64_t tiles, int64_t m, int kc, int& bn_out, int& splits_out)
{
    const int64_t groups = ceil_div(tiles, 8);
    const int64_t sms = device_sm_count();
    int dev = -1;                                             // looked up once: the capacity cache is per device
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    const char* ebn = getenv("VOX_GEMM_BN");
    const char* esp = getenv("VOX_GEMM_SPLITS");
    const int fbn = ebn ? atoi(ebn) : 0, fsp = esp ? atoi(esp) : 0;
    double best_cost = 1e300;
    int best_bn = 256, best_s = 1;
    for (int bn = 256; bn >= 32; bn >>= 1) {
        if (fbn && bn != fbn) continue;
        if (!fbn && bn > 32 && (bn >> 1) >= m) continue;    // a smaller tile already covers every row
        // measured on B200 (one wave): a K chunk costs about 0.53 us whatever the
        // tile width (its 128 x 64 weights are dequantised once per CTA), and a
        // CTA's fixed cost grows with the tile (accumulator read-out, epilogue)
        const double t_chunk = 0.53;
        const double fixed = bn == 256 ? 8.5 : bn == 128 ? 6.0 : bn == 64 ? 4.3 : 3.5;
        for (int sp = 1; sp <= 8; ++sp) {
            if (fsp && sp != fsp) continue;
            if (sp > 1 && kc / sp < 2) break;
            const int64_t clusters = groups * ceil_div(m, bn);
            int64_t waves = ceil_div(clusters * sp, sms);
            if (sp > 1) {
                const int mc = max_clusters(dev, bn, sp);
                if (mc < 1) continue;
                waves = ceil_div(clusters, mc);
                if (!fsp && waves > 1) continue;
            }
            // the cluster reduction: each rank sums bn / sp tokens x 128 rows over the ranks
            const double reduce = sp > 1 ? 0.5 + 0.23e-3 * (double)(bn * kGemmRows / sp) : 0.0;
            const double cost = (double)waves * ((double)ceil_div(kc, sp) * t_chunk + fixed + reduce);
            if (cost < best_cost) {
                best_cost = cost;
                best_bn = bn;
                best_s = sp;
            }
        }
    }
    bn_out = best_bn;
    splits_out = best_s;
}

vox_status launch_q4_gemm(const uint8_t* w, int64_t n, int64_t k, const void* x, int64_t m, int64_t ldx, void* y,
                          int y_dtype, int64_t ldy, const vox_epilogue* ep, cudaStream_t s)
{
    GemmArgs a = {};
    a.w = w;
    a.n = n;
    a.k = k;
    a.tiles = (int32_t)ceil_div(n, 16);
    a.kc = (int32_t)(k / 64);
    a.m = m;
    a.y = y;
    a.y_bf16 = y_dtype == VOX_BF16;
    a.ldy = ldy;
    a.op = ep ? ep->op : VOX_EP_NONE;
    a.res = ep ? ep->residual : nullptr;
    a.ldr = ep ? ep->ldr : 0;
    int bn = 256, splits = 1;
    pick_tile(a.tiles, m, a.kc, bn, splits);
    a.splits = splits;
    switch (bn) {
    case 32: return launch_gemm_bn<32>(a, x, ldx, s);
    case 64: return launch_gemm_bn<64>(a, x, ldx, s);
    case 128: return launch_gemm_bn<128>(a, x, ldx, s);
    default: return launch_gemm_bn<256>(a, x, ldx, s);
    }
}

}  // namespace vox
