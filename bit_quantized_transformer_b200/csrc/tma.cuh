// Tensor-map (TMA) helpers: host-side encoding through the driver entry
// point, device-side tiled loads, and the 128-byte swizzle address rule.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "vox_internal.cuh"

namespace vox {

// Encode a 2-D row-major tensor map: `rows` rows of `cols` elements with a
// row pitch of `pitch_bytes`, loaded in boxes of box_rows x box_cols with the
// 128-byte swizzle (box_cols * elem_bytes must be 128).  Out-of-range box
// elements read as zero.
vox_status make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                        uint64_t cols, uint64_t rows, uint64_t pitch_bytes, uint32_t box_cols,
                        uint32_t box_rows, CUtensorMapSwizzle swizzle);

// Byte offset of the 16-byte unit `unit` (0..7) of row `row` inside a tile
// written by TMA with the 128-byte swizzle (rows of 128 bytes, tile base
// 1024-byte aligned): the unit index is XORed with the row index mod 8.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t unit)
{
    return row * 128u + ((unit ^ (row & 7u)) << 4);
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int32_t x, int32_t y, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int32_t x, int32_t y, int32_t z,
                                            uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_addr(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}

// Two fp32 -> packed bf16x2 (round to nearest even); `lo` goes to bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Split a pair of floats into bf16 hi + bf16 lo parts (v ~= hi + lo to ~2^-16).
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo)
{
    hi = pack_bf16x2(a, b);
    const float ah = __uint_as_float(hi << 16), bh = __uint_as_float(hi & 0xFFFF0000u);
    lo = pack_bf16x2(a - ah, b - bh);
}

}  // namespace vox
