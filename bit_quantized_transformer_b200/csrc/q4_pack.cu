// Q4_0 repack (GGUF blocks -> tiled tensor-core layout) and dequantisation.
//
// Q4_0 ("Voxtral Mini 4B Realtime (Rust)", page 5, "Arquitetura": GGUF Q4_0):
// 32 weights per block, fp16 scale d, 4-bit codes q, w = (q - 8) * d; element
// j < 16 is the low nibble of byte j, element j + 16 the high nibble.
//
// Packed layout (one 576-byte record per 16-row tile and 64-column chunk):
//   bytes [16L, 16L+16) for lane L = 4g + t (g = L/4, t = L%4): four 32-bit
//   words; word 2bb+w serves block bb (0, 1) of the chunk and column pair
//   p0 = 2t + 8w (and p0 + 1) of each half of that block.  Nibble slot s of
//   a word (bits 4s..4s+3) holds
//       row   g + 8*((s >> 1) & 1)
//       half  s & 1                  (0: block elements 0..15, 1: 16..31)
//       elem  (s >> 2) & 1           (first or second of the column pair)
//   so one LOP3 with mask 0x000F000F (slots 0, 4) or 0x00F000F0 (slots 1, 5),
//   after an 8-bit shift for slots 2, 6 / 3, 7, yields a half2 that is
//   exactly one register of the m16n8k16 A fragment of that lane.
//   bytes [512 + 8g, 512 + 8g + 8): fp16 d of (row g, block 0), (row g+8,
//   block 0), (row g, block 1), (row g+8, block 1).
#include "vox_internal.cuh"

namespace vox {

__device__ __forceinline__ int gguf_code(const uint8_t* blk18, int e)
{
    uint8_t byte = blk18[2 + (e & 15)];
    return e < 16 ? (byte & 0x0F) : (byte >> 4);
}

// Source row of packed row pr (VOX_PACK_GATE_UP interleaves groups of 8).
__device__ __forceinline__ int64_t pack_src_row(int64_t pr, int gate_up, int64_t half_n)
{
    if (!gate_up) return pr;
    int64_t j = pr >> 4, i = pr & 15;
    return i < 8 ? (j * 8 + i) : (half_n + j * 8 + (i - 8));
}

// One thread per (tile, chunk, lane): writes that lane's 16 code bytes and,
// for t == 0, the 8 scale bytes of its row pair.
__global__ void q4_pack_kernel(const uint8_t* __restrict__ gguf, int64_t n, int64_t k, int gate_up,
                               uint8_t* __restrict__ packed, int64_t tiles, int64_t kc)
{
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int64_t total = tiles * kc * 32;
    if (gid >= total) return;
    int lane = (int)(gid & 31);
    int64_t rec = gid >> 5;                 // tile * kc + chunk
    int64_t tile = rec / kc, chunk = rec % kc;
    int g = lane >> 2, t = lane & 3;
    int64_t nb = k / 32;
    int64_t half_n = n / 2;

    uint32_t words[4] = {0, 0, 0, 0};
    for (int j = 0; j < 4; ++j) {
        int bb = j >> 1, w = j & 1;
        int64_t blk = chunk * 2 + bb;
        for (int s = 0; s < 8; ++s) {
            int rowsel = (s >> 1) & 1, half = s & 1, elem = (s >> 2) & 1;
            int64_t pr = tile * 16 + g + 8 * rowsel;
            int e = half * 16 + 2 * t + 8 * w + elem;
            int code = 8;                                   // padding: weight 0
            if (pr < n && blk < nb) {
                int64_t sr = pack_src_row(pr, gate_up, half_n);
                code = gguf_code(gguf + (sr * nb + blk) * 18, e);
            }
            words[j] |= (uint32_t)code << (4 * s);
        }
    }
    uint8_t* dst = packed + rec * kChunkBytes;
    *reinterpret_cast<uint4*>(dst + 16 * lane) = make_uint4(words[0], words[1], words[2], words[3]);

    if (t == 0) {
        uint16_t dv[4];
        for (int i = 0; i < 4; ++i) {
            int bb = i >> 1, rowsel = i & 1;
            int64_t pr = tile * 16 + g + 8 * rowsel;
            int64_t blk = chunk * 2 + bb;
            uint16_t bits = 0;                              // padding: d = +0
            if (pr < n && blk < nb) {
                const uint8_t* b18 = gguf + (pack_src_row(pr, gate_up, half_n) * nb + blk) * 18;
                bits = (uint16_t)(b18[0] | (b18[1] << 8));
            }
            dv[i] = bits;
        }
        uint2 dd = make_uint2(dv[0] | ((uint32_t)dv[1] << 16), dv[2] | ((uint32_t)dv[3] << 16));
        *reinterpret_cast<uint2*>(dst + kChunkQsBytes + 8 * g) = dd;
    }
}

// One thread per (row, block): decodes 32 weights from the packed layout.
// If row_dev is given, the first row is read from device memory (embedding
// lookup of a token produced on the GPU) after the upstream kernel finishes;
// with `gather`, output row i is packed row row_dev[i] (one token per
// sequence of a batch).
__global__ void q4_dequant_kernel(const uint8_t* __restrict__ packed, int64_t n, int64_t k, int64_t kc,
                                  int64_t row0, const int32_t* __restrict__ row_dev, int64_t nrows,
                                  void* __restrict__ out, int dtype, int64_t ldo, int gather)
{
    // dependents may launch once every CTA has started (a one-row dequant is
    // a few CTAs, so the next projection's CTAs start their weight copies
    // beside it); they still wait for this grid to complete
    pdl_launch_dependents();
    pdl_wait();
    int64_t nb = k / 32;
    int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= nrows * nb) return;
    int64_t rr = gid / nb, b = gid % nb;
    int64_t r;
    if (gather) {
        r = (int64_t)row_dev[rr];
        if (r < 0 || r >= n) {                           // device-side lookup out of range
            if (b == 0) atomicCAS(&g_vox_device_status, 0, 0x0D0);
            return;
        }
    } else {
        const int64_t r0 = row_dev ? (int64_t)(*row_dev) : row0;
        if (r0 < 0 || r0 + nrows > n) {                  // device-side lookup out of range
            if (gid == 0) atomicCAS(&g_vox_device_status, 0, 0x0D0);
            return;
        }
        r = r0 + rr;
    }
    int64_t tile = r >> 4;
    int i = (int)(r & 15), g = i & 7, rowsel = i >> 3;
    int64_t chunk = b >> 1;
    int bb = (int)(b & 1);
    const uint8_t* rec = packed + (tile * kc + chunk) * kChunkBytes;
    uint16_t dbits = *reinterpret_cast<const uint16_t*>(rec + kChunkQsBytes + 8 * g + 2 * (bb * 2 + rowsel));
    float d = __half2float(__ushort_as_half(dbits));

    float w[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        int half = e >> 4, ep = e & 15, wsel = ep >> 3, pp = ep & 7, t = pp >> 1, elem = pp & 1;
        int s = rowsel * 2 + half + elem * 4;
        uint32_t word = *reinterpret_cast<const uint32_t*>(rec + 16 * (4 * g + t) + 4 * (2 * bb + wsel));
        int q = (int)((word >> (4 * s)) & 15u);
        w[e] = (float)(q - 8) * d;                       // exact: 4-bit integer times fp16
    }
    if (dtype == VOX_F32) {
        float* o = reinterpret_cast<float*>(out) + rr * ldo + b * 32;
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = w[e];
    } else {
        uint16_t* o = reinterpret_cast<uint16_t*>(out) + rr * ldo + b * 32;
#pragma unroll
        for (int e = 0; e < 32; ++e) o[e] = f32_to_bf16_bits(w[e]);
    }
}

vox_status launch_q4_pack(const uint8_t* gguf, int64_t n, int64_t k, int gate_up, uint8_t* packed,
                          cudaStream_t s)
{
    int64_t tiles = ceil_div(n, 16), kc = ceil_div(k, 64);
    int64_t total = tiles * kc * 32;
    int threads = 256;
    int64_t blocks = ceil_div(total, threads);
    q4_pack_kernel<<<(unsigned)blocks, threads, 0, s>>>(gguf, n, k, gate_up, packed, tiles, kc);
    return check_launch();
}

vox_status launch_q4_dequant(const uint8_t* packed, int64_t n, int64_t k, int64_t row0,
                             const int32_t* row_dev, int64_t nrows, void* out, int dtype, int64_t ldo,
                             cudaStream_t s, int gather)
{
    int64_t kc = ceil_div(k, 64);
    int64_t total = nrows * (k / 32);
    int threads = 128;
    int64_t blocks = ceil_div(total, threads);
    return launch_pdl(q4_dequant_kernel, dim3((unsigned)blocks), dim3(threads), 0, s,
                      packed, n, k, kc, row0, row_dev, nrows, out, dtype, ldo, gather && row_dev ? 1 : 0);
}

}  // namespace vox
