// Host plumbing (error state, device queries, tensor-map encoding) and the
// small glue kernels: RMSNorm with fp32/bf16 output and the end-of-step
// position advance.
#include <mutex>
#include <stdio.h>
#include <string.h>

#include "tma.cuh"

namespace vox {

__device__ int32_t g_vox_device_status = 0;

static thread_local char t_last_error[256] = "";

void set_cuda_error(cudaError_t e)
{
    snprintf(t_last_error, sizeof(t_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
}

const char* last_error_text() { return t_last_error; }

void set_error_text(const char* text)
{
    snprintf(t_last_error, sizeof(t_last_error), "%s", text);
}

vox_status check_launch()
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        set_cuda_error(e);
        return VOX_ERR_CUDA;
    }
    return VOX_OK;
}

int device_sm_count()
{
    static int cached[64];
    static bool init[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!init[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
        init[dev] = true;
    }
    return cached[dev];
}

// ------------------------------------------------------------ tensor maps
static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

vox_status make_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype, int elem_bytes,
                        uint64_t cols, uint64_t rows, uint64_t pitch_bytes, uint32_t box_cols, uint32_t box_rows,
                        CUtensorMapSwizzle swizzle)
{
    (void)elem_bytes;
    auto fn = get_encode_fn();
    if (!fn) {
        snprintf(t_last_error, sizeof(t_last_error), "cuTensorMapEncodeTiled unavailable");
        return VOX_ERR_CUDA;
    }
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(t_last_error, sizeof(t_last_error), "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return VOX_ERR_CUDA;
    }
    return VOX_OK;
}

// ------------------------------------------------------------------ RMSNorm
// One CTA per row: y = x / sqrt(mean(x^2) + eps) * g (g = 1 when NULL);
// with normalize == 0 the row is only converted (y = x * g).
__global__ void rmsnorm_kernel(const float* __restrict__ x, int64_t n, int64_t ldx, float eps,
                               const float* __restrict__ g, void* __restrict__ out, int out_bf16, int64_t ldo,
                               int normalize)
{
    pdl_wait();
    pdl_launch_dependents();
    __shared__ float red[32];
    const int64_t row = blockIdx.x;
    const float* xr = x + row * ldx;
    float ssq = 0.f;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) ssq = fmaf(xr[i], xr[i], ssq);
    for (int o = 16; o > 0; o >>= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ssq;
    __syncthreads();
    if (threadIdx.x == 0) {
        float s = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += red[w];
        red[0] = normalize ? 1.0f / sqrtf(s / (float)n + eps) : 1.0f;
    }
    __syncthreads();
    const float r = red[0];
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
        float v = xr[i] * r;
        if (g) v *= g[i];
        if (out_bf16)
            static_cast<uint16_t*>(out)[row * ldo + i] = f32_to_bf16_bits(v);
        else
            static_cast<float*>(out)[row * ldo + i] = v;
    }
}

// The same with 16-byte accesses: each thread keeps its VPT float4 of the
// row in registers between the sum of squares and the scaling (one pass over
// x), and stores 4 outputs at once.  Per element the arithmetic is that of
// rmsnorm_kernel; the sum of squares is accumulated in another order, so the
// two agree to rounding.
template <int VPT>
__global__ void rmsnorm_vec_kernel(const float* __restrict__ x, int64_t n4, int64_t ldx, float eps,
                                   const float* __restrict__ g, void* __restrict__ out, int out_bf16, int64_t ldo,
                                   int normalize)
{
    pdl_wait();
    pdl_launch_dependents();
    __shared__ float red[32];
    const int64_t row = blockIdx.x;
    const float4* xr = reinterpret_cast<const float4*>(x + row * ldx);
    float4 v[VPT];
    float ssq = 0.f;
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int64_t i = threadIdx.x + (int64_t)k * blockDim.x;
        v[k] = i < n4 ? xr[i] : make_float4(0.f, 0.f, 0.f, 0.f);
        ssq = fmaf(v[k].x, v[k].x, ssq);
        ssq = fmaf(v[k].y, v[k].y, ssq);
        ssq = fmaf(v[k].z, v[k].z, ssq);
        ssq = fmaf(v[k].w, v[k].w, ssq);
    }
    for (int o = 16; o > 0; o >>= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ssq;
    __syncthreads();
    if (threadIdx.x == 0) {
        float sum = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) sum += red[w];
        red[0] = normalize ? 1.0f / sqrtf(sum / (float)(4 * n4) + eps) : 1.0f;
    }
    __syncthreads();
    const float r = red[0];
#pragma unroll
    for (int k = 0; k < VPT; ++k) {
        const int64_t i = threadIdx.x + (int64_t)k * blockDim.x;
        if (i >= n4) break;
        float4 y = make_float4(v[k].x * r, v[k].y * r, v[k].z * r, v[k].w * r);
        if (g) {
            const float4 gv = reinterpret_cast<const float4*>(g)[i];
            y = make_float4(y.x * gv.x, y.y * gv.y, y.z * gv.z, y.w * gv.w);
        }
        if (out_bf16) {
            const uint2 pk = make_uint2((uint32_t)f32_to_bf16_bits(y.x) | ((uint32_t)f32_to_bf16_bits(y.y) << 16),
                                        (uint32_t)f32_to_bf16_bits(y.z) | ((uint32_t)f32_to_bf16_bits(y.w) << 16));
            reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + row * ldo)[i] = pk;
        } else {
            reinterpret_cast<float4*>(static_cast<float*>(out) + row * ldo)[i] = y;
        }
    }
}

// Rows of x -> out through the 16-byte kernel when the row length, strides
// and pointers allow it, else through rmsnorm_kernel.
static vox_status launch_rows(const float* x, int64_t m, int64_t n, int64_t ldx, float eps, const float* g, void* out,
                              int out_bf16, int64_t ldo, int normalize, cudaStream_t s)
{
    auto al = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; };
    const bool vec = n % 4 == 0 && ldx % 4 == 0 && ldo % 4 == 0 && al(x, 16) && (!g || al(g, 16)) &&
                     al(out, out_bf16 ? 8 : 16) && n / 4 <= 8 * 1024;
    if (!vec)
        return launch_pdl(rmsnorm_kernel, dim3((unsigned)m), dim3(256), 0, s, x, n, ldx, eps, g, out, out_bf16, ldo,
                          normalize);
    const int64_t n4 = n / 4;
    const int vpt = n4 <= 1024 ? 1 : n4 <= 2048 ? 2 : n4 <= 4096 ? 4 : 8;
    const unsigned threads = (unsigned)((ceil_div(n4, vpt) + 31) / 32 * 32);
    switch (vpt) {
    case 1:
        return launch_pdl(rmsnorm_vec_kernel<1>, dim3((unsigned)m), dim3(threads), 0, s, x, n4, ldx, eps, g, out,
                          out_bf16, ldo, normalize);
    case 2:
        return launch_pdl(rmsnorm_vec_kernel<2>, dim3((unsigned)m), dim3(threads), 0, s, x, n4, ldx, eps, g, out,
                          out_bf16, ldo, normalize);
    case 4:
        return launch_pdl(rmsnorm_vec_kernel<4>, dim3((unsigned)m), dim3(threads), 0, s, x, n4, ldx, eps, g, out,
                          out_bf16, ldo, normalize);
    default:
        return launch_pdl(rmsnorm_vec_kernel<8>, dim3((unsigned)m), dim3(threads), 0, s, x, n4, ldx, eps, g, out,
                          out_bf16, ldo, normalize);
    }
}

vox_status launch_rmsnorm(const float* x, int64_t m, int64_t n, int64_t ldx, float eps, const float* g, void* out,
                          int out_dtype, int64_t ldo, cudaStream_t s)
{
    return launch_rows(x, m, n, ldx, eps, g, out, (int)(out_dtype == VOX_BF16), ldo, 1, s);
}

vox_status launch_cast_rows(const float* x, int64_t m, int64_t n, int64_t ldx, void* out, int out_dtype,
                            int64_t ldo, cudaStream_t s)
{
    return launch_rows(x, m, n, ldx, 0.0f, nullptr, out, (int)(out_dtype == VOX_BF16), ldo, 0, s);
}

// ------------------------------------------------------------ history roll
// Streaming encoder chunks ("주요 기능": the encoder takes the audio in
// overlapping chunks): the next chunk's history of one layer is the last
// `window` rows of this chunk's history followed by its own R new rows.
// Row i of the result is history row i + R while i + R < window, else new
// row i - (window - R) (when R >= window only new rows remain).  bf16 rows
// of `dim` elements, copied 16 bytes at a time; the output never aliases the
// inputs.
__global__ void hist_roll_kernel(const uint16_t* __restrict__ hist, int64_t ld_hist, const uint16_t* __restrict__ nw,
                                 int64_t ld_new, int64_t R, int64_t window, int64_t dim, uint16_t* __restrict__ out,
                                 int64_t ld_out)
{
    pdl_wait();
    pdl_launch_dependents();
    const int64_t per_row = dim / 8;
    const int64_t total = window * per_row;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / per_row, c = (i - r * per_row) * 8;
        const int64_t src_h = r + R;
        const uint16_t* src = src_h < window ? hist + src_h * ld_hist + c : nw + (src_h - window) * ld_new + c;
        *reinterpret_cast<uint4*>(out + r * ld_out + c) = *reinterpret_cast<const uint4*>(src);
    }
}

vox_status launch_hist_roll(const void* hist, int64_t ld_hist, const void* nw, int64_t ld_new, int64_t R,
                            int64_t window, int64_t dim, void* out, int64_t ld_out, cudaStream_t s)
{
    const int64_t total = window * (dim / 8);
    int64_t blocks = ceil_div(total, 256);
    if (blocks > 4 * 148) blocks = 4 * 148;
    return launch_pdl(hist_roll_kernel, dim3((unsigned)blocks), dim3(256), 0, s, static_cast<const uint16_t*>(hist),
                      ld_hist, static_cast<const uint16_t*>(nw), ld_new, R, window, dim, static_cast<uint16_t*>(out),
                      ld_out);
}

// --------------------------------------------------------- position advance
__global__ void advance_pos_kernel(int64_t* pos, int n)
{
    // one CTA: the next kernels may launch at once and start their weight
    // copies beside it; they still wait for this grid to complete
    pdl_launch_dependents();
    pdl_wait();
    if ((int)threadIdx.x < n) pos[threadIdx.x] += 1;
}

// Positions pos[0 .. n) advance by one (n <= 32).
vox_status launch_advance_pos(int64_t* pos, cudaStream_t s, int n)
{
    return launch_pdl(advance_pos_kernel, dim3(1), dim3(32), 0, s, pos, n);
}

}  // namespace vox
