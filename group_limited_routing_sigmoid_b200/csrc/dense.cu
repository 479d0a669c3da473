// The dense SwiGLU MLP of Beam's first three layers (launch blog
// "Introducing Beam", section "Mixture of Experts": the first 3 layers use a
// dense SwiGLU MLP; section "Residual Stream": SwiGLU product in FP32, norms
// in FP32, depth-scaled residual).  It runs on the same grouped GEMMs as the
// experts, as one expert that every token takes with weight 1 and no
// routed scaling.  This file holds its two small kernels:
//   dense_setup_kernel   the GEMMs' tables for one expert of T rows, and the
//                        identity row map / unit weights the combine reads;
//   dense_swiglu_kernel  h = bf16(silu(sum_s g_s) * sum_s u_s) over the FP32
//                        partial sums of split-K gate|up slices, summed in
//                        slice order.
#include "gemm_common.cuh"

namespace beam {

__global__ void __launch_bounds__(256) dense_setup_kernel(int T, int tiles, int32_t *counts,
                                                          int32_t *offsets, int32_t *tile_off,
                                                          int32_t *pair_row, int32_t *row_pair,
                                                          float *w)
{
    pdl_launch_dependents();
    pdl_wait();
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t == 0) {
        counts[0] = T;
        offsets[0] = 0;
        offsets[1] = T;
        tile_off[0] = 0;
        tile_off[1] = tiles;
    }
    if (t < T) {
        pair_row[t] = t;
        row_pair[t] = t;
        w[t] = 1.0f;
    }
}

// part: [S][T][2I] fp32 (gate in columns 0..I-1, up in I..2I-1), slices
// slice_stride elements apart; h: [T, I] bf16.  Four columns per thread.
__global__ void __launch_bounds__(256) dense_swiglu_kernel(const float *__restrict__ part, int S,
                                                           long long slice_stride, int T, int I,
                                                           __nv_bfloat16 *__restrict__ h)
{
    pdl_launch_dependents();
    pdl_wait();
    const long long q = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // float4 index in [T, I]
    const int nq = I / 4;
    if (q >= (long long)T * nq) return;
    const int t = (int)(q / nq);
    const int i = (int)(q - (long long)t * nq) * 4;
    float4 g = make_float4(0.f, 0.f, 0.f, 0.f), u = g;
    for (int s = 0; s < S; ++s) {
        const float *row = part + (size_t)s * (size_t)slice_stride + (size_t)t * 2 * I;
        const float4 a = *reinterpret_cast<const float4 *>(row + i);
        const float4 b = *reinterpret_cast<const float4 *>(row + I + i);
        g.x += a.x; g.y += a.y; g.z += a.z; g.w += a.w;
        u.x += b.x; u.y += b.y; u.z += b.z; u.w += b.w;
    }
    const __nv_bfloat162 lo =
        __floats2bfloat162_rn(gemm::silu_f32(g.x) * u.x, gemm::silu_f32(g.y) * u.y);
    const __nv_bfloat162 hi =
        __floats2bfloat162_rn(gemm::silu_f32(g.z) * u.z, gemm::silu_f32(g.w) * u.w);
    uint2 packed;
    packed.x = *reinterpret_cast<const uint32_t *>(&lo);
    packed.y = *reinterpret_cast<const uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(h + (size_t)t * I + i) = packed;
}

cudaError_t launch_dense_setup(int T, int tiles, int32_t *counts, int32_t *offsets,
                               int32_t *tile_off, int32_t *pair_row, int32_t *row_pair, float *w,
                               cudaStream_t stream)
{
    return launch_pdl(dense_setup_kernel, dim3((T + 255) / 256), dim3(256), 0, stream, T, tiles,
                      counts, offsets, tile_off, pair_row, row_pair, w);
}

cudaError_t launch_dense_swiglu(const float *part, int S, long long slice_stride, int T, int I,
                                __nv_bfloat16 *h, cudaStream_t stream)
{
    const long long n = (long long)T * (I / 4);
    return launch_pdl(dense_swiglu_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, stream,
                      part, S, slice_stride, T, I, h);
}

}  // namespace beam
