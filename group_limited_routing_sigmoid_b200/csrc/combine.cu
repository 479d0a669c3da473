// Combine of the Beam MoE block, with the optional post-norm and
// depth-scaled residual update fused in.
//
//   o[t]   = routed_scaling * sum_j w[t,j] * y[row(t,j)]     (FP32 or bf16 y, FP32 sum,
//                                                             slot order)
//   out[t] = bf16_rn(o[t])
//   n[t]   = o[t] / sqrt(mean(o[t]^2) + eps) * gamma          (if gamma)
//   stream[t] <- sqrt((k-1)/k) * stream[t] + n[t] / sqrt(k)
// Launch blog "Introducing Beam": section "Mixture of Experts" (normalised
// router weights, x2.5) and section "Residual Stream" (weights sqrt((k-1)/k)
// and 1/sqrt(k); every sub-layer normalised before and after; norms in FP32).
#include "kernels.cuh"

namespace beam {

namespace {
// 16-byte vectors (8 hidden values each) per thread: one while a row fits
// 640 threads (H <= 5120: every load of a thread in flight at once), else two
// (H <= 8192)
constexpr int kCombOneVecThreads = 640;
constexpr int kCombTwoVecThreads = 512;
constexpr int kCombBatch = 4;           // expert slots whose loads are in flight together

__device__ __forceinline__ void unpack8(const uint4 &raw, float (&v)[8])
{
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
}  // namespace

// Block per token; thread q takes the 16-byte vectors q (and q + blockDim.x
// when VECS is 2) of the row (8 hidden values each).  The loads of kCombBatch expert slots of a
// vector are issued before their sums, which take the slots in order (FP32
// FMA), so every value is the same slot-order sum.
// WIDE: FP32 expert outputs (a.y32), all top_k slots' loads in flight at
// once; otherwise bf16 outputs (a.y).
template <bool WIDE, int VECS>
__global__ void __launch_bounds__(VECS == 1 ? kCombOneVecThreads : kCombTwoVecThreads)
    combine_kernel(CombineArgs a)
{
    constexpr int kCombVecs = VECS;
    constexpr int kCombMaxThreads = VECS == 1 ? kCombOneVecThreads : kCombTwoVecThreads;
    pdl_launch_dependents();
    pdl_wait();
    if (a.status && status_is_set(a.status)) return;   // a check failed earlier in this pass
    __shared__ int rows[32];
    __shared__ float wts[32];
    __shared__ float red[kCombMaxThreads / 32];
    const int t = blockIdx.x;
    const int tid = threadIdx.x;
    const int nvec = a.H / 8;
    const int nsum = a.top_k;                  // expert slots
    constexpr bool wide = WIDE;                // FP32 expert outputs
    if (tid < nsum) {
        rows[tid] = a.pair_row[(size_t)t * a.top_k + tid];
        wts[tid] = a.w[(size_t)t * a.top_k + tid];
    }
    __syncthreads();

    float acc[kCombVecs][8];
    float ss = 0.f;
#pragma unroll
    for (int v = 0; v < kCombVecs; ++v) {
        const int q = tid + v * blockDim.x;   // vector index in the row
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[v][i] = 0.f;
        if (q >= nvec) continue;
        if constexpr (wide) {
            constexpr int B = 8;   // slots in flight
            for (int j0 = 0; j0 < nsum; j0 += B) {
                float4 lo[B], hi[B];
#pragma unroll
                for (int j = 0; j < B; ++j)
                    if (j0 + j < nsum) {
                        const float4 *src = reinterpret_cast<const float4 *>(
                            a.y32 + (size_t)rows[j0 + j] * a.H + 8 * q);
                        lo[j] = src[0];
                        hi[j] = src[1];
                    }
#pragma unroll
                for (int j = 0; j < B; ++j) {
                    if (j0 + j < nsum) {
                        const float y[8] = {lo[j].x, lo[j].y, lo[j].z, lo[j].w,
                                            hi[j].x, hi[j].y, hi[j].z, hi[j].w};
                        const float wj = wts[j0 + j];
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[v][i] = fmaf(wj, y[i], acc[v][i]);
                    }
                }
            }
        } else {
            for (int j0 = 0; j0 < nsum; j0 += kCombBatch) {
                uint4 raw[kCombBatch];
#pragma unroll
                for (int j = 0; j < kCombBatch; ++j)
                    if (j0 + j < nsum)
                        raw[j] = reinterpret_cast<const uint4 *>(a.y + (size_t)rows[j0 + j] * a.H)[q];
#pragma unroll
                for (int j = 0; j < kCombBatch; ++j) {
                    if (j0 + j < nsum) {
                        float y[8];
                        unpack8(raw[j], y);
                        const float wj = wts[j0 + j];
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[v][i] = fmaf(wj, y[i], acc[v][i]);
                    }
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[v][i] *= a.scaling;
        if (a.out) {
            uint4 packed;
            __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&packed);
#pragma unroll
            for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(acc[v][2 * i], acc[v][2 * i + 1]);
            reinterpret_cast<uint4 *>(a.out + (size_t)t * a.H)[q] = packed;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) ss += acc[v][i] * acc[v][i];
    }
    if (!a.residual) return;

    float scale = 1.0f;
    if (a.gamma) {
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if ((tid & 31) == 0) red[tid >> 5] = ss;
        __syncthreads();
        float tot = 0.f;
        const int nw = (blockDim.x + 31) >> 5;
        for (int wv = 0; wv < nw; ++wv) tot += red[wv];
        scale = 1.0f / sqrtf(tot / (float)a.H + a.eps);
    }
#pragma unroll
    for (int v = 0; v < kCombVecs; ++v) {
        const int q = tid + v * blockDim.x;
        if (q >= nvec) continue;
        float4 *st = reinterpret_cast<float4 *>(a.residual + (size_t)t * a.H + 8 * q);
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
            float4 sv = st[h2];
            float n[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) n[i] = acc[v][4 * h2 + i];
            if (a.gamma) {
                const float4 g = reinterpret_cast<const float4 *>(a.gamma + 8 * q)[h2];
                n[0] = n[0] * scale * g.x;
                n[1] = n[1] * scale * g.y;
                n[2] = n[2] * scale * g.z;
                n[3] = n[3] * scale * g.w;
            }
            sv.x = fmaf(a.keep, sv.x, n[0] * a.add);
            sv.y = fmaf(a.keep, sv.y, n[1] * a.add);
            sv.z = fmaf(a.keep, sv.z, n[2] * a.add);
            sv.w = fmaf(a.keep, sv.w, n[3] * a.add);
            st[h2] = sv;
        }
    }
}

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t stream)
{
    if (a.H % 8 != 0 || a.top_k > 32) return cudaErrorInvalidValue;
    const int nvec = a.H / 8;
    const int one = (nvec + 31) / 32 * 32;
    if (one <= kCombOneVecThreads) {
        if (a.y32) return launch_pdl(combine_kernel<true, 1>, dim3(a.T), dim3(one), 0, stream, a);
        return launch_pdl(combine_kernel<false, 1>, dim3(a.T), dim3(one), 0, stream, a);
    }
    const int two = ((nvec + 1) / 2 + 31) / 32 * 32;
    if (two > kCombTwoVecThreads) return cudaErrorInvalidValue;
    if (a.y32) return launch_pdl(combine_kernel<true, 2>, dim3(a.T), dim3(two), 0, stream, a);
    return launch_pdl(combine_kernel<false, 2>, dim3(a.T), dim3(two), 0, stream, a);
}

__global__ void wait_timeout_check_kernel(WaitCtl ctl)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_barrier_init();
        mbar_wait(smem_u32(&bar), 0, ctl);
    }
}

cudaError_t launch_wait_timeout_check(WaitCtl ctl, cudaStream_t stream)
{
    wait_timeout_check_kernel<<<1, 32, 0, stream>>>(ctl);
    return cudaGetLastError();
}

}  // namespace beam
