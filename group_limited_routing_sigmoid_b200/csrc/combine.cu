// Combine of the Beam MoE block, with the optional post-norm and
// depth-scaled residual update fused in.
//
//   o[t]   = routed_scaling * sum_j w[t,j] * y[row(t,j)]     (bf16 y, fp32 sum, slot order)
//            (dense layer: o[t] = sum_s y_s[t] over FP32 split-K slices, in slice order)
//   out[t] = bf16_rn(o[t])
//   n[t]   = o[t] / sqrt(mean(o[t]^2) + eps) * gamma          (if gamma)
//   stream[t] <- sqrt((k-1)/k) * stream[t] + n[t] / sqrt(k)
// Launch blog "Introducing Beam": section "Mixture of Experts" (normalised
// router weights, x2.5) and section "Residual Stream" (weights sqrt((k-1)/k)
// and 1/sqrt(k); every sub-layer normalised before and after; norms in FP32).
#include "kernels.cuh"

namespace beam {

namespace {
constexpr int kCombThreads = 256;
constexpr int kMaxVec = 8;   // float4 per thread: H <= 8 * 4 * 256 = 8192
}  // namespace

__global__ void __launch_bounds__(kCombThreads) combine_kernel(CombineArgs a)
{
    pdl_launch_dependents();
    pdl_wait();
    const int t = blockIdx.x;
    const int tid = threadIdx.x;
    const int nvec = a.H / 4;
    int rows[32];
    float wts[32];
    const int nsum = a.y_f32 ? 0 : a.top_k;   // expert slots (none for FP32 slices)
    for (int j = 0; j < nsum; ++j) {
        rows[j] = a.pair_row[(size_t)t * a.top_k + j];
        wts[j] = a.w[(size_t)t * a.top_k + j];
    }
    float4 o[kMaxVec];
    float ss = 0.f;
#pragma unroll
    for (int v = 0; v < kMaxVec; ++v) {
        const int i = tid + v * kCombThreads;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < nvec) {
            if (a.y_f32) {
                for (int sl = 0; sl < a.nslice; ++sl) {
                    const float4 y = reinterpret_cast<const float4 *>(
                        a.y_f32 + (size_t)sl * (size_t)a.slice_stride + (size_t)t * a.H)[i];
                    acc.x += y.x;
                    acc.y += y.y;
                    acc.z += y.z;
                    acc.w += y.w;
                }
            }
            for (int j = 0; j < nsum; ++j) {
                const uint2 raw = reinterpret_cast<const uint2 *>(a.y + (size_t)rows[j] * a.H)[i];
                const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
                const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
                const float4 y = make_float4(lo.x, lo.y, hi.x, hi.y);
                acc.x = fmaf(wts[j], y.x, acc.x);
                acc.y = fmaf(wts[j], y.y, acc.y);
                acc.z = fmaf(wts[j], y.z, acc.z);
                acc.w = fmaf(wts[j], y.w, acc.w);
            }
            acc.x *= a.scaling;
            acc.y *= a.scaling;
            acc.z *= a.scaling;
            acc.w *= a.scaling;
            if (a.out) {
                __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
                __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
                uint2 packed;
                packed.x = *reinterpret_cast<uint32_t *>(&lo);
                packed.y = *reinterpret_cast<uint32_t *>(&hi);
                reinterpret_cast<uint2 *>(a.out + (size_t)t * a.H)[i] = packed;
            }
            ss += acc.x * acc.x + acc.y * acc.y + acc.z * acc.z + acc.w * acc.w;
        }
        o[v] = acc;
    }
    if (!a.residual) return;

    float scale = 1.0f;
    if (a.gamma) {
        __shared__ float red[kCombThreads / 32];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
        if ((tid & 31) == 0) red[tid >> 5] = ss;
        __syncthreads();
        float tot = 0.f;
#pragma unroll
        for (int wv = 0; wv < kCombThreads / 32; ++wv) tot += red[wv];
        scale = 1.0f / sqrtf(tot / (float)a.H + a.eps);
    }
    float *st = a.residual + (size_t)t * a.H;
#pragma unroll
    for (int v = 0; v < kMaxVec; ++v) {
        const int i = tid + v * kCombThreads;
        if (i >= nvec) continue;
        float4 s = reinterpret_cast<float4 *>(st)[i];
        float4 n = o[v];
        if (a.gamma) {
            const float4 g = reinterpret_cast<const float4 *>(a.gamma)[i];
            n.x = n.x * scale * g.x;
            n.y = n.y * scale * g.y;
            n.z = n.z * scale * g.z;
            n.w = n.w * scale * g.w;
        }
        s.x = fmaf(a.keep, s.x, n.x * a.add);
        s.y = fmaf(a.keep, s.y, n.y * a.add);
        s.z = fmaf(a.keep, s.z, n.z * a.add);
        s.w = fmaf(a.keep, s.w, n.w * a.add);
        reinterpret_cast<float4 *>(st)[i] = s;
    }
}

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t stream)
{
    if (a.H % 4 != 0 || a.H > kMaxVec * 4 * kCombThreads || a.top_k > 32)
        return cudaErrorInvalidValue;
    return launch_pdl(combine_kernel, dim3(a.T), dim3(kCombThreads), 0, stream, a);
}

// ---------------------------------------------------------------------------
// Failure-detection self-check: one thread waits on a barrier that nothing
// completes.  The bounded wait must give up, record the timeout in the status
// word and let the kernel return.
// ---------------------------------------------------------------------------
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
