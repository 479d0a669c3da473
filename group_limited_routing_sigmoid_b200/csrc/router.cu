// Router of the Beam MoE block: FP32 logits, sigmoid scores, per-expert bias
// for selection, group-limited top-k, normalised weights.
//
// Method: launch blog "Introducing Beam", section "Mixture of Experts" (score
// every expert with a sigmoid, 8 groups of 32, a group's score is the sum of
// its two best scores, keep 4 groups, top-8 experts inside them, normalised
// router weights); transformers page "Beam", "Overview", "Sparse MoE" bullet
// (learned per-expert bias instead of an auxiliary loss, n_group /
// topk_group) and the paragraph fixing the router in FP32 with FP32 router
// weights and bias.
#include "kernels.cuh"

namespace beam {

// ---------------------------------------------------------------------------
// Logits: partial[s][t][e] = sum over the s-th K slice of x[t,h] * W[e,h].
// 128 tokens x 64 experts per block, 256 threads, 8 x 4 outputs per thread.
// K goes through shared memory 32 at a time; the next 32 are loaded into
// registers while the current ones are used.  Each thread folds its running
// FP32 sums into a second accumulator every 256 K, so no FP32 chain is
// longer than 256 terms.
// ---------------------------------------------------------------------------
namespace {
constexpr int kLT = 128;  // tokens per block
constexpr int kLE = 64;   // experts per block
constexpr int kLK = 32;   // K per shared-memory stage
}  // namespace

__global__ void __launch_bounds__(256) router_logits_kernel(const __nv_bfloat16 *__restrict__ x,
                                                            const float *__restrict__ w, int T,
                                                            int H, int E, int kslice,
                                                            float *__restrict__ partial)
{
    __shared__ __align__(16) float xs[kLK][kLT + 4];
    __shared__ __align__(16) float ws[kLK][kLE + 4];
    const int tid = threadIdx.x;
    const int t0 = blockIdx.x * kLT;
    const int e0 = blockIdx.y * kLE;
    const int kbeg = blockIdx.z * kslice;
    const int kend = min(H, kbeg + kslice);
    const int tx = tid & 15;   // 4 experts: e0 + 4*tx ..
    const int ty = tid >> 4;   // 8 tokens:  t0 + 8*ty ..

    float acc[8][4], tot[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = tot[i][j] = 0.f;

    // loaders: x -- 128 tokens x 32 K bf16 = 4096 values: 16 per thread
    //          (token tid/2, K half (tid&1)*16);
    //          W -- 64 experts x 32 K fp32 = 2048 values: 8 per thread
    //          (expert tid/4, K quarter (tid&3)*8).
    const int xr = tid >> 1, xk = (tid & 1) * 16;
    const int wr = tid >> 2, wk = (tid & 3) * 8;
    const bool xvalid = t0 + xr < T;
    const bool wvalid = e0 + wr < E;
    const __nv_bfloat16 *xp = x + (size_t)(t0 + xr) * H + xk;
    const float *wp = w + (size_t)(e0 + wr) * H + wk;
    uint4 xa = make_uint4(0, 0, 0, 0), xb = make_uint4(0, 0, 0, 0);
    float4 wa = make_float4(0.f, 0.f, 0.f, 0.f), wb = make_float4(0.f, 0.f, 0.f, 0.f);
    auto fetch = [&](int k0) {
        if (xvalid) {
            const uint4 *src = reinterpret_cast<const uint4 *>(xp + k0);
            xa = src[0];
            xb = src[1];
        }
        if (wvalid) {
            const float4 *src = reinterpret_cast<const float4 *>(wp + k0);
            wa = src[0];
            wb = src[1];
        }
    };
    auto stash = [&]() {
        const __nv_bfloat162 *p2 = reinterpret_cast<const __nv_bfloat162 *>(&xa);
        const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&xb);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(p2[i]);
            const float2 g = __bfloat1622float2(q2[i]);
            xs[xk + 2 * i][xr] = f.x;
            xs[xk + 2 * i + 1][xr] = f.y;
            xs[xk + 8 + 2 * i][xr] = g.x;
            xs[xk + 8 + 2 * i + 1][xr] = g.y;
        }
        ws[wk + 0][wr] = wa.x;
        ws[wk + 1][wr] = wa.y;
        ws[wk + 2][wr] = wa.z;
        ws[wk + 3][wr] = wa.w;
        ws[wk + 4][wr] = wb.x;
        ws[wk + 5][wr] = wb.y;
        ws[wk + 6][wr] = wb.z;
        ws[wk + 7][wr] = wb.w;
    };

    int folded = 0;
    if (kbeg < kend) fetch(kbeg);
    for (int k0 = kbeg; k0 < kend; k0 += kLK) {
        stash();
        __syncthreads();
        if (k0 + kLK < kend) fetch(k0 + kLK);   // in flight while the tile below is used
#pragma unroll 8
        for (int kk = 0; kk < kLK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4 *>(&xs[kk][ty * 8]);
            const float4 a1 = *reinterpret_cast<const float4 *>(&xs[kk][ty * 8 + 4]);
            const float4 b = *reinterpret_cast<const float4 *>(&ws[kk][tx * 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
        folded += kLK;
        if (folded == 256) {
            folded = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    tot[i][j] += acc[i][j];
                    acc[i][j] = 0.f;
                }
        }
    }
    float *dst = partial + (size_t)blockIdx.z * T * E;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int t = t0 + ty * 8 + i;
        if (t >= T) continue;
        const int e = e0 + tx * 4;
        if (e + 3 < E) {
            *reinterpret_cast<float4 *>(dst + (size_t)t * E + e) =
                make_float4(tot[i][0] + acc[i][0], tot[i][1] + acc[i][1], tot[i][2] + acc[i][2],
                            tot[i][3] + acc[i][3]);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (e + j < E) dst[(size_t)t * E + e + j] = tot[i][j] + acc[i][j];
        }
    }
}

// ---------------------------------------------------------------------------
// Selection: one warp per token; lane l owns experts l*EPL .. l*EPL+EPL-1,
// so a group of g experts spans g/EPL consecutive lanes.
// ---------------------------------------------------------------------------
template <int EPL>
__global__ void __launch_bounds__(256) router_select_kernel(
    const float *__restrict__ partial, int nslice, int T, int E, int n_group, int topk_group,
    int top_k, const float *__restrict__ bias, int32_t *__restrict__ idx_out,
    float *__restrict__ w_out, float *__restrict__ logits_out)
{
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    const int lpg = (E / n_group) / EPL;   // lanes per group (power of two)
    const int my_group = lane / lpg;
    const int e_base = lane * EPL;

    float s[EPL], b[EPL];
#pragma unroll
    for (int m = 0; m < EPL; ++m) {
        const int e = e_base + m;
        float l = 0.f;
        for (int q = 0; q < nslice; ++q) l += partial[((size_t)q * T + t) * E + e];
        if (logits_out) logits_out[(size_t)t * E + e] = l;
        s[m] = 1.0f / (1.0f + expf(-l));
        b[m] = s[m] + bias[e];
    }

    // group score: sum of the group's two largest biased scores
    float t1 = -INFINITY, t2 = -INFINITY;
#pragma unroll
    for (int m = 0; m < EPL; ++m) {
        if (b[m] > t1) {
            t2 = t1;
            t1 = b[m];
        } else if (b[m] > t2) {
            t2 = b[m];
        }
    }
    for (int off = 1; off < lpg; off <<= 1) {
        const float o1 = __shfl_xor_sync(0xffffffffu, t1, off);
        const float o2 = __shfl_xor_sync(0xffffffffu, t2, off);
        const float hi = fmaxf(t1, o1);
        const float lo = fmaxf(fminf(t1, o1), fmaxf(t2, o2));
        t1 = hi;
        t2 = lo;
    }
    const float gs = t1 + t2;

    // keep the topk_group best groups (ties to the lower group index)
    int rank = 0;
    for (int j = 0; j < n_group; ++j) {
        const float v = __shfl_sync(0xffffffffu, gs, j * lpg);
        rank += (v > gs || (v == gs && j < my_group)) ? 1 : 0;
    }
    const bool kept = rank < topk_group;

    float cand[EPL];
#pragma unroll
    for (int m = 0; m < EPL; ++m) cand[m] = kept ? b[m] : -INFINITY;
    uint32_t taken = 0;
    int my_idx = 0;
    float my_s = 0.f, ssum = 0.f;
    for (int r = 0; r < top_k; ++r) {
        float bv = -INFINITY, bs = 0.f;
        int bi = 0x7fffffff;
#pragma unroll
        for (int m = 0; m < EPL; ++m) {
            if (taken & (1u << m)) continue;
            const int e = e_base + m;
            if (cand[m] > bv || (cand[m] == bv && e < bi)) {
                bv = cand[m];
                bi = e;
                bs = s[m];
            }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            const float os = __shfl_xor_sync(0xffffffffu, bs, off);
            if (ov > bv || (ov == bv && oi < bi)) {
                bv = ov;
                bi = oi;
                bs = os;
            }
        }
        if (bi / EPL == lane) taken |= 1u << (bi - e_base);
        if (lane == r) {
            my_idx = bi;
            my_s = bs;
        }
        ssum += bs;
    }
    if (lane < top_k) {
        idx_out[(size_t)t * top_k + lane] = my_idx;
        w_out[(size_t)t * top_k + lane] = my_s / ssum;
    }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------

// K slices of the logits: enough blocks for several per SM (the selection
// sums the slices in a fixed order).  Slices stay a multiple of 32 wide and
// at least 1024 wide, or 256 when the grid would not fill the GPU anyway.
int router_slices(int T, int H, int E, int num_sms)
{
    const int base = ((T + kLT - 1) / kLT) * ((E + kLE - 1) / kLE);
    const int min_width = base < num_sms ? 256 : 1024;
    int ns = 1;
    while (ns * base < 6 * num_sms && (H / (ns * 2)) >= min_width && H % (ns * 2 * kLK) == 0)
        ns *= 2;
    return ns;
}

cudaError_t launch_router(const RouterArgs &a, cudaStream_t stream)
{
    const int ns = a.nslice;
    const int kslice = a.H / ns;
    dim3 grid((a.T + kLT - 1) / kLT, (a.E + kLE - 1) / kLE, ns);
    router_logits_kernel<<<grid, 256, 0, stream>>>(a.x, a.router_w, a.T, a.H, a.E, kslice,
                                                   a.partial);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const int warps = 8;
    dim3 sgrid((a.T + warps - 1) / warps);
    const int epl = a.E / 32;
#define BEAM_SELECT(EPLV)                                                                        \
    case EPLV:                                                                                   \
        router_select_kernel<EPLV><<<sgrid, warps * 32, 0, stream>>>(                            \
            a.partial, ns, a.T, a.E, a.n_group, a.topk_group, a.top_k, a.bias, a.idx, a.w,       \
            a.logits_out);                                                                       \
        break;
    switch (epl) {
        BEAM_SELECT(1)
        BEAM_SELECT(2)
        BEAM_SELECT(4)
        BEAM_SELECT(8)
        BEAM_SELECT(16)
        BEAM_SELECT(32)
        default:
            return cudaErrorInvalidValue;
    }
#undef BEAM_SELECT
    return cudaGetLastError();
}

}  // namespace beam
