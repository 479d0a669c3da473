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
    pdl_launch_dependents();
    pdl_wait();
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
// Logits for small batches (T <= 64, decode): a block per (16 experts, K
// slice of width ks), all tokens.  The block stages its slice of the router
// matrix (16 rows of ks floats) with cp.async and its slice of x (T rows of
// ks bf16, converted once to FP32; rows T..63 zero) in shared memory, so the
// slice costs one memory round trip.  Each of the 16 warps then sums the K
// range [w*ks/16, (w+1)*ks/16) for all 64 x 16 outputs: lane l holds tokens
// (l & 7) + 8i and experts (l >> 3) + 4j.  The products go through packed
// FP32 FMAs (fma.rn.f32x2), each output keeping two running sums, of its
// even and of its odd K terms, added at the end.  The sixteen warps' sums are
// added in warp order into partial[slice][t][e]; the selection adds the
// slices in slice order.  The padded rows put the 8 rows one 128-bit load
// instruction reads per quarter-warp in distinct banks.
// ---------------------------------------------------------------------------
constexpr int kSmallT = 64;        // tokens per block (the largest T of this path)
constexpr int kSmallE = 16;        // experts per block
constexpr int kSmallMaxK = 640;    // widest K slice (shared memory)
constexpr int kSmallWarps = 16;
constexpr int kSmallThreads = 32 * kSmallWarps;

__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// d = a * b + c on two FP32 lanes at once (element 0 in the low word).
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ float pair_sum(uint64_t v)
{
    return __uint_as_float((uint32_t)v) + __uint_as_float((uint32_t)(v >> 32));
}

__global__ void __launch_bounds__(kSmallThreads, 1) router_logits_small_kernel(
    const __nv_bfloat16 *__restrict__ x, const float *__restrict__ w, int T, int H, int E, int ks,
    float *__restrict__ partial)
{
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ __align__(16) uint8_t small_smem[];
    const int stride = ks + 4;   // floats per staged row (16 bytes of padding)
    float *xs = reinterpret_cast<float *>(small_smem);                 // [64][stride]
    float *ws = xs + (size_t)kSmallT * stride;                         // [16][stride]
    const int e0 = blockIdx.x * kSmallE;
    const int k0 = blockIdx.y * ks;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // router rows: one per warp, asynchronous
    {
        const float *src = w + (size_t)(e0 + warp) * H + k0;
        float *dst = ws + (size_t)warp * stride;
        for (int q = lane; q < ks / 4; q += 32) cp_async16(dst + 4 * q, src + 4 * q);
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    // token rows: four per warp (rows warp + 16 r), every load of the four in
    // flight before any is converted; rows T..63 are zero
    {
        constexpr int kRows = kSmallT / kSmallWarps;          // 4
        constexpr int kPer = (kSmallMaxK / 8 + 31) / 32;      // 16-byte vectors per lane and row, at most
        uint4 raw[kRows][kPer];
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            const int t = warp + kSmallWarps * r;
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int q = lane + 32 * u;
                raw[r][u] = make_uint4(0, 0, 0, 0);
                if (t < T && q < ks / 8)
                    raw[r][u] = *reinterpret_cast<const uint4 *>(x + (size_t)t * H + k0 + 8 * q);
            }
        }
#pragma unroll
        for (int r = 0; r < kRows; ++r) {
            float *dst = xs + (size_t)(warp + kSmallWarps * r) * stride;
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int q = lane + 32 * u;
                if (q < ks / 8) {
                    const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&raw[r][u]);
                    const float2 f0 = __bfloat1622float2(h2[0]), f1 = __bfloat1622float2(h2[1]);
                    const float2 f2 = __bfloat1622float2(h2[2]), f3 = __bfloat1622float2(h2[3]);
                    reinterpret_cast<float4 *>(dst + 8 * q)[0] = make_float4(f0.x, f0.y, f1.x, f1.y);
                    reinterpret_cast<float4 *>(dst + 8 * q)[1] = make_float4(f2.x, f2.y, f3.x, f3.y);
                }
            }
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();

    const int tg = lane & 7, eg = lane >> 3;
    const int kw = ks / kSmallWarps;   // a multiple of 4
    uint64_t acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0ull;
#pragma unroll 1
    for (int k = warp * kw; k < (warp + 1) * kw; k += 4) {
        ulonglong2 wv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
            wv[j] = *reinterpret_cast<const ulonglong2 *>(ws + (size_t)(eg + 4 * j) * stride + k);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const ulonglong2 xv = *reinterpret_cast<const ulonglong2 *>(xs + (size_t)(tg + 8 * i) * stride + k);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                acc[i][j] = fma_f32x2(xv.x, wv[j].x, acc[i][j]);
                acc[i][j] = fma_f32x2(xv.y, wv[j].y, acc[i][j]);
            }
        }
    }
    __syncthreads();   // every warp is done with the staged rows
    float *red = reinterpret_cast<float *>(small_smem);   // [16 warps][64 tokens][16 experts]
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
            red[((size_t)warp * kSmallT + tg + 8 * i) * kSmallE + eg + 4 * j] = pair_sum(acc[i][j]);
    __syncthreads();
    const int t = threadIdx.x >> 2, ec = (threadIdx.x & 3) * 4;
    if (t < T) {
        float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int wv2 = 0; wv2 < kSmallWarps; ++wv2) {
            const float4 v = *reinterpret_cast<const float4 *>(red + ((size_t)wv2 * kSmallT + t) * kSmallE + ec);
            sum.x += v.x;
            sum.y += v.y;
            sum.z += v.z;
            sum.w += v.w;
        }
        *reinterpret_cast<float4 *>(partial + ((size_t)blockIdx.y * T + t) * E + e0 + ec) = sum;
    }
}

// ---------------------------------------------------------------------------
// Selection: one warp per token; lane l owns experts l*EPL .. l*EPL+EPL-1,
// so a group of g experts spans g/EPL consecutive lanes.  Grid-stride over
// the tokens.  Optional extras (SelectExtra):
//   margin > 0: tokens whose decision margin -- the smallest gap between
//     neighbours in the ranking of the top k+1 candidates of the kept groups
//     (it decides the chosen set and its order), or the weakest kept group's
//     score minus the strongest dropped one's -- is below `margin` are
//     appended to fix_list (their logits are recomputed on CUDA cores);
//   token_list: select only the listed tokens, whose logits are the compact
//     rows 0..*list_count-1 of `partial` (one slice).
// ---------------------------------------------------------------------------
// Candidate keys for the top-k: the biased score's bits made order-preserving
// as an unsigned integer in the high word, ~expert in the low word, so that
// the larger key is the larger score and, between equal scores, the lower
// expert index (the ranking's tie rule).
__device__ __forceinline__ uint64_t rank_key(float v, int e)
{
    uint32_t u = __float_as_uint(v);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((uint64_t)u << 32) | (uint32_t)~(uint32_t)e;
}

__device__ __forceinline__ float key_value(uint64_t k)
{
    uint32_t u = (uint32_t)(k >> 32);
    u = (u & 0x80000000u) ? (u & 0x7fffffffu) : ~u;
    return __uint_as_float(u);
}

__device__ __forceinline__ int key_expert(uint64_t k) { return (int)~(uint32_t)k; }

// Larger key to a, smaller to b.
__device__ __forceinline__ void key_cas(uint64_t &a, uint64_t &b)
{
    const uint64_t hi = a > b ? a : b, lo = a > b ? b : a;
    a = hi;
    b = lo;
}

// Sorts 8 keys in descending order (Batcher's odd-even merge sort network).
__device__ __forceinline__ void sort8_desc(uint64_t (&k)[8])
{
    key_cas(k[0], k[1]); key_cas(k[2], k[3]); key_cas(k[4], k[5]); key_cas(k[6], k[7]);
    key_cas(k[0], k[2]); key_cas(k[1], k[3]); key_cas(k[4], k[6]); key_cas(k[5], k[7]);
    key_cas(k[1], k[2]); key_cas(k[5], k[6]);
    key_cas(k[0], k[4]); key_cas(k[1], k[5]); key_cas(k[2], k[6]); key_cas(k[3], k[7]);
    key_cas(k[2], k[4]); key_cas(k[3], k[5]);
    key_cas(k[1], k[2]); key_cas(k[3], k[4]); key_cas(k[5], k[6]);
}

// Top-8 selection for 8 experts per lane and top_k <= 8: each lane sorts its
// 8 candidate keys, then five butterfly steps (partners lane ^ 1 .. lane ^
// 16) each keep the 8 largest keys of the two lanes' sorted lists: the
// elementwise maximum of one list and the other reversed holds them as a
// bitonic sequence, which three compare-exchange steps sort.  Every lane
// ends with the same ranked top 8: the ranking the one-at-a-time warp argmax
// produces, with the same tie rule.  The chosen experts' unbiased scores are
// fetched from their owner lanes, summed in rank order and normalised; the
// margin check (ex.margin > 0) takes the gaps between neighbours in the
// ranking of the top k + 1 candidates and the group gap, as in the general
// path.
__device__ __forceinline__ void select_top8(const float (&cand)[8], const float (&s)[8], int e_base,
                                            int lane, int t, int T, int top_k, bool kept, float gs,
                                            int32_t *__restrict__ idx_out, float *__restrict__ w_out,
                                            const SelectExtra &ex)
{
    uint64_t k[8], loc[8];
#pragma unroll
    for (int m = 0; m < 8; ++m) k[m] = rank_key(cand[m], e_base + m);
    sort8_desc(k);
#pragma unroll
    for (int m = 0; m < 8; ++m) loc[m] = k[m];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        uint64_t o[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) o[m] = __shfl_xor_sync(0xffffffffu, k[m], off);
#pragma unroll
        for (int m = 0; m < 8; ++m) k[m] = k[m] > o[7 - m] ? k[m] : o[7 - m];
        key_cas(k[0], k[4]); key_cas(k[1], k[5]); key_cas(k[2], k[6]); key_cas(k[3], k[7]);
        key_cas(k[0], k[2]); key_cas(k[1], k[3]); key_cas(k[4], k[6]); key_cas(k[5], k[7]);
        key_cas(k[0], k[1]); key_cas(k[2], k[3]); key_cas(k[4], k[5]); key_cas(k[6], k[7]);
    }
    // lane j < top_k takes the j-th ranked expert and its unbiased score
    uint64_t mine = k[0];
#pragma unroll
    for (int m = 1; m < 8; ++m)
        if (lane == m) mine = k[m];
    const int my_idx = key_expert(mine);
    const int owner = (my_idx >> 3) & 31, slot = my_idx & 7;
    float my_s = 0.f;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const float v = __shfl_sync(0xffffffffu, s[m], owner);
        if (slot == m) my_s = v;
    }
    float ssum = 0.f;
    for (int j = 0; j < top_k; ++j) ssum += __shfl_sync(0xffffffffu, my_s, j);
    if (lane < top_k) {
        idx_out[(size_t)t * top_k + lane] = my_idx;
        w_out[(size_t)t * top_k + lane] = my_s / ssum;
    }
    if (ex.margin > 0.f) {
        // the (k+1)-th candidate: the 9th key when top_k is 8 (each lane's
        // best key outside the top 8, then the warp's best of those)
        uint64_t next = 0;
        if (top_k < 8) {
            next = __shfl_sync(0xffffffffu, mine, top_k);   // lane j holds the j-th ranked key
        } else {
            uint64_t c = 0;
#pragma unroll
            for (int m = 7; m >= 0; --m)
                if (loc[m] < k[7]) c = loc[m];
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                const uint64_t o = __shfl_xor_sync(0xffffffffu, c, off);
                c = o > c ? o : c;
            }
            next = c;
        }
        float min_gap = INFINITY, prev = key_value(k[0]);
#pragma unroll
        for (int m = 1; m < 8; ++m) {
            if (m < top_k) {
                const float v = key_value(k[m]);
                min_gap = fminf(min_gap, prev - v);
                prev = v;
            }
        }
        min_gap = fminf(min_gap, prev - key_value(next));
        float kmin = kept ? gs : INFINITY, dmax = kept ? -INFINITY : gs;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            kmin = fminf(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
            dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, off));
        }
        const float gap_group = kmin - dmax;
        if (lane == 0 && !(fminf(gap_group, min_gap) >= ex.margin)) {
            const int slot2 = atomicAdd(ex.fix_count, 1);
            if (slot2 < T) ex.fix_list[slot2] = t;
        }
    }
}

template <int EPL>
__global__ void __launch_bounds__(256) router_select_kernel(
    const float *__restrict__ partial, int nslice, int T, int E, int n_group, int topk_group,
    int top_k, const float *__restrict__ bias, int32_t *__restrict__ idx_out,
    float *__restrict__ w_out, float *__restrict__ logits_out, SelectExtra ex)
{
    pdl_launch_dependents();
    pdl_wait();
    const int lane = threadIdx.x & 31;
    const int lpg = (E / n_group) / EPL;   // lanes per group (power of two)
    const int my_group = lane / lpg;
    const int e_base = lane * EPL;
    const int limit = ex.token_list ? min(*ex.list_count, T) : T;
    const int stride = gridDim.x * (blockDim.x >> 5);
    float bias_r[EPL];   // the lane's experts' bias, the same for every token
#pragma unroll
    for (int m = 0; m < EPL; ++m) bias_r[m] = bias[e_base + m];
    for (int wi = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); wi < limit; wi += stride) {
        const int t = ex.token_list ? ex.token_list[wi] : wi;   // output row
        const int r = wi;                                         // logits row

        // the lane's logits: slices summed in order; the loads of one slice
        // are independent of each other (vectors when EPL allows)
        float l[EPL];
#pragma unroll
        for (int m = 0; m < EPL; ++m) l[m] = 0.f;
#pragma unroll 8
        for (int q = 0; q < nslice; ++q) {
            const float *src = partial + ((size_t)q * T + r) * E + e_base;
            if constexpr (EPL % 4 == 0) {
#pragma unroll
                for (int m = 0; m < EPL; m += 4) {
                    const float4 v = *reinterpret_cast<const float4 *>(src + m);
                    l[m] += v.x;
                    l[m + 1] += v.y;
                    l[m + 2] += v.z;
                    l[m + 3] += v.w;
                }
            } else {
#pragma unroll
                for (int m = 0; m < EPL; ++m) l[m] += src[m];
            }
        }
        float s[EPL], b[EPL];
#pragma unroll
        for (int m = 0; m < EPL; ++m) {
            const int e = e_base + m;
            if (logits_out) logits_out[(size_t)t * E + e] = l[m];
            s[m] = __frcp_rn(1.0f + expf(-l[m]));   // the correctly rounded 1 / (1 + e^-l)
            b[m] = s[m] + bias_r[m];
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
        if constexpr (EPL == 8) {
            if (top_k <= 8) {
                select_top8(cand, s, e_base, lane, t, T, top_k, kept, gs, idx_out, w_out, ex);
                continue;
            }
        }
        uint32_t taken = 0;
        int my_idx = 0;
        float my_s = 0.f, ssum = 0.f, prev = INFINITY, min_gap = INFINITY;
        const int rounds = ex.margin > 0.f ? top_k + 1 : top_k;   // one more for the margin
        for (int rr = 0; rr < rounds; ++rr) {
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
            // adjacent gap in the ranking: decides both the order of the
            // chosen experts and (at rr == top_k) which of them are chosen
            if (rr > 0) min_gap = fminf(min_gap, prev - bv);
            if (rr == top_k) break;   // the (k+1)-th candidate only feeds the margin
            if (bi / EPL == lane) taken |= 1u << (bi - e_base);
            if (lane == rr) {
                my_idx = bi;
                my_s = bs;
            }
            ssum += bs;
            prev = bv;
        }
        if (lane < top_k) {
            idx_out[(size_t)t * top_k + lane] = my_idx;
            w_out[(size_t)t * top_k + lane] = my_s / ssum;
        }
        if (ex.margin > 0.f) {
            // weakest kept group vs strongest dropped group
            float kmin = kept ? gs : INFINITY, dmax = kept ? -INFINITY : gs;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                kmin = fminf(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
                dmax = fmaxf(dmax, __shfl_xor_sync(0xffffffffu, dmax, off));
            }
            const float gap_group = kmin - dmax;      // +inf when every group is kept
            if (lane == 0 && !(fminf(gap_group, min_gap) >= ex.margin)) {
                const int slot = atomicAdd(ex.fix_count, 1);
                if (slot < T) ex.fix_list[slot] = t;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Exact-path logits for listed tokens: FP32 dot products on CUDA cores.
// A work unit is (8 listed tokens, 16 experts): the tokens' rows are staged
// in shared memory as bf16, each warp takes one expert, the lanes split K
// (lane l reads the 16-byte chunks l, l+32, ... of the weight row, so every
// load is 512 contiguous bytes), and the 8 per-lane sums (chains of at most
// 256 terms, folded) are combined by a shuffle tree: logits[slot][e] for
// list slots 0..*count-1.
// ---------------------------------------------------------------------------
constexpr int kFixTokens = 8;
constexpr int kFixExperts = 16;  // one per warp
constexpr int kFixThreads = 32 * kFixExperts;
constexpr int kFixLoads = 8;     // weight vectors in flight per lane

__global__ void __launch_bounds__(kFixThreads) router_fix_kernel(const __nv_bfloat16 *__restrict__ x,
                                                         const float *__restrict__ w, int H, int E,
                                                         int T, const int *__restrict__ list,
                                                         const int *__restrict__ count,
                                                         float *__restrict__ logits)
{
    pdl_launch_dependents();
    pdl_wait();
    extern __shared__ __align__(16) __nv_bfloat16 xs[];   // [kFixTokens][H]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n = min(*count, T);
    const int nchunk = (E + kFixExperts - 1) / kFixExperts;
    const int units = ((n + kFixTokens - 1) / kFixTokens) * nchunk;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int b0 = (u / nchunk) * kFixTokens, c = u % nchunk;
        const int nb = min(kFixTokens, n - b0);
        __syncthreads();
        for (int i = threadIdx.x; i < kFixTokens * H / 8; i += blockDim.x) {
            const int j = i / (H / 8), q = i - j * (H / 8);
            uint4 v = make_uint4(0, 0, 0, 0);
            if (j < nb) v = reinterpret_cast<const uint4 *>(x + (size_t)list[b0 + j] * H)[q];
            reinterpret_cast<uint4 *>(xs + (size_t)j * H)[q] = v;
        }
        __syncthreads();
        {
            const int e = c * kFixExperts + warp;
            if (e >= E) continue;
            const float4 *wr = reinterpret_cast<const float4 *>(w + (size_t)e * H);
            float acc[kFixTokens], tot[kFixTokens];
#pragma unroll
            for (int j = 0; j < kFixTokens; ++j) acc[j] = tot[j] = 0.f;
            int terms = 0;
            // kFixLoads weight vectors in flight per lane; the sums take them
            // in the same order (q = lane, lane + 32, ...) and fold at the
            // same points as a one-at-a-time loop would
            for (int q0 = lane; q0 < H / 4; q0 += 32 * kFixLoads) {
                float4 wv[kFixLoads];
#pragma unroll
                for (int u = 0; u < kFixLoads; ++u) {
                    const int q = q0 + 32 * u;
                    wv[u] = q < H / 4 ? wr[q] : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int u = 0; u < kFixLoads; ++u) {
                    const int q = q0 + 32 * u;
                    if (q >= H / 4) break;
#pragma unroll
                    for (int j = 0; j < kFixTokens; ++j) {
                        const __nv_bfloat162 *p2 =
                            reinterpret_cast<const __nv_bfloat162 *>(xs + (size_t)j * H + 4 * q);
                        const float2 a = __bfloat1622float2(p2[0]);
                        const float2 b = __bfloat1622float2(p2[1]);
                        acc[j] = fmaf(wv[u].x, a.x, acc[j]);
                        acc[j] = fmaf(wv[u].y, a.y, acc[j]);
                        acc[j] = fmaf(wv[u].z, b.x, acc[j]);
                        acc[j] = fmaf(wv[u].w, b.y, acc[j]);
                    }
                    terms += 4;
                    if (terms == 256) {
                        terms = 0;
#pragma unroll
                        for (int j = 0; j < kFixTokens; ++j) {
                            tot[j] += acc[j];
                            acc[j] = 0.f;
                        }
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < kFixTokens; ++j) {
                float v = tot[j] + acc[j];
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0 && j < nb) logits[(size_t)(b0 + j) * E + e] = v;
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Host launchers
// ---------------------------------------------------------------------------

// K slices of the logits: enough blocks for several per SM (the selection
// sums the slices in a fixed order).  Slices stay a multiple of 32 wide and
// at least 1024 wide, or 128 when the grid would not fill the GPU anyway.
int router_slices(int T, int H, int E, int num_sms)
{
    const int base = ((T + kLT - 1) / kLT) * ((E + kLE - 1) / kLE);
    const int min_width = base < num_sms ? 128 : 1024;
    int ns = 1;
    while (ns * base < 6 * num_sms && (H / (ns * 2)) >= min_width && H % (ns * 2 * kLK) == 0)
        ns *= 2;
    return ns;
}

// Small-batch path: the K slice count (each slice a multiple of 64 wide and
// at most kSmallMaxK) with the shortest estimated kernel: the busiest SM's
// blocks, each costing its slice width plus a fixed 128 for the staging
// round trip and the warps' reduction.  A block's work does not depend on T
// (its lanes cover 64 token rows), and two blocks sharing an SM share its
// issue slots, so 160 blocks on 148 SMs take about twice as long as 128.
// Ties go to fewer slices (less for the selection to add).  0 when the path
// does not apply (T > 64, or H or E off its grid).
int router_small_slices(int T, int H, int E, int num_sms)
{
    if (T < 1 || T > kSmallT || E % kSmallE != 0 || H % 64 != 0 || num_sms < 1) return 0;
    int best = 0;
    long long best_cost = 0;
    for (int ns = 1; ns <= H / 64; ++ns) {
        if (H % (ns * 64) != 0 || H / ns > kSmallMaxK) continue;
        const long long per_sm = ((long long)(E / kSmallE) * ns + num_sms - 1) / num_sms;
        const long long cost = per_sm * (H / ns + 128);
        if (best == 0 || cost < best_cost) {
            best = ns;
            best_cost = cost;
        }
    }
    return best;
}

// Staged rows, or the warps' sums that reuse them, whichever is larger.
static size_t small_smem_bytes(int ks)
{
    const size_t staged = (size_t)(kSmallT + kSmallE) * (ks + 4) * 4;
    const size_t red = (size_t)kSmallWarps * kSmallT * kSmallE * 4;
    return staged > red ? staged : red;
}

cudaError_t prepare_router_small()
{
    return cudaFuncSetAttribute(router_logits_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)small_smem_bytes(kSmallMaxK));
}

cudaError_t launch_router(const RouterArgs &a, cudaStream_t stream)
{
    const int ns = a.nslice;
    const int kslice = a.H / ns;
    cudaError_t err;
    if (a.small) {
        if (a.T > kSmallT || a.E % kSmallE != 0 || kslice % 64 != 0 || kslice > kSmallMaxK ||
            kslice * ns != a.H)
            return cudaErrorInvalidValue;
        const size_t smem = small_smem_bytes(kslice);
        err = launch_pdl(router_logits_small_kernel, dim3(a.E / kSmallE, ns), dim3(kSmallThreads), smem, stream,
                         a.x, a.router_w, a.T, a.H, a.E, kslice, a.partial);
    } else {
        dim3 grid((a.T + kLT - 1) / kLT, (a.E + kLE - 1) / kLE, ns);
        err = launch_pdl(router_logits_kernel, grid, dim3(256), 0, stream, a.x, a.router_w, a.T, a.H,
                         a.E, kslice, a.partial);
    }
    if (err != cudaSuccess) return err;
    // the selection is a chain of dependent steps per token: few warps per
    // block spread the tokens' warps over more SMs and scheduler slots
    const int warps = a.small ? 2 : 8;
    dim3 sgrid((a.T + warps - 1) / warps);
    const int epl = a.E / 32;
#define BEAM_SELECT(EPLV)                                                                        \
    case EPLV:                                                                                   \
        err = launch_pdl(router_select_kernel<EPLV>, sgrid, dim3(warps * 32), 0, stream,         \
                         a.partial, ns, a.T, a.E, a.n_group, a.topk_group, a.top_k, a.bias, a.idx, \
                         a.w, a.logits_out, SelectExtra{});                                      \
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
    return err;
}

}  // namespace beam

namespace beam {

// ---------------------------------------------------------------------------
// Tensor-core logits for large T.  The FP32 router weight is split once into
// three bf16 pieces, W = w0 + w1 + w2 (each the nearest bf16 to what the
// previous pieces leave; the remainder is below 2^-27 |W|), stored side by
// side as Wcat [E, 3H].  A product of a bf16 token value and a bf16 piece is
// exact in FP32, so x . W = sum over k < 3H of Wcat[e,k] * x[t, k mod H] is
// an FP32 sum of exact products: the tensor core accumulates it in TMEM.
// Work items: (128-expert tile, BN-token tile, K slice of H); the MMA has
// the experts as M (A = Wcat rows) and the tokens as N (B = x rows), and
// writes partial[slice][t][e] like the SIMT kernel, so the selection is
// shared.  A pipeline stage holds one 64-wide K step of the token tile and
// the same K step of all three pieces, so each token tile crosses into
// shared memory once for the three pieces (the pieces' twelve MMAs per
// stage go into one accumulator).
// ---------------------------------------------------------------------------

__global__ void router_split_kernel(const float *__restrict__ w, int n, __nv_bfloat16 *__restrict__ wcat,
                                    int H)
{
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const int e = i / H, h = i - e * H;
    const float v = w[i];
    const __nv_bfloat16 p0 = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(p0);        // exact in FP32
    const __nv_bfloat16 p1 = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(p1);       // exact in FP32
    const __nv_bfloat16 p2 = __float2bfloat16_rn(r2);
    __nv_bfloat16 *row = wcat + (size_t)e * 3 * H;
    row[h] = p0;
    row[H + h] = p1;
    row[2 * H + h] = p2;
}

cudaError_t launch_router_split(const float *w, int E, int H, __nv_bfloat16 *wcat, cudaStream_t s)
{
    const int n = E * H;
    router_split_kernel<<<(n + 255) / 256, 256, 0, s>>>(w, n, wcat, H);
    return cudaGetLastError();
}

namespace {
constexpr int kRBM = 128;   // experts per tile (UMMA M)
constexpr int kRBN = 128;   // tokens per tile (UMMA N)
constexpr int kRBK = 64;
constexpr int kRPieces = 3;
constexpr int kRTileA = kRBM * kRBK * 2;                 // one piece's weight tile
constexpr int kRStageBytes = kRPieces * kRTileA + kRBN * kRBK * 2;
constexpr int kRStages = 3;
constexpr int kRAccCols = kRBN;
constexpr int kRSmem = 1024 + kRStages * kRStageBytes + 256;
}  // namespace

__global__ void __launch_bounds__(192, 1)
    router_mma_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                      RouterMmaArgs p)
{
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *bar_ptr = smem_raw + (base - raw_addr) + kRStages * kRStageBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(bar_ptr);
    uint64_t *empty = full + kRStages;
    uint64_t *tfull = empty + kRStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < kRStages; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 128);
        }
        mbar_init(smem_u32(drain), 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        __syncwarp();
        tmem_alloc(smem_u32(tmem_slot), 2 * kRAccCols);
        tmem_relinquish();
    }
    pdl_launch_dependents();
    pdl_wait();   // set-up above overlaps the previous kernel; data from here on
    if (p.fix_count && blockIdx.x == 0 && threadIdx.x == 0) *p.fix_count = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int n_mt = (p.E + kRBM - 1) / kRBM;
    const int n_tt = (p.T + kRBN - 1) / kRBN;
    const int total = n_mt * n_tt * p.nslice;
    // item = ((tt * nslice) + s) * n_mt + mt: neighbours share the token tile

    if (warp == 0 && lane == 0) {
        const uint64_t pol = l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0;
        long long issued = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            const int mt = item % n_mt, rest = item / n_mt;
            const int s = rest % p.nslice, tt = rest / p.nslice;
            for (int j = 0; j < p.kb_per_slice; ++j) {
                const int kb = s * p.kb_per_slice + j;   // over H
                if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, p.ctl)) {
                    ok = false;
                    break;
                }
                const uint32_t sa = base + stage * kRStageBytes;
                const uint32_t fb = smem_u32(&full[stage]);
                mbar_arrive_expect_tx(fb, kRStageBytes);
#pragma unroll
                for (int pc = 0; pc < kRPieces; ++pc)
                    tma_load_2d(sa + pc * kRTileA, &tmW, (pc * p.kb_per_h + kb) * kRBK, mt * kRBM, fb, pol);
                tma_load_2d(sa + kRPieces * kRTileA, &tmX, kb * kRBK, tt * kRBN, fb, pol);
                ++issued;
                if (++stage == kRStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok) {
            long long n = issued < kRStages ? issued : kRStages;
            int st = stage;
            uint32_t ph = phase;
            for (long long j = 0; j < n; ++j) {
                if (st == 0) {
                    st = kRStages - 1;
                    ph ^= 1u;
                } else {
                    --st;
                }
                mbar_wait_drain(smem_u32(&full[st]), ph, p.ctl.limit_ns);
            }
        }
    } else if (warp == 1 && lane == 0) {
        constexpr uint32_t idesc = umma_idesc_bf16_f32(kRBM, kRBN);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true, issued_any = false;
        int iter = 0;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++iter) {
            const int acc = iter & 1;
            const uint32_t acc_phase = (uint32_t)(iter >> 1) & 1u;
            if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, p.ctl)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem_base + (uint32_t)(acc * kRAccCols);
            for (int j = 0; j < p.kb_per_slice; ++j) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, p.ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = base + stage * kRStageBytes;
                const uint32_t sb = sa + kRPieces * kRTileA;
#pragma unroll
                for (int pc = 0; pc < kRPieces; ++pc)
#pragma unroll
                    for (int k = 0; k < kRBK / 16; ++k) {
                        umma_bf16(d, umma_desc_sw128(sa + pc * kRTileA + k * 32), umma_desc_sw128(sb + k * 32),
                                  idesc, (j > 0 || pc > 0 || k > 0) ? 1u : 0u);
                        issued_any = true;
                    }
                umma_commit(smem_u32(&empty[stage]));
                if (++stage == kRStages) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            umma_commit(smem_u32(&tfull[acc]));
        }
        if (issued_any) {
            umma_commit(smem_u32(drain));
            mbar_wait_drain(smem_u32(drain), 0, p.ctl.limit_ns);
        }
    } else if (warp >= 2) {
        const int quad = warp & 3;
        int iter = 0;
        for (int item = blockIdx.x; item < total; item += gridDim.x, ++iter) {
            const int acc = iter & 1;
            const uint32_t acc_phase = (uint32_t)(iter >> 1) & 1u;
            const bool ok = mbar_wait(smem_u32(&tfull[acc]), acc_phase, p.ctl);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int mt = item % n_mt, rest = item / n_mt;
            const int s = rest % p.nslice, tt = rest / p.nslice;
            const int e = mt * kRBM + quad * 32 + lane;
            const int t0 = tt * kRBN;
            float *dst = p.partial + (size_t)s * p.T * p.E;
            const uint32_t taddr =
                tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * kRAccCols);
#pragma unroll 1
            for (int c0 = 0; c0 < kRBN && t0 + c0 < p.T; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(taddr + c0, v);
                tmem_ld_wait();
                if (e < p.E) {
#pragma unroll
                    for (int n = 0; n < 32; ++n)
                        if (t0 + c0 + n < p.T) dst[(size_t)(t0 + c0 + n) * p.E + e] = __uint_as_float(v[n]);
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty[acc]));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, 2 * kRAccCols);
    }
}

cudaError_t prepare_router_mma()
{
    return cudaFuncSetAttribute(router_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kRSmem);
}

cudaError_t launch_router_mma(const CUtensorMap &tmW, const CUtensorMap &tmX, const RouterMmaArgs &a,
                              int grid, cudaStream_t stream)
{
    cudaError_t e = launch_pdl(router_mma_kernel, dim3(grid), dim3(192), kRSmem, stream, tmW, tmX, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

int router_mma_tokens_per_tile() { return kRBN; }
int router_mma_experts_per_tile() { return kRBM; }

cudaError_t launch_router_select(const RouterArgs &a, const SelectExtra &ex, int max_blocks,
                                 cudaStream_t stream)
{
    const int warps = 8;
    int blocks = (a.T + warps - 1) / warps;
    if (max_blocks > 0 && blocks > max_blocks) blocks = max_blocks;
    const int epl = a.E / 32;
    cudaError_t err = cudaSuccess;
#define BEAM_SELECT2(EPLV)                                                                       \
    case EPLV:                                                                                   \
        err = launch_pdl(router_select_kernel<EPLV>, dim3(blocks), dim3(warps * 32), 0, stream,  \
                         a.partial, a.nslice, a.T, a.E, a.n_group, a.topk_group, a.top_k, a.bias, \
                         a.idx, a.w, a.logits_out, ex);                                          \
        break;
    switch (epl) {
        BEAM_SELECT2(1)
        BEAM_SELECT2(2)
        BEAM_SELECT2(4)
        BEAM_SELECT2(8)
        BEAM_SELECT2(16)
        BEAM_SELECT2(32)
        default:
            return cudaErrorInvalidValue;
    }
#undef BEAM_SELECT2
    return err;
}

cudaError_t prepare_router_fix(int H)
{
    return cudaFuncSetAttribute(router_fix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(kFixTokens * (size_t)H * 2));
}

cudaError_t launch_router_fix(const __nv_bfloat16 *x, const float *w, int H, int E, int T,
                              const int *list, const int *count, float *logits, int grid,
                              cudaStream_t stream)
{
    cudaError_t e = launch_pdl(router_fix_kernel, dim3(grid), dim3(kFixThreads),
                               kFixTokens * (size_t)H * 2, stream, x, w, H, E, T, list, count, logits);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace beam
