// Sparse dispatch of the Beam MoE block: a stable counting sort of the
// (token, slot) pairs by expert, and the gather of each pair's token into an
// expert-sorted activation buffer.  Only the routed experts run (launch blog
// "Introducing Beam", section "Mixture of Experts": 8 of 256 experts per
// token); how pairs reach their experts is not described on the pages, so
// this is a plain counting sort: histogram, exclusive prefix sum, scatter.
#include "kernels.cuh"

namespace beam {

// Per block of 1024 pairs: each warp counts its pairs per expert with
// match.any, the block turns the per-warp counts into per-warp prefixes, and
// every pair gets its rank among the block's pairs of the same expert
// (ordered by pair index).
__global__ void __launch_bounds__(kDispatchBlock) dispatch_count_kernel(
    const int *status, const int32_t *__restrict__ idx, int P, int E, int32_t *__restrict__ block_cnt,
    int32_t *__restrict__ rank)
{
    pdl_launch_dependents();
    pdl_wait();
    if (status_is_set(status)) return;   // a check failed earlier in this pass
    extern __shared__ int32_t wcnt[];   // [32 warps][E]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < 32 * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const int p = blockIdx.x * kDispatchBlock + tid;
    const int e = p < P ? idx[p] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rk = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && rk == 0) wcnt[warp * E + e] = __popc(peers);
    __syncthreads();
    for (int ee = tid; ee < E; ee += blockDim.x) {
        int run = 0;
        for (int w = 0; w < 32; ++w) {
            const int c = wcnt[w * E + ee];
            wcnt[w * E + ee] = run;
            run += c;
        }
        block_cnt[(size_t)blockIdx.x * E + ee] = run;
    }
    __syncthreads();
    if (e >= 0) rank[p] = wcnt[warp * E + e] + rk;
}

// One block, thread e = expert: per-block bases, expert counts, exclusive
// offsets and the prefix of token tiles of BN rows.
__global__ void __launch_bounds__(1024) dispatch_scan_kernel(
    const int *status, const int32_t *__restrict__ block_cnt, int nblk, int E, int BN,
    int32_t *__restrict__ block_base, int32_t *__restrict__ counts,
    int32_t *__restrict__ offsets, int32_t *__restrict__ tile_off)
{
    pdl_launch_dependents();
    pdl_wait();
    if (status_is_set(status)) return;   // a check failed earlier in this pass
    __shared__ int32_t wsum_c[32], wsum_t[32];
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    int run = 0;
    if (e < E) {
        for (int b = 0; b < nblk; ++b) {
            const int c = block_cnt[(size_t)b * E + e];
            block_base[(size_t)b * E + e] = run;
            run += c;
        }
        counts[e] = run;
    }
    const int nt = (run + BN - 1) / BN;
    int ic = run, it = nt;   // inclusive warp scans
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int vc = __shfl_up_sync(0xffffffffu, ic, off);
        const int vt = __shfl_up_sync(0xffffffffu, it, off);
        if (lane >= off) {
            ic += vc;
            it += vt;
        }
    }
    if (lane == 31) {
        wsum_c[warp] = ic;
        wsum_t[warp] = it;
    }
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int vc = lane < nw ? wsum_c[lane] : 0;
        int vt = lane < nw ? wsum_t[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int uc = __shfl_up_sync(0xffffffffu, vc, off);
            const int ut = __shfl_up_sync(0xffffffffu, vt, off);
            if (lane >= off) {
                vc += uc;
                vt += ut;
            }
        }
        if (lane < nw) {
            wsum_c[lane] = vc;   // inclusive over warps
            wsum_t[lane] = vt;
        }
    }
    __syncthreads();
    const int bc = warp > 0 ? wsum_c[warp - 1] : 0;
    const int bt = warp > 0 ? wsum_t[warp - 1] : 0;
    if (e < E) {
        offsets[e] = bc + ic - run;
        tile_off[e] = bt + it - nt;
        if (e == E - 1) {
            offsets[E] = bc + ic;
            tile_off[E] = bt + it;
        }
    }
}

// One warp per pair: its row in the sorted buffer, the maps both ways, and
// the copy of the token's hidden vector (16-byte vectors).  With to_f16 the
// copy holds f16 values of x x 2^-8, the operand type of the NVFP4 GEMMs
// (the MMA takes A and B of one type); a value beyond the f16 range sets
// BEAM_ERR_RANGE in the status word.
__global__ void __launch_bounds__(256) dispatch_permute_kernel(
    const int *status, const int32_t *__restrict__ idx, const int32_t *__restrict__ rank,
    const int32_t *__restrict__ block_base, const int32_t *__restrict__ offsets,
    const __nv_bfloat16 *__restrict__ x, int P, int H, int E, int top_k,
    int32_t *__restrict__ pair_row, int32_t *__restrict__ row_pair, __nv_bfloat16 *__restrict__ xp,
    int to_f16)
{
    pdl_launch_dependents();
    pdl_wait();
    if (status_is_set(status)) return;   // a check failed earlier in this pass
    const int p = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (p >= P) return;
    const int lane = threadIdx.x & 31;
    const int e = idx[p];
    const int row = offsets[e] + block_base[(size_t)(p / kDispatchBlock) * E + e] + rank[p];
    if (lane == 0) {
        pair_row[p] = row;
        row_pair[row] = p;
    }
    const int t = p / top_k;
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)t * H);
    uint4 *dst = reinterpret_cast<uint4 *>(xp + (size_t)row * H);
    if (!to_f16) {
        for (int i = lane; i < H / 8; i += 32) dst[i] = src[i];
        return;
    }
    bool fits = true;
    for (int i = lane; i < H / 8; i += 32) {
        const uint4 v = src[i];
        uint4 o;
        const uint32_t *vw = &v.x;
        uint32_t *ow = &o.x;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float lo = __uint_as_float(vw[q] << 16) * 0.00390625f;
            const float hi = __uint_as_float(vw[q] & 0xffff0000u) * 0.00390625f;
            asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(ow[q]) : "f"(hi), "f"(lo));
            if (fabsf(lo) > 65504.0f || fabsf(hi) > 65504.0f) fits = false;
        }
        dst[i] = o;
    }
    if (!fits) record_status(const_cast<int *>(status), kStatusRange);
}

// The maps only, a thread per pair: used when the gate|up GEMM gathers its
// token rows from x, so no sorted copy of x is made.
__global__ void __launch_bounds__(256) dispatch_rows_kernel(
    const int *status, const int32_t *__restrict__ idx, const int32_t *__restrict__ rank,
    const int32_t *__restrict__ block_base, const int32_t *__restrict__ offsets, int P, int E,
    int32_t *__restrict__ pair_row, int32_t *__restrict__ row_pair)
{
    pdl_launch_dependents();
    pdl_wait();
    if (status_is_set(status)) return;   // a check failed earlier in this pass
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= P) return;
    const int e = idx[p];
    const int row = offsets[e] + block_base[(size_t)(p / kDispatchBlock) * E + e] + rank[p];
    pair_row[p] = row;
    row_pair[row] = p;
}

// All of the above in one block, for at most kDispatchBlock pairs when no
// sorted copy is made (the decode path): the count kernel's ranks, the scan
// kernel's counts, offsets and tile prefix, and the row maps.  Thread p
// takes pair p; threads e < E also take expert e in the scans.
__global__ void __launch_bounds__(kDispatchBlock) dispatch_small_kernel(
    const int *status, const int32_t *__restrict__ idx, int P, int E, int BN,
    int32_t *__restrict__ counts, int32_t *__restrict__ offsets, int32_t *__restrict__ tile_off,
    int32_t *__restrict__ pair_row, int32_t *__restrict__ row_pair)
{
    pdl_launch_dependents();
    pdl_wait();
    if (status_is_set(status)) return;   // a check failed earlier in this pass
    extern __shared__ int32_t wcnt[];   // [32 warps][E], then the experts' offsets [E]
    int32_t *off_s = wcnt + 32 * E;
    __shared__ int32_t wsum_c[32], wsum_t[32];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < 32 * E; i += blockDim.x) wcnt[i] = 0;
    __syncthreads();
    const int e = tid < P ? idx[tid] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rk = __popc(peers & ((1u << lane) - 1u));
    if (e >= 0 && rk == 0) wcnt[warp * E + e] = __popc(peers);
    __syncthreads();
    int run = 0;   // thread tid < E: expert tid's pairs before each warp, and in all
    if (tid < E) {
        for (int w = 0; w < 32; ++w) {
            const int c = wcnt[w * E + tid];
            wcnt[w * E + tid] = run;
            run += c;
        }
    }
    const int nt = (run + BN - 1) / BN;
    int ic = run, it = nt;   // inclusive warp scans over the experts
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int vc = __shfl_up_sync(0xffffffffu, ic, off);
        const int vt = __shfl_up_sync(0xffffffffu, it, off);
        if (lane >= off) {
            ic += vc;
            it += vt;
        }
    }
    if (lane == 31) {
        wsum_c[warp] = ic;
        wsum_t[warp] = it;
    }
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        int vc = lane < nw ? wsum_c[lane] : 0;
        int vt = lane < nw ? wsum_t[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int uc = __shfl_up_sync(0xffffffffu, vc, off);
            const int ut = __shfl_up_sync(0xffffffffu, vt, off);
            if (lane >= off) {
                vc += uc;
                vt += ut;
            }
        }
        if (lane < nw) {
            wsum_c[lane] = vc;
            wsum_t[lane] = vt;
        }
    }
    __syncthreads();
    if (tid < E) {
        const int bc = warp > 0 ? wsum_c[warp - 1] : 0;
        const int bt = warp > 0 ? wsum_t[warp - 1] : 0;
        const int o = bc + ic - run;
        counts[tid] = run;
        offsets[tid] = o;
        off_s[tid] = o;
        tile_off[tid] = bt + it - nt;
        if (tid == E - 1) {
            offsets[E] = bc + ic;
            tile_off[E] = bt + it;
        }
    }
    __syncthreads();
    if (e >= 0) {
        const int row = off_s[e] + wcnt[warp * E + e] + rk;
        pair_row[tid] = row;
        row_pair[row] = tid;
    }
}

cudaError_t prepare_dispatch(int E)
{
    cudaError_t err = cudaFuncSetAttribute(dispatch_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)(sizeof(int32_t) * 32 * (size_t)E));
    if (err != cudaSuccess) return err;
    return cudaFuncSetAttribute(dispatch_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)(sizeof(int32_t) * 33 * (size_t)E));
}

cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t stream)
{
    const int P = a.T * a.top_k;
    const int nblk = (P + kDispatchBlock - 1) / kDispatchBlock;
    const size_t smem = sizeof(int32_t) * 32 * (size_t)a.E;
    if (nblk <= 1 && !a.copy_rows && a.E <= kDispatchBlock)
        return launch_pdl(dispatch_small_kernel, dim3(1), dim3(kDispatchBlock), smem + sizeof(int32_t) * a.E,
                          stream, a.status, a.idx, P, a.E, a.tile_rows, a.counts, a.offsets, a.tile_off,
                          a.pair_row, a.row_pair);
    cudaError_t err = launch_pdl(dispatch_count_kernel, dim3(nblk), dim3(kDispatchBlock), smem,
                                 stream, a.status, a.idx, P, a.E, a.block_cnt, a.rank);
    if (err != cudaSuccess) return err;
    const int threads = ((a.E + 31) / 32) * 32;
    err = launch_pdl(dispatch_scan_kernel, dim3(1), dim3(threads), 0, stream, a.status, a.block_cnt, nblk,
                     a.E, a.tile_rows, a.block_base, a.counts, a.offsets, a.tile_off);
    if (err != cudaSuccess) return err;
    if (a.copy_rows)
        return launch_pdl(dispatch_permute_kernel, dim3((P + 7) / 8), dim3(256), 0, stream, a.status, a.idx,
                          a.rank, a.block_base, a.offsets, a.x, P, a.H, a.E, a.top_k, a.pair_row,
                          a.row_pair, a.xp, a.xp_f16);
    return launch_pdl(dispatch_rows_kernel, dim3((P + 255) / 256), dim3(256), 0, stream, a.status, a.idx,
                      a.rank, a.block_base, a.offsets, P, a.E, a.pair_row, a.row_pair);
}

}  // namespace beam
