// Checked mode of the Beam MoE block: device-side validation that stands in
// for a memory checker (which this pool does not offer).  The kernels never
// trap: a failed check records kStatusCheck in the handle's status word (and
// the first failing index), and every later kernel of the forward pass sees
// the word and skips its work, so no kernel indexes memory with a bad
// expert or row.  beam_moe_get_status reports it.
#include "kernels.cuh"

namespace beam {

namespace {
__device__ __forceinline__ void fail_at(int *status, int *where, int index)
{
    atomicCAS(status, 0, kStatusCheck);
    atomicMin(where, index);
}
}  // namespace

// Warp per token: every chosen expert in [0, E), no expert twice, every
// weight finite and positive (the weights are normalised sigmoid scores).
__global__ void __launch_bounds__(256) check_routing_kernel(const int32_t *__restrict__ idx,
                                                            const float *__restrict__ w, int T,
                                                            int E, int top_k, int *status,
                                                            int *where)
{
    pdl_launch_dependents();
    pdl_wait();
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (t >= T) return;
    const bool mine = lane < top_k;
    const int e = mine ? idx[(size_t)t * top_k + lane] : -1 - lane;   // distinct fillers
    const float wv = mine ? w[(size_t)t * top_k + lane] : 1.0f;
    bool bad = mine && (e < 0 || e >= E || !(wv > 0.f) || !(wv <= 1.0f));
    const unsigned same = __match_any_sync(0xffffffffu, e);
    bad = bad || (mine && __popc(same) != 1);
    if (__any_sync(0xffffffffu, bad) && lane == 0) fail_at(status, where, t);
}

// Thread per (token, slot) pair: its row lies in its expert's row range and
// the two row maps are inverse.  Thread 0 also checks the tables: offsets
// start at 0, grow by the counts and end at P; each expert's token-tile
// count is ceil(count / tile_rows).
__global__ void __launch_bounds__(256) check_dispatch_kernel(
    const int32_t *__restrict__ idx, const int32_t *__restrict__ counts,
    const int32_t *__restrict__ offsets, const int32_t *__restrict__ tile_off,
    const int32_t *__restrict__ pair_row, const int32_t *__restrict__ row_pair, int P, int E,
    int tile_rows, int *status, int *where)
{
    pdl_launch_dependents();
    pdl_wait();
    if (*(volatile const int *)status != 0) return;   // routing already failed its check
    const int p = blockIdx.x * blockDim.x + threadIdx.x;
    if (p == 0) {
        bool ok = offsets[0] == 0 && tile_off[0] == 0 && offsets[E] == P;
        for (int e = 0; e < E && ok; ++e) {
            const int c = counts[e];
            ok = c >= 0 && offsets[e + 1] == offsets[e] + c &&
                 tile_off[e + 1] - tile_off[e] == (c + tile_rows - 1) / tile_rows;
        }
        if (!ok) fail_at(status, where, P);   // index P: the tables themselves
    }
    if (p >= P) return;
    const int e = idx[p];
    const int row = pair_row[p];
    const bool ok = row >= offsets[e] && row < offsets[e] + counts[e] && row_pair[row] == p;
    if (!ok) fail_at(status, where, p);
}

__global__ void corrupt_routing_kernel(int32_t *idx, int E)
{
    pdl_launch_dependents();
    pdl_wait();
    idx[0] = E;
}

cudaError_t launch_check_routing(const int32_t *idx, const float *w, int T, int E, int top_k,
                                 int *status, int *where, cudaStream_t stream)
{
    return launch_pdl(check_routing_kernel, dim3((T + 7) / 8), dim3(256), 0, stream, idx, w, T, E,
                      top_k, status, where);
}

cudaError_t launch_check_dispatch(const int32_t *idx, const int32_t *counts,
                                  const int32_t *offsets, const int32_t *tile_off,
                                  const int32_t *pair_row, const int32_t *row_pair, int P, int E,
                                  int tile_rows, int *status, int *where, cudaStream_t stream)
{
    return launch_pdl(check_dispatch_kernel, dim3((P + 255) / 256), dim3(256), 0, stream, idx,
                      counts, offsets, tile_off, pair_row, row_pair, P, E, tile_rows, status,
                      where);
}

cudaError_t launch_corrupt_routing(int32_t *idx, int E, cudaStream_t stream)
{
    return launch_pdl(corrupt_routing_kernel, dim3(1), dim3(1), 0, stream, idx, E);
}

}  // namespace beam
