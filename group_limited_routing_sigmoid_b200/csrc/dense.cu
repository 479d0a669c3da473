// The dense SwiGLU MLP of Beam's first three layers (launch blog
// "Introducing Beam", section "Mixture of Experts": the first 3 layers use a
// dense SwiGLU MLP; section "Residual Stream": SwiGLU product in FP32, norms
// in FP32, depth-scaled residual).  It runs on the same grouped GEMMs as the
// experts, as one expert that every token takes with weight 1 and no
// routed scaling.  This file holds its set-up kernel:
//   dense_setup_kernel   the GEMMs' tables for one expert of T rows, the
//                        identity row map / unit weights the combine reads,
//                        and zeroed stream-K arrival counters.
// The stream-K GEMMs for decode-sized batches are in dense_sk.cu.
#include "gemm_common.cuh"

namespace beam {

__global__ void __launch_bounds__(256) dense_setup_kernel(int T, int tiles, int32_t *counts,
                                                          int32_t *offsets, int32_t *tile_off,
                                                          int32_t *pair_row, int32_t *row_pair,
                                                          float *w, int *cnt, int ncnt)
{
    pdl_launch_dependents();
    pdl_wait();
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    const int stride = gridDim.x * blockDim.x;
    if (cnt)
        for (int i = t; i < ncnt; i += stride) cnt[i] = 0;
    if (t == 0) {
        counts[0] = T;
        offsets[0] = 0;
        offsets[1] = T;
        tile_off[0] = 0;
        tile_off[1] = tiles;
    }
    for (int i = t; i < T; i += stride) {
        pair_row[i] = i;
        row_pair[i] = i;
        w[i] = 1.0f;
    }
}

cudaError_t launch_dense_setup(int T, int tiles, int32_t *counts, int32_t *offsets,
                               int32_t *tile_off, int32_t *pair_row, int32_t *row_pair, float *w,
                               int *cnt, int ncnt, cudaStream_t stream)
{
    const int nc = cnt ? ncnt : 0;
    const int n = T > nc ? T : nc;
    const int blocks = (n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024;
    return launch_pdl(dense_setup_kernel, dim3(blocks > 0 ? blocks : 1), dim3(256), 0, stream, T,
                      tiles, counts, offsets, tile_off, pair_row, row_pair, w, cnt, ncnt);
}

}  // namespace beam
