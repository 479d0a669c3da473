// Launch interfaces of the Beam MoE kernels (host side).
#pragma once

#include "common.cuh"

namespace beam {

// ----------------------------------------------------------------- launch
// Launch `kernel` on `stream` as a programmatic dependent of the previous
// kernel there (it may start while that one finishes; it waits for it with
// pdl_wait before touching its results).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// ----------------------------------------------------------------- router
struct RouterArgs {
    const __nv_bfloat16 *x;   // [T, H]
    const float *router_w;    // [E, H]
    const float *bias;        // [E]
    int T, H, E, n_group, topk_group, top_k;
    int nslice;               // K slices of the logits (router_slices or router_small_slices)
    int small = 0;            // 1: the small-batch logits kernel (T <= 64)
    float *partial;           // [nslice, T, E] workspace
    int32_t *idx;             // [T, top_k]
    float *w;                 // [T, top_k]
    float *logits_out;        // [T, E] or nullptr
};
int router_slices(int T, int H, int E, int num_sms);
int router_small_slices(int T, int H, int E, int num_sms);   // 0: the small path does not apply
cudaError_t prepare_router_small();
cudaError_t launch_router(const RouterArgs &a, cudaStream_t stream);          // SIMT logits + selection

// Selection extras: a decision-margin check that lists tokens for the exact
// path, or selection of listed tokens only (logits in compact rows).
struct SelectExtra {
    float margin = 0.f;
    int *fix_list = nullptr;
    int *fix_count = nullptr;
    const int *token_list = nullptr;
    const int *list_count = nullptr;
};
cudaError_t launch_router_select(const RouterArgs &a, const SelectExtra &ex, int max_blocks,
                                 cudaStream_t stream);
cudaError_t prepare_router_fix(int H);
// FP32 CUDA-core logits of the listed tokens into compact rows of `logits`.
cudaError_t launch_router_fix(const __nv_bfloat16 *x, const float *w, int H, int E, int T,
                              const int *list, const int *count, float *logits, int grid,
                              cudaStream_t stream);

// Tensor-core logits: W split into bf16 pieces (Wcat [E, 3H]) x tokens.
struct RouterMmaArgs {
    int T, E;
    int nslice;          // K slices of H
    int kb_per_slice;    // 64-wide K steps per slice
    int kb_per_h;        // H / 64 (piece p's K step kb is Wcat column block p * kb_per_h + kb)
    float *partial;      // [nslice, T, E]
    int *fix_count;      // zeroed by the kernel (the re-derivation list's length), or nullptr
    WaitCtl ctl;
};
cudaError_t launch_router_split(const float *w, int E, int H, __nv_bfloat16 *wcat, cudaStream_t s);
cudaError_t prepare_router_mma();
cudaError_t launch_router_mma(const CUtensorMap &tmW, const CUtensorMap &tmX,
                              const RouterMmaArgs &a, int grid, cudaStream_t stream);
int router_mma_tokens_per_tile();
int router_mma_experts_per_tile();

// --------------------------------------------------------------- dispatch
constexpr int kDispatchBlock = 1024;   // pairs per counting block

struct DispatchArgs {
    const int *status;           // the handle's status word: no work while it is set
    const int32_t *idx;          // [P] expert of pair p = t*top_k + j
    const __nv_bfloat16 *x;      // [T, H]
    int T, H, E, top_k;
    int tile_rows;               // token rows per GEMM tile (BN)
    int32_t *block_cnt;          // [nblk, E]
    int32_t *block_base;         // [nblk, E]
    int32_t *rank;               // [P] rank of the pair among its block's pairs of that expert
    int32_t *counts;             // [E]
    int32_t *offsets;            // [E+1]
    int32_t *tile_off;           // [E+1] prefix of ceil(counts/BN)
    int32_t *pair_row;           // [P]
    int32_t *row_pair;           // [P]
    __nv_bfloat16 *xp;           // [P, H] expert-sorted activations
    int copy_rows;               // 0: maps only (the gate|up GEMM gathers from x)
    int xp_f16 = 0;              // 1: sorted rows as f16 x 2^-8 (NVFP4 GEMM operands)
};
cudaError_t launch_dispatch(const DispatchArgs &a, cudaStream_t stream);
cudaError_t prepare_dispatch(int E);   // shared-memory limit of the counting kernel

// ----------------------------------------------------------- grouped GEMM
struct GemmArgs {
    int K;                       // reduction length
    int R;                       // weight rows per expert (= output row stride)
    int E;
    const int32_t *counts;       // [E]
    const int32_t *offsets;      // [E+1]
    const int32_t *tile_off;     // [E+1]
    __nv_bfloat16 *out;          // bf16 [P, R]: h (gate|up) or y (down)
    // gate|up only: when `gather` is set, token rows come straight from x
    // (BoxMaps::gather), row r of the sorted order being token row_pair[r] / top_k
    const int32_t *row_pair;     // [P]
    int top_k;
    int gather;
    // FP32 outputs (kDownF32, kDownY32, kDownPairedY32): [P, R] instead of out
    float *out_f32;
    // CTA-pair kernel: depth of the token-row ring (0 = default); the weight
    // ring's depth is derived at launch (a_stages)
    int b_stages;
    int a_stages;
    WaitCtl ctl;
};

// Tensor maps of one activation buffer with boxes of 8, 16, 32, 64, 128 and
// 256 rows (64 columns each): a token tile is loaded as a sum of these; or,
// for the gate|up GEMM with gathering on, four token rows at a time from x.
struct BoxMaps {
    CUtensorMap m[6];
    CUtensorMap gather;          // x [T, H] with a 64-column, one-row box (tile::gather4)
};

enum class GemmKind {
    kGateUp,       // gate and up tiles, SwiGLU epilogue, bf16 out
    kDown,         // one 128-row tile, bf16 out
    kDownPaired,   // two consecutive 128-row tiles sharing the token tile, bf16 out
    kDownF32,      // one 128-row tile, FP32 expert outputs y ([P][R]) in out_f32
    kGateUpI,      // CTA-pair kernel: one interleaved tile (64 gate + 64 up rows per CTA,
                   // 16-row box maps), SwiGLU epilogue, bf16 out; one accumulator of N columns
    kDownY32,      // CTA-pair kernel: one 256-row block, FP32 expert outputs y ([P][R])
    kDownPairedY32 // CTA-pair kernel: two 256-row blocks sharing the token tile, FP32 y
};
// BN: largest token tile (16..256, power of two).
cudaError_t launch_grouped_gemm(GemmKind kind, int BN, const CUtensorMap &a0,
                                const CUtensorMap &a1, const BoxMaps &b, const GemmArgs &args,
                                int grid, cudaStream_t stream);
cudaError_t prepare_grouped_gemm(int E);   // sets shared-memory limits once per device
bool gemm_tile_supported(int BN);

// CTA-pair version (cta_group::2, clusters of two CTAs) for token tiles of
// 64..256 rows: the pair shares each MMA, each CTA holding half the token
// tile.  `grid` must be even.
cudaError_t launch_grouped_gemm_pair(GemmKind kind, int BN, const CUtensorMap &a0,
                                     const CUtensorMap &a1, const BoxMaps &b,
                                     const GemmArgs &args, int grid, cudaStream_t stream);
cudaError_t prepare_grouped_gemm_pair();
bool gemm_pair_supported(int BN);
int gemm_pair_max_ctas();   // CTAs of the pair kernels that can be resident at once (even)

// ---------------------------------------------------------------- combine
struct CombineArgs {
    const int *status;           // the handle's status word: no work while it is set
    const __nv_bfloat16 *y;      // [P, H] expert outputs (bf16), or
    const float *y32;            // [P, H] expert outputs (FP32); exactly one of y, y32 is set
                                 // for a sparse block
    const int32_t *pair_row;     // [P]
    const float *w;              // [T, top_k]
    int T, H, top_k;
    float scaling;
    __nv_bfloat16 *out;          // [T, H] or nullptr
    float *residual;             // [T, H] or nullptr
    const float *gamma;          // [H] or nullptr
    float eps;
    float keep, add;             // sqrt((k-1)/k), 1/sqrt(k)
};
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t stream);

// ------------------------------------------------------------- checked mode
// Validation of the routing and of the dispatch tables (see checks.cu); a
// failure records kStatusCheck and the first failing index in *where.
cudaError_t launch_check_routing(const int32_t *idx, const float *w, int T, int E, int top_k,
                                 int *status, int *where, cudaStream_t stream);
cudaError_t launch_check_dispatch(const int32_t *idx, const int32_t *counts,
                                  const int32_t *offsets, const int32_t *tile_off,
                                  const int32_t *pair_row, const int32_t *row_pair, int P, int E,
                                  int tile_rows, int *status, int *where, cudaStream_t stream);
// Test hook: write an out-of-range expert into slot 0 of the routing.
cudaError_t launch_corrupt_routing(int32_t *idx, int E, cudaStream_t stream);

// ------------------------------------------------------------- dense layer
cudaError_t launch_dense_setup(int T, int tiles, int32_t *counts, int32_t *offsets,
                               int32_t *tile_off, int32_t *pair_row, int32_t *row_pair, float *w,
                               int *cnt, int ncnt, cudaStream_t stream);
// Stream-K GEMMs of a dense layer (dense_sk.cu): gate|up (SwiGLU to bf16 h)
// or down (bf16 out), token tiles of BN = 16, 32 or 64 rows; `part` holds
// dense_sk_part_floats(BN, gate_up, grid) floats; `cnt` one zeroed counter per
// (weight tile, token tile).
cudaError_t launch_dense_sk(bool gate_up, int BN, const CUtensorMap &a0, const CUtensorMap &a1,
                            const BoxMaps &b, const GemmArgs &args, int T, float *part, int *cnt, int grid,
                            cudaStream_t stream);
size_t dense_sk_part_floats(int BN, bool gate_up, int grid);
cudaError_t prepare_dense_sk();

// ------------------------------------------------------------- self-check
cudaError_t launch_wait_timeout_check(WaitCtl ctl, cudaStream_t stream);

}  // namespace beam
