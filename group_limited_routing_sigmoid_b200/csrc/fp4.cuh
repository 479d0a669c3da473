// NVFP4 expert weights: the 4-bit checkpoint format the Beam pages name for
// Blackwell GPUs (launch blog "Introducing Beam", section "Mixture of
// Experts": most parameters stored at 4-bit precision).  Each weight is an
// E2M1 element times an FP8 E4M3 scale shared by 16 consecutive elements of
// its row, times one FP32 scale per tensor.
//
// The grouped GEMM takes the weights in a tiled copy made at create: for
// every (expert, 128-row tile, 64-column K step) the 128 x 32 bytes of codes
// and the 128 x 4 bytes of scales are contiguous, so each stage is two plain
// bulk copies.  Inside a tile the four 16-element blocks of a row are
// planes: codes [block][row][8 bytes], scales [block][row], so the 32 rows a
// converter warp decodes for one block are 256 contiguous bytes.  Converter warps turn a stage into the bf16 tile the tensor
// cores read, in tensor memory (every E2M1 x E4M3 product has at most 6
// significant bits, so it is exact in bf16); the per-tensor scale multiplies
// the FP32 accumulators in the epilogue.
#pragma once

#include "kernels.cuh"

namespace beam {

constexpr int kFp4TileRows = 128;                     // weight rows per tile
constexpr int kFp4TileK = 64;                         // K per stage
constexpr int kFp4CodeTile = kFp4TileRows * kFp4TileK / 2;    // 4096 bytes
constexpr int kFp4ScaleTile = kFp4TileRows * kFp4TileK / 16;  // 512 bytes

// One NVFP4 tensor in the tiled layout: codes [E][R/128][K/64][4][128][8],
// scales [E][R/128][K/64][4][128], and its per-tensor scale.
struct Fp4Tensor {
    const uint8_t *codes;
    const uint8_t *scales;
    float global;
};

// The expert tensors of one grouped GEMM: gate and up (same rows), or down.
struct Fp4Operands {
    Fp4Tensor a[2];
    int row_tiles;     // R / 128 of the tensor
    int k_steps;       // K / 64
};

// Repack an NVFP4 tensor from the row-major layout (codes [rows][K/2],
// scales [rows][K/16]) into the tiled layout.  rows a multiple of 128, K of
// 64; codes 16-byte and scales 4-byte aligned.
cudaError_t launch_fp4_repack(const uint8_t *codes, const uint8_t *scales, long long rows, int K,
                              uint8_t *codes_t, uint8_t *scales_t, cudaStream_t stream);

// Row-major NVFP4 elements (a multiple of 16) -> bf16 [elements]: each
// element times its block scale (the per-tensor scale not applied), decoded
// as the GEMM's converters decode it.  codes 8-byte aligned, out 16-byte.
cudaError_t launch_fp4_dequant(const uint8_t *codes, const uint8_t *scales, long long elements,
                               __nv_bfloat16 *out, cudaStream_t stream);

cudaError_t prepare_grouped_gemm_fp4();
// Grouped GEMM with NVFP4 A operands (single CTA per SM): kind kGateUp (two
// tensors, SwiGLU epilogue) or kDown (one tensor); token tiles (BN) of 16,
// 32, 64 or 128 rows.  b: token-row boxes of the sorted activations.
cudaError_t launch_grouped_gemm_fp4(GemmKind kind, int BN, const Fp4Operands &w,
                                    const BoxMaps &b, const GemmArgs &args, int grid,
                                    cudaStream_t stream);

}  // namespace beam
