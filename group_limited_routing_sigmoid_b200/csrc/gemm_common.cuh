// Helpers shared by the single-CTA and the CTA-pair grouped GEMMs.
#pragma once

#include "kernels.cuh"

namespace beam {
namespace gemm {

constexpr int kBM = 128;          // weight rows per A tile per CTA (UMMA M per CTA)
constexpr int kBK = 64;           // K per stage: one 128-byte swizzle row of bf16
constexpr int kEpiWarps = 8;      // two per TMEM lane quadrant, alternating column chunks
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxDynSmem = 232448;
constexpr int kTableBytes = 3 * (1024 + 1) * 4 + 4;   // counts, offsets, tile_off (E <= 1024)
constexpr int kBarrierBytes = 256;
constexpr int kStagingWarpBytes = 2048;                // one 32-row x CH-column block per epilogue warp
constexpr int kStagingBytes = kEpiWarps * kStagingWarpBytes;
constexpr int kStageBudget = kMaxDynSmem - 1024 - kBarrierBytes - kTableBytes - kStagingBytes;

// Epilogues: gate|up with SwiGLU; plain bf16 (down); FP32 (kStoreF32);
// gate|up with SwiGLU from one interleaved weight tile (kSwiGLUI, CTA-pair
// kernel): in each 32-row quarter of the tile, rows 0-15 are 16 gate rows
// and rows 16-31 the up rows of the same intermediate indices.
enum Epi { kSwiGLU = 0, kStoreBF16 = 1, kStoreF32 = 3, kSwiGLUI = 4 };

// Whether the second A tile holds the same weight rows of a second matrix
// (gate|up) rather than the next 128 rows of the same one (paired down).
constexpr bool same_rows(int epi) { return epi == kSwiGLU; }

constexpr int pow2_at_least(int v, int lo)
{
    int p = lo;
    while (p < v) p <<= 1;
    return p;
}

struct Item {
    int e, wt, row0, nrows;
};

// Item i of the list ordered (expert, weight tile, token tile): the expert is
// the largest e with WT * tile_off[e] <= i; its count c is split into
// nt = tile_off[e+1] - tile_off[e] tiles of ceil(c / nt) rows (the last may
// be shorter).
__device__ __forceinline__ Item decode_item(int i, int WT, int E, const int *s_counts,
                                            const int *s_offsets, const int *s_tile)
{
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (WT * s_tile[mid] <= i) lo = mid;
        else hi = mid - 1;
    }
    Item it;
    it.e = lo;
    const int local = i - WT * s_tile[lo];
    const int nt = s_tile[lo + 1] - s_tile[lo];
    it.wt = local / nt;
    const int tt = local - it.wt * nt;
    const int c = s_counts[lo];
    const int bal = (c + nt - 1) / nt;
    it.row0 = s_offsets[lo] + tt * bal;
    it.nrows = min(bal, c - tt * bal);
    return it;
}

// Rows of x for this CTA's gather4 copies of a token tile: copy j (this lane
// takes j = lane, lane + 32, ...) fills tile rows first + 4j .. first + 4j + 3.
// Row r of the expert-sorted order is pair row_pair[r] = t * top_k + slot, so
// its token is row_pair[r] / top_k.  Rows past the tile's valid rows (the MMA
// N is rounded up to 16) repeat the tile's first row; their results are
// never stored.
template <int G>
__device__ __forceinline__ void gather_tokens(const GemmArgs &p, const Item &it, int first,
                                              int n_ops, int lane, int (&tok)[G][4])
{
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const int op = lane + 32 * g;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int r = first + 4 * op + q;
            const int row = (op < n_ops && r < it.nrows) ? it.row0 + r : it.row0;
            tok[g][q] = p.row_pair[row] / p.top_k;
        }
    }
}

// silu(g) = g / (1 + e^-g) in FP32 with the fast exponential and divide; the
// product with u is rounded to bf16 right after, which the approximations
// (a few FP32 ulps) do not reach but in rare rounding-boundary cases.
__device__ __forceinline__ float silu_f32(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&v)[N])
{
    if constexpr (N == 32) tmem_ld32(taddr, v);
    else tmem_ld16(taddr, v);
}

// Load the expert counts, offsets and token-tile prefix into shared memory.
__device__ __forceinline__ void load_tables(const GemmArgs &p, int *s_counts, int *s_offsets,
                                            int *s_tile)
{
    for (int i = threadIdx.x; i < p.E; i += blockDim.x) s_counts[i] = p.counts[i];
    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
        s_offsets[i] = p.offsets[i];
        s_tile[i] = p.tile_off[i];
    }
}

// Epilogue of one accumulator (32 TMEM lanes of this warp, `nrows` columns)
// to bf16 outputs: SwiGLU of (gate, up) column pairs or the plain value;
// chunks of CH columns, alternating between the two warps of a quadrant,
// transposed through the warp's staging block and stored as 16-byte vectors.
//   out:   first output element of this warp's 32-row slice (token row 0)
//   ldo:   output row stride in elements
template <int EPI, int CH, int UP_OFFSET>
__device__ __forceinline__ void epilogue_block(uint32_t taddr, int nrows, int row0, int half,
                                               int lane, uint8_t *stg, __nv_bfloat16 *out, int ldo)
{
    constexpr int VPR = 4;   // 16-byte vectors per 32 bf16
#pragma unroll 1
    for (int c0 = half * CH; c0 < nrows; c0 += 2 * CH) {
        uint32_t g[CH];
        tmem_ld<CH>(taddr + c0, g);
        __nv_bfloat16 *sh = reinterpret_cast<__nv_bfloat16 *>(stg);
        if constexpr (EPI == kSwiGLU) {
            uint32_t u[CH];
            tmem_ld<CH>(taddr + UP_OFFSET + c0, u);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < CH; ++j)
                sh[j * 32 + lane] =
                    __float2bfloat16_rn(silu_f32(__uint_as_float(g[j])) * __uint_as_float(u[j]));
        } else {
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < CH; ++j) sh[j * 32 + lane] = __float2bfloat16_rn(__uint_as_float(g[j]));
        }
        __syncwarp();
#pragma unroll
        for (int v = lane; v < CH * VPR; v += 32) {
            const int j = v / VPR, part = v - j * VPR;
            if (c0 + j < nrows) {
                const uint4 val = *reinterpret_cast<const uint4 *>(stg + v * 16);
                *reinterpret_cast<uint4 *>(out + (size_t)(row0 + c0 + j) * ldo + part * 8) = val;
            }
        }
        __syncwarp();
    }
}

// SwiGLU epilogue of an interleaved gate|up accumulator (kSwiGLUI): TMEM
// lanes 0-15 of this warp's quarter hold gate rows, lanes 16-31 the up rows
// of the same 16 intermediate indices.  Per chunk of 32 token columns, lane l
// and lane l ^ 16 swap half their columns, so lane l < 16 holds gate and up
// of columns 0-15 and lane l + 16 those of columns 16-31 for intermediate
// index l; the 16 x 32 bf16 results go through the warp's staging block to
// 32-byte row stores.
//   out:   first output element of this warp's 16 intermediate columns (token row 0)
__device__ __forceinline__ void epilogue_swiglu_interleaved(uint32_t taddr, int nrows, int row0,
                                                            int half, int lane, uint8_t *stg,
                                                            __nv_bfloat16 *out, int ldo)
{
    __nv_bfloat16 *sh = reinterpret_cast<__nv_bfloat16 *>(stg);   // [32 tokens][16 columns]
    const bool up_lane = lane >= 16;
    const int icol = lane & 15;
#pragma unroll 1
    for (int c0 = half * 32; c0 < nrows; c0 += 64) {
        uint32_t v[32];
        tmem_ld32(taddr + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint32_t send = up_lane ? v[j] : v[16 + j];
            const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 16);
            const float g = __uint_as_float(up_lane ? recv : v[j]);
            const float u = __uint_as_float(up_lane ? v[16 + j] : recv);
            const int tok = up_lane ? 16 + j : j;
            sh[tok * 16 + icol] = __float2bfloat16_rn(silu_f32(g) * u);
        }
        __syncwarp();
#pragma unroll
        for (int w = lane; w < 64; w += 32) {
            const int tok = w >> 1, part = w & 1;
            if (c0 + tok < nrows) {
                const uint4 val = *reinterpret_cast<const uint4 *>(stg + tok * 32 + part * 16);
                *reinterpret_cast<uint4 *>(out + (size_t)(row0 + c0 + tok) * ldo + part * 8) = val;
            }
        }
        __syncwarp();
    }
}

// FP32 values of one accumulator (32 TMEM lanes of this warp = 32 output
// columns, `nrows` token columns), transposed through the warp's staging
// block so that each store is a 16-byte vector: chunks of 16 token rows
// alternate between the two warps of a quadrant; a chunk is 16 rows x 128
// bytes, four vectors per lane.
//   out:   this warp's first output column in token row 0
//   ldo:   output row stride in elements
__device__ __forceinline__ void epilogue_f32_staged(uint32_t taddr, int nrows, int row0, int half,
                                                    int lane, uint8_t *stg, float *out, int ldo)
{
    float *sh = reinterpret_cast<float *>(stg);   // [16 token rows][32 columns]
#pragma unroll 1
    for (int c0 = half * 16; c0 < nrows; c0 += 32) {
        uint32_t v[16];
        tmem_ld16(taddr + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) sh[j * 32 + lane] = __uint_as_float(v[j]);
        __syncwarp();
#pragma unroll
        for (int w = lane; w < 128; w += 32) {
            const int j = w >> 3, part = w & 7;
            if (c0 + j < nrows) {
                const float4 val = *reinterpret_cast<const float4 *>(sh + j * 32 + part * 4);
                *reinterpret_cast<float4 *>(out + (size_t)(row0 + c0 + j) * ldo + part * 4) = val;
            }
        }
        __syncwarp();
    }
}

}  // namespace gemm
}  // namespace beam
