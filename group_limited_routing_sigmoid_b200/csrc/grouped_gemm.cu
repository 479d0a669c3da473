// Grouped expert GEMMs of the Beam MoE block on the 5th-generation tensor
// cores (tcgen05 / TMEM), fed by TMA.
//
// Each Beam expert is a SwiGLU MLP with hidden 5120 and intermediate 2560
// (launch blog "Introducing Beam", section "Mixture of Experts"); the SwiGLU
// product is taken in FP32 (section "Residual Stream", FP32 sites).  Two
// kernels per forward pass:
//   gate|up:  h[row, i] = bf16( silu(W_g[e,i,:] . xp[row,:]) * (W_u[e,i,:] . xp[row,:]) )
//   down:     y[row, c] = W_d[e,c,:] . h[row,:]                      (fp32 out)
// for every row of the expert-sorted activation buffer, e = the row's expert.
//
// Tiling (weights as the MMA's M operand).  A work item is (expert e, a
// 128-row tile of that expert's weight matrix, a tile of BN token rows of
// e).  The weight tile is the UMMA A operand (M = 128) and the token tile is
// B (N = BN), so a decode batch with a handful of tokens per expert still
// uses full 128-row MMAs while streaming every weight byte exactly once.
// Gate and up go to two accumulators in TMEM (columns [0,BN) and [BN,2BN)),
// so TMEM lane r holds gate and up of the same intermediate row and the
// SwiGLU needs no data exchange between threads.
//
// Warp roles (192 threads, one CTA per SM, persistent over the item list):
//   warp 0      TMA producer: K-slices of 64 into a ring of smem stages;
//   warp 1      TMEM allocator and UMMA issuer (one thread);
//   warps 2..5  epilogue: tcgen05.ld from TMEM, SwiGLU or fp32 store.
// Accumulators are double-buffered in TMEM so the epilogue of one item
// overlaps the mainloop of the next.  Every wait is bounded (WaitCtl).
#include "kernels.cuh"

namespace beam {

namespace {

constexpr int kBM = 128;          // weight rows per tile (UMMA M)
constexpr int kBK = 64;           // K per stage: one 128-byte swizzle row of bf16
constexpr int kThreads = 192;
constexpr int kMaxDynSmem = 232448;
constexpr int kTableBytes = 3 * (1024 + 1) * 4 + 4;   // counts, offsets, tile_off (E <= 1024)
constexpr int kBarrierBytes = 256;

constexpr int pow2_at_least(int v, int lo)
{
    int p = lo;
    while (p < v) p <<= 1;
    return p;
}

template <int BN, int NUM_A>
struct Cfg {
    static constexpr int A_BYTES = kBM * kBK * 2;
    static constexpr int B_BYTES = BN * kBK * 2;
    static constexpr int STAGE_BYTES = NUM_A * A_BYTES + B_BYTES;
    static constexpr int STAGE_BUDGET = kMaxDynSmem - 1024 - kBarrierBytes - kTableBytes;
    static constexpr int STAGES_FIT = STAGE_BUDGET / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr int ACC_COLS = NUM_A * BN;            // one accumulator buffer
    static constexpr int TMEM_COLS = pow2_at_least(2 * ACC_COLS, 32);
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + kBarrierBytes + kTableBytes;
    static_assert(STAGES >= 2, "pipeline needs two stages");
    static_assert(TMEM_COLS <= 512, "TMEM holds 512 columns");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
    static_assert(B_BYTES % 1024 == 0, "B tile must keep 1024-byte alignment of the next tile");
    static_assert(SMEM_BYTES <= kMaxDynSmem, "shared memory");
};

struct Item {
    int e, wt, row0, nrows;
};

// Item i of the list ordered (expert, weight tile, token tile): the expert is
// the largest e with WT * tile_off[e] <= i.
__device__ __forceinline__ Item decode_item(int i, int WT, int E, int BN, const int *s_counts,
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
    it.row0 = s_offsets[lo] + tt * BN;
    it.nrows = min(BN, s_counts[lo] - tt * BN);
    return it;
}

__device__ __forceinline__ float silu_f32(float g) { return g / (1.0f + expf(-g)); }

}  // namespace

template <int BN, int NUM_A>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA0,
                        const __grid_constant__ CUtensorMap tmA1,
                        const __grid_constant__ CUtensorMap tmB, GemmArgs p)
{
    using C = Cfg<BN, NUM_A>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw_addr);
    uint8_t *bar_ptr = base_ptr + C::STAGES * C::STAGE_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(bar_ptr);
    uint64_t *empty = full + C::STAGES;
    uint64_t *tfull = empty + C::STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    int *s_counts = reinterpret_cast<int *>(bar_ptr + kBarrierBytes);
    int *s_offsets = s_counts + p.E;
    int *s_tile = s_offsets + (p.E + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    for (int i = threadIdx.x; i < p.E; i += kThreads) s_counts[i] = p.counts[i];
    for (int i = threadIdx.x; i <= p.E; i += kThreads) {
        s_offsets[i] = p.offsets[i];
        s_tile[i] = p.tile_off[i];
    }
    if (warp == 0 && lane == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 128);
        }
        mbar_init(smem_u32(drain), 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmA0);
        if (NUM_A == 2) tma_prefetch_desc(&tmA1);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 1) {
        __syncwarp();
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int WT = p.R / kBM;
    const int total = WT * s_tile[p.E];
    const int KB = p.K / kBK;

    if (warp == 0 && lane == 0) {
        // ------------------------------------------------ TMA producer
        const uint64_t pol_w = l2_policy_evict_first();   // weights: streamed
        const uint64_t pol_x = l2_policy_evict_last();    // activations: reused across tiles
        int stage = 0;
        uint32_t phase = 0;
        long long issued = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            const Item it = decode_item(item, WT, p.E, BN, s_counts, s_offsets, s_tile);
            const int a_row = it.e * p.R + it.wt * kBM;
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, p.ctl)) {
                    ok = false;
                    break;
                }
                const uint32_t sa = base + stage * C::STAGE_BYTES;
                const uint32_t fb = smem_u32(&full[stage]);
                mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
                tma_load_2d(sa, &tmA0, kb * kBK, a_row, fb, pol_w);
                if (NUM_A == 2) tma_load_2d(sa + C::A_BYTES, &tmA1, kb * kBK, a_row, fb, pol_w);
                tma_load_2d(sa + NUM_A * C::A_BYTES, &tmB, kb * kBK, it.row0, fb, pol_x);
                ++issued;
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok) {
            // Give the copies already in flight time to land before the CTA
            // exits: wait (time-bounded, status ignored) on the last ones.
            long long n = issued < C::STAGES ? issued : C::STAGES;
            int s = stage;
            uint32_t ph = phase;
            for (long long j = 0; j < n; ++j) {
                if (s == 0) {
                    s = C::STAGES - 1;
                    ph ^= 1u;
                } else {
                    --s;
                }
                mbar_wait_drain(smem_u32(&full[s]), ph, p.ctl.limit_ns);
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ UMMA issuer
        constexpr uint32_t idesc = umma_idesc_bf16_f32(kBM, BN);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        bool issued_any = false;
        int iter = 0;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++iter) {
            const int acc = iter & 1;
            const uint32_t acc_phase = (uint32_t)(iter >> 1) & 1u;
            if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, p.ctl)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d0 = tmem_base + (uint32_t)(acc * C::ACC_COLS);
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, p.ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = base + stage * C::STAGE_BYTES;
                const uint32_t sb = sa + NUM_A * C::A_BYTES;
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k) {
                    const uint64_t bdesc = umma_desc_sw128(sb + k * 32);
                    const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
                    umma_bf16(d0, umma_desc_sw128(sa + k * 32), bdesc, idesc, accum);
                    issued_any = true;
                    if (NUM_A == 2)
                        umma_bf16(d0 + BN, umma_desc_sw128(sa + C::A_BYTES + k * 32), bdesc, idesc,
                                  accum);
                }
                umma_commit(smem_u32(&empty[stage]));
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            umma_commit(smem_u32(&tfull[acc]));
        }
        // Every MMA issued must be complete before TMEM is released.
        if (issued_any) {
            umma_commit(smem_u32(drain));
            mbar_wait_drain(smem_u32(drain), 0, p.ctl.limit_ns);
        }
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue
        const int quad = warp & 3;            // TMEM lanes this warp may access
        const int r_in_tile = quad * 32 + lane;
        int iter = 0;
        for (int item = blockIdx.x; item < total; item += gridDim.x, ++iter) {
            const int acc = iter & 1;
            const uint32_t acc_phase = (uint32_t)(iter >> 1) & 1u;
            const bool ok = mbar_wait(smem_u32(&tfull[acc]), acc_phase, p.ctl);
            if (!__all_sync(0xffffffffu, ok)) break;   // warp-uniform from here on
            tc_fence_after();
            const Item it = decode_item(item, WT, p.E, BN, s_counts, s_offsets, s_tile);
            const uint32_t taddr =
                tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * C::ACC_COLS);
            const int r = it.wt * kBM + r_in_tile;   // row of this expert's weight matrix
            for (int c = 0; c < it.nrows; c += 16) {
                uint32_t g[16];
                tmem_ld16(taddr + c, g);
                if (NUM_A == 2) {
                    uint32_t u[16];
                    tmem_ld16(taddr + BN + c, u);
                    tmem_ld_wait();
                    __nv_bfloat16 *h = reinterpret_cast<__nv_bfloat16 *>(p.out);
#pragma unroll
                    for (int n = 0; n < 16; ++n) {
                        if (c + n < it.nrows) {
                            const float gv = __uint_as_float(g[n]);
                            const float uv = __uint_as_float(u[n]);
                            h[(size_t)(it.row0 + c + n) * p.R + r] = __float2bfloat16_rn(silu_f32(gv) * uv);
                        }
                    }
                } else {
                    tmem_ld_wait();
                    float *y = reinterpret_cast<float *>(p.out);
#pragma unroll
                    for (int n = 0; n < 16; ++n)
                        if (c + n < it.nrows)
                            y[(size_t)(it.row0 + c + n) * p.R + r] = __uint_as_float(g[n]);
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
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

namespace {
template <int BN, int NUM_A>
cudaError_t set_smem()
{
    return cudaFuncSetAttribute(grouped_gemm_kernel<BN, NUM_A>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<BN, NUM_A>::SMEM_BYTES);
}

template <int BN, int NUM_A>
cudaError_t launch(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b,
                   const GemmArgs &args, int grid, cudaStream_t stream)
{
    grouped_gemm_kernel<BN, NUM_A>
        <<<grid, kThreads, Cfg<BN, NUM_A>::SMEM_BYTES, stream>>>(a0, a1, b, args);
    return cudaGetLastError();
}
}  // namespace

bool gemm_tile_supported(int BN) { return BN == 16 || BN == 32 || BN == 64 || BN == 128; }

cudaError_t prepare_grouped_gemm(int E)
{
    if (E > 1024) return cudaErrorInvalidValue;
    cudaError_t err;
#define BEAM_PREP(BN)                                  \
    if ((err = set_smem<BN, 1>()) != cudaSuccess) return err; \
    if ((err = set_smem<BN, 2>()) != cudaSuccess) return err;
    BEAM_PREP(16)
    BEAM_PREP(32)
    BEAM_PREP(64)
    BEAM_PREP(128)
#undef BEAM_PREP
    return cudaSuccess;
}

cudaError_t launch_grouped_gemm(bool swiglu, int BN, const CUtensorMap &a0, const CUtensorMap &a1,
                                const CUtensorMap &b, const GemmArgs &args, int grid,
                                cudaStream_t stream)
{
#define BEAM_CASE(BNV)                                                          \
    case BNV:                                                                   \
        return swiglu ? launch<BNV, 2>(a0, a1, b, args, grid, stream)           \
                      : launch<BNV, 1>(a0, a1, b, args, grid, stream);
    switch (BN) {
        BEAM_CASE(16)
        BEAM_CASE(32)
        BEAM_CASE(64)
        BEAM_CASE(128)
        default:
            return cudaErrorInvalidValue;
    }
#undef BEAM_CASE
}

}  // namespace beam
