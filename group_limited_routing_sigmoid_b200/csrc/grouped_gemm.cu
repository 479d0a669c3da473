// Grouped expert GEMMs of the Beam MoE block on the 5th-generation tensor
// cores (tcgen05 / TMEM), fed by TMA: the single-CTA kernel, used for small
// token tiles (decode).  The CTA-pair kernel for large tiles is in
// grouped_gemm_pair.cu.
//
// Each Beam expert is a SwiGLU MLP with hidden 5120 and intermediate 2560
// (launch blog "Introducing Beam", section "Mixture of Experts"); the SwiGLU
// product is taken in FP32 (section "Residual Stream", FP32 sites).  Two
// kernels per forward pass:
//   gate|up:  h[row, i] = bf16( silu(W_g[e,i,:] . xp[row,:]) * (W_u[e,i,:] . xp[row,:]) )
//   down:     y[row, c] = bf16( W_d[e,c,:] . h[row,:] )
// for every row of the expert-sorted activation buffer, e = the row's expert.
//
// Tiling (weights as the MMA's M operand).  A work item is (expert e, a
// weight tile of e, a token tile of e).  Weight rows are the UMMA A operand
// (M = 128) and the token rows are B, so a decode batch with a handful of
// tokens per expert still issues full 128-row MMAs and streams every weight
// byte once.  An expert's tokens are split into ceil(count / BN) tiles of
// equal size, and each item's MMA N is its tile size rounded up to 16 (a
// runtime field of the instruction descriptor), so ragged experts waste at
// most 15 rows per tile.  The TMA loads of a token tile fetch exactly those
// rows, as a sum of power-of-two boxes of the sorted buffer, or (gate|up,
// by default) four rows at a time straight from x, which spares the sorted
// copy of x altogether.
//   gate|up: two A tiles (gate and up rows i0..i0+127) into two TMEM
//            accumulators, so TMEM lane r holds gate and up of one
//            intermediate row and the SwiGLU needs no exchange;
//   down:    one or two A tiles (rows c0..c0+127 and c0+128..c0+255) that
//            share the token tile, halving the token bytes per MMA.
//
// Warp roles (320 threads, one CTA per SM, persistent over the item list):
//   warp 0      TMA producer (lane 0; all lanes when gate|up gathers token
//               rows from x with tile::gather4);
//   warp 1      TMEM allocator and UMMA issuer (one thread);
//   warps 2..9  epilogue (two per TMEM lane quadrant): tcgen05.ld, SwiGLU or
//               the plain accumulator, rounded to bf16, a 32x32 transpose
//               through shared memory, 16-byte stores.
// Accumulators are double-buffered in TMEM when two fit in its 512 columns,
// so the epilogue of one item overlaps the mainloop of the next.  Every wait
// is bounded (WaitCtl).
#include "gemm_common.cuh"

namespace beam {

using namespace gemm;

namespace {

template <int BN, int NUM_A, int EPI>
struct Cfg {
    static constexpr int A_BYTES = kBM * kBK * 2;
    static constexpr int B_BYTES = BN * kBK * 2;
    static constexpr int STAGE_BYTES = NUM_A * A_BYTES + B_BYTES;
    static constexpr int STAGES_FIT = kStageBudget / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr int ACC_COLS = NUM_A * BN;             // one accumulator buffer
    static constexpr int NBUF = 2 * ACC_COLS <= 512 ? 2 : 1;
    static constexpr int TMEM_COLS = pow2_at_least(NBUF * ACC_COLS, 32);
    static constexpr int CH = BN >= 32 ? 32 : 16;           // epilogue columns per chunk
    static constexpr int ROWS_PER_ITEM = same_rows(EPI) ? kBM : NUM_A * kBM;
    static constexpr bool F32 = EPI == kStoreF32;   // FP32 expert outputs
    static constexpr int SMEM_BYTES =
        1024 + STAGES * STAGE_BYTES + kStagingBytes + kBarrierBytes + kTableBytes;
    static_assert(STAGES >= 2, "pipeline needs two stages");
    static_assert(TMEM_COLS <= 512, "TMEM holds 512 columns");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
    static_assert(B_BYTES % 1024 == 0, "B tile must keep 1024-byte alignment of the next tile");
    static_assert(SMEM_BYTES <= kMaxDynSmem, "shared memory");
    static_assert(!same_rows(EPI) || NUM_A == 2, "gate|up needs the gate and up tiles");
    static_assert(!F32 || NUM_A == 1, "FP32 down: one tile");
    static_assert(32 * CH * 2 <= kStagingWarpBytes, "staging block");
};

}  // namespace

template <int BN, int NUM_A, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA0,
                        const __grid_constant__ CUtensorMap tmA1,
                        const __grid_constant__ BoxMaps tmB, GemmArgs p)
{
    using C = Cfg<BN, NUM_A, EPI>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw_addr);
    uint8_t *staging = base_ptr + C::STAGES * C::STAGE_BYTES;   // 1024-aligned
    uint8_t *bar_ptr = staging + kStagingBytes;
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

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 32 * kEpiWarps);
        }
        mbar_init(smem_u32(drain), 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmA0);
        if (NUM_A == 2) tma_prefetch_desc(&tmA1);
    }
    if (warp == 1) {
        __syncwarp();
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    pdl_launch_dependents();
    pdl_wait();   // set-up above overlaps the previous kernel; data from here on
    load_tables(p, s_counts, s_offsets, s_tile);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int WT = p.R / C::ROWS_PER_ITEM;
    // no work while the status word is set (a failed check or wait)
    const int total = status_is_set(p.ctl.status) ? 0 : WT * s_tile[p.E];
    const int KB = p.K / kBK;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        // Lane 0 loads the weight tiles (and the token tile from the sorted
        // buffer); with gathering, every lane also issues its gather4 copies
        // of token rows straight from x.
        const uint64_t pol_w = l2_policy_evict_first();   // weights: streamed
        const uint64_t pol_x = l2_policy_evict_last();    // activations: reused across tiles
        constexpr int G = (BN / 4 + 31) / 32;             // gather4 copies per lane, at most
        const bool gather = EPI == kSwiGLU && p.gather != 0;
        int stage = 0;
        uint32_t phase = 0;
        long long issued = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            const Item it = decode_item(item, WT, p.E, s_counts, s_offsets, s_tile);
            const int kb0 = 0;
            const int a_row = it.e * p.R + it.wt * C::ROWS_PER_ITEM;
            const int n_load = (it.nrows + 15) & ~15;
            const uint32_t bytes = NUM_A * C::A_BYTES + n_load * (kBK * 2);
            int tok[G][4];
            if (gather) gather_tokens<G>(p, it, 0, n_load >> 2, lane, tok);
            for (int kb = kb0; kb < kb0 + KB; ++kb) {
                bool got = true;
                if (lane == 0 || gather) got = mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, p.ctl);
                ok = __all_sync(0xffffffffu, got);
                if (!ok) break;
                const uint32_t sa = base + stage * C::STAGE_BYTES;
                const uint32_t sb = sa + NUM_A * C::A_BYTES;
                const uint32_t fb = smem_u32(&full[stage]);
                if (lane == 0) {
                    mbar_arrive_expect_tx(fb, bytes);
                    tma_load_2d(sa, &tmA0, kb * kBK, a_row, fb, pol_w);
                    if (NUM_A == 2) {
                        // gate|up: the up matrix at the same rows; down: the next 128 rows
                        const int a_row1 = same_rows(EPI) ? a_row : a_row + kBM;
                        tma_load_2d(sa + C::A_BYTES, &tmA1, kb * kBK, a_row1, fb, pol_w);
                    }
                    if (!gather) {
                        int off = 0;
#pragma unroll
                        for (int bi = 5; bi >= 1; --bi) {   // boxes of 256, 128, 64, 32, 16 rows
                            const int hgt = 8 << bi;
                            if (hgt <= BN && n_load - off >= hgt) {
                                tma_load_2d(sb + off * (kBK * 2), &tmB.m[bi], kb * kBK,
                                            it.row0 + off, fb, pol_x);
                                off += hgt;
                            }
                        }
                    }
                }
                if (gather) {
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const int op = lane + 32 * g;
                        if (op < (n_load >> 2))
                            tma_gather4(sb + op * (4 * kBK * 2), &tmB.gather, kb * kBK, tok[g][0],
                                        tok[g][1], tok[g][2], tok[g][3], fb, pol_x);
                    }
                }
                ++issued;
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
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
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        bool issued_any = false;
        int iter = 0;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++iter) {
            const Item it = decode_item(item, WT, p.E, s_counts, s_offsets, s_tile);
            const int n_mma = (it.nrows + 15) & ~15;
            const uint32_t idesc = umma_idesc_bf16_f32(kBM, n_mma);
            const int acc = iter % C::NBUF;
            const uint32_t acc_phase = (uint32_t)(iter / C::NBUF) & 1u;
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
                    if (NUM_A == 2)
                        umma_bf16(d0 + BN, umma_desc_sw128(sa + C::A_BYTES + k * 32), bdesc, idesc,
                                  accum);
                    issued_any = true;
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
        const int quad = warp & 3;                         // TMEM lanes this warp may access
        const int half = (warp - 2) >> 2;                  // which alternate column chunks
        uint8_t *stg = staging + (warp - 2) * kStagingWarpBytes;
        int iter = 0;
        for (int item = blockIdx.x; item < total; item += gridDim.x, ++iter) {
            const int acc = iter % C::NBUF;
            const uint32_t acc_phase = (uint32_t)(iter / C::NBUF) & 1u;
            const bool ok = mbar_wait(smem_u32(&tfull[acc]), acc_phase, p.ctl);
            if (!__all_sync(0xffffffffu, ok)) break;   // warp-uniform from here on
            tc_fence_after();
            const Item it = decode_item(item, WT, p.E, s_counts, s_offsets, s_tile);
            const uint32_t taddr =
                tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * C::ACC_COLS);
            if constexpr (C::F32) {
                const int col0 = it.wt * kBM + quad * 32;
                epilogue_f32_staged(taddr, it.nrows, it.row0, half, lane, stg, p.out_f32 + col0, p.R);
            } else if constexpr (EPI == kSwiGLU) {
                const int col0 = it.wt * C::ROWS_PER_ITEM + quad * 32;
                epilogue_block<EPI, C::CH, BN>(taddr, it.nrows, it.row0, half, lane, stg,
                                               p.out + col0, p.R);
            } else {
#pragma unroll 1
                for (int a = 0; a < NUM_A; ++a) {
                    const int col0 = it.wt * C::ROWS_PER_ITEM + a * kBM + quad * 32;
                    epilogue_block<EPI, C::CH, 0>(taddr + a * BN, it.nrows, it.row0, half, lane,
                                                  stg, p.out + col0, p.R);
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
template <int BN, int NUM_A, int EPI>
cudaError_t set_smem()
{
    return cudaFuncSetAttribute(grouped_gemm_kernel<BN, NUM_A, EPI>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Cfg<BN, NUM_A, EPI>::SMEM_BYTES);
}

template <int BN, int NUM_A, int EPI>
cudaError_t launch(const CUtensorMap &a0, const CUtensorMap &a1, const BoxMaps &b,
                   const GemmArgs &args, int grid, cudaStream_t stream)
{
    return launch_pdl(grouped_gemm_kernel<BN, NUM_A, EPI>, dim3(grid), dim3(kThreads),
                      Cfg<BN, NUM_A, EPI>::SMEM_BYTES, stream, a0, a1, b, args);
}

template <int BN>
cudaError_t launch_kind(GemmKind kind, const CUtensorMap &a0, const CUtensorMap &a1,
                        const BoxMaps &b, const GemmArgs &args, int grid, cudaStream_t stream)
{
    switch (kind) {
        case GemmKind::kGateUp:
            return launch<BN, 2, kSwiGLU>(a0, a1, b, args, grid, stream);
        case GemmKind::kDown:
            return launch<BN, 1, kStoreBF16>(a0, a1, b, args, grid, stream);
        case GemmKind::kDownPaired:
            return launch<BN, 2, kStoreBF16>(a0, a1, b, args, grid, stream);
        case GemmKind::kDownF32:
            return launch<BN, 1, kStoreF32>(a0, a1, b, args, grid, stream);
        default:
            break;
    }
    return cudaErrorInvalidValue;
}
}  // namespace

bool gemm_tile_supported(int BN)
{
    return BN == 16 || BN == 32 || BN == 64 || BN == 128 || BN == 256;
}

cudaError_t prepare_grouped_gemm(int E)
{
    if (E > 1024) return cudaErrorInvalidValue;
    cudaError_t err;
#define BEAM_PREP(BN)                                                        \
    if ((err = set_smem<BN, 2, kSwiGLU>()) != cudaSuccess) return err;       \
    if ((err = set_smem<BN, 1, kStoreBF16>()) != cudaSuccess) return err;    \
    if ((err = set_smem<BN, 2, kStoreBF16>()) != cudaSuccess) return err;    \
    if ((err = set_smem<BN, 1, kStoreF32>()) != cudaSuccess) return err;
    BEAM_PREP(16)
    BEAM_PREP(32)
    BEAM_PREP(64)
    BEAM_PREP(128)
    BEAM_PREP(256)
#undef BEAM_PREP
    return prepare_grouped_gemm_pair();
}

cudaError_t launch_grouped_gemm(GemmKind kind, int BN, const CUtensorMap &a0, const CUtensorMap &a1,
                                const BoxMaps &b, const GemmArgs &args, int grid,
                                cudaStream_t stream)
{
    switch (BN) {
        case 16: return launch_kind<16>(kind, a0, a1, b, args, grid, stream);
        case 32: return launch_kind<32>(kind, a0, a1, b, args, grid, stream);
        case 64: return launch_kind<64>(kind, a0, a1, b, args, grid, stream);
        case 128: return launch_kind<128>(kind, a0, a1, b, args, grid, stream);
        case 256: return launch_kind<256>(kind, a0, a1, b, args, grid, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace beam
