// Grouped expert GEMMs of the Beam MoE block on CTA pairs: clusters of two
// CTAs on two SMs share each tcgen05 MMA (cta_group::2).  Used for large
// token tiles (prefill).  Same computation and item order as
// grouped_gemm.cu; see there for the block's definition.
//
// A pair item covers 256 weight rows per A matrix and up to BN tokens.  CTA r
// of the pair holds weight rows r*128 .. r*128+127 (its half of the MMA's
// M = 256) and token rows r*N/2 .. r*N/2+N/2-1 (its half of N); the MMA,
// issued by CTA 0, reads both CTAs' shared memory and writes each CTA's TMEM
// (128 lanes, its weight rows, all N token columns).
//
// Two rings.  The weight tiles stream from HBM with a loaded latency of a
// few microseconds, the token rows come from L2 (an expert's token tile is
// reused by all of its weight blocks) with about a third of that.  So the
// weights get a ring of their own, as deep as shared memory allows, and the
// token rows a shallow one; each has its own producer warp, so neither ring
// waits on the other's slots.  With 256-token tiles this keeps 4 weight
// stages (128 KB per SM) in flight instead of 3 in one shared ring.
//
// Synchronisation (every wait bounded):
//   fullA[s], fullB[s]  in CTA 0: CTA 0's producers expect the bytes of both
//                       CTAs; both CTAs' TMA loads complete on them;
//   emptyA[s], emptyB[s] in each CTA: the MMAs' completion, multicast to both;
//   tfull[a]   in each CTA: accumulator ready, multicast to both;
//   tempty[a]  in CTA 0: both CTAs' epilogue threads arrive;
//   drain      in each CTA: all MMAs complete, before TMEM is released.
// Only local TMA loads (no multicast).  The expert tables are read from
// global memory (a few hundred bytes, L1-resident), which leaves their
// shared memory to the rings.
#include "gemm_common.cuh"

namespace beam {

using namespace gemm;

namespace {

constexpr int kPairThreads = kThreads + 32;     // + warp 10: token-row producer
constexpr int kPairMaxStages = 16;              // barrier slots per ring
constexpr int kPairBarrierBytes = 1024;
constexpr int kPairRingBytes = kMaxDynSmem - 1024 - kPairBarrierBytes - kStagingBytes;
constexpr int kPairDefaultBStages = 3;
constexpr int kPairCh = 32;                     // epilogue token columns per chunk (bf16 paths)

template <int BN, int NUM_A, int EPI>
struct PairCfg {
    static constexpr int HALF = BN / 2;                    // token rows per CTA, at most
    static constexpr int A_BYTES = kBM * kBK * 2;          // one 128 x 64 weight tile
    static constexpr int A_STAGE = NUM_A * A_BYTES;
    static constexpr int B_STAGE = HALF * kBK * 2;
    static constexpr int ACC_COLS = NUM_A * BN;            // per CTA: 128 lanes x N per matrix
    static constexpr int NBUF = 2 * ACC_COLS <= 512 ? 2 : 1;
    static constexpr int TMEM_COLS = pow2_at_least(NBUF * ACC_COLS, 32);
    // weight rows of one matrix per item: gate|up 256 (128 per CTA, both
    // matrices), interleaved gate|up 128 (64 gate + 64 up rows per CTA),
    // down 256 per weight block
    static constexpr int ROWS_PER_ITEM = EPI == kSwiGLUI ? kBM : 2 * kBM * (EPI == kSwiGLU ? 1 : NUM_A);
    static constexpr int SMEM_BYTES = kMaxDynSmem;
    static_assert(TMEM_COLS <= 512, "TMEM holds 512 columns");
    static_assert(BN % 32 == 0 && BN >= 64 && BN <= 256, "pair UMMA N");
    static_assert(A_STAGE % 1024 == 0 && B_STAGE % 1024 == 0, "stages keep 1024-byte alignment");
    static_assert(kPairRingBytes >= 2 * A_STAGE + 2 * B_STAGE, "two stages per ring");
    static_assert(EPI != kSwiGLU || NUM_A == 2, "SwiGLU needs the gate and up tiles");
    static_assert(EPI == kSwiGLU || EPI == kStoreBF16 || EPI == kStoreF32 || EPI == kSwiGLUI,
                  "pair epilogues");
    static_assert(EPI != kSwiGLUI || NUM_A == 1, "one interleaved tile holds gate and up");
    static_assert(4 * kPairMaxStages * 8 + 5 * 8 + 4 <= kPairBarrierBytes, "barrier block");
};

constexpr uint16_t kPairMask = 0x3;

__device__ __forceinline__ void ring_next(int &s, uint32_t &ph, int n)
{
    if (++s == n) {
        s = 0;
        ph ^= 1u;
    }
}

// Wait (time-bounded, status ignored) for the last min(issued, n) copies a
// ring's producer issued to land, so that no copy is in flight when the CTA
// leaves after a failed wait.  CTA 0's barriers count both CTAs' copies.
__device__ __forceinline__ void drain_ring(uint64_t *full, int s, uint32_t ph, long long issued,
                                           int n, long long limit_ns)
{
    const long long m = issued < n ? issued : n;
    for (long long j = 0; j < m; ++j) {
        if (s == 0) {
            s = n - 1;
            ph ^= 1u;
        } else {
            --s;
        }
        mbar_wait_drain(smem_u32(&full[s]), ph, limit_ns);
    }
}

}  // namespace

template <int BN, int NUM_A, int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA0,
                             const __grid_constant__ CUtensorMap tmA1,
                             const __grid_constant__ BoxMaps tmB, GemmArgs p)
{
    using C = PairCfg<BN, NUM_A, EPI>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw_addr);
    const int SA = p.a_stages, SB = p.b_stages;            // ring depths (host-checked)
    const uint32_t ring_b = base + (uint32_t)(SA * C::A_STAGE);
    uint8_t *staging = base_ptr + SA * C::A_STAGE + SB * C::B_STAGE;
    uint64_t *bars = reinterpret_cast<uint64_t *>(staging + kStagingBytes);
    uint64_t *fullA = bars;
    uint64_t *emptyA = fullA + kPairMaxStages;
    uint64_t *fullB = emptyA + kPairMaxStages;
    uint64_t *emptyB = fullB + kPairMaxStages;
    uint64_t *tfull = emptyB + kPairMaxStages;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();     // 0: issues the MMAs
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < SA; ++s) {
            mbar_init(smem_u32(&fullA[s]), 1);
            mbar_init(smem_u32(&emptyA[s]), 1);
        }
        for (int s = 0; s < SB; ++s) {
            mbar_init(smem_u32(&fullB[s]), 1);
            mbar_init(smem_u32(&emptyB[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), 1);
            mbar_init(smem_u32(&tempty[a]), 2 * 32 * kEpiWarps);
        }
        mbar_init(smem_u32(drain), 1);
        fence_barrier_init();
        tma_prefetch_desc(&tmA0);
        if (NUM_A == 2) tma_prefetch_desc(&tmA1);
    }
    if (warp == 1) {
        __syncwarp();
        tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    pdl_launch_dependents();
    pdl_wait();   // set-up above overlaps the previous kernel; data from here on
    tc_fence_before();
    __syncthreads();
    __syncwarp();
    cluster_sync();   // both CTAs' barriers exist before either signals the other
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int WT = p.R / C::ROWS_PER_ITEM;
    // no work while the status word is set (a failed check or wait)
    const int total = status_is_set(p.ctl.status) ? 0 : WT * __ldg(&p.tile_off[p.E]);
    const int KB = p.K / kBK;

    if (warp == 0) {
        if (lane == 0) {
            // -------------------------------------------- weight producer
            const uint64_t pol_w = l2_policy_evict_first();   // weights: streamed once
            int sa = 0;
            uint32_t pa = 0;
            long long issued = 0;
            bool ok = true;
            for (int item = pair; item < total && ok; item += npairs) {
                const Item it = decode_item(item, WT, p.E, p.counts, p.offsets, p.tile_off);
                // A rows of this CTA: its 128-row half of each 256-row block
                // (interleaved gate|up: its 64 intermediate rows of the 128)
                const int a_base = it.e * p.R + it.wt * C::ROWS_PER_ITEM +
                                   (int)rank * (EPI == kSwiGLUI ? kBM / 2 : kBM);
                // gate|up: the up matrix at the same rows; down: the next 256-row block
                const int a_row1 = EPI == kSwiGLU ? a_base : a_base + 2 * kBM;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(smem_u32(&emptyA[sa]), pa ^ 1u, p.ctl)) {
                        ok = false;
                        break;
                    }
                    const uint32_t dst = base + (uint32_t)(sa * C::A_STAGE);
                    const uint32_t f_local = smem_u32(&fullA[sa]);
                    const uint32_t f = mapa_shared(f_local, 0);   // CTA 0's barrier
                    if (rank == 0) mbar_arrive_expect_tx(f_local, 2u * C::A_STAGE);
                    if constexpr (EPI == kSwiGLUI) {
                        // 16-row boxes: gate rows to rows 32q..32q+15 of the
                        // tile, the same up rows to 32q+16..32q+31
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            tma_load_2d_pair(dst + (uint32_t)(32 * q) * (kBK * 2), &tmA0, kb * kBK,
                                             a_base + 16 * q, f, pol_w);
                            tma_load_2d_pair(dst + (uint32_t)(32 * q + 16) * (kBK * 2), &tmA1,
                                             kb * kBK, a_base + 16 * q, f, pol_w);
                        }
                    } else {
                        tma_load_2d_pair(dst, &tmA0, kb * kBK, a_base, f, pol_w);
                        if (NUM_A == 2)
                            tma_load_2d_pair(dst + C::A_BYTES, &tmA1, kb * kBK, a_row1, f, pol_w);
                    }
                    ++issued;
                    ring_next(sa, pa, SA);
                }
            }
            if (!ok && rank == 0) drain_ring(fullA, sa, pa, issued, SA, p.ctl.limit_ns);
        }
    } else if (warp == kPairThreads / 32 - 1) {
        // ------------------------------------------------ token-row producer
        // Lane 0 loads boxes of the sorted rows; with gathering every lane
        // issues its gather4 copies of rows straight from x.
        const uint64_t pol_x = l2_policy_evict_last();    // activations: reused across tiles
        constexpr int G = (C::HALF / 4 + 31) / 32;          // gather4 copies per lane, at most
        const bool gather = (EPI == kSwiGLU || EPI == kSwiGLUI) && p.gather != 0;
        int sb = 0;
        uint32_t pb = 0;
        long long issued = 0;
        bool ok = true;
        for (int item = pair; item < total && ok; item += npairs) {
            const Item it = decode_item(item, WT, p.E, p.counts, p.offsets, p.tile_off);
            const int n_mma = (it.nrows + 15) & ~15;
            const int half = n_mma >> 1;                    // this CTA's token rows
            const int b_row = it.row0 + (int)rank * half;
            const uint32_t pair_bytes = 2u * (uint32_t)(half * (kBK * 2));
            int tok[G][4];
            if (gather) gather_tokens<G>(p, it, (int)rank * half, half >> 2, lane, tok);
            for (int kb = 0; kb < KB; ++kb) {
                bool got = true;
                if (lane == 0 || gather) got = mbar_wait(smem_u32(&emptyB[sb]), pb ^ 1u, p.ctl);
                ok = __all_sync(0xffffffffu, got);
                if (!ok) break;
                const uint32_t dst = ring_b + (uint32_t)(sb * C::B_STAGE);
                const uint32_t f_local = smem_u32(&fullB[sb]);
                const uint32_t f = mapa_shared(f_local, 0);   // CTA 0's barrier
                if (lane == 0) {
                    if (rank == 0) mbar_arrive_expect_tx(f_local, pair_bytes);
                    if (!gather) {
                        int off = 0;
#pragma unroll
                        for (int bi = 4; bi >= 0; --bi) {   // boxes of 128, 64, 32, 16, 8 rows
                            const int hgt = 8 << bi;
                            if (hgt <= C::HALF && half - off >= hgt) {
                                tma_load_2d_pair(dst + off * (kBK * 2), &tmB.m[bi], kb * kBK,
                                                 b_row + off, f, pol_x);
                                off += hgt;
                            }
                        }
                    }
                }
                if (gather) {
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const int op = lane + 32 * g;
                        if (op < (half >> 2))
                            tma_gather4_pair(dst + op * (4 * kBK * 2), &tmB.gather, kb * kBK,
                                             tok[g][0], tok[g][1], tok[g][2], tok[g][3], f, pol_x);
                    }
                }
                ++issued;
                ring_next(sb, pb, SB);
            }
        }
        if (!ok && lane == 0 && rank == 0) drain_ring(fullB, sb, pb, issued, SB, p.ctl.limit_ns);
    } else if (warp == 1 && lane == 0 && rank == 0) {
        // ------------------------------------------------ UMMA issuer (CTA 0)
        int sa = 0, sb = 0;
        uint32_t pa = 0, pb = 0;
        bool ok = true;
        bool issued_any = false;
        int iter = 0;
        for (int item = pair; item < total && ok; item += npairs, ++iter) {
            const Item it = decode_item(item, WT, p.E, p.counts, p.offsets, p.tile_off);
            const int n_mma = (it.nrows + 15) & ~15;
            const uint32_t idesc = umma_idesc_bf16_f32(2 * kBM, n_mma);
            const int acc = iter % C::NBUF;
            const uint32_t acc_phase = (uint32_t)(iter / C::NBUF) & 1u;
            if (!mbar_wait_cluster(smem_u32(&tempty[acc]), acc_phase ^ 1u, p.ctl)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d0 = tmem_base + (uint32_t)(acc * C::ACC_COLS);
            for (int kb = 0; kb < KB; ++kb) {
                if (!mbar_wait(smem_u32(&fullA[sa]), pa, p.ctl) ||
                    !mbar_wait(smem_u32(&fullB[sb]), pb, p.ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a_addr = base + (uint32_t)(sa * C::A_STAGE);
                const uint32_t b_addr = ring_b + (uint32_t)(sb * C::B_STAGE);
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k) {
                    const uint64_t bdesc = umma_desc_sw128(b_addr + k * 32);
                    const uint32_t accum = (kb > 0 || k > 0) ? 1u : 0u;
                    umma_bf16_pair(d0, umma_desc_sw128(a_addr + k * 32), bdesc, idesc, accum);
                    if (NUM_A == 2)
                        umma_bf16_pair(d0 + BN, umma_desc_sw128(a_addr + C::A_BYTES + k * 32), bdesc,
                                       idesc, accum);
                    issued_any = true;
                }
                umma_commit_pair(smem_u32(&emptyA[sa]), kPairMask);
                umma_commit_pair(smem_u32(&emptyB[sb]), kPairMask);
                ring_next(sa, pa, SA);
                ring_next(sb, pb, SB);
            }
            if (!ok) break;
            umma_commit_pair(smem_u32(&tfull[acc]), kPairMask);
        }
        if (issued_any) umma_commit_pair(smem_u32(drain), kPairMask);
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue (both CTAs)
        const int quad = warp & 3;
        const int half_sel = (warp - 2) >> 2;
        uint8_t *stg = staging + (warp - 2) * kStagingWarpBytes;
        const uint32_t tempty_remote0 = mapa_shared(smem_u32(&tempty[0]), 0);
        const uint32_t tempty_remote1 = mapa_shared(smem_u32(&tempty[1]), 0);
        int iter = 0;
        for (int item = pair; item < total; item += npairs, ++iter) {
            const int acc = iter % C::NBUF;
            const uint32_t acc_phase = (uint32_t)(iter / C::NBUF) & 1u;
            const bool ok = mbar_wait(smem_u32(&tfull[acc]), acc_phase, p.ctl);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const Item it = decode_item(item, WT, p.E, p.counts, p.offsets, p.tile_off);
            const uint32_t taddr =
                tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * C::ACC_COLS);
            if constexpr (EPI == kSwiGLU) {
                const int col0 = it.wt * C::ROWS_PER_ITEM + (int)rank * kBM + quad * 32;
                epilogue_block<EPI, kPairCh, BN>(taddr, it.nrows, it.row0, half_sel, lane, stg,
                                               p.out + col0, p.R);
            } else if constexpr (EPI == kSwiGLUI) {
                const int col0 = it.wt * C::ROWS_PER_ITEM + (int)rank * (kBM / 2) + quad * 16;
                epilogue_swiglu_interleaved(taddr, it.nrows, it.row0, half_sel, lane, stg,
                                            p.out + col0, p.R);
            } else if constexpr (EPI == kStoreF32) {
                // FP32 expert outputs through the staging block, 16-byte stores
#pragma unroll 1
                for (int a = 0; a < NUM_A; ++a) {
                    const int col0 =
                        it.wt * C::ROWS_PER_ITEM + a * 2 * kBM + (int)rank * kBM + quad * 32;
                    epilogue_f32_staged(taddr + a * BN, it.nrows, it.row0, half_sel, lane, stg,
                                        p.out_f32 + col0, p.R);
                }
            } else {
#pragma unroll 1
                for (int a = 0; a < NUM_A; ++a) {
                    const int col0 =
                        it.wt * C::ROWS_PER_ITEM + a * 2 * kBM + (int)rank * kBM + quad * 32;
                    epilogue_block<EPI, kPairCh, 0>(taddr + a * BN, it.nrows, it.row0, half_sel,
                                                  lane, stg, p.out + col0, p.R);
                }
            }
            tc_fence_before();
            mbar_arrive_cluster(acc == 0 ? tempty_remote0 : tempty_remote1);
        }
    }

    // Both CTAs: no TMEM release until CTA 0's MMAs are complete.
    if (warp == 1 && lane == 0 && pair < total)
        mbar_wait_drain(smem_u32(drain), 0, p.ctl.limit_ns);
    tc_fence_before();
    __syncthreads();
    __syncwarp();
    cluster_sync();   // no CTA leaves while the other may still signal it
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

namespace {
int g_pair_max_ctas = 0;

template <int BN, int NUM_A, int EPI>
cudaError_t set_smem_pair()
{
    return cudaFuncSetAttribute(grouped_gemm_pair_kernel<BN, NUM_A, EPI>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                PairCfg<BN, NUM_A, EPI>::SMEM_BYTES);
}

template <int BN, int NUM_A, int EPI>
cudaError_t launch_pair(const CUtensorMap &a0, const CUtensorMap &a1, const BoxMaps &b,
                        const GemmArgs &args, int grid, cudaStream_t stream)
{
    using C = PairCfg<BN, NUM_A, EPI>;
    // ring depths: the token rows' ring as asked (default 3), the weights'
    // ring as deep as the rest of shared memory allows
    GemmArgs a = args;
    a.b_stages = args.b_stages > 0 ? args.b_stages : kPairDefaultBStages;
    if (a.b_stages < 2 || a.b_stages > kPairMaxStages) return cudaErrorInvalidValue;
    a.a_stages = (kPairRingBytes - a.b_stages * C::B_STAGE) / C::A_STAGE;
    if (a.a_stages > kPairMaxStages) a.a_stages = kPairMaxStages;
    if (a.a_stages < 2) return cudaErrorInvalidValue;
    return launch_pdl(grouped_gemm_pair_kernel<BN, NUM_A, EPI>, dim3(grid), dim3(kPairThreads),
                      C::SMEM_BYTES, stream, a0, a1, b, a);
}

template <int BN>
cudaError_t launch_pair_kind(GemmKind kind, const CUtensorMap &a0, const CUtensorMap &a1,
                             const BoxMaps &b, const GemmArgs &args, int grid, cudaStream_t stream)
{
    switch (kind) {
        case GemmKind::kGateUp:
            return launch_pair<BN, 2, kSwiGLU>(a0, a1, b, args, grid, stream);
        case GemmKind::kDown:
            return launch_pair<BN, 1, kStoreBF16>(a0, a1, b, args, grid, stream);
        case GemmKind::kDownPaired:
            return launch_pair<BN, 2, kStoreBF16>(a0, a1, b, args, grid, stream);
        case GemmKind::kGateUpI:
            return launch_pair<BN, 1, kSwiGLUI>(a0, a1, b, args, grid, stream);
        case GemmKind::kDownY32:
            return launch_pair<BN, 1, kStoreF32>(a0, a1, b, args, grid, stream);
        case GemmKind::kDownPairedY32:
            return launch_pair<BN, 2, kStoreF32>(a0, a1, b, args, grid, stream);
        default:
            break;
    }
    return cudaErrorInvalidValue;
}
}  // namespace

bool gemm_pair_supported(int BN) { return BN == 64 || BN == 128 || BN == 256; }

int gemm_pair_max_ctas() { return g_pair_max_ctas; }

cudaError_t prepare_grouped_gemm_pair()
{
    cudaError_t err;
#define BEAM_PREP_PAIR(BN)                                                        \
    if ((err = set_smem_pair<BN, 2, kSwiGLU>()) != cudaSuccess) return err;       \
    if ((err = set_smem_pair<BN, 1, kStoreBF16>()) != cudaSuccess) return err;    \
    if ((err = set_smem_pair<BN, 2, kStoreBF16>()) != cudaSuccess) return err;    \
    if ((err = set_smem_pair<BN, 1, kStoreF32>()) != cudaSuccess) return err;     \
    if ((err = set_smem_pair<BN, 1, kSwiGLUI>()) != cudaSuccess) return err;      \
    if ((err = set_smem_pair<BN, 2, kStoreF32>()) != cudaSuccess) return err;
    BEAM_PREP_PAIR(64)
    BEAM_PREP_PAIR(128)
    BEAM_PREP_PAIR(256)
#undef BEAM_PREP_PAIR
    // How many pairs fit at once (one CTA per SM; pairs must sit on SM pairs
    // of one GPC), so that the persistent grid is fully resident.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = PairCfg<256, 2, kSwiGLU>::SMEM_BYTES;
    cfg.numAttrs = 0;   // the cluster shape comes from the kernel's __cluster_dims__
    int clusters = 0;
    err = cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_pair_kernel<256, 2, kSwiGLU>, &cfg);
    if (err != cudaSuccess) return err;
    g_pair_max_ctas = 2 * clusters;
    return cudaSuccess;
}

cudaError_t launch_grouped_gemm_pair(GemmKind kind, int BN, const CUtensorMap &a0,
                                     const CUtensorMap &a1, const BoxMaps &b,
                                     const GemmArgs &args, int grid, cudaStream_t stream)
{
    if (grid < 2 || grid % 2 != 0) return cudaErrorInvalidValue;
    switch (BN) {
        case 64: return launch_pair_kind<64>(kind, a0, a1, b, args, grid, stream);
        case 128: return launch_pair_kind<128>(kind, a0, a1, b, args, grid, stream);
        case 256: return launch_pair_kind<256>(kind, a0, a1, b, args, grid, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace beam
