// Stream-K GEMMs of the dense SwiGLU MLP layer (launch blog "Introducing
// Beam", section "Mixture of Experts": the first three layers use a dense
// SwiGLU MLP; section "Residual Stream": the SwiGLU product in FP32) for
// decode-sized batches, where the weight tiles alone give too few work items
// to fill every SM evenly.
//
// The work is (weight tile of 128 rows, token tile of BN rows) x K steps of
// 64.  Unit u = tile * KB + kb; CTA b of G takes units [b*U/G, (b+1)*U/G),
// i.e. the same number of K steps (within one) on every SM.  A CTA's range
// cuts it into segments, each a K range of one tile:
//   - a segment that covers its whole tile finishes it in the epilogue
//     (SwiGLU to bf16 h for gate|up; bf16 out for down);
//   - a tile cut between CTAs b0 < ... < b1 is finished by b0, the owner of
//     its first K steps.  That piece is the last segment of b0's range, so b0
//     reaches it last.  Every other piece writes its FP32 sums to its CTA's
//     slot (slot 0 for the CTA's first segment, 1 for its last) and counts
//     itself in the tile's counter.  b0 waits (bounded) for the count, then
//     adds the pieces in K order to its own sums, read straight from TMEM, and
//     applies the epilogue.  A CTA waits only on higher-numbered CTAs, which
//     publish their pieces of the tile before any wait of their own, and all
//     CTAs are resident (one per SM, the grid no larger than the SM count).
// The counters are zeroed by the layer's set-up kernel before each pass.
//
// Roles as the single-CTA grouped GEMM (grouped_gemm.cu): warp 0 TMA
// producer, warp 1 TMEM allocator and MMA issuer, warps 2..9 epilogue, two
// accumulators in TMEM so one segment's epilogue overlaps the next
// segment's MMAs.  Every wait is bounded.
#include "gemm_common.cuh"

namespace beam {

using namespace gemm;

namespace {

template <int BN, bool GATEUP>
struct SkCfg {
    static constexpr int NUM_A = GATEUP ? 2 : 1;
    static constexpr int A_BYTES = kBM * kBK * 2;
    static constexpr int B_BYTES = BN * kBK * 2;
    static constexpr int STAGE_BYTES = NUM_A * A_BYTES + B_BYTES;
    static constexpr int STAGES_FIT = (kStageBudget + kTableBytes) / STAGE_BYTES;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr int ACC_COLS = NUM_A * BN;
    static constexpr int NBUF = 2;
    static constexpr int TMEM_COLS = pow2_at_least(NBUF * ACC_COLS, 32);
    static constexpr int CH = BN >= 32 ? 32 : 16;
    static constexpr int PART = BN * NUM_A * kBM;   // floats of one segment's sums
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + kStagingBytes + kBarrierBytes;
    static_assert((2 * STAGES + 6) * 8 + 4 <= kBarrierBytes, "barrier block");
    static_assert(STAGES >= 2, "pipeline needs two stages");
    static_assert(TMEM_COLS <= 512, "TMEM holds 512 columns");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 64, "stream-K token tiles of 16..64 rows");
    static_assert(SMEM_BYTES <= kMaxDynSmem, "shared memory");
};

// Prefetch of one tile of a 2-D tensor into L2 (no shared memory, no
// completion to wait for).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *map, int32_t x, int32_t y)
{
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}

struct Seg {
    int t;        // tile
    int k0, k1;   // K steps [k0, k1)
    int first;    // 1: the CTA's first segment (slot 0), else slot 1
};

__device__ __forceinline__ long long unit_start(int b, long long U, int G)
{
    return (long long)b * U / G;
}

// CTA whose range holds unit u: the largest b with floor(b*U/G) <= u.
__device__ __forceinline__ int unit_owner(long long u, long long U, int G)
{
    return (int)(((u + 1) * (long long)G - 1) / U);
}

// Segment j of CTA b (j counts from 0); false past its range.
__device__ __forceinline__ bool segment(int b, int j, long long U, int G, int KB, Seg &s)
{
    const long long u0 = unit_start(b, U, G), u1 = unit_start(b + 1, U, G);
    if (u0 >= u1) return false;
    const int t0 = (int)(u0 / KB);
    const int t = t0 + j;
    const long long a = (long long)t * KB > u0 ? (long long)t * KB : u0;
    const long long e = (long long)(t + 1) * KB < u1 ? (long long)(t + 1) * KB : u1;
    if (a >= e) return false;
    s.t = t;
    s.k0 = (int)(a - (long long)t * KB);
    s.k1 = (int)(e - (long long)t * KB);
    s.first = j == 0;
    return true;
}

// Barrier of the 256 epilogue threads on an mbarrier, with the bounded wait:
// if a warp has left after a failed wait, the others give up too.
__device__ __forceinline__ bool epi_sync(uint64_t *bar, uint32_t &phase, const WaitCtl &ctl)
{
    mbar_arrive(smem_u32(bar));
    const bool ok = mbar_wait(smem_u32(bar), phase, ctl);
    phase ^= 1u;
    return ok;
}

// Wait (bounded) until *count reaches target: the other pieces of a tile are
// published.  Their CTAs are resident (one CTA per SM, the grid no larger
// than the SM count) and never wait for this one, since a CTA waits only on
// pieces of higher-numbered CTAs.  Gives up as mbar_wait does.
__device__ __forceinline__ bool wait_count(const int *count, int target, const WaitCtl &ctl)
{
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        int v;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(count) : "memory");
        if (v >= target) return true;
        __nanosleep(64);
        if ((it & 15u) == 15u) {
            if (status_is_set(ctl.status)) return false;
            if ((long long)(global_timer_ns() - t0) > ctl.limit_ns) {
                record_status(ctl.status, kStatusTimeout);
                return false;
            }
        }
    }
}

}  // namespace

// GATEUP: A = W_gate and W_up tiles [I, H], B = x; h = bf16(silu(g) * u).
// Otherwise: A = W_down tiles [H, I], B = h; out = bf16(sum).
//   p.R: weight rows (I or H); p.K: reduction length; out: [T, R] bf16.
//   part: [2 G][PART] FP32 slots; cnt: [tiles] arrival counters (zero on entry).
template <int BN, bool GATEUP>
__global__ void __launch_bounds__(kThreads, 1)
    dense_sk_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                    const __grid_constant__ BoxMaps tmB, GemmArgs p, int T, float *part, int *cnt)
{
    using C = SkCfg<BN, GATEUP>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw_addr);
    uint8_t *staging = base_ptr + C::STAGES * C::STAGE_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(staging + kStagingBytes);
    uint64_t *empty = full + C::STAGES;
    uint64_t *tfull = empty + C::STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint64_t *epi_bar = drain + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(epi_bar + 1);
    __shared__ int s_last;

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
        mbar_init(smem_u32(epi_bar), 32 * kEpiWarps);
        fence_barrier_init();
        tma_prefetch_desc(&tmA0);
        if (GATEUP) tma_prefetch_desc(&tmA1);
        // the first 8 weight tiles of this CTA's range into L2 while the
        // preceding kernel finishes; a prefetch only warms the coherent L2,
        // so issuing it before the wait for that kernel is safe
        {
            const int NT0 = (T + BN - 1) / BN, KB0 = p.K / kBK;
            const long long U0 = (long long)(p.R / kBM) * NT0 * KB0;
            Seg s0;
            if (U0 > 0 && segment(blockIdx.x, 0, U0, gridDim.x, KB0, s0)) {
                const int wt0 = s0.t / NT0;
                const int kend = s0.k0 + 8 < s0.k1 ? s0.k0 + 8 : s0.k1;
                for (int kb = s0.k0; kb < kend; ++kb) {
                    tma_prefetch_l2_2d(&tmA0, kb * kBK, wt0 * kBM);
                    if (GATEUP) tma_prefetch_l2_2d(&tmA1, kb * kBK, wt0 * kBM);
                }
            }
        }
    }
    if (warp == 1) {
        __syncwarp();
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    pdl_launch_dependents();
    pdl_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int NT = (T + BN - 1) / BN;                 // token tiles
    const int WT = p.R / kBM;                         // weight tiles
    const int KB = p.K / kBK;
    const long long U = status_is_set(p.ctl.status) ? 0 : (long long)WT * NT * KB;
    const int G = gridDim.x;
    const int b = blockIdx.x;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ TMA producer
            const uint64_t pol_w = l2_policy_evict_first();
            const uint64_t pol_x = l2_policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            Seg sg;
            for (int j = 0; U > 0 && ok && segment(b, j, U, G, KB, sg); ++j) {
                const int wt = sg.t / NT, tt = sg.t - wt * NT;
                const int row0 = tt * BN, nrows = min(BN, T - row0);
                const int n_load = (nrows + 15) & ~15;
                const uint32_t bytes = C::NUM_A * C::A_BYTES + n_load * (kBK * 2);
                for (int kb = sg.k0; kb < sg.k1; ++kb) {
                    if (!mbar_wait(smem_u32(&empty[stage]), phase ^ 1u, p.ctl)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sa = base + stage * C::STAGE_BYTES;
                    const uint32_t sb = sa + C::NUM_A * C::A_BYTES;
                    const uint32_t fb = smem_u32(&full[stage]);
                    mbar_arrive_expect_tx(fb, bytes);
                    tma_load_2d(sa, &tmA0, kb * kBK, wt * kBM, fb, pol_w);
                    if (GATEUP) tma_load_2d(sa + C::A_BYTES, &tmA1, kb * kBK, wt * kBM, fb, pol_w);
                    int off = 0;
#pragma unroll
                    for (int bi = 3; bi >= 1; --bi) {   // boxes of 64, 32, 16 rows
                        const int hgt = 8 << bi;
                        if (hgt <= BN && n_load - off >= hgt) {
                            tma_load_2d(sb + off * (kBK * 2), &tmB.m[bi], kb * kBK, row0 + off, fb, pol_x);
                            off += hgt;
                        }
                    }
                    ++issued;
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                const long long n = issued < C::STAGES ? issued : C::STAGES;
                int s = stage;
                uint32_t ph = phase;
                for (long long i = 0; i < n; ++i) {
                    if (s == 0) {
                        s = C::STAGES - 1;
                        ph ^= 1u;
                    } else {
                        --s;
                    }
                    mbar_wait_drain(smem_u32(&full[s]), ph, p.ctl.limit_ns);
                }
            }
        }
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------ UMMA issuer
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        bool issued_any = false;
        Seg sg;
        for (int j = 0; U > 0 && ok && segment(b, j, U, G, KB, sg); ++j) {
            const int tt = sg.t % NT;
            const int nrows = min(BN, T - tt * BN);
            const uint32_t idesc = umma_idesc_bf16_f32(kBM, (nrows + 15) & ~15);
            const int acc = j & 1;
            const uint32_t acc_phase = (uint32_t)(j >> 1) & 1u;
            if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, p.ctl)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d0 = tmem_base + (uint32_t)(acc * C::ACC_COLS);
            for (int kb = sg.k0; kb < sg.k1; ++kb) {
                if (!mbar_wait(smem_u32(&full[stage]), phase, p.ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sa = base + stage * C::STAGE_BYTES;
                const uint32_t sb = sa + C::NUM_A * C::A_BYTES;
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k) {
                    const uint64_t bdesc = umma_desc_sw128(sb + k * 32);
                    const uint32_t accum = (kb > sg.k0 || k > 0) ? 1u : 0u;
                    umma_bf16(d0, umma_desc_sw128(sa + k * 32), bdesc, idesc, accum);
                    if (GATEUP)
                        umma_bf16(d0 + BN, umma_desc_sw128(sa + C::A_BYTES + k * 32), bdesc, idesc, accum);
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
        if (issued_any) {
            umma_commit(smem_u32(drain));
            mbar_wait_drain(smem_u32(drain), 0, p.ctl.limit_ns);
        }
    } else if (warp >= 2) {
        // ------------------------------------------------ epilogue
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const int et = threadIdx.x - 64;             // 0..255 among the epilogue threads
        uint8_t *stg = staging + (warp - 2) * kStagingWarpBytes;
        uint32_t ephase = 0;
        Seg sg;
        for (int j = 0; U > 0 && segment(b, j, U, G, KB, sg); ++j) {
            const int acc = j & 1;
            const uint32_t acc_phase = (uint32_t)(j >> 1) & 1u;
            const bool ok = mbar_wait(smem_u32(&tfull[acc]), acc_phase, p.ctl);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const int wt = sg.t / NT, tt = sg.t - wt * NT;
            const int row0 = tt * BN, nrows = min(BN, T - row0);
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * C::ACC_COLS);
            const int col0 = wt * kBM + quad * 32;
            if (sg.k0 == 0 && sg.k1 == KB) {
                // the whole tile: finish it here
                if constexpr (GATEUP)
                    epilogue_block<kSwiGLU, C::CH, BN>(taddr, nrows, row0, half, lane, stg, p.out + col0, p.R);
                else
                    epilogue_block<kStoreBF16, C::CH, 0>(taddr, nrows, row0, half, lane, stg, p.out + col0, p.R);
                tc_fence_before();
                mbar_arrive(smem_u32(&tempty[acc]));
                continue;
            }
            // a partial K range of tile sg.t, whose pieces belong to CTAs
            // b0 .. b1 in K order.  b0's piece (the tile's first K steps) is
            // the last segment of b0's range, so b0 reaches it last: b0 adds
            // the others' published pieces to its own, still in TMEM.
            const int b0 = unit_owner((long long)sg.t * KB, U, G);
            const int b1 = unit_owner((long long)(sg.t + 1) * KB - 1, U, G);
            if (b != b0) {
                // FP32 sums to this CTA's slot, [token][matrix][128], then publish
                float *slot = part + (size_t)(2 * b + (sg.first ? 0 : 1)) * C::PART;
#pragma unroll 1
                for (int a = 0; a < C::NUM_A; ++a)
                    epilogue_f32_staged(taddr + a * BN, nrows, 0, half, lane, stg, slot + a * kBM + quad * 32,
                                        C::NUM_A * kBM);
                tc_fence_before();
                mbar_arrive(smem_u32(&tempty[acc]));   // TMEM is free again
                __threadfence();
                if (!__all_sync(0xffffffffu, epi_sync(epi_bar, ephase, p.ctl))) break;
                if (et == 0) atomicAdd(&cnt[sg.t], 1);
                continue;
            }
            // b0: wait (bounded) until the b1 - b0 other pieces are published
            if (et == 0) s_last = wait_count(&cnt[sg.t], b1 - b0, p.ctl) ? 1 : 0;
            if (!__all_sync(0xffffffffu, epi_sync(epi_bar, ephase, p.ctl))) break;
            if (!s_last) break;
            __threadfence();
            // Thread (quad, lane) holds weight row r = quad * 32 + lane of its
            // token chunks (CH columns, alternating between the quadrant's two
            // warps): its own sums from TMEM, then the pieces of b0 + 1 ..
            // b1 in order, SG pieces' loads at once.
            const int r = quad * 32 + lane;
            constexpr int CH = C::CH;
            constexpr int SG = GATEUP ? 1 : 2;          // pieces per batch of loads
            constexpr int LDN = C::NUM_A * kBM;         // floats per token row of a slot
#pragma unroll 1
            for (int c0 = half * CH; c0 < nrows; c0 += 2 * CH) {
                float v[C::NUM_A][CH];
#pragma unroll
                for (int a = 0; a < C::NUM_A; ++a) {
                    uint32_t u[CH];
                    tmem_ld<CH>(taddr + a * BN + c0, u);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < CH; ++j) v[a][j] = 0.f + __uint_as_float(u[j]);
                }
#pragma unroll 1
                for (int q0 = b0 + 1; q0 <= b1; q0 += SG) {
                    float ld[SG][C::NUM_A][CH];
#pragma unroll
                    for (int q = 0; q < SG; ++q) {
                        const int cb = q0 + q;
                        const float *src = part + r;
                        if (cb <= b1) {
                            const int ft = (int)(unit_start(cb, U, G) / KB);   // cb's first tile
                            src += (size_t)(2 * cb + (sg.t == ft ? 0 : 1)) * C::PART;
                        }
#pragma unroll
                        for (int a = 0; a < C::NUM_A; ++a)
#pragma unroll
                            for (int j = 0; j < CH; ++j)
                                ld[q][a][j] = (cb <= b1 && c0 + j < nrows)
                                                  ? __ldcg(src + (size_t)(c0 + j) * LDN + a * kBM)
                                                  : 0.f;
                    }
#pragma unroll
                    for (int q = 0; q < SG; ++q) {
                        if (q0 + q > b1) break;
#pragma unroll
                        for (int a = 0; a < C::NUM_A; ++a)
#pragma unroll
                            for (int j = 0; j < CH; ++j) v[a][j] += ld[q][a][j];
                    }
                }
#pragma unroll
                for (int j = 0; j < CH; ++j) {
                    if (c0 + j >= nrows) break;
                    float o;
                    if constexpr (GATEUP) o = silu_f32(v[0][j]) * v[C::NUM_A - 1][j];
                    else o = v[0][j];
                    p.out[(size_t)(row0 + c0 + j) * p.R + wt * kBM + r] = __float2bfloat16_rn(o);
                }
            }
            tc_fence_before();
            mbar_arrive(smem_u32(&tempty[acc]));
            if (et == 0) cnt[sg.t] = 0;   // ready for the next pass
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
template <int BN, bool GATEUP>
cudaError_t set_smem_sk()
{
    return cudaFuncSetAttribute(dense_sk_kernel<BN, GATEUP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SkCfg<BN, GATEUP>::SMEM_BYTES);
}

template <int BN, bool GATEUP>
cudaError_t launch_sk(const CUtensorMap &a0, const CUtensorMap &a1, const BoxMaps &b, const GemmArgs &args,
                      int T, float *part, int *cnt, int grid, cudaStream_t stream)
{
    return launch_pdl(dense_sk_kernel<BN, GATEUP>, dim3(grid), dim3(kThreads), SkCfg<BN, GATEUP>::SMEM_BYTES,
                      stream, a0, a1, b, args, T, part, cnt);
}
}  // namespace

cudaError_t prepare_dense_sk()
{
    cudaError_t e;
    if ((e = set_smem_sk<16, true>()) != cudaSuccess) return e;
    if ((e = set_smem_sk<32, true>()) != cudaSuccess) return e;
    if ((e = set_smem_sk<64, true>()) != cudaSuccess) return e;
    if ((e = set_smem_sk<16, false>()) != cudaSuccess) return e;
    if ((e = set_smem_sk<32, false>()) != cudaSuccess) return e;
    return set_smem_sk<64, false>();
}

size_t dense_sk_part_floats(int BN, bool gate_up, int grid)
{
    return (size_t)2 * grid * BN * (gate_up ? 2 : 1) * gemm::kBM;
}

cudaError_t launch_dense_sk(bool gate_up, int BN, const CUtensorMap &a0, const CUtensorMap &a1,
                            const BoxMaps &b, const GemmArgs &args, int T, float *part, int *cnt, int grid,
                            cudaStream_t stream)
{
    // every CTA needs a non-empty range (an empty one would never arrive)
    const long long U = (long long)(args.R / gemm::kBM) * ((T + BN - 1) / BN) * (args.K / gemm::kBK);
    if (grid > U) grid = (int)U;
    if (grid < 1 || args.R % gemm::kBM != 0 || args.K % gemm::kBK != 0) return cudaErrorInvalidValue;
    switch (BN) {
        case 16: return gate_up ? launch_sk<16, true>(a0, a1, b, args, T, part, cnt, grid, stream)
                                : launch_sk<16, false>(a0, a1, b, args, T, part, cnt, grid, stream);
        case 32: return gate_up ? launch_sk<32, true>(a0, a1, b, args, T, part, cnt, grid, stream)
                                : launch_sk<32, false>(a0, a1, b, args, T, part, cnt, grid, stream);
        case 64: return gate_up ? launch_sk<64, true>(a0, a1, b, args, T, part, cnt, grid, stream)
                                : launch_sk<64, false>(a0, a1, b, args, T, part, cnt, grid, stream);
        default: return cudaErrorInvalidValue;
    }
}

// Failure-detection check of wait_count: one thread polls a counter that
// nothing increments, with the caller's limit; it must give up and record
// kStatusTimeout.
namespace {
__device__ int g_unset_count;   // zero, never written
}

__global__ void count_wait_check_kernel(WaitCtl ctl)
{
    if (threadIdx.x == 0) wait_count(&g_unset_count, 1, ctl);
}

cudaError_t launch_count_wait_check(WaitCtl ctl, cudaStream_t stream)
{
    count_wait_check_kernel<<<1, 32, 0, stream>>>(ctl);
    return cudaGetLastError();
}

}  // namespace beam
