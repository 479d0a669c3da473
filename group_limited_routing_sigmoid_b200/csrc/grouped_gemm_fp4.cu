// Grouped expert GEMMs of the Beam MoE block with NVFP4 expert weights (the
// format is described in fp4.cuh).  Same work items, token tiles and
// epilogue as the single-CTA bf16 kernel (grouped_gemm.cu); what differs is
// the path of a weight tile to the tensor cores:
//
//   warp 0        producer: per stage of KS K steps, bulk copies of KS tiles'
//                 4096 bytes of codes and 512 bytes of block scales each (per
//                 matrix, consecutive in the layout) and the TMA boxes of the
//                 token rows of each step, into a ring in shared memory;
//   warps 6..21   converters, four per TMEM lane quadrant: thread r of the
//                 g-th warp of a quadrant decodes the g-th 16-element block
//                 of weight row r of each K step to f16 (hardware E2M1 -> f16
//                 conversion and one f16 multiply by the block scale: every
//                 product has at most 6 significant bits and lies between
//                 2^-10 and 2688 in magnitude, so it is exact) and writes it
//                 to TMEM lane r with tcgen05.st.  The token rows arrive as
//                 f16 times 2^-8 (the MMA takes A and B of one type): the
//                 dispatch writes x's sorted rows that way, and the gate|up
//                 epilogue writes h that way (the bf16 rounding of h first,
//                 as for bf16 weights).  That is exact for every |x| from
//                 2^-9 up to 65504 x 2^8 and within 2^-17 below that; a
//                 larger value sets the status word (BEAM_ERR_RANGE).  The
//                 epilogue multiplies by 2^8 again;
//   warps 1, 22   MMA issuers (lane 0): A (the decoded weights) from TMEM,
//                 two to four stages deep, B (the token rows) from the
//                 shared-memory stage.  gate|up: warp 1 issues the gate MMAs
//                 and warp 22 the up MMAs; down: warp 1 alone.  At 16-row
//                 token tiles the issuing thread, not the tensor pipe, sets
//                 the pace (an issued MMA of this shape is ~100 cycles of
//                 issue for a few cycles of tensor work), so two issuers cut
//                 the gate|up time by about a tenth; splitting down the same
//                 way was slower.  An issuer waits only for the converters'
//                 arrival: they waited for the raw stage before converting;
//   warps 2..5    epilogue, one per quadrant: as the bf16 kernel, with the
//                 FP32 accumulators first multiplied by the per-tensor scales.
//
// Stages: a pipeline stage holds KS 64-wide K steps (the codes and scales
// of KS consecutive tiles of the layout, the token rows of each step): 2 for
// gate|up; for down 5 when K/64 allows it and the token tile has at most 32
// rows, else 4 when K/64 allows.  Every per-stage cost of the issuing
// threads and the converters (barrier waits, fences, commits) is then paid
// once per 64 KS of K.  At 16-row tiles those costs, not the tensor core,
// set the pace: one wait less per stage took 8% off the decode step, two
// steps per stage 20% more, four for down another 7%.
//
// Accumulator chains: small tiles spread the four K sub-steps of a step over
// CHAINS independent accumulators per matrix, so consecutive MMAs never add
// into the same accumulator; the epilogue adds the chains in chain order in
// FP32.
//
// Why TMEM for A: a decode token tile has 16 rows, so each MMA reads a
// 128 x 16 weight block for a 16 x 16 token block.  Staging the decoded
// weights in shared memory would cost a write and a read of 2 bytes per
// weight there for every 0.5625 bytes fetched from HBM, more than shared
// memory delivers at HBM speed; from TMEM the tensor core reads them
// directly, and shared memory carries only the 4.5-bit ring.  The decode is
// a chain of short dependent steps per element, so many converter warps
// keep the SM sub-partitions busy while each waits on its own steps.  Every
// wait is bounded.
#include "fp4.cuh"
#include "gemm_common.cuh"

namespace beam {

using namespace gemm;

namespace {

constexpr int kFp4EpiWarps = 4;                            // one per TMEM lane quadrant
constexpr int kFp4ConvWarps = 16;                          // four per quadrant, a block each
constexpr int kFp4ConvFirst = 2 + kFp4EpiWarps;            // first converter warp
constexpr int kFp4Issuer2 = kFp4ConvFirst + kFp4ConvWarps;  // warp of the second MMA issuer
constexpr int kFp4Threads = 32 * (kFp4Issuer2 + 1);          // 736
constexpr int kFp4AStagesMax = 4;                          // decoded A stages in TMEM, at most
// 64-wide K steps per pipeline stage: 2 for gate|up (what TMEM holds with two
// accumulator buffers), 4 for down when K allows
constexpr int kFp4Ch = 16;                                 // epilogue columns per chunk
constexpr int kFp4MaxRaw = 24;
constexpr int kFp4BarrierBytes = 1024;
constexpr float kFp4TokenScale = 0.00390625f;              // 2^-8: token rows as f16
constexpr float kFp4TokenUnscale = 256.0f;
constexpr int kAColsPerTile = kBK / 2;                     // 64 bf16 of a row: 32 TMEM columns

template <int BN, int NUM_A, int EPI, int KS>
struct Fp4Cfg {
    static constexpr int B_BYTES = BN * kBK * 2;                 // token rows of one K step
    static constexpr int CODES = KS * kFp4CodeTile;           // one matrix's codes per stage
    static constexpr int SCALES = KS * kFp4ScaleTile;
    static constexpr int RAW_USED = KS * B_BYTES + NUM_A * (CODES + SCALES);
    static constexpr int RAW_STAGE = (RAW_USED + 1023) / 1024 * 1024;   // keeps B 1024-aligned
    static constexpr int STAGING = kFp4EpiWarps * kStagingWarpBytes;
    static constexpr int FIXED = 1024 + STAGING + kFp4BarrierBytes + kTableBytes;
    static constexpr int RAW_FIT = (kMaxDynSmem - FIXED) / RAW_STAGE;
    static constexpr int RAW_STAGES = RAW_FIT > kFp4MaxRaw ? kFp4MaxRaw : RAW_FIT;
    static constexpr int CHAINS = BN >= 64 ? 1 : 64 / BN;        // 4 for 16 rows, 2 for 32
    static constexpr int ACC_COLS = CHAINS * NUM_A * BN;         // [chain][matrix][BN]
    static constexpr int A_STAGE_COLS = NUM_A * KS * kAColsPerTile;
    // as many A stages as tensor memory holds beside two accumulator
    // buffers, up to four (two at least: then one accumulator buffer)
    static constexpr int A_STAGES_FIT = (512 - 2 * ACC_COLS) / A_STAGE_COLS;
    static constexpr int A_STAGES =
        A_STAGES_FIT > kFp4AStagesMax ? kFp4AStagesMax : (A_STAGES_FIT < 2 ? 2 : A_STAGES_FIT);
    static constexpr int A_COLS = A_STAGES * A_STAGE_COLS;
    // MMA issuers: gate and up each from their own thread (measured: the
    // gate|up GEMM 10% faster at 16-row tiles); down keeps one (splitting
    // its chains between two threads measured 15% slower)
    static constexpr int ISSUERS = NUM_A == 2 ? 2 : 1;
    static constexpr int NBUF = A_COLS + 2 * ACC_COLS <= 512 ? 2 : 1;
    static constexpr int TMEM_COLS = pow2_at_least(A_COLS + NBUF * ACC_COLS, 32);
    static constexpr int SMEM_BYTES = FIXED + RAW_STAGES * RAW_STAGE;
    static_assert(RAW_STAGES >= 2, "raw ring needs two stages");
    static_assert(SMEM_BYTES <= kMaxDynSmem, "shared memory");
    static_assert(TMEM_COLS <= 512, "TMEM holds 512 columns");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 128, "token tiles of 16..128 rows");
    static_assert(EPI != kSwiGLU || NUM_A == 2, "SwiGLU needs the gate and up tiles");
    static_assert(EPI == kSwiGLU || NUM_A == 1, "one matrix for the store epilogues");
    static_assert(EPI == kSwiGLU || EPI == kStoreBF16 || EPI == kStoreF32, "fp4 epilogues");
    static_assert(32 * kFp4Ch * 4 <= kStagingWarpBytes, "staging block (FP32)");
    static_assert((2 * kFp4MaxRaw + 2 * kFp4AStagesMax + 6) * 8 + 4 <= kFp4BarrierBytes, "barriers");
    static_assert(KS * B_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "token tiles 1024-aligned");
    static_assert(32 * kFp4Ch * 2 <= kStagingWarpBytes, "staging block");
    static_assert(kFp4ConvWarps == 4 * (kFp4TileK / 16), "a converter warp per quadrant and block");
    static_assert(CHAINS <= kBK / 16, "a chain per K sub-step at most");
};

// One bulk copy global -> shared completing on a local mbarrier.  Both
// addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T: A is 128 TMEM lanes (one weight row
// each) by 8 columns (16 bf16 along K, element 2c in the low half of
// column c).
__device__ __forceinline__ void umma_bf16_tmem_a(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                                 uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Warp-wide: thread i writes 8 consecutive 32-bit columns of TMEM lane
// (taddr.lane + i).
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&v)[8])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(
                     taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_st_wait()
{
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void ring_step(int &s, uint32_t &ph, int n)
{
    if (++s == n) {
        s = 0;
        ph ^= 1u;
    }
}

// Sum of the CHAINS partial accumulators of one matrix (columns `stride`
// apart) over CH columns, in chain order, in FP32.
template <int CH, int CHAINS>
__device__ __forceinline__ void load_chains(uint32_t taddr, int stride, float (&acc)[CH])
{
    uint32_t v[CH];
    tmem_ld<CH>(taddr, v);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < CH; ++j) acc[j] = __uint_as_float(v[j]);
#pragma unroll 1
    for (int c = 1; c < CHAINS; ++c) {
        tmem_ld<CH>(taddr + c * stride, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < CH; ++j) acc[j] += __uint_as_float(v[j]);
    }
}

// The bf16 kernel's epilogue with per-tensor scales on the FP32
// accumulators: SwiGLU of (gate x sa, up x sb), or the value x sa; one warp
// per lane quadrant takes every chunk of CH columns.  The up accumulator is
// UP_OFFSET columns after the gate's; chain c of either CHAIN_STRIDE x c.
// SwiGLU writes h as the down GEMM's operand: f16 of bf16(h) x 2^-8, and
// BEAM_ERR_RANGE in the status word if a stored value is beyond f16 range.
template <int EPI, int CH, int UP_OFFSET, int CHAINS, int CHAIN_STRIDE>
__device__ __forceinline__ void fp4_epilogue_block(uint32_t taddr, int nrows, int row0, int lane,
                                                   uint8_t *stg, __nv_bfloat16 *out, int ldo,
                                                   float sa, float sb, int *status)
{
    bool fits = true;
    constexpr int VPR = 4;   // 16-byte vectors per 32 bf16
#pragma unroll 1
    for (int c0 = 0; c0 < nrows; c0 += CH) {
        float g[CH];
        load_chains<CH, CHAINS>(taddr + c0, CHAIN_STRIDE, g);
        __nv_bfloat16 *sh = reinterpret_cast<__nv_bfloat16 *>(stg);
        if constexpr (EPI == kSwiGLU) {
            float u[CH];
            load_chains<CH, CHAINS>(taddr + UP_OFFSET + c0, CHAIN_STRIDE, u);
            unsigned short *shu = reinterpret_cast<unsigned short *>(sh);
#pragma unroll
            for (int j = 0; j < CH; ++j) {
                const float hv = __bfloat162float(__float2bfloat16_rn(silu_f32(g[j] * sa) * (u[j] * sb))) * kFp4TokenScale;
                if (c0 + j < nrows && fabsf(hv) > 65504.0f) fits = false;
                shu[j * 32 + lane] = __half_as_ushort(__float2half_rn(hv));
            }
        } else {
#pragma unroll
            for (int j = 0; j < CH; ++j) sh[j * 32 + lane] = __float2bfloat16_rn(g[j] * sa);
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
    if (!fits) record_status(status, kStatusRange);
}

// FP32 outputs: the chains' sum times sa, 16 token rows at a time through
// the warp's staging block, each row's 32 columns (this warp's output
// columns) stored as 16-byte vectors.
template <int CH, int CHAINS, int CHAIN_STRIDE>
__device__ __forceinline__ void fp4_epilogue_f32(uint32_t taddr, int nrows, int row0, int lane,
                                                 uint8_t *stg, float *out, int ldo, float sa)
{
    float *sh = reinterpret_cast<float *>(stg);   // [CH token rows][32 columns]
#pragma unroll 1
    for (int c0 = 0; c0 < nrows; c0 += CH) {
        float g[CH];
        load_chains<CH, CHAINS>(taddr + c0, CHAIN_STRIDE, g);
#pragma unroll
        for (int j = 0; j < CH; ++j) sh[j * 32 + lane] = g[j] * sa;
        __syncwarp();
#pragma unroll
        for (int w = lane; w < CH * 8; w += 32) {
            const int j = w >> 3, part = w & 7;
            if (c0 + j < nrows) {
                const float4 val = *reinterpret_cast<const float4 *>(sh + j * 32 + part * 4);
                *reinterpret_cast<float4 *>(out + (size_t)(row0 + c0 + j) * ldo + part * 4) = val;
            }
        }
        __syncwarp();
    }
}

// E4M3 value from the format's definition (exact in float): sign, 4-bit
// exponent with bias 7, 3-bit mantissa; exponent 0 is subnormal; S.1111.111
// is NaN.
__device__ __forceinline__ float e4m3_float(uint32_t byte)
{
    const uint32_t e = (byte >> 3) & 15u, m = byte & 7u;
    float v;
    if (e == 15u && m == 7u) v = __int_as_float(0x7fc00000);
    else if (e == 0u) v = ldexpf((float)m * 0.125f, -6);
    else v = ldexpf(1.0f + (float)m * 0.125f, (int)e - 7);
    return (byte & 0x80u) ? -v : v;
}

// The bf16 encoding of (E4M3 value x 2^112): finite for every E4M3 value
// (at most 448 x 2^112 < 2^121) and normal (at least 2^-9 x 2^112).
__device__ __forceinline__ uint32_t fp4_scale_bits(uint32_t byte)
{
    return __bfloat16_as_ushort(__float2bfloat16_rn(ldexpf(e4m3_float(byte), 112)));
}

// Four code bytes (eight E2M1 elements, element 2j in the low nibble of byte
// j) times one block scale, as four bf16x2 words (element 2j in the low
// half).  The hardware converts a byte to two f16 values; an f16 value
// shifted right by three bits, sign kept in place, is the bf16 encoding of
// the same value times 2^-112 (the exponent bias goes from 15 to 127, the
// mantissa from 10 to 7 bits; E2M1 values have one mantissa bit, so nothing
// is lost); the multiply by bf16(scale x 2^112) restores the magnitude and
// is exact, since the product of an E2M1 and an E4M3 value has at most 6
// significant bits.
__device__ __forceinline__ void fp4_decode4(uint32_t codes, uint32_t scale_bits, uint32_t (&o)[4])
{
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(codes));
    const uint32_t s2u = scale_bits | (scale_bits << 16);
    const __nv_bfloat162 s2 = *reinterpret_cast<const __nv_bfloat162 *>(&s2u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t r = ((h[i] >> 3) & 0x0FFF0FFFu) | (h[i] & 0x80008000u);
        const __nv_bfloat162 prod = __hmul2(*reinterpret_cast<const __nv_bfloat162 *>(&r), s2);
        o[i] = *reinterpret_cast<const uint32_t *>(&prod);
    }
}


// Four code bytes (eight E2M1 elements, element 2j in the low nibble of byte
// j) times one block scale, as four f16x2 words (element 2j in the low
// half): the hardware converts a byte to two f16 values, one f16 multiply by
// the scale (both halves of `scale2`) gives the exact product.
__device__ __forceinline__ void fp4_decode4_f16(uint32_t codes, uint32_t scale2, uint32_t (&o)[4])
{
    uint32_t h[4];
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(codes));
#pragma unroll
    for (int i = 0; i < 4; ++i) asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(o[i]) : "r"(h[i]), "r"(scale2));
}

}  // namespace

template <int BN, int NUM_A, int EPI, int KS>
__global__ void __launch_bounds__(kFp4Threads, 1)
    grouped_gemm_fp4_kernel(const __grid_constant__ BoxMaps tmB, const Fp4Operands w, GemmArgs p)
{
    using C = Fp4Cfg<BN, NUM_A, EPI, KS>;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    uint8_t *base_ptr = smem_raw + (base - raw_addr);
    uint8_t *staging = base_ptr + C::RAW_STAGES * C::RAW_STAGE;
    uint64_t *rfull = reinterpret_cast<uint64_t *>(staging + C::STAGING);
    uint64_t *rempty = rfull + kFp4MaxRaw;
    uint64_t *cfull = rempty + kFp4MaxRaw;
    uint64_t *cempty = cfull + kFp4AStagesMax;
    uint64_t *tfull = cempty + kFp4AStagesMax;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;                                          // one per issuer
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 2);
    int *s_counts = reinterpret_cast<int *>(staging + C::STAGING + kFp4BarrierBytes);
    int *s_offsets = s_counts + p.E;
    int *s_tile = s_offsets + (p.E + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const bool converter = warp >= kFp4ConvFirst && warp < kFp4Issuer2;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < C::RAW_STAGES; ++s) {
            mbar_init(smem_u32(&rfull[s]), 1);
            mbar_init(smem_u32(&rempty[s]), C::ISSUERS);   // a commit from each issuer
        }
        for (int s = 0; s < C::A_STAGES; ++s) {
            mbar_init(smem_u32(&cfull[s]), kFp4ConvWarps);   // one elected lane per warp
            mbar_init(smem_u32(&cempty[s]), C::ISSUERS);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&tfull[a]), C::ISSUERS);
            mbar_init(smem_u32(&tempty[a]), 32 * kFp4EpiWarps);
        }
        mbar_init(smem_u32(&drain[0]), 1);
        mbar_init(smem_u32(&drain[1]), 1);
        fence_barrier_init();
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

    const int WT = p.R / kBM;
    // no work while the status word is set (a failed check or wait)
    const int total = status_is_set(p.ctl.status) ? 0 : WT * s_tile[p.E];
    // stages of KS K steps (hidden and inter are multiples of 128)
    const int KB = p.K / (kBK * KS);

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ producer
            const uint64_t pol_w = l2_policy_evict_first();   // weights: streamed
            const uint64_t pol_x = l2_policy_evict_last();    // token rows: reused across tiles
            int rs = 0;
            uint32_t rp = 0;
            long long issued = 0;
            bool ok = true;
            for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
                const Item it = decode_item(item, WT, p.E, s_counts, s_offsets, s_tile);
                const size_t rt = (size_t)it.e * w.row_tiles + it.wt;
                const int n_load = (it.nrows + 15) & ~15;
                const uint32_t bytes = NUM_A * (C::CODES + C::SCALES) +
                                       (uint32_t)(KS * n_load * (kBK * 2));
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait(smem_u32(&rempty[rs]), rp ^ 1u, p.ctl)) {
                        ok = false;
                        break;
                    }
                    const uint32_t dst = base + (uint32_t)(rs * C::RAW_STAGE);
                    const uint32_t fb = smem_u32(&rfull[rs]);
                    mbar_arrive_expect_tx(fb, bytes);
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        int off = 0;
#pragma unroll
                        for (int bi = 4; bi >= 1; --bi) {   // token rows: boxes of 128, 64, 32, 16 rows
                            const int hgt = 8 << bi;
                            if (hgt <= BN && n_load - off >= hgt) {
                                tma_load_2d(dst + ks * C::B_BYTES + off * (kBK * 2), &tmB.m[bi],
                                            (kb * KS + ks) * kBK, it.row0 + off, fb, pol_x);
                                off += hgt;
                            }
                        }
                    }
                    // the stage's K steps are consecutive tiles of the layout
                    const size_t tile = rt * (size_t)w.k_steps + (size_t)kb * KS;
#pragma unroll
                    for (int a = 0; a < NUM_A; ++a) {
                        bulk_load(dst + KS * C::B_BYTES + a * C::CODES,
                                  w.a[a].codes + tile * kFp4CodeTile, C::CODES, fb, pol_w);
                        bulk_load(dst + KS * C::B_BYTES + NUM_A * C::CODES + a * C::SCALES,
                                  w.a[a].scales + tile * kFp4ScaleTile, C::SCALES, fb, pol_w);
                    }
                    ++issued;
                    ring_step(rs, rp, C::RAW_STAGES);
                }
            }
            if (!ok) {
                // copies in flight land before the CTA leaves (time-bounded)
                const long long m = issued < C::RAW_STAGES ? issued : C::RAW_STAGES;
                int s = rs;
                uint32_t ph = rp;
                for (long long j = 0; j < m; ++j) {
                    if (s == 0) {
                        s = C::RAW_STAGES - 1;
                        ph ^= 1u;
                    } else {
                        --s;
                    }
                    mbar_wait_drain(smem_u32(&rfull[s]), ph, p.ctl.limit_ns);
                }
            }
        }
    } else if (converter) {
        // ------------------------------------------------ converters
        const int quad = warp & 3;                     // the TMEM lanes this warp may access
        const int blk = (warp - kFp4ConvFirst) >> 2;   // its 16-element block of the K step
        const int r = quad * 32 + lane;                // weight row of the tile = TMEM lane
        const uint32_t lane_base = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(blk * 8);
        int rs = 0, cs = 0;
        uint32_t rp = 0, cp = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x) {
            for (int kb = 0; kb < KB; ++kb) {
                const bool got = mbar_wait(smem_u32(&rfull[rs]), rp, p.ctl) &&
                                 mbar_wait(smem_u32(&cempty[cs]), cp ^ 1u, p.ctl);
                ok = __all_sync(0xffffffffu, got);
                if (!ok) break;
                tc_fence_after();
                const uint8_t *raw = base_ptr + rs * C::RAW_STAGE + KS * C::B_BYTES;
#pragma unroll
                for (int a = 0; a < NUM_A; ++a)
#pragma unroll
                    for (int ks = 0; ks < KS; ++ks) {
                        // this block of row r in K step ks: 8 code bytes and one scale byte
                        const uint2 c = *reinterpret_cast<const uint2 *>(
                            raw + a * C::CODES + ks * kFp4CodeTile + blk * (kFp4TileRows * 8) + r * 8);
                        // the scale byte in both halves, widened to f16x2 by
                        // the hardware (exact: every E4M3 value is a normal f16)
                        const uint32_t sbyte = raw[NUM_A * C::CODES + a * C::SCALES +
                                                   ks * kFp4ScaleTile + blk * kFp4TileRows + r];
                        const unsigned short pair = (unsigned short)(sbyte | (sbyte << 8));
                        uint32_t s2;
                        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(s2) : "h"(pair));
                        uint32_t lo[4], hi[4];
                        fp4_decode4_f16(c.x, s2, lo);
                        fp4_decode4_f16(c.y, s2, hi);
                        const uint32_t v[8] = {lo[0], lo[1], lo[2], lo[3], hi[0], hi[1], hi[2], hi[3]};
                        tmem_st8(lane_base + (uint32_t)(cs * C::A_STAGE_COLS + (a * KS + ks) * kAColsPerTile), v);
                    }
                // every lane's stores complete, then one arrival for the
                // warp (512 same-address arrivals a stage would serialise)
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&cfull[cs]));
                ring_step(rs, rp, C::RAW_STAGES);
                ring_step(cs, cp, C::A_STAGES);
            }
        }
    } else if ((warp == 1 || (warp == kFp4Issuer2 && C::ISSUERS == 2)) && lane == 0) {
        // ------------------------------------------------ UMMA issuers
        // issuer mi: matrix mi of gate|up, or the chains of parity mi of down
        const int mi = warp == 1 ? 0 : 1;
        int rs = 0, cs = 0;
        uint32_t rp = 0, cp = 0;
        bool ok = true;
        bool issued_any = false;
        int iter = 0;
        for (int item = blockIdx.x; item < total && ok; item += gridDim.x, ++iter) {
            const Item it = decode_item(item, WT, p.E, s_counts, s_offsets, s_tile);
            const int n_mma = (it.nrows + 15) & ~15;
            const uint32_t idesc = umma_idesc_f16_f32(kBM, n_mma);
            const int acc = iter % C::NBUF;
            const uint32_t acc_phase = (uint32_t)(iter / C::NBUF) & 1u;
            if (!mbar_wait(smem_u32(&tempty[acc]), acc_phase ^ 1u, p.ctl)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d0 = tmem_base + (uint32_t)(C::A_COLS + acc * C::ACC_COLS);
            for (int kb = 0; kb < KB; ++kb) {
                // the converters' arrival implies the stage's raw data landed
                // (they waited for it) and its token rows are converted: no
                // wait on the raw ring here (one wait less per stage measured
                // 8% off the step: the issuing thread sets the pace)
                if (!mbar_wait(smem_u32(&cfull[cs]), cp, p.ctl)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t a0 = tmem_base + (uint32_t)(cs * C::A_STAGE_COLS);
                const uint32_t b_addr = base + (uint32_t)(rs * C::RAW_STAGE);
#pragma unroll
                for (int ks = 0; ks < KS; ++ks)
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k) {
                        // K sub-step k of step ks adds into chain k % CHAINS, first
                        // written in the first stage's first step
                        const int chain = k % C::CHAINS;
                        if (NUM_A == 1 && C::ISSUERS == 2 && (chain & 1) != mi) continue;
                        const int a = NUM_A == 2 ? mi : 0;
                        const uint32_t d = d0 + (uint32_t)((chain * NUM_A + a) * BN);
                        const uint64_t bdesc = umma_desc_sw128(b_addr + ks * C::B_BYTES + k * 32);
                        const uint32_t accum = (kb > 0 || ks > 0 || k >= C::CHAINS) ? 1u : 0u;
                        umma_bf16_tmem_a(d, a0 + (a * KS + ks) * kAColsPerTile + k * 8, bdesc, idesc,
                                         accum);
                        issued_any = true;
                    }
                umma_commit(smem_u32(&rempty[rs]));
                umma_commit(smem_u32(&cempty[cs]));
                ring_step(rs, rp, C::RAW_STAGES);
                ring_step(cs, cp, C::A_STAGES);
            }
            if (!ok) break;
            umma_commit(smem_u32(&tfull[acc]));
        }
        // every MMA issued completes before TMEM is released
        if (issued_any) {
            umma_commit(smem_u32(&drain[mi]));
            mbar_wait_drain(smem_u32(&drain[mi]), 0, p.ctl.limit_ns);
        }
    } else if (warp >= 2 && warp < 2 + kFp4EpiWarps) {
        // ------------------------------------------------ epilogue
        const int quad = warp & 3;
        uint8_t *stg = staging + (warp - 2) * kStagingWarpBytes;
        int iter = 0;
        for (int item = blockIdx.x; item < total; item += gridDim.x, ++iter) {
            const int acc = iter % C::NBUF;
            const uint32_t acc_phase = (uint32_t)(iter / C::NBUF) & 1u;
            const bool ok = mbar_wait(smem_u32(&tfull[acc]), acc_phase, p.ctl);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            const Item it = decode_item(item, WT, p.E, s_counts, s_offsets, s_tile);
            const uint32_t taddr = tmem_base + ((uint32_t)(quad * 32) << 16) +
                                   (uint32_t)(C::A_COLS + acc * C::ACC_COLS);
            const int col0 = it.wt * kBM + quad * 32;
            if constexpr (EPI == kSwiGLU)
                fp4_epilogue_block<EPI, kFp4Ch, BN, C::CHAINS, NUM_A * BN>(
                    taddr, it.nrows, it.row0, lane, stg, p.out + col0, p.R,
                    w.a[0].global * kFp4TokenUnscale, w.a[1].global * kFp4TokenUnscale, p.ctl.status);
            else if constexpr (EPI == kStoreF32)
                fp4_epilogue_f32<kFp4Ch, C::CHAINS, NUM_A * BN>(
                    taddr, it.nrows, it.row0, lane, stg, p.out_f32 + col0, p.R,
                    w.a[0].global * kFp4TokenUnscale);
            else
                fp4_epilogue_block<EPI, kFp4Ch, 0, C::CHAINS, NUM_A * BN>(
                    taddr, it.nrows, it.row0, lane, stg, p.out + col0, p.R,
                    w.a[0].global * kFp4TokenUnscale, 1.0f, p.ctl.status);
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

// Row-major NVFP4 (codes [rows][K/2], scales [rows][K/16]) -> tiled layout
// (fp4.cuh): a block per (128-row tile, K step), a thread per row.
__global__ void __launch_bounds__(128) fp4_repack_kernel(const uint8_t *__restrict__ codes,
                                                         const uint8_t *__restrict__ scales,
                                                         int K, int k_steps,
                                                         uint8_t *__restrict__ codes_t,
                                                         uint8_t *__restrict__ scales_t)
{
    const size_t tile = blockIdx.x;             // rt * k_steps + kb
    const size_t rt = tile / k_steps, kb = tile - rt * k_steps;
    const int r = threadIdx.x;
    const size_t row = rt * kFp4TileRows + r;
    const uint2 *src = reinterpret_cast<const uint2 *>(codes + row * (size_t)(K / 2) + kb * 32);
    const uint8_t *ssrc = scales + row * (size_t)(K / 16) + kb * 4;
#pragma unroll
    for (int b = 0; b < kFp4TileK / 16; ++b) {   // block b of the row -> plane b of the tile
        *reinterpret_cast<uint2 *>(codes_t + tile * kFp4CodeTile + b * (kFp4TileRows * 8) + r * 8) = src[b];
        scales_t[tile * kFp4ScaleTile + b * kFp4TileRows + r] = ssrc[b];
    }
}

// Row-major NVFP4 -> bf16 products (element x block scale): a thread per
// 16-element block, through the converters' decode.
__global__ void __launch_bounds__(256) fp4_dequant_kernel(const uint8_t *__restrict__ codes,
                                                          const uint8_t *__restrict__ scales,
                                                          long long blocks,
                                                          __nv_bfloat16 *__restrict__ out)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= blocks) return;
    const uint2 c = *reinterpret_cast<const uint2 *>(codes + i * 8);
    const uint32_t sb = fp4_scale_bits(scales[i]);
    uint32_t lo[4], hi[4];
    fp4_decode4(c.x, sb, lo);
    fp4_decode4(c.y, sb, hi);
    uint4 *dst = reinterpret_cast<uint4 *>(out + i * 16);
    dst[0] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    dst[1] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
}

namespace {
template <int BN, int NUM_A, int EPI, int KS>
cudaError_t set_smem_fp4()
{
    return cudaFuncSetAttribute(grouped_gemm_fp4_kernel<BN, NUM_A, EPI, KS>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Fp4Cfg<BN, NUM_A, EPI, KS>::SMEM_BYTES);
}

template <int BN, int EPI, int KS>
cudaError_t launch_fp4_down(const Fp4Operands &w, const BoxMaps &b, const GemmArgs &args, int grid,
                            cudaStream_t stream)
{
    return launch_pdl(grouped_gemm_fp4_kernel<BN, 1, EPI, KS>, dim3(grid), dim3(kFp4Threads),
                      Fp4Cfg<BN, 1, EPI, KS>::SMEM_BYTES, stream, b, w, args);
}

template <int BN>
cudaError_t launch_fp4_kind(GemmKind kind, const Fp4Operands &w, const BoxMaps &b,
                            const GemmArgs &args, int grid, cudaStream_t stream)
{
    if (kind == GemmKind::kGateUp)
        return launch_pdl(grouped_gemm_fp4_kernel<BN, 2, kSwiGLU, 2>, dim3(grid), dim3(kFp4Threads),
                          Fp4Cfg<BN, 2, kSwiGLU, 2>::SMEM_BYTES, stream, b, w, args);
    // down: five K steps per stage when K is a multiple of 320 and the token
    // tile has at most 32 rows (two raw stages of five steps then fit in
    // shared memory), else four when K is a multiple of 256
    if constexpr (BN <= 32) {
        if (args.K % (5 * kBK) == 0) {
            if (kind == GemmKind::kDown) return launch_fp4_down<BN, kStoreBF16, 5>(w, b, args, grid, stream);
            if (kind == GemmKind::kDownF32 && args.out_f32 != nullptr)
                return launch_fp4_down<BN, kStoreF32, 5>(w, b, args, grid, stream);
        }
    }
    const bool ks4 = args.K % (4 * kBK) == 0;
    if (kind == GemmKind::kDown)
        return ks4 ? launch_fp4_down<BN, kStoreBF16, 4>(w, b, args, grid, stream)
                   : launch_fp4_down<BN, kStoreBF16, 2>(w, b, args, grid, stream);
    if (kind == GemmKind::kDownF32 && args.out_f32 != nullptr)
        return ks4 ? launch_fp4_down<BN, kStoreF32, 4>(w, b, args, grid, stream)
                   : launch_fp4_down<BN, kStoreF32, 2>(w, b, args, grid, stream);
    return cudaErrorInvalidValue;
}
}  // namespace

cudaError_t prepare_grouped_gemm_fp4()
{
    cudaError_t err;
#define BEAM_PREP_FP4(BN)                                                       \
    if ((err = set_smem_fp4<BN, 2, kSwiGLU, 2>()) != cudaSuccess) return err;   \
    if ((err = set_smem_fp4<BN, 1, kStoreBF16, 2>()) != cudaSuccess) return err; \
    if ((err = set_smem_fp4<BN, 1, kStoreF32, 2>()) != cudaSuccess) return err;  \
    if ((err = set_smem_fp4<BN, 1, kStoreBF16, 4>()) != cudaSuccess) return err; \
    if ((err = set_smem_fp4<BN, 1, kStoreF32, 4>()) != cudaSuccess) return err;
    if ((err = set_smem_fp4<16, 1, kStoreBF16, 5>()) != cudaSuccess) return err;
    if ((err = set_smem_fp4<16, 1, kStoreF32, 5>()) != cudaSuccess) return err;
    if ((err = set_smem_fp4<32, 1, kStoreBF16, 5>()) != cudaSuccess) return err;
    if ((err = set_smem_fp4<32, 1, kStoreF32, 5>()) != cudaSuccess) return err;
    BEAM_PREP_FP4(16)
    BEAM_PREP_FP4(32)
    BEAM_PREP_FP4(64)
    BEAM_PREP_FP4(128)
#undef BEAM_PREP_FP4
    return cudaSuccess;
}

cudaError_t launch_grouped_gemm_fp4(GemmKind kind, int BN, const Fp4Operands &w,
                                    const BoxMaps &b, const GemmArgs &args, int grid,
                                    cudaStream_t stream)
{
    switch (BN) {
        case 16: return launch_fp4_kind<16>(kind, w, b, args, grid, stream);
        case 32: return launch_fp4_kind<32>(kind, w, b, args, grid, stream);
        case 64: return launch_fp4_kind<64>(kind, w, b, args, grid, stream);
        case 128: return launch_fp4_kind<128>(kind, w, b, args, grid, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_fp4_repack(const uint8_t *codes, const uint8_t *scales, long long rows, int K,
                              uint8_t *codes_t, uint8_t *scales_t, cudaStream_t stream)
{
    if (rows % kFp4TileRows != 0 || K % kFp4TileK != 0) return cudaErrorInvalidValue;
    const long long k_steps = K / kFp4TileK;
    const long long blocks = rows / kFp4TileRows * k_steps;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (blocks == 0) return cudaSuccess;
    fp4_repack_kernel<<<(unsigned)blocks, kFp4TileRows, 0, stream>>>(codes, scales, K, (int)k_steps,
                                                                     codes_t, scales_t);
    return cudaGetLastError();
}

cudaError_t launch_fp4_dequant(const uint8_t *codes, const uint8_t *scales, long long elements,
                               __nv_bfloat16 *out, cudaStream_t stream)
{
    if (elements % 16 != 0) return cudaErrorInvalidValue;
    const long long blocks = elements / 16;
    const long long grid = (blocks + 255) / 256;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (blocks == 0) return cudaSuccess;
    fp4_dequant_kernel<<<(unsigned)grid, 256, 0, stream>>>(codes, scales, blocks, out);
    return cudaGetLastError();
}

}  // namespace beam
