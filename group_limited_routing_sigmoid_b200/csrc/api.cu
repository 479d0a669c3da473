// C ABI of the Beam MoE block (declared in include/beam_moe.h): argument
// validation, workspace, TMA descriptors, and the stream-ordered launch
// sequence router -> dispatch -> gate|up GEMM -> down GEMM -> combine.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "beam_moe.h"
#include "fp4.cuh"
#include "kernels.cuh"

namespace beam {
// The dense stream-K GEMMs' wait on a global counter, checked the same way
// (defined in dense_sk.cu beside the wait).
cudaError_t launch_count_wait_check(WaitCtl ctl, cudaStream_t stream);
}  // namespace beam

using namespace beam;

struct beam_moe {
    int H, E, I, n_group, topk_group, top_k;
    float scaling;
    const float *router_w, *bias, *gamma;
    const __nv_bfloat16 *w_gate, *w_up, *w_down;
    float eps;
    int max_tokens;
    int device, num_sms;
    int gemm_ctas;           // 0: num_sms
    long long wait_limit_ns;

    void *ws;
    size_t ws_bytes;
    int dense;               // 1: dense SwiGLU MLP (one expert, no router)
    int fp4;                 // 1: NVFP4 expert weights
    // NVFP4: the caller's row-major tensors (read at create only), the
    // tiled copy the GEMMs stream (owned), and its operand sets
    const uint8_t *fp4_codes_in[3], *fp4_scales_in[3];
    float fp4_global[3];
    uint8_t *fp4_buf;
    Fp4Operands fp4_gate_up, fp4_down;
    float *partial;          // [nslice_max * T_max * E]
    float *sk_part;          // dense layers: stream-K slots, two per CTA
    int *sk_cnt;             // dense layers: stream-K arrival counter per tile
    int sk_cnt_n;
    int32_t *idx;            // [P]
    float *w;                // [P]
    int32_t *block_cnt, *block_base, *rank, *counts, *offsets, *tile_off, *pair_row, *row_pair;
    __nv_bfloat16 *xp;       // [P, H]
    __nv_bfloat16 *hbuf;     // [P, I]
    __nv_bfloat16 *ybuf;     // [P, H] bf16 expert outputs, or
    float *y32;              // [P, H] FP32 expert outputs (same memory; sparse blocks)
    int *status;             // device status word
    // host-buffer path: two staging slots, so one call's copies overlap the
    // neighbouring calls' compute; a copy-in and a copy-out stream; per slot
    // the events copy-in done, compute done, copy-out done
    __nv_bfloat16 *x_stage[2], *out_stage[2];
    float *res_stage[2];
    cudaStream_t copy_in, copy_out;
    cudaEvent_t ev_in[2], ev_comp[2], ev_out[2];
    cudaEvent_t ev_fence;            // host_fence: the caller's stream position
    int host_slot;

    CUtensorMap tm_gate, tm_up, tm_down;
    CUtensorMap tm_gate16, tm_up16;  // the same with 16-row boxes (interleaved gate|up tiles)
    CUtensorMap tm_wcat;             // router weight as three bf16 pieces [E, 3H]
    __nv_bfloat16 *wcat;
    int router_mode;                 // -1: auto, 0: FP32 SIMT, 1: tensor cores, 2: 1 + every token re-derived
    int *fix_list;                   // [max_tokens] tokens re-derived on the exact path
    int *fix_count;
    BoxMaps tm_xp, tm_h;             // box rows 8, 16, 32, 64, 128, 256
    BoxMaps tm_x;                    // dense layers: boxes of the caller's x ...
    const void *tm_x_ptr;            // ... for this pointer and token count
    int tm_x_T;
    int tile_rows;                   // 0: chosen from T
    int down_pair;                   // -1: auto, 0: single tiles, 1: paired tiles
    int use_pair;                    // 1: CTA-pair kernels for large token tiles (default)
    int gather_rows;                 // -1: auto (default), 0: never, 1: always
    int y_mode;                      // 1: FP32 expert outputs y (default), 0: bf16 y
    int gu_layout;                   // -1: auto, 0: separate gate and up tiles, 1: interleaved
    int token_stages;                // CTA-pair kernels: token-row ring depth (0: default)
    int checks;                      // 1: validate routing and dispatch tables on the device
    int corrupt_next;                // test hook: forward passes left whose routing is corrupted
    int *check_where;                // device: first index a check failed at
    int last_T;
    std::vector<cudaEvent_t> prof_events;   // 6 per profiled forward pass
    int prof_max, prof_calls;
    char err[512];
};

namespace {

thread_local char g_create_err[512] = "";   // per calling thread

int fail(beam_moe *h, int code, const char *fmt, ...)
{
    char *dst = h ? h->err : g_create_err;
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(dst, 512, fmt, ap);
    va_end(ap);
    return code;
}

int cuda_fail(beam_moe *h, cudaError_t e, const char *what)
{
    return fail(h, BEAM_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D bf16 tensor [rows, cols] row-major, box {64 cols, box_rows}, 128B swizzle.
bool make_map(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t es[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Largest token tile of the GEMMs from the mean load per expert (the host
// never reads the routing, so the choice depends on T only).
int choose_tile_rows(int T, int top_k, int E)
{
    const double mean = (double)T * top_k / E;
    if (mean <= 24) return 16;
    if (mean <= 48) return 32;
    if (mean <= 96) return 64;
    if (mean <= 160) return 128;
    return 256;
}

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int check_device(beam_moe *h)
{
    int cur = -1;
    cudaError_t e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return cuda_fail(h, e, "cudaGetDevice");
    if (cur != h->device)
        return fail(h, BEAM_ERR_INVALID_ARG, "current device %d is not the handle's device %d", cur,
                    h->device);
    return BEAM_OK;
}

// Tensor-core router slices: the fewest K slices (dividing the 3H/64 steps,
// each at least 16 steps) that give two work items per SM.
int router_mma_slices(int T, int H, int E, int num_sms)
{
    const int items = ((E + router_mma_experts_per_tile() - 1) / router_mma_experts_per_tile()) *
                      ((T + router_mma_tokens_per_tile() - 1) / router_mma_tokens_per_tile());
    // K slices of H (each at least 16 steps of 64): the fewest that minimise
    // the busiest SM's K steps, (waves of items) x (steps per item)
    const int kb = H / 64;
    int best = 1;
    long long best_cost = 0;
    for (int d = 1; d <= kb / 16 || d == 1; ++d) {
        if (kb % d) continue;
        const long long waves = ((long long)items * d + num_sms - 1) / num_sms;
        const long long cost = waves * (kb / d);
        if (d == 1 || cost < best_cost) {
            best = d;
            best_cost = cost;
        }
    }
    return best;
}

bool router_on_tensor_cores(const beam_moe *h, int T)
{
    if (h->router_mode >= 0) return h->router_mode >= 1;
    return T >= 512;
}

// Decision margin below which a token's routing is re-derived from FP32
// CUDA-core logits: the tensor-core logits' accumulation error stays below
// 4e-5 (logit units, measured against exact sums at 320-step chains), i.e.
// below 1e-5 in sigmoid-score units; 4e-5 leaves a factor of four.
constexpr float kRouterMargin = 4e-5f;

int run_router(beam_moe *h, cudaStream_t s, const void *x, int T, int32_t *idx, float *w,
               float *logits)
{
    RouterArgs a;
    a.x = static_cast<const __nv_bfloat16 *>(x);
    a.router_w = h->router_w;
    a.bias = h->bias;
    a.T = T;
    a.H = h->H;
    a.E = h->E;
    a.n_group = h->n_group;
    a.topk_group = h->topk_group;
    a.top_k = h->top_k;
    a.partial = h->partial;
    a.idx = idx;
    a.w = w;
    a.logits_out = logits;
    cudaError_t e;
    if (!logits && router_on_tensor_cores(h, T)) {
        CUtensorMap tmx;
        if (!make_map(&tmx, x, (uint64_t)T, (uint64_t)h->H, (uint32_t)router_mma_tokens_per_tile()))
            return fail(h, BEAM_ERR_CUDA, "cuTensorMapEncodeTiled failed for x");
        RouterMmaArgs m;
        m.T = T;
        m.E = h->E;
        m.nslice = router_mma_slices(T, h->H, h->E, h->num_sms);
        m.kb_per_slice = h->H / 64 / m.nslice;
        m.kb_per_h = h->H / 64;
        m.partial = h->partial;
        m.fix_count = h->fix_count;   // the kernel zeroes the re-derivation count
        m.ctl.status = h->status;
        m.ctl.limit_ns = h->wait_limit_ns;
        const int items = ((h->E + router_mma_experts_per_tile() - 1) / router_mma_experts_per_tile()) *
                          ((T + router_mma_tokens_per_tile() - 1) / router_mma_tokens_per_tile()) *
                          m.nslice;
        e = launch_router_mma(h->tm_wcat, tmx, m, items < h->num_sms ? items : h->num_sms, s);
        if (e == cudaSuccess) {
            // select on the tensor-core logits, listing tokens whose margins
            // are too thin for their accumulation error ...
            a.nslice = m.nslice;
            SelectExtra ex;
            ex.margin = h->router_mode == 2 ? INFINITY : kRouterMargin;
            ex.fix_list = h->fix_list;
            ex.fix_count = h->fix_count;
            e = launch_router_select(a, ex, 0, s);
        }
        if (e == cudaSuccess)   // ... recompute theirs in FP32 on CUDA cores ...
            e = launch_router_fix(a.x, h->router_w, h->H, h->E, T, h->fix_list, h->fix_count,
                                  h->partial, 4 * h->num_sms, s);
        if (e == cudaSuccess) {   // ... and select them again
            RouterArgs b = a;
            b.nslice = 1;
            SelectExtra ex;
            ex.token_list = h->fix_list;
            ex.list_count = h->fix_count;
            e = launch_router_select(b, ex, 4 * h->num_sms, s);
        }
    } else {
        // the workspace holds nslice * T rows of either path
        const int ns_small = router_small_slices(T, h->H, h->E, h->num_sms);
        a.small = ns_small > 0;
        a.nslice = ns_small > 0 ? ns_small : router_slices(T, h->H, h->E, h->num_sms);
        e = launch_router(a, s);
    }
    return e == cudaSuccess ? BEAM_OK : cuda_fail(h, e, "router launch");
}

void prof_mark(beam_moe *h, cudaStream_t s, int stage)
{
    if (h->prof_calls < h->prof_max)
        cudaEventRecord(h->prof_events[(size_t)h->prof_calls * 6 + stage], s);
}

// The kernels and launch shapes a forward pass of T tokens uses.  A function
// of the handle's tuning and of T only, so that the host never waits on the
// routing to launch the GEMMs.
struct ForwardPlan {
    int tile_rows;     // largest token tile of the grouped GEMMs
    int cta_pairs;     // 1: cta_group::2 kernels
    int grid;          // CTAs of each grouped GEMM
    int down_paired;   // 1: two weight blocks per down work item
    int router_tc;     // 1: tensor-core logits with exact re-derivation
    int router_slices; // K slices of the router logits
    int gather;        // 1: gate|up gathers token rows from x; no sorted copy
    int stream_k;         // dense layers: 1 = both GEMMs stream-K (decode-sized token tiles)
    int y_f32;            // 1: the down GEMM writes the expert outputs y in FP32
    int gu_interleaved;   // 1: CTA-pair gate|up with interleaved gate and up rows per tile
};

// Dense layers: stream-K for token tiles of up to 64 rows (decode-sized
// batches), where the weight tiles alone give too few work items to spread
// evenly over the SMs.
bool dense_stream_k(const beam_moe *h, int BN) { return h->dense && BN <= 64; }

// Stream-K grid of a dense GEMM: every SM, or the tuning's CTA count.
int dense_sk_grid(const beam_moe *h)
{
    const int g = h->gemm_ctas > 0 ? h->gemm_ctas : h->num_sms;
    return g < h->num_sms ? g : h->num_sms;
}

// Dense layers: the smallest power-of-two token tile (16..256) that holds T.
int dense_tile_rows(int T)
{
    int bn = 16;
    while (bn < T && bn < 256) bn <<= 1;
    return bn;
}

ForwardPlan plan_forward(const beam_moe *h, int T)
{
    ForwardPlan p;
    p.tile_rows = h->tile_rows ? h->tile_rows
                               : (h->dense ? dense_tile_rows(T) : choose_tile_rows(T, h->top_k, h->E));
    // CTA pairs (cta_group::2) for large token tiles when the weight rows
    // split into 256-row blocks; single CTAs otherwise
    p.cta_pairs = h->use_pair != 0 && gemm_pair_supported(p.tile_rows) && h->I % 256 == 0 &&
                  h->H % 256 == 0 && gemm_pair_max_ctas() >= 2;
    p.grid = h->gemm_ctas > 0 ? h->gemm_ctas : h->num_sms;
    if (p.cta_pairs) {
        const int cap = gemm_pair_max_ctas();
        p.grid = p.grid > cap ? cap : p.grid;
        p.grid &= ~1;
        if (p.grid < 2) p.grid = 2;
    }
    // pair the down projection's weight blocks (two blocks share a token
    // tile) when H allows; lone blocks for decode-sized token tiles keep more
    // items in flight
    const int block_rows = p.cta_pairs ? 512 : 256;
    p.down_paired = h->H % block_rows == 0 &&
                    (h->down_pair == 1 || (h->down_pair < 0 && p.tile_rows >= 64));
    // Gathered token rows spare dispatch the sorted copy of x, but each
    // gather4 copy costs the TMA unit about as much as a whole box: with
    // large token tiles the gathers of a stage outlast its MMAs.  Automatic
    // only for tiles of up to 32 rows, where the weight stream sets the pace.
    p.gather = h->gather_rows < 0 ? (p.tile_rows <= 32 ? 1 : 0) : h->gather_rows;
    p.stream_k = 0;
    // Expert outputs y in FP32: the combine then rounds only once, to the
    // block's bf16 output.  The single-CTA FP32 down GEMM takes one weight
    // block per item.
    p.y_f32 = !h->dense && h->y_mode != 0;
    if (p.y_f32 && !p.cta_pairs) p.down_paired = 0;
    // Interleaved gate|up tiles on CTA pairs (on request only): one
    // accumulator of N columns instead of two, so two fit TMEM and one
    // item's epilogue overlaps the next item's MMAs; but each token tile is
    // then loaded for 128 intermediate rows instead of 256, and the extra
    // token-row traffic costs more than the overlap gains (measured at the
    // Beam prefill shape: gate|up 4.30 -> 5.87 ms).
    p.gu_interleaved = h->gu_layout == 1 && p.cta_pairs && h->I % 128 == 0;
    if (h->fp4) {
        // NVFP4 weights: the single-CTA kernel with token tiles of up to 128
        // rows from the sorted copy, one weight block per down item, FP32 y
        // as for bf16 weights
        if (p.tile_rows > 128) p.tile_rows = 128;
        p.cta_pairs = 0;
        p.grid = h->gemm_ctas > 0 ? h->gemm_ctas : h->num_sms;
        p.down_paired = 0;
        p.gather = 0;
        p.y_f32 = h->y_mode != 0;
        p.gu_interleaved = 0;
    }
    if (h->dense) {
        // one expert: with decode-sized T the weight tiles alone give too few
        // work items, so both GEMMs run stream-K (an equal run of K steps per
        // CTA; tiles cut between CTAs are finished by the last to arrive)
        p.gather = 0;
        p.router_tc = 0;
        p.router_slices = 0;
        p.stream_k = dense_stream_k(h, p.tile_rows);
        if (p.stream_k) {
            p.cta_pairs = 0;
            p.gu_interleaved = 0;
            p.down_paired = 0;
            p.grid = dense_sk_grid(h);
        }
        return p;
    }
    p.router_tc = router_on_tensor_cores(h, T);
    const int ns_small = router_small_slices(T, h->H, h->E, h->num_sms);
    p.router_slices = p.router_tc ? router_mma_slices(T, h->H, h->E, h->num_sms)
                                  : (ns_small > 0 ? ns_small : router_slices(T, h->H, h->E, h->num_sms));
    return p;
}

void finish_profile(beam_moe *h, cudaStream_t s, int T)
{
    prof_mark(h, s, 5);
    if (h->prof_calls < h->prof_max) ++h->prof_calls;
    h->last_T = T;
}

// The dense SwiGLU MLP: the grouped GEMMs over one expert of T rows that
// reads x directly, stream-K for decode-sized token tiles; the combine only
// for the post-norm and residual update.  Stage marks as the sparse block's,
// with empty router and a table set-up in place of the dispatch.
int run_forward_dense(beam_moe *h, cudaStream_t s, const void *x, int T, void *out,
                      float *residual, int k)
{
    prof_mark(h, s, 0);
    prof_mark(h, s, 1);
    const ForwardPlan plan = plan_forward(h, T);
    const int BN = plan.tile_rows;
    const int tiles = (T + BN - 1) / BN;
    cudaError_t e = launch_dense_setup(T, tiles, h->counts, h->offsets, h->tile_off, h->pair_row,
                                       h->row_pair, h->w, plan.stream_k ? h->sk_cnt : nullptr,
                                       h->sk_cnt_n, s);
    if (e != cudaSuccess) return cuda_fail(h, e, "dense set-up launch");
    prof_mark(h, s, 2);
    if (h->tm_x_ptr != x || h->tm_x_T != T) {
        for (int i = 0; i < 6; ++i)
            if (!make_map(&h->tm_x.m[i], x, (uint64_t)T, (uint64_t)h->H, 8u << i)) {
                h->tm_x_ptr = nullptr;
                return fail(h, BEAM_ERR_CUDA, "tensor map of x");
            }
        h->tm_x_ptr = x;
        h->tm_x_T = T;
    }
    GemmArgs g;
    g.E = 1;
    g.counts = h->counts;
    g.offsets = h->offsets;
    g.tile_off = h->tile_off;
    g.row_pair = h->row_pair;
    g.top_k = 1;
    g.gather = 0;
    g.ctl.status = h->status;
    g.ctl.limit_ns = h->wait_limit_ns;
    g.b_stages = h->token_stages;
    g.a_stages = 0;
    g.out_f32 = nullptr;
    // counters of the gate|up tiles, then of the down tiles
    const int nt = (T + BN - 1) / BN;
    int *cnt_gu = h->sk_cnt, *cnt_d = h->sk_cnt + (size_t)(h->I / 128) * nt;

    g.K = h->H;
    g.R = h->I;
    g.out = h->hbuf;
    if (plan.stream_k) {
        e = launch_dense_sk(true, BN, h->tm_gate, h->tm_up, h->tm_x, g, T, h->sk_part, cnt_gu,
                            plan.grid, s);
    } else {
        e = plan.gu_interleaved
                ? launch_grouped_gemm_pair(GemmKind::kGateUpI, BN, h->tm_gate16, h->tm_up16, h->tm_x,
                                           g, plan.grid, s)
            : plan.cta_pairs
                ? launch_grouped_gemm_pair(GemmKind::kGateUp, BN, h->tm_gate, h->tm_up, h->tm_x, g,
                                           plan.grid, s)
                : launch_grouped_gemm(GemmKind::kGateUp, BN, h->tm_gate, h->tm_up, h->tm_x, g,
                                      plan.grid, s);
    }
    if (e != cudaSuccess) return cuda_fail(h, e, "gate/up GEMM launch");
    prof_mark(h, s, 3);

    g.K = h->I;
    g.R = h->H;
    // without a residual the down projection's bf16 rows are the output
    g.out = residual ? h->ybuf : static_cast<__nv_bfloat16 *>(out);
    if (plan.stream_k) {
        e = launch_dense_sk(false, BN, h->tm_down, h->tm_down, h->tm_h, g, T, h->sk_part, cnt_d,
                            plan.grid, s);
    } else {
        const GemmKind dk = plan.down_paired ? GemmKind::kDownPaired : GemmKind::kDown;
        e = plan.cta_pairs ? launch_grouped_gemm_pair(dk, BN, h->tm_down, h->tm_down, h->tm_h, g,
                                                      plan.grid, s)
                           : launch_grouped_gemm(dk, BN, h->tm_down, h->tm_down, h->tm_h, g,
                                                 plan.grid, s);
    }
    if (e != cudaSuccess) return cuda_fail(h, e, "down GEMM launch");
    prof_mark(h, s, 4);

    if (residual) {
        CombineArgs c;
        c.status = h->status;
        c.y = h->ybuf;
        c.y32 = nullptr;
        c.pair_row = h->pair_row;
        c.w = h->w;
        c.T = T;
        c.H = h->H;
        c.top_k = 1;
        c.scaling = 1.0f;
        c.out = static_cast<__nv_bfloat16 *>(out);
        c.residual = residual;
        c.gamma = residual ? h->gamma : nullptr;
        c.eps = h->eps;
        const int kk = k >= 1 ? k : 1;
        c.keep = (float)std::sqrt((double)(kk - 1) / (double)kk);
        c.add = (float)(1.0 / std::sqrt((double)kk));
        e = launch_combine(c, s);
        if (e != cudaSuccess) return cuda_fail(h, e, "combine launch");
    }
    finish_profile(h, s, T);
    return BEAM_OK;
}

int run_forward(beam_moe *h, cudaStream_t s, const void *x, int T, void *out, float *residual,
                int k)
{
    if (h->dense) return run_forward_dense(h, s, x, T, out, residual, k);
    prof_mark(h, s, 0);
    int rc = run_router(h, s, x, T, h->idx, h->w, nullptr);
    if (rc != BEAM_OK) return rc;
    if (h->checks) {
        cudaError_t ce = cudaSuccess;
        if (h->corrupt_next > 0) {
            --h->corrupt_next;
            ce = launch_corrupt_routing(h->idx, h->E, s);
        }
        if (ce == cudaSuccess)
            ce = launch_check_routing(h->idx, h->w, T, h->E, h->top_k, h->status, h->check_where, s);
        if (ce != cudaSuccess) return cuda_fail(h, ce, "routing check launch");
    }
    prof_mark(h, s, 1);
    const ForwardPlan plan = plan_forward(h, T);
    const int BN = plan.tile_rows;
    DispatchArgs d;
    d.status = h->status;
    d.idx = h->idx;
    d.x = static_cast<const __nv_bfloat16 *>(x);
    d.T = T;
    d.H = h->H;
    d.E = h->E;
    d.top_k = h->top_k;
    d.tile_rows = BN;
    d.block_cnt = h->block_cnt;
    d.block_base = h->block_base;
    d.rank = h->rank;
    d.counts = h->counts;
    d.offsets = h->offsets;
    d.tile_off = h->tile_off;
    d.pair_row = h->pair_row;
    d.row_pair = h->row_pair;
    d.xp = h->xp;
    d.copy_rows = !plan.gather;
    d.xp_f16 = h->fp4 ? 1 : 0;
    cudaError_t e = launch_dispatch(d, s);
    if (e == cudaSuccess && h->checks)
        e = launch_check_dispatch(h->idx, h->counts, h->offsets, h->tile_off, h->pair_row,
                                  h->row_pair, T * h->top_k, h->E, BN, h->status, h->check_where, s);
    if (e != cudaSuccess) return cuda_fail(h, e, "dispatch launch");
    prof_mark(h, s, 2);

    GemmArgs g;
    g.E = h->E;
    g.counts = h->counts;
    g.offsets = h->offsets;
    g.tile_off = h->tile_off;
    g.ctl.status = h->status;
    g.ctl.limit_ns = h->wait_limit_ns;
    g.b_stages = h->token_stages;
    g.a_stages = 0;
    g.row_pair = h->row_pair;
    g.top_k = h->top_k;
    g.gather = plan.gather;
    g.out_f32 = nullptr;
    // token rows of the gate|up GEMM: x itself, four rows per gather4 copy,
    // or boxes of the sorted copy
    BoxMaps bx_local;
    const BoxMaps *bx = &h->tm_xp;
    if (plan.gather) {
        bx_local = h->tm_xp;
        if (!make_map(&bx_local.gather, x, (uint64_t)T, (uint64_t)h->H, 1u))
            return fail(h, BEAM_ERR_CUDA, "tensor map of x");
        bx = &bx_local;
    }
    const bool use_pair = plan.cta_pairs != 0;
    const int grid = plan.grid;
    g.K = h->H;
    g.R = h->I;
    g.out = h->hbuf;
    if (h->fp4)
        e = launch_grouped_gemm_fp4(GemmKind::kGateUp, BN, h->fp4_gate_up, *bx, g, grid, s);
    else
        e = plan.gu_interleaved
                ? launch_grouped_gemm_pair(GemmKind::kGateUpI, BN, h->tm_gate16, h->tm_up16, *bx, g,
                                           grid, s)
            : use_pair ? launch_grouped_gemm_pair(GemmKind::kGateUp, BN, h->tm_gate, h->tm_up, *bx,
                                                  g, grid, s)
                       : launch_grouped_gemm(GemmKind::kGateUp, BN, h->tm_gate, h->tm_up, *bx, g,
                                             grid, s);
    if (e != cudaSuccess) return cuda_fail(h, e, "gate/up GEMM launch");
    prof_mark(h, s, 3);
    g.K = h->I;
    g.R = h->H;
    g.out = h->ybuf;
    g.out_f32 = plan.y_f32 ? h->y32 : nullptr;
    g.gather = 0;
    GemmKind dk = plan.down_paired ? GemmKind::kDownPaired : GemmKind::kDown;
    if (plan.y_f32)
        dk = use_pair ? (plan.down_paired ? GemmKind::kDownPairedY32 : GemmKind::kDownY32)
                      : GemmKind::kDownF32;
    if (h->fp4)
        e = launch_grouped_gemm_fp4(plan.y_f32 ? GemmKind::kDownF32 : GemmKind::kDown, BN, h->fp4_down,
                                    h->tm_h, g, grid, s);
    else
        e = use_pair ? launch_grouped_gemm_pair(dk, BN, h->tm_down, h->tm_down, h->tm_h, g, grid, s)
                     : launch_grouped_gemm(dk, BN, h->tm_down, h->tm_down, h->tm_h, g, grid, s);
    if (e != cudaSuccess) return cuda_fail(h, e, "down GEMM launch");
    prof_mark(h, s, 4);

    CombineArgs c;
    c.status = h->status;
    c.y = plan.y_f32 ? nullptr : h->ybuf;
    c.y32 = plan.y_f32 ? h->y32 : nullptr;
    c.pair_row = h->pair_row;
    c.w = h->w;
    c.T = T;
    c.H = h->H;
    c.top_k = h->top_k;
    c.scaling = h->scaling;
    c.out = static_cast<__nv_bfloat16 *>(out);
    c.residual = residual;
    c.gamma = residual ? h->gamma : nullptr;
    c.eps = h->eps;
    const int kk = k >= 1 ? k : 1;
    c.keep = (float)std::sqrt((double)(kk - 1) / (double)kk);
    c.add = (float)(1.0 / std::sqrt((double)kk));
    e = launch_combine(c, s);
    if (e != cudaSuccess) return cuda_fail(h, e, "combine launch");
    finish_profile(h, s, T);
    return BEAM_OK;
}

int check_tokens(beam_moe *h, const void *x, int T)
{
    if (T < 0 || T > h->max_tokens)
        return fail(h, BEAM_ERR_INVALID_ARG, "T=%d outside [0, max_tokens=%d]", T, h->max_tokens);
    if (T > 0 && (!x || !aligned16(x)))
        return fail(h, BEAM_ERR_INVALID_ARG, "x must be a non-NULL 16-byte aligned device pointer");
    return BEAM_OK;
}

void release_host_path(beam_moe *h)
{
    for (int i = 0; i < 2; ++i) {
        if (h->ev_in[i]) cudaEventDestroy(h->ev_in[i]);
        if (h->ev_comp[i]) cudaEventDestroy(h->ev_comp[i]);
        if (h->ev_out[i]) cudaEventDestroy(h->ev_out[i]);
    }
    if (h->ev_fence) cudaEventDestroy(h->ev_fence);
    if (h->copy_in) cudaStreamDestroy(h->copy_in);
    if (h->copy_out) cudaStreamDestroy(h->copy_out);
}

// Device set-up common to both handle kinds: workspace, kernel attributes,
// the router weight's bf16 pieces (sparse blocks) and the tensor maps.
int finish_create(beam_moe *h, beam_moe_t *out)
{
    const int hidden = h->H, inter = h->I, n_experts = h->E, top_k = h->top_k;
    const int max_tokens = h->max_tokens;
    h->wait_limit_ns = 2000000000LL;
    h->down_pair = -1;
    h->use_pair = 1;
    h->gather_rows = -1;
    h->router_mode = -1;
    h->y_mode = 1;
    h->gu_layout = -1;

    cudaError_t e = cudaGetDevice(&h->device);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device);
    if (e != cudaSuccess) {
        int rc = cuda_fail(nullptr, e, "device query");
        delete h;
        return rc;
    }

    // Workspace
    const size_t T = (size_t)max_tokens, E = (size_t)n_experts, P = T * top_k;
    const size_t nblk = (P + kDispatchBlock - 1) / kDispatchBlock;
    // router partial sums: the largest nslice(t) * t over t <= max_tokens, for
    // either router path
    size_t partial_rows = 0;
    // dense layers: stream-K slots (two per CTA, at the largest stream-K
    // token tile) and an arrival counter per tile of either GEMM, for every
    // token tile a tuning may ask for (16 rows: the most tiles)
    const size_t sk_floats = h->dense ? dense_sk_part_floats(64, true, h->num_sms) : 0;
    h->sk_cnt_n = h->dense ? (int)((size_t)(hidden > inter ? hidden : inter) / 128 * 2 *
                                   ((size_t)(max_tokens + 15) / 16))
                           : 0;
    for (int t = 1; t <= max_tokens && !h->dense; ++t) {
        const size_t r0 = (size_t)router_small_slices(t, hidden, n_experts, h->num_sms) * t;
        if (r0 > partial_rows) partial_rows = r0;
        const size_t r1 = (size_t)router_slices(t, hidden, n_experts, h->num_sms) * t;
        const size_t r2 = (size_t)router_mma_slices(t, hidden, n_experts, h->num_sms) * t;
        if (r1 > partial_rows) partial_rows = r1;
        if (r2 > partial_rows) partial_rows = r2;
    }
    size_t off = 0;
    auto carve = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + bytes, 256);
        return o;
    };
    const size_t o_partial = carve(partial_rows * E * 4);
    const size_t o_skpart = carve(sk_floats * 4);
    const size_t o_skcnt = carve((size_t)h->sk_cnt_n * 4);
    const size_t o_idx = carve(P * 4);
    const size_t o_w = carve(P * 4);
    const size_t o_bcnt = carve(nblk * E * 4);
    const size_t o_bbase = carve(nblk * E * 4);
    const size_t o_rank = carve(P * 4);
    const size_t o_counts = carve(E * 4);
    const size_t o_offsets = carve((E + 1) * 4);
    const size_t o_tile = carve((E + 1) * 4);
    const size_t o_prow = carve(P * 4);
    const size_t o_rpair = carve(P * 4);
    const size_t o_xp = carve(h->dense ? 0 : P * hidden * 2);   // dense: the GEMM reads x
    const size_t o_h = carve(P * inter * 2);
    const size_t o_y = carve(P * hidden * (h->dense ? 2 : 4));   // bf16 or FP32 y
    const size_t o_status = carve(256);
    size_t o_xs[2], o_os[2], o_rs[2];
    for (int i = 0; i < 2; ++i) {
        o_xs[i] = carve(T * hidden * 2);
        o_os[i] = carve(T * hidden * 2);
        o_rs[i] = carve(T * hidden * 4);
    }
    const size_t o_wcat = carve(h->dense ? 0 : E * 3 * (size_t)hidden * 2);
    const size_t o_fix = carve((T + 1) * 4);
    h->ws_bytes = off;
    e = cudaMalloc(&h->ws, h->ws_bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        int rc = fail(nullptr, BEAM_ERR_OOM, "workspace of %zu bytes: %s", h->ws_bytes,
                      cudaGetErrorString(e));
        delete h;
        return rc;
    }
    char *b = static_cast<char *>(h->ws);
    h->partial = reinterpret_cast<float *>(b + o_partial);
    h->sk_part = reinterpret_cast<float *>(b + o_skpart);
    h->sk_cnt = reinterpret_cast<int *>(b + o_skcnt);
    h->idx = reinterpret_cast<int32_t *>(b + o_idx);
    h->w = reinterpret_cast<float *>(b + o_w);
    h->block_cnt = reinterpret_cast<int32_t *>(b + o_bcnt);
    h->block_base = reinterpret_cast<int32_t *>(b + o_bbase);
    h->rank = reinterpret_cast<int32_t *>(b + o_rank);
    h->counts = reinterpret_cast<int32_t *>(b + o_counts);
    h->offsets = reinterpret_cast<int32_t *>(b + o_offsets);
    h->tile_off = reinterpret_cast<int32_t *>(b + o_tile);
    h->pair_row = reinterpret_cast<int32_t *>(b + o_prow);
    h->row_pair = reinterpret_cast<int32_t *>(b + o_rpair);
    h->xp = reinterpret_cast<__nv_bfloat16 *>(b + o_xp);
    h->hbuf = reinterpret_cast<__nv_bfloat16 *>(b + o_h);
    h->ybuf = reinterpret_cast<__nv_bfloat16 *>(b + o_y);
    h->y32 = reinterpret_cast<float *>(b + o_y);
    h->status = reinterpret_cast<int *>(b + o_status);
    for (int i = 0; i < 2; ++i) {
        h->x_stage[i] = reinterpret_cast<__nv_bfloat16 *>(b + o_xs[i]);
        h->out_stage[i] = reinterpret_cast<__nv_bfloat16 *>(b + o_os[i]);
        h->res_stage[i] = reinterpret_cast<float *>(b + o_rs[i]);
    }
    h->wcat = reinterpret_cast<__nv_bfloat16 *>(b + o_wcat);
    h->fix_count = reinterpret_cast<int *>(b + o_fix);
    h->fix_list = h->fix_count + 1;
    h->check_where = h->status + 1;
    e = cudaMemset(h->fix_count, 0, sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(h->status, 0, sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(h->check_where, 0x7f, sizeof(int));
    if (e == cudaSuccess) e = prepare_grouped_gemm(n_experts);
    if (e == cudaSuccess) e = prepare_dispatch(n_experts);
    if (e == cudaSuccess && h->dense) e = prepare_dense_sk();
    if (e == cudaSuccess && h->fp4) {
        // the tiled copy of the three NVFP4 tensors (gate, up: [E*I, H];
        // down: [E*H, I]), made once on the legacy default stream
        const long long rows[3] = {(long long)E * inter, (long long)E * inter, (long long)E * hidden};
        const int kdim[3] = {hidden, hidden, inter};
        size_t code_off[3], scale_off[3], total = 0;
        for (int i = 0; i < 3; ++i) {
            code_off[i] = total;
            total = align_up(total + (size_t)rows[i] * kdim[i] / 2, 256);
            scale_off[i] = total;
            total = align_up(total + (size_t)rows[i] * kdim[i] / 16, 256);
        }
        e = cudaMalloc(&h->fp4_buf, total);
        if (e != cudaSuccess) {
            cudaGetLastError();
            h->fp4_buf = nullptr;
            int rc = fail(nullptr, BEAM_ERR_OOM, "NVFP4 weight copy of %zu bytes: %s", total,
                          cudaGetErrorString(e));
            cudaFree(h->ws);
            delete h;
            return rc;
        }
        Fp4Tensor t[3] = {};
        for (int i = 0; i < 3 && e == cudaSuccess; ++i) {
            t[i].codes = h->fp4_buf + code_off[i];
            t[i].scales = h->fp4_buf + scale_off[i];
            t[i].global = h->fp4_global[i];
            e = launch_fp4_repack(h->fp4_codes_in[i], h->fp4_scales_in[i], rows[i], kdim[i],
                                  h->fp4_buf + code_off[i], h->fp4_buf + scale_off[i], 0);
        }
        h->fp4_gate_up.a[0] = t[0];
        h->fp4_gate_up.a[1] = t[1];
        h->fp4_gate_up.row_tiles = inter / kFp4TileRows;
        h->fp4_gate_up.k_steps = hidden / kFp4TileK;
        h->fp4_down.a[0] = t[2];
        h->fp4_down.a[1] = t[2];
        h->fp4_down.row_tiles = hidden / kFp4TileRows;
        h->fp4_down.k_steps = inter / kFp4TileK;
        if (e == cudaSuccess) e = prepare_grouped_gemm_fp4();
        for (int i = 0; i < 3; ++i)   // read at create only: not kept
            h->fp4_codes_in[i] = h->fp4_scales_in[i] = nullptr;
    }
    if (!h->dense) {
        if (e == cudaSuccess) e = prepare_router_mma();
        if (e == cudaSuccess) e = prepare_router_small();
        if (e == cudaSuccess) e = prepare_router_fix(hidden);
        // the router weight's bf16 pieces for the tensor-core router (the
        // weight is borrowed and must not change while the handle lives)
        if (e == cudaSuccess) e = launch_router_split(h->router_w, n_experts, hidden, h->wcat, 0);
    }
    if (e == cudaSuccess) e = cudaStreamSynchronize(0);
    if (e != cudaSuccess) {
        int rc = cuda_fail(nullptr, e, "workspace / kernel set-up");
        if (h->fp4_buf) cudaFree(h->fp4_buf);
        cudaFree(h->ws);
        delete h;
        return rc;
    }

    bool ok = h->fp4 || (make_map(&h->tm_gate, h->w_gate, E * inter, hidden, 128) &&
                         make_map(&h->tm_up, h->w_up, E * inter, hidden, 128) &&
                         make_map(&h->tm_gate16, h->w_gate, E * inter, hidden, 16) &&
                         make_map(&h->tm_up16, h->w_up, E * inter, hidden, 16) &&
                         make_map(&h->tm_down, h->w_down, E * hidden, inter, 128));
    if (!h->dense) ok = ok && make_map(&h->tm_wcat, h->wcat, E, 3 * (uint64_t)hidden, 128);
    for (int i = 0; i < 6 && ok; ++i) {
        ok = make_map(&h->tm_h.m[i], h->hbuf, P, inter, 8u << i);
        if (ok && !h->dense) ok = make_map(&h->tm_xp.m[i], h->xp, P, hidden, 8u << i);
    }
    if (!ok) {
        if (h->fp4_buf) cudaFree(h->fp4_buf);
        cudaFree(h->ws);
        delete h;
        return fail(nullptr, BEAM_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    }
    e = cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_fence, cudaEventDisableTiming);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
        e = cudaEventCreateWithFlags(&h->ev_in[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_comp[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->ev_out[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) {
        int rc = cuda_fail(nullptr, e, "host-path streams / events");
        release_host_path(h);
        if (h->fp4_buf) cudaFree(h->fp4_buf);
        cudaFree(h->ws);
        delete h;
        return rc;
    }
    *out = h;
    return BEAM_OK;
}

// Argument checks shared by the sparse-block create calls: shapes, routing
// parameters, the router and norm pointers.
int check_sparse_args(int hidden, int n_experts, int inter, int n_group, int topk_group, int top_k,
                      float routed_scaling, const float *router_w, const float *expert_bias,
                      const float *post_norm_w, float norm_eps, int max_tokens)
{
    if (hidden <= 0 || n_experts <= 0 || inter <= 0 || n_group <= 0 || max_tokens < 1)
        return fail(nullptr, BEAM_ERR_INVALID_ARG, "sizes must be positive");
    if (n_experts % n_group != 0)
        return fail(nullptr, BEAM_ERR_INVALID_ARG, "n_experts %% n_group != 0");
    const int gsize = n_experts / n_group;
    if (gsize < 2) return fail(nullptr, BEAM_ERR_INVALID_ARG, "group size must be >= 2");
    if (topk_group < 1 || topk_group > n_group)
        return fail(nullptr, BEAM_ERR_INVALID_ARG, "topk_group outside [1, n_group]");
    if (top_k < 1 || top_k > topk_group * gsize)
        return fail(nullptr, BEAM_ERR_INVALID_ARG, "top_k outside [1, topk_group * group size]");
    if (!(routed_scaling == routed_scaling) || !(norm_eps >= 0.f))
        return fail(nullptr, BEAM_ERR_INVALID_ARG, "routed_scaling / norm_eps not valid");
    if (!router_w || !expert_bias)
        return fail(nullptr, BEAM_ERR_INVALID_ARG, "weight pointer is NULL");
    if (!aligned16(router_w) || !aligned16(expert_bias) || (post_norm_w && !aligned16(post_norm_w)))
        return fail(nullptr, BEAM_ERR_INVALID_ARG, "weight pointers must be 16-byte aligned");
    if (hidden % 128 != 0 || inter % 128 != 0)
        return fail(nullptr, BEAM_ERR_UNSUPPORTED, "hidden and inter must be multiples of 128");
    if (hidden > 8192)
        return fail(nullptr, BEAM_ERR_UNSUPPORTED, "hidden > 8192");
    if (n_experts % 32 != 0 || n_experts > 1024 || !is_pow2(n_experts / 32))
        return fail(nullptr, BEAM_ERR_UNSUPPORTED,
                    "n_experts must be 32 x a power of two, at most 1024");
    const int epl = n_experts / 32;
    if (gsize % epl != 0 || !is_pow2(gsize / epl) || n_group > 32)
        return fail(nullptr, BEAM_ERR_UNSUPPORTED, "group size not supported by the router kernel");
    if (top_k > 32) return fail(nullptr, BEAM_ERR_UNSUPPORTED, "top_k > 32");
    if ((long long)max_tokens * top_k > (1LL << 30))
        return fail(nullptr, BEAM_ERR_UNSUPPORTED, "max_tokens * top_k too large");
    return BEAM_OK;
}

beam_moe *new_sparse_handle(int hidden, int n_experts, int inter, int n_group, int topk_group,
                            int top_k, float routed_scaling, const float *router_w,
                            const float *expert_bias, const float *post_norm_w, float norm_eps,
                            int max_tokens)
{
    beam_moe *h = new beam_moe();   // value-initialised: every plain field starts at zero
    h->H = hidden;
    h->E = n_experts;
    h->I = inter;
    h->n_group = n_group;
    h->topk_group = topk_group;
    h->top_k = top_k;
    h->scaling = routed_scaling;
    h->router_w = router_w;
    h->bias = expert_bias;
    h->gamma = post_norm_w;
    h->eps = norm_eps;
    h->max_tokens = max_tokens;
    return h;
}

}  // namespace

extern "C" {

const char *beam_moe_create_error(void) { return g_create_err; }

int beam_moe_create(beam_moe_t *out, int hidden, int n_experts, int inter, int n_group,
                    int topk_group, int top_k, float routed_scaling, const float *router_w,
                    const float *expert_bias, const void *w_gate, const void *w_up,
                    const void *w_down, const float *post_norm_w, float norm_eps, int max_tokens)
{
    g_create_err[0] = 0;
    if (!out) return fail(nullptr, BEAM_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    int rc = check_sparse_args(hidden, n_experts, inter, n_group, topk_group, top_k, routed_scaling,
                               router_w, expert_bias, post_norm_w, norm_eps, max_tokens);
    if (rc != BEAM_OK) return rc;
    if (!w_gate || !w_up || !w_down)
        return fail(nullptr, BEAM_ERR_INVALID_ARG, "weight pointer is NULL");
    if (!aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down))
        return fail(nullptr, BEAM_ERR_INVALID_ARG, "weight pointers must be 16-byte aligned");
    beam_moe *h = new_sparse_handle(hidden, n_experts, inter, n_group, topk_group, top_k,
                                    routed_scaling, router_w, expert_bias, post_norm_w, norm_eps,
                                    max_tokens);
    h->w_gate = static_cast<const __nv_bfloat16 *>(w_gate);
    h->w_up = static_cast<const __nv_bfloat16 *>(w_up);
    h->w_down = static_cast<const __nv_bfloat16 *>(w_down);
    return finish_create(h, out);
}

int beam_moe_create_nvfp4(beam_moe_t *out, int hidden, int n_experts, int inter, int n_group,
                          int topk_group, int top_k, float routed_scaling, const float *router_w,
                          const float *expert_bias, const uint8_t *gate_codes,
                          const uint8_t *gate_scales, float gate_global, const uint8_t *up_codes,
                          const uint8_t *up_scales, float up_global, const uint8_t *down_codes,
                          const uint8_t *down_scales, float down_global, const float *post_norm_w,
                          float norm_eps, int max_tokens)
{
    g_create_err[0] = 0;
    if (!out) return fail(nullptr, BEAM_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    int rc = check_sparse_args(hidden, n_experts, inter, n_group, topk_group, top_k, routed_scaling,
                               router_w, expert_bias, post_norm_w, norm_eps, max_tokens);
    if (rc != BEAM_OK) return rc;
    const uint8_t *ptrs[6] = {gate_codes, gate_scales, up_codes, up_scales, down_codes, down_scales};
    for (const uint8_t *q : ptrs) {
        if (!q) return fail(nullptr, BEAM_ERR_INVALID_ARG, "NVFP4 tensor pointer is NULL");
        if (!aligned16(q))
            return fail(nullptr, BEAM_ERR_INVALID_ARG, "NVFP4 tensor pointers must be 16-byte aligned");
    }
    const float gl[3] = {gate_global, up_global, down_global};
    for (float g : gl)
        if (!(std::isfinite(g)))
            return fail(nullptr, BEAM_ERR_INVALID_ARG, "per-tensor scales must be finite");
    beam_moe *h = new_sparse_handle(hidden, n_experts, inter, n_group, topk_group, top_k,
                                    routed_scaling, router_w, expert_bias, post_norm_w, norm_eps,
                                    max_tokens);
    h->fp4 = 1;
    for (int i = 0; i < 3; ++i) {
        h->fp4_codes_in[i] = ptrs[2 * i];
        h->fp4_scales_in[i] = ptrs[2 * i + 1];
        h->fp4_global[i] = gl[i];
    }
    return finish_create(h, out);
}

int beam_nvfp4_dequant(void *stream, const uint8_t *codes, const uint8_t *scales, long long rows,
                       int K, void *out)
{
    if (rows < 0 || K <= 0 || K % 16 != 0) return BEAM_ERR_INVALID_ARG;
    if (rows == 0) return BEAM_OK;
    if (!codes || !scales || !out || !aligned16(codes) || !aligned16(out)) return BEAM_ERR_INVALID_ARG;
    const cudaError_t e = launch_fp4_dequant(codes, scales, rows * (long long)K,
                                             static_cast<__nv_bfloat16 *>(out),
                                             static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BEAM_OK : BEAM_ERR_CUDA;
}

int beam_moe_create_dense(beam_moe_t *out, int hidden, int inter, const void *w_gate,
                          const void *w_up, const void *w_down, const float *post_norm_w,
                          float norm_eps, int max_tokens)
{
    g_create_err[0] = 0;
    if (!out) return fail(nullptr, BEAM_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (hidden <= 0 || inter <= 0 || max_tokens < 1)
        return fail(nullptr, BEAM_ERR_INVALID_ARG, "sizes must be positive");
    if (!(norm_eps >= 0.f)) return fail(nullptr, BEAM_ERR_INVALID_ARG, "norm_eps not valid");
    if (!w_gate || !w_up || !w_down)
        return fail(nullptr, BEAM_ERR_INVALID_ARG, "weight pointer is NULL");
    if (!aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) ||
        (post_norm_w && !aligned16(post_norm_w)))
        return fail(nullptr, BEAM_ERR_INVALID_ARG, "weight pointers must be 16-byte aligned");
    if (hidden % 128 != 0 || inter % 128 != 0)
        return fail(nullptr, BEAM_ERR_UNSUPPORTED, "hidden and inter must be multiples of 128");
    if (hidden > 8192) return fail(nullptr, BEAM_ERR_UNSUPPORTED, "hidden > 8192");
    if ((long long)max_tokens > (1LL << 30))
        return fail(nullptr, BEAM_ERR_UNSUPPORTED, "max_tokens too large");

    beam_moe *h = new beam_moe();
    h->dense = 1;
    h->H = hidden;
    h->E = 1;
    h->I = inter;
    h->n_group = 1;
    h->topk_group = 1;
    h->top_k = 1;
    h->scaling = 1.0f;
    h->gamma = post_norm_w;
    h->w_gate = static_cast<const __nv_bfloat16 *>(w_gate);
    h->w_up = static_cast<const __nv_bfloat16 *>(w_up);
    h->w_down = static_cast<const __nv_bfloat16 *>(w_down);
    h->eps = norm_eps;
    h->max_tokens = max_tokens;
    return finish_create(h, out);
}

int beam_moe_route(beam_moe_t h, void *stream, const void *x, int T, int32_t *topk_idx,
                   float *topk_w)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    if (h->dense) return fail(h, BEAM_ERR_UNSUPPORTED, "a dense layer has no router");
    h->err[0] = 0;
    int rc = check_tokens(h, x, T);
    if (rc != BEAM_OK) return rc;
    if (T == 0) return BEAM_OK;
    if (!topk_idx || !topk_w) return fail(h, BEAM_ERR_INVALID_ARG, "output pointer is NULL");
    if ((rc = check_device(h)) != BEAM_OK) return rc;
    return run_router(h, static_cast<cudaStream_t>(stream), x, T, topk_idx, topk_w, nullptr);
}

int beam_moe_router_logits(beam_moe_t h, void *stream, const void *x, int T, float *logits)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    if (h->dense) return fail(h, BEAM_ERR_UNSUPPORTED, "a dense layer has no router");
    h->err[0] = 0;
    int rc = check_tokens(h, x, T);
    if (rc != BEAM_OK) return rc;
    if (T == 0) return BEAM_OK;
    if (!logits) return fail(h, BEAM_ERR_INVALID_ARG, "logits is NULL");
    if ((rc = check_device(h)) != BEAM_OK) return rc;
    return run_router(h, static_cast<cudaStream_t>(stream), x, T, h->idx, h->w, logits);
}

int beam_moe_route_logits(beam_moe_t h, void *stream, const float *logits, int T,
                          const float *expert_bias, int32_t *topk_idx, float *topk_w)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    if (h->dense) return fail(h, BEAM_ERR_UNSUPPORTED, "a dense layer has no router");
    h->err[0] = 0;
    if (T < 0 || T > h->max_tokens)
        return fail(h, BEAM_ERR_INVALID_ARG, "T=%d outside [0, max_tokens=%d]", T, h->max_tokens);
    if (T == 0) return BEAM_OK;
    if (!logits || !topk_idx || !topk_w)
        return fail(h, BEAM_ERR_INVALID_ARG, "logits, topk_idx and topk_w must be non-NULL");
    if (!aligned16(logits) || (expert_bias && !aligned16(expert_bias)))
        return fail(h, BEAM_ERR_INVALID_ARG, "logits / expert_bias must be 16-byte aligned");
    int rc = check_device(h);
    if (rc != BEAM_OK) return rc;
    // the selection kernel over one K slice that already holds the logits
    RouterArgs a;
    a.x = nullptr;
    a.router_w = nullptr;
    a.bias = expert_bias ? expert_bias : h->bias;
    a.T = T;
    a.H = h->H;
    a.E = h->E;
    a.n_group = h->n_group;
    a.topk_group = h->topk_group;
    a.top_k = h->top_k;
    a.nslice = 1;
    a.partial = const_cast<float *>(logits);   // read only by the selection
    a.idx = topk_idx;
    a.w = topk_w;
    a.logits_out = nullptr;
    cudaError_t e = launch_router_select(a, SelectExtra(), 0, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BEAM_OK : cuda_fail(h, e, "selection launch");
}

int beam_moe_forward(beam_moe_t h, void *stream, const void *x, int T, void *out,
                     float *residual, int k)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    h->err[0] = 0;
    int rc = check_tokens(h, x, T);
    if (rc != BEAM_OK) return rc;
    if (T == 0) return BEAM_OK;
    if (!out && !residual) return fail(h, BEAM_ERR_INVALID_ARG, "out and residual are both NULL");
    if ((out && !aligned16(out)) || (residual && !aligned16(residual)))
        return fail(h, BEAM_ERR_INVALID_ARG, "out / residual must be 16-byte aligned");
    if (residual && k < 1) return fail(h, BEAM_ERR_INVALID_ARG, "residual step k must be >= 1");
    if ((rc = check_device(h)) != BEAM_OK) return rc;
    return run_forward(h, static_cast<cudaStream_t>(stream), x, T, out, residual, k);
}

int beam_moe_forward_host_async(beam_moe_t h, void *stream, const void *x_host, int T,
                                void *out_host, float *residual_host, int k)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    h->err[0] = 0;
    if (T < 0 || T > h->max_tokens)
        return fail(h, BEAM_ERR_INVALID_ARG, "T=%d outside [0, max_tokens=%d]", T, h->max_tokens);
    if (T == 0) return BEAM_OK;
    if (!out_host && !residual_host)
        return fail(h, BEAM_ERR_INVALID_ARG, "out_host and residual_host are both NULL");
    if (!x_host) return fail(h, BEAM_ERR_INVALID_ARG, "x_host is NULL");
    if (residual_host && k < 1) return fail(h, BEAM_ERR_INVALID_ARG, "residual step k must be >= 1");
    int rc = check_device(h);
    if (rc != BEAM_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int slot = h->host_slot;
    const size_t n = (size_t)T * h->H;
    // copy in once this slot's previous pass has read its inputs and its
    // previous results have left
    cudaError_t e = cudaStreamWaitEvent(h->copy_in, h->ev_comp[slot], 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->copy_in, h->ev_out[slot], 0);
    if (e == cudaSuccess)
        e = cudaMemcpyAsync(h->x_stage[slot], x_host, n * 2, cudaMemcpyHostToDevice, h->copy_in);
    if (e == cudaSuccess && residual_host)
        e = cudaMemcpyAsync(h->res_stage[slot], residual_host, n * 4, cudaMemcpyHostToDevice,
                            h->copy_in);
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_in[slot], h->copy_in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, h->ev_in[slot], 0);
    if (e != cudaSuccess) return cuda_fail(h, e, "host-to-device copy");
    rc = run_forward(h, s, h->x_stage[slot], T, out_host ? h->out_stage[slot] : nullptr,
                     residual_host ? h->res_stage[slot] : nullptr, k);
    if (rc != BEAM_OK) return rc;
    e = cudaEventRecord(h->ev_comp[slot], s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->copy_out, h->ev_comp[slot], 0);
    if (e == cudaSuccess && out_host)
        e = cudaMemcpyAsync(out_host, h->out_stage[slot], n * 2, cudaMemcpyDeviceToHost, h->copy_out);
    if (e == cudaSuccess && residual_host)
        e = cudaMemcpyAsync(residual_host, h->res_stage[slot], n * 4, cudaMemcpyDeviceToHost,
                            h->copy_out);
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_out[slot], h->copy_out);
    if (e != cudaSuccess) return cuda_fail(h, e, "device-to-host copy");
    h->host_slot = slot ^ 1;
    return BEAM_OK;
}

int beam_moe_host_fence(beam_moe_t h, void *stream)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    cudaError_t e = cudaEventRecord(h->ev_fence, static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->copy_in, h->ev_fence, 0);
    return e == cudaSuccess ? BEAM_OK : cuda_fail(h, e, "fence of the host-buffer copies");
}

int beam_moe_host_join(beam_moe_t h, void *stream)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamWaitEvent(s, h->ev_out[0], 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, h->ev_out[1], 0);
    return e == cudaSuccess ? BEAM_OK : cuda_fail(h, e, "join of the host-buffer copies");
}

int beam_moe_forward_host(beam_moe_t h, void *stream, const void *x_host, int T, void *out_host,
                          float *residual_host, int k)
{
    int rc = beam_moe_forward_host_async(h, stream, x_host, T, out_host, residual_host, k);
    if (rc != BEAM_OK) return rc;
    if (T == 0) return BEAM_OK;
    rc = beam_moe_host_join(h, stream);
    if (rc != BEAM_OK) return rc;
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? BEAM_OK : cuda_fail(h, e, "host-buffer pass");
}

int beam_moe_dispatch_info(beam_moe_t h, void *stream, int T, int32_t *counts_host,
                           int32_t *offsets_host, int32_t *pair_row_host)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    h->err[0] = 0;
    if (T != h->last_T || T <= 0)
        return fail(h, BEAM_ERR_INVALID_ARG, "T=%d is not the T of the last forward pass (%d)", T,
                    h->last_T);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (counts_host)
        e = cudaMemcpyAsync(counts_host, h->counts, sizeof(int32_t) * h->E, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess && offsets_host)
        e = cudaMemcpyAsync(offsets_host, h->offsets, sizeof(int32_t) * (h->E + 1),
                            cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess && pair_row_host)
        e = cudaMemcpyAsync(pair_row_host, h->pair_row, sizeof(int32_t) * (size_t)T * h->top_k,
                            cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return e == cudaSuccess ? BEAM_OK : cuda_fail(h, e, "dispatch info copy");
}

int beam_moe_router_stats(beam_moe_t h, void *stream, int32_t *rederived_host)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    if (!rederived_host) return fail(h, BEAM_ERR_INVALID_ARG, "rederived_host is NULL");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(rederived_host, h->fix_count, sizeof(int32_t),
                                    cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    return e == cudaSuccess ? BEAM_OK : cuda_fail(h, e, "router stats copy");
}

int beam_moe_launch_plan(beam_moe_t h, int T, int32_t *plan_host)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    if (!plan_host) return fail(h, BEAM_ERR_INVALID_ARG, "plan_host is NULL");
    if (T < 0 || T > h->max_tokens)
        return fail(h, BEAM_ERR_INVALID_ARG, "T=%d outside [0, max_tokens=%d]", T, h->max_tokens);
    const ForwardPlan p = plan_forward(h, T);
    plan_host[0] = p.tile_rows;
    plan_host[1] = p.cta_pairs;
    plan_host[2] = p.grid;
    plan_host[3] = p.down_paired;
    plan_host[4] = p.router_tc;
    plan_host[5] = p.router_slices;
    plan_host[6] = p.gather;
    plan_host[7] = p.stream_k;
    plan_host[8] = p.stream_k;
    plan_host[9] = p.y_f32;
    plan_host[10] = p.gu_interleaved;
    return BEAM_OK;
}

int beam_moe_get_status(beam_moe_t h, void *stream)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int v[2] = {0, 0};   // the status word and the first index a check failed at
    cudaError_t e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemcpy(v, h->status, sizeof(v), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && v[0] != 0) e = cudaMemset(h->status, 0, sizeof(int));
    if (e == cudaSuccess && v[0] != 0) e = cudaMemset(h->check_where, 0x7f, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(h, e, "status read");
    if (v[0] == BEAM_ERR_CHECK)
        fail(h, v[0], "checked mode: validation failed at index %d (T*top_k: the dispatch tables)", v[1]);
    else if (v[0] != 0)
        fail(h, v[0], "device-side wait ran out (status %d)", v[0]);
    return v[0];
}

int beam_moe_set_checks(beam_moe_t h, int on)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    if (on < 0 || on > 1) return fail(h, BEAM_ERR_INVALID_ARG, "checks must be 0 or 1");
    h->checks = on;
    if (!on) h->corrupt_next = 0;
    return BEAM_OK;
}

int beam_moe_debug_corrupt_routing(beam_moe_t h, int passes)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    if (h->dense) return fail(h, BEAM_ERR_UNSUPPORTED, "a dense layer has no router");
    if (!h->checks) return fail(h, BEAM_ERR_INVALID_ARG, "corrupted routing needs checked mode");
    if (passes < 0) return fail(h, BEAM_ERR_INVALID_ARG, "passes < 0");
    h->corrupt_next = passes;
    return BEAM_OK;
}

int beam_moe_set_wait_limit(beam_moe_t h, int64_t limit_ns)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    if (limit_ns < 1000) return fail(h, BEAM_ERR_INVALID_ARG, "wait limit below 1000 ns");
    h->wait_limit_ns = limit_ns;
    return BEAM_OK;
}

static void prof_release(beam_moe *h)
{
    for (cudaEvent_t ev : h->prof_events) cudaEventDestroy(ev);
    h->prof_events.clear();
    h->prof_max = h->prof_calls = 0;
}

int beam_moe_profile_begin(beam_moe_t h, int max_calls)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    if (max_calls < 1 || max_calls > 100000)
        return fail(h, BEAM_ERR_INVALID_ARG, "max_calls outside [1, 100000]");
    int rc = check_device(h);
    if (rc != BEAM_OK) return rc;
    prof_release(h);
    h->prof_events.resize((size_t)max_calls * 6);
    for (auto &ev : h->prof_events) {
        cudaError_t e = cudaEventCreate(&ev);
        if (e != cudaSuccess) {
            ev = nullptr;
            prof_release(h);
            return cuda_fail(h, e, "cudaEventCreate");
        }
    }
    h->prof_max = max_calls;
    h->prof_calls = 0;
    return BEAM_OK;
}

int beam_moe_profile_end(beam_moe_t h, float *stage_ms, int *calls)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    if (!stage_ms || !calls) return fail(h, BEAM_ERR_INVALID_ARG, "output pointer is NULL");
    for (int i = 0; i < 5; ++i) stage_ms[i] = 0.f;
    *calls = h->prof_calls;
    if (h->prof_calls > 0) {
        cudaError_t e = cudaEventSynchronize(h->prof_events[(size_t)h->prof_calls * 6 - 1]);
        for (int c = 0; c < h->prof_calls && e == cudaSuccess; ++c)
            for (int i = 0; i < 5 && e == cudaSuccess; ++i) {
                float ms = 0.f;
                e = cudaEventElapsedTime(&ms, h->prof_events[(size_t)c * 6 + i],
                                         h->prof_events[(size_t)c * 6 + i + 1]);
                stage_ms[i] += ms;
            }
        if (e != cudaSuccess) {
            prof_release(h);
            return cuda_fail(h, e, "profile events");
        }
    }
    prof_release(h);
    return BEAM_OK;
}

int beam_moe_set_gemm_tuning(beam_moe_t h, int ctas, int tile_rows, int down_pair, int cta_pairs,
                             int router_mode, int gather_rows, int token_stages)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    if (ctas < 0 || ctas > 65535) return fail(h, BEAM_ERR_INVALID_ARG, "ctas outside [0, 65535]");
    if (tile_rows != 0 && !gemm_tile_supported(tile_rows))
        return fail(h, BEAM_ERR_INVALID_ARG, "tile_rows must be 0, 16, 32, 64, 128 or 256");
    if (down_pair < -1 || down_pair > 1)
        return fail(h, BEAM_ERR_INVALID_ARG, "down_pair outside [-1, 1]");
    if (cta_pairs < 0 || cta_pairs > 1) return fail(h, BEAM_ERR_INVALID_ARG, "cta_pairs must be 0 or 1");
    if (router_mode < -1 || router_mode > 2)
        return fail(h, BEAM_ERR_INVALID_ARG, "router_mode outside [-1, 2]");
    if (gather_rows < -1 || gather_rows > 1)
        return fail(h, BEAM_ERR_INVALID_ARG, "gather_rows outside [-1, 1]");
    if (token_stages != 0 && (token_stages < 2 || token_stages > 8))
        return fail(h, BEAM_ERR_INVALID_ARG, "token_stages must be 0 or in [2, 8]");
    h->token_stages = token_stages;
    h->router_mode = router_mode;
    h->gather_rows = gather_rows;
    h->gemm_ctas = ctas;
    h->tile_rows = tile_rows;
    h->down_pair = down_pair;
    h->use_pair = cta_pairs;
    return BEAM_OK;
}

int beam_moe_set_gate_up_layout(beam_moe_t h, int layout)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    if (layout < -1 || layout > 1) return fail(h, BEAM_ERR_INVALID_ARG, "layout outside [-1, 1]");
    h->gu_layout = layout;
    return BEAM_OK;
}

int beam_moe_check_wait_timeout(beam_moe_t h, void *stream)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    int rc = check_device(h);
    if (rc != BEAM_OK) return rc;
    WaitCtl ctl;
    ctl.status = h->status;
    ctl.limit_ns = h->wait_limit_ns;
    cudaError_t e = launch_wait_timeout_check(ctl, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(h, e, "self-check launch");
    const int first = beam_moe_get_status(h, stream);   // read and cleared
    e = launch_count_wait_check(ctl, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(h, e, "self-check launch");
    const int second = beam_moe_get_status(h, stream);
    return first != BEAM_ERR_TIMEOUT ? first : second;
}

const char *beam_moe_last_error(beam_moe_t h) { return h ? h->err : g_create_err; }

int beam_moe_destroy(beam_moe_t h)
{
    if (!h) return BEAM_ERR_INVALID_ARG;
    int prev = -1;
    cudaGetDevice(&prev);
    if (prev != h->device) cudaSetDevice(h->device);
    cudaError_t e = cudaDeviceSynchronize();
    prof_release(h);
    release_host_path(h);
    if (h->ws) cudaFree(h->ws);
    if (h->fp4_buf) cudaFree(h->fp4_buf);
    if (prev >= 0 && prev != h->device) cudaSetDevice(prev);
    delete h;
    return e == cudaSuccess ? BEAM_OK : BEAM_ERR_CUDA;
}

}  // extern "C"
