// Router entry point that allocates no device memory.
//
// Some callers cannot call cudaMalloc: an inference engine that reserves
// nearly all of the GPU's memory for its own pools at start-up and lets no
// library allocate beside it, or a latency-critical path that must not enter
// the CUDA allocator (cudaMalloc and cudaFree can synchronise the device).
// beam_moe_route_static serves them: the router's scratch (the per-slice
// partial logits) lives in the fixed device array below, which every GPU that
// loads this library holds until the process exits.  The caller passes only
// the inputs (tokens, router weight, bias) and the outputs.
#include <mutex>

#include "beam_moe.h"
#include "kernels.cuh"

namespace {
constexpr size_t kScratchFloats = (size_t)2 * 1024 * 1024;   // 8 MiB of partial logits
constexpr int kMaxDevices = 64;
}  // namespace

// Shared by every call on a device; keeps the last call's contents.
static __device__ __align__(256) float beam_route_scratch[kScratchFloats];

namespace {

std::mutex g_setup_mu;
float *g_scratch_ptr[kMaxDevices];   // device address of beam_route_scratch, per device
int g_num_sms[kMaxDevices];

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Once per device, with that device current: the array's device address.
// In host code the array's name is only a host-side stand-in, so the
// address must come from cudaGetSymbolAddress.
int scratch_for_current_device(float **scratch, int *num_sms)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return BEAM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return BEAM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, beam_route_scratch) != cudaSuccess || !p) return BEAM_ERR_CUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return BEAM_ERR_CUDA;
        g_num_sms[dev] = sms;
        g_scratch_ptr[dev] = static_cast<float *>(p);
    }
    *scratch = g_scratch_ptr[dev];
    *num_sms = g_num_sms[dev];
    return BEAM_OK;
}

}  // namespace

extern "C" int beam_moe_route_static(void *stream, const void *x, int T, int hidden, int n_experts,
                                     int n_group, int topk_group, int top_k, const float *router_w,
                                     const float *expert_bias, int32_t *topk_idx, float *topk_w)
{
    if (T < 0 || hidden <= 0 || hidden % 32 != 0 || n_experts <= 0 || n_group <= 0)
        return BEAM_ERR_INVALID_ARG;
    if (n_experts % n_group != 0 || n_experts / n_group < 2) return BEAM_ERR_INVALID_ARG;
    const int gsize = n_experts / n_group;
    if (topk_group < 1 || topk_group > n_group || top_k < 1 || top_k > topk_group * gsize)
        return BEAM_ERR_INVALID_ARG;
    if (n_experts % 32 != 0 || n_experts > 1024 || !is_pow2(n_experts / 32) || n_group > 32 ||
        top_k > 32)
        return BEAM_ERR_UNSUPPORTED;
    const int epl = n_experts / 32;
    if (gsize % epl != 0 || !is_pow2(gsize / epl)) return BEAM_ERR_UNSUPPORTED;
    if (T == 0) return BEAM_OK;
    if (!x || !router_w || !expert_bias || !topk_idx || !topk_w) return BEAM_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(router_w) || !aligned16(expert_bias))
        return BEAM_ERR_INVALID_ARG;
    if ((size_t)T * (size_t)n_experts > kScratchFloats) return BEAM_ERR_INVALID_ARG;

    float *scratch = nullptr;
    int num_sms = 0;
    int rc = scratch_for_current_device(&scratch, &num_sms);
    if (rc != BEAM_OK) return rc;

    beam::RouterArgs a;
    a.x = static_cast<const __nv_bfloat16 *>(x);
    a.router_w = router_w;
    a.bias = expert_bias;
    a.T = T;
    a.H = hidden;
    a.E = n_experts;
    a.n_group = n_group;
    a.topk_group = topk_group;
    a.top_k = top_k;
    a.nslice = beam::router_slices(T, hidden, n_experts, num_sms);
    while (a.nslice > 1 && (size_t)a.nslice * T * n_experts > kScratchFloats) a.nslice /= 2;
    a.partial = scratch;   // every element the selection reads is written first, in this call
    a.idx = topk_idx;
    a.w = topk_w;
    a.logits_out = nullptr;
    return beam::launch_router(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? BEAM_OK
                                                                                    : BEAM_ERR_CUDA;
}
