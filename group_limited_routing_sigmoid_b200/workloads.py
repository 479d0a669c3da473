"""Seeded synthetic workloads for the Beam MoE block.

This module holds shapes, distributions and a fixed draw order, and nothing
of the block's arithmetic.  Both the CUDA path (through the tests and the
benchmark) and the CPU oracle consume the tensors it draws; neither side
computes anything here.

Shapes come from the Beam pages: hidden 5120 and 256 SwiGLU experts of
intermediate size 2560 in 8 groups of 32, 4 groups kept, top-8, scaling 2.5
(launch blog "Introducing Beam", sections "Attention" and "Mixture of
Experts").  The pages publish no weights, so every tensor is random:

* x ~ N(0, 1) rounded to bf16;
* router weight fp32 ~ N(0, 1/H) (variance 1/H, so logits are ~N(0, 1));
* expert bias fp32 ~ U(lo, hi), optionally 16 "hot" experts (chosen by a
  seeded permutation) set to a fixed value;
* expert gate/up/down ~ N(0, 0.02^2) (std 0.02) rounded to bf16;
* post-norm weight fp32 ~ N(1, 0.02^2); residual stream fp32 ~ N(0, 1).

Draw order from one generator seeded with ``seed``: router weight, bias,
hot-expert permutation, then per expert (gate, up, down), then x, stream,
post-norm weight.  bf16 tensors are drawn in fp32 and rounded to nearest even
by ``Tensor.to(torch.bfloat16)``.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    hidden: int
    n_experts: int
    n_group: int
    topk_group: int
    top_k: int
    inter: int
    routed_scaling: float = 2.5
    bias_lo: float = -0.1
    bias_hi: float = 0.1
    hot_experts: int = 0
    hot_bias: float = 0.0
    post_norm: bool = False
    residual_k: int = 0          # 0: no residual update
    norm_eps: float = 1e-6
    expert_std: float = 0.02
    seed: int = 0
    sample: int = 0              # tokens the oracle checks (0 = all)
    weight_format: str = "bf16"  # "bf16" or "nvfp4" (expert weights)

    def with_tokens(self, T: int) -> "Workload":
        return replace(self, T=T)


_BEAM = dict(hidden=5120, n_experts=256, n_group=8, topk_group=4, top_k=8, inter=2560,
             routed_scaling=2.5)

WORKLOADS: Dict[str, Workload] = {
    # small block: H=256, 32 experts in 8 groups of 4, I=128
    "tiny": Workload("tiny", T=64, hidden=256, n_experts=32, n_group=8, topk_group=4, top_k=8,
                     inter=128),
    # small block whose weight rows split into 256-row blocks (H=512, I=256):
    # covers the CTA-pair GEMM path at sizes the oracle checks in full
    "small": Workload("small", T=1024, hidden=512, n_experts=32, n_group=8, topk_group=4, top_k=8,
                      inter=256),
    # Beam shape, decode batch of 64 tokens
    "decode": Workload("decode", T=64, **_BEAM),
    # Beam shape, prefill of 8192 tokens, near-uniform routing
    "prefill": Workload("prefill", T=8192, bias_lo=-0.01, bias_hi=0.01, sample=512, **_BEAM),
    # Beam shape, 8192 tokens, 16 experts carry bias +3.0
    "skewed": Workload("skewed", T=8192, hot_experts=16, hot_bias=3.0, sample=512, **_BEAM),
    # Beam shape, 32768 tokens, post-MoE RMSNorm + depth-scaled residual at step 20
    "long": Workload("long", T=32768, post_norm=True, residual_k=20, sample=512, **_BEAM),
    # profiling case: Beam-shaped experts (H=5120, I=2560), only 32 of them
    # (2.5 GB of weights), 8 tokens: the decode kernels on a few GB of memory
    "decode_small": Workload("decode_small", T=8, hidden=5120, n_experts=32, n_group=8,
                             topk_group=4, top_k=8, inter=2560),
    # profiling case: the same 32 Beam-shaped experts with 1024 tokens, i.e.
    # ~256 tokens per expert as in the 8192-token prefill
    "prefill_small": Workload("prefill_small", T=1024, hidden=5120, n_experts=32, n_group=8,
                              topk_group=4, top_k=8, inter=2560, bias_lo=-0.01, bias_hi=0.01),
    # dense SwiGLU MLP layers (the first three layers): one expert that every
    # token takes with weight 1, no routing and no routed scaling.  The pages
    # do not give the layers' intermediate size; 20480 (= 8 x 2560, the
    # routed width a token sees in a MoE layer) fits the pages' parameter
    # counts.  The router weight and bias are drawn (draw order) but unused.
    # (dense_tiny: K long enough that stream-K cuts tiles between CTAs)
    "dense_tiny": Workload("dense_tiny", T=64, hidden=1024, n_experts=1, n_group=1, topk_group=1,
                           top_k=1, inter=2048, routed_scaling=1.0),
    "dense_decode": Workload("dense_decode", T=64, hidden=5120, n_experts=1, n_group=1,
                             topk_group=1, top_k=1, inter=20480, routed_scaling=1.0),
    "dense_prefill": Workload("dense_prefill", T=8192, hidden=5120, n_experts=1, n_group=1,
                              topk_group=1, top_k=1, inter=20480, routed_scaling=1.0, sample=256),
    # NVFP4 expert weights (the 4-bit checkpoint format the pages recommend for
    # Blackwell): the same draws, quantised by nvfp4_quantize
    "tiny_nvfp4": Workload("tiny_nvfp4", T=64, hidden=256, n_experts=32, n_group=8, topk_group=4,
                           top_k=8, inter=128, weight_format="nvfp4"),
    "decode_nvfp4": Workload("decode_nvfp4", T=64, weight_format="nvfp4", **_BEAM),
    # profiling-sized NVFP4 case: 32 Beam-shaped experts (0.7 GB of weights), 8 tokens
    "decode_small_nvfp4": Workload("decode_small_nvfp4", T=8, hidden=5120, n_experts=32, n_group=8,
                                   topk_group=4, top_k=8, inter=2560, routed_scaling=2.5,
                                   weight_format="nvfp4"),
}


def generator(wl: Workload, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed)
    return g


def make_weights(wl: Workload, device, g: Optional[torch.Generator] = None) -> Dict[str, torch.Tensor]:
    """Router weight, bias and expert weights (draws 1-3 of the fixed order)."""
    if g is None:
        g = generator(wl, device)
    E, H, I = wl.n_experts, wl.hidden, wl.inter
    router_w = torch.randn(E, H, generator=g, device=device, dtype=torch.float32) * (1.0 / math.sqrt(H))
    bias = torch.rand(E, generator=g, device=device, dtype=torch.float32) * (wl.bias_hi - wl.bias_lo) + wl.bias_lo
    hot = None
    if wl.hot_experts:
        hot = torch.randperm(E, generator=g, device=device)[: wl.hot_experts]
        bias[hot] = wl.hot_bias
    w_gate = torch.empty(E, I, H, device=device, dtype=torch.bfloat16)
    w_up = torch.empty(E, I, H, device=device, dtype=torch.bfloat16)
    w_down = torch.empty(E, H, I, device=device, dtype=torch.bfloat16)
    for e in range(E):
        w_gate[e] = (torch.randn(I, H, generator=g, device=device) * wl.expert_std).to(torch.bfloat16)
        w_up[e] = (torch.randn(I, H, generator=g, device=device) * wl.expert_std).to(torch.bfloat16)
        w_down[e] = (torch.randn(H, I, generator=g, device=device) * wl.expert_std).to(torch.bfloat16)
    return dict(router_w=router_w.contiguous(), bias=bias.contiguous(), w_gate=w_gate, w_up=w_up,
                w_down=w_down, hot=hot)


E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def nvfp4_quantize(w: torch.Tensor, global_scale: float):
    """Round-to-nearest NVFP4 encoding of w [..., R, K] (K a multiple of 16)
    with the given per-tensor scale: one E4M3 scale per 16 elements (the
    block's absolute maximum / 6, over the tensor scale, rounded to E4M3 by
    torch's cast) and each element's nearest E2M1 magnitude and its sign.
    Returns codes uint8 [..., R, K/2] (element 2j in the low nibble of byte
    j) and scales uint8 [..., R, K/16].  This makes synthetic inputs; the
    block's arithmetic only ever decodes them."""
    *lead, K = w.shape
    blocks = w.float().reshape(*lead, K // 16, 16)
    bscale = (blocks.abs().amax(-1) / 6.0 / global_scale).to(torch.float8_e4m3fn)
    eff = bscale.float() * global_scale
    q = torch.where(eff[..., None] > 0, blocks / eff[..., None].clamp_min(1e-30), torch.zeros_like(blocks))
    mids = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], device=w.device)
    mag = torch.bucketize(q.abs().clamp(max=6.0), mids)
    code = (mag | ((q < 0).to(torch.int64) << 3)).reshape(*lead, K)
    packed = (code[..., 0::2] | (code[..., 1::2] << 4)).to(torch.uint8)
    return packed.contiguous(), bscale.view(torch.uint8).contiguous()


def nvfp4_global_scale(w: torch.Tensor) -> float:
    """The per-tensor scale that maps the tensor's absolute maximum to the
    largest NVFP4 value (6 x 448)."""
    amax = float(w.abs().max())
    return amax / (6.0 * 448.0) if amax > 0 else 1.0


def make_nvfp4_weights(wl: Workload, device, g: Optional[torch.Generator] = None) -> Dict[str, torch.Tensor]:
    """make_weights, then the expert tensors in NVFP4: {gate,up,down}_codes,
    _scales and _global (per tensor); the bf16 tensors are dropped."""
    d = make_weights(wl, device, g)
    for name in ("gate", "up", "down"):
        w = d.pop("w_" + name)
        gs = nvfp4_global_scale(w)
        codes, scales = [], []
        for e in range(w.shape[0]):        # per expert: bounded temporaries
            c, s = nvfp4_quantize(w[e], gs)
            codes.append(c)
            scales.append(s)
        d[name + "_codes"] = torch.stack(codes)
        d[name + "_scales"] = torch.stack(scales)
        d[name + "_global"] = gs
        del w
    return d


def make_tokens(wl: Workload, device, g: torch.Generator, T: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """x, then the residual stream and post-norm weight when the workload has them."""
    T = wl.T if T is None else T
    H = wl.hidden
    x = torch.randn(T, H, generator=g, device=device).to(torch.bfloat16)
    out = dict(x=x, stream=None, gamma=None)
    if wl.residual_k:
        out["stream"] = torch.randn(T, H, generator=g, device=device, dtype=torch.float32)
    if wl.post_norm:
        out["gamma"] = 1.0 + 0.02 * torch.randn(H, generator=g, device=device, dtype=torch.float32)
    return out


def make_inputs(wl: Workload, device) -> Dict[str, torch.Tensor]:
    """All tensors of a workload, in the fixed draw order, from one generator."""
    g = generator(wl, device)
    d = make_weights(wl, device, g)
    d.update(make_tokens(wl, device, g))
    return d


def sample_tokens(wl: Workload) -> torch.Tensor:
    """Tokens the oracle checks: all of them, or the first ``sample`` entries of a
    permutation of range(T) drawn on the CPU from seed + 1, sorted."""
    if not wl.sample or wl.sample >= wl.T:
        return torch.arange(wl.T)
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed + 1)
    return torch.sort(torch.randperm(wl.T, generator=g)[: wl.sample]).values


def bf16_bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (a view of the bytes; no arithmetic)."""
    assert t.dtype == torch.bfloat16, f"expected a bf16 tensor, got {t.dtype}"
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
