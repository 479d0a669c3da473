#!/usr/bin/env python
"""Benchmark of the Beam MoE block forward pass on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode]
                    [--impl ours|reference]

A step is one forward pass of the whole block (router, dispatch, gate|up
GEMM with SwiGLU, down GEMM, combine [+ post-norm and residual]) over one
batch of T synthetic tokens, with weights and tokens already in HBM.  Each
rank runs its own replica on its own batches (tokens are independent: weak
scaling, no data-path collective); ``value`` is all ranks' tokens over the
slowest rank's device time.

``--workload`` picks one of the seeded workloads: the Beam block at decode
(``decode``, the default) and prefill sizes, skewed routing, the long
sequence with post-norm and residual, the dense layers, and the same decode
batch with NVFP4 expert weights (``decode_nvfp4``, whose HBM roofline counts
0.5625 bytes per weight).

``--impl reference`` times the plain CPU oracle on the host cores instead,
one bounded sample of tokens per step (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from group_limited_routing_sigmoid_b200 import workloads as W  # noqa: E402

METRIC = "MoE-layer tokens/s (Beam shape, bf16) and % of HBM / tensor-core roofline"
# workloads whose dominant kernel streams weights (roofline against HBM)
HBM_BOUND = ("decode", "tiny", "decode_small", "dense_decode", "dense_tiny", "decode_nvfp4",
             "tiny_nvfp4", "decode_small_nvfp4")
TOKEN_BATCHES = 8           # distinct token batches cycled through the steps
MIN_WINDOWS = 5             # headline windows of --steps steps, at least
MAX_WINDOWS = 200
TIMED_SPAN_S = 2.0          # headline windows cover about this much device time
STAGE_WINDOWS = 7           # stage-timed windows (median per stage)
E2E_WINDOWS = 7             # host-buffer windows (median)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], bf16=p["bf16_tflops"], bf16_sus=p["bf16_tflops_sustained"],
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, sampled every 20 ms)
# ---------------------------------------------------------------------------
REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks",
           0x10: "sync_boost", 0x1: "gpu_idle"}


class ClockSampler:
    def __init__(self, cuda_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            phys = int(vis.split(",")[cuda_index]) if vis and vis.split(",")[0].isdigit() else cuda_index
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._reason_fn = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons")
        except Exception as e:  # NVML missing: report no clocks rather than guess
            self._nv = None
            self.error = str(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                bits = self._reason_fn(self._h)
                for b, name in REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.02)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def report(self):
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

# the sources of the bf16 grouped GEMMs: the default for a traffic entry
# that names no sources of its own
GEMM_SOURCES = ("grouped_gemm.cu", "grouped_gemm_pair.cu", "gemm_common.cuh", "common.cuh", "kernels.cuh")


def kernel_hash(files=GEMM_SOURCES) -> str:
    h = hashlib.sha256()
    for fn in files:
        with open(os.path.join(ROOT, "group_limited_routing_sigmoid_b200", "csrc", fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per launch of the gate|up GEMM from the committed ncu summary,
    scaled to this workload; None if absent or taken on other kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    entry = t.get(workload)
    if not entry or entry.get("kernel_hash") != kernel_hash(tuple(entry.get("sources", GEMM_SOURCES))):
        return None
    return entry.get("dram_bytes_per_launch")


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def token_seed(wl: W.Workload, rank: int) -> int:
    """Seed of a rank's token batches: every rank shares the weights (seed
    wl.seed) and draws its own tokens."""
    return wl.seed + 1000 * (rank + 1)


def max_over_ranks(value: float, dist, device) -> float:
    """The slowest rank's time (all ranks take this collective step)."""
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_config(name: str, wl) -> dict:
    """The workload's identity and shape (the same keys on both arms)."""
    return {"workload": f"beam_{name}", "T": wl.T, "hidden": wl.hidden, "n_experts": wl.n_experts,
            "n_group": wl.n_group, "topk_group": wl.topk_group, "top_k": wl.top_k,
            "inter": wl.inter, "routed_scaling": wl.routed_scaling, "residual_k": wl.residual_k,
            "post_norm": wl.post_norm, "expert_weights": wl.weight_format}


def kernels_per_forward(plan: dict, dense: bool, residual: bool, pairs: int, n_experts: int) -> int:
    """Kernels of this library one forward pass launches, from its launch plan."""
    if dense:
        # table set-up, gate|up, down, combine (only for the residual update)
        return 1 + 1 + 1 + int(residual)
    # router: logits + selection (CUDA cores) or tensor-core logits, selection,
    # exact re-derivation, selection of the re-derived tokens; dispatch:
    # count, scan, permute or row maps, or one block for at most 1024 pairs
    # when the GEMM gathers its token rows; the two GEMMs; combine
    one_block = plan["gather_rows"] == 1 and pairs <= 1024 and n_experts <= 1024
    return (4 if plan["router_tensor_cores"] else 2) + (1 if one_block else 3) + 2 + 1


def expert_weight_bytes(wl) -> float:
    """Bytes per expert weight as stored: bf16, or NVFP4 (4-bit element plus
    an 8-bit scale per 16 elements)."""
    return 0.5625 if wl.weight_format == "nvfp4" else 2.0


def make_weights(wl, dev, g):
    return W.make_nvfp4_weights(wl, dev, g) if wl.weight_format == "nvfp4" else W.make_weights(wl, dev, g)


def whole_job_tokens_per_s(world: int, steps: int, T: int, ms_max: float) -> float:
    """All ranks' tokens over the slowest rank's device time."""
    return world * steps * T / (ms_max * 1e-3)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import torch.distributed as dist
    from group_limited_routing_sigmoid_b200.build import build
    from group_limited_routing_sigmoid_b200.binding import BeamMoE

    ws, rank, local = dist_env()
    if ws != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={ws}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    if rank == 0 or ws == 1:
        build(quiet=True)
    if ws > 1:
        dist.barrier()

    wl = W.WORKLOADS[args.workload]
    T, H, I, E, k = wl.T, wl.hidden, wl.inter, wl.n_experts, wl.top_k
    g = W.generator(wl, dev)
    weights = make_weights(wl, dev, g)
    wb = expert_weight_bytes(wl)
    # distinct token batches per rank (weights identical on every rank)
    tg = torch.Generator(device=dev)
    tg.manual_seed(token_seed(wl, rank))
    batches = [W.make_tokens(wl, dev, tg) for _ in range(TOKEN_BATCHES)]
    if wl.post_norm:
        weights["gamma"] = batches[0]["gamma"]
    moe = BeamMoE.from_workload(wl, weights)
    moe.set_gemm_tuning(0, args.gemm_tile, args.down_pair, args.cta_pairs, args.router, args.gather,
                        args.token_stages)
    outs = [torch.empty(T, H, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    streams = [b["stream"] for b in batches]

    # distinct experts each batch touches (for the algorithmic byte count);
    # a dense layer is one expert that every token takes
    dense = E == 1
    distinct = []
    for b in batches:
        if dense:
            distinct.append(1)
            continue
        idx, _ = moe.route(b["x"])
        distinct.append(int((torch.bincount(idx.reshape(-1).long(), minlength=E) > 0).sum()))
    torch.cuda.synchronize(dev)

    def step(i):
        b = batches[i % TOKEN_BATCHES]
        if wl.residual_k:
            moe.forward(b["x"], out=outs[i & 1], residual=streams[i % TOKEN_BATCHES], k=wl.residual_k)
        else:
            moe.forward(b["x"], out=outs[i & 1])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    assert moe.get_status() == 0

    stream = torch.cuda.current_stream(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def window(first: int, n: int, fn) -> float:
        """Device time (ms) of n steps fn(first + i), bracketed by a barrier
        and a synchronize on both sides; the slowest rank's time."""
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        for i in range(n):
            fn(first + i)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        if ws > 1:
            dist.barrier()
        return max_over_ranks(ev0.elapsed_time(ev1), dist, dev)

    # headline: windows of exactly --steps steps each, enough of them (at
    # least MIN_WINDOWS) that the timed span covers TIMED_SPAN_S seconds of
    # clock samples; every rank takes the same number (decided from the
    # slowest rank's first window)
    sampler = ClockSampler(local)
    win_ms = []
    with sampler:
        win_ms.append(window(args.warmup, args.steps, step))
        n_win = max(MIN_WINDOWS, min(MAX_WINDOWS, int(TIMED_SPAN_S * 1e3 / max(win_ms[0], 1e-3)) + 1))
        if args.windows > 0:
            n_win = max(MIN_WINDOWS, args.windows)
        for w in range(1, n_win):
            win_ms.append(window(args.warmup + w * args.steps, args.steps, step))
    rederived = moe.router_stats()
    if moe.get_status() != 0:
        raise SystemExit("a device-side wait ran out during the timed region")
    ms_max = statistics.median(win_ms)

    # per-stage device times: windows of the same steps again with the
    # library's CUDA events around each stage (kept out of the headline
    # region: an event between two kernels stops the second from starting
    # early); each stage's per-launch time is the median over the windows
    stage_steps = min(args.steps, 50)
    stage_windows = []
    for w in range(min(n_win, STAGE_WINDOWS)):
        moe.profile_begin(stage_steps)
        for i in range(stage_steps):
            step(args.warmup + i)
        calls, st = moe.profile_end()
        stage_windows.append({kname: v / max(calls, 1) for kname, v in st.items()})
    if moe.get_status() != 0:
        raise SystemExit("a device-side wait ran out during the stage-timed steps")
    stage_med = {kname: statistics.median(sw[kname] for sw in stage_windows) for kname in stage_windows[0]}

    # end to end through the host-buffer entry points (pinned buffers): each
    # step copies its batch in and its result out; the pipelined call lets a
    # step's copies overlap its neighbours' compute
    x_host = [b["x"].cpu().pin_memory() for b in batches]
    out_host = [torch.empty(T, H, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    res_host = [s.cpu().pin_memory() for s in streams] if wl.residual_k else None
    e2e_steps = max(3, min(args.steps, 50))

    def e2e_step(i):
        j = i % TOKEN_BATCHES
        moe.forward_host_async(x_host[j], out_host=out_host[i & 1],
                               residual_host=res_host[j] if res_host else None,
                               k=max(1, wl.residual_k))

    def e2e_window(first: int, n: int) -> float:
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        moe.host_fence()          # the first copy in starts after ev0
        for i in range(n):
            e2e_step(first + i)
        moe.host_join()           # ev1 after the last copy out
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        if ws > 1:
            dist.barrier()
        return max_over_ranks(ev0.elapsed_time(ev1), dist, dev)

    for i in range(args.warmup):
        e2e_step(i)
    moe.host_join()
    e2e_win = [e2e_window(w * e2e_steps, e2e_steps) for w in range(min(n_win, E2E_WINDOWS))]
    e2e_ms = statistics.median(e2e_win)

    # roofline of the dominant kernel
    pk = peaks()
    steps_done = args.steps
    d_mean = sum(distinct[(args.warmup + i) % TOKEN_BATCHES] for i in range(stage_steps)) / stage_steps
    P = T * k
    gate_up_ms = stage_med["gate_up_gemm"]
    if args.workload in HBM_BOUND:
        alg_bytes = d_mean * 2 * I * H * wb + P * H * 2 + P * I * 2
        achieved = alg_bytes / (gate_up_ms * 1e-3) / 1e9
        roof = {"bound": "hbm",
                "achieved": round(achieved, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4), "peak_source": pk["source"],
                "algorithmic_bytes_per_launch": int(alg_bytes), "launch_ms": round(gate_up_ms, 4)}
    else:
        flops = 4.0 * H * I * P
        achieved = flops / (gate_up_ms * 1e-3) / 1e12
        roof = {"bound": "tensor",
                "achieved": round(achieved, 1), "peak": pk["bf16_sus"], "unit": "TFLOP/s",
                "frac": round(achieved / pk["bf16_sus"], 4), "peak_source": pk["source"] + " sustained",
                "algorithmic_flops_per_launch": flops, "launch_ms": round(gate_up_ms, 4)}
    plan = moe.launch_plan(T)
    if plan["stream_k_gate_up"]:
        roof["kernel"] = ("gate_up_gemm (dense_sk_kernel<%d,true>, stream-K, grid %d)"
                          % (plan["tile_rows"], plan["grid"]))
    elif wl.weight_format == "nvfp4":
        roof["kernel"] = ("gate_up_gemm (grouped_gemm_fp4_kernel<%d,2,0>, NVFP4 weights, grid %d)"
                          % (plan["tile_rows"], plan["grid"]))
    else:
        roof["kernel"] = ("gate_up_gemm (grouped_gemm_pair_kernel<%d,2,0>, CTA pairs, grid %d)"
                          if plan["cta_pairs"] else
                          "gate_up_gemm (grouped_gemm_kernel<%d,2,0>, grid %d)") % (plan["tile_rows"], plan["grid"])
    roof["traffic"] = ncu_traffic(args.workload)
    # the nominal datasheet peaks beside the measured ones (context, not the denominator)
    nominal = 8000.0 if roof["bound"] == "hbm" else 2250.0
    roof["nominal_peak"] = nominal
    roof["frac_of_nominal"] = round(roof["achieved"] / nominal, 4)
    timed = n_win * steps_done
    d_steps = sum(distinct[(args.warmup + i) % TOKEN_BATCHES] for i in range(timed)) / timed
    step_bytes = (d_steps * 3 * H * I * wb + (0 if dense else E * H * 4) + T * H * 4
                  + (T * H * 8 if wl.residual_k else 0))
    stage_avg = {kname: round(v, 4) for kname, v in stage_med.items()}
    gu = sorted(sw["gate_up_gemm"] for sw in stage_windows)
    roof["launch_ms_min"], roof["launch_ms_max"] = round(gu[0], 4), round(gu[-1], 4)
    roof["launch_ms_windows"] = len(gu)

    line = {
        "metric": METRIC,
        "value": round(whole_job_tokens_per_s(ws, steps_done, T, ms_max), 1),
        "unit": "tokens/s",
        "n_gpus": ws,
        "steps": steps_done,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max / steps_done, 4),
        "ms_per_step_min": round(min(win_ms) / steps_done, 4),
        "ms_per_step_max": round(max(win_ms) / steps_done, 4),
        "windows": n_win,
        "timing": (f"median of {n_win} windows of {steps_done} steps, each bracketed by a barrier "
                   f"and a synchronize; CUDA events on the launching stream; max over ranks per window"),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded random weights and tokens of the Beam block shape)",
        "config": {**workload_config(args.workload, wl), "token_batches": TOKEN_BATCHES,
                   "distinct_experts_per_step": round(d_steps, 2),
                   "l2": f"inputs larger than L2: each step streams {d_steps * 3 * H * I * wb / 1e9:.1f} GB of expert weights",
                   "parallelism": f"{ws} independent replicas (data parallel, no collective on the data path)"},
        "hbm_fraction_whole_step": round(step_bytes / (ms_max / steps_done * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
        "stage_ms": stage_avg,
        "router_tokens_rederived_last_step": rederived,
        "clocks": sampler.report(),
        "e2e": {"value": round(whole_job_tokens_per_s(ws, e2e_steps, T, e2e_ms), 1), "unit": "tokens/s",
                "windows": len(e2e_win), "steps_per_window": e2e_steps,
                "h2d_bytes_per_step": T * H * 2 + (T * H * 4 if wl.residual_k else 0),
                "d2h_bytes_per_step": T * H * 2 + (T * H * 4 if wl.residual_k else 0)},
        "gpu_launches": kernels_per_forward(plan, dense, bool(wl.residual_k), wl.T * wl.top_k, wl.n_experts) * steps_done * n_win,
        "gpu_launches_per_step": kernels_per_forward(plan, dense, bool(wl.residual_k), wl.T * wl.top_k, wl.n_experts),
        "roofline": roof,
        "launch_plan": plan,
    }
    if ws == 1 and not args.no_cpu_baseline:
        pool = torch.cat([b["x"] for b in batches])
        # the NVFP4 oracle decodes every weight it touches: a quarter of the
        # sample keeps it near the bf16 workloads' CPU time
        n_cpu = args.cpu_tokens if wl.weight_format != "nvfp4" else max(1, args.cpu_tokens // 4)
        line["cpu_baseline"] = cpu_baseline(wl, weights, pool, min(n_cpu, pool.shape[0]))
    if rank == 0:
        print(json.dumps(line), flush=True)
    moe.close()
    if ws > 1:
        dist.barrier()
        dist.destroy_process_group()


def _oracle_on_tokens(wl, weights, x, n_tokens):
    """Time the oracle on the first n_tokens of x (expert weights copied to
    the host before the clock starts)."""
    import oracle
    oracle.build()
    xs = W.bf16_bits(x[:n_tokens])
    gamma = None if weights.get("gamma") is None else weights["gamma"].cpu().numpy()
    stream = torch.zeros(n_tokens, wl.hidden).numpy() if wl.residual_k else None
    if wl.n_experts == 1:   # a dense layer: no routing
        wg, wu, wd = (W.bf16_bits(weights[k][0]) for k in ("w_gate", "w_up", "w_down"))
        t0 = time.perf_counter()
        oracle.dense_block(xs, wg, wu, wd, gamma=gamma, eps=wl.norm_eps, stream=stream,
                           kstep=wl.residual_k)
        return time.perf_counter() - t0
    rw = weights["router_w"].cpu().numpy()
    bias = weights["bias"].cpu().numpy()
    r = oracle.route(xs, rw, bias, wl.n_group, wl.topk_group, wl.top_k)
    cache = {}
    for e in sorted(set(int(v) for v in r.idx.reshape(-1))):
        if wl.weight_format == "nvfp4":
            cache[e] = tuple(oracle.Nvfp4Matrix(weights[n + "_codes"][e].cpu().numpy(),
                                                weights[n + "_scales"][e].cpu().numpy(),
                                                weights[n + "_global"]) for n in ("gate", "up", "down"))
        else:
            cache[e] = (W.bf16_bits(weights["w_gate"][e]), W.bf16_bits(weights["w_up"][e]),
                        W.bf16_bits(weights["w_down"][e]))
    t0 = time.perf_counter()
    oracle.moe_block(xs, rw, bias, cache.__getitem__, wl.n_group, wl.topk_group, wl.top_k,
                     wl.routed_scaling, gamma=gamma, eps=wl.norm_eps, stream=stream, kstep=wl.residual_k)
    return time.perf_counter() - t0


def cpu_baseline(wl, weights, x, n_tokens):
    import oracle
    sec = _oracle_on_tokens(wl, weights, x, n_tokens)
    return {"value": round(n_tokens / sec, 3), "unit": "tokens/s", "cores": oracle.threads(),
            "kind": "oracle",
            "sample": f"the first {n_tokens} tokens of the bench's token batches, all {wl.top_k} "
                      f"experts each, fp64 oracle ({sec:.1f} s)"}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle on the host cores
# ---------------------------------------------------------------------------

def run_reference(args):
    ws, rank, local = dist_env()
    if rank != 0:
        return
    import oracle
    wl = W.WORKLOADS[args.workload]
    dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    g = W.generator(wl, dev)
    weights = make_weights(wl, dev, g)
    tg = torch.Generator(device=dev)
    tg.manual_seed(token_seed(wl, 0))
    x = W.make_tokens(wl, dev, tg)["x"]
    if wl.post_norm:
        weights["gamma"] = 1.0 + 0.02 * torch.randn(wl.hidden, generator=tg, device=dev)
    per_step = 1
    times = []
    for i in range(args.warmup + args.steps):
        j = i % wl.T
        sec = _oracle_on_tokens(wl, weights, x[j:j + 1].contiguous(), per_step)
        if i >= args.warmup:
            times.append(sec)
    total = sum(times)
    value = round(args.steps * per_step / total, 4)
    line = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded random weights and tokens of the Beam block shape)",
        "config": workload_config(args.workload, wl),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads(), "kind": "oracle",
                         "sample": f"{per_step} token per step (all {wl.top_k} experts), tokens "
                                   f"cycled through one {wl.T}-token batch"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=128,
                    help="tokens in the CPU-baseline sample (about 10 s of oracle work at the decode shape)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--windows", type=int, default=0,
                    help="headline windows (0 = enough for about 2 s of device time; at least 5)")
    ap.add_argument("--gemm-tile", type=int, default=0, help="largest GEMM token tile (0 = auto)")
    ap.add_argument("--gather", type=int, default=-1,
                    help="gate|up token rows gathered from x: -1 auto (tiles <= 32 rows), 0 never, 1 always")
    ap.add_argument("--token-stages", type=int, default=0,
                    help="CTA-pair GEMMs: token-row ring depth (0 = default 3)")
    ap.add_argument("--down-pair", type=int, default=-1, help="paired down tiles: -1 auto, 0, 1")
    ap.add_argument("--cta-pairs", type=int, default=1, help="SM-pair GEMMs for large tiles: 1 or 0")
    ap.add_argument("--router", type=int, default=-1, help="router logits: -1 auto, 0 CUDA cores, 1 tensor cores")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
