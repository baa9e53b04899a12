#!/usr/bin/env python
"""Throughput of the MoE FFN layer forward on B200.

One step = one ``moe_forward`` over a batch of T tokens (router GEMM + softmax/
top-k, histogram/scan/permute, grouped expert GEMMs, shared experts, combine),
inputs already resident in HBM. Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--workloads LIST|all|none] [--impl ours|reference]

Every fourth timed step records CUDA events at the start of its expert FFNs and of
its combine (``moe_forward_staged``), so the expert GEMMs' time comes from the
timed steps themselves; the same number of steps follows with an event at every stage
boundary, for the per-stage breakdown. After the headline workload the other workloads of the layer run
the same way, each reported under ``workloads``.

Multi-GPU (torchrun, one rank per GPU): every rank runs the same layer on its
own batch of T tokens (weak scaling, no data-path collective); the elapsed time
is the max over ranks. With N > 1 the token-sharded layer also runs: one batch
of N x T Switch-layer tokens split over the ranks, with the all-gather of the
pre-drop counts and the all-reduce of the statistics sums inside its timed
steps (``sharded``).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from sparse_mixture_experts_12_b200 import synth  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# datasheet dense peaks of a B200 (HGX), reported beside the measured denominators
NOMINAL_PEAKS = {"hbm_gbs": 7700.0, "bf16_tflops": 2250.0}
METRIC = "MoE-layer tokens/s"
STAGES = ("route", "scan", "permute", "shared_ffn", "expert_ffn", "combine")
# the workloads reported under "workloads" after the headline one (bench --workloads all)
SIDE_WORKLOADS = ("tiny", "deepseek", "switch", "decode32", "decode8", "decode1",
                  "mixtral_ec", "mixtral_noisy")
L2_BYTES = 126 * 1024 * 1024
FLUSH_BYTES = 2 * L2_BYTES  # a write of this many bytes evicts the L2


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks sampler
class ClockSampler:
    """Polls the GPU's SM clock and clock-event reasons through NVML every 5 ms
    (read-only queries) while the timed region runs."""

    # NVML clock-event reason bits (nvmlClocksEventReason*)
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device: int):
        self.samples: list = []
        self.nv = None
        self.mark = None
        self.max_mhz = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.h = nv.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM))
            self.nv = nv
        except Exception as e:  # no NVML: clocks are reported as unknown
            log(f"clock sampler unavailable: {e}")

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return int(fn(self.h))

    def _poll(self):
        while not self.done.is_set():
            try:
                sm = float(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.samples.append((time.time(), sm, self._reasons()))
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        if self.nv is None:
            return
        self.done = threading.Event()
        self.thread = threading.Thread(target=self._poll, daemon=True)
        self.thread.start()

    def begin_load(self):
        self.mark = time.time()

    def stop(self):
        end = time.time()
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": "unavailable"}
        self.done.set()
        self.thread.join(timeout=2)
        rows = [(sm, r) for (t, sm, r) in self.samples if self.mark is None or self.mark <= t <= end]
        if not rows:  # a region shorter than the poll period: the first sample after it began
            rows = [(sm, r) for (t, sm, r) in self.samples if self.mark is None or t >= self.mark][:1]
        reasons = sorted({n for (_, r) in rows for n, b in self.REASON_BITS.items() if r & b})
        sm = [x for (x, _) in rows]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(sm), "source": "NVML, 5 ms polling"}


# ----------------------------------------------------------- multi-rank plumbing
def dist_env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 when absent)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int, device=None) -> float:
    """The slowest rank's value: the job takes as long as its last rank."""
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def tokens_per_second(T: int, world: int, steps: int, ms: float) -> float:
    """Whole-job throughput: every rank processes its own batch of T tokens per step."""
    return T * world * steps / (ms / 1000.0)


# ---------------------------------------------------------------- oracle helpers
def oracle_params_f64(inp: dict) -> dict:
    """Every input upcast to fp64 numpy once, so that the timed oracle calls do only
    the oracle's own arithmetic (input marshalling, not part of the method)."""
    return {k: (None if v is None else v.to(torch.float64).numpy()) for k, v in inp.items()}


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample_rate(wl, P, n_tokens: int):
    """Time the CPU oracle as it stands: routing of all T tokens (capacity needs the
    whole batch's order) plus the expert FFNs of ``n_tokens`` strided tokens (tokens
    are independent once routed). P holds fp64 inputs. Returns (tokens/s estimate
    for the full workload, description, seconds of CPU work)."""
    from oracle import moe_oracle as O

    acts = {0: "relu", 1: "gelu", 2: "swiglu"}
    modes = {0: "topk_softmax", 1: "softmax_topk_renorm", 2: "softmax_topk_raw"}
    toks = synth.token_sample(wl.T, n_tokens).numpy()
    if wl.routing == synth.ROUTING_EXPERT_CHOICE:
        t0 = time.perf_counter()
        logits = O.router_logits(P["x"], P["w_router"], P.get("b_router"), P.get("logit_bias"))
        O.expert_choice_select(logits, O.expert_choice_capacity(wl.capacity_factor, wl.T,
                                                                wl.n_experts))
        t_route = time.perf_counter() - t0
        t0 = time.perf_counter()
        O.expert_choice_forward(P["x"], P, capacity_factor=wl.capacity_factor,
                                act=acts[wl.act], logits=logits, tokens=toks)
        t_ffn = time.perf_counter() - t0  # includes the (cheap) re-selection
        kind = "expert choice"
    else:
        kw = dict(top_k=wl.top_k, act=acts[wl.act], gate_mode=modes[wl.gate_mode],
                  capacity_factor=wl.capacity_factor, n_shared=wl.n_shared)
        t0 = time.perf_counter()
        noisy = None
        if wl.noisy:  # the counter-based draws of the GPU arm's first step
            eps = O.noise_draws(wl.T, wl.n_experts, 1234, 1)[0]
            noisy = O.noisy_router_logits(P["x"], P["w_router"], P["w_noise"], eps,
                                          P.get("b_router"), P.get("logit_bias"))
        r = O.route(P["x"], P, top_k=wl.top_k, gate_mode=kw["gate_mode"],
                    capacity_factor=wl.capacity_factor, logits=noisy)
        t_route = time.perf_counter() - t0
        t0 = time.perf_counter()
        O.moe_forward(P["x"], P, tokens=toks, logits=r["logits"], **kw)
        t_ffn = time.perf_counter() - t0  # includes the (cheap) re-selection
        kind = "token choice"
    per_token = t_route / wl.T + t_ffn / len(toks)
    desc = (f"oracle (numpy fp64, inputs upcast once outside the timing), {kind}: routing "
            f"of all {wl.T} tokens ({t_route:.2f} s) + expert FFNs of {len(toks)} strided "
            f"tokens ({t_ffn:.2f} s); tokens/s = 1 / (t_route/T + t_ffn/n)")
    return 1.0 / per_token, desc, t_route + t_ffn


# ---------------------------------------------------------------- the reference arm
def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    inp = synth.generate(wl, seed=0)
    P = oracle_params_f64(inp)
    n = args.ref_sample
    for _ in range(args.warmup):
        oracle_sample_rate(wl, P, n)
    rates, secs = [], 0.0
    desc = ""
    for _ in range(args.steps):
        r, desc, s = oracle_sample_rate(wl, P, n)
        rates.append(1.0 / r)
        secs += s
    value = len(rates) / sum(rates)
    cores = _oracle_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * secs / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": _config(wl, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _config(wl, world):
    return {"workload": wl.name, "T": wl.T, "d_model": wl.d_model, "n_experts": wl.n_experts,
            "top_k": wl.top_k, "d_ff": wl.d_ff, "n_shared": wl.n_shared,
            "d_ff_shared": wl.d_ff_shared, "capacity_factor": wl.capacity_factor,
            "routing": ("expert choice" if wl.routing == synth.ROUTING_EXPERT_CHOICE
                        else "token choice") + (", noisy gating" if wl.noisy else ""),
            "global_batch": wl.T * world, "seq_len": wl.T,
            "parallelism": f"dp{world} (independent token batches, no data-path collective)",
            "l2": "working set > L2 (weights >= 2.8 GB per step); no flush"}


def _traffic(workload_name):
    """DRAM bytes per expert-FFN call (all its kernel launches) from the committed ncu
    summary, valid only while every kernel source it lists is unchanged since the
    capture; None otherwise."""
    p = os.path.join(ROOT, "profiles", "ffn_traffic.json")
    if not os.path.exists(p):
        return None
    try:
        with open(p) as f:
            ent = json.load(f).get(workload_name)
        if ent is None:
            return None
        for rel, sha in ent["sources"].items():
            with open(os.path.join(ROOT, rel), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != sha:
                    return None
        return ent["dram_bytes_per_call"]
    except (OSError, ValueError, KeyError, TypeError):
        return None


def kernels_per_step(step, dev) -> int:
    """Kernel launches of one step, counted from a CUDA-graph capture of it (the
    graph is built, its kernel nodes counted, and destroyed without running)."""
    from cuda.bindings import runtime as cudart

    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream())
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        (e,) = cudart.cudaStreamBeginCapture(
            s.cuda_stream, cudart.cudaStreamCaptureMode.cudaStreamCaptureModeThreadLocal)
        if e != cudart.cudaError_t.cudaSuccess:
            raise RuntimeError(f"stream capture: {e}")
        try:
            step()
        finally:
            e, graph = cudart.cudaStreamEndCapture(s.cuda_stream)
    if e != cudart.cudaError_t.cudaSuccess:
        raise RuntimeError(f"stream capture: {e}")
    try:
        e, _, n = cudart.cudaGraphGetNodes(graph, 0)
        e, nodes, n = cudart.cudaGraphGetNodes(graph, n)
        kernels = 0
        for node in nodes[:n]:
            e, kind = cudart.cudaGraphNodeGetType(node)
            kernels += kind == cudart.cudaGraphNodeType.cudaGraphNodeTypeKernel
        return int(kernels)
    finally:
        cudart.cudaGraphDestroy(graph)


# ------------------------------------------------------ algorithmic work per stage
def routing_stats(wl, counts, offsets) -> dict:
    """Rows kept, touched experts and pre-drop loads of one step's routing."""
    counts = np.asarray(counts)
    kept = np.diff(np.asarray(offsets))
    return {"rows_kept": int(kept.sum()), "touched_experts": int((kept > 0).sum()),
            "dropped": int(counts.sum() - kept.sum()),
            "max_expert_load": int(counts.max()), "min_expert_load": int(counts.min())}


def stage_work(wl, rs, want_aux: bool) -> dict:
    """Algorithmic bytes (HBM side) or flops (expert FFN) of each stage of one step:
    what the method must read and write once, not what a kernel happens to move.
    rs: routing_stats; tokens_read = tokens with at least one kept slot."""
    b = wl.elem_bytes
    T, d, E, k, F = wl.T, wl.d_model, wl.n_experts, wl.top_k, wl.d_ff
    R = rs["rows_kept"]
    ec = wl.routing == synth.ROUTING_EXPERT_CHOICE
    n_proj = 2 if wl.noisy else 1
    # router: x and W_r (and W_noise) read, selection (+ logits) written
    route = n_proj * (T * d * b + E * d * b) + T * k * 8
    if want_aux or wl.noisy or ec:
        route += T * E * 4 * (3 if wl.noisy else 1)
    # permute: each token with a kept slot read once, every kept row written
    permute = rs.get("tokens_read", T) * d * b + R * d * b + T * k * 12
    # combine: kept rows read, y written (+ the shared experts' fp32 rows)
    combine = R * d * b + T * d * b + T * k * 8 + (T * d * 4 if wl.n_shared else 0)
    n_mats = 3 if wl.act == synth.ACT_SWIGLU else 2
    flops = 2.0 * R * n_mats * d * F
    w_bytes = rs["touched_experts"] * n_mats * d * F * b
    ffn_bytes = w_bytes + 2.0 * R * d * b
    sh_flops = sh_bytes = 0.0
    if wl.n_shared:
        Fs = wl.n_shared * wl.d_ff_shared
        sh_flops = 2.0 * T * 3 * d * Fs
        sh_bytes = 3.0 * d * Fs * b + T * d * b + T * d * 4
    return {"route": {"bytes": route}, "permute": {"bytes": permute},
            "combine": {"bytes": combine},
            "expert_ffn": {"flops": flops, "bytes": ffn_bytes},
            "shared_ffn": {"flops": sh_flops, "bytes": sh_bytes}}


def ffn_roofline(wl, work, ffn_ms, peaks, peaks_src):
    """Roofline of the grouped expert GEMMs (routed + shared experts) from their
    stage time inside the timed steps: tensor-bound when the arithmetic intensity
    is above the ridge of the measured peaks, HBM-bound below it."""
    flops = work["expert_ffn"]["flops"] + work["shared_ffn"]["flops"]
    byts = work["expert_ffn"]["bytes"] + work["shared_ffn"]["bytes"]
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if wl.dtype == synth.DT_BF16 and flops / byts >= ridge:
        roof = {"bound": "tensor", "achieved": flops / (ffn_ms * 1e-3) / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
        sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        roof["frac_of_sustained"] = roof["achieved"] / sus
        roof["peak_source"] = f"{peaks_src} (burst: the timed region is under a second)"
    else:
        roof = {"bound": "hbm", "achieved": byts / (ffn_ms * 1e-3) / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "peak_source": f"{peaks_src} (copy)"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    nominal = NOMINAL_PEAKS["bf16_tflops" if roof["bound"] == "tensor" else "hbm_gbs"]
    roof["nominal_peak"] = nominal
    roof["frac_of_nominal"] = roof["achieved"] / nominal
    roof["ms_per_step"] = ffn_ms
    roof["algorithmic"] = {"flops": flops, "bytes": byts}
    return roof


def stage_report(work, stage_ms, peaks) -> dict:
    """Per-stage device time per step, with the HBM fraction of the bandwidth-bound
    stages (algorithmic bytes / time against the measured copy bandwidth)."""
    out = {}
    for name, ms in zip(STAGES, stage_ms):
        ent = {"ms": ms}
        w = work.get(name)
        if w is not None and "flops" not in w and ms > 0:
            gbs = w["bytes"] / (ms * 1e-3) / 1e9
            ent.update({"bytes": w["bytes"], "gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"]})
        out[name] = ent
    return out


# ------------------------------------------------------------ timing of one layer
class StepTimer:
    """K steps with events at every stage boundary (moe_forward_staged) and around
    the loop. flush: an L2-evicting write between steps (outside the stage events),
    for workloads whose working set fits in L2."""

    def __init__(self, steps: int):
        self.steps = steps
        self.ev = [_made_events(len(STAGES) + 1) for _ in range(steps)]
        self.e0 = torch.cuda.Event(enable_timing=True)
        self.e1 = torch.cuda.Event(enable_timing=True)

    def run(self, step, stream, flush=None):
        self.e0.record(stream)
        for i in range(self.steps):
            if flush is not None:
                flush()
            step(self.ev[i])
        self.e1.record(stream)

    def loop_ms(self) -> float:
        return self.e0.elapsed_time(self.e1)

    def stage_ms(self):
        """Mean device time per step of every stage."""
        tot = np.zeros(len(STAGES))
        for ev in self.ev:
            for s in range(len(STAGES)):
                tot[s] += ev[s].elapsed_time(ev[s + 1])
        return list(tot / self.steps)

    def step_ms(self) -> float:
        """Mean device time per step from each step's first to last stage event."""
        return float(np.mean([ev[0].elapsed_time(ev[-1]) for ev in self.ev]))


class Workbench:
    """One workload's layer on the GPU, ready to time."""

    def __init__(self, wl, dev, rank=0, inp=None):
        from sparse_mixture_experts_12_b200 import binding as B

        self.wl, self.dev = wl, dev
        if inp is None:
            inp = synth.generate(wl, seed=0)
        if rank > 0:  # same weights, an independent batch per rank
            g = torch.Generator().manual_seed(1000 + rank)
            inp["x"] = torch.empty((wl.T, wl.d_model)).normal_(0, 1, generator=g).to(
                wl.torch_dtype)
        self.inp = inp
        self.layer = B.MoELayer(wl, inp, dev)
        self.x = inp["x"].to(dev)
        self.y = torch.empty_like(self.x)
        self.ec = wl.routing == synth.ROUTING_EXPERT_CHOICE
        # the capacity workloads also emit f, P and the aux loss (token choice only)
        self.want_aux = wl.capacity_factor > 0 and not self.ec
        self.aux = self.layer.new_aux() if self.want_aux else None
        # noisy gating: the step routes on logits + softplus(x W_noise^T) * eps, the
        # draws eps made inside the library for (seed, offset), a new offset per step
        self.noise_seed = 1234 + rank if wl.noisy else None
        self.noise_offset = 0

    def forward(self, x=None, y=None, aux=None, taps=None, events=None):
        x = self.x if x is None else x
        y = self.y if y is None else y
        aux = self.aux if aux is None else aux
        if self.noise_seed is None:
            return self.layer.forward(x, y, aux, taps=taps, events=events)
        self.noise_offset += 1
        return self.layer.forward_noisy(x, None, y, aux, taps=taps, events=events,
                                        seed=self.noise_seed, offset=self.noise_offset)

    def check(self, where):
        code, info = self.layer.last_device_error()
        if code != 0:
            raise RuntimeError(f"{self.wl.name}: device error {code} ({info}) {where}")

    def routing(self) -> dict:
        """Routing statistics of one step (from a forward with taps)."""
        taps = self.layer.new_taps()
        if self.ec:
            self.forward(taps=taps)
            E = self.wl.n_experts
            C = int(math.floor(self.wl.capacity_factor * self.wl.T / E))
            lg = torch.empty((self.wl.T, E), dtype=torch.float32, device=self.dev)
            eci = torch.empty((E, C), dtype=torch.int32, device=self.dev)
            ecs = torch.empty((E, C), dtype=torch.float32, device=self.dev)
            self.layer.route_expert_choice(self.x, lg, eci, ecs)
            torch.cuda.synchronize()
            rs = routing_stats(self.wl, np.full(E, C), np.arange(E + 1) * C)
            rs["tokens_read"] = int(torch.unique(eci).numel())
        else:
            self.forward(taps=taps)
            torch.cuda.synchronize()
            rs = routing_stats(self.wl, taps["counts"].cpu().numpy(),
                               taps["offsets"].cpu().numpy())
            inv = taps["inv"].cpu().numpy().reshape(self.wl.T, self.wl.top_k)
            rs["tokens_read"] = int((inv >= 0).any(axis=1).sum())
        self.check("in the routing pass")
        return rs


def _made_events(n: int):
    """n timing events, each already created on the device (torch creates an event
    at its first record, and the library records the raw handle)."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for e in evs:
        e.record()
    torch.cuda.synchronize()
    return evs


FFN_FIRST, FFN_END = STAGES.index("shared_ffn"), STAGES.index("combine")
FFN_EVERY = 4  # every 4th timed step also times its expert GEMMs


def time_workload(wb: Workbench, steps: int, warmup: int, peaks, peaks_src, local_rank,
                  world=1, flush_buf=None):
    """Warm-up, then the timed region: K steps of the layer call; every FFN_EVERY-th
    step records two events, at the start of its expert FFNs (shared experts first)
    and at the start of its combine, so that the expert GEMMs' time comes from the
    timed steps. The layer launches each kernel so that it may begin while the one
    before it finishes; the kernel right after an event does not, so these events
    cost those steps a little.
    Then, for the breakdown, K more steps with an event at every stage boundary.
    Returns the workload's report, the timed loop's time (max over ranks) and the
    kernels per step."""
    wl, dev = wb.wl, wb.dev
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        wb.forward()
    torch.cuda.synchronize()
    wb.check("during warm-up")
    launches = kernels_per_step(lambda: wb.forward(), dev)
    timer = StepTimer(steps)
    ffn_ev = [_made_events(2) for _ in range(0, steps, FFN_EVERY)]
    flush = None
    if flush_buf is not None:
        flush = flush_buf.zero_
    clocks = ClockSampler(local_rank)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    clocks.begin_load()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        if flush is not None:
            flush()
        if i % FFN_EVERY == 0:
            ev = [None] * (len(STAGES) + 1)
            ev[FFN_FIRST], ev[FFN_END] = ffn_ev[i // FFN_EVERY]
            wb.forward(events=ev)
        else:
            wb.forward()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    wb.check("in the timed region")
    ffn_ms = float(np.mean([a.elapsed_time(b) for a, b in ffn_ev]))
    timer.run(lambda ev: wb.forward(events=ev), stream, flush)  # the breakdown
    torch.cuda.synchronize()
    wb.check("in the breakdown steps")
    stage_ms = timer.stage_ms()
    if flush is None:
        loop_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
        ms_step = loop_ms / steps
        timing = "back-to-back steps, working set > L2"
    else:
        ms_step = max_over_ranks(timer.step_ms(), world, dev)
        loop_ms = ms_step * steps
        timing = "per step (first to last stage event), L2 flushed between steps"
    rs = wb.routing()
    work = stage_work(wl, rs, wb.want_aux)
    rep = {"workload": wl.name, "T": wl.T, "ms_per_step": ms_step,
           "tokens_per_s": wl.T * world / (ms_step * 1e-3), "timing": timing,
           "stages": stage_report(work, stage_ms, peaks),
           "stages_note": "a second run of K steps with an event at every stage boundary; "
                          "the kernel after each event starts after it",
           "roofline": ffn_roofline(wl, work, ffn_ms, peaks, peaks_src),
           "kernels_per_step": launches, "routing": rs, "clocks": clk}
    return rep, loop_ms, launches


# ---------------------------------------------------------------------- our arm
def run_ours(args, wl, rank, world, local_rank):
    from sparse_mixture_experts_12_b200 import build as BUILD

    BUILD.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks, peaks_src = load_peaks()
    t0 = time.time()
    wb = Workbench(wl, dev, rank)
    log(f"[rank {rank}] {wl.name}: inputs drawn and placed in {time.time() - t0:.1f} s")

    rep, loop_ms, launches = time_workload(wb, args.steps, args.warmup, peaks, peaks_src,
                                           local_rank, world)
    value = tokens_per_second(wl.T, world, args.steps, loop_ms)
    roof = dict(rep["roofline"])
    roof["traffic"] = _traffic(wl.name)
    roof["kernel"] = ("grouped expert GEMMs (up + down projections of the routed experts, "
                      "and of the shared experts), timed by the stage events of the timed "
                      "steps")

    # ---- end to end through the public API with host buffers. Every step copies
    # its input from pinned host memory, runs moe_forward and copies its output
    # (and the aux statistics) back to pinned host memory. Two buffer slots and
    # three streams (copy in, compute, copy out) let step i+1's input copy and step
    # i-1's output copy run under step i's compute; events order each slot's reuse.
    e2e = measure_e2e(wb, args.steps, world, dev)
    wb.check("in the end-to-end loop")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        P = oracle_params_f64(wb.inp)
        rate, desc, _ = oracle_sample_rate(wl, P, args.cpu_sample)
        del P
        cpu = {"value": rate, "unit": "tokens/s", "cores": _oracle_threads(), "kind": "oracle",
               "sample": desc}

    side = {}
    names = _side_workloads(args, wl, world)
    sharded = None
    del wb
    torch.cuda.empty_cache()
    flush_buf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev) if names else None
    for name in names:
        swl = synth.WORKLOADS[name]
        t0 = time.time()
        swb = Workbench(swl, dev, rank)
        log(f"[rank {rank}] {swl.name}: inputs drawn and placed in {time.time() - t0:.1f} s")
        small = _working_set_bytes(swl) < L2_BYTES
        srep, _, _ = time_workload(swb, args.steps, args.warmup, peaks, peaks_src, local_rank,
                                   world, flush_buf if small else None)
        srep["roofline"]["traffic"] = _traffic(swl.name)
        if swl.n_shared and srep["roofline"]["traffic"] is not None:
            srep["roofline"]["traffic_scope"] = "routed experts only (the shared ones not captured)"
        side[name] = srep
        del swb
        torch.cuda.empty_cache()
    if world > 1 and not args.no_sharded:
        sharded = run_sharded_gpu(args, world, rank, local_rank, dev)

    if rank != 0:
        return
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": loop_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16"
            if wl.dtype == synth.DT_BF16 else "f32",
            "data": "synthetic (seeded N(0,1) activations, random-init weights)",
            "config": _config(wl, world), "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches * args.steps, "clocks": rep["clocks"],
            "stages": rep["stages"], "routing": rep["routing"], "workloads": side}
    if sharded is not None:
        line["sharded"] = sharded
    print(json.dumps(line), flush=True)


def _working_set_bytes(wl) -> int:
    """Bytes one step touches at least (weights and activations)."""
    b = wl.elem_bytes
    n_mats = 3 if wl.act == synth.ACT_SWIGLU else 2
    w = wl.n_experts * n_mats * wl.d_model * wl.d_ff * b
    if wl.T * wl.top_k < wl.n_experts:  # decode: only the touched experts are read
        w = w * wl.T * wl.top_k // wl.n_experts
    return w + 2 * wl.T * wl.d_model * b


def _side_workloads(args, wl, world):
    """The other workloads to time after the headline one. By default only one-GPU
    runs time them (N > 1 runs time the headline and the sharded batch)."""
    if args.workloads == "none" or (args.workloads == "all" and world > 1):
        return []
    names = SIDE_WORKLOADS if args.workloads == "all" else tuple(args.workloads.split(","))
    for n in names:
        if n not in synth.WORKLOADS:
            raise SystemExit(f"unknown workload {n}")
    return [n for n in names if synth.WORKLOADS[n].name != wl.name]


def measure_e2e(wb: Workbench, steps: int, world: int, dev) -> dict:
    x, y, aux, inp = wb.x, wb.y, wb.aux, wb.inp
    stream = torch.cuda.current_stream()
    xh = inp["x"].pin_memory()
    slots = []
    for _ in range(2):
        slots.append({"x": torch.empty_like(x), "y": torch.empty_like(y),
                      "aux": None if aux is None else torch.empty_like(aux),
                      "yh": torch.empty(x.shape, dtype=x.dtype).pin_memory(),
                      "auxh": None if aux is None else torch.empty(aux.shape).pin_memory(),
                      "in": torch.cuda.Event(), "comp": torch.cuda.Event(),
                      "out": torch.cuda.Event()})
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_steps(n):
        for i in range(n):
            sl = slots[i % 2]
            with torch.cuda.stream(s_in):
                s_in.wait_event(sl["comp"])  # the slot's previous forward has read x
                sl["x"].copy_(xh, non_blocking=True)
                sl["in"].record(s_in)
            stream.wait_event(sl["in"])
            stream.wait_event(sl["out"])     # the slot's previous output has left
            wb.forward(sl["x"], sl["y"], sl["aux"])
            sl["comp"].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(sl["comp"])
                sl["yh"].copy_(sl["y"], non_blocking=True)
                if sl["aux"] is not None:
                    sl["auxh"].copy_(sl["aux"], non_blocking=True)
                sl["out"].record(s_out)

    e2e_steps(4)
    torch.cuda.synchronize()
    barrier(world)
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    g0.record(s_in)
    s_in.wait_event(g0)
    stream.wait_event(g0)
    s_out.wait_event(g0)
    e2e_steps(steps)
    for sl in slots:  # the end: both slots' last outputs are on the host
        s_out.wait_event(sl["out"])
    g1.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(g0.elapsed_time(g1), world, dev)
    return {"value": tokens_per_second(wb.wl.T, world, steps, e2e_ms), "unit": "tokens/s",
            "h2d_bytes_per_step": int(xh.numel() * xh.element_size()),
            "d2h_bytes_per_step": int(slots[0]["yh"].numel() * slots[0]["yh"].element_size()) +
            (int(aux.numel() * 4) if aux is not None else 0),
            "pipelining": "2 slots, copy-in / compute / copy-out streams"}


# ------------------------------------------------- one batch sharded over the ranks
SHARDED_WORKLOAD = "switch"


def sharded_steps_timing(steps_obj, x_local, n_experts, steps, warmup, group, clock,
                         want_aux=True):
    """Time `steps` calls of the token-sharded layer (sharded.forward_sharded: route,
    all-gather of the pre-drop counts, all-reduce of the statistics sums, then the
    shard's permute / expert FFNs / combine and the statistics) after `warmup` calls.
    clock() returns a pair (start, stop) of callables; stop() returns elapsed ms
    including a synchronisation. Every rank takes the same collectives in the same
    order. Returns (ms of the timed calls on this rank, last (y, aux))."""
    from sparse_mixture_experts_12_b200 import sharded as S

    out = None
    for _ in range(warmup):
        out = S.forward_sharded(steps_obj, x_local, n_experts, group, want_aux)
    start, stop = clock()
    start()
    for _ in range(steps):
        out = S.forward_sharded(steps_obj, x_local, n_experts, group, want_aux)
    return stop(), out


def run_sharded_gpu(args, world, rank, local_rank, dev):
    """One batch of world x T Switch-layer tokens, rank r holding the r-th slice; the
    weights are the same seeded draws on every rank."""
    from sparse_mixture_experts_12_b200 import sharded as S

    base = synth.WORKLOADS[SHARDED_WORKLOAD]
    wl = base.replace(T=base.T * world)
    inp = synth.generate(base, seed=0)
    a, b = S.shard_bounds(wl.T, world)[rank]
    g = torch.Generator().manual_seed(2000)  # the whole batch, drawn alike on every rank
    xall = torch.empty((wl.T, wl.d_model)).normal_(0, 1, generator=g).to(wl.torch_dtype)
    layer = S.ShardedMoELayer(wl, inp, rank, world, dev)
    x = xall[a:b].to(dev)

    def clock():
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def start():
            barrier(world)
            torch.cuda.synchronize()
            e0.record()

        def stop():
            e1.record()
            torch.cuda.synchronize()
            barrier(world)
            return e0.elapsed_time(e1)

        return start, stop

    ms, _ = sharded_steps_timing(layer, x, wl.n_experts, args.steps, args.warmup, None, clock)
    code, info = layer.layer.last_device_error()
    if code != 0:
        raise RuntimeError(f"sharded layer: device error {code} ({info})")
    ms = max_over_ranks(ms, world, dev)
    return {"workload": wl.name + f" (one batch of {wl.T} tokens over {world} ranks)",
            "tokens_per_s": tokens_per_second(wl.T, 1, args.steps, ms),
            "ms_per_step": ms / args.steps, "collectives": "NCCL all-gather of [E] int32 "
            "counts, sum all-reduce of [1 + 2E] fp64 sums, per step",
            "scaling": "weak (T tokens per rank)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mixtral_prefill", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--workloads", default="all",
                    help="the other workloads reported under 'workloads': 'all', 'none' or "
                         "a comma-separated list")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sharded", action="store_true",
                    help="skip the token-sharded batch that N > 1 runs also time")
    ap.add_argument("--cpu-sample", type=int, default=512,
                    help="tokens whose expert FFNs the CPU oracle computes")
    ap.add_argument("--ref-sample", type=int, default=256,
                    help="tokens per step of the reference (oracle) arm")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local_rank = dist_env()
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, wl, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
