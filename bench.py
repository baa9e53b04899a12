#!/usr/bin/env python
"""Throughput of the MoE FFN layer forward on B200.

One step = one ``moe_forward`` over a batch of T tokens (router GEMM + softmax/
top-k, histogram/scan/permute, grouped expert GEMMs, shared experts, combine),
inputs already resident in HBM. Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs the same layer on its
own batch of T tokens (weak scaling, no data-path collective); the elapsed time
is the max over ranks.
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
METRIC = "MoE-layer tokens/s"


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
class _F64View:
    """Lazily upcast slices of a CPU tensor to fp64 numpy (input marshalling only)."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, i):
        return self.t[i].to(torch.float64).numpy()


def _oracle_params(inp):
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif v.numel() > (1 << 22) and k not in ("x", "w_router"):
            out[k] = _F64View(v)
        else:
            out[k] = v.to(torch.float64).numpy()
    return out


def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample_rate(wl, inp, n_tokens: int):
    """Time the CPU oracle: routing of all T tokens plus the expert FFNs of
    ``n_tokens`` strided tokens. Returns (tokens/s estimate for the full
    workload, description)."""
    from oracle import moe_oracle as O

    acts = {0: "relu", 1: "gelu", 2: "swiglu"}
    modes = {0: "topk_softmax", 1: "softmax_topk_renorm", 2: "softmax_topk_raw"}
    P = _oracle_params(inp)
    if wl.routing == synth.ROUTING_EXPERT_CHOICE:
        t0 = time.perf_counter()
        logits = O.router_logits(P["x"], P["w_router"], P.get("b_router"), P.get("logit_bias"))
        O.expert_choice_select(logits, O.expert_choice_capacity(wl.capacity_factor, wl.T,
                                                                wl.n_experts))
        t_route = time.perf_counter() - t0
        toks = synth.token_sample(wl.T, n_tokens).numpy()
        t0 = time.perf_counter()
        O.expert_choice_forward(P["x"], P, capacity_factor=wl.capacity_factor,
                                act=acts[wl.act], logits=logits, tokens=toks)
        t_ffn = time.perf_counter() - t0  # includes the (cheap) re-selection
        per_token = t_route / wl.T + t_ffn / len(toks)
        desc = (f"oracle (numpy fp64), expert choice: routing of all {wl.T} tokens "
                f"({t_route:.2f} s) + expert FFNs of {len(toks)} strided tokens ({t_ffn:.2f} s)"
                f"; tokens/s = 1 / (t_route/T + t_ffn/n)")
        return 1.0 / per_token, desc, t_route + t_ffn
    kw = dict(top_k=wl.top_k, act=acts[wl.act], gate_mode=modes[wl.gate_mode],
              capacity_factor=wl.capacity_factor, n_shared=wl.n_shared)
    t0 = time.perf_counter()
    noisy = None
    if wl.noisy:  # the same seeded draws as the GPU arm
        eps = synth.noise_draws(wl.T, wl.n_experts, 99).numpy()
        noisy = O.noisy_router_logits(P["x"], P["w_router"], P["w_noise"], eps,
                                      P.get("b_router"), P.get("logit_bias"))
    r = O.route(P["x"], P, top_k=wl.top_k, gate_mode=kw["gate_mode"],
                capacity_factor=wl.capacity_factor, logits=noisy)
    t_route = time.perf_counter() - t0
    toks = synth.token_sample(wl.T, n_tokens).numpy()
    t0 = time.perf_counter()
    O.moe_forward(P["x"], P, tokens=toks, logits=r["logits"], **kw)
    t_ffn = time.perf_counter() - t0  # includes the (cheap) re-selection from given logits
    per_token = t_route / wl.T + t_ffn / len(toks)
    desc = (f"oracle (numpy fp64): routing of all {wl.T} tokens ({t_route:.2f} s) + expert "
            f"FFNs of {len(toks)} strided tokens ({t_ffn:.2f} s); tokens/s = 1 / "
            f"(t_route/T + t_ffn/n)")
    return 1.0 / per_token, desc, t_route + t_ffn


# ---------------------------------------------------------------- the reference arm
def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    inp = synth.generate(wl, seed=0)
    n = args.ref_sample
    for _ in range(args.warmup):
        oracle_sample_rate(wl, inp, n)
    rates, secs = [], 0.0
    desc = ""
    for _ in range(args.steps):
        r, desc, s = oracle_sample_rate(wl, inp, n)
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


# ---------------------------------------------------------------------- our arm
def run_ours(args, wl, rank, world, local_rank):
    from sparse_mixture_experts_12_b200 import binding as B
    from sparse_mixture_experts_12_b200 import build as BUILD

    BUILD.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    peaks, peaks_src = load_peaks()
    t0 = time.time()
    inp = synth.generate(wl, seed=0)
    if rank > 0:  # same weights, an independent batch per rank
        g = torch.Generator().manual_seed(1000 + rank)
        inp["x"] = torch.empty((wl.T, wl.d_model)).normal_(0, 1, generator=g).to(wl.torch_dtype)
    log(f"[rank {rank}] inputs drawn in {time.time() - t0:.1f} s")
    layer = B.MoELayer(wl, inp, dev)
    x = inp["x"].to(dev)
    y = torch.empty_like(x)
    ec = wl.routing == synth.ROUTING_EXPERT_CHOICE
    # the Switch workload also emits f, P and the aux loss (token choice only)
    want_aux = wl.capacity_factor > 0 and not ec
    aux = layer.new_aux() if want_aux else None
    stream = torch.cuda.current_stream()
    # noisy gating: the step routes on logits + softplus(x W_noise^T) * eps; the draws
    # eps are made once (seeded) and stay resident, like x
    eps = synth.noise_draws(wl.T, wl.n_experts, 99 + rank).to(dev) if wl.noisy else None

    def forward(xx, yy, aa, taps=None):
        if eps is None:
            return layer.forward(xx, yy, aa, taps=taps)
        return layer.forward_noisy(xx, eps, yy, aa, taps=taps)

    clocks = ClockSampler(local_rank)
    clocks.start()
    for _ in range(args.warmup):
        forward(x, y, aux)
    torch.cuda.synchronize()
    code, info = layer.last_device_error()
    if code != 0:
        raise RuntimeError(f"device error {code} ({info}) during warm-up")
    clocks.stop()
    per_step_launches = kernels_per_step(lambda: forward(x, y, aux), dev)
    clocks = ClockSampler(local_rank)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    clocks.begin_load()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        forward(x, y, aux)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    clk = clocks.stop()
    code, info = layer.last_device_error()
    if code != 0:
        raise RuntimeError(f"device error {code} ({info}) in the timed region")
    value = tokens_per_second(wl.T, world, args.steps, ms)

    # ---- expert FFN (grouped GEMMs) timed alone on the same stream, for the roofline
    E, k = wl.n_experts, wl.top_k
    if ec:  # each expert's C picked rows, expert-contiguous
        C = int(math.floor(wl.capacity_factor * wl.T / E))
        lg = torch.empty((wl.T, E), dtype=torch.float32, device=dev)
        eci = torch.empty((E, C), dtype=torch.int32, device=dev)
        ecs = torch.empty((E, C), dtype=torch.float32, device=dev)
        layer.route_expert_choice(x, lg, eci, ecs)
        xp = x[eci.reshape(-1).long()].contiguous()
        off = (torch.arange(E + 1, device=dev, dtype=torch.int32) * C).contiguous()
    else:
        taps = layer.new_taps()
        forward(x, y, aux, taps=taps)
        xp = torch.empty((wl.T * k, wl.d_model), dtype=wl.torch_dtype, device=dev)
        cnt = torch.empty(E, dtype=torch.int32, device=dev)
        off = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(wl.T * k, dtype=torch.int32, device=dev)
        inv = torch.empty(wl.T * k, dtype=torch.int32, device=dev)
        layer.permute(x, taps["topk_idx"], cnt, off, perm, inv, xp)
    yp = torch.empty_like(xp)
    counts = np.diff(off.cpu().numpy()) if ec else taps["counts"].cpu().numpy()
    for _ in range(3):
        layer.expert_ffn(xp, off, yp)
    torch.cuda.synchronize()
    n_ffn = max(args.steps, 10)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(n_ffn):
        layer.expert_ffn(xp, off, yp)
    f1.record(stream)
    torch.cuda.synchronize()
    ffn_ms = f0.elapsed_time(f1) / n_ffn
    R = int(off[-1].item())
    kept = np.diff(off.cpu().numpy())
    touched = int((kept > 0).sum())
    F, d = wl.d_ff, wl.d_model
    n_mats = 3 if wl.act == synth.ACT_SWIGLU else 2
    flops = 2.0 * R * n_mats * d * F
    w_bytes = touched * n_mats * d * F * wl.elem_bytes
    alg_bytes = w_bytes + 2.0 * R * d * wl.elem_bytes  # weights + x_perm read + y_perm write
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if flops / alg_bytes >= ridge:
        roof = {"bound": "tensor", "achieved": flops / (ffn_ms * 1e-3) / 1e12,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
        roof["frac_of_sustained"] = roof["achieved"] / peaks.get("bf16_tflops_sustained",
                                                                 peaks["bf16_tflops"])
    else:
        roof = {"bound": "hbm", "achieved": alg_bytes / (ffn_ms * 1e-3) / 1e9,
                "peak": peaks["hbm_gbs"], "unit": "GB/s"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = _traffic(wl.name)
    roof["kernel"] = "grouped expert FFN (moe_expert_ffn: up-projection + down-projection tcgen05 GEMMs)"
    roof["ms_per_launch"] = ffn_ms
    roof["peak_source"] = f"{peaks_src} ({'burst' if roof['bound'] == 'tensor' else 'copy'})"
    roof["algorithmic"] = {"flops": flops, "bytes": alg_bytes, "rows": R,
                           "touched_experts": touched}

    # ---- end to end through the public API with host buffers. Every step copies
    # its input from pinned host memory, runs moe_forward and copies its output
    # (and the aux statistics) back to pinned host memory. Two buffer slots and
    # three streams (copy in, compute, copy out) let step i+1's input copy and step
    # i-1's output copy run under step i's compute; events order each slot's reuse.
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
            forward(sl["x"], sl["y"], sl["aux"])
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
    e2e_steps(args.steps)
    for sl in slots:  # the end: both slots' last outputs are on the host
        s_out.wait_event(sl["out"])
    g1.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(g0.elapsed_time(g1), world, dev)
    e2e = {"value": tokens_per_second(wl.T, world, args.steps, e2e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": int(xh.numel() * xh.element_size()),
           "d2h_bytes_per_step": int(slots[0]["yh"].numel() * slots[0]["yh"].element_size()) +
           (int(aux.numel() * 4) if aux is not None else 0),
           "pipelining": "2 slots, copy-in / compute / copy-out streams"}
    code, info = layer.last_device_error()
    if code != 0:
        raise RuntimeError(f"device error {code} ({info}) in the end-to-end loop")

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        rate, desc, _ = oracle_sample_rate(wl, inp, args.cpu_sample)
        cpu = {"value": rate, "unit": "tokens/s", "cores": _oracle_threads(), "kind": "oracle",
               "sample": desc}
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16"
            if wl.dtype == synth.DT_BF16 else "f32",
            "data": "synthetic (seeded N(0,1) activations, random-init weights)",
            "config": _config(wl, world), "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": per_step_launches * args.steps, "clocks": clk,
            "routing": {"kind": "expert choice" if ec else "token choice", "rows_kept": R,
                        "dropped": 0 if ec else int(wl.T * k - R),
                        "max_expert_load": int(counts.max()), "min_expert_load": int(counts.min())}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mixtral_prefill", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample", type=int, default=8,
                    help="tokens whose expert FFNs the CPU oracle computes")
    ap.add_argument("--ref-sample", type=int, default=2,
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
