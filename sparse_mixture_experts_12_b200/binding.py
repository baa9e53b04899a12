"""Thin ctypes binding over ``libmoe.so`` (argument marshalling only).

Every step of the layer runs in the library's CUDA kernels; PyTorch only
provides device memory and the current stream. There is no fallback: if the
library is missing or no CUDA device is present, the calls raise.

Function names follow the C ABI in ``include/moe.h``.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

from . import synth

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")
_lib = None

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_MISALIGNED", 4: "MOE_ERR_WORKSPACE", 5: "MOE_ERR_CUDA",
                6: "MOE_ERR_DEVICE"}
DEVERR_NAMES = {0: "none", 1: "expert index out of range", 2: "invalid offsets",
                3: "row index out of range", 4: "pipeline wait timeout"}

EXPORTED = ("moe_workspace_size", "moe_workspace_init", "moe_route", "moe_route_noisy",
            "moe_route_expert_choice", "moe_permute", "moe_permute_noalloc", "moe_forward_noisy",
            "moe_expert_ffn", "moe_combine", "moe_aux_stats", "moe_forward",
            "moe_route_shard", "moe_permute_shard", "moe_forward_shard", "moe_aux_finalize",
            "moe_forward_staged", "moe_noise_draws", "moe_route_noisy_seeded",
            "moe_forward_noisy_seeded", "moe_test_set_wait_limit", "moe_test_withhold_load",
            "moe_last_device_error", "moe_status_string")

# stages of one layer call (MOE_STAGE_*), in launch order
STAGES = ("route", "scan", "permute", "shared_ffn", "expert_ffn", "combine")


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")
        self.status = status


class MoeCfg(ctypes.Structure):
    _fields_ = [("n_tokens", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("d_ff", ctypes.c_int32), ("act", ctypes.c_int32),
                ("gate_mode", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("capacity_factor", ctypes.c_float), ("aux_alpha", ctypes.c_float),
                ("n_shared", ctypes.c_int32), ("d_ff_shared", ctypes.c_int32),
                ("routing", ctypes.c_int32)]


class MoeWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("w_router", "b_router", "logit_bias", "w1", "w3", "w2", "b1", "b2",
                 "ws_gate", "ws_up", "ws_down", "w_noise")]


class MoeTaps(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("logits", "topk_idx", "topk_gate", "counts", "offsets", "perm", "inv")]


class MoeShard(ctypes.Structure):
    _fields_ = [("n_tokens_total", ctypes.c_longlong), ("n_shards", ctypes.c_int32),
                ("shard", ctypes.c_int32), ("counts_all", ctypes.c_void_p)]


class MoeStageEvents(ctypes.Structure):
    _fields_ = [("ev", ctypes.c_void_p * (len(STAGES) + 1))]


class MoeNoise(ctypes.Structure):
    _fields_ = [("eps", ctypes.c_void_p), ("seed", ctypes.c_uint64), ("offset", ctypes.c_uint64)]


def lib_path() -> str:
    return _LIB_PATH


def load() -> ctypes.CDLL:
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m sparse_mixture_experts_12_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, S = ctypes.c_void_p, ctypes.c_size_t
    cfgp, wp = ctypes.POINTER(MoeCfg), ctypes.POINTER(MoeWeights)
    sig = {
        "moe_workspace_size": [cfgp, ctypes.POINTER(ctypes.c_size_t)],
        "moe_workspace_init": [P, S, P],
        "moe_route": [cfgp, wp, P, P, P, P, P, S, P],
        "moe_permute": [cfgp, P, P, P, P, P, P, P, P, S, P],
        "moe_permute_noalloc": [cfgp, P, P, P, P, P, P, P, P],
        "moe_expert_ffn": [cfgp, wp, P, P, P, P, S, P],
        "moe_combine": [cfgp, P, P, P, P, P, P, S, P],
        "moe_aux_stats": [cfgp, P, P, P, P, S, P],
        "moe_forward": [cfgp, wp, P, P, P, ctypes.POINTER(MoeTaps), P, S, P],
        "moe_route_shard": [cfgp, wp, P, P, P, P, P, P, P, S, P],
        "moe_permute_shard": [cfgp, ctypes.POINTER(MoeShard), P, P, P, P, P, P, P, P, S, P],
        "moe_forward_shard": [cfgp, ctypes.POINTER(MoeShard), wp, P, ctypes.POINTER(MoeTaps), P,
                              P, S, P],
        "moe_aux_finalize": [cfgp, ctypes.c_longlong, P, P, P],
        "moe_forward_staged": [cfgp, wp, P, ctypes.POINTER(MoeNoise), P, P,
                               ctypes.POINTER(MoeTaps), ctypes.POINTER(MoeStageEvents), P, S,
                               P],
        "moe_noise_draws": [ctypes.c_int32, ctypes.c_int32, ctypes.c_uint64, ctypes.c_uint64, P,
                            P, P],
        "moe_route_noisy_seeded": [cfgp, wp, P, ctypes.c_uint64, ctypes.c_uint64, P, P, P, P, S,
                                   P],
        "moe_forward_noisy_seeded": [cfgp, wp, P, ctypes.c_uint64, ctypes.c_uint64, P, P,
                                     ctypes.POINTER(MoeTaps), P, S, P],
        "moe_test_set_wait_limit": [ctypes.c_uint64],
        "moe_test_withhold_load": [ctypes.c_int32],
        "moe_last_device_error": [P, ctypes.POINTER(ctypes.c_int32),
                                  ctypes.POINTER(ctypes.c_int32), P],
    }
    for name, args in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    lib.moe_status_string.argtypes = [ctypes.c_int]
    lib.moe_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def expert_rows(cfg: MoeCfg) -> int:
    """Rows of the expert-contiguous buffers (x_perm, y_perm) the library reads and
    writes for this configuration: T * k under token choice, E * C with
    C = floor(cf * T / E) under expert choice (evaluated in double, as the library
    does)."""
    if cfg.routing == synth.ROUTING_EXPERT_CHOICE:
        if not cfg.capacity_factor > 0:
            return 0
        return cfg.n_experts * math.floor(float(cfg.capacity_factor) * cfg.n_tokens /
                                          cfg.n_experts)
    return cfg.n_tokens * cfg.top_k


def check_rows(t: Optional[torch.Tensor], rows: int, cols: int, name: str):
    """The C ABI takes raw pointers and cannot see a buffer's size: a tensor with
    fewer than the `rows` rows of `cols` elements that the library will access is
    refused here, before anything is launched."""
    if t is None:
        return
    if t.dim() != 2 or t.shape[0] < rows or t.shape[1] != cols or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [>= {rows}, {cols}] tensor, "
                         f"not {tuple(t.shape)}")


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _taps(taps: Optional[dict]):
    if taps is None:
        return None
    return MoeTaps(**{k: _ptr(taps.get(k)) for k, _ in MoeTaps._fields_})


def stage_events(events) -> MoeStageEvents:
    """MoeStageEvents from len(STAGES) + 1 torch.cuda.Event (None entries allowed)."""
    if len(events) != len(STAGES) + 1:
        raise ValueError(f"{len(STAGES) + 1} events expected, got {len(events)}")
    ev = MoeStageEvents()
    for i, e in enumerate(events):
        if e is not None and not e.cuda_event:
            raise ValueError("a torch.cuda.Event has no CUDA event until its first record()")
        ev.ev[i] = None if e is None else e.cuda_event
    return ev


def make_cfg(w: synth.Workload, **over) -> MoeCfg:
    c = MoeCfg(n_tokens=w.T, d_model=w.d_model, n_experts=w.n_experts, top_k=w.top_k,
               d_ff=w.d_ff, act=w.act, gate_mode=w.gate_mode, dtype=w.dtype,
               capacity_factor=w.capacity_factor, aux_alpha=w.aux_alpha,
               n_shared=w.n_shared, d_ff_shared=w.d_ff_shared, routing=w.routing)
    for k, v in over.items():
        setattr(c, k, v)
    return c


def workspace_size(cfg: MoeCfg) -> int:
    n = ctypes.c_size_t(0)
    _check(load().moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def new_workspace(cfg: MoeCfg, device="cuda") -> torch.Tensor:
    nbytes = workspace_size(cfg)
    ws = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    ws = ws[off:off + nbytes]
    _check(load().moe_workspace_init(_ptr(ws), nbytes, _stream()), "moe_workspace_init")
    return ws


class MoELayer:
    """One MoE FFN layer whose weights live on the GPU.

    ``params`` is the dict of ``synth.generate`` (CPU or CUDA tensors); they are
    moved to ``device`` once. ``forward`` runs the whole layer through
    ``moe_forward`` on the current stream.
    """

    def __init__(self, workload: synth.Workload, params: dict, device="cuda"):
        self.w = workload
        self.cfg = make_cfg(workload)
        self.device = torch.device(device)
        self.p = {k: (None if v is None else v.to(self.device).contiguous())
                  for k, v in params.items() if k != "x"}
        self.weights = MoeWeights(**{k: _ptr(self.p.get(k)) for k, _ in MoeWeights._fields_})
        self.ws = new_workspace(self.cfg, self.device)
        self.lib = load()

    # -------------------------------------------------------------- whole layer
    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None,
                aux: Optional[torch.Tensor] = None, taps: Optional[dict] = None,
                events: Optional[list] = None) -> torch.Tensor:
        """The whole layer (moe_forward). ``events``: len(STAGES) + 1 torch.cuda.Event
        objects recorded at the stage boundaries (moe_forward_staged)."""
        if y is None:
            y = torch.empty_like(x)
        tp = _taps(taps)
        tpr = ctypes.byref(tp) if tp is not None else None
        if events is None:
            _check(self.lib.moe_forward(ctypes.byref(self.cfg), ctypes.byref(self.weights),
                                        _ptr(x), _ptr(y), _ptr(aux), tpr, _ptr(self.ws),
                                        self.ws.numel(), _stream()), "moe_forward")
        else:
            self._staged(x, None, y, aux, tpr, events)
        return y

    def _staged(self, x, noise, y, aux, tpr, events):
        ev = stage_events(events)
        _check(self.lib.moe_forward_staged(ctypes.byref(self.cfg), ctypes.byref(self.weights),
                                           _ptr(x), ctypes.byref(noise) if noise else None,
                                           _ptr(y), _ptr(aux), tpr, ctypes.byref(ev),
                                           _ptr(self.ws), self.ws.numel(), _stream()),
               "moe_forward_staged")

    def forward_noisy(self, x: torch.Tensor, eps: Optional[torch.Tensor] = None,
                      y: Optional[torch.Tensor] = None, aux: Optional[torch.Tensor] = None,
                      taps: Optional[dict] = None, events: Optional[list] = None,
                      seed: Optional[int] = None, offset: int = 0) -> torch.Tensor:
        """The layer with noisy top-k gating: eps [T, E] fp32 standard normal draws, or
        (eps None) the library's counter-based draws for (seed, offset)."""
        if (eps is None) == (seed is None):
            raise ValueError("give either eps or seed")
        if y is None:
            y = torch.empty_like(x)
        tp = _taps(taps)
        tpr = ctypes.byref(tp) if tp is not None else None
        if events is not None:
            self._staged(x, MoeNoise(eps=_ptr(eps), seed=seed or 0, offset=offset), y, aux, tpr,
                         events)
        elif eps is not None:
            _check(self.lib.moe_forward_noisy(ctypes.byref(self.cfg), ctypes.byref(self.weights),
                                              _ptr(x), _ptr(eps), _ptr(y), _ptr(aux), tpr,
                                              _ptr(self.ws), self.ws.numel(), _stream()),
                   "moe_forward_noisy")
        else:
            _check(self.lib.moe_forward_noisy_seeded(
                ctypes.byref(self.cfg), ctypes.byref(self.weights), _ptr(x), seed, offset,
                _ptr(y), _ptr(aux), tpr, _ptr(self.ws), self.ws.numel(), _stream()),
                "moe_forward_noisy_seeded")
        return y

    def new_taps(self) -> dict:
        T, E, k = self.w.T, self.w.n_experts, self.w.top_k
        dev = self.device
        i32 = dict(dtype=torch.int32, device=dev)
        return {"logits": torch.empty((T, E), dtype=torch.float32, device=dev),
                "topk_idx": torch.empty((T, k), **i32),
                "topk_gate": torch.empty((T, k), dtype=torch.float32, device=dev),
                "counts": torch.empty((E,), **i32), "offsets": torch.empty((E + 1,), **i32),
                "perm": torch.empty((T * k,), **i32), "inv": torch.empty((T * k,), **i32)}

    def new_aux(self) -> torch.Tensor:
        return torch.zeros(3 + 2 * self.w.n_experts, dtype=torch.float32, device=self.device)

    # ------------------------------------------------------------- single steps
    def route(self, x: Optional[torch.Tensor], logits: torch.Tensor, topk_idx: torch.Tensor,
              topk_gate: torch.Tensor):
        _check(self.lib.moe_route(ctypes.byref(self.cfg), ctypes.byref(self.weights), _ptr(x),
                                  _ptr(logits), _ptr(topk_idx), _ptr(topk_gate), _ptr(self.ws),
                                  self.ws.numel(), _stream()), "moe_route")

    def route_noisy(self, x: torch.Tensor, eps: torch.Tensor, logits: torch.Tensor,
                    topk_idx: torch.Tensor, topk_gate: torch.Tensor):
        _check(self.lib.moe_route_noisy(ctypes.byref(self.cfg), ctypes.byref(self.weights),
                                        _ptr(x), _ptr(eps), _ptr(logits), _ptr(topk_idx),
                                        _ptr(topk_gate), _ptr(self.ws), self.ws.numel(),
                                        _stream()), "moe_route_noisy")

    def route_noisy_seeded(self, x: torch.Tensor, seed: int, offset: int, logits: torch.Tensor,
                           topk_idx: torch.Tensor, topk_gate: torch.Tensor):
        _check(self.lib.moe_route_noisy_seeded(ctypes.byref(self.cfg), ctypes.byref(self.weights),
                                               _ptr(x), seed, offset, _ptr(logits),
                                               _ptr(topk_idx), _ptr(topk_gate), _ptr(self.ws),
                                               self.ws.numel(), _stream()),
               "moe_route_noisy_seeded")

    def route_expert_choice(self, x: Optional[torch.Tensor], logits: torch.Tensor,
                            ec_idx: torch.Tensor, ec_score: torch.Tensor):
        """Expert-Choice routing: logits [T, E] (input when x is None), ec_idx [E, C],
        ec_score [E, C]."""
        _check(self.lib.moe_route_expert_choice(
            ctypes.byref(self.cfg), ctypes.byref(self.weights), _ptr(x), _ptr(logits),
            _ptr(ec_idx), _ptr(ec_score), _ptr(self.ws), self.ws.numel(), _stream()),
            "moe_route_expert_choice")

    def permute(self, x, topk_idx, counts, offsets, perm, inv, x_perm):
        check_rows(x_perm, expert_rows(self.cfg), self.cfg.d_model, "x_perm")
        _check(self.lib.moe_permute(ctypes.byref(self.cfg), _ptr(x), _ptr(topk_idx), _ptr(counts),
                                    _ptr(offsets), _ptr(perm), _ptr(inv), _ptr(x_perm),
                                    _ptr(self.ws), self.ws.numel(), _stream()), "moe_permute")

    def expert_ffn(self, x_perm, offsets, y_perm, cfg: Optional[MoeCfg] = None,
                   weights: Optional[MoeWeights] = None):
        c = cfg or self.cfg
        check_rows(x_perm, expert_rows(c), c.d_model, "x_perm")
        check_rows(y_perm, expert_rows(c), c.d_model, "y_perm")
        _check(self.lib.moe_expert_ffn(ctypes.byref(cfg or self.cfg),
                                       ctypes.byref(weights or self.weights), _ptr(x_perm),
                                       _ptr(offsets), _ptr(y_perm), _ptr(self.ws),
                                       self.ws.numel(), _stream()), "moe_expert_ffn")

    def combine(self, y_perm, inv, topk_gate, shared_y, y):
        check_rows(y_perm, expert_rows(self.cfg), self.cfg.d_model, "y_perm")
        _check(self.lib.moe_combine(ctypes.byref(self.cfg), _ptr(y_perm), _ptr(inv),
                                    _ptr(topk_gate), _ptr(shared_y), _ptr(y), _ptr(self.ws),
                                    self.ws.numel(), _stream()), "moe_combine")

    def aux_stats(self, logits, topk_idx, out):
        _check(self.lib.moe_aux_stats(ctypes.byref(self.cfg), _ptr(logits), _ptr(topk_idx),
                                      _ptr(out), _ptr(self.ws), self.ws.numel(), _stream()),
               "moe_aux_stats")

    # ------------------------------------------------- one shard of a larger batch
    def route_shard(self, x: Optional[torch.Tensor], logits: Optional[torch.Tensor],
                    topk_idx: torch.Tensor, topk_gate: torch.Tensor, counts: torch.Tensor,
                    aux_part: Optional[torch.Tensor] = None):
        """moe_route on this shard + its pre-drop counts [E] int32 and, optionally, its
        fp64 sums aux_part [1 + 2E] for the statistics."""
        _check(self.lib.moe_route_shard(ctypes.byref(self.cfg), ctypes.byref(self.weights),
                                        _ptr(x), _ptr(logits), _ptr(topk_idx), _ptr(topk_gate),
                                        _ptr(counts), _ptr(aux_part), _ptr(self.ws),
                                        self.ws.numel(), _stream()), "moe_route_shard")

    def permute_shard(self, shard: MoeShard, x, topk_idx, counts, offsets, perm, inv, x_perm):
        check_rows(x_perm, expert_rows(self.cfg), self.cfg.d_model, "x_perm")
        _check(self.lib.moe_permute_shard(ctypes.byref(self.cfg), ctypes.byref(shard), _ptr(x),
                                          _ptr(topk_idx), _ptr(counts), _ptr(offsets),
                                          _ptr(perm), _ptr(inv), _ptr(x_perm), _ptr(self.ws),
                                          self.ws.numel(), _stream()), "moe_permute_shard")

    def forward_shard(self, shard: MoeShard, x: torch.Tensor, taps: dict,
                      y: Optional[torch.Tensor] = None) -> torch.Tensor:
        """The layer on this shard, routed by route_shard: taps["topk_idx"] and
        taps["topk_gate"] are inputs."""
        if y is None:
            y = torch.empty_like(x)
        tp = MoeTaps(**{k: _ptr(taps.get(k)) for k, _ in MoeTaps._fields_})
        _check(self.lib.moe_forward_shard(ctypes.byref(self.cfg), ctypes.byref(shard),
                                          ctypes.byref(self.weights), _ptr(x), ctypes.byref(tp),
                                          _ptr(y), _ptr(self.ws), self.ws.numel(), _stream()),
               "moe_forward_shard")
        return y

    def aux_finalize(self, n_tokens_total: int, aux_part: torch.Tensor,
                     out: Optional[torch.Tensor] = None) -> torch.Tensor:
        if out is None:
            out = self.new_aux()
        _check(self.lib.moe_aux_finalize(ctypes.byref(self.cfg), int(n_tokens_total),
                                         _ptr(aux_part), _ptr(out), _stream()),
               "moe_aux_finalize")
        return out

    def last_device_error(self):
        code, info = ctypes.c_int32(0), ctypes.c_int32(0)
        st = self.lib.moe_last_device_error(_ptr(self.ws), ctypes.byref(code), ctypes.byref(info),
                                            _stream())
        if st not in (MOE_OK, 6):
            raise MoeError(st, "moe_last_device_error")
        return code.value, info.value


def noise_draws(n_tokens: int, n_experts: int, seed: int, offset: int, eps: torch.Tensor,
                raw: Optional[torch.Tensor] = None):
    """moe_noise_draws: eps [T, E] fp32 and optionally raw [T, ceil(E/4), 4] int32 words
    (the uint32 bit patterns), both on the current device and stream."""
    _check(load().moe_noise_draws(n_tokens, n_experts, seed, offset, _ptr(eps), _ptr(raw),
                                  _stream()), "moe_noise_draws")


def shared_as_experts(layer: MoELayer):
    """(cfg, weights) that run the layer's shared experts through moe_expert_ffn:
    one group, d_ff = n_shared * d_ff_shared, rows = all tokens."""
    w = layer.w
    cfg = make_cfg(w, n_experts=1, top_k=1, d_ff=w.n_shared * w.d_ff_shared,
                   act=synth.ACT_SWIGLU, n_shared=0, d_ff_shared=0, capacity_factor=0.0)
    p = layer.p
    wt = MoeWeights(w1=_ptr(p["ws_gate"]), w3=_ptr(p["ws_up"]), w2=_ptr(p["ws_down"]))
    return cfg, wt
