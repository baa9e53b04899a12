"""Seeded synthetic workloads for the sparse MoE FFN forward.

This module only draws inputs: it holds none of the layer's arithmetic, so both
the CPU oracle's tests and the CUDA path's tests/benchmark take their inputs
from here and nowhere else.

Recipe (identical for every workload, one torch CPU ``Generator`` per call,
seeded with ``seed``; every draw is fp32 ``normal_`` in this fixed order):

1. ``x``           [T, d]      ~ N(0, 1)
2. ``w_router``    [E, d]      ~ N(0, 0.02^2)
3. ``b_router``    [E]         ~ N(0, bias_std^2)   (only if the router has a bias)
4. ``logit_bias``  [E]         ~ N(0, logit_bias_std^2) (only if set)
5. per routed expert e = 0..E-1: ``w1[e]`` [F, d], then ``w3[e]`` [F, d] (SwiGLU
   only), then ``w2[e]`` [d, F], each ~ N(0, 1/fan_in) with fan_in = in_features
6. expert biases ``b1`` [E, F], ``b2`` [E, d] ~ N(0, bias_std^2) (MLP experts only)
7. per shared expert j: gate [F_sh, d], up [F_sh, d], down [d, F_sh] ~ N(0, 1/fan_in);
   the shared experts are stored concatenated along F_sh
   (``ws_gate``/``ws_up`` [n_sh*F_sh, d], ``ws_down`` [d, n_sh*F_sh]).
8. ``w_noise`` [E, d] ~ N(0, 0.02^2) (noisy gating only); the noise draws eps
   [T, E] ~ N(0, 1) come from ``noise_draws`` with a seed of their own.

Weights and activations are then rounded once (round-to-nearest-even) to the
workload's storage dtype (bf16 or fp32). Biases and ``logit_bias`` stay fp32.
``bias_std`` defaults to 0 (the named workloads initialise biases to zero);
tests pass a non-zero value so that the bias paths are exercised.

Weight layout is the ``nn.Linear`` one, [out_features, in_features] row-major,
stacked over experts.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

ACT_RELU, ACT_GELU, ACT_SWIGLU = 0, 1, 2
ROUTING_TOKEN_CHOICE, ROUTING_EXPERT_CHOICE = 0, 1
# gate modes: A = softmax over the top-k logits; B = top-k of the full softmax,
# divided by their sum; C = top-k of the full softmax, raw (Switch).
GATE_TOPK_SOFTMAX, GATE_SOFTMAX_TOPK_RENORM, GATE_SOFTMAX_TOPK_RAW = 0, 1, 2
DT_F32, DT_BF16 = 0, 1

ACT_NAMES = {ACT_RELU: "relu", ACT_GELU: "gelu", ACT_SWIGLU: "swiglu"}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d_model: int
    n_experts: int
    top_k: int
    d_ff: int
    act: int
    gate_mode: int
    dtype: int
    capacity_factor: float = 0.0  # <= 0: no capacity limit
    router_bias: bool = False
    expert_bias: bool = False
    logit_bias_std: float = 0.0  # > 0: per-expert logit bias drawn and added
    n_shared: int = 0
    d_ff_shared: int = 0
    aux_alpha: float = 0.01
    router_std: float = 0.02
    bias_std: float = 0.0
    routing: int = ROUTING_TOKEN_CHOICE  # expert choice: C = floor(cf * T / E) per expert
    noisy: bool = False  # noisy top-k gating: draws w_noise (the draws of eps are separate)

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == DT_F32 else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == DT_F32 else 2


# ---- the five workloads the layer is measured on ---------------------------------
TINY_FP32 = Workload("tiny_top2_fp32_T64_d64_E8_k2_relu256", T=64, d_model=64, n_experts=8,
                     top_k=2, d_ff=256, act=ACT_RELU, gate_mode=GATE_TOPK_SOFTMAX,
                     dtype=DT_F32, router_bias=True, expert_bias=True)
MIXTRAL_PREFILL = Workload("mixtral_prefill_bf16_T4096_d4096_E8_k2_swiglu14336", T=4096,
                           d_model=4096, n_experts=8, top_k=2, d_ff=14336, act=ACT_SWIGLU,
                           gate_mode=GATE_TOPK_SOFTMAX, dtype=DT_BF16)
DEEPSEEK_FINE = Workload("deepseek_bf16_T8192_d2048_E64_k6_swiglu4096_shared2x8192", T=8192,
                         d_model=2048, n_experts=64, top_k=6, d_ff=4096, act=ACT_SWIGLU,
                         gate_mode=GATE_SOFTMAX_TOPK_RENORM, dtype=DT_BF16, n_shared=2,
                         d_ff_shared=8192)
SWITCH_CAPACITY = Workload("switch_top1_bf16_T16384_d1024_E128_gelu4096_cf1.25", T=16384,
                           d_model=1024, n_experts=128, top_k=1, d_ff=4096, act=ACT_GELU,
                           gate_mode=GATE_SOFTMAX_TOPK_RAW, dtype=DT_BF16,
                           capacity_factor=1.25, expert_bias=True, logit_bias_std=1.5)


# Expert-Choice routing on the Mixtral prefill layer: cf = 2 gives each of the 8
# experts C = 1024 of the 4096 tokens (the same expert work as top-2 token choice)
MIXTRAL_EC = MIXTRAL_PREFILL.replace(name="mixtral_ec_bf16_T4096_d4096_E8_cf2_swiglu14336",
                                     capacity_factor=2.0, top_k=1,
                                     routing=ROUTING_EXPERT_CHOICE)


# Noisy top-k gating (training mode of the ja page's TopKGating: softmax, top-2,
# renormalised) on the Mixtral prefill shapes
MIXTRAL_NOISY = MIXTRAL_PREFILL.replace(
    name="mixtral_noisy_bf16_T4096_d4096_E8_k2_swiglu14336", gate_mode=GATE_SOFTMAX_TOPK_RENORM,
    noisy=True)


def mixtral_decode(T: int) -> Workload:
    return MIXTRAL_PREFILL.replace(name=f"mixtral_decode_bf16_T{T}_d4096_E8_k2_swiglu14336", T=T)


WORKLOADS = {
    "tiny": TINY_FP32,
    "mixtral_prefill": MIXTRAL_PREFILL,
    "deepseek": DEEPSEEK_FINE,
    "switch": SWITCH_CAPACITY,
    "decode32": mixtral_decode(32),
    "decode8": mixtral_decode(8),
    "decode1": mixtral_decode(1),
    "mixtral_ec": MIXTRAL_EC,
    "mixtral_noisy": MIXTRAL_NOISY,
}

# ---- reduced shapes of the same families (several tiles plus a ragged tail) ------
SMALL = {
    "tiny": TINY_FP32.replace(name="tiny_bias", bias_std=0.1),
    "mixtral_small": MIXTRAL_PREFILL.replace(name="mixtral_small", T=333, d_model=256, d_ff=384),
    "deepseek_small": DEEPSEEK_FINE.replace(name="deepseek_small", T=517, d_model=256, d_ff=256,
                                            d_ff_shared=384),
    "switch_small": SWITCH_CAPACITY.replace(name="switch_small", T=2111, d_model=128, d_ff=256,
                                            n_experts=32, bias_std=0.1),
    "decode_small": MIXTRAL_PREFILL.replace(name="decode_small", T=5, d_model=256, d_ff=384),
    "deepseek_decode": DEEPSEEK_FINE.replace(name="deepseek_decode", T=20, d_model=256, d_ff=256,
                                             d_ff_shared=384),
    # a small batch whose down projection splits K: the combine reads its partials
    # and adds the shared experts' row
    "deepseek_decode_split": DEEPSEEK_FINE.replace(name="deepseek_decode_split", T=20,
                                                   d_model=128, d_ff=512, d_ff_shared=384),
    "decode_chunks": MIXTRAL_PREFILL.replace(name="decode_chunks", T=64, d_model=256, d_ff=384,
                                             n_experts=2, top_k=1),
    # decode-sized batches routed in one launch: capacity drops (cap 4 of 8 x 3
    # pairs over 6 experts), and 32 experts with top-8, router and logit biases
    "decode_cap": MIXTRAL_PREFILL.replace(name="decode_cap", T=8, d_model=256, d_ff=384,
                                          n_experts=6, top_k=3, capacity_factor=1.0),
    "decode_e32": DEEPSEEK_FINE.replace(name="decode_e32", T=8, d_model=192, d_ff=128,
                                        n_experts=32, top_k=8, n_shared=1, d_ff_shared=128,
                                        router_bias=True, bias_std=0.1, logit_bias_std=0.5),
    # SwiGLU experts with a capacity of 112 rows each
    "mixtral_cap": MIXTRAL_PREFILL.replace(name="mixtral_cap", T=900, d_model=256, d_ff=384,
                                           capacity_factor=0.5),
    # noisy top-k gating (softmax, top-2, renormalised, as the ja page's TopKGating):
    # bf16 with 16 experts (tensor-core router), fp32 with 8 (CUDA-core router)
    "noisy_small": MIXTRAL_PREFILL.replace(name="noisy_small", T=500, d_model=256, d_ff=128,
                                           n_experts=16, gate_mode=GATE_SOFTMAX_TOPK_RENORM,
                                           noisy=True),
    "noisy_fp32": TINY_FP32.replace(name="noisy_fp32", T=100, gate_mode=GATE_SOFTMAX_TOPK_RENORM,
                                    noisy=True, bias_std=0.1),
    # bf16 routers with 20 and 256 experts (expert counts that pad to the MMA's N),
    # router and logit biases, ragged token tiles
    "router_e20": DEEPSEEK_FINE.replace(name="router_e20", T=700, d_model=256, d_ff=128,
                                        n_experts=20, top_k=3, n_shared=0, d_ff_shared=0,
                                        router_bias=True, bias_std=0.1, logit_bias_std=0.5),
    "router_e256": SWITCH_CAPACITY.replace(name="router_e256", T=300, d_model=128, d_ff=64,
                                           n_experts=256, top_k=8, capacity_factor=0.0,
                                           bias_std=0.1),
    # Expert-Choice routing: bf16 SwiGLU (C = 93 of 300 tokens for each of 8 experts),
    # fp32 ReLU with biases, a bf16 GELU layer with 20 experts (C = 17)
    "ec_small": MIXTRAL_EC.replace(name="ec_small", T=300, d_model=256, d_ff=384,
                                   capacity_factor=2.5),
    "ec_fp32": TINY_FP32.replace(name="ec_fp32", T=64, top_k=1, capacity_factor=1.0,
                                 routing=ROUTING_EXPERT_CHOICE, bias_std=0.1),
    "ec_gelu20": SWITCH_CAPACITY.replace(name="ec_gelu20", T=347, d_model=128, d_ff=192,
                                         n_experts=20, capacity_factor=1.0, bias_std=0.1,
                                         routing=ROUTING_EXPERT_CHOICE),
    "fp32_swiglu": DEEPSEEK_FINE.replace(name="fp32_swiglu", T=150, d_model=96, d_ff=160,
                                         n_experts=16, top_k=3, dtype=DT_F32,
                                         d_ff_shared=64),
    "fp32_gelu_cap": SWITCH_CAPACITY.replace(name="fp32_gelu_cap", T=300, d_model=64, d_ff=128,
                                             n_experts=8, top_k=2, dtype=DT_F32,
                                             gate_mode=GATE_SOFTMAX_TOPK_RENORM,
                                             bias_std=0.2, router_bias=True),
}


def _normal(g: torch.Generator, shape, std: float) -> torch.Tensor:
    t = torch.empty(shape, dtype=torch.float32)
    t.normal_(0.0, std, generator=g)
    return t


def generate(w: Workload, seed: int = 0, with_weights: bool = True) -> dict:
    """Draw one workload's inputs on the CPU, following the module docstring's recipe.

    Returns a dict of CPU tensors: activations/weights in ``w.torch_dtype``,
    biases fp32, absent items as ``None``.
    """
    g = torch.Generator().manual_seed(seed)
    T, d, E, F = w.T, w.d_model, w.n_experts, w.d_ff
    dt = w.torch_dtype
    out: dict = {}
    out["x"] = _normal(g, (T, d), 1.0).to(dt)
    out["w_router"] = _normal(g, (E, d), w.router_std).to(dt)
    out["b_router"] = _normal(g, (E,), w.bias_std) if w.router_bias else None
    out["logit_bias"] = _normal(g, (E,), w.logit_bias_std) if w.logit_bias_std > 0 else None
    if not with_weights:
        return out
    swiglu = w.act == ACT_SWIGLU
    w1 = torch.empty((E, F, d), dtype=dt)
    w3 = torch.empty((E, F, d), dtype=dt) if swiglu else None
    w2 = torch.empty((E, d, F), dtype=dt)
    for e in range(E):
        w1[e] = _normal(g, (F, d), 1.0 / math.sqrt(d)).to(dt)
        if swiglu:
            w3[e] = _normal(g, (F, d), 1.0 / math.sqrt(d)).to(dt)
        w2[e] = _normal(g, (d, F), 1.0 / math.sqrt(F)).to(dt)
    out["w1"], out["w3"], out["w2"] = w1, w3, w2
    if w.expert_bias and not swiglu:
        out["b1"] = _normal(g, (E, F), w.bias_std)
        out["b2"] = _normal(g, (E, d), w.bias_std)
    else:
        out["b1"] = out["b2"] = None
    if w.n_shared > 0:
        Fs, ns = w.d_ff_shared, w.n_shared
        gate = torch.empty((ns * Fs, d), dtype=dt)
        up = torch.empty((ns * Fs, d), dtype=dt)
        down = torch.empty((d, ns * Fs), dtype=dt)
        for j in range(ns):
            gate[j * Fs:(j + 1) * Fs] = _normal(g, (Fs, d), 1.0 / math.sqrt(d)).to(dt)
            up[j * Fs:(j + 1) * Fs] = _normal(g, (Fs, d), 1.0 / math.sqrt(d)).to(dt)
            down[:, j * Fs:(j + 1) * Fs] = _normal(g, (d, Fs), 1.0 / math.sqrt(Fs)).to(dt)
        out["ws_gate"], out["ws_up"], out["ws_down"] = gate, up, down
    else:
        out["ws_gate"] = out["ws_up"] = out["ws_down"] = None
    # 8. (noisy gating only) the noise projection, drawn last so that every other
    #    draw is the same with and without it
    out["w_noise"] = _normal(g, (E, d), w.router_std).to(dt) if w.noisy else None
    return out


def noise_draws(T: int, E: int, seed: int) -> torch.Tensor:
    """Standard normal draws eps [T, E] fp32 of noisy top-k gating, seeded."""
    g = torch.Generator().manual_seed(seed)
    return _normal(g, (T, E), 1.0)


def random_logits(T: int, E: int, seed: int = 0, std: float = 1.0,
                  tie_fraction: float = 0.0) -> torch.Tensor:
    """Seeded fp32 router logits [T, E] fed identically to both routing implementations.

    With ``tie_fraction`` > 0 that share of rows is snapped to a coarse grid
    (multiples of 0.25) so that exact ties between experts occur.
    """
    g = torch.Generator().manual_seed(seed)
    z = _normal(g, (T, E), std)
    if tie_fraction > 0:
        pick = torch.rand((T,), generator=g) < tie_fraction
        z[pick] = torch.round(z[pick] * 4.0) / 4.0
    return z


def token_sample(T: int, n: int) -> torch.Tensor:
    """A fixed strided subset of ``n`` token indices (always includes the first and last)."""
    if n >= T:
        return torch.arange(T)
    idx = torch.linspace(0, T - 1, n).round().long()
    return torch.unique(idx)


def to_f64_numpy(t: Optional[torch.Tensor]):
    """Exact upcast of a CPU tensor to an fp64 numpy array (None passes through)."""
    if t is None:
        return None
    return t.detach().to(torch.float64).cpu().numpy()
