"""The seeded input recipe, as the module docstring of ``synth`` states it: one torch
CPU generator per call, fp32 normal draws in a fixed order, then one rounding to
the storage dtype. Re-drawn here step by step for two small workloads."""
import math

import torch

from sparse_mixture_experts_12_b200 import synth


def _draws(g, shape, std):
    return torch.empty(shape).normal_(0.0, std, generator=g)


def test_recipe_order_tiny_fp32():
    w = synth.SMALL["tiny"]  # fp32, router bias, expert biases (bias_std 0.1), ReLU
    inp = synth.generate(w, seed=3)
    g = torch.Generator().manual_seed(3)
    T, d, E, F = w.T, w.d_model, w.n_experts, w.d_ff
    assert torch.equal(inp["x"], _draws(g, (T, d), 1.0))
    assert torch.equal(inp["w_router"], _draws(g, (E, d), w.router_std))
    assert torch.equal(inp["b_router"], _draws(g, (E,), w.bias_std))
    for e in range(E):
        assert torch.equal(inp["w1"][e], _draws(g, (F, d), 1 / math.sqrt(d)))
        assert torch.equal(inp["w2"][e], _draws(g, (d, F), 1 / math.sqrt(F)))
    assert torch.equal(inp["b1"], _draws(g, (E, F), w.bias_std))
    assert torch.equal(inp["b2"], _draws(g, (E, d), w.bias_std))
    assert inp["w3"] is None and inp["logit_bias"] is None and inp["w_noise"] is None


def test_recipe_order_bf16_swiglu_shared_and_noise():
    w = synth.SMALL["deepseek_small"].replace(T=10, d_model=64, d_ff=64, d_ff_shared=64,
                                               n_experts=3, top_k=2, noisy=True)
    inp = synth.generate(w, seed=5)
    g = torch.Generator().manual_seed(5)
    T, d, E, F, Fs = w.T, w.d_model, w.n_experts, w.d_ff, w.d_ff_shared
    bf = torch.bfloat16
    assert torch.equal(inp["x"], _draws(g, (T, d), 1.0).to(bf))
    assert torch.equal(inp["w_router"], _draws(g, (E, d), w.router_std).to(bf))
    for e in range(E):
        assert torch.equal(inp["w1"][e], _draws(g, (F, d), 1 / math.sqrt(d)).to(bf))
        assert torch.equal(inp["w3"][e], _draws(g, (F, d), 1 / math.sqrt(d)).to(bf))
        assert torch.equal(inp["w2"][e], _draws(g, (d, F), 1 / math.sqrt(F)).to(bf))
    for j in range(w.n_shared):
        sl = slice(j * Fs, (j + 1) * Fs)
        assert torch.equal(inp["ws_gate"][sl], _draws(g, (Fs, d), 1 / math.sqrt(d)).to(bf))
        assert torch.equal(inp["ws_up"][sl], _draws(g, (Fs, d), 1 / math.sqrt(d)).to(bf))
        assert torch.equal(inp["ws_down"][:, sl], _draws(g, (d, Fs), 1 / math.sqrt(Fs)).to(bf))
    # the noise projection is drawn last, so every other draw matches the plain layer
    assert torch.equal(inp["w_noise"], _draws(g, (E, d), w.router_std).to(bf))
    plain = synth.generate(w.replace(noisy=False), seed=5)
    for key in ("x", "w_router", "w1", "w3", "w2", "ws_gate", "ws_up", "ws_down"):
        assert torch.equal(plain[key], inp[key]), key


def test_noise_draws_are_seeded_standard_normal():
    a = synth.noise_draws(7, 3, seed=11)
    b = synth.noise_draws(7, 3, seed=11)
    g = torch.Generator().manual_seed(11)
    assert torch.equal(a, b) and torch.equal(a, _draws(g, (7, 3), 1.0))
    assert a.dtype == torch.float32
