"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Every input is seeded and synthetic (sparse_mixture_experts_12_b200.synth); no
expected value comes from the CUDA path. Integer outputs (indices, counts,
offsets, permutation, drop decisions) must be bit-exact when both sides see the
same logits / routing; floating outputs must be within the per-token max
relative error of 1e-5 (fp32 layers) or 2e-2 (bf16 storage, fp32 accumulation).
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_12_b200 import binding as B
from sparse_mixture_experts_12_b200 import build as BUILD
from sparse_mixture_experts_12_b200 import synth
from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    BUILD.build()
    B.load()


def _raw_ws(cfg):
    return B.new_workspace(cfg, DEV)


def _s():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _devcheck(ws, expect=0):
    code, info = ctypes.c_int32(0), ctypes.c_int32(0)
    B.load().moe_last_device_error(_p(ws), ctypes.byref(code), ctypes.byref(info), _s())
    assert code.value == expect, (code.value, info.value)
    return info.value


# =============================================================== routing (bit-exact)
ROUTE_CASES = [(E, k, mode) for E in (1, 3, 8, 16, 20, 33, 64, 65, 128, 129, 256)
               for k in sorted({1, 2, min(6, E), min(8, E)}) if k <= E
               for mode in (0, 1, 2)]


@pytest.mark.parametrize("E,k,mode", ROUTE_CASES)
def test_route_given_logits_bitexact(E, k, mode):
    T = 301
    z = synth.random_logits(T, E, seed=E * 100 + k * 10 + mode, std=1.5, tie_fraction=0.3)
    wl = synth.SMALL["mixtral_small"].replace(T=T, n_experts=E, top_k=k, gate_mode=mode)
    cfg = B.make_cfg(wl)
    ws = _raw_ws(cfg)
    logits = z.to(DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gate = torch.empty((T, k), dtype=torch.float32, device=DEV)
    W = B.MoeWeights()
    st = B.load().moe_route(ctypes.byref(cfg), ctypes.byref(W), None, _p(logits), _p(idx),
                            _p(gate), _p(ws), ws.numel(), _s())
    assert st == 0
    torch.cuda.synchronize()
    zn = z.numpy()
    ref_idx = O.select_topk(zn, k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    ref_g = O.gate_values(zn, ref_idx, H.MODE[mode])
    assert np.allclose(gate.cpu().numpy(), ref_g, rtol=4e-6, atol=1e-7)
    _devcheck(ws)


# shapes of the tensor-core router: expert counts padded to N = 16 .. 256, K split
# over 1, 2 or 4 CTAs of a cluster, token tiles with ragged tails, one-token batches
ROUTE_TC_CASES = [
    # E, k, T, d, gate mode, biases
    (1, 1, 77, 128, 0, False), (8, 2, 1, 4096, 0, False), (8, 2, 129, 256, 1, True),
    (8, 2, 4096, 4096, 0, False), (16, 4, 300, 192, 2, True), (33, 3, 1000, 512, 0, True),
    (64, 6, 257, 2048, 1, False), (64, 6, 8192, 2048, 1, False), (128, 1, 5000, 1024, 2, True),
    (200, 8, 130, 256, 1, True), (256, 8, 64, 128, 0, False), (20, 5, 33, 64, 2, True),
]


@pytest.mark.parametrize("E,k,T,d,mode,bias", ROUTE_TC_CASES,
                         ids=[f"E{c[0]}_k{c[1]}_T{c[2]}_d{c[3]}" for c in ROUTE_TC_CASES])
def test_route_tc_matches_oracle(E, k, T, d, mode, bias):
    """moe_route with x (bf16): logits within the fp32 accumulation bound; the
    selection and the gates exactly those the oracle takes from the same logits."""
    wl = synth.SMALL["mixtral_small"].replace(T=T, n_experts=E, top_k=k, gate_mode=mode,
                                              d_model=d, router_bias=bias, bias_std=0.1,
                                              logit_bias_std=0.5 if bias else 0.0)
    inp = synth.generate(wl, seed=E + T + d, with_weights=False)
    layer = B.MoELayer(wl, inp, DEV)
    x = inp["x"].to(DEV)
    logits = torch.empty((T, E), dtype=torch.float32, device=DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gate = torch.empty((T, k), dtype=torch.float32, device=DEV)
    layer.route(x, logits, idx, gate)
    torch.cuda.synchronize()
    P = H.oracle_params(inp)
    extra = np.zeros(E)
    for key in ("b_router", "logit_bias"):
        if P[key] is not None:
            extra += np.abs(P[key])
    z64 = O.router_logits(P["x"], P["w_router"], P["b_router"], P["logit_bias"])
    zg = logits.cpu().numpy()
    assert np.all(np.abs(zg.astype(np.float64) - z64) <=
                  H.logits_bound(P["x"], P["w_router"], extra))
    ref_idx = O.select_topk(zg, k)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    assert np.allclose(gate.cpu().numpy(), O.gate_values(zg, ref_idx, H.MODE[mode]),
                       rtol=4e-6, atol=1e-7)
    _devcheck(layer.ws)


# ============================================================= permute (bit-exact)
PERMUTE_CASES = [
    # E, k, T, cf, dtype
    (8, 2, 1000, 0.0, synth.DT_BF16),
    (8, 2, 1000, 1.0, synth.DT_BF16),
    (64, 6, 777, 0.0, synth.DT_BF16),
    (128, 1, 3001, 1.25, synth.DT_BF16),
    (256, 8, 513, 0.5, synth.DT_BF16),
    (3, 3, 65, 0.8, synth.DT_F32),
    (33, 4, 129, 0.0, synth.DT_F32),
    (1, 1, 50, 0.3, synth.DT_BF16),
]


@pytest.mark.parametrize("E,k,T,cf,dt", PERMUTE_CASES)
def test_permute_given_routing_bitexact(E, k, T, cf, dt):
    d = 192 if dt == synth.DT_BF16 else 36
    wl = synth.SMALL["mixtral_small"].replace(T=T, n_experts=E, top_k=k, capacity_factor=cf,
                                              d_model=d, dtype=dt)
    cfg = B.make_cfg(wl)
    ws = _raw_ws(cfg)
    z = synth.random_logits(T, E, seed=E + T, std=2.0)
    if E >= 64:  # skew the load so that capacity bites
        z = z + torch.linspace(3.0, -3.0, E)[None, :]
    ref_idx = O.select_topk(z.numpy(), k)
    x = synth.generate(wl, seed=T, with_weights=False)["x"]
    xd = x.to(DEV)
    idx = torch.from_numpy(ref_idx).to(DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.full((T * k,), -7, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    x_perm = torch.zeros((T * k, d), dtype=x.dtype, device=DEV)
    st = B.load().moe_permute(ctypes.byref(cfg), _p(xd), _p(idx), _p(counts), _p(offsets),
                              _p(perm), _p(inv), _p(x_perm), _p(ws), ws.numel(), _s())
    assert st == 0
    torch.cuda.synchronize()
    cap = O.capacity(cf, T, k, E)
    rc, rank, kept = O.dispatch(ref_idx, E, cap)
    roff, rperm, rinv = O.expert_layout(ref_idx, rank, kept, E)
    R = int(roff[-1])
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), roff)
    assert np.array_equal(perm.cpu().numpy()[:R], rperm)
    assert np.array_equal(inv.cpu().numpy().reshape(T, k), rinv)
    xp = x_perm.cpu()
    assert torch.equal(xp[:R], x[torch.from_numpy(rperm)])
    if cap is not None:
        assert (~kept).any() or E == 1
    H.report("permute", E=E, k=k, T=T, cap=cap, dropped=int((~kept).sum()))
    _devcheck(ws)


def test_permute_reports_bad_expert_index():
    """A corrupted routing index is reported through the device error word (no fault)."""
    T, E, k = 100, 8, 2
    wl = synth.SMALL["mixtral_small"].replace(T=T, n_experts=E, top_k=k, d_model=64)
    cfg = B.make_cfg(wl)
    ws = _raw_ws(cfg)
    ref_idx = O.select_topk(synth.random_logits(T, E, seed=5).numpy(), k)
    bad = ref_idx.copy()
    bad[37, 1] = 99
    x = synth.generate(wl, seed=1, with_weights=False)["x"].to(DEV)
    outs = [torch.empty(E, dtype=torch.int32, device=DEV),
            torch.empty(E + 1, dtype=torch.int32, device=DEV),
            torch.empty(T * k, dtype=torch.int32, device=DEV),
            torch.empty(T * k, dtype=torch.int32, device=DEV),
            torch.empty((T * k, 64), dtype=torch.bfloat16, device=DEV)]
    bad_d = torch.from_numpy(bad).to(DEV)
    st = B.load().moe_permute(ctypes.byref(cfg), _p(x), _p(bad_d), *[_p(o) for o in outs],
                              _p(ws), ws.numel(), _s())
    assert st == 0
    info = _devcheck(ws, expect=1)
    assert info == 37 * k + 1
    assert int(outs[3].cpu()[37 * k + 1]) == -1
    _devcheck(ws, expect=0)  # the word is cleared after reading


# ========================================================== expert FFN (tolerance)
FFN_CASES = [
    # name, act, dtype, d, F, E, rows per expert
    ("swiglu_bf16", synth.ACT_SWIGLU, synth.DT_BF16, 256, 384, 5, [0, 1, 129, 300, 64]),
    ("swiglu_bf16_ntail", synth.ACT_SWIGLU, synth.DT_BF16, 192, 192, 3, [200, 0, 17]),
    ("gelu_bf16_bias", synth.ACT_GELU, synth.DT_BF16, 128, 320, 4, [5, 260, 0, 128]),
    ("relu_bf16_bias", synth.ACT_RELU, synth.DT_BF16, 320, 256, 2, [131, 7]),
    ("swiglu_f32", synth.ACT_SWIGLU, synth.DT_F32, 96, 160, 4, [3, 140, 0, 33]),
    ("relu_f32_bias", synth.ACT_RELU, synth.DT_F32, 64, 256, 8, [16] * 8),
    ("gelu_f32_odd", synth.ACT_GELU, synth.DT_F32, 36, 50, 3, [1, 2, 300]),
    # at most 32 rows in all: the small-batch path (weights on the MMA's M side,
    # split-K down projection)
    ("swiglu_bf16_decode", synth.ACT_SWIGLU, synth.DT_BF16, 256, 384, 5, [0, 1, 3, 7, 2]),
    ("gelu_bf16_decode_bias", synth.ACT_GELU, synth.DT_BF16, 128, 320, 4, [5, 0, 9, 2]),
    ("relu_bf16_decode_ntail", synth.ACT_RELU, synth.DT_BF16, 192, 192, 2, [1, 12]),
    # still the small-batch path, with an expert spanning two 32-row chunks
    ("swiglu_bf16_decode_chunks", synth.ACT_SWIGLU, synth.DT_BF16, 256, 384, 2, [33, 20]),
    # at most 8 rows in all (decode T = 1..4)
    ("swiglu_bf16_decode_tiny", synth.ACT_SWIGLU, synth.DT_BF16, 256, 384, 2, [1, 1]),
    ("swiglu_bf16_decode_tiny_k", synth.ACT_SWIGLU, synth.DT_BF16, 512, 384, 3, [1, 0, 1]),
    ("gelu_bf16_decode_chunks", synth.ACT_GELU, synth.DT_BF16, 128, 256, 2, [45, 10]),
    # 190..256 rows in all: one or two 128-row tiles per expert
    ("swiglu_bf16_medium", synth.ACT_SWIGLU, synth.DT_BF16, 256, 384, 5, [0, 1, 129, 60, 30]),
    ("gelu_bf16_medium_bias", synth.ACT_GELU, synth.DT_BF16, 128, 320, 4, [200, 0, 17, 33]),
    ("relu_bf16_medium_ntail", synth.ACT_RELU, synth.DT_BF16, 192, 192, 2, [100, 90]),
    # reductions of 2048 and more over experts averaging 256+ rows: the 256 x 512
    # CTA-pair tile (ragged N, pair tiles whose second CTA holds no row or one row)
    ("swiglu_bf16_wide_up", synth.ACT_SWIGLU, synth.DT_BF16, 2112, 320, 3, [300, 0, 529]),
    ("gelu_bf16_wide_down_bias", synth.ACT_GELU, synth.DT_BF16, 192, 2112, 3, [260, 5, 600]),
    ("relu_bf16_wide_both", synth.ACT_RELU, synth.DT_BF16, 2048, 2048, 2, [129, 400]),
    # the same reduction lengths over experts with few rows: 128-row single-CTA tiles
    ("swiglu_bf16_long_k_few_rows", synth.ACT_SWIGLU, synth.DT_BF16, 2112, 320, 3,
     [100, 0, 200]),
    # 80 wide tiles over the 74 CTA pairs of a B200: the last round runs as half tiles
    ("relu_bf16_wide_tail", synth.ACT_RELU, synth.DT_BF16, 2048, 2048, 4,
     [1300, 1300, 1000, 1000]),
    ("swiglu_bf16_wide_tail", synth.ACT_SWIGLU, synth.DT_BF16, 2048, 1024, 4,
     [1300, 1300, 1000, 1000]),
]


# Capacity-limited layers (name, act, d, F, E, rows per expert, capacity): experts
# at and below the capacity, the 128-row tiles of the single-CTA kernel split over
# a capacity of 131-160 rows, and an expert given more rows than the capacity
# (moe_expert_ffn takes any offsets).
FFN_CAP_CASES = [
    ("gelu_bf16_cap160", synth.ACT_GELU, 128, 320, 4, [5, 160, 0, 131], 160),
    ("swiglu_bf16_cap128", synth.ACT_SWIGLU, 256, 384, 5, [0, 1, 128, 77, 40], 128),
    ("relu_bf16_cap_over", synth.ACT_RELU, 192, 192, 3, [200, 17, 96], 96),
    ("gelu_bf16_cap_long_k", synth.ACT_GELU, 1024, 4096, 3, [150, 3, 100], 160),
]


@pytest.mark.parametrize("name,act,dt,d,F,E,rows", FFN_CASES, ids=[c[0] for c in FFN_CASES])
def test_expert_ffn_matches_oracle(name, act, dt, d, F, E, rows):
    _expert_ffn_case(name, act, dt, d, F, E, rows)


@pytest.mark.parametrize("name,act,d,F,E,rows,cap", FFN_CAP_CASES,
                         ids=[c[0] for c in FFN_CAP_CASES])
def test_expert_ffn_capacity_layers_match_oracle(name, act, d, F, E, rows, cap):
    _expert_ffn_case(name, act, synth.DT_BF16, d, F, E, rows, cap=cap)


def _expert_ffn_case(name, act, dt, d, F, E, rows, cap=None):
    R = int(sum(rows))
    k = 2
    T = (R + k - 1) // k + 3  # x_perm holds T*k rows; the tail rows are unused
    # capacity floor(cf * T * k / E) == cap
    cf = 0.0 if cap is None else (cap + 0.5) * E / (T * k)
    wl = synth.Workload(name, T=T, d_model=d, n_experts=E, top_k=k, d_ff=F, act=act,
                        gate_mode=0, dtype=dt, expert_bias=act != synth.ACT_SWIGLU,
                        bias_std=0.3, capacity_factor=cf)
    if cap is not None:
        assert O.capacity(cf, T, k, E) == cap
    inp = synth.generate(wl, seed=R)
    layer = B.MoELayer(wl, inp, DEV)
    g = torch.Generator().manual_seed(R + 1)
    xp = torch.randn((T * k, d), generator=g).to(wl.torch_dtype)
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(rows)]), dtype=torch.int32)
    y = torch.full((T * k, d), float("nan"), dtype=wl.torch_dtype, device=DEV)
    layer.expert_ffn(xp.to(DEV), offsets.to(DEV), y)
    torch.cuda.synchronize()
    yc = y.cpu().to(torch.float64).numpy()
    P = H.oracle_params(inp)
    worst = 0.0
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b == a:
            continue
        ref = O.expert_ffn(synth.to_f64_numpy(xp[a:b]), H.ACT[act], P["w1"][e], P["w2"][e],
                           None if P["w3"] is None else P["w3"][e],
                           None if P["b1"] is None else P["b1"][e],
                           None if P["b2"] is None else P["b2"][e])
        err = H.max_rel_err(yc[a:b], ref)
        worst = max(worst, float(err.max()))
    H.report("expert_ffn", case=name, worst_rel_err=worst)
    assert worst <= H.TOL[dt], worst
    # rows outside every expert's range are never written
    assert np.isnan(yc[R:]).all()
    _devcheck(layer.ws)


def test_expert_ffn_rejects_bad_offsets():
    wl = synth.SMALL["mixtral_small"].replace(T=64, d_model=128, d_ff=128)
    layer = B.MoELayer(wl, synth.generate(wl, seed=2), DEV)
    xp = torch.zeros((128, 128), dtype=torch.bfloat16, device=DEV)
    y = torch.zeros_like(xp)
    bad = torch.tensor([0, 10, 5, 20, 20, 30, 40, 50, 60], dtype=torch.int32, device=DEV)
    layer.expert_ffn(xp, bad, y)
    code, info = layer.last_device_error()
    assert code == 2 and info == 1


def test_shared_experts_through_expert_ffn():
    wl = synth.SMALL["deepseek_small"]
    inp = synth.generate(wl, seed=3)
    layer = B.MoELayer(wl, inp, DEV)
    cfg, wt = B.shared_as_experts(layer)
    x = inp["x"].to(DEV)
    y = torch.empty_like(x)
    offsets = torch.tensor([0, wl.T], dtype=torch.int32, device=DEV)
    layer.expert_ffn(x, offsets, y, cfg=cfg, weights=wt)
    torch.cuda.synchronize()
    P = H.oracle_params(inp)
    ref = O.shared_experts(P["x"], P["ws_gate"], P["ws_up"], P["ws_down"], wl.n_shared)
    err = H.max_rel_err(y.cpu().to(torch.float64).numpy(), ref)
    assert err.max() <= H.TOL[wl.dtype], err.max()


# =================================================================== combine
# k = 1 without a shared row takes the 8-tokens-per-warp kernel (T = 333 leaves a
# last warp with 5 tokens)
@pytest.mark.parametrize("dt,with_shared,k", [(synth.DT_BF16, False, 3), (synth.DT_BF16, True, 3),
                                              (synth.DT_F32, True, 3), (synth.DT_BF16, False, 1),
                                              (synth.DT_F32, False, 1), (synth.DT_BF16, True, 1)])
def test_combine_matches_oracle(dt, with_shared, k):
    T, d = 333, 128
    wl = synth.SMALL["mixtral_small"].replace(T=T, top_k=k, d_model=d, dtype=dt)
    cfg = B.make_cfg(wl)
    ws = _raw_ws(cfg)
    g = torch.Generator().manual_seed(9)
    R = T * k
    y_rows = torch.randn((R, d), generator=g).to(wl.torch_dtype)
    inv = torch.randperm(R, generator=g)[:T * k].reshape(T, k).to(torch.int32)
    drop = torch.rand((T, k), generator=g) < 0.2
    inv[drop] = -1
    inv[5] = -1  # a token with every slot dropped
    gates = torch.rand((T, k), generator=g)
    shared = torch.randn((T, d), generator=g) if with_shared else None
    y = torch.empty((T, d), dtype=wl.torch_dtype, device=DEV)
    # keep every device tensor referenced until the kernels have run
    yr_d, inv_d, g_d = y_rows.to(DEV), inv.to(DEV), gates.to(DEV)
    sh_d = None if shared is None else shared.to(DEV)
    st = B.load().moe_combine(ctypes.byref(cfg), _p(yr_d), _p(inv_d), _p(g_d), _p(sh_d), _p(y),
                              _p(ws), ws.numel(), _s())
    assert st == 0
    torch.cuda.synchronize()
    ref = O.combine(synth.to_f64_numpy(y_rows), inv.numpy(), gates.numpy().astype(np.float64),
                    None if shared is None else shared.numpy())
    err = H.max_rel_err(y.cpu().to(torch.float64).numpy(), ref)
    assert err.max() <= H.TOL[dt], err.max()
    if not with_shared:
        assert torch.all(y[5] == 0)
    _devcheck(ws)


# ================================================================= aux statistics
@pytest.mark.parametrize("E,k", [(8, 2), (64, 6), (128, 1), (5, 5)])
def test_aux_stats_matches_oracle(E, k):
    T = 1237
    wl = synth.SMALL["mixtral_small"].replace(T=T, n_experts=E, top_k=k)
    cfg = B.make_cfg(wl)
    ws = _raw_ws(cfg)
    z = synth.random_logits(T, E, seed=E, std=2.0)
    idx = O.select_topk(z.numpy(), k)
    out = torch.zeros(3 + 2 * E, dtype=torch.float32, device=DEV)
    z_d, idx_d = z.to(DEV), torch.from_numpy(idx).to(DEV)
    st = B.load().moe_aux_stats(ctypes.byref(cfg), _p(z_d), _p(idx_d), _p(out), _p(ws),
                                ws.numel(), _s())
    assert st == 0
    torch.cuda.synchronize()
    o = out.cpu().numpy().astype(np.float64)
    f, P, aux = O.aux_stats(z.numpy(), idx, E, k, wl.aux_alpha)
    assert np.allclose(o[3:3 + E], f, rtol=1e-6, atol=0)
    assert np.allclose(o[3 + E:], P, rtol=2e-5, atol=1e-7)
    assert abs(o[0] - aux) <= 2e-5 * aux
    assert abs(o[1] - O.router_z_loss(z.numpy())) <= 2e-5 * O.router_z_loss(z.numpy())
    assert abs(o[2] - O.balance_sq_loss(idx, E)) <= 1e-6 + 1e-5 * O.balance_sq_loss(idx, E)


# ====================================================================== whole layer
NOISE_OFFSET = 7


def _forward_and_compare(wl: synth.Workload, seed: int, n_sample=None, check_full_routing=True,
                         noise_seed=None, with_aux=True):
    """noise_seed (noisy workloads): the library draws the noise for (noise_seed,
    NOISE_OFFSET) and the oracle the same counter-based draws; otherwise the noise is
    a seeded input both sides read. with_aux=False: the forward without the
    load-balancing statistics (the path of a layer that does not ask for them)."""
    inp = synth.generate(wl, seed=seed)
    layer = B.MoELayer(wl, inp, DEV)
    x = inp["x"].to(DEV)
    taps = layer.new_taps()
    aux = layer.new_aux() if with_aux else None
    eps = e64 = None
    if wl.noisy and noise_seed is None:
        eps = synth.noise_draws(wl.T, wl.n_experts, seed + 99)
        e64 = eps.numpy().astype(np.float64)
    elif wl.noisy:
        e64 = O.noise_draws(wl.T, wl.n_experts, noise_seed, NOISE_OFFSET)[0]
    if not wl.noisy:
        y = layer.forward(x, taps=taps, aux=aux)
    elif eps is not None:
        y = layer.forward_noisy(x, eps.to(DEV), taps=taps, aux=aux)
    else:
        y = layer.forward_noisy(x, seed=noise_seed, offset=NOISE_OFFSET, taps=taps, aux=aux)
    torch.cuda.synchronize()
    code, info = layer.last_device_error()
    assert code == 0, (code, info)
    P = H.oracle_params(inp)
    T, E, k = wl.T, wl.n_experts, wl.top_k
    ref_logits = None
    if wl.noisy:
        ref_logits = O.noisy_router_logits(P["x"], P["w_router"], P["w_noise"], e64,
                                           P["b_router"], P["logit_bias"])
    kw = H.oracle_kwargs(wl)
    tokens = tiles = None
    if n_sample is not None:
        # compared tokens from the oracle's routing: the first and the last row of
        # every (expert, 128-row tile) of the grouped GEMMs, of every tile of the
        # shared experts' GEMM (its rows are the tokens), some dropped tokens, and
        # a strided sample
        r0 = O.route(P["x"], P, top_k=k, gate_mode=kw["gate_mode"],
                     capacity_factor=wl.capacity_factor, logits=ref_logits)
        ref_logits = r0["logits"]
        dropped = np.nonzero(~r0["kept"].all(axis=1))[0]
        extra = list(dropped[np.unique(np.linspace(0, len(dropped) - 1, 8).astype(int))]) \
            if len(dropped) else []
        if wl.n_shared > 0:
            for t0 in range(0, T, H.ROW_TILE):
                extra += [t0, min(t0 + H.ROW_TILE, T) - 1]
        tokens, tiles = H.tile_cover_tokens(r0["perm"], r0["offsets"], T, n_sample, extra)
    yref, r = O.moe_forward(P["x"], P, tokens=tokens, logits=ref_logits, **kw)
    # logits against the fp32 accumulation bound
    extra = np.zeros(E)
    if P["b_router"] is not None:
        extra += np.abs(P["b_router"])
    if P["logit_bias"] is not None:
        extra += np.abs(P["logit_bias"])
    bound = H.logits_bound(P["x"], P["w_router"], extra)
    if wl.noisy:  # + |eps| (bound of x W_noise^T + softplus rounding) + final roundings
        zn = P["x"] @ P["w_noise"].T
        sp = O.softplus(zn)
        zpl = P["x"] @ P["w_router"].T
        bound = bound + np.abs(e64) * (H.logits_bound(P["x"], P["w_noise"]) + 8 * H.U32 * sp) \
            + 4 * H.U32 * (np.abs(zpl) + extra[None, :] + sp * np.abs(e64))
        if eps is None:  # the device's fp32 draws differ from the fp64 ones by <= 8 ulp
            bound = bound + sp * H.EPS_REL * np.abs(e64)
    zg = taps["logits"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(zg - r["logits"]) <= bound)
    if wl.noisy:  # the forward's selection, on its own noisy logits, is bit-exact
        gi = torch.empty((T, k), dtype=torch.int32, device=DEV)
        gg = torch.empty((T, k), dtype=torch.float32, device=DEV)
        layer.route(None, taps["logits"], gi, gg)
        torch.cuda.synchronize()
        assert torch.equal(gi, taps["topk_idx"])
        li = torch.empty((T, E), dtype=torch.float32, device=DEV)
        if eps is not None:
            layer.route_noisy(x, eps.to(DEV), li, gi, gg)
        else:
            layer.route_noisy_seeded(x, noise_seed, NOISE_OFFSET, li, gi, gg)
        torch.cuda.synchronize()
        assert torch.equal(li, taps["logits"]) and torch.equal(gi, taps["topk_idx"])
    # the forward's own routing: differences only on near-ties
    gidx = taps["topk_idx"].cpu().numpy()
    mism, affected, n_near = H.routing_compare(gidx, r["logits"], r["idx"], k, r["capacity"])
    if len(mism) == 0:
        assert np.array_equal(taps["counts"].cpu().numpy(), r["counts"])
        assert np.array_equal(taps["offsets"].cpu().numpy(), r["offsets"])
        R = int(r["offsets"][-1])
        assert np.array_equal(taps["perm"].cpu().numpy()[:R], r["perm"])
        assert np.array_equal(taps["inv"].cpu().numpy().reshape(T, k), r["inv"])
        gg = taps["topk_gate"].cpu().numpy()
        assert np.allclose(gg, r["gates"], rtol=2e-5, atol=1e-6)
    # outputs on the compared tokens
    sel = np.arange(T) if tokens is None else tokens
    keep = np.array([t not in affected for t in sel])
    yg = y.cpu().to(torch.float64).numpy()[sel]
    err = H.max_rel_err(yg[keep], yref[keep])
    if with_aux:  # aux statistics (f from the forward's own routing)
        a = aux.cpu().numpy().astype(np.float64)
        f, Pm, auxv = O.aux_stats(r["logits"], r["idx"], E, k, wl.aux_alpha)
        assert np.abs(a[3:3 + E] - f).max() <= len(mism) / (T * k) + 1e-7
        assert np.allclose(a[3 + E:], Pm, rtol=1e-4, atol=1e-6)
        assert abs(a[0] - auxv) <= 1e-4 * auxv + wl.aux_alpha * E * len(mism) / (T * k)
    cover = {}
    if tiles is not None:
        covered = H.tiles_covered(tiles, r["perm"], sel[keep])
        cover = dict(tiles=len(tiles), tiles_covered=covered)
        if len(mism) == 0:  # every expert tile of the GEMMs has a compared row
            assert covered == len(tiles), (covered, len(tiles))
    H.report("forward", workload=wl.name, T=T, compared=int(keep.sum()), **cover,
             worst_rel_err=float(err.max()) if len(err) else 0.0,
             p99_rel_err=float(np.quantile(err, 0.99)) if len(err) else 0.0,
             routing_mismatch=len(mism), near_tie_tokens=n_near, excluded=len(affected),
             dropped=int((~r["kept"]).sum()), R=int(r["offsets"][-1]))
    assert err.max() <= H.TOL[wl.dtype], (wl.name, float(err.max()))
    if check_full_routing:
        _routing_on_oracle_logits(wl, layer, inp, r)
    return layer, y


def _routing_on_oracle_logits(wl, layer, inp, r):
    """Feed the oracle's fp32 logits and routing to the GPU routing and permute
    steps: everything integer must then be bit-exact at full size."""
    T, E, k = wl.T, wl.n_experts, wl.top_k
    logits = torch.from_numpy(r["logits"]).to(DEV)
    idx = torch.empty((T, k), dtype=torch.int32, device=DEV)
    gate = torch.empty((T, k), dtype=torch.float32, device=DEV)
    layer.route(None, logits, idx, gate)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
    perm = torch.empty(T * k, dtype=torch.int32, device=DEV)
    inv = torch.empty(T * k, dtype=torch.int32, device=DEV)
    xp = torch.empty((T * k, wl.d_model), dtype=wl.torch_dtype, device=DEV)
    layer.permute(inp["x"].to(DEV), torch.from_numpy(r["idx"]).to(DEV), counts, offsets, perm,
                  inv, xp)
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), r["idx"])
    assert np.allclose(gate.cpu().numpy(), r["gates"], rtol=4e-6, atol=1e-7)
    assert np.array_equal(counts.cpu().numpy(), r["counts"])
    assert np.array_equal(offsets.cpu().numpy(), r["offsets"])
    R = int(r["offsets"][-1])
    assert np.array_equal(perm.cpu().numpy()[:R], r["perm"])
    assert np.array_equal(inv.cpu().numpy().reshape(T, k), r["inv"])
    code, _ = layer.last_device_error()
    assert code == 0


TOKEN_CHOICE_SMALL = sorted(n for n, w in synth.SMALL.items()
                            if w.routing == synth.ROUTING_TOKEN_CHOICE)
EXPERT_CHOICE_SMALL = sorted(n for n, w in synth.SMALL.items()
                             if w.routing == synth.ROUTING_EXPERT_CHOICE)


@pytest.mark.parametrize("name", TOKEN_CHOICE_SMALL)
def test_forward_small_matches_oracle(name):
    _forward_and_compare(synth.SMALL[name], seed=0)


FULL = ["tiny", "mixtral_prefill", "deepseek", "switch", "decode32", "decode8", "decode1",
        "mixtral_noisy"]


@pytest.mark.parametrize("name", FULL)
def test_forward_full_size_sampled(name):
    wl = synth.WORKLOADS[name]
    n = None if wl.T <= 64 else 48
    # the noisy layer at full size draws its noise inside the library, as in the benchmark
    _forward_and_compare(wl, seed=0, n_sample=n, noise_seed=2024 if wl.noisy else None)
    torch.cuda.empty_cache()


# Decode-sized batches whose layer asks for no statistics: with at most 8 tokens
# and 32 experts (bf16) the router also lays out the experts (counts, capacity,
# offsets, tile table) in the same launch, the path of the benchmark's decode steps
# at T = 1 and 8; deepseek_decode (64 experts) and T = 32 take the tensor-core
# router and the scan.
SMALL_BATCH = ["decode_small", "decode_cap", "decode_e32", "deepseek_decode"]


@pytest.mark.parametrize("name", SMALL_BATCH)
def test_forward_small_batch_without_statistics(name):
    _forward_and_compare(synth.SMALL[name], seed=0, with_aux=False)


# edge shapes of the one-launch decode routing: one expert, k = E, 32 experts with
# top-8, odd expert counts, a d that leaves most threads without columns, each gate
# mode, capacity drops
SMALL_ROUTE_EDGES = [
    # T, E, k, d, gate mode, capacity factor
    (1, 1, 1, 64, 0, 0.0),
    (3, 4, 4, 128, 1, 0.0),
    (8, 32, 8, 192, 1, 0.0),
    (7, 17, 5, 64, 2, 0.0),
    (8, 9, 2, 256, 0, 0.6),   # capacity 1
    (5, 32, 1, 128, 2, 7.0),  # capacity 1
]


@pytest.mark.parametrize("T,E,k,d,mode,cf", SMALL_ROUTE_EDGES)
def test_forward_small_batch_routing_edges(T, E, k, d, mode, cf):
    wl = synth.SMALL["decode_small"].replace(name=f"edge_T{T}_E{E}_k{k}", T=T, n_experts=E,
                                             top_k=k, d_model=d, d_ff=128, gate_mode=mode,
                                             capacity_factor=cf, router_bias=True,
                                             bias_std=0.1, logit_bias_std=0.3)
    _forward_and_compare(wl, seed=T + E, with_aux=False)


@pytest.mark.parametrize("name", ["decode1", "decode8", "decode32"])
def test_forward_decode_without_statistics(name):
    _forward_and_compare(synth.WORKLOADS[name], seed=0, with_aux=False)
    torch.cuda.empty_cache()


NOISY_SMALL = sorted(n for n, w in synth.SMALL.items() if w.noisy)


@pytest.mark.parametrize("name", NOISY_SMALL)
def test_forward_noisy_seeded_matches_oracle(name):
    """The noise drawn inside the library for (seed, offset), the oracle drawing the
    same counter-based noise: the whole layer as with the noise as an input."""
    _forward_and_compare(synth.SMALL[name], seed=0, noise_seed=(1 << 40) + 17)


NOISE_CASES = [(1, 1, 0, 0), (333, 6, 42, 3), (4096, 64, (1 << 40) + 3, (1 << 33) + 5),
               (5000, 128, 7, 123456789), (17, 250, 2 ** 64 - 1, 2 ** 64 - 1)]


@pytest.mark.parametrize("T,E,seed,offset", NOISE_CASES)
def test_noise_draws_match_oracle(T, E, seed, offset):
    """moe_noise_draws: the Philox words bit-exact, the normal draws within 8 ulp
    (relative) of the oracle's fp64 Box-Muller on the same uniforms."""
    Q = (E + 3) // 4
    eps = torch.full((T, E), float("nan"), dtype=torch.float32, device=DEV)
    raw = torch.zeros((T, Q, 4), dtype=torch.int32, device=DEV)
    B.noise_draws(T, E, seed, offset, eps, raw)
    torch.cuda.synchronize()
    ref, ref_raw = O.noise_draws(T, E, seed, offset)
    got_raw = raw.cpu().numpy().view(np.uint32)
    assert np.array_equal(got_raw, ref_raw)
    got = eps.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= H.EPS_REL * np.abs(ref) + 1e-30), float((err / np.abs(ref)).max())
    H.report("noise_draws", T=T, E=E, max_rel_err=float((err / np.abs(ref)).max()),
             max_ulp=float((err / (np.abs(ref) * 2.0 ** -23)).max()))


def test_forward_is_deterministic():
    wl = synth.SMALL["switch_small"]
    inp = synth.generate(wl, seed=4)
    layer = B.MoELayer(wl, inp, DEV)
    x = inp["x"].to(DEV)
    y1 = layer.forward(x).clone()
    y2 = layer.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_zero_tokens_is_a_noop():
    wl = synth.SMALL["mixtral_small"].replace(T=0)
    layer = B.MoELayer(wl, synth.generate(wl.replace(T=1), seed=0), DEV)
    x = torch.empty((0, wl.d_model), dtype=torch.bfloat16, device=DEV)
    y = layer.forward(x)
    assert y.shape == (0, wl.d_model)
    assert layer.last_device_error() == (0, 0)


# ============================================================ Expert-Choice routing
EC_ROUTE_CASES = [
    # E, T, cf (C = floor(cf * T / E))
    (8, 300, 2.5), (20, 347, 1.0), (64, 1000, 1.0), (1, 64, 1.0), (3, 5000, 0.5),
    (128, 4096, 1.0), (256, 2048, 3.0), (8, 32768, 2.0),
]


@pytest.mark.parametrize("E,T,cf", EC_ROUTE_CASES)
def test_ec_route_given_logits_bitexact(E, T, cf):
    """Each expert's picks (order included) are bit-exact and the scores match when
    both sides see the same fp32 logits, ties included."""
    wl = synth.SMALL["ec_small"].replace(T=T, n_experts=E, capacity_factor=cf)
    C = O.expert_choice_capacity(cf, T, E)
    z = synth.random_logits(T, E, seed=E * 7 + T, std=1.5, tie_fraction=0.3)
    layer = B.MoELayer(wl, synth.generate(wl.replace(T=1), seed=0, with_weights=False), DEV)
    logits = z.to(DEV)
    idx = torch.empty((E, C), dtype=torch.int32, device=DEV)
    score = torch.empty((E, C), dtype=torch.float32, device=DEV)
    layer.route_expert_choice(None, logits, idx, score)
    torch.cuda.synchronize()
    zn = z.numpy()
    ref_idx = O.expert_choice_select(zn, C)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    ref_s = np.take_along_axis(O.expert_choice_scores(zn), ref_idx.astype(np.int64), axis=1)
    assert np.allclose(score.cpu().numpy(), ref_s, rtol=2e-5, atol=1e-9)
    _devcheck(layer.ws)


def _ec_forward_and_compare(wl: synth.Workload, seed: int, n_sample=None):
    inp = synth.generate(wl, seed=seed)
    layer = B.MoELayer(wl, inp, DEV)
    x = inp["x"].to(DEV)
    taps = layer.new_taps()
    y = layer.forward(x, taps=taps)
    torch.cuda.synchronize()
    code, info = layer.last_device_error()
    assert code == 0, (code, info)
    P = H.oracle_params(inp)
    T, E = wl.T, wl.n_experts
    tokens = tiles = None
    z0 = None
    if n_sample is not None:
        # the first and the last row of every 128-row tile of every expert's C picks
        # (expert e owns rows [e*C, (e+1)*C), row e*C + j holding its j-th pick)
        z0 = O.router_logits(P["x"], P["w_router"], P["b_router"], P["logit_bias"])
        C0 = O.expert_choice_capacity(wl.capacity_factor, T, E)
        picks = O.expert_choice_select(z0, C0)
        tokens, tiles = H.tile_cover_tokens(picks.ravel(), np.arange(E + 1) * C0, T, n_sample)
    yref, r = O.expert_choice_forward(P["x"], P, capacity_factor=wl.capacity_factor,
                                      act=H.ACT[wl.act], logits=z0, tokens=tokens)
    extra = np.zeros(E)
    if P["b_router"] is not None:
        extra += np.abs(P["b_router"])
    if P["logit_bias"] is not None:
        extra += np.abs(P["logit_bias"])
    zg = taps["logits"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(zg - r["logits"]) <= H.logits_bound(P["x"], P["w_router"], extra))
    # the forward's picks from its own logits: tokens within 1e-4 of an expert's
    # C-th logit may be picked differently and are not compared
    C = r["C"]
    near = set()
    zr = np.asarray(r["logits"], dtype=np.float64)
    for e in range(E):
        col = zr[:, e]
        kth = np.sort(col)[::-1][C - 1]
        near |= set(np.nonzero(np.abs(col - kth) < H.MARGIN)[0].tolist()) if C < T else set()
    gidx = torch.empty((E, C), dtype=torch.int32, device=DEV)
    gsc = torch.empty((E, C), dtype=torch.float32, device=DEV)
    layer.route_expert_choice(None, taps["logits"], gidx, gsc)
    torch.cuda.synchronize()
    ref_own = O.expert_choice_select(taps["logits"].cpu().numpy(), C)
    assert np.array_equal(gidx.cpu().numpy(), ref_own)  # bit-exact on the GPU's logits
    sel = np.arange(T) if tokens is None else tokens
    keep = np.array([t not in near for t in sel])
    yg = y.cpu().to(torch.float64).numpy()[sel]
    err = H.max_rel_err(yg[keep], yref[keep])
    taken = np.zeros(T, dtype=bool)
    taken[np.asarray(r["idx"]).ravel()] = True
    cover = {}
    if tiles is not None:
        covered = H.tiles_covered(tiles, np.asarray(r["idx"]).ravel(), sel[keep])
        cover = dict(tiles=len(tiles), tiles_covered=covered)
        assert covered == len(tiles), (covered, len(tiles))
    H.report("forward_expert_choice", workload=wl.name, T=T, C=C, compared=int(keep.sum()),
             **cover,
             near_tie_tokens=len(near), untaken_tokens=int((~taken).sum()),
             worst_rel_err=float(err.max()) if len(err) else 0.0)
    assert err.max() <= H.TOL[wl.dtype], (wl.name, float(err.max()))


@pytest.mark.parametrize("name", EXPERT_CHOICE_SMALL)
def test_ec_forward_small_matches_oracle(name):
    _ec_forward_and_compare(synth.SMALL[name], seed=0)


def test_ec_forward_full_size_sampled():
    _ec_forward_and_compare(synth.WORKLOADS["mixtral_ec"], seed=0, n_sample=48)


def test_ec_forward_is_deterministic():
    wl = synth.SMALL["ec_gelu20"]
    inp = synth.generate(wl, seed=4)
    layer = B.MoELayer(wl, inp, DEV)
    x = inp["x"].to(DEV)
    y1 = layer.forward(x).clone()
    y2 = layer.forward(x).clone()
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_ec_forward_rejects_aux():
    wl = synth.SMALL["ec_small"]
    layer = B.MoELayer(wl, synth.generate(wl, seed=1), DEV)
    x = torch.zeros((wl.T, wl.d_model), dtype=wl.torch_dtype, device=DEV)
    with pytest.raises(B.MoeError):
        layer.forward(x, aux=layer.new_aux())
