"""Checks that pin the CPU oracle to what the pages and the mathematics fix.

Each ``check_*`` raises AssertionError on a mismatch. They take the oracle module
as an argument so that the mutant tests can hand in a deliberately broken copy
and confirm that at least one check catches every planted mistake.
"""
from __future__ import annotations

import itertools
import json
import math
import os

import numpy as np
import torch

from sparse_mixture_experts_12_b200 import synth
from tests import pages_torch_ref as ref

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
ACT = {synth.ACT_RELU: "relu", synth.ACT_GELU: "gelu", synth.ACT_SWIGLU: "swiglu"}
MODE = {synth.GATE_TOPK_SOFTMAX: "topk_softmax",
        synth.GATE_SOFTMAX_TOPK_RENORM: "softmax_topk_renorm",
        synth.GATE_SOFTMAX_TOPK_RAW: "softmax_topk_raw"}


def params_f64(inp: dict) -> dict:
    return {k: synth.to_f64_numpy(v) for k, v in inp.items()}


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ------------------------------------------------------------------------ top-k
def _brute_topk(zrow, k):
    """All k-permutations; keep the one that is ordered by (value desc, index asc)
    and that no unselected expert beats under the same order."""
    E = len(zrow)
    key = lambda e: (-float(zrow[e]), e)  # noqa: E731
    found = []
    for perm in itertools.permutations(range(E), k):
        ordered = all(key(perm[j]) < key(perm[j + 1]) for j in range(k - 1))
        rest = [e for e in range(E) if e not in perm]
        dominated = all(key(perm[-1]) < key(e) for e in rest)
        if ordered and dominated:
            found.append(list(perm))
    assert len(found) == 1
    return found[0]


def check_topk_bruteforce(O):
    rng = np.random.default_rng(1)
    for E in (1, 2, 3, 5, 6):
        for k in range(1, E + 1):
            z = rng.normal(size=(12, E)).astype(np.float32)
            # constructed ties: a coarse grid makes many equal values
            zt = (np.round(rng.normal(size=(12, E)) * 2) / 2).astype(np.float32)
            for zz in (z, zt):
                got = O.select_topk(zz, k)
                for t in range(zz.shape[0]):
                    assert list(got[t]) == _brute_topk(zz[t], k), (E, k, zz[t], got[t])


# ------------------------------------------------------------------------ gates
def check_gate_sums_and_ranges(O):
    rng = np.random.default_rng(2)
    for E, k in ((8, 2), (64, 6), (5, 5), (3, 1)):
        z = (rng.normal(size=(40, E)) * 3).astype(np.float32)
        idx = O.select_topk(z, k)
        for mode in ("topk_softmax", "softmax_topk_renorm"):
            g = O.gate_values(z, idx, mode)
            assert np.all(np.abs(g.sum(axis=1) - 1.0) <= 4 * k * 2.0 ** -52)
            assert np.all(g >= 0) and np.all(np.diff(g, axis=1) <= 1e-15)
        graw = O.gate_values(z, idx, "softmax_topk_raw")
        p = O.softmax(z)
        assert np.all(graw[:, 0] >= 1.0 / E - 1e-15) and np.all(graw[:, 0] <= 1.0)
        # the raw Switch gate of slot 0 is the largest probability
        assert np.allclose(graw[:, 0], p.max(axis=1), rtol=0, atol=1e-15)
        # modes A and B select the same set and give the same gates up to rounding
        ga = O.gate_values(z, idx, "topk_softmax")
        gb = O.gate_values(z, idx, "softmax_topk_renorm")
        assert np.allclose(ga, gb, rtol=1e-12, atol=1e-15)


def check_worked_gates(O):
    for c in _golden("worked_gates.json")["cases"]:
        z = np.array([c["logits"]], dtype=np.float32)
        idx = O.select_topk(z, c["k"])
        assert list(idx[0]) == c["expect_idx"], c["cite"]
        for mode in ("topk_softmax", "softmax_topk_renorm"):
            g = O.gate_values(z, idx, mode)[0]
            assert np.allclose(g, c["expect_gates"], rtol=0, atol=2e-7), (c["cite"], mode, g)


def check_softmax_closed_forms(O):
    z = np.zeros((3, 7), dtype=np.float32)
    assert np.allclose(O.softmax(z), 1.0 / 7, rtol=0, atol=1e-16)
    z = np.array([[0.0, math.log(3.0)]], dtype=np.float64)
    assert np.allclose(O.softmax(z), [[0.25, 0.75]], rtol=0, atol=1e-15)
    # invariance to a per-row shift, and to huge logits (no overflow)
    z = np.array([[1000.0, 999.0, 998.0]])
    e = np.exp([0.0, -1.0, -2.0])
    assert np.allclose(O.softmax(z), e / e.sum(), rtol=1e-14)


# --------------------------------------------------------------------- logits
def check_router_logits_exact(O):
    rng = np.random.default_rng(3)
    # small integers: every product and sum is exact in fp32 and fp64
    x = rng.integers(-4, 5, size=(9, 16)).astype(np.float64)
    w = rng.integers(-3, 4, size=(5, 16)).astype(np.float64)
    b = rng.integers(-2, 3, size=(5,)).astype(np.float64)
    lb = rng.integers(-2, 3, size=(5,)).astype(np.float64)
    z = O.router_logits(x, w, b, lb)
    want = np.zeros((9, 5))
    for t in range(9):
        for e in range(5):
            want[t, e] = sum(x[t, j] * w[e, j] for j in range(16)) + b[e] + lb[e]
    assert z.dtype == np.float32 and np.array_equal(z.astype(np.float64), want)
    # non-integer inputs: the result is the fp32 rounding of the exact dot product
    x = rng.normal(size=(4, 33))
    w = rng.normal(size=(3, 33))
    z = O.router_logits(x, w)
    exact = np.array([[math.fsum(x[t] * w[e]) for e in range(3)] for t in range(4)])
    assert np.array_equal(z, exact.astype(np.float32))


# ------------------------------------------------------------ capacity / drops
def check_capacity_golden(O):
    for c in _golden("capacity.json")["cases"]:
        assert O.capacity(c["cf"], c["T"], c["k"], c["E"]) == c["expect"], c["cite"]


def check_counts_and_drop_order(O):
    rng = np.random.default_rng(4)
    for T, E, k, cap in ((50, 4, 1, 9), (64, 8, 2, 10), (33, 3, 3, 5), (20, 5, 2, None)):
        z = rng.normal(size=(T, E)).astype(np.float32)
        idx = O.select_topk(z, k)
        counts, rank, kept = O.dispatch(idx, E, cap)
        assert counts.sum() == T * k
        for e in range(E):
            # the pairs routed to e, listed token-major then slot
            pairs = [(t, s) for t in range(T) for s in range(k) if idx[t, s] == e]
            assert counts[e] == len(pairs)
            for r, (t, s) in enumerate(pairs):
                assert rank[t, s] == r
                assert kept[t, s] == (cap is None or r < cap)
            n_kept = sum(kept[t, s] for (t, s) in pairs)
            assert n_kept == (len(pairs) if cap is None else min(len(pairs), cap))
        n_drop = int((~kept).sum())
        assert int(kept.sum()) == T * k - n_drop
    # every token on one expert: exactly the first ``cap`` tokens survive
    idx = np.zeros((30, 1), dtype=np.int32)
    _, _, kept = O.dispatch(idx, 4, 7)
    assert list(np.nonzero(kept[:, 0])[0]) == list(range(7))


def check_layout(O):
    rng = np.random.default_rng(5)
    T, E, k, cap = 40, 6, 2, 11
    idx = O.select_topk(rng.normal(size=(T, E)).astype(np.float32), k)
    counts, rank, kept = O.dispatch(idx, E, cap)
    offsets, perm, inv = O.expert_layout(idx, rank, kept, E)
    assert offsets[0] == 0 and offsets[-1] == kept.sum()
    for e in range(E):
        rows = range(offsets[e], offsets[e + 1])
        toks = [perm[r] for r in rows]
        assert toks == sorted(toks)  # token order inside an expert
        for r in rows:
            t = perm[r]
            s = [s for s in range(k) if idx[t, s] == e][0]
            assert inv[t, s] == r
    assert np.all((inv >= 0) == kept)


# ------------------------------------------------------------------ forward
def _small_inputs(wl, seed=0):
    inp = synth.generate(wl, seed=seed)
    return inp, params_f64(inp)


def check_forward_vs_pages_torch(O):
    """The numpy oracle and the torch restatement of the pages' listings agree."""
    cases = [synth.SMALL["tiny"].replace(T=48),
             synth.SMALL["mixtral_small"].replace(T=40, d_model=32, d_ff=48),
             synth.SMALL["deepseek_small"].replace(T=30, d_model=32, d_ff=24, d_ff_shared=40),
             synth.SMALL["switch_small"].replace(T=90, d_model=24, d_ff=40, n_experts=6),
             synth.SMALL["fp32_gelu_cap"].replace(T=35, capacity_factor=0.0)]
    for wl in cases:
        inp, p = _small_inputs(wl, seed=7)
        act, mode = ACT[wl.act], MODE[wl.gate_mode]
        cap = O.capacity(wl.capacity_factor, wl.T, wl.top_k, wl.n_experts)
        y, r = O.moe_forward(p["x"], p, top_k=wl.top_k, act=act, gate_mode=mode,
                             capacity_factor=wl.capacity_factor, n_shared=wl.n_shared)
        yt, zt, it, wt, pt = ref.moe_layer(p["x"], p, k=wl.top_k, act=act, mode=mode,
                                           cap=cap, n_shared=wl.n_shared)
        # the torch restatement keeps fp64 logits; both must pick the same experts
        assert np.min(O.topk_margin(r["logits"], wl.top_k)) > 1e-5, wl.name
        assert np.array_equal(r["idx"], it.numpy()), wl.name
        assert np.allclose(r["logits"], zt.numpy(), rtol=1e-6, atol=1e-6), wl.name
        assert np.allclose(r["gates"], wt.numpy(), rtol=1e-6, atol=1e-7), wl.name
        scale = np.abs(yt.numpy()).max()
        assert np.abs(y - yt.numpy()).max() <= 1e-6 * scale, wl.name
        f, P, aux = O.aux_stats(r["logits"], r["idx"], wl.n_experts, wl.top_k, wl.aux_alpha)
        ft, Pt, auxt = ref.load_balancing_loss(pt, it, wl.n_experts, wl.top_k, wl.aux_alpha)
        assert np.allclose(f, ft.numpy(), rtol=0, atol=1e-15)
        assert np.allclose(P, Pt.numpy(), rtol=1e-6, atol=1e-9)
        assert abs(aux - float(auxt)) <= 1e-6 * abs(float(auxt)) + 1e-12


def _dense_expert(p, e, act, x):
    """One expert through torch.nn.functional in fp64 (a library restatement)."""
    X = torch.as_tensor(x)
    w1 = torch.as_tensor(p["w1"][e]); w2 = torch.as_tensor(p["w2"][e])
    if act == "swiglu":
        h = F.silu(F.linear(X, w1)) * F.linear(X, torch.as_tensor(p["w3"][e]))
        return F.linear(h, w2).numpy()
    b1 = None if p.get("b1") is None else torch.as_tensor(p["b1"][e])
    b2 = None if p.get("b2") is None else torch.as_tensor(p["b2"][e])
    v = F.linear(X, w1, b1)
    h = F.relu(v) if act == "relu" else F.gelu(v)
    return F.linear(h, w2, b2).numpy()


import torch.nn.functional as F  # noqa: E402


def check_sparse_equals_dense_masked(O):
    """Computing every expert for every token and weighting by the full gate
    matrix G (zero outside the kept top-k) gives the sparse result."""
    for wl in (synth.SMALL["fp32_gelu_cap"].replace(T=60, capacity_factor=0.6),
               synth.SMALL["deepseek_small"].replace(T=25, d_model=16, d_ff=24, d_ff_shared=8,
                                                     n_experts=9, top_k=3),
               synth.SMALL["tiny"].replace(T=20)):
        inp, p = _small_inputs(wl, seed=11)
        act, mode = ACT[wl.act], MODE[wl.gate_mode]
        y, r = O.moe_forward(p["x"], p, top_k=wl.top_k, act=act, gate_mode=mode,
                             capacity_factor=wl.capacity_factor, n_shared=wl.n_shared)
        T, E = r["logits"].shape
        G = np.zeros((T, E))
        for t in range(T):
            for s in range(wl.top_k):
                if r["kept"][t, s]:
                    G[t, r["idx"][t, s]] += r["gates"][t, s]
        dense = np.zeros_like(y)
        for e in range(E):
            dense += G[:, e:e + 1] * _dense_expert(p, e, act, p["x"])
        if wl.n_shared:
            Fs = wl.d_ff_shared
            for j in range(wl.n_shared):
                sl = slice(j * Fs, (j + 1) * Fs)
                X = torch.as_tensor(p["x"])
                h = F.silu(F.linear(X, torch.as_tensor(p["ws_gate"][sl]))) * \
                    F.linear(X, torch.as_tensor(p["ws_up"][sl]))
                dense += F.linear(h, torch.as_tensor(p["ws_down"][:, sl])).numpy()
        assert np.abs(y - dense).max() <= 1e-12 * max(1.0, np.abs(dense).max()), wl.name
        if wl.capacity_factor > 0:
            assert (~r["kept"]).any(), "the capped case must drop something"


def check_special_cases(O):
    # E = 1, k = 1, mode A: the layer is the plain expert FFN (gate 1)
    for act_id in (synth.ACT_RELU, synth.ACT_GELU, synth.ACT_SWIGLU):
        wl = synth.SMALL["tiny"].replace(T=10, d_model=8, d_ff=12, n_experts=1, top_k=1,
                                         act=act_id, expert_bias=act_id != synth.ACT_SWIGLU)
        inp, p = _small_inputs(wl, seed=3)
        act = ACT[act_id]
        y, r = O.moe_forward(p["x"], p, top_k=1, act=act, gate_mode="topk_softmax")
        assert np.all(r["gates"] == 1.0)
        assert np.allclose(y, _dense_expert(p, 0, act, p["x"]), rtol=1e-13, atol=1e-13)
    # k = E, mode B: a dense soft mixture under the full softmax
    wl = synth.SMALL["fp32_swiglu"].replace(T=12, d_model=8, d_ff=6, n_experts=4, top_k=4,
                                            n_shared=0)
    inp, p = _small_inputs(wl, seed=4)
    y, r = O.moe_forward(p["x"], p, top_k=4, act="swiglu", gate_mode="softmax_topk_renorm")
    probs = torch.softmax(torch.as_tensor(r["logits"], dtype=torch.float64), dim=-1).numpy()
    dense = sum(probs[:, e:e + 1] * _dense_expert(p, e, "swiglu", p["x"]) for e in range(4))
    assert np.allclose(y, dense, rtol=1e-12, atol=1e-13)
    # SwiGLU with W_gate = 0: silu(0) = 0, so every routed output is 0
    p0 = dict(p)
    p0["w1"] = np.zeros_like(p["w1"])
    y0, _ = O.moe_forward(p["x"], p0, top_k=2, act="swiglu", gate_mode="topk_softmax")
    assert np.all(y0 == 0.0)
    # two shared experts equal one expert with their weights concatenated along d_ff
    wl = synth.SMALL["deepseek_small"].replace(T=9, d_model=16, d_ff=8, d_ff_shared=12)
    inp, p = _small_inputs(wl, seed=5)
    two = O.shared_experts(p["x"], p["ws_gate"], p["ws_up"], p["ws_down"], 2)
    one = O.shared_experts(p["x"], p["ws_gate"], p["ws_up"], p["ws_down"], 1)
    assert np.allclose(two, one, rtol=1e-12, atol=1e-13)
    # the GELU and SiLU element functions against library routines
    v = np.linspace(-6, 6, 101)
    assert np.allclose(O.gelu(v), F.gelu(torch.as_tensor(v)).numpy(), rtol=1e-14, atol=1e-15)
    assert np.allclose(O.silu(v), F.silu(torch.as_tensor(v)).numpy(), rtol=1e-14, atol=1e-15)


# -------------------------------------------------------------------- aux stats
def check_aux_closed_forms(O):
    c = _golden("aux_small.json")
    z = np.array(c["logits"], dtype=np.float32)
    idx = O.select_topk(z, c["k"])
    assert idx.tolist() == c["expect_idx"]
    f, P, aux = O.aux_stats(z, idx, c["E"], c["k"], c["alpha"])
    assert np.allclose(f, c["expect_f"], atol=1e-15)
    assert np.allclose(P, c["expect_P"], atol=1e-7)
    assert abs(aux - c["expect_aux"]) < 1e-8
    a = 0.01
    # uniform logits: P_i = 1/E, and with a balanced assignment f_i = 1/E -> aux = alpha
    for E, k in ((8, 1), (8, 2), (4, 4)):
        T = 4 * E
        z = np.zeros((T, E), dtype=np.float32)
        idx = np.array([[(t + s) % E for s in range(k)] for t in range(T)], dtype=np.int32)
        f, P, aux = O.aux_stats(z, idx, E, k, a)
        assert np.allclose(P, 1.0 / E, atol=1e-16) and np.allclose(f, 1.0 / E, atol=1e-16)
        assert abs(aux - a) < 1e-15
    # every token on expert 0 with a one-hot probability: aux -> alpha * E
    E = 16
    z = np.full((10, E), -200.0, dtype=np.float32)
    z[:, 0] = 0.0
    idx = O.select_topk(z, 1)
    f, P, aux = O.aux_stats(z, idx, E, 1, a)
    assert abs(aux - a * E) < 1e-12
    # extra outputs: z-loss of zero logits is (log E)^2; squared balance loss
    z = np.zeros((5, 8), dtype=np.float32)
    assert abs(O.router_z_loss(z) - math.log(8) ** 2) < 1e-12
    idx = np.zeros((6, 1), dtype=np.int32)
    assert abs(O.balance_sq_loss(idx, 4) - ((1 - 0.25) ** 2 + 3 * 0.25 ** 2)) < 1e-15
    idx = np.array([[0], [1], [2], [3]], dtype=np.int32)
    assert O.balance_sq_loss(idx, 4) == 0.0


def check_combine(O):
    """Layout -> per-row expert -> combine reproduces the masked loop; closed forms."""
    wl = synth.SMALL["fp32_gelu_cap"].replace(T=40, capacity_factor=0.7)
    inp, p = _small_inputs(wl, seed=13)
    act, mode = ACT[wl.act], MODE[wl.gate_mode]
    y, r = O.moe_forward(p["x"], p, top_k=wl.top_k, act=act, gate_mode=mode,
                         capacity_factor=wl.capacity_factor)
    rows = np.zeros((len(r["perm"]), wl.d_model))
    for e in range(wl.n_experts):
        a, b = r["offsets"][e], r["offsets"][e + 1]
        if b > a:
            rows[a:b] = _dense_expert(p, e, act, p["x"][r["perm"][a:b]])
    assert np.allclose(O.combine(rows, r["inv"], r["gates"]), y, rtol=1e-12, atol=1e-13)
    # one-hot gates pick the rows; all slots dropped gives the shared part only
    rng = np.random.default_rng(14)
    yr = rng.normal(size=(6, 5))
    inv = np.array([[0, 3], [5, -1], [-1, -1]])
    g = np.array([[1.0, 0.0], [0.0, 0.5], [0.3, 0.7]])
    sh = rng.normal(size=(3, 5))
    out = O.combine(yr, inv, g, sh)
    assert np.allclose(out[0], yr[0] + sh[0], rtol=0, atol=1e-15)
    assert np.allclose(out[1], sh[1], rtol=0, atol=1e-15)
    assert np.allclose(out[2], sh[2], rtol=0, atol=1e-15)


# ------------------------------------------------------------ Expert-Choice routing
def check_expert_choice_capacity(O):
    """int(cf * N / E) (P3 ``ExpertChoiceRouter``, P4 ``ExpertChoiceGating``), by hand."""
    for cf, T, E, want in ((1.0, 16384, 128, 128), (1.0, 10, 3, 3), (2.0, 4096, 8, 1024),
                           (1.25, 7, 2, 4), (0.5, 9, 4, 1), (3.0, 5, 3, 5)):
        assert O.expert_choice_capacity(cf, T, E) == want, (cf, T, E)


def check_expert_choice_bruteforce(O):
    """Each expert's C tokens, by enumeration over all ordered C-subsets of the
    tokens (value descending, equal values to the lower token first)."""
    rng = np.random.default_rng(5)
    for T, E in ((5, 2), (6, 3), (7, 1)):
        for C in range(1, T + 1):
            z = rng.normal(size=(T, E)).astype(np.float32)
            zt = (np.round(rng.normal(size=(T, E)) * 2) / 2).astype(np.float32)
            for zz in (z, zt):
                got = O.expert_choice_select(zz, C)
                assert got.shape == (E, C)
                for e in range(E):
                    assert list(got[e]) == _brute_topk(zz[:, e], C), (T, E, C, zz[:, e])


def check_expert_choice_scores(O):
    """Per expert, a softmax over the tokens: each expert's scores sum to 1 over
    the tokens, and score ratios are exp of logit differences along a column."""
    rng = np.random.default_rng(6)
    z = (rng.normal(size=(9, 4)) * 3).astype(np.float32)
    S = O.expert_choice_scores(z)
    assert S.shape == (4, 9)
    assert np.allclose(S.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    for e in range(4):
        for t in range(1, 9):
            assert abs(S[e, t] / S[e, 0] - math.exp(float(z[t, e]) - float(z[0, e]))) <= \
                1e-12 * math.exp(float(z[t, e]) - float(z[0, e]))
    # a column that is constant gives the uniform distribution over the tokens
    S1 = O.expert_choice_scores(np.zeros((5, 2), dtype=np.float32))
    assert np.allclose(S1, 0.2, rtol=0, atol=1e-15)


def check_expert_choice_dense(O):
    """The pages' form: dispatch mask [E, N] = scores scattered at each expert's
    top-C tokens (torch.topk on torch.softmax over the token dim, P4
    ``ExpertChoiceGating``), every expert computed on every token, masked and
    summed, equals the oracle's sparse loop; with C = N it is the dense soft mix."""
    for wl, cf in ((synth.SMALL["tiny"].replace(T=24), 1.0),
                   (synth.SMALL["mixtral_small"].replace(T=20, d_model=16, d_ff=24, n_experts=4),
                    1.5),
                   (synth.SMALL["switch_small"].replace(T=12, d_model=8, d_ff=16, n_experts=3),
                    3.0)):
        inp, p = _small_inputs(wl, seed=13)
        act = ACT[wl.act]
        y, r = O.expert_choice_forward(p["x"], p, capacity_factor=cf, act=act)
        T, E = r["logits"].shape
        assert np.min(O.expert_choice_margin(r["logits"], r["C"])) > 1e-6, wl.name
        zt = torch.as_tensor(np.asarray(r["logits"], dtype=np.float64))
        scores = torch.softmax(zt.T, dim=-1)
        top_s, top_i = torch.topk(scores, r["C"], dim=-1)
        dispatch = torch.zeros(E, T, dtype=torch.float64)
        dispatch.scatter_(1, top_i, top_s)
        assert np.array_equal(np.asarray(r["idx"]), top_i.numpy()), wl.name
        dense = np.zeros_like(y)
        for e in range(E):
            dense += dispatch[e].numpy()[:, None] * _dense_expert(p, e, act, p["x"])
        assert np.abs(y - dense).max() <= 1e-12 * max(1.0, np.abs(dense).max()), wl.name
        if r["C"] == T:
            assert (dispatch > 0).all(), "C = N: every expert takes every token"
        else:
            assert (dispatch.sum(dim=0) == 0).any() or r["C"] * E >= T


# -------------------------------------------------------------- noisy top-k gating
def check_noisy_logits(O):
    """P4 ``TopKGating`` training logits: zero noise gives the plain router; a zero
    noise projection adds ln(2) * eps; the noise term is linear in eps; softplus
    against torch's, including its switch to the identity above 20."""
    rng = np.random.default_rng(8)
    T, d, E = 7, 6, 5
    x = rng.integers(-3, 4, size=(T, d)).astype(np.float64)
    wr = rng.integers(-2, 3, size=(E, d)).astype(np.float64) / 4
    wn = rng.integers(-2, 3, size=(E, d)).astype(np.float64) / 8
    eps = rng.normal(size=(T, E))
    plain = O.router_logits(x, wr)
    assert np.array_equal(O.noisy_router_logits(x, wr, wn, np.zeros((T, E))), plain)
    z0 = O.noisy_router_logits(x, wr, np.zeros((E, d)), eps)
    assert np.allclose(z0, (x @ wr.T + math.log(2.0) * eps).astype(np.float32), rtol=0,
                       atol=1e-6)
    z1 = O.noisy_router_logits(x, wr, wn, eps).astype(np.float64) - plain
    z2 = O.noisy_router_logits(x, wr, wn, 2 * eps).astype(np.float64) - plain
    assert np.allclose(z2, 2 * z1, rtol=1e-6, atol=1e-5)
    v = np.array([-30.0, -3.0, -0.5, 0.0, 0.5, 3.0, 19.9, 20.0, 20.5, 40.0])
    ref = F.softplus(torch.as_tensor(v)).numpy()
    assert np.allclose(O.softplus(v), ref, rtol=1e-15, atol=1e-300)
    assert O.softplus(np.array([0.0]))[0] == math.log(2.0)


# ---------------------------------------------------------- token-sharded capacity
def check_sharded_capacity(O):
    """Splitting the tokens into consecutive shards, each dropping against the capacity
    the earlier shards left, keeps exactly the (token, slot) pairs the single call
    keeps (enumerated over shard splits of random routings with drops)."""
    rng = np.random.default_rng(12)
    for T, E, k, cf in ((30, 4, 2, 0.7), (25, 3, 1, 0.5), (40, 6, 3, 1.0)):
        z = rng.normal(size=(T, E)).astype(np.float32)
        idx = O.select_topk(z, k)
        cap = O.capacity(cf, T, k, E)
        _, _, kept = O.dispatch(idx, E, cap)
        assert (~kept).any()
        for cuts in ((T // 2,), (7, 19), (1, 2, T - 1)):
            bounds = [0, *cuts, T]
            shards = [idx[a:b] for a, b in zip(bounds, bounds[1:])]
            counts_all = np.stack([np.bincount(sh.ravel(), minlength=E) for sh in shards])
            got = []
            for r, sh in enumerate(shards):
                caps = O.shard_capacity(counts_all, r, cap)
                got.append(O.dispatch_with_caps(sh, E, caps)[2])
            assert np.array_equal(np.concatenate(got), kept), (T, E, k, cuts)
    assert O.shard_capacity(np.ones((2, 3)), 1, None) is None


# ------------------------------------------------- counter-based noise (Philox, Box-Muller)
def check_philox_kat(O):
    """Philox4x32-10 reproduces the generator's published known-answer vectors."""
    kat = _golden("philox_kat.json")
    for case in kat["cases"]:
        ctr = np.array([int(v, 16) for v in case["counter"]], dtype=np.uint64)
        key = np.array([int(v, 16) for v in case["key"]], dtype=np.uint64)
        out = O.philox4x32(ctr, key, rounds=kat["rounds"])
        assert [int(v) for v in out] == [int(v, 16) for v in case["out"]], case


def check_noise_draws(O):
    """The seeded noise: uniforms strictly inside (0, 1) and exact in fp32; the draws
    a function of (seed, offset) alone; standard normal (Kolmogorov-Smirnov, mean,
    variance) with the two members of a Box-Muller pair uncorrelated, also in their
    squares (which a shared uniform would correlate)."""
    from scipy import stats

    u = O.uniform_open(np.array([0, 1, 511, 512, 2 ** 31, 2 ** 32 - 1], dtype=np.uint64))
    assert u.min() > 0 and u.max() < 1
    assert np.array_equal(u.astype(np.float32).astype(np.float64), u)
    assert u[0] == 2.0 ** -24 and u[-1] == 1.0 - 2.0 ** -24 and u[2] == u[0] and u[3] > u[2]
    T, E = 4096, 64
    eps, raw = O.noise_draws(T, E, seed=1234, offset=5)
    assert eps.shape == (T, E) and raw.shape == (T, E // 4, 4)
    again, _ = O.noise_draws(T, E, seed=1234, offset=5)
    assert np.array_equal(eps, again)
    assert not np.array_equal(O.noise_draws(8, E, seed=1234, offset=6)[0], eps[:8])
    assert not np.array_equal(O.noise_draws(8, E, seed=1235, offset=5)[0], eps[:8])
    # a ragged expert count takes the first E columns of the same draws
    assert np.array_equal(O.noise_draws(16, 6, seed=1234, offset=5)[0], eps[:16, :6])
    n = eps.size
    v = eps.ravel()
    assert abs(v.mean()) < 5.0 / math.sqrt(n)
    assert abs(v.var() - 1.0) < 5.0 * math.sqrt(2.0 / n)
    assert stats.kstest(v, "norm").pvalue > 1e-4
    a, b = eps[:, 0::2].ravel(), eps[:, 1::2].ravel()  # the two members of each pair
    assert abs(np.corrcoef(a, b)[0, 1]) < 5.0 / math.sqrt(a.size)
    assert abs(np.corrcoef(a * a, b * b)[0, 1]) < 5.0 / math.sqrt(a.size)
    # nothing repeats across tokens, expert groups or offsets
    words = np.concatenate([raw.ravel(), O.noise_draws(64, E, 1234, 6)[1].ravel()])
    assert len(np.unique(words)) > 0.999 * len(words)


ALL_CHECKS = [check_combine, check_topk_bruteforce, check_gate_sums_and_ranges, check_worked_gates,
              check_softmax_closed_forms, check_router_logits_exact, check_capacity_golden,
              check_counts_and_drop_order, check_layout, check_forward_vs_pages_torch,
              check_sparse_equals_dense_masked, check_special_cases, check_aux_closed_forms,
              check_expert_choice_capacity, check_expert_choice_bruteforce,
              check_expert_choice_scores, check_expert_choice_dense, check_noisy_logits,
              check_sharded_capacity, check_philox_kat, check_noise_draws]
