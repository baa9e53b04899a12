"""A token-sharded batch through the C ABI against the CPU oracle, on one GPU.

The shards run one after another on the same device (their kernels never wait on
one another); the two collectives of the sharded layer are done by hand between
the phases: the counts are stacked shard-major (the all-gather) and the fp64 sums
added (the sum all-reduce). Put together, the shards must give the single-batch
oracle's results: the same kept pairs (bit-exact), the same permutation inside
each shard, y within the layer tolerance, the statistics of the whole batch.
The oracle routes on the GPU's own fp32 logits, which are checked against the
fp64 logits' accumulation bound first.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_12_b200 import binding as B
from sparse_mixture_experts_12_b200 import build as BUILD
from sparse_mixture_experts_12_b200 import sharded as S
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


CASES = [
    ("mixtral_cap", synth.SMALL["mixtral_cap"], 3),          # bf16 SwiGLU, cf 0.5, GEMV router
    ("switch_small", synth.SMALL["switch_small"], 2),        # bf16 GELU, 32 experts, TC router
    ("deepseek_small", synth.SMALL["deepseek_small"], 2),    # shared experts, top-6 of 64
    ("fp32_gelu_cap", synth.SMALL["fp32_gelu_cap"], 4),      # fp32 path with capacity
    ("empty_shard", synth.SMALL["mixtral_cap"].replace(T=3, capacity_factor=2.0), 4),
]


@pytest.mark.parametrize("name,wl,world", CASES, ids=[c[0] for c in CASES])
def test_sharded_batch_matches_oracle(name, wl, world):
    inp = synth.generate(wl, seed=5)
    P = H.oracle_params(inp)
    T, E, k = wl.T, wl.n_experts, wl.top_k
    x = inp["x"].to(DEV)
    # every shard in this one process: the test gathers the counts itself
    shards = [S.ShardedMoELayer(wl, inp, s, world, DEV, caller_exchanges=True)
              for s in range(world)]
    # phase 1: every shard routes its tokens, counts them and sums its statistics
    logits, taps, counts, parts = [], [], [], []
    for sh in shards:
        a, b = sh.rows
        n = b - a
        z = torch.empty((n, E), dtype=torch.float32, device=DEV)
        tp = {"topk_idx": torch.empty((n, k), dtype=torch.int32, device=DEV),
              "topk_gate": torch.empty((n, k), dtype=torch.float32, device=DEV),
              "counts": torch.empty(E, dtype=torch.int32, device=DEV),
              "offsets": torch.empty(E + 1, dtype=torch.int32, device=DEV),
              "perm": torch.empty(max(n * k, 1), dtype=torch.int32, device=DEV),
              "inv": torch.empty(max(n * k, 1), dtype=torch.int32, device=DEV)}
        c = torch.empty(E, dtype=torch.int32, device=DEV)
        p = torch.empty(1 + 2 * E, dtype=torch.float64, device=DEV)
        sh.layer.route_shard(x[a:b], z, tp["topk_idx"], tp["topk_gate"], c, p)
        logits.append(z)
        taps.append(tp)
        counts.append(c)
        parts.append(p)
    counts_all = torch.stack(counts)          # the all-gather
    part = torch.stack(parts).sum(dim=0)      # the sum all-reduce
    # phase 2: every shard's layer with its share of the capacity
    ys = []
    for sh, tp in zip(shards, taps):
        a, b = sh.rows
        ys.append(sh.forward_shard(x[a:b], tp, counts_all))
    aux = shards[-1].aux_finalize(part)
    torch.cuda.synchronize()
    for sh in shards:
        assert sh.layer.last_device_error() == (0, 0)

    zg = torch.cat(logits).cpu().numpy()
    extra = np.zeros(E)
    for key in ("b_router", "logit_bias"):
        if P[key] is not None:
            extra += np.abs(P[key])
    z64 = O.router_logits(P["x"], P["w_router"], P["b_router"], P["logit_bias"])
    assert np.all(np.abs(zg.astype(np.float64) - z64) <= H.logits_bound(P["x"], P["w_router"], extra))
    yref, r = O.moe_forward(P["x"], P, logits=zg, **H.oracle_kwargs(wl))
    gidx = torch.cat([tp["topk_idx"] for tp in taps]).cpu().numpy()
    assert np.array_equal(gidx, r["idx"])
    cnt = counts_all.cpu().numpy()
    for s, sh in enumerate(shards):
        a, b = sh.rows
        assert np.array_equal(cnt[s], np.bincount(r["idx"][a:b].ravel(), minlength=E))
    # kept pairs: the single batch's, across the shard boundaries
    kept = np.concatenate([(tp["inv"][:(sh.rows[1] - sh.rows[0]) * k].cpu().numpy() >= 0)
                           .reshape(-1, k) for sh, tp in zip(shards, taps)])
    assert np.array_equal(kept, r["kept"])
    # each shard's layout is the oracle's for its tokens and its capacities
    cap = O.capacity(wl.capacity_factor, T, k, E)
    for s, (sh, tp) in enumerate(zip(shards, taps)):
        a, b = sh.rows
        n = b - a
        if n == 0:  # as moe_forward with no tokens, an empty shard writes no taps
            continue
        caps = O.shard_capacity(cnt, s, cap)
        c_s, rank, kp = O.dispatch_with_caps(r["idx"][a:b], E, caps)
        off, perm, inv = O.expert_layout(r["idx"][a:b], rank, kp, E)
        assert np.array_equal(tp["counts"].cpu().numpy(), c_s)
        assert np.array_equal(tp["offsets"].cpu().numpy(), off)
        R = int(off[-1])
        assert np.array_equal(tp["perm"].cpu().numpy()[:R], perm)
        assert np.array_equal(tp["inv"].cpu().numpy()[:n * k].reshape(n, k), inv)
    y = torch.cat(ys).cpu().to(torch.float64).numpy()
    err = H.max_rel_err(y, yref)
    # the whole batch's statistics
    a = aux.cpu().numpy().astype(np.float64)
    f, Pm, auxv = O.aux_stats(zg, r["idx"], E, k, wl.aux_alpha)
    assert np.allclose(a[3:3 + E], f, rtol=1e-6, atol=0)
    assert np.allclose(a[3 + E:], Pm, rtol=2e-5, atol=1e-7)
    assert abs(a[0] - auxv) <= 2e-5 * auxv
    zl = O.router_z_loss(zg)
    assert abs(a[1] - zl) <= 2e-5 * zl
    bsq = O.balance_sq_loss(r["idx"], E)
    assert abs(a[2] - bsq) <= 1e-6 + 1e-5 * bsq
    H.report("sharded", workload=name, T=T, shards=world, worst_rel_err=float(err.max()),
             dropped=int((~r["kept"]).sum()))
    assert err.max() <= H.TOL[wl.dtype], (name, float(err.max()))
    if cap is not None and T > 100:
        assert (~r["kept"]).any()


def test_permute_shard_matches_oracle_bitexact():
    """moe_permute_shard on given routing: the layout of each shard of a batch whose
    capacity bites across the shard boundaries (skewed logits, 64 experts)."""
    T, E, k, world = 1000, 64, 2, 3
    wl = synth.SMALL["mixtral_small"].replace(T=T, n_experts=E, top_k=k, capacity_factor=0.7,
                                              d_model=192)
    z = synth.random_logits(T, E, seed=11, std=2.0) + torch.linspace(3.0, -3.0, E)[None, :]
    idx = O.select_topk(z.numpy(), k)
    x = synth.generate(wl, seed=1, with_weights=False)["x"]
    bounds = S.shard_bounds(T, world)
    counts_all = torch.from_numpy(np.stack(
        [np.bincount(idx[a:b].ravel(), minlength=E) for a, b in bounds]).astype(np.int32)).to(DEV)
    cap = O.capacity(wl.capacity_factor, T, k, E)
    _, _, kept_ref = O.dispatch(idx, E, cap)
    kept = []
    for s, (a, b) in enumerate(bounds):
        n = b - a
        layer = B.MoELayer(wl.replace(T=n), {"w_router": None}, DEV)
        desc = B.MoeShard(n_tokens_total=T, n_shards=world, shard=s,
                          counts_all=counts_all.data_ptr())
        counts = torch.empty(E, dtype=torch.int32, device=DEV)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=DEV)
        perm = torch.full((n * k,), -7, dtype=torch.int32, device=DEV)
        inv = torch.empty(n * k, dtype=torch.int32, device=DEV)
        xp = torch.zeros((n * k, wl.d_model), dtype=x.dtype, device=DEV)
        xs = x[a:b].to(DEV)
        layer.permute_shard(desc, xs, torch.from_numpy(idx[a:b]).to(DEV), counts, offsets,
                            perm, inv, xp)
        torch.cuda.synchronize()
        assert layer.last_device_error() == (0, 0)
        caps = O.shard_capacity(counts_all.cpu().numpy(), s, cap)
        c_s, rank, kp = O.dispatch_with_caps(idx[a:b], E, caps)
        off, rperm, rinv = O.expert_layout(idx[a:b], rank, kp, E)
        R = int(off[-1])
        assert np.array_equal(counts.cpu().numpy(), c_s)
        assert np.array_equal(offsets.cpu().numpy(), off)
        assert np.array_equal(perm.cpu().numpy()[:R], rperm)
        assert np.array_equal(inv.cpu().numpy().reshape(n, k), rinv)
        assert torch.equal(xp.cpu()[:R], x[a:b][torch.from_numpy(rperm)])
        kept.append(kp)
    assert np.array_equal(np.concatenate(kept), kept_ref)
    assert (~kept_ref).any()
