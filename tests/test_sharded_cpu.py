"""Token sharding of one batch over ranks, without a GPU.

The exchange logic of ``sharded.forward_sharded`` (an all-gather of the ranks'
pre-drop counts, a sum all-reduce of their statistics sums) runs here on 2 and 3
gloo ranks, each rank's three steps computed by the oracle. The ranks' outputs put
together must be the single-batch oracle's: the same kept pairs, the same y, the
same statistics. The C entry points' host-side checks are tested without a launch.
"""
import ctypes
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import moe_oracle as O
from sparse_mixture_experts_12_b200 import binding as B
from sparse_mixture_experts_12_b200 import build as BUILD
from sparse_mixture_experts_12_b200 import sharded as S
from sparse_mixture_experts_12_b200 import synth
from tests import gpu_harness as H

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
# fp32 GELU experts, 8 experts, top-2, capacity factor 1.0: drops in several experts
WL = synth.SMALL["fp32_gelu_cap"].replace(T=301)


def test_shard_bounds():
    assert S.shard_bounds(10, 3) == [(0, 4), (4, 7), (7, 10)]
    assert S.shard_bounds(2, 4) == [(0, 1), (1, 2), (2, 2), (2, 2)]
    assert S.shard_bounds(0, 2) == [(0, 0), (0, 0)]
    for T, W in ((301, 2), (301, 3), (7, 7), (1000, 8)):
        b = S.shard_bounds(T, W)
        assert b[0][0] == 0 and b[-1][1] == T
        assert all(x[1] == y[0] for x, y in zip(b, b[1:]))
        assert max(y - x for x, y in b) - min(y - x for x, y in b) <= 1


class OracleSteps:
    """The three per-rank steps of forward_sharded, computed by the oracle in fp64."""

    def __init__(self, wl, P, rank, world):
        self.wl, self.P, self.rank, self.world = wl, P, rank, world
        self.kw = H.oracle_kwargs(wl)
        self.kept = None

    def route_shard(self, x, want_aux):
        E, k = self.wl.n_experts, self.wl.top_k
        z = O.router_logits(x, self.P["w_router"], self.P["b_router"], self.P["logit_bias"])
        z = np.asarray(z, dtype=np.float32)
        idx = O.select_topk(z, k)
        gates = O.gate_values(z, idx, self.kw["gate_mode"])
        counts = torch.from_numpy(np.bincount(idx.ravel(), minlength=E).astype(np.int32))
        part = None
        if want_aux:
            zz = z.astype(np.float64)
            m = zz.max(axis=1)
            lse = m + np.log(np.exp(zz - m[:, None]).sum(axis=1))
            part = torch.from_numpy(np.concatenate(
                [[(lse ** 2).sum()], counts.numpy().astype(np.float64),
                 O.softmax(z).sum(axis=0)]))
        return counts, part, dict(idx=idx, gates=gates)

    def forward_shard(self, x, routed, counts_all, y=None):
        wl, P = self.wl, self.P
        cap = O.capacity(wl.capacity_factor, wl.T, wl.top_k, wl.n_experts)
        caps = O.shard_capacity(counts_all.numpy(), self.rank, cap)
        _, _, kept = O.dispatch_with_caps(routed["idx"], wl.n_experts, caps)
        self.kept = kept
        out = np.zeros_like(x)
        if wl.n_shared:
            out += O.shared_experts(x, P["ws_gate"], P["ws_up"], P["ws_down"], wl.n_shared)
        for t in range(x.shape[0]):
            for s in range(wl.top_k):
                if kept[t, s]:
                    e = int(routed["idx"][t, s])
                    b1 = P["b1"][e] if P.get("b1") is not None else None
                    b2 = P["b2"][e] if P.get("b2") is not None else None
                    w3 = P["w3"][e] if P.get("w3") is not None else None
                    out[t] += routed["gates"][t, s] * O.expert_ffn(
                        x[t:t + 1], self.kw["act"], P["w1"][e], P["w2"][e], w3, b1, b2)[0]
        return out

    def aux_finalize(self, part):
        E, k, T = self.wl.n_experts, self.wl.top_k, self.wl.T
        p = part.numpy()
        f = p[1:1 + E] / (T * k)
        Pm = p[1 + E:] / T
        return dict(f=f, P=Pm, aux=self.wl.aux_alpha * E * float((f * Pm).sum()),
                    z=p[0] / T, bsq=float(((f - 1.0 / E) ** 2).sum()))


def test_one_shard_needs_no_process_group():
    """Without a process group the exchange is the identity: one shard is the batch."""
    P = H.oracle_params(synth.generate(WL, seed=3))
    steps = OracleSteps(WL, P, 0, 1)
    y, aux = S.forward_sharded(steps, P["x"], WL.n_experts, want_aux=True)
    yref, r = O.moe_forward(P["x"], P, **H.oracle_kwargs(WL))
    assert np.array_equal(steps.kept, r["kept"])
    assert np.allclose(y, yref, rtol=1e-12, atol=1e-12)
    _, _, auxv = O.aux_stats(r["logits"], r["idx"], WL.n_experts, WL.top_k, WL.aux_alpha)
    assert aux["aux"] == pytest.approx(auxv, rel=1e-12)


def test_sharded_layer_checks_its_place():
    with pytest.raises(ValueError):
        S.ShardedMoELayer(WL, {}, shard=2, n_shards=2, device="cpu")


def test_several_shards_need_a_process_group():
    """Without a process group, shard 1 of 2 would pass a one-row counts_all while
    the library reads the counts of shard 0 from a second row: rejected up front."""
    assert not dist.is_initialized()
    with pytest.raises(ValueError, match="process group"):
        S.ShardedMoELayer(WL, {}, shard=1, n_shards=2, device="cpu")
    with pytest.raises(ValueError, match="process group"):
        S.ShardedMoELayer(WL, {}, shard=0, n_shards=2, device="cpu")
    S.check_placement(0, 1)  # one shard is the whole batch
    S.check_placement(1, 2, caller_exchanges=True)  # the caller gathers the counts itself
    with pytest.raises(ValueError):
        S.check_placement(2, 2, caller_exchanges=True)


def test_counts_all_is_checked_before_the_descriptor_is_built():
    E = WL.n_experts
    ok = torch.zeros((2, E), dtype=torch.int32)
    S.check_counts_all(ok, 2, E, "cpu")
    with pytest.raises(ValueError, match="shape"):
        S.check_counts_all(torch.zeros((1, E), dtype=torch.int32), 2, E, "cpu")
    with pytest.raises(ValueError, match="shape"):
        S.check_counts_all(torch.zeros((2, E + 1), dtype=torch.int32), 2, E, "cpu")
    with pytest.raises(ValueError, match="int32"):
        S.check_counts_all(torch.zeros((2, E), dtype=torch.int64), 2, E, "cpu")
    with pytest.raises(ValueError, match="is on"):
        S.check_counts_all(ok.to("meta"), 2, E, "cpu")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        P = H.oracle_params(synth.generate(WL, seed=3))
        a, b = S.shard_bounds(WL.T, world)[rank]
        steps = OracleSteps(WL, P, rank, world)
        y, aux = S.forward_sharded(steps, P["x"][a:b], WL.n_experts, want_aux=True)
        q.put((rank, y, steps.kept, aux))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_batch_matches_the_single_batch(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=300) for _ in range(world)), key=lambda g: g[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    P = H.oracle_params(synth.generate(WL, seed=3))
    yref, r = O.moe_forward(P["x"], P, **H.oracle_kwargs(WL))
    assert (~r["kept"]).any()  # the capacity bites, across the shard boundary too
    kept = np.concatenate([g[2] for g in got])
    assert np.array_equal(kept, r["kept"])
    y = np.concatenate([g[1] for g in got])
    assert np.allclose(y, yref, rtol=1e-12, atol=1e-12)
    f, Pm, auxv = O.aux_stats(r["logits"], r["idx"], WL.n_experts, WL.top_k, WL.aux_alpha)
    for _, _, _, aux in got:  # every rank holds the whole batch's statistics
        assert np.allclose(aux["f"], f, rtol=1e-12) and np.allclose(aux["P"], Pm, rtol=1e-12)
        assert aux["aux"] == pytest.approx(auxv, rel=1e-12)
        assert aux["z"] == pytest.approx(O.router_z_loss(r["logits"]), rel=1e-12)
        assert aux["bsq"] == pytest.approx(O.balance_sq_loss(r["idx"], WL.n_experts), rel=1e-9)


def _bench_worker(rank, world, port, q):
    """bench.py's sharded timing path on gloo ranks, the oracle doing the steps."""
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        P = H.oracle_params(synth.generate(WL, seed=3))
        a, b = S.shard_bounds(WL.T, world)[rank]
        steps = OracleSteps(WL, P, rank, world)

        def clock():
            t = {}

            def start():
                bench.barrier(world)
                t[0] = time.perf_counter()

            def stop():
                bench.barrier(world)
                return 1000.0 * (time.perf_counter() - t[0])

            return start, stop

        ms, (y, aux) = bench.sharded_steps_timing(steps, P["x"][a:b], WL.n_experts, 2, 3,
                                                  None, clock)
        worst = bench.max_over_ranks(ms, world)
        q.put((rank, y, steps.kept, aux, ms, worst))
    finally:
        dist.destroy_process_group()


def test_bench_sharded_path_on_two_ranks():
    """The timed loop bench.py runs for one batch split over N GPUs: every rank takes
    the same collectives per step, the ranks' outputs put together are the single
    batch's, and the reported time is the slowest rank's."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_bench_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted((q.get(timeout=300) for _ in range(world)), key=lambda g: g[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    P = H.oracle_params(synth.generate(WL, seed=3))
    yref, r = O.moe_forward(P["x"], P, **H.oracle_kwargs(WL))
    assert np.array_equal(np.concatenate([g[2] for g in got]), r["kept"])
    assert np.allclose(np.concatenate([g[1] for g in got]), yref, rtol=1e-12, atol=1e-12)
    _, _, auxv = O.aux_stats(r["logits"], r["idx"], WL.n_experts, WL.top_k, WL.aux_alpha)
    worst = max(g[4] for g in got)
    for g in got:
        assert g[3]["aux"] == pytest.approx(auxv, rel=1e-12)
        assert g[5] == worst > 0


# ----------------------------------------------------- C entry points, host checks
@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.load()


def test_shard_entry_points_reject_before_launching(lib):
    """Every failure here is decided on the host: no CUDA call is made."""
    wl = synth.SMALL["mixtral_cap"]
    cfg = B.make_cfg(wl)
    ws_bytes = B.workspace_size(cfg)
    ws = ctypes.c_void_p(0x100000)          # fake, 256-aligned: never dereferenced
    good = ctypes.c_void_p(0x200000)
    odd = ctypes.c_void_p(0x200008)
    W = B.MoeWeights(w_router=good, w1=good, w3=good, w2=good)
    taps = B.MoeTaps(topk_idx=good, topk_gate=good)

    def sh(**kw):
        d = dict(n_tokens_total=2 * wl.T, n_shards=2, shard=1, counts_all=good)
        d.update(kw)
        return B.MoeShard(**d)

    def fwd(shard, taps_=taps, cfg_=cfg):
        return lib.moe_forward_shard(ctypes.byref(cfg_), ctypes.byref(shard) if shard else None,
                                     ctypes.byref(W), good, ctypes.byref(taps_) if taps_ else None,
                                     good, ws, ws_bytes, None)
    assert fwd(None) == 1
    assert fwd(sh(shard=2)) == 1                         # shard out of range
    assert fwd(sh(shard=-1)) == 1
    assert fwd(sh(n_shards=0, shard=0)) == 1
    assert fwd(sh(n_tokens_total=wl.T - 1)) == 1         # batch smaller than this shard
    assert fwd(sh(counts_all=None)) == 1
    assert fwd(sh(), taps_=None) == 1                    # the routing is an input
    assert fwd(sh(), taps_=B.MoeTaps(topk_idx=good)) == 1
    ec = B.make_cfg(synth.SMALL["ec_small"])
    assert lib.moe_forward_shard(ctypes.byref(ec), ctypes.byref(sh()), ctypes.byref(W), good,
                                 ctypes.byref(taps), good, ws, B.workspace_size(ec), None) == 1
    assert lib.moe_permute_shard(ctypes.byref(cfg), ctypes.byref(sh(counts_all=odd)), good, good,
                                 good, good, good, good, good, ws, ws_bytes, None) == 3
    assert lib.moe_permute_shard(ctypes.byref(cfg), ctypes.byref(sh()), good, good, good, good,
                                 good, odd, good, ws, ws_bytes, None) == 3
    assert lib.moe_route_shard(ctypes.byref(cfg), ctypes.byref(W), good, None, good, good, None,
                               None, ws, ws_bytes, None) == 1      # counts missing
    assert lib.moe_route_shard(ctypes.byref(cfg), ctypes.byref(W), good, None, good, good, good,
                               odd, ws, ws_bytes, None) == 3       # aux_part misaligned
    assert lib.moe_aux_finalize(ctypes.byref(cfg), 0, good, good, None) == 1
    assert lib.moe_aux_finalize(ctypes.byref(cfg), 10, None, good, None) == 1
