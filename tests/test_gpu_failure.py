"""Failure detection on the GPU without a fault: a bounded pipeline wait runs out.

Every pipeline wait in the tensor-core kernels has a time limit; when one runs out
the kernel records MOE_DEVERR_WAIT_TIMEOUT in the workspace's error word, lets the
copies and MMAs it issued finish, frees its tensor memory and returns. Here the
single-CTA expert GEMM is made to withhold one operand load per CTA (a test hook),
with a short limit, so its MMA issuer waits for data that never comes: the call
must return the timeout through the error word, quickly, and the same workspace
must then give the oracle's result on a normal call.
"""
import ctypes
import time

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
LIMIT_NS = 20_000_000  # 20 ms


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.fail("the GPU tests need a CUDA device")
    BUILD.build()
    lib = B.load()
    yield lib
    lib.moe_test_withhold_load(0)
    lib.moe_test_set_wait_limit(0)


def _layer_and_rows(act, d, F, rows, seed):
    """A layer whose expert FFN takes the single-CTA GEMM (reductions under 2048,
    experts averaging under 256 rows) and its permuted rows."""
    R = int(sum(rows))
    k = 2
    T = (R + k - 1) // k + 3
    wl = synth.Workload("timeout_case", T=T, d_model=d, n_experts=len(rows), top_k=k, d_ff=F,
                        act=act, gate_mode=0, dtype=synth.DT_BF16,
                        expert_bias=act != synth.ACT_SWIGLU, bias_std=0.3)
    inp = synth.generate(wl, seed=seed)
    layer = B.MoELayer(wl, inp, DEV)
    g = torch.Generator().manual_seed(seed + 1)
    xp = torch.randn((T * k, d), generator=g).to(torch.bfloat16)
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(rows)]), dtype=torch.int32)
    return wl, inp, layer, xp, offsets


@pytest.mark.parametrize("act,d,F,rows", [
    (synth.ACT_GELU, 128, 320, [5, 260, 0, 128]),
    (synth.ACT_SWIGLU, 256, 384, [0, 1, 129, 300, 64]),
], ids=["gelu", "swiglu"])
def test_pipeline_wait_runs_out_and_the_context_recovers(_lib, act, d, F, rows):
    lib = _lib
    wl, inp, layer, xp, offsets = _layer_and_rows(act, d, F, rows, seed=sum(rows))
    xpd, offd = xp.to(DEV), offsets.to(DEV)
    y = torch.zeros((xp.shape[0], d), dtype=torch.bfloat16, device=DEV)
    torch.cuda.synchronize()
    assert layer.last_device_error() == (0, 0)

    # 1. a load that never comes: the bounded wait runs out, the call comes back
    assert lib.moe_test_set_wait_limit(LIMIT_NS) == 0
    assert lib.moe_test_withhold_load(1) == 0
    t0 = time.perf_counter()
    layer.expert_ffn(xpd, offd, y)
    code, info = layer.last_device_error()  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert code == 4, (code, info)          # MOE_DEVERR_WAIT_TIMEOUT
    assert info in (1, 2, 3, 4), info        # the site of the wait that ran out
    assert elapsed < 5.0, elapsed            # bounded: no 2 s default waits, no hang
    assert layer.last_device_error() == (0, 0)  # the word was cleared by the read

    # 2. the same workspace, the default limit, no hook: the oracle's result
    assert lib.moe_test_set_wait_limit(0) == 0
    y2 = torch.full((xp.shape[0], d), float("nan"), dtype=torch.bfloat16, device=DEV)
    layer.expert_ffn(xpd, offd, y2)
    torch.cuda.synchronize()
    assert layer.last_device_error() == (0, 0)
    yc = y2.cpu().to(torch.float64).numpy()
    P = H.oracle_params(inp)
    worst = 0.0
    for e in range(len(rows)):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b == a:
            continue
        ref = O.expert_ffn(synth.to_f64_numpy(xp[a:b]), H.ACT[act], P["w1"][e], P["w2"][e],
                           None if P["w3"] is None else P["w3"][e],
                           None if P["b1"] is None else P["b1"][e],
                           None if P["b2"] is None else P["b2"][e])
        worst = max(worst, float(H.max_rel_err(yc[a:b], ref).max()))
    H.report("wait_timeout", act=H.ACT[act], code=code, site=info, seconds=elapsed,
             recovered_worst_rel_err=worst)
    assert worst <= H.TOL[synth.DT_BF16], worst
