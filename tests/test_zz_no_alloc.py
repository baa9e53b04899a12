"""moe_permute_noalloc against moe_permute, through the C ABI.

The no-allocation variant serves callers that own no device memory beyond their
inputs and outputs (a plugin inside a framework with its own memory arena, a
loop where cudaMalloc's possible device synchronisation is not acceptable), so
it keeps its scratch in a static device array instead of a caller workspace.
Its outputs must equal the workspace entry point's exactly (indices, counts,
offsets, permutation and the gathered rows), on two calls in a row whose
routings differ, so that nothing left in the shared array by one call leaks
into the next. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_12_b200 import binding as B
from sparse_mixture_experts_12_b200 import build as BUILD
from sparse_mixture_experts_12_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _outputs(T, E, k, d, dtype):
    i32 = dict(dtype=torch.int32, device=DEV)
    return {"counts": torch.full((E,), -5, **i32), "offsets": torch.full((E + 1,), -5, **i32),
            "perm": torch.full((T * k,), -5, **i32), "inv": torch.full((T * k,), -5, **i32),
            "x_perm": torch.zeros((T * k, d), dtype=dtype, device=DEV)}


@pytest.mark.parametrize("E,k,T,cf,dt", [(8, 2, 1000, 0.0, synth.DT_BF16),
                                          (128, 1, 3001, 1.25, synth.DT_BF16),
                                          (64, 6, 777, 0.5, synth.DT_F32)])
def test_noalloc_permute_matches_workspace_permute(E, k, T, cf, dt):
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device")
    BUILD.build()
    lib = B.load()
    d = 128
    wl = synth.SMALL["mixtral_small"].replace(T=T, n_experts=E, top_k=k, capacity_factor=cf,
                                              d_model=d, dtype=dt)
    cfg = B.make_cfg(wl)
    ws = B.new_workspace(cfg, DEV)
    x = synth.generate(wl, seed=T, with_weights=False)["x"].to(DEV)
    for call in range(2):  # two calls in a row, different routings
        z = synth.random_logits(T, E, seed=100 * call + E, std=2.0)
        z = z + torch.linspace(2.0 * (call + 1), -2.0, E)[None, :]
        idx = torch.from_numpy(O.select_topk(z.numpy(), k)).to(DEV)
        ref = _outputs(T, E, k, d, x.dtype)
        got = _outputs(T, E, k, d, x.dtype)
        st = lib.moe_permute(ctypes.byref(cfg), _p(x), _p(idx), _p(ref["counts"]),
                             _p(ref["offsets"]), _p(ref["perm"]), _p(ref["inv"]),
                             _p(ref["x_perm"]), _p(ws), ws.numel(), _s())
        assert st == 0
        st = lib.moe_permute_noalloc(ctypes.byref(cfg), _p(x), _p(idx), _p(got["counts"]),
                                     _p(got["offsets"]), _p(got["perm"]), _p(got["inv"]),
                                     _p(got["x_perm"]), _s())
        assert st == 0
        torch.cuda.synchronize()
        R = int(ref["offsets"][-1].item())
        for key in ("counts", "offsets", "inv"):
            assert torch.equal(got[key], ref[key]), (call, key)
        assert torch.equal(got["perm"][:R], ref["perm"][:R]), call
        assert torch.equal(got["x_perm"][:R], ref["x_perm"][:R]), call
        if cf > 0:
            assert R < T * k  # capacity dropped something: the drop path was exercised


def test_noalloc_permute_rejects_sizes_beyond_its_scratch():
    BUILD.build()
    lib = B.load()
    # E = 256 uses 32-token tiles: 256 * ceil(T / 32) must stay <= 65536, i.e. T <= 8192
    wl = synth.SMALL["mixtral_small"].replace(T=8193, n_experts=256, top_k=2, d_model=128)
    cfg = B.make_cfg(wl)
    fake = ctypes.c_void_p(0x200000)  # never dereferenced: rejected on the host
    st = lib.moe_permute_noalloc(ctypes.byref(cfg), fake, fake, fake, fake, fake, fake, fake,
                                 None)
    assert st == 4  # MOE_ERR_WORKSPACE


def test_noalloc_permute_drops_out_of_range_indices():
    """With no workspace there is no error word: a pair whose expert index is out of
    range is dropped (inv = -1) and left out of every count, and the other pairs are
    laid out as if it were absent. The workspace entry point treats such a pair the
    same way (and also reports it), so the two must agree exactly."""
    BUILD.build()
    lib = B.load()
    T, E, k, d = 700, 16, 2, 128
    wl = synth.SMALL["mixtral_small"].replace(T=T, n_experts=E, top_k=k, capacity_factor=0.9,
                                              d_model=d)
    cfg = B.make_cfg(wl)
    ws = B.new_workspace(cfg, DEV)
    x = synth.generate(wl, seed=11, with_weights=False)["x"].to(DEV)
    idx_np = O.select_topk(synth.random_logits(T, E, seed=12, std=2.0).numpy(), k)
    bad = [(3, 0, E), (3, 1, -1), (250, 1, 1000), (699, 0, -7)]
    for t, s, v in bad:
        idx_np[t, s] = v
    idx = torch.from_numpy(idx_np).to(DEV)
    ref = _outputs(T, E, k, d, x.dtype)
    got = _outputs(T, E, k, d, x.dtype)
    assert lib.moe_permute(ctypes.byref(cfg), _p(x), _p(idx), _p(ref["counts"]),
                           _p(ref["offsets"]), _p(ref["perm"]), _p(ref["inv"]),
                           _p(ref["x_perm"]), _p(ws), ws.numel(), _s()) == 0
    assert lib.moe_permute_noalloc(ctypes.byref(cfg), _p(x), _p(idx), _p(got["counts"]),
                                   _p(got["offsets"]), _p(got["perm"]), _p(got["inv"]),
                                   _p(got["x_perm"]), _s()) == 0
    torch.cuda.synchronize()
    code, info = ctypes.c_int32(0), ctypes.c_int32(0)
    lib.moe_last_device_error(_p(ws), ctypes.byref(code), ctypes.byref(info), _s())
    assert code.value == 1  # the workspace path reports the first bad pair it met
    inv = got["inv"].cpu().numpy().reshape(T, k)
    for t, s, _ in bad:
        assert inv[t, s] == -1
    valid = (idx_np >= 0) & (idx_np < E)
    counts = np.bincount(idx_np[valid], minlength=E)
    assert np.array_equal(got["counts"].cpu().numpy(), counts)
    R = int(ref["offsets"][-1].item())
    for key in ("counts", "offsets", "inv"):
        assert torch.equal(got[key], ref[key]), key
    assert torch.equal(got["perm"][:R], ref["perm"][:R])
    assert torch.equal(got["x_perm"][:R], ref["x_perm"][:R])
    # the kept pairs are exactly the oracle's for the routing with the bad pairs
    # removed: give each bad pair an expert of its own past the end, then drop it
    cap = O.capacity(wl.capacity_factor, T, k, E)
    fixed = idx_np.copy()
    fixed[~valid] = E
    caps = np.full(E + 1, cap)
    caps[E] = 0
    _, rank, kept = O.dispatch_with_caps(fixed, E + 1, caps)
    assert np.array_equal(inv >= 0, kept)
