"""The C-ABI library without a GPU: it loads, exports exactly what include/moe.h
declares, its struct layouts match the ctypes binding, and host-side validation
rejects bad arguments before anything is launched."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest
import torch

from sparse_mixture_experts_12_b200 import binding as B
from sparse_mixture_experts_12_b200 import build as BUILD
from sparse_mixture_experts_12_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


@pytest.fixture(scope="module")
def lib():
    BUILD.build()
    return B.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_]+)\s*\(", src)))


def test_header_declares_the_abi():
    names = declared_functions()
    assert names == sorted(B.EXPORTED), names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", B.lib_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (moe_[a-z_]+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None
    # nothing else of ours leaks out of the library
    ours = set(re.findall(r"\bT (moe[A-Za-z_0-9]*)$", out, flags=re.M))
    assert ours == set(declared_functions())


def test_struct_layout_matches_header(tmp_path):
    prog = tmp_path / "layout.c"
    prog.write_text(
        '#include <stddef.h>\n#include <stdio.h>\n#include "moe.h"\n'
        "#define F(s, m) printf(#s \" \" #m \" %zu\\n\", offsetof(s, m))\n"
        "int main(void) {\n"
        + "".join(f"  F(moe_cfg_t, {n});\n" for n, _ in B.MoeCfg._fields_)
        + "".join(f"  F(moe_weights_t, {n});\n" for n, _ in B.MoeWeights._fields_)
        + "".join(f"  F(moe_taps_t, {n});\n" for n, _ in B.MoeTaps._fields_)
        + "".join(f"  F(moe_shard_t, {n});\n" for n, _ in B.MoeShard._fields_)
        + "".join(f"  F(moe_noise_t, {n});\n" for n, _ in B.MoeNoise._fields_)
        + '  printf("size moe_cfg_t %zu\\nsize moe_weights_t %zu\\nsize moe_taps_t %zu\\n",'
          " sizeof(moe_cfg_t), sizeof(moe_weights_t), sizeof(moe_taps_t));\n"
        + '  printf("size moe_shard_t %zu\\n", sizeof(moe_shard_t));\n'
        + '  printf("size moe_stage_events_t %zu\\n", sizeof(moe_stage_events_t));\n'
        + '  printf("size moe_noise_t %zu\\n", sizeof(moe_noise_t));\n'
        + '  printf("stages count %d\\n", (int)MOE_STAGE_COUNT);\n  return 0;\n}\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", f"-I{os.path.dirname(HEADER)}", str(prog), "-o", str(exe)],
                   check=True)
    lines = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split("\n")
    got = {}
    for ln in lines:
        if ln:
            a, b, c = ln.split()
            got[(a, b)] = int(c)
    for st, cls in (("moe_cfg_t", B.MoeCfg), ("moe_weights_t", B.MoeWeights),
                    ("moe_taps_t", B.MoeTaps), ("moe_shard_t", B.MoeShard)):
        for n, _ in cls._fields_:
            assert got[(st, n)] == getattr(cls, n).offset, (st, n)
        assert got[("size", st)] == ctypes.sizeof(cls)
    assert got[("size", "moe_stage_events_t")] == ctypes.sizeof(B.MoeStageEvents)
    for n, _ in B.MoeNoise._fields_:
        assert got[("moe_noise_t", n)] == getattr(B.MoeNoise, n).offset, n
    assert got[("size", "moe_noise_t")] == ctypes.sizeof(B.MoeNoise)
    assert got[("stages", "count")] == len(B.STAGES)


def _status(lib, cfg):
    n = ctypes.c_size_t(0)
    return lib.moe_workspace_size(ctypes.byref(cfg), ctypes.byref(n)), n.value


@pytest.mark.parametrize("over,expect", [
    ({}, B.MOE_OK),
    ({"n_experts": 0}, 1), ({"n_experts": 257}, 1), ({"top_k": 0}, 1), ({"top_k": 9}, 1),
    ({"n_experts": 4, "top_k": 5}, 1), ({"n_tokens": -1}, 1), ({"d_model": 0}, 1),
    ({"d_ff": -5}, 1), ({"act": 3}, 1), ({"gate_mode": 7}, 1), ({"dtype": 2}, 1),
    ({"capacity_factor": float("nan")}, 1), ({"n_shared": -1}, 1),
    ({"n_shared": 1, "d_ff_shared": 0}, 1),
    ({"d_model": 4000}, 2), ({"d_ff": 14300}, 2), ({"n_shared": 1, "d_ff_shared": 100}, 2),
])
def test_config_validation(lib, over, expect):
    cfg = B.make_cfg(synth.MIXTRAL_PREFILL, **over)
    st, n = _status(lib, cfg)
    assert st == expect, (over, st)
    if expect == B.MOE_OK:
        assert n > 0


def test_fp32_path_accepts_unaligned_sizes(lib):
    cfg = B.make_cfg(synth.SMALL["fp32_swiglu"], d_ff=161)
    assert _status(lib, cfg)[0] == B.MOE_OK
    cfg = B.make_cfg(synth.SMALL["fp32_swiglu"], d_model=98)
    assert _status(lib, cfg)[0] == 2


def test_workspace_grows_with_the_problem(lib):
    small = _status(lib, B.make_cfg(synth.SMALL["mixtral_small"]))[1]
    big = _status(lib, B.make_cfg(synth.MIXTRAL_PREFILL))[1]
    shared = _status(lib, B.make_cfg(synth.DEEPSEEK_FINE))[1]
    noshared = _status(lib, B.make_cfg(synth.DEEPSEEK_FINE, n_shared=0))[1]
    assert 0 < small < big and shared > noshared


def test_entry_points_reject_bad_pointers_before_launching(lib):
    """Every failure here is decided on the host: no CUDA call is made."""
    wl = synth.SMALL["mixtral_small"]
    cfg = B.make_cfg(wl)
    ws_bytes = B.workspace_size(cfg)
    ws = ctypes.c_void_p(0x100000)          # fake, 256-aligned: never dereferenced
    good = ctypes.c_void_p(0x200000)
    odd = ctypes.c_void_p(0x200008)
    W = B.MoeWeights(w_router=good, w1=good, w3=good, w2=good)
    fwd = lambda x, y, w=W, ws_=ws, n=ws_bytes: lib.moe_forward(  # noqa: E731
        ctypes.byref(cfg), ctypes.byref(w), x, y, None, None, ws_, n, None)
    assert fwd(None, good) == 1                          # x missing
    assert fwd(odd, good) == 3                           # x misaligned
    assert fwd(good, good, ws_=ctypes.c_void_p(0x100080)) == 3   # ws not 256-aligned
    assert fwd(good, good, n=ws_bytes - 1) == 4          # workspace too small
    assert fwd(good, good, ws_=None) == 1
    assert fwd(good, good, w=B.MoeWeights(w_router=good, w1=good, w2=good)) == 1  # no w_up
    assert fwd(good, good, w=B.MoeWeights(w_router=good, w1=good, w3=good, w2=good,
                                          b1=good)) == 1  # SwiGLU experts take no bias
    assert lib.moe_route(ctypes.byref(cfg), ctypes.byref(W), None, None, good, good, ws,
                         ws_bytes, None) == 1            # logits input missing
    assert lib.moe_permute(ctypes.byref(cfg), good, good, good, good, good, odd, good, ws,
                           ws_bytes, None) == 3
    assert lib.moe_combine(ctypes.byref(cfg), good, good, good, odd, good, ws, ws_bytes,
                           None) == 3
    assert lib.moe_aux_stats(ctypes.byref(cfg), good, None, good, ws, ws_bytes, None) == 1
    assert lib.moe_expert_ffn(ctypes.byref(cfg), ctypes.byref(W), good, good, None, ws,
                              ws_bytes, None) == 1
    code = ctypes.c_int32(0)
    assert lib.moe_last_device_error(None, ctypes.byref(code), None, None) == 1
    assert lib.moe_status_string(4) == b"workspace too small"


@pytest.mark.parametrize("over,expect", [
    ({}, B.MOE_OK),
    ({"routing": 2}, 1),                           # no such routing
    ({"capacity_factor": 0.0}, 1),                 # expert choice needs cf > 0
    ({"capacity_factor": 0.001}, 1),               # C = 0: an expert would take nothing
    ({"capacity_factor": 9.0}, 1),                 # C > T
    ({"n_tokens": 40000, "capacity_factor": 0.1}, 2),   # T beyond one CTA's column
    ({"capacity_factor": 8.0, "n_tokens": 16384}, 2),   # C = 16384 > 8192 picks
    ({"n_shared": 2, "d_ff_shared": 8192}, 2),     # shared experts with expert choice
])
def test_expert_choice_config_validation(lib, over, expect):
    cfg = B.make_cfg(synth.MIXTRAL_EC, **over)
    st, n = _status(lib, cfg)
    assert st == expect, (over, st)


def test_expert_choice_workspace_holds_its_rows(lib):
    """cf = 2 over 8 experts: 2T expert rows, twice top-1 token choice's."""
    ec = _status(lib, B.make_cfg(synth.MIXTRAL_EC))[1]
    tc = _status(lib, B.make_cfg(synth.MIXTRAL_EC, routing=0, capacity_factor=0.0))[1]
    assert ec > tc


def test_expert_choice_entry_points_reject_before_launching(lib):
    wl = synth.SMALL["ec_small"]
    cfg = B.make_cfg(wl)
    ws_bytes = B.workspace_size(cfg)
    ws = ctypes.c_void_p(0x100000)
    good = ctypes.c_void_p(0x200000)
    odd = ctypes.c_void_p(0x200008)
    W = B.MoeWeights(w_router=good, w1=good, w3=good, w2=good)
    route = lib.moe_route_expert_choice
    assert route(ctypes.byref(cfg), ctypes.byref(W), None, None, good, good, ws, ws_bytes,
                 None) == 1                          # logits input missing
    assert route(ctypes.byref(cfg), ctypes.byref(W), None, good, odd, good, ws, ws_bytes,
                 None) == 3                          # ec_idx misaligned
    tc = B.make_cfg(wl, routing=0)
    assert route(ctypes.byref(tc), ctypes.byref(W), None, good, good, good, ws,
                 B.workspace_size(tc), None) == 1    # a token-choice configuration
    # moe_forward: expert choice produces no load-balancing statistics
    assert lib.moe_forward(ctypes.byref(cfg), ctypes.byref(W), good, good, good, None, ws,
                           ws_bytes, None) == 1


# ------------------------------------------------------ buffer sizes in the binding
def test_binding_expert_rows_follow_the_routing():
    """x_perm / y_perm hold T*k rows under token choice and E*C under expert choice,
    C = floor(cf*T/E) (the oracle's expert-choice capacity)."""
    from sparse_mixture_experts_12_b200 import binding as Bd
    from oracle import moe_oracle as Or
    tc = synth.WORKLOADS["mixtral_prefill"]
    assert Bd.expert_rows(Bd.make_cfg(tc)) == tc.T * tc.top_k
    ec = synth.WORKLOADS["mixtral_ec"]
    C = Or.expert_choice_capacity(ec.capacity_factor, ec.T, ec.n_experts)
    assert Bd.expert_rows(Bd.make_cfg(ec)) == ec.n_experts * C == 8192
    assert Bd.expert_rows(Bd.make_cfg(ec.replace(capacity_factor=0.0))) == 0


def test_binding_refuses_short_expert_buffers():
    """A tensor with fewer rows than the library will touch is refused before any
    launch (the C ABI only sees a pointer): an expert-choice layer's x_perm sized for
    token choice (T*k = 4096 rows instead of E*C = 8192) among them."""
    from sparse_mixture_experts_12_b200 import binding as Bd
    ec = synth.WORKLOADS["mixtral_ec"]
    R, d = Bd.expert_rows(Bd.make_cfg(ec)), ec.d_model
    Bd.check_rows(torch.empty((R, d)), R, d, "x_perm")
    Bd.check_rows(torch.empty((R + 5, d)), R, d, "x_perm")
    Bd.check_rows(None, R, d, "x_perm")
    for bad in (torch.empty((ec.T * ec.top_k, d)), torch.empty((R, d + 1)),
                torch.empty((d, R)).t(), torch.empty(R * d)):
        with pytest.raises(ValueError):
            Bd.check_rows(bad, R, d, "x_perm")
