"""Helpers shared by the GPU parity tests: oracle-side views of the inputs,
the per-token error measure, the fp32 error bound of the router GEMM, and a
small JSON report of what each parity test saw (near-tie tokens and so on)."""
from __future__ import annotations

import json
import os

import numpy as np
import torch

from oracle import moe_oracle as O
from sparse_mixture_experts_12_b200 import synth
from tests.oracle_pins import ACT, MODE

# Tolerance on the per-token max relative error (see ``max_rel_err``).
TOL = {synth.DT_F32: 1e-5, synth.DT_BF16: 2e-2}
# Tokens whose sorted top-(k+1) logits are closer than this are near-ties.
MARGIN = 1e-4
U32 = 2.0 ** -24
# the device's fp32 Box-Muller draws against the oracle's fp64 ones (logf, sincospif
# within 1 ulp each, sqrtf and the products correctly rounded): 8 ulp, relative
EPS_REL = 8 * 2.0 ** -23


class F64View:
    """Indexable fp64 view of a (possibly bf16) CPU tensor, converted slice by slice
    so that the oracle can walk multi-GB weight stacks expert by expert."""

    def __init__(self, t: torch.Tensor):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, i):
        return synth.to_f64_numpy(self.t[i])


def oracle_params(inp: dict) -> dict:
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif v.numel() > (1 << 22) and k not in ("x", "w_router"):
            out[k] = F64View(v)
        else:
            out[k] = synth.to_f64_numpy(v)
    return out


def oracle_kwargs(wl: synth.Workload) -> dict:
    return dict(top_k=wl.top_k, act=ACT[wl.act], gate_mode=MODE[wl.gate_mode],
                capacity_factor=wl.capacity_factor, n_shared=wl.n_shared)


def max_rel_err(y, yref) -> np.ndarray:
    """Per token ||y_t - yref_t||_inf / ||yref_t||_inf; a token whose reference is
    exactly zero must be exactly zero (inf otherwise, 0 if so)."""
    y = np.asarray(y, dtype=np.float64)
    yref = np.asarray(yref, dtype=np.float64)
    num = np.abs(y - yref).max(axis=1)
    den = np.abs(yref).max(axis=1)
    out = np.zeros(len(y))
    nz = den > 0
    out[nz] = num[nz] / den[nz]
    out[~nz] = np.where(num[~nz] == 0, 0.0, np.inf)
    return out


def logits_bound(x64, w64, extra_abs=None) -> np.ndarray:
    """Worst-case fp32 accumulation error of x W^T with d terms (plus the bias
    additions): gamma_(d+2) * (|x| |W|^T + |biases|), with a 2x safety factor."""
    d = x64.shape[1]
    s = np.abs(x64) @ np.abs(w64).T
    if extra_abs is not None:
        s = s + extra_abs[None, :]
    return 2.0 * (d + 2) * U32 * s + 1e-30


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy() if t.is_floating_point() \
        else t.detach().to("cpu").numpy()


def report(name: str, **fields):
    d = os.environ.get("MOE_TEST_REPORT_DIR")
    if not d:
        return
    os.makedirs(d, exist_ok=True)
    with open(os.path.join(d, "parity_report.jsonl"), "a") as f:
        f.write(json.dumps({"test": name, **fields}, default=float) + "\n")


def routing_compare(gpu_idx: np.ndarray, ref_logits: np.ndarray, ref_idx: np.ndarray, k: int,
                    cap):
    """Tokens routed differently must all be near-ties. Returns (mismatched tokens,
    tokens whose output may legitimately differ because of them)."""
    mism = np.nonzero((gpu_idx != ref_idx).any(axis=1))[0]
    margin = O.topk_margin(ref_logits, k)
    assert np.all(margin[mism] < MARGIN), (
        f"tokens routed differently without a near-tie: {mism[margin[mism] >= MARGIN][:10]}")
    affected = set(int(t) for t in mism)
    if cap is not None and len(mism):
        # a flipped token shifts the capacity ranks of later tokens in both experts
        experts = set(ref_idx[mism].ravel().tolist()) | set(gpu_idx[mism].ravel().tolist())
        t0 = int(mism.min())
        later = np.arange(len(ref_idx)) >= t0
        hit = np.isin(ref_idx, list(experts)).any(axis=1) | np.isin(gpu_idx, list(experts)).any(axis=1)
        affected |= set(np.nonzero(later & hit)[0].tolist())
    return mism, affected, int((margin < MARGIN).sum())


ROW_TILE = 128  # rows of one grouped-GEMM M tile


def tile_rows(offsets) -> list:
    """(expert, first row, last row) of every ROW_TILE-row tile of the expert-contiguous
    rows: expert e owns rows [offsets[e], offsets[e+1])."""
    out = []
    offsets = np.asarray(offsets, dtype=np.int64)
    for e in range(len(offsets) - 1):
        a, b = int(offsets[e]), int(offsets[e + 1])
        for r0 in range(a, b, ROW_TILE):
            out.append((e, r0, min(r0 + ROW_TILE, b) - 1))
    return out


def tile_cover_tokens(row_token, offsets, T: int, n_strided: int = 48, extra=()):
    """Tokens to compare at full size: the tokens of the first, the middle and the
    last row of every expert tile (row_token maps a row to its token), plus a strided
    sample and ``extra``. Returns (sorted unique tokens, tile list)."""
    tiles = tile_rows(offsets)
    toks = set(synth.token_sample(T, n_strided).tolist())
    toks |= set(int(t) for t in extra)
    for _, r0, r1 in tiles:
        for r in (r0, (r0 + r1) // 2, r1):
            toks.add(int(row_token[r]))
    return np.array(sorted(toks), dtype=np.int64), tiles


def tiles_covered(tiles, row_token, compared) -> int:
    """Tiles with at least one row whose token is among ``compared``."""
    cmp = set(int(t) for t in compared)
    n = 0
    for _, r0, r1 in tiles:
        if any(int(row_token[r]) in cmp for r in range(r0, r1 + 1)):
            n += 1
    return n
