"""A second, independent statement of the MoE layer in torch (CPU, fp64), following
the module structure of the pages' listings: nn.Linear experts, torch.topk,
F.softmax, boolean masks and per-expert loops. It is used only to pin the numpy
oracle at small sizes; it shares no code with it.

Listings restated (page titles as in the oracle's header):
P1 ``MoELayer`` (biased gate, top-k then softmax, ReLU experts),
P3 ``MoELayer`` (GELU experts), ``SwitchRouter`` (top-1 with capacity),
``MixtralMoELayer`` / ``SwiGLUExpert``, ``DeepSeekMoELayer`` (shared + routed),
P4 ``TopKGating`` (softmax, top-k, renormalise) and ``compute_load_balancing_loss``.
"""
from __future__ import annotations

import torch
import torch.nn as nn
import torch.nn.functional as F


def _lin(w, b=None):
    m = nn.Linear(w.shape[1], w.shape[0], bias=b is not None).double()
    with torch.no_grad():
        m.weight.copy_(torch.as_tensor(w, dtype=torch.float64))
        if b is not None:
            m.bias.copy_(torch.as_tensor(b, dtype=torch.float64))
    return m


class MLPExpert(nn.Module):
    def __init__(self, w1, b1, w2, b2, act):
        super().__init__()
        self.net = nn.Sequential(_lin(w1, b1), nn.ReLU() if act == "relu" else nn.GELU(),
                                 _lin(w2, b2))

    def forward(self, x):
        return self.net(x)


class SwiGLUExpert(nn.Module):
    def __init__(self, w_gate, w_up, w_down):
        super().__init__()
        self.w_gate, self.w_up, self.w_down = _lin(w_gate), _lin(w_up), _lin(w_down)

    def forward(self, x):
        return self.w_down(F.silu(self.w_gate(x)) * self.w_up(x))


def build_experts(p, act):
    E = p["w1"].shape[0]
    out = []
    for e in range(E):
        if act == "swiglu":
            out.append(SwiGLUExpert(p["w1"][e], p["w3"][e], p["w2"][e]))
        else:
            b1 = None if p.get("b1") is None else p["b1"][e]
            b2 = None if p.get("b2") is None else p["b2"][e]
            out.append(MLPExpert(p["w1"][e], b1, p["w2"][e], b2, act))
    return out


def gating(logits, k, mode):
    """Returns (weights [T,k], indices [T,k], probs [T,E])."""
    probs = F.softmax(logits, dim=-1)
    if mode == "topk_softmax":
        top, ind = torch.topk(logits, k, dim=-1)
        return F.softmax(top, dim=-1), ind, probs
    top, ind = torch.topk(probs, k, dim=-1)
    if mode == "softmax_topk_renorm":
        top = top / top.sum(dim=-1, keepdim=True)
    return top, ind, probs


def switch_keep_mask(indices, num_experts, cap):
    """P3 SwitchRouter drop rule for top-1 (flattened tokens): for each expert,
    keep the first ``cap`` positions returned by nonzero()."""
    keep = torch.zeros_like(indices, dtype=torch.bool)
    for i in range(num_experts):
        m = indices == i
        pos = m.nonzero(as_tuple=True)[0]
        if cap is not None and len(pos) > cap:
            m[pos[cap:]] = False
        keep |= m
    return keep


def moe_layer(x, p, *, k, act, mode, cap=None, n_shared=0):
    """Forward of the layer, loop form of the pages. ``cap`` applies to top-1 only."""
    x = torch.as_tensor(x, dtype=torch.float64)
    gate = _lin(p["w_router"], p.get("b_router"))
    logits = gate(x)
    if p.get("logit_bias") is not None:
        logits = logits + torch.as_tensor(p["logit_bias"], dtype=torch.float64)
    weights, indices, probs = gating(logits, k, mode)
    experts = build_experts(p, act)
    keep = torch.ones_like(indices, dtype=torch.bool)
    if cap is not None:
        assert k == 1
        keep = switch_keep_mask(indices[:, 0], len(experts), cap)[:, None]
    out = torch.zeros_like(x)
    for i in range(k):
        ei = indices[:, i]
        wi = weights[:, i]
        for j in range(len(experts)):
            mask = (ei == j) & keep[:, i]
            if mask.any():
                out[mask] += wi[mask].unsqueeze(-1) * experts[j](x[mask])
    if n_shared:
        Fs = p["ws_gate"].shape[0] // n_shared
        shared = [SwiGLUExpert(p["ws_gate"][j * Fs:(j + 1) * Fs], p["ws_up"][j * Fs:(j + 1) * Fs],
                               p["ws_down"][:, j * Fs:(j + 1) * Fs]) for j in range(n_shared)]
        out = out + sum(e(x) for e in shared)
    return out.detach(), logits.detach(), indices, weights.detach(), probs.detach()


def load_balancing_loss(probs, indices, num_experts, top_k, alpha):
    """P4 compute_load_balancing_loss times the aux weight."""
    mask = F.one_hot(indices, num_experts).double().sum(dim=1)
    f = mask.sum(dim=0) / (probs.shape[0] * top_k)
    P = probs.mean(dim=0)
    return f, P, alpha * num_experts * (f * P).sum()
