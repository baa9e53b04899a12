"""CPU oracle of the sparse Mixture-of-Experts FFN forward.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module:
only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may call it. It shares no code with the CUDA library.

It is written for a reader who checks it against the pages by eye: fp64 numpy,
plain loops where the pages loop, a library matmul / sort / erf as single steps,
no blocking, fusion or reordering. Inputs are the dtype-rounded values (bf16 or
fp32) upcast exactly to fp64.

Pages cited (by title and the listing or section that defines each step):

* P1 — devtips.kr, "MoE (Mixture of Experts) 아키텍처 완전 정복: Mixtral부터
  DeepSeek-MoE까지 구현 원리와 실전 최적화 기법": ``MoELayer``, ``DeepSeekMoE``, the
  capacity snippet, ``load_balancing_loss``.
* P2 — ricepunchb.github.io, "MoE" study note: §4 diagram (gate scores 0.8/0.2),
  §5 formulas (garbled), §7 stabilisation list.
* P3 — youngju.dev, "Mixture of Experts（MoE）架构深度解析：从 Switch Transformer 到
  Mixtral 的演进与高效扩展策略": ``GatingNetwork``, ``MoELayer`` (GELU),
  ``SwitchRouter``, ``load_balancing_loss``, ``MixtralMoELayer``, ``SwiGLUExpert``,
  ``DeepSeekMoELayer``, ``ExpertChoiceRouter``.
* P4 — youngju.dev, "Sparse Mixture of Experts（MoE）アーキテクチャ深層分析：設計原理
  からDeepSeek-V3・Qwen3まで": the gating equation, ``SwiGLUExpert``, ``TopKGating``,
  ``ExpertChoiceGating``, ``compute_load_balancing_loss``, ``MoELayerWithAuxLoss``,
  ``router_z_loss``.
* P5 — study-site lecture 03, "Mixture of Experts": "Token Routing" (gates 0.7/0.3,
  unselected experts are not computed), "SiLU · SwiGLU · MoE" table.

Readings taken where the pages are silent or disagree (each is also pinned by a
test):

* top-k is selected on the fp32 logits in every gate mode (softmax is monotone;
  P4 selects on probabilities, P1/P3 on logits); slots are in descending value,
  equal values go to the lower expert index first.
* capacity = floor(cf * T * k / E) in double, T = every token of the call; no
  minimum capacity; cf <= 0 means unlimited.
* overflow is dropped in token-major, then slot, order; a dropped slot adds 0 and
  the surviving gates are not renormalised.
* f_i counts pre-drop assignments over T*k; P_i is the mean full softmax of the
  router logits (router bias and logit bias included).
* GELU is the exact erf form; dropout and routing noise are off (inference).
* Noisy top-k gating (training mode of P4 ``TopKGating``): the standard normal
  draws eps [T, E] are either an input, so both sides see the same draws, or the
  counter-based draws of ``noise_draws`` (Philox4x32-10 and Box-Muller) for a seed
  and an offset, which both sides compute from the generator's published
  definition.
* Expert-Choice routing: each expert takes int(cf * T / E) tokens, chosen on the
  fp32 logits (equal logits: lower token index first); a token's output is the
  score-weighted sum over the experts that took it (P4's dispatch mask used as
  the gate), 0 if none did.
* A batch split by tokens over several shards gives every token what the single
  call over the whole batch gives: the capacity is that of the whole batch, and
  each shard keeps per expert what the earlier shards' pre-drop pairs left.
* No intermediate rounding: everything after the fp32 logits is fp64.

Parity status: every function below is pinned by the CPU test suite; none is
"parity unpinned".
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np
from scipy.special import erf as _erf

ACTS = ("relu", "gelu", "swiglu")
GATE_MODES = ("topk_softmax", "softmax_topk_renorm", "softmax_topk_raw")


def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------- router
def router_logits(x, w_router, b_router=None, logit_bias=None) -> np.ndarray:
    """z = x W_r^T (+ b_r) (+ logit_bias), exact in fp64, rounded once to fp32.

    P1 ``MoELayer``: the gate is ``nn.Linear(hidden, E)`` with a bias.
    P3 ``GatingNetwork`` / ``SwitchRouter`` / ``MixtralMoELayer``: bias-free gate.
    ``logit_bias`` is the per-expert skew of the Switch workload, added to the logits.
    """
    z = _f64(x) @ _f64(w_router).T
    if b_router is not None:
        z = z + _f64(b_router)[None, :]
    if logit_bias is not None:
        z = z + _f64(logit_bias)[None, :]
    return z.astype(np.float32)


def softmax(z) -> np.ndarray:
    """Row softmax over experts in fp64, max-subtracted (P3 ``SwitchRouter``, P4 ``TopKGating``)."""
    z = _f64(z)
    m = z.max(axis=-1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=-1, keepdims=True)


def select_topk(logits32, k: int) -> np.ndarray:
    """Indices [T, k] of the k largest fp32 logits per token, in descending order.

    P1 ``MoELayer`` and P3 ``GatingNetwork``: ``torch.topk`` over the gate scores.
    Ties: the lower expert index comes first (a stable sort of the negated values).
    """
    z = np.asarray(logits32, dtype=np.float32).astype(np.float64)
    order = np.argsort(-z, axis=1, kind="stable")
    return order[:, :k].astype(np.int32)


def gate_values(logits32, idx, mode: str) -> np.ndarray:
    """Gate weight per selected slot, fp64 [T, k].

    * ``topk_softmax`` (P1 ``MoELayer``, P3 ``GatingNetwork``/``MixtralMoELayer``/
      ``DeepSeekMoELayer``): softmax over the k selected logits only.
    * ``softmax_topk_renorm`` (P4 ``TopKGating``): full softmax over E, keep the
      selected probabilities, divide by their sum.
    * ``softmax_topk_raw`` (P3 ``SwitchRouter``; P4 gating equation, where G is the
      softmax inside the top-k and 0 elsewhere): the selected probabilities as they are.
    """
    z = np.asarray(logits32, dtype=np.float32).astype(np.float64)
    idx = np.asarray(idx)
    T, k = idx.shape
    g = np.zeros((T, k), dtype=np.float64)
    if mode == "topk_softmax":
        for t in range(T):
            sel = z[t, idx[t]]
            e = np.exp(sel - sel.max())
            g[t] = e / e.sum()
    elif mode in ("softmax_topk_renorm", "softmax_topk_raw"):
        p = softmax(z)
        for t in range(T):
            sel = p[t, idx[t]]
            g[t] = sel / sel.sum() if mode == "softmax_topk_renorm" else sel
    else:
        raise ValueError(mode)
    return g


def topk_margin(logits32, k: int) -> np.ndarray:
    """Smallest gap between consecutive values among the sorted top-(k+1) logits.

    A token whose margin is tiny (below 1e-4) can legitimately be routed
    differently by two correct fp32 implementations; such tokens are reported
    apart from the parity failures.
    """
    z = np.sort(np.asarray(logits32, dtype=np.float32).astype(np.float64), axis=1)[:, ::-1]
    m = min(k + 1, z.shape[1])
    if m < 2:
        return np.full(z.shape[0], np.inf)
    gaps = z[:, :m - 1] - z[:, 1:m]
    return gaps.min(axis=1)


# ------------------------------------------------------------------- dispatch / drop
def capacity(capacity_factor: float, T: int, k: int, E: int) -> Optional[int]:
    """Per-expert row capacity, or None when unlimited.

    P1 capacity snippet: (tokens * top_k / E) * capacity_factor.
    P3 ``SwitchRouter``: ``int(capacity_factor * T / E)`` (top-1).
    Taken as floor(cf * T * k / E) evaluated in double.
    """
    if capacity_factor is None or capacity_factor <= 0:
        return None
    return int(math.floor(float(capacity_factor) * T * k / E))


def dispatch(idx, E: int, cap: Optional[int]):
    """Walk (token, slot) pairs in token-major order and assign per-expert ranks.

    P3 ``SwitchRouter``: for each expert, the positions routed to it are listed
    in token order and those past ``capacity`` are dropped.

    Returns ``counts`` [E] (before drops), ``rank`` [T, k] (the pair's position
    inside its expert, before drops) and ``kept`` [T, k] bool.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    counts = np.zeros(E, dtype=np.int64)
    rank = np.zeros((T, k), dtype=np.int64)
    kept = np.zeros((T, k), dtype=bool)
    for t in range(T):
        for s in range(k):
            e = int(idx[t, s])
            rank[t, s] = counts[e]
            counts[e] += 1
            kept[t, s] = cap is None or rank[t, s] < cap
    return counts, rank, kept


def expert_layout(idx, rank, kept, E: int):
    """Expert-contiguous row order of the kept pairs.

    Rows of expert e occupy [offsets[e], offsets[e+1]) in token order;
    ``perm[row]`` is the token of that row, ``inv[t, s]`` the row of pair (t, s)
    or -1 when it was dropped.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    kept_counts = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for s in range(k):
            if kept[t, s]:
                kept_counts[idx[t, s]] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept_counts)
    perm = np.full(int(offsets[-1]), -1, dtype=np.int64)
    inv = np.full((T, k), -1, dtype=np.int64)
    for t in range(T):
        for s in range(k):
            if kept[t, s]:
                row = offsets[idx[t, s]] + rank[t, s]
                perm[row] = t
                inv[t, s] = row
    return offsets, perm, inv


# -------------------------------------------------------------------------- experts
def gelu(v):
    """Exact GELU, 0.5 v (1 + erf(v / sqrt 2)) (``nn.GELU()`` default in P3 ``MoELayer``)."""
    return 0.5 * v * (1.0 + _erf(v / math.sqrt(2.0)))


def silu(v):
    """SiLU(v) = v * sigmoid(v) (P5 table: scalar x sigma(x))."""
    return v / (1.0 + np.exp(-v))


def expert_ffn(x_rows, act: str, w1, w2, w3=None, b1=None, b2=None) -> np.ndarray:
    """One expert on a block of rows, fp64.

    * ``relu`` — P1 ``MoELayer`` experts: Linear(d, F) -> ReLU -> Linear(F, d), with bias.
    * ``gelu`` — P3 ``MoELayer`` experts: Linear(d, F) -> GELU -> Linear(F, d), with bias.
    * ``swiglu`` — P3/P4 ``SwiGLUExpert``, P5 table: w_down(silu(w_gate x) * w_up x),
      no bias; ``w1`` is w_gate, ``w3`` is w_up, ``w2`` is w_down.
    Weights use the nn.Linear [out, in] layout.
    """
    x = _f64(x_rows)
    if act == "swiglu":
        h = silu(x @ _f64(w1).T) * (x @ _f64(w3).T)
    else:
        v = x @ _f64(w1).T
        if b1 is not None:
            v = v + _f64(b1)[None, :]
        h = np.maximum(v, 0.0) if act == "relu" else gelu(v)
    o = h @ _f64(w2).T
    if b2 is not None:
        o = o + _f64(b2)[None, :]
    return o


def shared_experts(x, ws_gate, ws_up, ws_down, n_shared: int) -> np.ndarray:
    """Sum of the always-on SwiGLU experts, unweighted (P3 ``DeepSeekMoELayer``;
    P1 ``DeepSeekMoE``). The weights arrive concatenated along d_ff; each expert's
    slice is applied separately and the outputs are added."""
    Fs = ws_gate.shape[0] // n_shared
    out = np.zeros((x.shape[0], ws_down.shape[0]), dtype=np.float64)
    for j in range(n_shared):
        sl = slice(j * Fs, (j + 1) * Fs)
        out += expert_ffn(x, "swiglu", ws_gate[sl], ws_down[:, sl], w3=ws_up[sl])
    return out


def combine(y_rows, inv, gates, shared=None) -> np.ndarray:
    """Gate-weighted combine of expert rows: y_t = sum_{s: inv[t,s] >= 0} g_{t,s} y_rows[inv[t,s]]
    (+ shared_t). The gating equation of P4 with the pages' scatter-add written as a
    gather; a dropped slot (inv = -1) contributes nothing (P3 ``SwitchRouter``)."""
    y_rows = _f64(y_rows)
    inv = np.asarray(inv).reshape(np.asarray(gates).shape)
    gates = _f64(gates)
    T, k = inv.shape
    y = np.zeros((T, y_rows.shape[1]), dtype=np.float64)
    if shared is not None:
        y += _f64(shared)
    for t in range(T):
        for s in range(k):
            if inv[t, s] >= 0:
                y[t] += gates[t, s] * y_rows[inv[t, s]]
    return y


# -------------------------------------------------------------------------- forward
def route(x, params: dict, *, top_k: int, gate_mode: str, capacity_factor: float = 0.0,
          logits=None) -> dict:
    """Router, selection, gates, counts and capacity drops for all T tokens."""
    if logits is None:
        logits = router_logits(x, params["w_router"], params.get("b_router"),
                               params.get("logit_bias"))
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    idx = select_topk(logits, top_k)
    gates = gate_values(logits, idx, gate_mode)
    cap = capacity(capacity_factor, T, top_k, E)
    counts, rank, kept = dispatch(idx, E, cap)
    offsets, perm, inv = expert_layout(idx, rank, kept, E)
    return dict(logits=logits, idx=idx, gates=gates, capacity=cap, counts=counts,
                rank=rank, kept=kept, offsets=offsets, perm=perm, inv=inv)


def moe_forward(x, params: dict, *, top_k: int, act: str, gate_mode: str,
                capacity_factor: float = 0.0, n_shared: int = 0,
                logits=None, tokens: Optional[Sequence[int]] = None):
    """y = sum_i G(x)_i E_i(x) (+ shared experts) for every token, or for ``tokens``.

    P4 gating equation y = sum_i G(x)_i E_i(x); the loop form is P1 ``MoELayer`` /
    P3 ``MixtralMoELayer`` / P4 ``MoELayerWithAuxLoss``: for every slot and every
    expert, gather the rows routed there, run only that expert, and add the
    gate-weighted result (P5 "Token Routing": unselected experts are not computed).
    Capacity drops follow P3 ``SwitchRouter``; shared experts P3 ``DeepSeekMoELayer``.

    Routing always covers all tokens (capacity depends on the global token
    order); only the expert work is restricted to ``tokens``.
    Returns (y [len(tokens) or T, d] fp64, routing dict).
    """
    x = _f64(x)
    r = route(x, params, top_k=top_k, gate_mode=gate_mode,
              capacity_factor=capacity_factor, logits=logits)
    T = x.shape[0]
    E = r["logits"].shape[1]
    sel = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    in_sel = np.zeros(T, dtype=bool)
    in_sel[sel] = True
    pos = np.full(T, -1, dtype=np.int64)
    pos[sel] = np.arange(len(sel))
    y = np.zeros((len(sel), x.shape[1]), dtype=np.float64)
    if n_shared > 0:
        y += shared_experts(x[sel], params["ws_gate"], params["ws_up"], params["ws_down"],
                            n_shared)
    for s in range(top_k):
        for e in range(E):
            mask = (r["idx"][:, s] == e) & r["kept"][:, s] & in_sel
            if not mask.any():
                continue
            w3 = params["w3"][e] if params.get("w3") is not None else None
            b1 = params["b1"][e] if params.get("b1") is not None else None
            b2 = params["b2"][e] if params.get("b2") is not None else None
            out = expert_ffn(x[mask], act, params["w1"][e], params["w2"][e], w3, b1, b2)
            y[pos[mask]] += r["gates"][mask, s][:, None] * out
    return y, r


# ---------------------------------------------------------------------- aux outputs
def aux_stats(logits32, idx, E: int, top_k: int, alpha: float):
    """Switch load-balancing statistics.

    P3 ``load_balancing_loss`` and P4 ``compute_load_balancing_loss``:
    f_i = (assignments to expert i) / (T * k), counted before capacity drops;
    P_i = mean over tokens of the full softmax over experts;
    aux = alpha * E * sum_i f_i P_i (alpha = ``aux_loss_weight``, 0.01 in
    P4 ``MoEConfig`` and P3's default).
    """
    idx = np.asarray(idx)
    T = idx.shape[0]
    counts = np.zeros(E, dtype=np.int64)
    for e in idx.ravel():
        counts[int(e)] += 1
    f = counts / float(T * top_k)
    P = softmax(logits32).mean(axis=0)
    aux = alpha * E * float((f * P).sum())
    return f, P, aux


def router_z_loss(logits32) -> float:
    """P4 ``router_z_loss``: mean over tokens of logsumexp(logits)^2."""
    z = _f64(logits32)
    m = z.max(axis=1)
    lse = m + np.log(np.exp(z - m[:, None]).sum(axis=1))
    return float((lse ** 2).mean())


def balance_sq_loss(idx, E: int) -> float:
    """P1 ``load_balancing_loss``: sum_i (share_i - 1/E)^2, share_i = count_i / sum(counts)."""
    counts = np.zeros(E, dtype=np.float64)
    for e in np.asarray(idx).ravel():
        counts[int(e)] += 1
    share = counts / counts.sum()
    return float(((share - 1.0 / E) ** 2).sum())


# ------------------------------------------------------------ Expert-Choice routing
def expert_choice_capacity(capacity_factor: float, T: int, E: int) -> int:
    """Tokens each expert takes: int(cf * N / E) with N = all tokens of the call
    (P3 ``ExpertChoiceRouter``, P4 ``ExpertChoiceGating``: ``expert_capacity``)."""
    return int(math.floor(float(capacity_factor) * T / E))


def expert_choice_scores(logits32) -> np.ndarray:
    """Scores [E, T]: for every expert, the softmax of its logits over the tokens
    (P3: ``F.softmax(logits, dim=0)``; P4: ``F.softmax(gate_logits.T, dim=-1)``), fp64."""
    z = _f64(logits32).T
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    return e / e.sum(axis=1, keepdims=True)


def expert_choice_select(logits32, C: int) -> np.ndarray:
    """Token indices [E, C] each expert takes: its C highest-scoring tokens, in
    descending score (``torch.topk(scores, C, dim=-1)``).

    The per-expert softmax over tokens is monotone in the logit, so the choice is
    made on the fp32 logits; equal logits go to the lower token index first.
    """
    z = np.asarray(logits32, dtype=np.float32)
    T, E = z.shape
    out = np.zeros((E, C), dtype=np.int32)
    for e in range(E):
        order = np.argsort(-z[:, e].astype(np.float64), kind="stable")
        out[e] = order[:C]
    return out


def expert_choice_forward(x, params: dict, *, capacity_factor: float, act: str,
                          logits=None, tokens: Optional[Sequence[int]] = None):
    """Expert-Choice layer output y[t] = sum over experts e that took t of
    score[e, t] * E_e(x_t): the dispatch mask of P4 ``ExpertChoiceGating``
    (``dispatch_mask.scatter_(1, top_k_indices, top_k_scores)``) applied as the
    gate of each expert's output. A token no expert took gets 0.

    Returns (y [len(tokens) or T, d] fp64, dict(logits, C, idx [E, C], scores [E, C])).
    """
    x = _f64(x)
    if logits is None:
        logits = router_logits(x, params["w_router"], params.get("b_router"),
                               params.get("logit_bias"))
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    C = expert_choice_capacity(capacity_factor, T, E)
    idx = expert_choice_select(logits, C)
    S = expert_choice_scores(logits)
    scores = np.take_along_axis(S, idx.astype(np.int64), axis=1)
    sel = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    pos = np.full(T, -1, dtype=np.int64)
    pos[sel] = np.arange(len(sel))
    y = np.zeros((len(sel), x.shape[1]), dtype=np.float64)
    for e in range(E):
        toks = idx[e].astype(np.int64)
        keep = pos[toks] >= 0
        if not keep.any():
            continue
        w3 = params["w3"][e] if params.get("w3") is not None else None
        b1 = params["b1"][e] if params.get("b1") is not None else None
        b2 = params["b2"][e] if params.get("b2") is not None else None
        out = expert_ffn(x[toks[keep]], act, params["w1"][e], params["w2"][e], w3, b1, b2)
        y[pos[toks[keep]]] += scores[e, keep][:, None] * out
    return y, dict(logits=logits, C=C, idx=idx, scores=scores)


def expert_choice_margin(logits32, C: int) -> np.ndarray:
    """Per expert, the gap between its C-th and (C+1)-th largest fp32 logits (inf
    when C >= T): a choice whose gap is tiny may flip under a different rounding
    of the logits."""
    z = np.asarray(logits32, dtype=np.float64)
    T, E = z.shape
    out = np.full(E, np.inf)
    if C >= T or C <= 0:
        return out
    for e in range(E):
        v = np.sort(z[:, e])[::-1]
        out[e] = v[C - 1] - v[C]
    return out


# ----------------------------------------------------------------- noisy top-k gating
def softplus(v):
    """softplus(v) = log(1 + e^v), fp64 (``F.softplus`` of P4 ``TopKGating``, whose
    default switches to the identity above 20)."""
    v = _f64(v)
    return np.where(v > 20.0, v, np.log1p(np.exp(np.minimum(v, 20.0))))


def noisy_router_logits(x, w_router, w_noise, eps, b_router=None,
                        logit_bias=None) -> np.ndarray:
    """Training-mode logits of P4 ``TopKGating`` (Noisy Top-K Gating):
    z + softplus(x W_noise^T) * eps, with z the plain router logits and eps [T, E]
    the standard normal draws (passed in), exact in fp64, rounded once to fp32."""
    x = _f64(x)
    z = x @ _f64(w_router).T
    if b_router is not None:
        z = z + _f64(b_router)[None, :]
    if logit_bias is not None:
        z = z + _f64(logit_bias)[None, :]
    zn = x @ _f64(w_noise).T
    return (z + softplus(zn) * _f64(eps)).astype(np.float32)


# ------------------------------------------- counter-based noise draws (Philox + Box-Muller)
# The noisy gate of P4 ``TopKGating`` draws ``torch.randn_like`` inside the layer. With
# a seed and an offset instead of a caller's tensor, the draws must be a pure function
# of (seed, offset, token, expert) so that the CUDA path and this oracle produce the
# same numbers: a counter-based generator. Philox4x32-10 is restated here from J. K.
# Salmon, M. A. Moraes, R. O. Dror and D. E. Shaw, "Parallel Random Numbers: As Easy
# as 1, 2, 3" (SC'11), and the normal deviates from its uniforms by the transform of
# G. E. P. Box and M. E. Muller, "A Note on the Generation of Random Normal Deviates"
# (Ann. Math. Statist. 29, 1958).
PHILOX_M0, PHILOX_M1 = 0xD2511F53, 0xCD9E8D57   # round multipliers
PHILOX_W0, PHILOX_W1 = 0x9E3779B9, 0xBB67AE85   # Weyl increments of the key
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32(counter, key, rounds: int = 10) -> np.ndarray:
    """Philox4x32-R: counter [..., 4] and key [..., 2] (uint32) -> [..., 4] uint32.

    One round maps (c0, c1, c2, c3) with key (k0, k1) to
    (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1, lo(M0*c0)), where hi/lo are
    the upper and lower 32 bits of the 64-bit product; the key is advanced by
    (W0, W1) mod 2^32 before every round but the first."""
    counter = np.asarray(counter, dtype=np.uint64)
    key = np.asarray(key, dtype=np.uint64)
    c0, c1, c2, c3 = (counter[..., i] for i in range(4))
    k0, k1 = key[..., 0], key[..., 1]
    for r in range(rounds):
        if r > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK32
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK32
        p0 = c0 * np.uint64(PHILOX_M0)   # < 2^64: exact in uint64
        p1 = c2 * np.uint64(PHILOX_M1)
        c0, c1, c2, c3 = ((p1 >> np.uint64(32)) ^ c1 ^ k0, p1 & _MASK32,
                          (p0 >> np.uint64(32)) ^ c3 ^ k1, p0 & _MASK32)
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def uniform_open(r) -> np.ndarray:
    """A uint32 word to a uniform in (0, 1): u = (2 * (r >> 9) + 1) * 2^-24, an odd
    multiple of 2^-24 (exact in fp32 and fp64; never 0 or 1)."""
    r = np.asarray(r, dtype=np.uint64)
    return ((r >> np.uint64(9)).astype(np.float64) * 2.0 + 1.0) * 2.0 ** -24


def box_muller(u_a, u_b):
    """Two independent standard normals from two uniforms in (0, 1):
    rho = sqrt(-2 ln u_a), (rho cos(2 pi u_b), rho sin(2 pi u_b)), in fp64."""
    rho = np.sqrt(-2.0 * np.log(u_a))
    ang = 2.0 * math.pi * np.asarray(u_b, dtype=np.float64)
    return rho * np.cos(ang), rho * np.sin(ang)


def noise_draws(T: int, E: int, seed: int, offset: int):
    """The noise eps [T, E] of the seeded noisy gate, fp64, and the raw Philox words
    [T, ceil(E/4), 4].

    Token t and expert group q = e // 4 use counter (t, q, offset mod 2^32,
    offset >> 32) and key (seed mod 2^32, seed >> 32); with the four words (r0, r1,
    r2, r3) and u_i = uniform_open(r_i), Box-Muller of (u0, u1) gives experts 4q and
    4q + 1 (cos, then sin) and of (u2, u3) experts 4q + 2 and 4q + 3."""
    Q = (E + 3) // 4
    t = np.arange(T, dtype=np.uint64)[:, None]
    q = np.arange(Q, dtype=np.uint64)[None, :]
    ctr = np.zeros((T, Q, 4), dtype=np.uint64)
    ctr[..., 0] = t
    ctr[..., 1] = q
    ctr[..., 2] = offset & 0xFFFFFFFF
    ctr[..., 3] = (offset >> 32) & 0xFFFFFFFF
    key = np.array([seed & 0xFFFFFFFF, (seed >> 32) & 0xFFFFFFFF], dtype=np.uint64)
    raw = philox4x32(ctr, np.broadcast_to(key, (T, Q, 2)))
    u = uniform_open(raw)
    eps = np.empty((T, Q, 4), dtype=np.float64)
    eps[..., 0], eps[..., 1] = box_muller(u[..., 0], u[..., 1])
    eps[..., 2], eps[..., 3] = box_muller(u[..., 2], u[..., 3])
    return eps.reshape(T, 4 * Q)[:, :E], raw


# ------------------------------------------------- token-sharded routing (several ranks)
def shard_capacity(counts_all, rank: int, cap: Optional[int]):
    """Capacity left to shard `rank` for each expert when the call's T tokens are
    split into consecutive shards: cap minus the (pre-drop) assignments of the earlier
    shards, at least 0 (None: unlimited). counts_all [W, E]. The drop order is then
    the same as for the whole batch in one call (token-major over all tokens)."""
    if cap is None:
        return None
    counts_all = np.asarray(counts_all, dtype=np.int64)
    before = counts_all[:rank].sum(axis=0)
    return np.maximum(0, cap - before)


def dispatch_with_caps(idx, E: int, caps):
    """``dispatch`` with a capacity per expert (token-major, then slot order)."""
    idx = np.asarray(idx)
    T, k = idx.shape
    counts = np.zeros(E, dtype=np.int64)
    rank = np.zeros((T, k), dtype=np.int64)
    kept = np.zeros((T, k), dtype=bool)
    for t in range(T):
        for s in range(k):
            e = int(idx[t, s])
            rank[t, s] = counts[e]
            kept[t, s] = caps is None or counts[e] < caps[e]
            counts[e] += 1
    return counts, rank, kept
