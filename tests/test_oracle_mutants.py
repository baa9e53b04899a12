"""Plant plausible mistakes in the CPU oracle and confirm the pins catch each one.

Every mutant replaces one oracle function with a subtly wrong version (a dropped
term, a wrong index, a swapped operand, a wrong normaliser). The pins must fail
for every mutant; a mutant that survives means a pin is missing.
"""
import math

import numpy as np
import pytest

from oracle import moe_oracle as O
from tests import oracle_pins as pins

_orig = {name: getattr(O, name) for name in dir(O) if callable(getattr(O, name))}


def _topk_ties_high(logits32, k):
    z = np.asarray(logits32, dtype=np.float32).astype(np.float64)
    E = z.shape[1]
    order = np.argsort(-z[:, ::-1], axis=1, kind="stable")
    return (E - 1 - order[:, :k]).astype(np.int32)


def _gates_no_renorm(logits32, idx, mode):
    g = _orig["gate_values"](logits32, idx, "softmax_topk_raw")
    return g if mode != "softmax_topk_raw" else g


def _gates_modeA_full_softmax(logits32, idx, mode):
    if mode == "topk_softmax":
        return _orig["gate_values"](logits32, idx, "softmax_topk_raw")
    return _orig["gate_values"](logits32, idx, mode)


def _capacity_no_k(cf, T, k, E):
    return _orig["capacity"](cf, T, 1, E)


def _dispatch_keep_last(idx, E, cap):
    counts, rank, kept = _orig["dispatch"](idx, E, None)
    if cap is not None:
        for e in range(E):
            kept[idx == e] = rank[idx == e] >= counts[e] - cap
    return counts, rank, kept


def _gelu_tanh(v):
    return 0.5 * v * (1 + np.tanh(math.sqrt(2 / math.pi) * (v + 0.044715 * v ** 3)))


def _ffn_swapped_gate_up(x_rows, act, w1, w2, w3=None, b1=None, b2=None):
    if act == "swiglu":
        return _orig["expert_ffn"](x_rows, act, w3, w2, w1, b1, b2)
    return _orig["expert_ffn"](x_rows, act, w1, w2, w3, b1, b2)


def _ffn_no_b2(x_rows, act, w1, w2, w3=None, b1=None, b2=None):
    return _orig["expert_ffn"](x_rows, act, w1, w2, w3, b1, None)


def _ffn_transposed_down(x_rows, act, w1, w2, w3=None, b1=None, b2=None):
    w2 = np.asarray(w2)
    if w2.shape[0] == w2.shape[1]:
        w2 = w2.T
    else:
        w2 = w2.T.reshape(w2.shape)
    return _orig["expert_ffn"](x_rows, act, w1, w2, w3, b1, b2)


def _logits_no_bias(x, w_router, b_router=None, logit_bias=None):
    return _orig["router_logits"](x, w_router, None, logit_bias)


def _aux_f_over_T(logits32, idx, E, top_k, alpha):
    f, P, aux = _orig["aux_stats"](logits32, idx, E, top_k, alpha)
    f = f * top_k
    return f, P, alpha * E * float((f * P).sum())


def _shared_dropped(x, ws_gate, ws_up, ws_down, n_shared):
    return np.zeros((x.shape[0], ws_down.shape[0]))


def _silu_sign(v):
    return v / (1.0 + np.exp(v))


def _layout_reverse(idx, rank, kept, E):
    offsets, perm, inv = _orig["expert_layout"](idx, rank, kept, E)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        perm[a:b] = perm[a:b][::-1].copy()
    return offsets, perm, inv


def _combine_ignores_gates(y_rows, inv, gates, shared=None):
    return _orig["combine"](y_rows, inv, np.ones_like(np.asarray(gates, dtype=float)), shared)


def _ec_softmax_over_experts(logits32):
    z = np.asarray(logits32, dtype=np.float64)
    e = np.exp(z - z.max(axis=1, keepdims=True))
    return (e / e.sum(axis=1, keepdims=True)).T


def _ec_ties_to_higher_token(logits32, C):
    z = np.asarray(logits32, dtype=np.float32)
    T, E = z.shape
    out = np.zeros((E, C), dtype=np.int32)
    for e in range(E):
        order = np.argsort(-z[::-1, e].astype(np.float64), kind="stable")
        out[e] = (T - 1 - order)[:C]
    return out


def _ec_capacity_rounds_up(cf, T, E):
    return int(np.ceil(float(cf) * T / E))


def _ec_forward_ignores_scores(x, params, *, capacity_factor, act, logits=None, tokens=None):
    orig = _orig["expert_choice_scores"]
    O.expert_choice_scores = lambda z: np.ones_like(orig(z))
    try:
        return _orig["expert_choice_forward"](x, params, capacity_factor=capacity_factor,
                                              act=act, logits=logits, tokens=tokens)
    finally:
        O.expert_choice_scores = orig


def _softplus_is_exp(v):
    return np.exp(np.asarray(v, dtype=np.float64))


def _noise_sign_flipped(x, w_router, w_noise, eps, b_router=None, logit_bias=None):
    return _orig["noisy_router_logits"](x, w_router, w_noise, -np.asarray(eps), b_router,
                                        logit_bias)


def _shard_capacity_ignores_earlier(counts_all, rank, cap):
    return _orig["shard_capacity"](counts_all, 0, cap)


def _philox_nine_rounds(counter, key, rounds=10):
    return _orig["philox4x32"](counter, key, rounds - 1)


def _philox_key_not_advanced(counter, key, rounds=10):
    c = [np.asarray(counter, dtype=np.uint64)[..., i] for i in range(4)]
    k0, k1 = (np.asarray(key, dtype=np.uint64)[..., i] for i in range(2))
    m = np.uint64(0xFFFFFFFF)
    for _ in range(rounds):
        p0 = c[0] * np.uint64(O.PHILOX_M0)
        p1 = c[2] * np.uint64(O.PHILOX_M1)
        c = [(p1 >> np.uint64(32)) ^ c[1] ^ k0, p1 & m, (p0 >> np.uint64(32)) ^ c[3] ^ k1,
             p0 & m]
    return np.stack(c, axis=-1).astype(np.uint32)


def _box_muller_without_two(u_a, u_b):
    rho = np.sqrt(-np.log(u_a))
    ang = 2.0 * math.pi * np.asarray(u_b, dtype=np.float64)
    return rho * np.cos(ang), rho * np.sin(ang)


def _box_muller_one_uniform(u_a, u_b):
    return _orig["box_muller"](u_a, u_a)


def _uniform_includes_zero(r):
    return (np.asarray(r, dtype=np.uint64) >> np.uint64(8)).astype(np.float64) * 2.0 ** -24


MUTANTS = {
    "philox_nine_rounds": ("philox4x32", _philox_nine_rounds),
    "philox_key_not_advanced": ("philox4x32", _philox_key_not_advanced),
    "box_muller_without_factor_two": ("box_muller", _box_muller_without_two),
    "box_muller_one_uniform_for_both": ("box_muller", _box_muller_one_uniform),
    "uniform_includes_zero": ("uniform_open", _uniform_includes_zero),
    "shard_capacity_ignores_earlier_shards": ("shard_capacity", _shard_capacity_ignores_earlier),
    "softplus_is_exp": ("softplus", _softplus_is_exp),
    "noise_sign_flipped": ("noisy_router_logits", _noise_sign_flipped),
    "ec_softmax_over_experts": ("expert_choice_scores", _ec_softmax_over_experts),
    "ec_ties_to_higher_token": ("expert_choice_select", _ec_ties_to_higher_token),
    "ec_capacity_rounds_up": ("expert_choice_capacity", _ec_capacity_rounds_up),
    "ec_output_ignores_scores": ("expert_choice_forward", _ec_forward_ignores_scores),
    "combine_ignores_gates": ("combine", _combine_ignores_gates),
    "topk_ties_to_higher_index": ("select_topk", _topk_ties_high),
    "gates_not_renormalised": ("gate_values", _gates_no_renorm),
    "modeA_softmax_over_all_experts": ("gate_values", _gates_modeA_full_softmax),
    "capacity_without_k": ("capacity", _capacity_no_k),
    "drop_keeps_last_tokens": ("dispatch", _dispatch_keep_last),
    "gelu_tanh_approximation": ("gelu", _gelu_tanh),
    "swiglu_gate_up_swapped": ("expert_ffn", _ffn_swapped_gate_up),
    "mlp_second_bias_dropped": ("expert_ffn", _ffn_no_b2),
    "down_projection_transposed": ("expert_ffn", _ffn_transposed_down),
    "router_bias_dropped": ("router_logits", _logits_no_bias),
    "aux_f_normalised_by_T": ("aux_stats", _aux_f_over_T),
    "shared_experts_not_added": ("shared_experts", _shared_dropped),
    "silu_sign_flipped": ("silu", _silu_sign),
    "layout_rows_reversed": ("expert_layout", _layout_reverse),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for check in pins.ALL_CHECKS:
        try:
            check(O)
        except Exception:  # an assertion, or a shape error from a transposed operand
            failed.append(check.__name__)
    assert failed, f"mutant {name} survived every pin"
