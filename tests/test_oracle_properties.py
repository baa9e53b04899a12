"""Randomised properties of the CPU oracle (hypothesis): invariants that must hold
for every small configuration, beyond the fixed pins. No GPU needed."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle import moe_oracle as O

MODES = ("topk_softmax", "softmax_topk_renorm", "softmax_topk_raw")


@st.composite
def routing_case(draw):
    T = draw(st.integers(1, 24))
    E = draw(st.integers(1, 9))
    k = draw(st.integers(1, min(E, 8)))
    grid = draw(st.booleans())  # a coarse grid makes exact ties likely
    seed = draw(st.integers(0, 2 ** 31 - 1))
    z = np.random.default_rng(seed).normal(size=(T, E)) * 2
    if grid:
        z = np.round(z * 2) / 2
    return z.astype(np.float32), k


@settings(max_examples=60, deadline=None)
@given(routing_case(), st.sampled_from(MODES))
def test_topk_and_gates(case, mode):
    z, k = case
    T, E = z.shape
    idx = O.select_topk(z, k)
    # k distinct experts per token, in descending logit, ties to the lower index
    for t in range(T):
        row = list(idx[t])
        assert len(set(row)) == k
        for a, b in zip(row, row[1:]):
            assert z[t, a] > z[t, b] or (z[t, a] == z[t, b] and a < b)
        worst = row[-1]
        for e in range(E):
            if e not in row:
                assert z[t, e] < z[t, worst] or (z[t, e] == z[t, worst] and e > worst)
    g = O.gate_values(z, idx, mode)
    assert np.all(g >= 0) and np.all(g <= 1 + 1e-12)
    if mode != "softmax_topk_raw":
        assert np.allclose(g.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    else:
        assert np.all(g.sum(axis=1) <= 1 + 1e-12)
    # within a token, gates follow the logits' order
    assert np.all(np.diff(g, axis=1) <= 1e-12)


@settings(max_examples=60, deadline=None)
@given(routing_case(), st.floats(0.1, 3.0))
def test_capacity_drops(case, cf):
    z, k = case
    T, E = z.shape
    idx = O.select_topk(z, k)
    cap = O.capacity(cf, T, k, E)
    counts, rank, kept = O.dispatch(idx, E, cap)
    assert counts.sum() == T * k
    for e in range(E):
        mine = idx == e
        assert int(mine.sum()) == counts[e]
        assert int((mine & kept).sum()) == min(counts[e], cap)
        # the kept ones are exactly the first `cap` in token-major order
        r = np.sort(rank[mine])
        assert np.array_equal(r, np.arange(counts[e]))
        assert np.all(kept[mine] == (rank[mine] < cap))
    offsets, perm, inv = O.expert_layout(idx, rank, kept, E)
    assert offsets[-1] == int(kept.sum())
    assert np.all(np.diff(offsets) >= 0)
    for t in range(T):
        for s in range(k):
            if kept[t, s]:
                assert perm[inv[t, s]] == t
            else:
                assert inv[t, s] == -1


@settings(max_examples=60, deadline=None)
@given(st.integers(1, 40), st.integers(1, 9), st.floats(0.05, 4.0), st.booleans(),
       st.integers(0, 2 ** 31 - 1))
def test_expert_choice_picks(T, E, cf, grid, seed):
    C = O.expert_choice_capacity(cf, T, E)
    if C < 1 or C > T:
        return
    z = np.random.default_rng(seed).normal(size=(T, E)) * 2
    if grid:
        z = np.round(z * 2) / 2
    z = z.astype(np.float32)
    idx = O.expert_choice_select(z, C)
    S = O.expert_choice_scores(z)
    assert np.allclose(S.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    for e in range(E):
        picks = list(idx[e])
        assert len(set(picks)) == C  # C distinct tokens per expert
        for a, b in zip(picks, picks[1:]):
            assert z[a, e] > z[b, e] or (z[a, e] == z[b, e] and a < b)
        last = picks[-1]
        for t in range(T):
            if t not in picks:
                assert z[t, e] < z[last, e] or (z[t, e] == z[last, e] and t > last)
        # the scores of the picks are the largest of the expert's column
        taken = S[e, picks]
        rest = np.delete(S[e], picks)
        assert rest.size == 0 or taken.min() >= rest.max()
