"""Property-based pins of the oracle (hypothesis): align & sort and gating
against brute force over random small shapes, including repeated ids,
tied logits, both bias modes and shared experts."""
import numpy as np
import scipy.special
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle.moe_oracle as mo
from test_oracle_gate_align import _brute_align, _brute_topk


@st.composite
def _align_case(draw):
    E = draw(st.integers(1, 9))
    k = draw(st.integers(1, min(E, 4)))
    T = draw(st.integers(0, 12))
    bm = draw(st.integers(1, 8))
    rows = [draw(st.permutations(range(E)))[:k] for _ in range(T)]
    ids = np.array(rows, dtype=np.int32).reshape(T, k)
    return ids, E, bm


@settings(max_examples=150, deadline=None)
@given(_align_case())
def test_align_matches_brute_force(case):
    ids, E, bm = case
    s, b, n = mo.align_sort(ids, E, bm)
    ref_s, ref_b = _brute_align(ids.reshape(-1), E, bm)
    assert n == len(ref_s) and list(s[:n]) == ref_s and list(b[:n // bm]) == ref_b
    P, NB = mo.expected_sizes(ids.shape[0], ids.shape[1], E, bm)
    assert n <= P and n // bm <= NB


@st.composite
def _gate_case(draw):
    E = draw(st.integers(1, 8))
    k = draw(st.integers(1, E))
    T = draw(st.integers(1, 6))
    vals = st.integers(-3, 3)           # small integers: ties are common
    logits = np.array([[draw(vals) for _ in range(E)] for _ in range(T)], dtype=np.float32)
    bias = np.array([draw(vals) for _ in range(E)], dtype=np.float32) if draw(st.booleans()) else None
    mode = draw(st.sampled_from(["logits", "select"]))
    S = draw(st.integers(0, 2))
    return logits, k, bias, mode, S


@settings(max_examples=150, deadline=None)
@given(_gate_case())
def test_gate_matches_brute_force(case):
    logits, k, bias, mode, S = case
    E = logits.shape[1]
    ids, w = mo.topk_gate(logits, k, bias, mode)
    if S:
        ids, w = mo.add_shared(ids, w, E, S)
    score = logits + (bias[None] if bias is not None else 0)
    for t in range(logits.shape[0]):
        assert list(ids[t, :k]) == _brute_topk(list(score[t]), k)
        src = score[t] if (mode == "logits") else logits[t]
        ref = scipy.special.softmax(src[ids[t, :k]].astype(np.float64))
        np.testing.assert_allclose(w[t, :k], ref, rtol=1e-6, atol=1e-7)
        assert list(ids[t, k:]) == list(range(E, E + S)) and np.all(w[t, k:] == 1.0)
