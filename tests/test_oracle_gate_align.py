"""Pins for the oracle's gating and align&sort.

Gate: brute force over all k-subsets (the selected set is the one whose every
member beats every non-member, ties to the lower index); the weights equal a
library softmax over the selected logits alone; with k = E they are the full
softmax; a bias is the same as shifting the logits; the selection-only bias
picks by logit + bias and weighs by the raw logits (brute force, a constant
bias, a bias that forces a set of experts).

Align&sort: brute force with Python's ``sorted`` on (expert, slot) pairs and
an explicit segment build; the structural invariants (non-sentinel entries
are a permutation of the slots, one expert per block, non-decreasing block
experts, segments of ceil(c/bm)*bm, ascending slots inside a segment); edge
cases (no tokens, one expert, bm = 1, all slots on one expert).
"""
import itertools

import numpy as np
import pytest
import scipy.special

import oracle.moe_oracle as mo
from moe_inputs import align_ids


def _brute_topk(row, k):
    E = len(row)
    for S in itertools.combinations(range(E), k):
        rest = [u for u in range(E) if u not in S]
        if all(row[s] > row[u] or (row[s] == row[u] and s < u) for s in S for u in rest):
            return sorted(S, key=lambda e: (-row[e], e))
    raise AssertionError("no dominating subset")


@pytest.mark.parametrize("E,k", [(4, 1), (6, 2), (8, 3), (8, 8), (7, 5)])
def test_gate_brute_force_with_ties(E, k):
    rng = np.random.default_rng(E * 10 + k)
    # integer-valued logits make ties common
    logits = rng.integers(-3, 4, size=(200, E)).astype(np.float32)
    ids, w = mo.topk_gate(logits, k)
    for t in range(logits.shape[0]):
        assert list(ids[t]) == _brute_topk(list(logits[t]), k)
        ref = scipy.special.softmax(logits[t, ids[t]].astype(np.float64))
        np.testing.assert_allclose(w[t], ref, rtol=1e-6, atol=1e-7)


def test_gate_k_equals_E_is_full_softmax():
    rng = np.random.default_rng(3)
    logits = rng.standard_normal((50, 16)).astype(np.float32)
    ids, w = mo.topk_gate(logits, 16)
    full = scipy.special.softmax(logits.astype(np.float64), axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(full, ids.astype(np.int64), 1), rtol=1e-6)
    assert np.all(np.diff(np.take_along_axis(logits, ids.astype(np.int64), 1), axis=1) <= 0)


def test_gate_weights_sum_to_one_and_bias_shift():
    rng = np.random.default_rng(4)
    logits = rng.standard_normal((300, 256)).astype(np.float32)
    bias = rng.standard_normal(256).astype(np.float32)
    ids, w = mo.topk_gate(logits, 8, bias)
    np.testing.assert_allclose(w.astype(np.float64).sum(1), 1.0, atol=1e-6)
    assert all(len(set(r)) == 8 for r in ids)
    ids2, w2 = mo.topk_gate((logits + bias[None]).astype(np.float32), 8)
    np.testing.assert_array_equal(ids, ids2)
    np.testing.assert_array_equal(w, w2)


@pytest.mark.parametrize("E,k", [(6, 2), (8, 3), (8, 8)])
def test_gate_bias_modes_brute_force(E, k):
    """Both bias modes select by brute force on logit + bias; "logits" weighs
    the chosen experts by a softmax of logit + bias, "select" by a softmax of
    the raw logits (library softmax over the chosen entries only)."""
    rng = np.random.default_rng(100 + E * 10 + k)
    logits = rng.integers(-3, 4, size=(150, E)).astype(np.float32)
    bias = rng.integers(-2, 3, size=E).astype(np.float32)
    score = logits + bias[None]
    for mode in ("logits", "select"):
        ids, w = mo.topk_gate(logits, k, bias, mode)
        for t in range(logits.shape[0]):
            assert list(ids[t]) == _brute_topk(list(score[t]), k)
            src = score[t] if mode == "logits" else logits[t]
            ref = scipy.special.softmax(src[ids[t]].astype(np.float64))
            np.testing.assert_allclose(w[t], ref, rtol=1e-6, atol=1e-7)


def test_gate_select_bias_constant_and_zero():
    """A bias equal for every expert changes nothing in "select" mode (and in
    "logits" mode the shift cancels in the softmax); a zero bias is no bias."""
    rng = np.random.default_rng(5)
    logits = rng.standard_normal((200, 64)).astype(np.float32)
    ids0, w0 = mo.topk_gate(logits, 6)
    for mode in ("select", "logits"):
        ids, w = mo.topk_gate(logits, 6, np.zeros(64, np.float32), mode)
        np.testing.assert_array_equal(ids, ids0)
        np.testing.assert_array_equal(w, w0)
    ids, w = mo.topk_gate(logits, 6, np.full(64, 0.5, np.float32), "select")
    np.testing.assert_array_equal(ids, ids0)
    np.testing.assert_allclose(w, w0, rtol=1e-6)


def test_gate_select_bias_steers_only_selection():
    """A large bias on a fixed set of k experts makes exactly that set the
    choice (ordered by logit + bias) while the weights stay the softmax of the
    raw logits of those experts."""
    rng = np.random.default_rng(6)
    E, k = 32, 4
    logits = rng.standard_normal((100, E)).astype(np.float32)
    favour = np.array([3, 11, 17, 29])
    bias = np.zeros(E, np.float32)
    bias[favour] = 1000.0 + np.arange(4, dtype=np.float32)
    ids, w = mo.topk_gate(logits, k, bias, "select")
    for t in range(100):
        assert sorted(ids[t]) == sorted(favour)
        ref = scipy.special.softmax(logits[t, ids[t]].astype(np.float64))
        np.testing.assert_allclose(w[t], ref, rtol=1e-6, atol=1e-7)


def test_add_shared_layout():
    ids = np.array([[3, 1], [0, 2]], np.int32)
    w = np.array([[0.7, 0.3], [0.6, 0.4]], np.float32)
    ids2, w2 = mo.add_shared(ids, w, 4, 2)
    np.testing.assert_array_equal(ids2, [[3, 1, 4, 5], [0, 2, 4, 5]])
    np.testing.assert_array_equal(w2, np.array([[0.7, 0.3, 1, 1], [0.6, 0.4, 1, 1]], np.float32))


def _brute_align(ids_flat, E, bm):
    N = len(ids_flat)
    pairs = sorted((int(e), i) for i, e in enumerate(ids_flat))
    out, blocks = [], []
    for e in range(E):
        seg = [i for (ee, i) in pairs if ee == e]
        n_blk = (len(seg) + bm - 1) // bm
        seg = seg + [N] * (n_blk * bm - len(seg))
        out += seg
        blocks += [e] * n_blk
    return out, blocks


@pytest.mark.parametrize("T,k,E,bm", [(5, 2, 4, 4), (9, 3, 5, 2), (16, 1, 3, 8),
                                      (7, 4, 8, 1), (1, 1, 1, 16), (12, 2, 6, 3)])
def test_align_brute_force(T, k, E, bm):
    rng = np.random.default_rng(T * 1000 + E)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    s, b, n = mo.align_sort(ids, E, bm)
    ref_s, ref_b = _brute_align(ids.reshape(-1), E, bm)
    assert n == len(ref_s)
    assert list(s) == ref_s and list(b) == ref_b


def check_align_invariants(ids, E, bm, s, b, n):
    flat = np.asarray(ids).reshape(-1)
    N = flat.size
    assert n % bm == 0 and len(s) == n and len(b) == n // bm
    real = s[s != N]
    assert np.array_equal(np.sort(real), np.arange(N))
    assert (s == N).sum() == n - N
    assert np.all(np.diff(b) >= 0)
    counts = np.bincount(flat, minlength=E)
    for e in range(E):
        blk = np.nonzero(b == e)[0]
        assert blk.size * bm == -(-counts[e] // bm) * bm
        if blk.size:
            seg = s[blk[0] * bm:(blk[-1] + 1) * bm]
            body = seg[seg != N]
            assert np.all(flat[body] == e)
            assert np.all(np.diff(body) > 0)             # stable
            assert np.all(seg[body.size:] == N)          # padding at the tail
    T, k = np.asarray(ids).shape
    P, NB = mo.expected_sizes(T, k, E, bm)
    assert n <= P and n // bm <= NB


@pytest.mark.parametrize("dist", ["zipf", "uniform"])
def test_align_invariants_generated(dist):
    ids = align_ids(2048, 256, 8, seed=7, dist=dist)
    s, b, n = mo.align_sort(ids, 256, 64)
    check_align_invariants(ids, 256, 64, s, b, n)


def test_align_edge_cases():
    s, b, n = mo.align_sort(np.zeros((0, 8), np.int32), 256, 64)
    assert n == 0 and s.size == 0 and b.size == 0
    ids = np.zeros((10, 1), np.int32)                   # everything on expert 0
    s, b, n = mo.align_sort(ids, 4, 4)
    assert n == 12 and list(s) == list(range(10)) + [10, 10] and list(b) == [0, 0, 0]
    ids = np.arange(6, dtype=np.int32).reshape(3, 2) % 3
    s, b, n = mo.align_sort(ids, 3, 1)                  # bm = 1: no padding
    assert n == 6 and list(b) == [0, 0, 1, 1, 2, 2] and list(s) == [0, 3, 1, 4, 2, 5]
    with pytest.raises(ValueError):
        mo.align_sort(np.array([[5]], np.int32), 4, 4)


def test_planted_unstable_sort_is_caught(monkeypatch):
    """An align that breaks the stable order (planted in the oracle) fails the brute-force pin."""
    orig = np.argsort

    def unstable(a, *args, **kw):
        kw["kind"] = "quicksort"
        r = orig(a, *args, **kw)
        return r[::-1] if np.ndim(a) == 1 else r

    monkeypatch.setattr(mo.np, "argsort", unstable)
    ids = np.array([[0, 1], [0, 1], [1, 0]], np.int32)
    s, b, n = mo.align_sort(ids, 2, 4)
    monkeypatch.undo()
    ref_s, _ = _brute_align(ids.reshape(-1), 2, 4)
    assert list(s) != ref_s
