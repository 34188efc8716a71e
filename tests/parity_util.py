"""Comparison helpers shared by the GPU parity tests."""
import numpy as np

# tolerances of the MoE layer forward (max-abs, relative Frobenius)
TOL_BF16 = (2e-2, 1e-2)
TOL_FP8 = (5e-2, 3e-2)


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    if got.size == 0:
        return 0.0, 0.0
    d = got - ref
    max_abs = float(np.max(np.abs(d)))
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(d) / den) if den > 0 else float(np.linalg.norm(d))
    return max_abs, rel


def assert_close(got, ref, tol, what=""):
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), f"{what}: non-finite output"
    max_abs, rel = errors(got, ref)
    assert max_abs <= tol[0] and rel <= tol[1], (
        f"{what}: max abs {max_abs:.3e} (limit {tol[0]}), rel fro {rel:.3e} (limit {tol[1]})")
    return max_abs, rel


def assert_close_scaled(got, ref, tol, what=""):
    """assert_close with the max-abs bar taken relative to the output's scale:
    |got - ref| <= tol[0] * max(1, max |ref|) (the relative Frobenius bar is
    unchanged).  For gradients summed over many tokens, whose entries grow with
    the sum while their bf16 operands keep 8 significant bits, an absolute bar
    meant for outputs of order 1 would be tighter than one bf16 ulp."""
    scale = max(1.0, float(np.max(np.abs(np.asarray(ref, dtype=np.float64)))) if np.size(ref) else 1.0)
    return assert_close(got, ref, (tol[0] * scale, tol[1]), what)


def bf16_ulp(v):
    """Spacing of bfloat16 values at |v| (normal range)."""
    a = np.maximum(np.abs(np.asarray(v, dtype=np.float64)), 2.0 ** -126)
    return np.ldexp(1.0, (np.floor(np.log2(a)) - 7).astype(np.int64))


class ExpertView:
    """Lazy per-expert float64 (or code) view of a torch weight tensor, so the
    oracle converts one expert at a time."""

    def __init__(self, t, codes=False):
        self.t = t
        self.codes = codes
        self.shape = tuple(t.shape)

    def __getitem__(self, e):
        x = self.t[int(e)].cpu()
        if self.codes:
            return x.view(__import__("torch").uint8).numpy()
        return x.float().numpy().astype(np.float64)


def cover_sample(ids, n_hot=8, group_rows=(64, 128, 256)):
    """Tokens whose outputs a full-size parity test compares, chosen from a
    routing table ``ids`` [T, k] (the oracle's): the first and last token; a
    greedy cover that reaches every expert in ``ids``; and, for the ``n_hot``
    most loaded experts, the tokens of the last slot and of the first slot of
    the last token group of each size in ``group_rows``.

    Returns (sorted token indices, experts the sample reaches, experts touched).
    """
    ids = np.asarray(ids, dtype=np.int64)
    T, k = ids.shape
    chosen = {0, T - 1}
    flat = ids.reshape(-1)
    touched = np.unique(flat)
    counts = np.bincount(flat, minlength=int(flat.max()) + 1)
    for e in np.argsort(-counts, kind="stable")[:n_hot]:
        slots = np.nonzero(flat == e)[0]          # ascending: the order inside the expert's segment
        if slots.size == 0:
            continue
        chosen.add(int(slots[-1] // k))
        for g in group_rows:
            chosen.add(int(slots[((slots.size - 1) // g) * g] // k))
    covered = set(flat[np.isin(np.arange(T * k) // k, list(chosen))].tolist())
    member = np.zeros((T, counts.size), dtype=bool)
    member[np.repeat(np.arange(T), k), flat] = True
    missing = np.ones(counts.size, dtype=bool)
    missing[list(covered)] = False
    missing &= counts > 0
    while missing.any():
        gain = member[:, missing].sum(axis=1)
        t = int(np.argmax(gain))
        chosen.add(t)
        missing &= ~member[t]
        covered.update(np.nonzero(member[t])[0].tolist())
    toks = np.array(sorted(chosen), dtype=np.int64)
    reached = np.unique(ids[toks].reshape(-1)).size
    return toks, int(reached), int(touched.size)
