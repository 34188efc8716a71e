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
