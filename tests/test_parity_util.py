"""Host logic of the full-size parity sample (CPU)."""
import numpy as np

from parity_util import cover_sample


def test_cover_sample_reaches_every_expert_and_the_hot_tails():
    rng = np.random.default_rng(3)
    T, E, k = 500, 40, 4
    p = 1.0 / np.arange(1, E + 1)
    ids = np.stack([rng.choice(E, size=k, replace=False, p=p / p.sum()) for _ in range(T)])
    toks, reached, touched = cover_sample(ids, n_hot=3, group_rows=(16,))
    assert reached == touched == np.unique(ids).size
    assert toks[0] == 0 and toks[-1] == T - 1 and np.all(np.diff(toks) > 0)
    flat = ids.reshape(-1)
    for e in np.argsort(-np.bincount(flat, minlength=E), kind="stable")[:3]:
        slots = np.nonzero(flat == e)[0]
        assert slots[-1] // k in toks                               # last slot of a hot expert
        assert slots[((slots.size - 1) // 16) * 16] // k in toks    # first slot of its last 16-row group


def test_cover_sample_single_token():
    toks, reached, touched = cover_sample(np.array([[3, 1, 2]]))
    assert list(toks) == [0] and reached == touched == 3


def test_pack_e2m1_layout_numpy_and_torch():
    import torch
    from moe_inputs import mx_weights, pack_e2m1
    codes, scales = mx_weights(2, 4, 64, "e2m1", seed=3)
    p = pack_e2m1(codes)
    assert p.shape == (2, 4, 32)
    assert np.array_equal(p & 0xF, codes[..., 0::2]) and np.array_equal(p >> 4, codes[..., 1::2])
    assert np.array_equal(pack_e2m1(torch.from_numpy(codes)).numpy(), p)
    tc, ts = mx_weights(2, 4, 64, "e4m3", seed=3, device="cpu")
    assert tc.dtype == torch.uint8 and ts.shape == (2, 4, 2)
    assert not bool(((tc & 0x7F) == 0x7F).any())        # no NaN codes
    assert int(ts.min()) >= 121 and int(ts.max()) <= 123


def test_scaled_tolerance_follows_the_output_scale():
    import pytest
    from parity_util import assert_close_scaled
    ref = np.array([100.0, -50.0, 1.0])
    assert_close_scaled(ref + 1.5, ref, (2e-2, 1.0))           # 1.5 <= 2e-2 * 100
    with pytest.raises(AssertionError):
        assert_close_scaled(ref + 2.5, ref, (2e-2, 1.0))
    small = np.array([0.5, -0.25])
    with pytest.raises(AssertionError):
        assert_close_scaled(small + 0.03, small, (2e-2, 1.0))  # scale floor 1: bar stays 2e-2
