"""Pins for the MX block-scaled oracle (oracle/mx_oracle.py).

E2M1: the format's value table; every code round-trips; encoding is the
brute-force nearest value with ties to the even code, saturating at +-6.
E8M0: 2^(code - 127), 255 is NaN.  MX quantisation: exact blocks (element
values times a power of two) come back exactly with their scale; the block
maximum lands in the top binade of the element format; zero blocks; MXFP8
elements agree with torch's float8_e4m3fn cast.  The block-sum GEMM equals
a library matmul of the decoded operands, and an MX FFN with identical
experts equals a dense SwiGLU FFN computed with torch on the same quantised
operands.
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as mo
import oracle.mx_oracle as mx

# the E2M1 format's non-negative values (OCP MX specification, FP4 E2M1)
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_table_and_round_trip():
    assert list(mx.e2m1_values()) == E2M1_TABLE
    assert list(mx.e2m1_decode(np.arange(8, 16))) == [-v for v in E2M1_TABLE]
    codes = np.arange(16)
    np.testing.assert_array_equal(mx.e2m1_encode(mx.e2m1_decode(codes)), codes)


def _brute_e2m1(v):
    best = None
    for c, q in enumerate(E2M1_TABLE):
        d = abs(abs(v) - q)
        if best is None or d < best[0] - 1e-15 or (abs(d - best[0]) <= 1e-15 and c % 2 == 0):
            best = (d, c)
    return best[1] | (8 if np.signbit(v) else 0)


def test_e2m1_encode_brute_force_and_midpoints():
    rng = np.random.default_rng(1)
    vals = np.concatenate([rng.uniform(-6.5, 6.5, 4000),
                           [(a + b) / 2 for a, b in zip(E2M1_TABLE, E2M1_TABLE[1:])],
                           [-(a + b) / 2 for a, b in zip(E2M1_TABLE, E2M1_TABLE[1:])]])
    got = mx.e2m1_encode(vals)
    want = np.array([_brute_e2m1(v) for v in np.minimum(np.maximum(vals, -6.0), 6.0)])
    np.testing.assert_array_equal(got, want)
    # every midpoint goes to the even code
    mids = np.array([(a + b) / 2 for a, b in zip(E2M1_TABLE, E2M1_TABLE[1:])])
    assert np.all(mx.e2m1_encode(mids) % 2 == 0)


def test_e2m1_saturates():
    np.testing.assert_array_equal(mx.e2m1_encode([6.0, 7.0, 1e9, -6.5, -1e9]), [7, 7, 7, 15, 15])


def test_e8m0_codes():
    np.testing.assert_array_equal(mx.e8m0_decode([127, 128, 126, 0, 254]),
                                  [1.0, 2.0, 0.5, 2.0 ** -127, 2.0 ** 127])
    assert np.isnan(mx.e8m0_decode(255))


@pytest.mark.parametrize("elem", ["e2m1", "e4m3"])
def test_mx_exact_blocks_reconstruct(elem):
    rng = np.random.default_rng(2)
    vals = mx.e2m1_values() if elem == "e2m1" else mo.e4m3_values()
    top = vals[-1]
    blocks, scales = [], []
    for b in range(40):
        q = rng.choice(vals, size=32) * rng.choice([-1.0, 1.0], size=32)
        q[rng.integers(32)] = top * rng.choice([-1.0, 1.0])     # the block's max is the format's max
        s = int(rng.integers(-20, 20))
        blocks.append(q * 2.0 ** s)
        scales.append(s + 127)
    a = np.concatenate(blocks)[None, :]
    codes, sc = mx.mx_quantize(a, elem)
    np.testing.assert_array_equal(sc[0], scales)
    np.testing.assert_array_equal(mx.mx_dequantize(codes, sc, elem), a)


@pytest.mark.parametrize("elem,emax,top", [("e2m1", 2, 6.0), ("e4m3", 8, 448.0)])
def test_mx_block_max_in_top_binade(elem, emax, top):
    rng = np.random.default_rng(3)
    a = rng.standard_normal((50, 256)) * np.exp(rng.uniform(-8, 8, size=(50, 1)))
    codes, sc = mx.mx_quantize(a, elem)
    dec = mx.e2m1_decode if elem == "e2m1" else mo.e4m3_decode
    q = np.abs(dec(codes)).reshape(50, 8, 32).max(axis=-1)
    assert np.all(q >= 2.0 ** emax) and np.all(q <= top)
    # scales are powers of two with the block max / X in [2^emax, 2^(emax+1))
    amax = np.abs(a).reshape(50, 8, 32).max(axis=-1)
    r = amax / mx.e8m0_decode(sc)
    assert np.all((r >= 2.0 ** emax) & (r < 2.0 ** (emax + 1)))


def test_mx_zero_block():
    a = np.zeros((1, 64))
    a[0, 40] = 3.0
    codes, sc = mx.mx_quantize(a, "e2m1")
    assert sc[0, 0] == 127 and np.all(codes[0, :32] == 0)
    assert mx.mx_dequantize(codes, sc, "e2m1")[0, 40] == 3.0


def test_mxfp8_elements_match_torch_cast():
    rng = np.random.default_rng(4)
    a = rng.standard_normal((20, 128)) * 3.0
    codes, sc = mx.mx_quantize(a, "e4m3")
    X = np.repeat(mx.e8m0_decode(sc), 32, axis=1)
    ref = torch.from_numpy(np.clip(a / X, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(codes, ref)


def test_block_sum_gemm_equals_decoded_matmul():
    rng = np.random.default_rng(5)
    a = rng.standard_normal((6, 128))
    w = rng.standard_normal((10, 128)) * 0.05
    ac, asc = mx.mx_quantize(a, "e4m3")
    wc, wsc = mx.mx_quantize(w, "e2m1")
    got = mx.mx_dot_blocks(ac, asc, "e4m3", wc, wsc, "e2m1")
    ref = torch.from_numpy(mx.mx_dequantize(ac, asc, "e4m3")) @ torch.from_numpy(mx.mx_dequantize(wc, wsc, "e2m1")).T
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("w_elem", ["e2m1", "e4m3"])
def test_mx_ffn_identical_experts_is_dense(w_elem):
    rng = np.random.default_rng(6)
    T, H, I, E, k = 12, 64, 32, 4, 2
    x = mo.bf16_round(rng.standard_normal((T, H)))
    w13 = rng.standard_normal((2 * I, H)) * 0.1
    w2 = rng.standard_normal((H, I)) * 0.1
    c13, s13 = mx.mx_quantize(w13, w_elem)
    c2, s2 = mx.mx_quantize(w2, w_elem)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    y = mx.ffn_mx(x, ids, [c13] * E, [s13] * E, [c2] * E, [s2] * E, w_elem=w_elem)
    # dense reference with torch on the same quantised operands
    xq = torch.from_numpy(mx.mx_dequantize(*mx.mx_quantize(x, "e4m3"), "e4m3"))
    gu = xq @ torch.from_numpy(mx.mx_dequantize(c13, s13, w_elem)).T
    h = (torch.nn.functional.silu(gu[:, :I]) * gu[:, I:]).float().to(torch.bfloat16).double().numpy()
    hq = torch.from_numpy(mx.mx_dequantize(*mx.mx_quantize(h, "e4m3"), "e4m3"))
    dense = (hq @ torch.from_numpy(mx.mx_dequantize(c2, s2, w_elem)).T).numpy()
    np.testing.assert_allclose(y, np.repeat(dense, k, axis=0), rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("w_elem", ["e2m1", "e4m3"])
def test_mx_layer_with_identical_experts_is_dense(w_elem):
    """Layer level: routing and the combine of MX expert outputs; with every
    expert (routed and shared) identical, out = (sum of the token's weights)
    x the dense FFN, and the routed weights sum to 1."""
    from moe_inputs import mx_weights
    rng = np.random.default_rng(8)
    T, H, I, E, k, S = 10, 64, 32, 6, 2, 1
    x = mo.bf16_round(rng.standard_normal((T, H)))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    c13, s13 = mx_weights(1, 2 * I, H, w_elem, seed=1)
    c2, s2 = mx_weights(1, H, I, w_elem, seed=2)
    out, ids, w = mx.moe_forward_mx(x, logits, k, [c13[0]] * (E + S), [s13[0]] * (E + S), [c2[0]] * (E + S),
                                    [s2[0]] * (E + S), w_elem=w_elem, n_shared=S)
    y1 = mx.ffn_mx(x, np.zeros((T, 1), np.int32), [c13[0]], [s13[0]], [c2[0]], [s2[0]], w_elem=w_elem)
    np.testing.assert_allclose(w[:, :k].astype(np.float64).sum(1), 1.0, atol=1e-6)
    np.testing.assert_allclose(out, y1 * w.astype(np.float64).sum(1, keepdims=True), rtol=1e-9, atol=1e-12)


def test_mx_weight_generator_codes_and_scales():
    from moe_inputs import mx_weights
    c, s = mx_weights(2, 8, 64, "e4m3", seed=3)
    assert c.shape == (2, 8, 64) and s.shape == (2, 8, 2)
    assert not np.any((c & 0x7F) == 0x7F)                 # no NaN codes
    assert set(np.unique(s)) <= {121, 122, 123}
    c4, _ = mx_weights(1, 4, 32, "e2m1", seed=4)
    assert c4.max() <= 15
