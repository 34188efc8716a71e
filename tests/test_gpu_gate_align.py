"""GPU parity of moe_topk_gate and moe_align_sort against the CPU oracle.

Routing and every align&sort output are compared bit-exactly; gate weights
within 1e-6 absolute.  Cases span several CTAs and ragged tails, the
align-only workload (16384 tokens, top-8 of 256, Zipf s=1, block 64) and its
block-size variants, the edge cases (no tokens, one expert, block size 1,
every slot on one expert, E = 1024), out-of-range ids and the bounded
grid-wide wait.
"""
import numpy as np
import pytest
import torch

import mixture_experts_expert_moe_b200 as m
import oracle
from moe_inputs import ALIGN_CONFIG, align_ids

pytestmark = pytest.mark.gpu


def _gate_case(T, E, k, bias, seed, ties=False):
    g = torch.Generator().manual_seed(seed)
    if ties:
        logits = torch.randint(-3, 4, (T, E), generator=g).float()
    else:
        logits = torch.randn(T, E, generator=g)
    b = torch.randn(E, generator=g) if bias else None
    return logits, b


@pytest.mark.parametrize("T,E,k,bias,ties", [
    (64, 8, 2, False, False), (4096, 8, 2, False, False), (2048, 256, 8, False, False),
    (2048, 256, 8, True, False), (1000, 1024, 32, False, False), (300, 33, 5, True, False),
    (50, 7, 7, False, False), (777, 64, 8, False, True), (5, 1, 1, False, False), (0, 16, 4, False, False),
])
def test_topk_gate_parity(cuda_device, T, E, k, bias, ties):
    logits, b = _gate_case(T, E, k, bias, seed=T * 7 + E, ties=ties)
    ids, w = m.topk_gate(logits.to(cuda_device), k, None if b is None else b.to(cuda_device))
    torch.cuda.synchronize()
    ref_ids, ref_w = oracle.topk_gate(logits.numpy(), k, None if b is None else b.numpy())
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    if T:
        assert np.max(np.abs(w.cpu().numpy().astype(np.float64) - ref_w)) <= 1e-6


@pytest.mark.parametrize("T,E,k,n_shared,mode", [
    (2048, 256, 8, 1, "select"), (2048, 256, 8, 0, "select"), (300, 33, 5, 2, "select"),
    (300, 33, 5, 2, "logits"), (64, 8, 2, 3, "logits"), (777, 64, 8, 1, "select"), (40, 1000, 24, 8, "select"),
])
def test_topk_gate_bias_modes_and_shared(cuda_device, T, E, k, n_shared, mode):
    logits, b = _gate_case(T, E, k, True, seed=T * 11 + E + n_shared, ties=False)
    ids, w = m.topk_gate(logits.to(cuda_device), k, b.to(cuda_device), bias_mode=mode, n_shared=n_shared)
    torch.cuda.synchronize()
    ref_ids, ref_w = oracle.topk_gate(logits.numpy(), k, b.numpy(), mode)
    ref_ids, ref_w = oracle.add_shared(ref_ids, ref_w, E, n_shared)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref_ids)
    assert np.max(np.abs(w.cpu().numpy().astype(np.float64) - ref_w)) <= 1e-6


def _align_case(T, k, E, bm, dist, seed):
    if dist == "same":
        return np.zeros((T, k), np.int32) + (E - 1)
    if k > E:
        raise ValueError
    return align_ids(T, E, k, seed=seed, dist=dist)


ALIGN_CASES = [
    (64, 2, 8, 16, "uniform"), (1, 1, 1, 1, "uniform"), (0, 8, 256, 64, "uniform"),
    (100, 8, 256, 64, "zipf"), (ALIGN_CONFIG["T"], 8, 256, 64, "zipf"),
    (ALIGN_CONFIG["T"], 8, 256, 32, "zipf"), (ALIGN_CONFIG["T"], 8, 256, 128, "zipf"),
    (4096, 2, 8, 128, "uniform"), (2048, 8, 256, 64, "uniform"), (3000, 32, 1024, 16, "zipf"),
    (999, 3, 17, 1, "zipf"), (5000, 1, 4, 64, "same"), (262144, 8, 256, 64, "zipf"),
    (1 << 20, 8, 256, 64, "uniform"), (12345, 4, 1000, 7, "zipf"),
]


def _run_align(ids_np, E, bm, dev, fill=-7):
    T, k = ids_np.shape
    P, NB, _ = m.align_sort_sizes(T, k, E, bm)
    out = (torch.full((P,), fill, dtype=torch.int32, device=dev),
           torch.full((NB,), fill, dtype=torch.int32, device=dev),
           torch.full((1,), fill, dtype=torch.int32, device=dev))
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    s, b, n = m.align_sort(torch.from_numpy(ids_np).to(dev), E, bm, dev_status=st, out=out)
    torch.cuda.synchronize()
    return s.cpu().numpy(), b.cpu().numpy(), int(n.item()), int(st.item())


@pytest.mark.parametrize("T,k,E,bm,dist", ALIGN_CASES)
def test_align_sort_bit_exact(cuda_device, T, k, E, bm, dist):
    ids = _align_case(T, k, E, bm, dist, seed=ALIGN_CONFIG["seed"] + T + bm)
    s, b, n, st = _run_align(ids, E, bm, cuda_device)
    assert st == 0
    ref_s, ref_b, ref_n = oracle.align_sort(ids, E, bm)
    assert n == ref_n
    np.testing.assert_array_equal(s[:n], ref_s)
    np.testing.assert_array_equal(b[:n // bm], ref_b)
    # the tails beyond num_post are not written
    assert np.all(s[n:] == -7) and np.all(b[n // bm:] == -7)


def test_align_sort_deterministic(cuda_device):
    ids = align_ids(ALIGN_CONFIG["T"], 256, 8, seed=3, dist="zipf")
    first = _run_align(ids, 256, 64, cuda_device)
    for _ in range(5):
        again = _run_align(ids, 256, 64, cuda_device)
        assert again[2] == first[2]
        np.testing.assert_array_equal(again[0][:first[2]], first[0][:first[2]])


def test_align_sort_flags_out_of_range_ids(cuda_device):
    ids = align_ids(1000, 64, 4, seed=5, dist="uniform")
    ids[3, 1] = 64
    ids[700, 0] = -1
    s, b, n, st = _run_align(ids, 64, 16, cuda_device)
    assert st & m.MOE_DEV_BAD_EXPERT_ID
    # the valid slots are still placed as the oracle places them without the bad ones
    placed = s[:n][s[:n] != ids.size]
    assert 3 * 4 + 1 not in placed and 700 * 4 not in placed
    assert placed.size == ids.size - 2


def test_grid_wait_times_out_cleanly(cuda_device):
    st = m.run_wait_timeout_check(50_000_000)
    assert st & m.MOE_DEV_TIMEOUT
    # the context is still usable afterwards
    ids = align_ids(64, 8, 2, seed=1, dist="uniform")
    s, b, n, st2 = _run_align(ids, 8, 16, cuda_device)
    assert st2 == 0 and n == oracle.align_sort(ids, 8, 16)[2]


@pytest.mark.parametrize("T,k,E,dist", [(200000, 1, 3, "uniform"), (60000, 2, 8, "zipf"), (30000, 4, 5, "zipf")])
def test_align_sort_stable_under_heavy_collisions(cuda_device, T, k, E, dist):
    """Many equal ids per warp step: the stable order inside every segment must
    match the oracle on every one of several runs."""
    ids = align_ids(T, E, k, seed=T + E, dist=dist)
    ref_s, ref_b, ref_n = oracle.align_sort(ids, E, 32)
    for _ in range(4):
        s, b, n, st = _run_align(ids, E, 32, cuda_device)
        assert st == 0 and n == ref_n
        np.testing.assert_array_equal(s[:n], ref_s)
        np.testing.assert_array_equal(b[:n // 32], ref_b)
