"""moe_align_sort_noalloc: the align&sort entry point for callers that cannot
allocate device memory (it uses a fixed scratch array inside the library
instead of a caller workspace).

Its outputs must equal those of moe_align_sort (bit-exact, the bar for index
outputs) on two calls in a row, since the second call reuses the scratch the
first one left behind.  This file is collected last on purpose: the entry
point's first call on a device performs its one-time set-up, and the test
must pass both alone in a fresh process and after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import mixture_experts_expert_moe_b200 as m
from moe_inputs import ALIGN_CONFIG, align_ids


def _noalloc(lib, ids, E, bm, dev, with_status=True):
    T, k = ids.shape
    P, NB, _ = m.align_sort_sizes(T, k, E, bm)
    s = torch.full((max(P, 1),), -7, dtype=torch.int32, device=dev)
    b = torch.full((max(NB, 1),), -7, dtype=torch.int32, device=dev)
    n = torch.full((1,), -7, dtype=torch.int32, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    rc = lib.moe_align_sort_noalloc(ctypes.c_void_p(ids.data_ptr()) if ids.numel() else None, T, k, E, bm,
                                    ctypes.c_void_p(s.data_ptr()), ctypes.c_void_p(b.data_ptr()),
                                    ctypes.c_void_p(n.data_ptr()),
                                    ctypes.c_void_p(st.data_ptr()) if with_status else None, stream)
    assert rc == 0, lib.moe_status_string(rc)
    torch.cuda.synchronize()
    return s.cpu().numpy(), b.cpu().numpy(), int(n.item()), int(st.item())


def _regular(ids, E, bm):
    s, b, n = m.align_sort(ids, E, bm)
    torch.cuda.synchronize()
    return s.cpu().numpy(), b.cpu().numpy(), int(n.item())


@pytest.mark.gpu
def test_noalloc_matches_align_sort_twice(cuda_device):
    lib = m.load_library()
    cases = [
        (align_ids(ALIGN_CONFIG["T"], 256, 8, seed=ALIGN_CONFIG["seed"], dist="zipf"), 256, 64),
        (align_ids(3000, 64, 4, seed=11, dist="uniform"), 64, 16),
    ]
    for ids_np, E, bm in cases:          # two calls in a row, different shapes
        ids = torch.from_numpy(ids_np).to(cuda_device)
        s, b, n, st = _noalloc(lib, ids, E, bm, cuda_device)
        rs, rb, rn = _regular(ids, E, bm)
        assert st == 0
        assert n == rn
        np.testing.assert_array_equal(s[:n], rs[:n])
        np.testing.assert_array_equal(b[:n // bm], rb[:n // bm])
    # and the first shape once more, after the scratch held the second call's data
    ids_np, E, bm = cases[0]
    ids = torch.from_numpy(ids_np).to(cuda_device)
    s, b, n, st = _noalloc(lib, ids, E, bm, cuda_device)
    rs, rb, rn = _regular(ids, E, bm)
    assert st == 0 and n == rn
    np.testing.assert_array_equal(s[:n], rs[:n])
    np.testing.assert_array_equal(b[:n // bm], rb[:n // bm])


def test_noalloc_rejects_more_experts_than_its_scratch():
    lib = m.load_library()
    # E beyond the built-in limit is refused before any device work
    assert lib.moe_align_sort_noalloc(None, 0, 1, 257, 16, ctypes.c_void_p(16), ctypes.c_void_p(16),
                                      ctypes.c_void_p(16), None, None) == 2


@pytest.mark.gpu
def test_noalloc_small_empty_and_without_status(cuda_device):
    """A batch small enough for one CTA (the count matrix in the scratch is
    then not used), an empty batch, and a call without a status word."""
    lib = m.load_library()
    small = torch.from_numpy(align_ids(64, 8, 2, seed=5, dist="uniform")).to(cuda_device)
    for with_status in (True, False):
        s, b, n, st = _noalloc(lib, small, 8, 16, cuda_device, with_status=with_status)
        rs, rb, rn = _regular(small, 8, 16)
        assert st == 0 and n == rn
        np.testing.assert_array_equal(s[:n], rs[:n])
        np.testing.assert_array_equal(b[:n // 16], rb[:n // 16])
    empty = torch.empty(0, 2, dtype=torch.int32, device=cuda_device)
    _, _, n, st = _noalloc(lib, empty, 8, 16, cuda_device)
    assert n == 0 and st == 0
