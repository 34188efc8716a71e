"""The C-ABI library loads and exports every entry point that
include/moe_b200.h declares; host-side argument checks and size queries
(no device work: these calls return before any launch)."""
import ctypes
import os
import re

import pytest

import mixture_experts_expert_moe_b200 as m

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "moe_b200.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = m.load_library()
    names = declared_symbols()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(m.EXPORTED) == names


def _debug_library_path():
    from mixture_experts_expert_moe_b200 import build_lib
    if not os.path.exists(build_lib.DEBUG_LIB):
        build_lib.build(debug=True)
    return build_lib.DEBUG_LIB


def test_debug_library_exports_the_same_abi():
    """libmoe_b200_debug.so (kernels compiled with MOE_DEBUG index checks)
    implements the same ABI: every declared symbol and the same version."""
    path = _debug_library_path()
    assert os.path.abspath(path) != os.path.abspath(m.LIB_PATH)
    lib = ctypes.CDLL(path)
    for n in declared_symbols():
        assert hasattr(lib, n), n
    lib.moe_version.restype = ctypes.c_int
    assert lib.moe_version() == m.ABI_VERSION
    assert m.MOE_DEV_BOUNDS == 0x10
    text = open(HEADER).read()
    assert re.search(r"#define MOE_DEV_BOUNDS\s+0x10\b", text)


def test_library_path_override_selects_the_debug_build():
    import subprocess
    import sys
    path = _debug_library_path()
    env = dict(os.environ, MOE_B200_LIB=path)
    code = ("import mixture_experts_expert_moe_b200 as m; lib = m.load_library(); "
            "print(m.LIB_PATH); print(lib.moe_version())")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], env=env, cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.split() == [path, str(m.ABI_VERSION)]


def test_status_strings_and_version():
    lib = m.load_library()
    assert lib.moe_status_string(0) == b"MOE_OK"
    assert lib.moe_status_string(3) == b"MOE_ERR_WORKSPACE"
    assert lib.moe_status_string(99) == b"MOE_ERR_UNKNOWN"
    assert lib.moe_version() == m.ABI_VERSION == 300


def test_align_sizes():
    assert m.align_sort_sizes(16384, 8, 256, 64) == (131072 + 256 * 63, -(-(131072 + 256 * 63) // 64),
                                                     256 + 1024 * 256 * 4)
    assert m.align_sort_sizes(0, 8, 256, 64)[0] == 256 * 63
    lib = m.load_library()
    P = ctypes.c_size_t()
    assert lib.moe_align_sort_sizes(4, 2, 0, 16, ctypes.byref(P), None, None) == 1
    assert lib.moe_align_sort_sizes(4, 2, 1025, 16, ctypes.byref(P), None, None) == 1
    assert lib.moe_align_sort_sizes(4, 0, 8, 16, ctypes.byref(P), None, None) == 1
    assert lib.moe_align_sort_sizes(-1, 2, 8, 16, ctypes.byref(P), None, None) == 1


@pytest.mark.parametrize("bad", [dict(E=0), dict(k=0), dict(k=9), dict(T=-1), dict(E=1025), dict(mode=2),
                                 dict(mode=-1), dict(S=-1), dict(k=8, E=40, S=25), dict(E=1020, S=5)])
def test_gate_rejects_bad_sizes(bad):
    lib = m.load_library()
    a = dict(T=4, E=8, k=2, mode=0, S=0)
    a.update(bad)
    assert lib.moe_topk_gate(None, None, a["mode"], a["T"], a["E"], a["k"], a["S"], None, None, None) == 1


@pytest.mark.parametrize("bad", [dict(bias_mode=2), dict(n_shared=-1), dict(n_shared=31), dict(E=1024, n_shared=1)])
def test_forward_workspace_rejects_bad_shared_and_mode(bad):
    lib = m.load_library()
    a = dict(T=64, H=256, I=128, E=8, k=2, block_size=16, wdtype=0, out_dtype=0, tile_tokens=0, n_shared=0,
             bias_mode=0)
    a.update(bad)
    n = ctypes.c_size_t()
    assert lib.moe_forward_workspace(ctypes.byref(m.ForwardArgs(**a)), ctypes.byref(n)) == 1


def test_forward_workspace_counts_shared_slots():
    """A shared expert adds one slot per token and one expert: the workspace
    grows accordingly."""
    lib = m.load_library()
    base = dict(T=64, H=256, I=128, E=8, k=2, block_size=16, wdtype=0, out_dtype=0, tile_tokens=0)
    n0, n1 = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.moe_forward_workspace(ctypes.byref(m.ForwardArgs(**base)), ctypes.byref(n0)) == 0
    assert lib.moe_forward_workspace(ctypes.byref(m.ForwardArgs(**base, n_shared=1)), ctypes.byref(n1)) == 0
    assert n1.value > n0.value


def _ffn(**kw):
    a = dict(T=64, H=256, I=128, E=8, k=2, block_size=16, wdtype=0, tile_tokens=0)
    a.update(kw)
    return m.FfnArgs(**a)


def test_ffn_workspace_and_validation():
    lib = m.load_library()
    n = ctypes.c_size_t()
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn()), ctypes.byref(n)) == 0 and n.value > 0
    n8 = ctypes.c_size_t()
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn(wdtype=1)), ctypes.byref(n8)) == 0
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn(H=200)), ctypes.byref(n)) == 2     # unsupported
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn(I=96)), ctypes.byref(n)) == 2
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn(wdtype=2)), ctypes.byref(n)) == 1
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn(tile_tokens=48)), ctypes.byref(n)) == 1
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn(k=9)), ctypes.byref(n)) == 1
    # missing pointers are rejected before any launch
    assert lib.moe_grouped_ffn(ctypes.byref(_ffn()), None, None, 0, None, None) == 1


def test_forward_workspace_and_validation():
    lib = m.load_library()
    a = m.ForwardArgs(T=64, H=256, I=128, E=8, k=2, block_size=16, wdtype=0, out_dtype=0)
    n = ctypes.c_size_t()
    assert lib.moe_forward_workspace(ctypes.byref(a), ctypes.byref(n)) == 0
    a.out_dtype = 1
    assert lib.moe_forward_workspace(ctypes.byref(a), ctypes.byref(n)) == 1
    a.out_dtype = 2
    assert lib.moe_forward(ctypes.byref(a), None, 0, None, None) == 1
    assert lib.moe_combine(None, None, 4, 2, 6, None, 0, None) == 1    # H % 4
    assert lib.moe_combine(None, None, 4, 2, 8, None, 5, None) == 1    # dtype


# ---------------------------------------------------------------------------
# argument errors are reported before anything touches the device
# ---------------------------------------------------------------------------
_HOST = (ctypes.c_uint8 * 4096)()          # a 16-byte-aligned host block used only as a non-null address
_ADDR = (ctypes.addressof(_HOST) + 15) // 16 * 16


def _fwd(**kw):
    a = dict(T=64, H=256, I=128, E=8, k=2, block_size=16, wdtype=0, out_dtype=0, x=_ADDR, logits=_ADDR,
             w13=_ADDR, w2=_ADDR, out=_ADDR)
    a.update(kw)
    return m.ForwardArgs(**a)


def test_forward_rejects_misaligned_and_missing_scales():
    lib = m.load_library()
    for bad in (dict(x=_ADDR + 2), dict(w13=_ADDR + 8), dict(out=_ADDR + 4)):
        assert lib.moe_forward(ctypes.byref(_fwd(**bad)), ctypes.c_void_p(_ADDR), 1 << 40, None, None) == 1
    # FP8 weights need their scales
    assert lib.moe_forward(ctypes.byref(_fwd(wdtype=1)), ctypes.c_void_p(_ADDR), 1 << 40, None, None) == 1
    # a misaligned workspace
    assert lib.moe_forward(ctypes.byref(_fwd()), ctypes.c_void_p(_ADDR + 1), 1 << 40, None, None) == 1


def test_forward_workspace_too_small():
    lib = m.load_library()
    a = _fwd()
    n = ctypes.c_size_t()
    assert lib.moe_forward_workspace(ctypes.byref(a), ctypes.byref(n)) == 0
    assert lib.moe_forward(ctypes.byref(a), ctypes.c_void_p(_ADDR), n.value - 1, None, None) == 3


def test_forward_without_a_device_fails_loudly():
    """Valid arguments on a machine without an sm_100 device: MOE_ERR_DEVICE
    (there is no CPU fallback)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a CUDA device is present")
    lib = m.load_library()
    a = _fwd()
    n = ctypes.c_size_t()
    assert lib.moe_forward_workspace(ctypes.byref(a), ctypes.byref(n)) == 0
    assert lib.moe_forward(ctypes.byref(a), ctypes.c_void_p(_ADDR), n.value, None, None) == 5


def test_forward_with_no_tokens_is_a_no_op():
    lib = m.load_library()
    assert lib.moe_forward(ctypes.byref(_fwd(T=0)), None, 0, None, None) == 0


def test_gate_with_no_tokens_is_a_no_op():
    lib = m.load_library()
    assert lib.moe_topk_gate(None, None, 0, 0, 8, 2, 0, None, None, None) == 0


def test_ffn_rejects_small_workspace_and_missing_scales():
    lib = m.load_library()
    a = _ffn(x=_ADDR, w13=_ADDR, w2=_ADDR, sorted_ids=_ADDR, expert_ids=_ADDR, num_post=_ADDR)
    n = ctypes.c_size_t()
    assert lib.moe_ffn_workspace(ctypes.byref(a), ctypes.byref(n)) == 0
    y = ctypes.c_void_p(_ADDR)
    assert lib.moe_grouped_ffn(ctypes.byref(a), y, ctypes.c_void_p(_ADDR), n.value - 16, None, None) == 3
    a8 = _ffn(wdtype=1, x=_ADDR, w13=_ADDR, w2=_ADDR, sorted_ids=_ADDR, expert_ids=_ADDR, num_post=_ADDR)
    assert lib.moe_grouped_ffn(ctypes.byref(a8), y, ctypes.c_void_p(_ADDR), 1 << 40, None, None) == 1


def test_align_sort_argument_errors():
    lib = m.load_library()
    p = ctypes.c_void_p(_ADDR)
    # outputs missing
    assert lib.moe_align_sort(p, 16, 2, 8, 16, None, p, p, p, 1 << 20, None, None) == 1
    # workspace below moe_align_sort_sizes' figure
    ws = ctypes.c_size_t()
    assert lib.moe_align_sort_sizes(16, 2, 8, 16, None, None, ctypes.byref(ws)) == 0
    assert lib.moe_align_sort(p, 16, 2, 8, 16, p, p, p, p, ws.value - 1, None, None) == 3
    # the no-allocation variant: more experts than its built-in scratch holds
    assert lib.moe_align_sort_noalloc(p, 16, 2, 257, 16, p, p, p, None, None) == 2
    assert lib.moe_align_sort_noalloc(p, 16, 2, 8, 16, None, p, p, None, None) == 1


def _fwd_ws(**kw):
    lib = m.load_library()
    a = dict(T=64, H=256, I=128, E=8, k=2, block_size=16, wdtype=0, out_dtype=0)
    a.update(kw)
    n = ctypes.c_size_t()
    assert lib.moe_forward_workspace(ctypes.byref(m.ForwardArgs(**a)), ctypes.byref(n)) == 0
    return n.value


def test_forward_workspace_follows_the_combine_rule():
    """k + n_shared >= 4: the combine is fused, the workspace holds an fp32
    token accumulator [T, H] only for bf16 output (an f32 output is the
    accumulator).  Fewer slots: per-slot rows [T*k, H] for either output."""
    T, H = 64, 256
    fused_bf16, fused_f32 = _fwd_ws(k=4, out_dtype=0), _fwd_ws(k=4, out_dtype=2)
    assert fused_bf16 - fused_f32 == T * H * 4
    assert _fwd_ws(k=2, out_dtype=0) == _fwd_ws(k=2, out_dtype=2)
    # a shared expert counts as a slot: k = 3 + 1 shared is fused as well
    assert _fwd_ws(k=3, n_shared=1, out_dtype=0) - _fwd_ws(k=3, n_shared=1, out_dtype=2) == T * H * 4


# ---------------------------------------------------------------------------
# MX block-scaled weights (MOE_MXFP8 = 3, MOE_MXFP4 = 4)
# ---------------------------------------------------------------------------
def test_mx_workspace_and_tile_limit():
    lib = m.load_library()
    n16, n8, nmx = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn()), ctypes.byref(n16)) == 0
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn(wdtype=3)), ctypes.byref(nmx)) == 0
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn(wdtype=4)), ctypes.byref(n8)) == 0
    assert n8.value == nmx.value < n16.value        # one-byte activations, no bf16 copy of h
    # MX token tiles hold at most 128 tokens
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn(wdtype=3, tile_tokens=256)), ctypes.byref(n8)) == 2
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn(wdtype=3, tile_tokens=128)), ctypes.byref(n8)) == 0
    assert lib.moe_ffn_workspace(ctypes.byref(_ffn(wdtype=5)), ctypes.byref(n8)) == 1


def test_mx_forward_needs_its_scales_and_alignment():
    lib = m.load_library()
    ws = ctypes.c_void_p(_ADDR)
    # MX weights without their tiled scales
    assert lib.moe_forward(ctypes.byref(_fwd(wdtype=3)), ws, 1 << 40, None, None) == 1
    assert lib.moe_forward(ctypes.byref(_fwd(wdtype=4, w13_mx_scale=_ADDR)), ws, 1 << 40, None, None) == 1
    # packed E2M1 weights need 32-byte aligned bases (the 4-bit tensor maps' rule)
    a32 = (_ADDR + 31) // 32 * 32
    bad = _fwd(wdtype=4, w13=a32 + 16, w2=a32, w13_mx_scale=_ADDR, w2_mx_scale=_ADDR)
    assert lib.moe_forward(ctypes.byref(bad), ws, 1 << 40, None, None) == 1


def test_mx_helpers_argument_errors():
    lib = m.load_library()
    p = ctypes.c_void_p(_ADDR)
    assert lib.moe_mx_tile_scales(p, 100, 256, p, None) == 1       # rows % 128
    assert lib.moe_mx_tile_scales(p, 128, 96, p, None) == 1        # K % 128
    assert lib.moe_mx_tile_scales(None, 128, 256, p, None) == 1
    assert lib.moe_mx_tile_scales(p, 0, 256, p, None) == 0         # nothing to do
    assert lib.moe_mx_quantize_rows(p, 4, 48, p, p, None) == 1     # C % 32
    assert lib.moe_mx_quantize_rows(p, -1, 64, p, p, None) == 1
    assert lib.moe_mx_quantize_rows(p, 0, 64, p, p, None) == 0
