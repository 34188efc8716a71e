"""Python binding of the B200 MoE layer-forward library (libmoe_b200.so).

Argument marshalling only: every step of the forward runs in the CUDA
kernels behind the C ABI declared in ``include/moe_b200.h``.  PyTorch is used
for device memory (workspaces and outputs are torch tensors) and for the
current CUDA stream.  There is no CPU fallback: if the shared library is not
built, importing the ops raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_B200_LIB selects another build of the same ABI (libmoe_b200_debug.so:
# kernels with index checks that report MOE_DEV_BOUNDS)
LIB_PATH = os.environ.get("MOE_B200_LIB") or os.path.join(_PKG, "libmoe_b200.so")

MOE_BF16, MOE_FP8_E4M3, MOE_F32, MOE_MXFP8, MOE_MXFP4 = 0, 1, 2, 3, 4
_MX_TYPES = {"mxfp8": MOE_MXFP8, "mxfp4": MOE_MXFP4}
MOE_DEV_BAD_EXPERT_ID, MOE_DEV_TIMEOUT, MOE_DEV_BAD_PLAN, MOE_DEV_DRAIN_TIMEOUT = 0x1, 0x2, 0x4, 0x8
MOE_DEV_BOUNDS = 0x10   # debug builds only: an out-of-range index was skipped
STAGES = ["gate", "align", "plan", "gather", "gateup", "requant", "down", "combine"]

EXPORTED = [
    "moe_status_string", "moe_last_cuda_error", "moe_version", "moe_topk_gate",
    "moe_align_sort_sizes", "moe_align_sort", "moe_ffn_workspace", "moe_grouped_ffn",
    "moe_combine", "moe_forward_workspace", "moe_forward", "moe_test_wait_timeout",
    "moe_align_sort_noalloc", "moe_test_quant_division", "moe_mx_tile_scales", "moe_mx_quantize_rows",
    "moe_backward_workspace", "moe_backward", "moe_ep_route_workspace", "moe_ep_route", "moe_permute_rows",
    "moe_scatter_rows",
]

_vp = ctypes.c_void_p
_i = ctypes.c_int


class FfnArgs(ctypes.Structure):
    _fields_ = [("T", _i), ("H", _i), ("I", _i), ("E", _i), ("k", _i), ("block_size", _i),
                ("wdtype", _i), ("x", _vp), ("w13", _vp), ("w13_scale", _vp), ("w2", _vp),
                ("w2_scale", _vp), ("sorted_ids", _vp), ("expert_ids", _vp), ("num_post", _vp),
                ("tile_tokens", _i), ("w13_mx_scale", _vp), ("w2_mx_scale", _vp)]


class ForwardArgs(ctypes.Structure):
    _fields_ = [("T", _i), ("H", _i), ("I", _i), ("E", _i), ("k", _i), ("block_size", _i),
                ("wdtype", _i), ("out_dtype", _i), ("x", _vp), ("logits", _vp), ("bias", _vp),
                ("w13", _vp), ("w13_scale", _vp), ("w2", _vp), ("w2_scale", _vp), ("out", _vp),
                ("topk_ids", _vp), ("topk_w", _vp), ("tile_tokens", _i), ("stage_events", _vp),
                ("n_shared", _i), ("bias_mode", _i), ("w13_mx_scale", _vp), ("w2_mx_scale", _vp)]


class BackwardArgs(ctypes.Structure):
    _fields_ = [("T", _i), ("H", _i), ("I", _i), ("E", _i), ("k", _i), ("block_size", _i), ("n_shared", _i),
                ("bias_mode", _i), ("x", _vp), ("logits", _vp), ("bias", _vp), ("w13", _vp), ("w2", _vp),
                ("dout", _vp), ("dx", _vp), ("dlogits", _vp), ("dw13", _vp), ("dw2", _vp)]


MOE_BIAS_LOGITS, MOE_BIAS_SELECT = 0, 1
ABI_VERSION = 300   # MOE_ABI_VERSION of include/moe_b200.h
_BIAS_MODES = {"logits": MOE_BIAS_LOGITS, "select": MOE_BIAS_SELECT}


_LIB = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoe_b200.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(path):
            raise ImportError(
                f"{path} is missing: build it with `python -m mixture_experts_expert_moe_b200.build_lib`")
        lib = ctypes.CDLL(path)
        sz = ctypes.POINTER(ctypes.c_size_t)
        sigs = {
            "moe_status_string": (ctypes.c_char_p, [_i]),
            "moe_last_cuda_error": (ctypes.c_char_p, []),
            "moe_version": (_i, []),
            "moe_topk_gate": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _vp, _vp, _vp]),
            "moe_align_sort_sizes": (_i, [_i, _i, _i, _i, sz, sz, sz]),
            "moe_align_sort": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp, _vp]),
            "moe_ffn_workspace": (_i, [ctypes.POINTER(FfnArgs), sz]),
            "moe_grouped_ffn": (_i, [ctypes.POINTER(FfnArgs), _vp, _vp, ctypes.c_size_t, _vp, _vp]),
            "moe_combine": (_i, [_vp, _vp, _i, _i, _i, _vp, _i, _vp]),
            "moe_forward_workspace": (_i, [ctypes.POINTER(ForwardArgs), sz]),
            "moe_forward": (_i, [ctypes.POINTER(ForwardArgs), _vp, ctypes.c_size_t, _vp, _vp]),
            "moe_test_wait_timeout": (_i, [_vp, _vp, ctypes.c_longlong, _vp]),
            "moe_align_sort_noalloc": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, _vp]),
            "moe_test_quant_division": (_i, [_vp, _vp]),
            "moe_mx_tile_scales": (_i, [_vp, ctypes.c_longlong, _i, _vp, _vp]),
            "moe_mx_quantize_rows": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
            "moe_backward_workspace": (_i, [ctypes.POINTER(BackwardArgs), sz]),
            "moe_backward": (_i, [ctypes.POINTER(BackwardArgs), _vp, ctypes.c_size_t, _vp, _vp]),
            "moe_ep_route_workspace": (_i, [_i, _i, _i, sz]),
            "moe_ep_route": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp, _vp]),
            "moe_permute_rows": (_i, [_vp, _i, _vp, _i, _i, _i, _vp, _vp]),
            "moe_scatter_rows": (_i, [_vp, _i, _vp, _i, _i, _vp, _vp]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        if lib.moe_version() != ABI_VERSION:
            raise ImportError(f"{path} implements ABI {lib.moe_version()}, this binding expects {ABI_VERSION}: "
                              "rebuild it with `python -m mixture_experts_expert_moe_b200.build_lib`")
        _LIB = lib
    return _LIB


class MoEError(RuntimeError):
    pass


def _check(status: int, what: str):
    if status != 0:
        lib = load_library()
        msg = lib.moe_status_string(status).decode()
        cuda = lib.moe_last_cuda_error().decode()
        raise MoEError(f"{what}: {msg}" + (f" ({cuda})" if cuda and status == 4 else ""))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device=None):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dev_status(dev_status, device):
    if dev_status is None:
        return None
    assert dev_status.dtype == torch.int32 and dev_status.device == device
    return _ptr(dev_status)


def _wdtype(w, mx=None):
    if mx is not None:
        if w.dtype != torch.uint8:
            raise TypeError("MX weights are uint8 codes (E4M3, or E2M1 packed two per byte)")
        return _MX_TYPES[mx]
    if w.dtype == torch.bfloat16:
        return MOE_BF16
    if w.dtype in (torch.float8_e4m3fn, torch.uint8):
        return MOE_FP8_E4M3
    raise TypeError(f"unsupported weight dtype {w.dtype}")


def _inner_k(w, mx):
    """Elements along K of a weight tensor (E2M1 codes are packed two per byte)."""
    return w.shape[-1] * (2 if mx == "mxfp4" else 1)


# ---------------------------------------------------------------------------
# ops
# ---------------------------------------------------------------------------

def topk_gate(logits: torch.Tensor, k: int, bias: torch.Tensor | None = None, bias_mode: str = "logits",
              n_shared: int = 0):
    """Softmax top-k gating: returns (ids int32 [T, k+n_shared], weights f32
    [T, k+n_shared]); the last n_shared columns are the shared experts E..
    with weight 1.  bias_mode "logits": the bias shifts the logits for both
    the choice and the weights; "select": it only steers the choice."""
    lib = load_library()
    assert logits.is_cuda and logits.dtype == torch.float32 and logits.is_contiguous()
    T, E = logits.shape
    ids = torch.empty(T, k + n_shared, dtype=torch.int32, device=logits.device)
    w = torch.empty(T, k + n_shared, dtype=torch.float32, device=logits.device)
    _check(lib.moe_topk_gate(_ptr(logits), _ptr(bias), _BIAS_MODES[bias_mode], T, E, k, n_shared, _ptr(ids),
                             _ptr(w), _stream(logits.device)), "moe_topk_gate")
    return ids, w


def align_sort_sizes(T: int, k: int, E: int, block_size: int):
    lib = load_library()
    P, NB, ws = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.moe_align_sort_sizes(T, k, E, block_size, ctypes.byref(P), ctypes.byref(NB),
                                    ctypes.byref(ws)), "moe_align_sort_sizes")
    return P.value, NB.value, ws.value


def align_sort(topk_ids: torch.Tensor, E: int, block_size: int, dev_status=None, ws=None, out=None):
    """Block-aligned align&sort.  Returns (sorted_ids [P], expert_ids [NB],
    num_post [1]); only the first num_post / num_post//block_size entries are
    defined."""
    lib = load_library()
    assert topk_ids.is_cuda and topk_ids.dtype == torch.int32 and topk_ids.is_contiguous()
    T, k = topk_ids.shape
    P, NB, wsb = align_sort_sizes(T, k, E, block_size)
    dev = topk_ids.device
    if out is None:
        out = (torch.empty(P, dtype=torch.int32, device=dev), torch.empty(NB, dtype=torch.int32, device=dev),
               torch.empty(1, dtype=torch.int32, device=dev))
    if ws is None:
        ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    s, b, n = out
    _check(lib.moe_align_sort(_ptr(topk_ids), T, k, E, block_size, _ptr(s), _ptr(b), _ptr(n), _ptr(ws),
                              ws.numel(), _dev_status(dev_status, dev), _stream(dev)), "moe_align_sort")
    return s, b, n


def _ffn_args(x, w13, w2, sorted_ids, expert_ids, num_post, T, k, E, block_size, w13_scale, w2_scale,
              tile_tokens, mx=None, w13_mx_scale=None, w2_mx_scale=None):
    H = x.shape[1]
    I = w13.shape[1] // 2
    a = FfnArgs(T=T, H=H, I=I, E=E, k=k, block_size=block_size, wdtype=_wdtype(w13, mx),
                x=x.data_ptr(), w13=w13.data_ptr(), w2=w2.data_ptr(),
                w13_scale=None if w13_scale is None else w13_scale.data_ptr(),
                w2_scale=None if w2_scale is None else w2_scale.data_ptr(),
                sorted_ids=sorted_ids.data_ptr(), expert_ids=expert_ids.data_ptr(),
                num_post=num_post.data_ptr(), tile_tokens=tile_tokens,
                w13_mx_scale=None if w13_mx_scale is None else w13_mx_scale.data_ptr(),
                w2_mx_scale=None if w2_mx_scale is None else w2_mx_scale.data_ptr())
    return a


def grouped_ffn(x, w13, w2, sorted_ids, expert_ids, num_post, k, block_size, w13_scale=None, w2_scale=None,
                tile_tokens=0, dev_status=None, y=None, ws=None, mx=None, w13_mx_scale=None, w2_mx_scale=None):
    """Per-slot expert FFN output y f32 [T*k, H] over align&sort's outputs.
    ``mx`` ("mxfp8" / "mxfp4"): MX weights (uint8 codes) with tiled E8M0
    scales ``w13_mx_scale`` / ``w2_mx_scale`` from ``mx_tile_scales``."""
    lib = load_library()
    T, H = x.shape
    E = w13.shape[0]
    a = _ffn_args(x, w13, w2, sorted_ids, expert_ids, num_post, T, k, E, block_size, w13_scale, w2_scale,
                  tile_tokens, mx, w13_mx_scale, w2_mx_scale)
    nbytes = ctypes.c_size_t()
    _check(lib.moe_ffn_workspace(ctypes.byref(a), ctypes.byref(nbytes)), "moe_ffn_workspace")
    if ws is None:
        ws = torch.empty(nbytes.value, dtype=torch.uint8, device=x.device)
    if y is None:
        y = torch.empty(T * k, H, dtype=torch.float32, device=x.device)
    _check(lib.moe_grouped_ffn(ctypes.byref(a), _ptr(y), _ptr(ws), ws.numel(),
                               _dev_status(dev_status, x.device), _stream(x.device)), "moe_grouped_ffn")
    return y


def combine(y: torch.Tensor, topk_w: torch.Tensor, out_dtype=torch.bfloat16, out=None):
    """out[t] = sum_j w[t,j] * y[t*k+j]."""
    lib = load_library()
    T, k = topk_w.shape
    H = y.shape[1]
    if out is None:
        out = torch.empty(T, H, dtype=out_dtype, device=y.device)
    od = MOE_BF16 if out.dtype == torch.bfloat16 else MOE_F32
    _check(lib.moe_combine(_ptr(y), _ptr(topk_w), T, k, H, _ptr(out), od, _stream(y.device)), "moe_combine")
    return out


class MoELayer:
    """One MoE layer forward through ``moe_forward`` with a reusable workspace.

    Weights: ``w13 [E + n_shared, 2I, H]`` (gate rows then up rows) and
    ``w2 [E + n_shared, H, I]``, bf16, or float8_e4m3fn codes with f32 per-row
    scales ``w13_scale [E + n_shared, 2I]`` and ``w2_scale [E + n_shared, H]``;
    the last ``n_shared`` experts are shared (every token, weight 1).
    ``bias_mode``: "logits" (the bias shifts the logits for the choice and the
    weights) or "select" (it only steers the choice).
    """

    def __init__(self, w13, w2, k, block_size, w13_scale=None, w2_scale=None, out_dtype=torch.bfloat16,
                 tile_tokens=0, n_shared=0, bias_mode="logits", mx=None, w13_mx_scale=None, w2_mx_scale=None):
        self.w13, self.w2, self.k, self.block_size = w13, w2, k, block_size
        self.w13_scale, self.w2_scale = w13_scale, w2_scale
        self.mx, self.w13_mx_scale, self.w2_mx_scale = mx, w13_mx_scale, w2_mx_scale
        self.out_dtype, self.tile_tokens = out_dtype, tile_tokens
        self.n_shared, self.bias_mode = n_shared, _BIAS_MODES[bias_mode]
        EW, twoI, _ = w13.shape
        self.H = _inner_k(w13, mx)
        self.E = EW - n_shared
        self.I = twoI // 2
        self._ws = None

    def _args(self, x, logits, bias, out, ids, w, events=None):
        T = x.shape[0]
        return ForwardArgs(
            T=T, H=self.H, I=self.I, E=self.E, k=self.k, block_size=self.block_size,
            wdtype=_wdtype(self.w13, self.mx), out_dtype=MOE_BF16 if out.dtype == torch.bfloat16 else MOE_F32,
            x=x.data_ptr(), logits=logits.data_ptr(), bias=None if bias is None else bias.data_ptr(),
            w13=self.w13.data_ptr(), w13_scale=None if self.w13_scale is None else self.w13_scale.data_ptr(),
            w2=self.w2.data_ptr(), w2_scale=None if self.w2_scale is None else self.w2_scale.data_ptr(),
            out=out.data_ptr(), topk_ids=None if ids is None else ids.data_ptr(),
            topk_w=None if w is None else w.data_ptr(), tile_tokens=self.tile_tokens,
            stage_events=None if events is None else ctypes.cast(events, ctypes.c_void_p),
            n_shared=self.n_shared, bias_mode=self.bias_mode,
            w13_mx_scale=None if self.w13_mx_scale is None else self.w13_mx_scale.data_ptr(),
            w2_mx_scale=None if self.w2_mx_scale is None else self.w2_mx_scale.data_ptr())

    def workspace_bytes(self, T):
        lib = load_library()
        a = ForwardArgs(T=T, H=self.H, I=self.I, E=self.E, k=self.k, block_size=self.block_size,
                        wdtype=_wdtype(self.w13, self.mx),
                        out_dtype=MOE_BF16 if self.out_dtype == torch.bfloat16 else MOE_F32,
                        tile_tokens=self.tile_tokens, n_shared=self.n_shared, bias_mode=self.bias_mode)
        n = ctypes.c_size_t()
        _check(lib.moe_forward_workspace(ctypes.byref(a), ctypes.byref(n)), "moe_forward_workspace")
        return n.value

    def __call__(self, x, logits, bias=None, out=None, topk_ids=None, topk_w=None, dev_status=None,
                 stage_events=None):
        """Run the layer.  ``stage_events``: optional list of len(STAGES)+1
        torch.cuda.Event objects recorded at the stage boundaries."""
        lib = load_library()
        T = x.shape[0]
        if out is None:
            out = torch.empty(T, self.H, dtype=self.out_dtype, device=x.device)
        need = self.workspace_bytes(T)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=x.device)
        evs = None
        if stage_events is not None:
            assert len(stage_events) == len(STAGES) + 1
            for e in stage_events:
                if e.cuda_event == 0:     # created lazily by torch
                    e.record()
            evs = (ctypes.c_void_p * len(stage_events))(*[e.cuda_event for e in stage_events])
        a = self._args(x, logits, bias, out, topk_ids, topk_w, evs)
        _check(lib.moe_forward(ctypes.byref(a), _ptr(self._ws), self._ws.numel(),
                               _dev_status(dev_status, x.device), _stream(x.device)), "moe_forward")
        return out


def backward(x, logits, w13, w2, dout, k, block_size, bias=None, bias_mode="logits", n_shared=0,
             dev_status=None, ws=None, outs=None):
    """Gradients of sum(out * dout) for the layer forward (bf16 weights):
    returns (dx f32 [T, H], dlogits f32 [T, E], dw13 f32 like w13, dw2 f32
    like w2), written into ``outs`` when given."""
    lib = load_library()
    T, H = x.shape
    E = logits.shape[1]
    I = w13.shape[1] // 2
    dev = x.device
    if outs is None:
        outs = (torch.empty(T, H, dtype=torch.float32, device=dev),
                torch.empty(T, E, dtype=torch.float32, device=dev),
                torch.empty(w13.shape, dtype=torch.float32, device=dev),
                torch.empty(w2.shape, dtype=torch.float32, device=dev))
    dx, dl, dw13, dw2 = outs
    a = BackwardArgs(T=T, H=H, I=I, E=E, k=k, block_size=block_size, n_shared=n_shared,
                     bias_mode=_BIAS_MODES[bias_mode], x=x.data_ptr(), logits=logits.data_ptr(),
                     bias=None if bias is None else bias.data_ptr(), w13=w13.data_ptr(), w2=w2.data_ptr(),
                     dout=dout.data_ptr(), dx=dx.data_ptr(), dlogits=dl.data_ptr(), dw13=dw13.data_ptr(),
                     dw2=dw2.data_ptr())
    n = ctypes.c_size_t()
    _check(lib.moe_backward_workspace(ctypes.byref(a), ctypes.byref(n)), "moe_backward_workspace")
    if ws is None or ws.numel() < n.value:
        ws = torch.empty(max(n.value, 1), dtype=torch.uint8, device=dev)
    _check(lib.moe_backward(ctypes.byref(a), _ptr(ws), ws.numel(), _dev_status(dev_status, dev), _stream(dev)),
           "moe_backward")
    return dx, dl, dw13, dw2


def ep_route(topk_ids: torch.Tensor, E: int, R: int, dev_status=None):
    """Destination ranks of the slots for R-way expert parallelism (rank r
    holds experts [r*E/R, (r+1)*E/R)): returns (order int32 [T*k]: the flat
    slots grouped by destination rank, send_counts int32 [R], local_ids int32
    [T*k]: the slots' expert ids local to their rank, in order's order)."""
    lib = load_library()
    assert topk_ids.is_cuda and topk_ids.dtype == torch.int32 and topk_ids.is_contiguous()
    T, k = topk_ids.shape
    dev = topk_ids.device
    n = ctypes.c_size_t()
    _check(lib.moe_ep_route_workspace(T, k, R, ctypes.byref(n)), "moe_ep_route_workspace")
    ws = torch.empty(max(n.value, 1), dtype=torch.uint8, device=dev)
    order = torch.empty(T * k, dtype=torch.int32, device=dev)
    counts = torch.empty(R, dtype=torch.int32, device=dev)
    local = torch.empty(T * k, dtype=torch.int32, device=dev)
    _check(lib.moe_ep_route(_ptr(topk_ids), T, k, E, R, _ptr(order), _ptr(counts), _ptr(local), _ptr(ws),
                            ws.numel(), _dev_status(dev_status, dev), _stream(dev)), "moe_ep_route")
    return order, counts, local


def permute_rows(src: torch.Tensor, index: torch.Tensor, div: int = 1) -> torch.Tensor:
    """out[i] = src[index[i] // div] (rows of a 2-D tensor)."""
    lib = load_library()
    assert src.is_cuda and src.is_contiguous() and index.dtype == torch.int32
    n = index.numel()
    out = torch.empty(n, src.shape[1], dtype=src.dtype, device=src.device)
    rb = src.shape[1] * src.element_size()
    _check(lib.moe_permute_rows(_ptr(src), rb, _ptr(index), n, div, src.shape[0], _ptr(out), _stream(src.device)),
           "moe_permute_rows")
    return out


def scatter_rows(src: torch.Tensor, index: torch.Tensor, rows: int) -> torch.Tensor:
    """out[index[i]] = src[i]; out has `rows` rows (rows no index names are 0)."""
    lib = load_library()
    assert src.is_cuda and src.is_contiguous() and index.dtype == torch.int32
    out = torch.zeros(rows, src.shape[1], dtype=src.dtype, device=src.device)
    rb = src.shape[1] * src.element_size()
    _check(lib.moe_scatter_rows(_ptr(src), rb, _ptr(index), index.numel(), rows, _ptr(out), _stream(src.device)),
           "moe_scatter_rows")
    return out


def mx_tile_scales(sf: torch.Tensor) -> torch.Tensor:
    """Per-row E8M0 weight scales ``sf`` uint8 [..., rows, K/32] (any leading
    dims folded into rows; rows % 128 == 0, K % 128 == 0) rearranged into the
    tiled layout the MX grouped GEMM reads (model preparation, done once)."""
    lib = load_library()
    assert sf.is_cuda and sf.dtype == torch.uint8 and sf.is_contiguous()
    K = sf.shape[-1] * 32
    rows = sf.numel() // sf.shape[-1]
    out = torch.empty_like(sf)
    _check(lib.moe_mx_tile_scales(_ptr(sf), rows, K, _ptr(out), _stream(sf.device)), "moe_mx_tile_scales")
    return out


def mx_quantize_rows(x: torch.Tensor):
    """MXFP8 quantisation of bf16 rows x [R, C]: (E4M3 codes uint8 [R, C],
    E8M0 scale codes uint8 [R, C/32])."""
    lib = load_library()
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2
    R, C = x.shape
    codes = torch.empty(R, C, dtype=torch.uint8, device=x.device)
    scales = torch.empty(R, C // 32, dtype=torch.uint8, device=x.device)
    _check(lib.moe_mx_quantize_rows(_ptr(x), R, C, _ptr(codes), _ptr(scales), _stream(x.device)),
           "moe_mx_quantize_rows")
    return codes, scales


def capture_graph(layer, x, logits, bias=None, out=None):
    """Capture one ``layer`` forward on these fixed buffers into a CUDA graph.

    Returns (graph, out); ``graph.replay()`` reruns the whole forward (the
    same kernels the C ABI launches) without host launch overhead.
    """
    out = layer(x, logits, bias, out=out)      # sizes the workspace outside the capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer(x, logits, bias, out=out)
    return g, out


def run_wait_timeout_check(timeout_ns: int, device="cuda"):
    """Run the bounded grid-wide wait on a barrier that never fills; returns
    the device status word (MOE_DEV_TIMEOUT expected)."""
    lib = load_library()
    ws = torch.zeros(64, dtype=torch.int32, device=device)
    st = torch.zeros(1, dtype=torch.int32, device=device)
    _check(lib.moe_test_wait_timeout(_ptr(ws), _ptr(st), int(timeout_ns), _stream(torch.device(device))),
           "moe_test_wait_timeout")
    torch.cuda.synchronize()
    return int(st.item())


def run_quant_division_check(device="cuda"):
    """Exhaustive check of the E4M3 quantiser's quotient path against IEEE
    division over all bf16 pairs (v, amax), |v| <= amax.  Returns
    (pairs checked, mismatches, one failing (v bits << 16 | amax bits))."""
    lib = load_library()
    ws = torch.zeros(4, dtype=torch.int64, device=device)
    _check(lib.moe_test_quant_division(_ptr(ws), _stream(torch.device(device))), "moe_test_quant_division")
    torch.cuda.synchronize()
    c = ws.cpu().tolist()
    return c[0], c[1], c[2] & 0xFFFFFFFF
