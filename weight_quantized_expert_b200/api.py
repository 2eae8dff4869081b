"""Thin Python binding of libfocr_moe (include/focr_moe.h).

Argument marshalling only: every step of the layer runs in the CUDA library.  PyTorch
provides device memory and the current stream.  There is no fallback: if the
shared library is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np

from . import synth

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfocr_moe.so")

H, E, TOPK, I, IS, VOCAB, DENSE_I = 1280, 64, 6, 896, 1792, 129280, 6848
T_MAX = 8192
W_BF16, W_INT8, W_INT4 = 0, 1, 2
(MAT_GATE, MAT_UP, MAT_DOWN, MAT_SHARED_GATE, MAT_SHARED_UP, MAT_SHARED_DOWN, MAT_ROUTER) = range(7)
STATUS = {0: "FOCR_OK", 1: "FOCR_ERR_INVALID_ARG", 2: "FOCR_ERR_UNSUPPORTED", 3: "FOCR_ERR_CUDA",
          4: "FOCR_ERR_OOM", 5: "FOCR_ERR_TIMEOUT", 6: "FOCR_ERR_RANGE"}

# every symbol include/focr_moe.h declares
EXPORTED = (
    "focr_moe_pack_weights", "focr_moe_layer_clone", "focr_moe_layer_free", "focr_moe_layer_device_bytes",
    "focr_moe_export_sizes", "focr_moe_export_quantized", "focr_moe_workspace_bytes",
    "focr_moe_workspace_zero_bytes", "focr_moe_layer_forward",
    "focr_moe_check", "focr_last_error", "focr_version", "focr_moe_layer_forward_noalloc", "focr_moe_check_noalloc",
    "focr_moe_layer_forward_ex", "focr_lm_head_pack", "focr_lm_head_free", "focr_lm_head_export",
    "focr_lm_head_workspace_bytes", "focr_lm_head_gemv", "focr_rmsnorm", "focr_dense_mlp_pack",
    "focr_dense_mlp_free", "focr_dense_mlp_export_quantized", "focr_dense_mlp_forward", "focr_tc_selftest",
    "focr_decode_step_workspace_bytes", "focr_decode_step", "focr_w8a8_pack", "focr_w8a8_free",
    "focr_w8a8_export", "focr_w8a8_quantize_x", "focr_w8a8_workspace_bytes", "focr_w8a8_gemv", "focr_w8a8_check",
    "focr_lm_head_check", "focr_rswa_workspace_bytes", "focr_rswa_decode",
)
FWD_RESIDUAL = 1
FWD_DETERMINISTIC = 2
NOALLOC_T_MAX = 320


class FocrError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class WeightsDesc(ctypes.Structure):
    _fields_ = [("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p),
                ("ws_gate", ctypes.c_void_p), ("ws_up", ctypes.c_void_p), ("ws_down", ctypes.c_void_p),
                ("w_router_bf16", ctypes.c_void_p), ("routed_type", ctypes.c_int32),
                ("shared_type", ctypes.c_int32), ("group_size", ctypes.c_int32)]


class RouteDebug(ctypes.Structure):
    _fields_ = [("logits", ctypes.c_void_p), ("topk_idx", ctypes.c_void_p), ("topk_w", ctypes.c_void_p),
                ("counts", ctypes.c_void_p), ("offsets", ctypes.c_void_p), ("perm", ctypes.c_void_p)]


_lib = None
_lock = threading.Lock()


class DecodeModelDesc(ctypes.Structure):
    _fields_ = [("dense", ctypes.c_void_p), ("moe", ctypes.POINTER(ctypes.c_void_p)), ("n_moe", ctypes.c_int32),
                ("gamma", ctypes.POINTER(ctypes.c_void_p)), ("eps", ctypes.c_float), ("head", ctypes.c_void_p)]


def lib():
    """Load libfocr_moe.so (built in-tree by weight_quantized_expert_b200/build.py)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with weight_quantized_expert_b200/build.py")
            L = ctypes.CDLL(LIB_PATH)
            P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
            sigs = {
                "focr_moe_pack_weights": (i32, [ctypes.POINTER(WeightsDesc), ctypes.POINTER(P), P]),
                "focr_moe_layer_clone": (i32, [P, ctypes.POINTER(P), P]),
                "focr_moe_layer_free": (None, [P]),
                "focr_moe_layer_device_bytes": (sz, [P]),
                "focr_moe_export_sizes": (i32, [P, i32, ctypes.POINTER(sz), ctypes.POINTER(sz)]),
                "focr_moe_export_quantized": (i32, [P, i32, i32, P, sz, P, sz]),
                "focr_moe_workspace_bytes": (sz, [i32]),
                "focr_moe_workspace_zero_bytes": (sz, []),
                "focr_moe_layer_forward": (i32, [P, P, i32, P, P, sz, ctypes.POINTER(RouteDebug), P]),
                "focr_moe_check": (i32, [P, P]),
                "focr_moe_layer_forward_noalloc": (i32, [P, P, i32, P, ctypes.POINTER(RouteDebug), P]),
                "focr_moe_check_noalloc": (i32, [P]),
                "focr_moe_layer_forward_ex": (i32, [P, P, i32, P, P, sz, ctypes.POINTER(RouteDebug), i32, P]),
                "focr_lm_head_pack": (i32, [P, ctypes.POINTER(P), P]),
                "focr_lm_head_free": (None, [P]),
                "focr_lm_head_export": (i32, [P, P, P]),
                "focr_lm_head_workspace_bytes": (sz, [i32]),
                "focr_lm_head_gemv": (i32, [P, P, i32, P, P, P, sz, P]),
                "focr_rmsnorm": (i32, [P, P, i32, ctypes.c_float, P, P]),
                "focr_dense_mlp_pack": (i32, [P, P, P, i32, i32, ctypes.POINTER(P), P]),
                "focr_dense_mlp_free": (None, [P]),
                "focr_dense_mlp_export_quantized": (i32, [P, i32, P, sz, P, sz]),
                "focr_dense_mlp_forward": (i32, [P, P, i32, P, P, sz, i32, P]),
                "focr_tc_selftest": (i32, [P, P, i32, i32, i32, P, P, P]),
                "focr_decode_step_workspace_bytes": (sz, [i32]),
                "focr_decode_step": (i32, [ctypes.POINTER(DecodeModelDesc), P, i32, P, P, P, P, sz, P]),
                "focr_w8a8_pack": (i32, [P, i64, i32, ctypes.POINTER(P), P]),
                "focr_w8a8_free": (None, [P]),
                "focr_w8a8_export": (i32, [P, P, P, ctypes.POINTER(i64), ctypes.POINTER(i32)]),
                "focr_w8a8_quantize_x": (i32, [P, i32, i32, P, P, P]),
                "focr_w8a8_workspace_bytes": (sz, [P, i32]),
                "focr_w8a8_gemv": (i32, [P, P, i32, P, P, sz, P]),
                "focr_w8a8_check": (i32, [P, P]),
                "focr_lm_head_check": (i32, [P, P]),
                "focr_rswa_workspace_bytes": (sz, [i32, i32]),
                "focr_rswa_decode": (i32, [P, P, P, P, P, P, i32, P, P, P, i32, P, P, sz, P]),
                "focr_last_error": (ctypes.c_char_p, []),
                "focr_version": (ctypes.c_char_p, []),
            }
            for name, (res, args) in sigs.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _check(status: int):
    if status != 0:
        raise FocrError(status, lib().focr_last_error().decode())


def _stream(stream=None) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t) -> int | None:
    if t is None:
        return None
    return int(t.data_ptr())


def focr_last_error() -> str:
    return lib().focr_last_error().decode()


def focr_version() -> str:
    return lib().focr_version().decode()


class MoELayer:
    """A packed, device-resident MoE layer (owns its device memory)."""

    def __init__(self, handle: int):
        self.handle = handle

    def __del__(self):
        h, self.handle = getattr(self, "handle", None), None
        if h and _lib is not None:
            _lib.focr_moe_layer_free(ctypes.c_void_p(h))

    @property
    def device_bytes(self) -> int:
        return lib().focr_moe_layer_device_bytes(ctypes.c_void_p(self.handle))


def focr_moe_pack_weights(layer: "synth.MoELayerInputs", stream=None) -> MoELayer:
    arrs = [np.ascontiguousarray(a, np.float32) for a in
            (layer.gate, layer.up, layer.down, layer.sgate, layer.sup, layer.sdown)]
    router = np.ascontiguousarray(layer.router_bf16, np.uint16)
    assert arrs[0].shape == (E, I, H) and arrs[2].shape == (E, H, I) and arrs[3].shape == (IS, H)
    desc = WeightsDesc(*[a.ctypes.data for a in arrs], router.ctypes.data,
                       int(layer.routed_type), int(layer.shared_type), int(layer.group))
    h = ctypes.c_void_p()
    _check(lib().focr_moe_pack_weights(ctypes.byref(desc), ctypes.byref(h), _stream(stream)))
    return MoELayer(h.value)


def focr_moe_layer_clone(layer: MoELayer, stream=None) -> MoELayer:
    h = ctypes.c_void_p()
    _check(lib().focr_moe_layer_clone(ctypes.c_void_p(layer.handle), ctypes.byref(h), _stream(stream)))
    return MoELayer(h.value)


def focr_moe_export_quantized(layer: MoELayer, matrix: int, expert: int = 0):
    """Canonical codes (bytes as np.uint8 / int8 / uint16) and f32 scales of one matrix."""
    L = lib()
    cb, ns = ctypes.c_size_t(), ctypes.c_size_t()
    _check(L.focr_moe_export_sizes(ctypes.c_void_p(layer.handle), matrix, ctypes.byref(cb), ctypes.byref(ns)))
    codes = np.empty(cb.value, np.uint8)
    scales = np.empty(ns.value, np.float32)
    _check(L.focr_moe_export_quantized(ctypes.c_void_p(layer.handle), matrix, expert, codes.ctypes.data, cb.value,
                                       scales.ctypes.data if ns.value else None, ns.value))
    return codes, scales


def focr_moe_workspace_bytes(T_max: int) -> int:
    return int(lib().focr_moe_workspace_bytes(int(T_max)))


def focr_moe_workspace_zero_bytes() -> int:
    """Bytes at the start of a workspace that are zero between forwards."""
    return int(lib().focr_moe_workspace_zero_bytes())


def new_workspace(T_max: int, device="cuda"):
    """A zero-filled workspace tensor for forwards with up to T_max tokens."""
    import torch
    return torch.zeros(focr_moe_workspace_bytes(T_max), dtype=torch.uint8, device=device)


def focr_moe_layer_forward(layer: MoELayer, hidden, out=None, workspace=None, debug: dict | None = None,
                           stream=None, flags: int = 0):
    """out[T, 1280] = MoE(hidden[T, 1280]) on the current (or given) stream.
    `debug`, if given, maps names of focr_moe_route_debug fields to device tensors to fill."""
    import torch
    assert hidden.is_cuda and hidden.dtype == torch.float32 and hidden.is_contiguous() and hidden.shape[-1] == H
    T = hidden.shape[0]
    if out is None:
        out = torch.empty_like(hidden)
    if workspace is None:
        workspace = new_workspace(T, hidden.device)
    dbg = None
    if debug:
        dbg = RouteDebug(*[_ptr(debug.get(f)) for f, _ in RouteDebug._fields_])
    _check(lib().focr_moe_layer_forward_ex(ctypes.c_void_p(layer.handle), _ptr(hidden), T, _ptr(out),
                                           _ptr(workspace), workspace.numel(),
                                           ctypes.byref(dbg) if dbg is not None else None, int(flags),
                                           _stream(stream)))
    return out


def focr_moe_layer_forward_noalloc(layer: MoELayer, hidden, out=None, debug: dict | None = None, stream=None):
    """The forward for callers that cannot allocate device memory: the library's own fixed
    scratch array replaces the workspace (T <= NOALLOC_T_MAX; calls must not overlap)."""
    import torch
    assert hidden.is_cuda and hidden.dtype == torch.float32 and hidden.is_contiguous() and hidden.shape[-1] == H
    T = hidden.shape[0]
    if out is None:
        out = torch.empty_like(hidden)
    dbg = None
    if debug:
        dbg = RouteDebug(*[_ptr(debug.get(f)) for f, _ in RouteDebug._fields_])
    _check(lib().focr_moe_layer_forward_noalloc(ctypes.c_void_p(layer.handle), _ptr(hidden), T, _ptr(out),
                                                ctypes.byref(dbg) if dbg is not None else None, _stream(stream)))
    return out


def focr_moe_check_noalloc(stream=None):
    """Report (FocrError TIMEOUT) a device wait of an earlier allocation-free forward that ran out."""
    _check(lib().focr_moe_check_noalloc(_stream(stream)))


def focr_moe_check(workspace, stream=None):
    _check(lib().focr_moe_check(_ptr(workspace), _stream(stream)))


# ---------------------------------------------------------------- decode-step companions

class LMHead:
    """A packed int8 lm_head (owns its device memory)."""

    def __init__(self, handle: int):
        self.handle = handle

    def __del__(self):
        h, self.handle = getattr(self, "handle", None), None
        if h and _lib is not None:
            _lib.focr_lm_head_free(ctypes.c_void_p(h))


def focr_lm_head_pack(w, stream=None) -> LMHead:
    w = np.ascontiguousarray(w, np.float32)
    assert w.shape == (VOCAB, H)
    h = ctypes.c_void_p()
    _check(lib().focr_lm_head_pack(w.ctypes.data, ctypes.byref(h), _stream(stream)))
    return LMHead(h.value)


def focr_lm_head_export(head: LMHead):
    codes = np.empty((VOCAB, H), np.int8)
    scales = np.empty(VOCAB, np.float32)
    _check(lib().focr_lm_head_export(ctypes.c_void_p(head.handle), codes.ctypes.data, scales.ctypes.data))
    return codes, scales


def focr_lm_head_workspace_bytes(T_max: int) -> int:
    return int(lib().focr_lm_head_workspace_bytes(int(T_max)))


def focr_lm_head_gemv(head: LMHead, x, argmax=None, logits=None, workspace=None, stream=None):
    """argmax[T] (int32) and optionally logits[T, 129280] of the int8 lm_head."""
    import torch
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous() and x.shape[-1] == H
    T = x.shape[0]
    if argmax is None:
        argmax = torch.empty(T, dtype=torch.int32, device=x.device)
    if workspace is None:
        workspace = torch.zeros(focr_lm_head_workspace_bytes(T), dtype=torch.uint8, device=x.device)
    _check(lib().focr_lm_head_gemv(ctypes.c_void_p(head.handle), _ptr(x), T, _ptr(logits), _ptr(argmax),
                                   _ptr(workspace), workspace.numel(), _stream(stream)))
    return argmax


# ---------------------------------------------------------------- W8A8 linear

W8A8_T_MAX = 64
W8A8_K_MAX = 133143


class W8A8:
    """A packed int8 matrix with one scale per row, for the W8A8 GEMV (owns its device memory)."""

    def __init__(self, handle: int, N: int, K: int):
        self.handle, self.N, self.K = handle, N, K

    def __del__(self):
        h, self.handle = getattr(self, "handle", None), None
        if h and _lib is not None:
            _lib.focr_w8a8_free(ctypes.c_void_p(h))


def focr_w8a8_pack(w, stream=None) -> W8A8:
    w = np.ascontiguousarray(w, np.float32)
    N, K = w.shape
    h = ctypes.c_void_p()
    _check(lib().focr_w8a8_pack(w.ctypes.data, N, K, ctypes.byref(h), _stream(stream)))
    return W8A8(h.value, N, K)


def focr_w8a8_export(m: W8A8):
    codes = np.empty((m.N, m.K), np.int8)
    scales = np.empty(m.N, np.float32)
    n, k = ctypes.c_int64(), ctypes.c_int32()
    _check(lib().focr_w8a8_export(ctypes.c_void_p(m.handle), codes.ctypes.data, scales.ctypes.data,
                                  ctypes.byref(n), ctypes.byref(k)))
    assert (n.value, k.value) == (m.N, m.K)
    return codes, scales


def focr_w8a8_quantize_x(x, stream=None):
    """Per-token int8 codes [T, K] and fp32 scales [T] of x (DEVICE fp32 [T, K])."""
    import torch
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous() and x.dim() == 2
    T, K = x.shape
    qx = torch.empty(T, K, dtype=torch.int8, device=x.device)
    sx = torch.empty(T, dtype=torch.float32, device=x.device)
    _check(lib().focr_w8a8_quantize_x(_ptr(x), T, K, _ptr(qx), _ptr(sx), _stream(stream)))
    return qx, sx


def focr_w8a8_workspace_bytes(m: W8A8, T_max: int) -> int:
    return int(lib().focr_w8a8_workspace_bytes(ctypes.c_void_p(m.handle), int(T_max)))


def focr_w8a8_gemv(m: W8A8, x, y=None, workspace=None, stream=None):
    """y[T, N] = W8A8(m, x) for x DEVICE fp32 [T, K]."""
    import torch
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous() and x.shape[-1] == m.K
    T = x.shape[0]
    if y is None:
        y = torch.empty(T, m.N, dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = torch.zeros(focr_w8a8_workspace_bytes(m, T), dtype=torch.uint8, device=x.device)
    _check(lib().focr_w8a8_gemv(ctypes.c_void_p(m.handle), _ptr(x), T, _ptr(y), _ptr(workspace),
                                workspace.numel(), _stream(stream)))
    return y


def focr_lm_head_check(workspace, stream=None):
    _check(lib().focr_lm_head_check(_ptr(workspace), _stream(stream)))


def focr_w8a8_check(workspace, stream=None):
    _check(lib().focr_w8a8_check(_ptr(workspace), _stream(stream)))


# ---------------------------------------------------------------- R-SWA decode attention

RSWA_HEADS, RSWA_DIM, RSWA_RING = 10, 128, 128


def focr_rswa_workspace_bytes(B: int, Rcap: int) -> int:
    return int(lib().focr_rswa_workspace_bytes(int(B), int(Rcap)))


def focr_rswa_decode(q, k_new, v_new, k_ref, v_ref, ref_len, k_ring, v_ring, n_gen, out=None, workspace=None,
                     stream=None):
    """out [B, 10, 128]: one R-SWA decode step; k_ring / v_ring [B, 10, 128, 128] get the current token."""
    import torch
    B, H, D = q.shape
    Rcap = k_ref.shape[2]
    for t in (q, k_new, v_new, k_ref, v_ref, k_ring, v_ring):
        assert t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()
    assert (H, D) == (RSWA_HEADS, RSWA_DIM) and k_ring.shape == (B, H, RSWA_RING, D) and v_ref.shape == k_ref.shape
    assert ref_len.dtype == torch.int32 and n_gen.dtype == torch.int32 and ref_len.is_cuda and n_gen.is_cuda
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.empty(focr_rswa_workspace_bytes(B, Rcap), dtype=torch.uint8, device=q.device)
    _check(lib().focr_rswa_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_ref), _ptr(v_ref), _ptr(ref_len), Rcap,
                                  _ptr(k_ring), _ptr(v_ring), _ptr(n_gen), B, _ptr(out), _ptr(workspace),
                                  workspace.numel(), _stream(stream)))
    return out


def focr_rmsnorm(x, gamma=None, eps: float = 1e-6, out=None, stream=None):
    import torch
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous() and x.shape[-1] == H
    if out is None:
        out = torch.empty_like(x)
    _check(lib().focr_rmsnorm(_ptr(x), _ptr(gamma), x.shape[0], float(eps), _ptr(out), _stream(stream)))
    return out


class DenseMLP:
    """A packed dense SwiGLU MLP (decoder layer 0; owns its device memory)."""

    def __init__(self, handle: int, wtype: int, group: int):
        self.handle, self.wtype, self.group = handle, wtype, group

    def __del__(self):
        h, self.handle = getattr(self, "handle", None), None
        if h and _lib is not None:
            _lib.focr_dense_mlp_free(ctypes.c_void_p(h))


def focr_dense_mlp_pack(gate, up, down, wtype: int = W_INT8, group: int = 128, stream=None) -> DenseMLP:
    arrs = [np.ascontiguousarray(a, np.float32) for a in (gate, up, down)]
    assert arrs[0].shape == (DENSE_I, H) and arrs[2].shape == (H, DENSE_I)
    h = ctypes.c_void_p()
    _check(lib().focr_dense_mlp_pack(arrs[0].ctypes.data, arrs[1].ctypes.data, arrs[2].ctypes.data, int(wtype),
                                     int(group), ctypes.byref(h), _stream(stream)))
    return DenseMLP(h.value, wtype, group)


def focr_dense_mlp_export_quantized(mlp: DenseMLP, matrix: int):
    rows, cols = (DENSE_I, H) if matrix < 2 else (H, DENSE_I)
    n = rows * cols
    cb = n // 2 if mlp.wtype == W_INT4 else (n if mlp.wtype == W_INT8 else 2 * n)
    ns = rows * ((cols + mlp.group - 1) // mlp.group) if mlp.wtype != W_BF16 else 0
    codes = np.empty(cb, np.uint8)
    scales = np.empty(ns, np.float32)
    _check(lib().focr_dense_mlp_export_quantized(ctypes.c_void_p(mlp.handle), matrix, codes.ctypes.data, cb,
                                                 scales.ctypes.data if ns else None, ns))
    return codes, scales


def focr_dense_mlp_forward(mlp: DenseMLP, x, out=None, workspace=None, flags: int = 0, stream=None):
    import torch
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous() and x.shape[-1] == H
    T = x.shape[0]
    if out is None:
        out = torch.empty_like(x)
    if workspace is None:
        workspace = new_workspace(T, x.device)
    _check(lib().focr_dense_mlp_forward(ctypes.c_void_p(mlp.handle), _ptr(x), T, _ptr(out), _ptr(workspace),
                                        workspace.numel(), int(flags), _stream(stream)))
    return out


def focr_tc_selftest(a, b, a_from_tmem: bool, stream=None):
    """D = a @ b.T (fp32) through the library's tcgen05 tile primitives; a [128, k], b [n, k] bf16
    device tensors.  Returns (D, err) with err nonzero if the kernel's bounded wait ran out."""
    import torch
    assert a.dtype == torch.bfloat16 and b.dtype == torch.bfloat16 and a.is_cuda and b.is_cuda
    n, k = b.shape
    d = torch.empty(128, n, dtype=torch.float32, device=a.device)
    err = torch.zeros(1, dtype=torch.int32, device=a.device)
    _check(lib().focr_tc_selftest(_ptr(a), _ptr(b), n, k, int(a_from_tmem), _ptr(d), _ptr(err), _stream(stream)))
    return d, err


# ---------------------------------------------------------------- decode step
class DecodeModel:
    """Handles of one decoder stack for focr_decode_step: the dense layer 0, the MoE layers, the
    RMSNorm weights (device tensors [1280] or None for ones) and the lm_head.  Keeps the
    Python objects alive; owns no device memory of its own."""

    def __init__(self, dense: "DenseMLP", moe_layers, head: LMHead, gammas=None, eps: float = 1e-6):
        self.dense, self.moe, self.head, self.gammas, self.eps = dense, list(moe_layers), head, gammas, float(eps)
        self._moe = (ctypes.c_void_p * max(1, len(self.moe)))(*[m.handle for m in self.moe])
        self._gam = None
        if gammas is not None:
            assert len(gammas) == len(self.moe) + 1
            self._gam = (ctypes.c_void_p * len(gammas))(*[_ptr(g) for g in gammas])
        self.desc = DecodeModelDesc(dense.handle, ctypes.cast(self._moe, ctypes.POINTER(ctypes.c_void_p)),
                                    len(self.moe),
                                    ctypes.cast(self._gam, ctypes.POINTER(ctypes.c_void_p)) if self._gam else None,
                                    self.eps, head.handle)


def new_decode_step_workspace(T_max: int, device=None):
    """A zero-filled workspace for focr_decode_step calls with up to T_max tokens."""
    import torch
    n = lib().focr_decode_step_workspace_bytes(T_max)
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def focr_decode_step(model: DecodeModel, x, argmax=None, logits=None, hidden_out=None, workspace=None, stream=None):
    """One decode step of the stack (dense layer 0, MoE layers, RMSNorms, lm_head + argmax).
    Returns argmax [T] int32 (device)."""
    import torch
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous() and x.shape[-1] == H
    T = x.shape[0]
    if argmax is None:
        argmax = torch.empty(T, dtype=torch.int32, device=x.device)
    if workspace is None:
        workspace = new_decode_step_workspace(T, x.device)
    _check(lib().focr_decode_step(ctypes.byref(model.desc), _ptr(x), T, _ptr(logits), _ptr(argmax), _ptr(hidden_out),
                                  _ptr(workspace), workspace.numel(), _stream(stream)))
    return argmax
