"""CPU oracle for the group-quantised MoE layer -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  The product (the CUDA library and its Python binding)
never does.  The arithmetic lives in ``focr_oracle.c`` (plain loops, fp64
accumulation); this file only marshals numpy arrays into it.

Every function cites its source inside the C file.  Parity pins for each of
them are in the CPU tests (``tests/test_oracle_pins.py``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "focr_oracle.c")
_SO = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None

ORC_DENSE, ORC_QUANT = 0, 1
W_BF16, W_INT8, W_INT4 = 0, 1, 2


def compile_to(src: str, out: str) -> str:
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-o", out, src, "-lm"]
    subprocess.check_call(cmd)
    return out


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain C, no fast-math, no FMA contraction).
    FOCR_ORACLE_SO names a prebuilt copy instead (the mutation tests use it to
    load a deliberately broken oracle in a child process)."""
    override = os.environ.get("FOCR_ORACLE_SO")
    if override:
        return override
    if not force and os.path.exists(_SO) and os.path.getmtime(_SO) >= os.path.getmtime(_SRC):
        return _SO
    os.makedirs(os.path.dirname(_SO), exist_ok=True)
    tmp = _SO + f".tmp{os.getpid()}"
    compile_to(_SRC, tmp)
    os.replace(tmp, _SO)
    return _SO


class Mat(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("group", ctypes.c_int32),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("f", ctypes.c_void_p), ("q", ctypes.c_void_p), ("s", ctypes.c_void_p)]


class Moe(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("Is", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("router", ctypes.c_void_p),
                ("gate", Mat), ("up", Mat), ("down", Mat),
                ("sgate", Mat), ("sup", Mat), ("sdown", Mat)]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            P, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
            L.orc_bf16_to_f32.restype = ctypes.c_float
            L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
            L.orc_f32_to_bf16.restype = ctypes.c_uint16
            L.orc_f32_to_bf16.argtypes = [ctypes.c_float]
            L.orc_round_bf16_array.argtypes = [P, i64, P]
            L.orc_num_groups.restype = i64
            L.orc_num_groups.argtypes = [i64, ctypes.c_int]
            L.orc_quantize_rows.argtypes = [P, i64, i64, ctypes.c_int, ctypes.c_int, P, P]
            L.orc_nibble_pack.argtypes = [P, i64, P]
            L.orc_nibble_unpack.argtypes = [P, i64, P]
            L.orc_gemv.argtypes = [ctypes.POINTER(Mat), P, P]
            L.orc_swiglu.argtypes = [ctypes.POINTER(Mat)] * 3 + [P, P]
            L.orc_router_logits.argtypes = [P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P]
            L.orc_softmax_topk.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
            L.orc_dispatch.argtypes = [P, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P]
            L.orc_moe_forward.argtypes = [ctypes.POINTER(Moe), P, ctypes.c_int, P, P, P, P, P, P, P,
                                          ctypes.c_int]
            L.orc_dense_mlp.argtypes = [ctypes.POINTER(Mat)] * 3 + [P, ctypes.c_int, P, ctypes.c_int]
            L.orc_rmsnorm.argtypes = [P, ctypes.c_int, ctypes.c_int, P, dbl, P]
            L.orc_lm_head.argtypes = [P, P, P, ctypes.c_int, i64, ctypes.c_int, P, P, ctypes.c_int]
            L.orc_w8a8_quantize_x.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P]
            L.orc_w8a8_gemv.argtypes = [P, P, i64, ctypes.c_int, P, P, ctypes.c_int, P, P]
            L.orc_rswa_decode.argtypes = [P, P, P, P, P, P, ctypes.c_int, P, P, P] + [ctypes.c_int] * 4 + [P]
            L.orc_max_threads.restype = ctypes.c_int
            for name in ("orc_round_bf16_array", "orc_quantize_rows", "orc_nibble_pack",
                         "orc_nibble_unpack", "orc_gemv", "orc_swiglu", "orc_router_logits",
                         "orc_softmax_topk", "orc_dispatch", "orc_moe_forward", "orc_dense_mlp",
                         "orc_rmsnorm", "orc_lm_head", "orc_w8a8_quantize_x", "orc_w8a8_gemv",
                         "orc_rswa_decode"):
                getattr(L, name).restype = None
            _lib = L
    return _lib


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- formats

def f32_to_bf16(a) -> np.ndarray:
    a = _c(a, np.float32).reshape(-1)
    L = lib()
    return np.array([L.orc_f32_to_bf16(float(v)) for v in a], dtype=np.uint16)


def round_bf16(a) -> np.ndarray:
    a = _c(a, np.float32)
    out = np.empty_like(a)
    lib().orc_round_bf16_array(_p(a), a.size, _p(out))
    return out


def bf16_to_f32(b) -> np.ndarray:
    b = _c(b, np.uint16).reshape(-1)
    L = lib()
    return np.array([L.orc_bf16_to_f32(int(v)) for v in b], dtype=np.float32)


def quantize_rows(w, group: int, bits: int):
    """Group-quantise each row of a 2-D fp32 matrix.  Returns (q int8 [rows, cols],
    scales f32 [rows, ceil(cols / group)])."""
    w = _c(w, np.float32)
    assert w.ndim == 2
    rows, cols = w.shape
    ng = (cols + group - 1) // group
    q = np.empty((rows, cols), dtype=np.int8)
    s = np.empty((rows, ng), dtype=np.float32)
    lib().orc_quantize_rows(_p(w), rows, cols, group, bits, _p(q), _p(s))
    return q, s


def nibble_pack(q) -> np.ndarray:
    q = _c(q, np.int8).reshape(-1)
    assert q.size % 2 == 0
    out = np.empty(q.size // 2, dtype=np.uint8)
    lib().orc_nibble_pack(_p(q), q.size, _p(out))
    return out


def nibble_unpack(packed, n: int) -> np.ndarray:
    packed = _c(packed, np.uint8).reshape(-1)
    q = np.empty(n, dtype=np.int8)
    lib().orc_nibble_unpack(_p(packed), n, _p(q))
    return q


# ---------------------------------------------------------------- matrices

class OMat:
    """A weight matrix in the oracle's form: bf16-rounded fp32 values, or int codes
    plus f32 group scales.  Keeps its arrays alive for the C struct."""

    def __init__(self, w, wtype: int, group: int = 0):
        w = _c(w, np.float32)
        assert w.ndim == 2
        self.rows, self.cols = w.shape
        self.wtype, self.group = wtype, group
        if wtype == W_BF16:
            self.f = round_bf16(w)
            self.q = self.s = None
        else:
            self.f = None
            self.q, self.s = quantize_rows(w, group, 4 if wtype == W_INT4 else 8)

    def struct(self) -> Mat:
        if self.f is not None:
            return Mat(ORC_DENSE, 0, self.rows, self.cols, _p(self.f), None, None)
        return Mat(ORC_QUANT, self.group, self.rows, self.cols, None, _p(self.q), _p(self.s))

    def dequant(self) -> np.ndarray:
        """fp64 values q*s (or the bf16 values) -- for the numpy cross-checks."""
        if self.f is not None:
            return self.f.astype(np.float64)
        ng = self.s.shape[1]
        sc = np.repeat(self.s.astype(np.float64), self.group, axis=1)[:, :self.cols]
        assert ng * self.group >= self.cols
        return self.q.astype(np.float64) * sc


def gemv(m: OMat, x) -> np.ndarray:
    x = _c(x, np.float64)
    y = np.empty(m.rows, dtype=np.float64)
    st = m.struct()
    lib().orc_gemv(ctypes.byref(st), _p(x), _p(y))
    return y


def swiglu(G: OMat, U: OMat, D: OMat, x) -> np.ndarray:
    x = _c(x, np.float64)
    y = np.empty(D.rows, dtype=np.float64)
    g, u, d = G.struct(), U.struct(), D.struct()
    lib().orc_swiglu(ctypes.byref(g), ctypes.byref(u), ctypes.byref(d), _p(x), _p(y))
    return y


# ---------------------------------------------------------------- router

def router_logits(x, router_bf16) -> np.ndarray:
    x = _c(x, np.float32)
    wr = _c(router_bf16, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    out = np.empty((T, E), dtype=np.float32)
    lib().orc_router_logits(_p(x), _p(wr), T, H, E, _p(out))
    return out


def softmax_topk(logits, k: int):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    p = np.empty((T, E), dtype=np.float64)
    lib().orc_softmax_topk(_p(logits), T, E, k, _p(idx), _p(w), _p(p))
    return idx, w, p


def dispatch(idx, E: int):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(T * k, dtype=np.int32)
    lib().orc_dispatch(_p(idx), T, k, E, _p(counts), _p(offsets), _p(perm))
    return counts, offsets, perm


# ---------------------------------------------------------------- MoE layer

class OracleMoE:
    """The oracle's copy of one MoE layer, quantised by the oracle's own quantiser."""

    def __init__(self, layer, topk: int = 6):
        E, I, H = layer.gate.shape
        self.E, self.I, self.H, self.topk = E, I, H, topk
        self.Is = layer.sgate.shape[0]
        self.router = _c(layer.router_bf16, np.uint16)
        rt, st, g = layer.routed_type, layer.shared_type, layer.group
        self.gate = OMat(layer.gate.reshape(E * I, H), rt, g)
        self.up = OMat(layer.up.reshape(E * I, H), rt, g)
        self.down = OMat(layer.down.reshape(E * H, I), rt, g)
        self.sgate = OMat(layer.sgate, st, g if st != W_BF16 else 0)
        self.sup = OMat(layer.sup, st, g if st != W_BF16 else 0)
        self.sdown = OMat(layer.sdown, st, g if st != W_BF16 else 0)

    def struct(self) -> Moe:
        return Moe(self.E, self.H, self.I, self.Is, self.topk, _p(self.router),
                   self.gate.struct(), self.up.struct(), self.down.struct(),
                   self.sgate.struct(), self.sup.struct(), self.sdown.struct())

    def forward(self, x, nthreads: int = 1) -> dict:
        x = _c(x, np.float32)
        T = x.shape[0]
        r = dict(out=np.empty((T, self.H), np.float32),
                 logits=np.empty((T, self.E), np.float32),
                 idx=np.empty((T, self.topk), np.int32),
                 w=np.empty((T, self.topk), np.float64),
                 counts=np.empty(self.E, np.int32),
                 offsets=np.empty(self.E + 1, np.int32),
                 perm=np.empty(T * self.topk, np.int32))
        st = self.struct()
        lib().orc_moe_forward(ctypes.byref(st), _p(x), T, _p(r["out"]), _p(r["logits"]),
                              _p(r["idx"]), _p(r["w"]), _p(r["counts"]), _p(r["offsets"]),
                              _p(r["perm"]), nthreads)
        return r


# ---------------------------------------------------------------- companions

class OracleDense:
    def __init__(self, gate, up, down, wtype: int = W_INT8, group: int = 128):
        self.G, self.U, self.D = OMat(gate, wtype, group), OMat(up, wtype, group), OMat(down, wtype, group)

    def forward(self, x, nthreads: int = 1) -> np.ndarray:
        x = _c(x, np.float32)
        T = x.shape[0]
        out = np.empty((T, self.D.rows), np.float32)
        g, u, d = self.G.struct(), self.U.struct(), self.D.struct()
        lib().orc_dense_mlp(ctypes.byref(g), ctypes.byref(u), ctypes.byref(d), _p(x), T, _p(out), nthreads)
        return out


def rmsnorm(x, gamma=None, eps: float = 1e-6) -> np.ndarray:
    x = _c(x, np.float32)
    T, H = x.shape
    g = None if gamma is None else _c(gamma, np.float32)
    out = np.empty_like(x)
    lib().orc_rmsnorm(_p(x), T, H, _p(g), eps, _p(out))
    return out


class OracleLMHead:
    """int8 lm_head with one scale per row (a group spanning the whole row)."""

    def __init__(self, w):
        self.q, s = quantize_rows(w, w.shape[1], 8)
        self.s = np.ascontiguousarray(s[:, 0])
        self.V, self.H = self.q.shape

    def forward(self, x, want_logits: bool = False, nthreads: int = 1):
        x = _c(x, np.float32)
        T = x.shape[0]
        logits = np.empty((T, self.V), np.float32) if want_logits else None
        am = np.empty(T, np.int32)
        lib().orc_lm_head(_p(self.q), _p(self.s), _p(x), T, self.V, self.H, _p(logits), _p(am), nthreads)
        return am, logits


def w8a8_quantize_x(x):
    """Per-token int8 activations and their fp32 scales ([P4-cpu] quantise-plus-GEMV)."""
    x = _c(x, np.float32)
    T, K = x.shape
    qx = np.empty((T, K), np.int8)
    sx = np.empty(T, np.float32)
    lib().orc_w8a8_quantize_x(_p(x), T, K, _p(qx), _p(sx))
    return qx, sx


class OracleW8A8:
    """An int8 weight matrix with one scale per row, applied to per-token int8 activations."""

    def __init__(self, w):
        w = _c(w, np.float32)
        self.N, self.K = w.shape
        q, s = quantize_rows(w, self.K, 8)
        self.q, self.s = q, np.ascontiguousarray(s[:, 0])

    def forward(self, x, want_acc: bool = False):
        qx, sx = w8a8_quantize_x(x)
        T = qx.shape[0]
        y = np.empty((T, self.N), np.float32)
        acc = np.empty((T, self.N), np.int64) if want_acc else None
        lib().orc_w8a8_gemv(_p(self.q), _p(self.s), self.N, self.K, _p(qx), _p(sx), T, _p(y), _p(acc))
        return (y, qx, sx, acc) if want_acc else (y, qx, sx)


RSWA_HEADS, RSWA_DIM, RSWA_RING = 10, 128, 128


def rswa_decode(q, k_new, v_new, k_ref, v_ref, ref_len, k_ring, v_ring, n_gen, W: int = RSWA_RING):
    """One R-SWA decode step ([P4-rswa]).  q, k_new, v_new [B, H, D]; k_ref, v_ref [B, H, Rcap, D];
    k_ring, v_ring [B, H, W, D]; ref_len, n_gen [B].  Returns (out [B, H, D], k_ring', v_ring')."""
    q, k_new, v_new = (_c(a, np.float32) for a in (q, k_new, v_new))
    k_ref, v_ref = _c(k_ref, np.float32), _c(v_ref, np.float32)
    k_ring, v_ring = np.array(k_ring, np.float32, copy=True), np.array(v_ring, np.float32, copy=True)
    ref_len, n_gen = _c(ref_len, np.int32), _c(n_gen, np.int32)
    B, H, D = q.shape
    Rcap = k_ref.shape[2]
    assert k_ring.shape == (B, H, W, D) and v_ref.shape == k_ref.shape
    out = np.empty((B, H, D), np.float32)
    lib().orc_rswa_decode(_p(q), _p(k_new), _p(v_new), _p(k_ref), _p(v_ref), _p(ref_len), Rcap, _p(k_ring),
                          _p(v_ring), _p(n_gen), B, H, D, W, _p(out))
    return out, k_ring, v_ring


def max_threads() -> int:
    return lib().orc_max_threads()
