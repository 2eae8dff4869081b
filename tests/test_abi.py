"""The C-ABI library builds, loads without a GPU, exports every declared symbol,
and rejects bad arguments before launching anything."""
import ctypes
import glob
import os
import re

import pytest

from weight_quantized_expert_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(focr_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return names


def test_library_builds_and_loads():
    path = build.build()
    assert os.path.exists(path)
    assert api.focr_version().startswith("focr_moe sm_100a")


def test_every_declared_symbol_is_exported():
    declared = _declared_symbols()
    assert {"focr_moe_pack_weights", "focr_moe_layer_forward", "focr_moe_export_quantized"} <= declared
    L = api.lib()
    for name in sorted(declared):
        assert hasattr(L, name), f"{name} declared in include/ but not exported"
    assert declared == set(api.EXPORTED), "binding and header disagree"


def test_workspace_size_grows_with_tokens():
    sizes = [api.focr_moe_workspace_bytes(t) for t in (1, 8, 289, 8192)]
    assert all(s % 256 == 0 for s in sizes)
    assert sizes == sorted(sizes) and sizes[0] < sizes[-1]
    # clamped outside [1, T_MAX]
    assert api.focr_moe_workspace_bytes(0) == sizes[0]
    assert api.focr_moe_workspace_bytes(10 ** 6) == sizes[-1]
    # the zero-on-entry prefix is the same for every T and lies inside every workspace
    z = api.focr_moe_workspace_zero_bytes()
    assert 0 < z < sizes[0] and z % 256 == 0


def test_forward_rejects_bad_arguments_without_launching():
    L = api.lib()
    ws = ctypes.create_string_buffer(1 << 16)
    st = L.focr_moe_layer_forward(None, None, 1, None, None, 0, None, None)
    assert st == 1 and "layer" in api.focr_last_error()


def test_pack_rejects_null_and_unsupported_types():
    L = api.lib()
    h = ctypes.c_void_p()
    assert L.focr_moe_pack_weights(None, ctypes.byref(h), None) == 1
    dummy = (ctypes.c_float * 4)()
    router = (ctypes.c_uint16 * 4)()
    p = ctypes.cast(dummy, ctypes.c_void_p).value
    r = ctypes.cast(router, ctypes.c_void_p).value
    for rt, st_, g in ((api.W_INT4, api.W_BF16, 48), (api.W_INT8, api.W_BF16, 64), (7, api.W_BF16, 64),
                       (api.W_INT4, 9, 64)):
        desc = api.WeightsDesc(p, p, p, p, p, p, r, rt, st_, g)
        assert L.focr_moe_pack_weights(ctypes.byref(desc), ctypes.byref(h), None) == 2
        assert "not supported" in api.focr_last_error()
        assert not h.value
    desc = api.WeightsDesc(p, None, p, p, p, p, r, api.W_INT4, api.W_BF16, 64)
    assert L.focr_moe_pack_weights(ctypes.byref(desc), ctypes.byref(h), None) == 1


def test_export_and_check_reject_null():
    L = api.lib()
    a, b = ctypes.c_size_t(), ctypes.c_size_t()
    assert L.focr_moe_export_sizes(None, 0, ctypes.byref(a), ctypes.byref(b)) == 1
    assert L.focr_moe_check(None, None) == 1


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(api, "LIB_PATH", str(tmp_path / "nope.so"))
    monkeypatch.setattr(api, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        api.lib()


def test_w8a8_rejects_bad_arguments_without_launching():
    L = api.lib()
    h = ctypes.c_void_p()
    w = (ctypes.c_float * 16)()
    p = ctypes.cast(w, ctypes.c_void_p).value
    assert L.focr_w8a8_pack(None, 1, 1, ctypes.byref(h), None) == 1
    for n, k in ((0, 16), (1, 0), (1, api.W8A8_K_MAX + 1), (1 << 27, 16)):
        assert L.focr_w8a8_pack(p, n, k, ctypes.byref(h), None) == 1
        assert "outside" in api.focr_last_error() and not h.value
    assert L.focr_w8a8_gemv(None, p, 1, p, p, 1 << 20, None) == 1
    assert L.focr_w8a8_workspace_bytes(None, 1) == 0
    assert L.focr_w8a8_export(None, None, None, None, None) == 1
    q = (ctypes.c_int8 * 16)()
    qp = ctypes.cast(q, ctypes.c_void_p).value
    for T, K in ((0, 16), (api.T_MAX + 1, 16), (1, 0),
                 (1, api.W8A8_K_MAX + 1)):
        assert L.focr_w8a8_quantize_x(p, T, K, qp, p, None) == 1


def test_rswa_workspace_and_argument_checks_without_launching():
    L = api.lib()
    assert api.focr_rswa_workspace_bytes(1, 289) % 256 == 0
    assert api.focr_rswa_workspace_bytes(8, 289) >= api.focr_rswa_workspace_bytes(1, 289)
    buf = (ctypes.c_float * 64)()
    p = ctypes.cast(buf, ctypes.c_void_p).value
    assert L.focr_rswa_decode(None, p, p, p, p, p, 1, p, p, p, 1, p, p, 1 << 20, None) == 1
    assert L.focr_rswa_decode(p, p, p, p, p, p, 0, p, p, p, 1, p, p, 1 << 20, None) == 1
    assert L.focr_rswa_decode(p, p, p, p, p, p, 1, p, p, p, 5000, p, p, 1 << 20, None) == 1
