"""Parity of the CUDA MoE layer against the CPU oracle, through the C ABI.

Bit-exact: the canonical quantised codes and scales, router expert indices, the
dispatch (counts, offsets, permutation).  Floating point: the layer output within a
per-token relative error (max |gpu - oracle| / max |oracle| over the 1280 outputs of a
token) of 2e-3 on the mma.sync kernels (T <= 64: f16 activations, fp32 accumulation) and
1e-2 on the tensor-core path (T > 64: f16 gate/up and bf16 down operands in tcgen05 MMAs,
fp32 accumulation), router weights within 1e-5.
"""
import functools
import os

import numpy as np
import pytest

import oracle
from conftest import moe_case, per_token_rel_err
from weight_quantized_expert_b200 import api, synth

pytestmark = pytest.mark.gpu
NTHREADS = max(1, (os.cpu_count() or 1))
TOL_DECODE = 2e-3   # T <= 64: the mma.sync kernels (f16 activations, fp32 accumulation)
TOL_TC = 1e-2       # T > 64: the tensor-core kernel (f16 gate/up, bf16 down operands, fp32 accumulation)
MID_T = 64


def tol_for(T):
    return TOL_DECODE if T <= MID_T else TOL_TC

W4, W8, WB = synth.W_INT4, synth.W_INT8, synth.W_BF16
LAYERS = {
    "int8_g128": (0, W8, W8, 128, False),
    "int4_g32": (1, W4, WB, 32, False),
    "int4_g64": (1, W4, WB, 64, False),
    "int4_g128": (1, W4, WB, 128, False),
    "int4_g64_skew": (2, W4, WB, 64, True),
    "int4_g64_prefill": (3, W4, WB, 64, False),
}


def _torch():
    import torch
    return torch


def run_gpu(packed, x, ws=None):
    torch = _torch()
    T = x.shape[0]
    xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    dbg = dict(logits=torch.empty(T, 64, device="cuda"), topk_idx=torch.empty(T, 6, dtype=torch.int32, device="cuda"),
               topk_w=torch.empty(T, 6, device="cuda"), counts=torch.empty(64, dtype=torch.int32, device="cuda"),
               offsets=torch.empty(65, dtype=torch.int32, device="cuda"),
               perm=torch.empty(T * 6, dtype=torch.int32, device="cuda"))
    if ws is None:
        ws = api.new_workspace(T)
    out = api.focr_moe_layer_forward(packed, xd, workspace=ws, debug=dbg)
    torch.cuda.synchronize()
    api.focr_moe_check(ws)
    r = {k: v.cpu().numpy() for k, v in dbg.items()}
    r["out"] = out.cpu().numpy()
    return r


def assert_parity(g, r, tol=None):
    if tol is None:
        tol = tol_for(g["out"].shape[0])
    np.testing.assert_array_equal(g["topk_idx"], r["idx"])
    np.testing.assert_array_max_ulp(g["logits"], r["logits"], maxulp=1)
    np.testing.assert_allclose(g["topk_w"], r["w"], rtol=1e-5, atol=1e-9)
    np.testing.assert_array_equal(g["counts"], r["counts"])
    np.testing.assert_array_equal(g["offsets"], r["offsets"])
    np.testing.assert_array_equal(g["perm"], r["perm"])
    err = per_token_rel_err(g["out"], r["out"])
    assert err.max() <= tol, f"max per-token relative error {err.max():.3e} > {tol}"


# ------------------------------------------------------------------ quantised codes

@pytest.mark.parametrize("name", ["int8_g128", "int4_g32", "int4_g64", "int4_g128"])
def test_export_is_bit_exact_with_oracle_quantiser(name):
    om, packed = moe_case(*LAYERS[name])
    I, H = 896, 1280
    for e in range(64):   # every expert of the layer
        for mat, omat, rows in ((api.MAT_GATE, om.gate, slice(e * I, (e + 1) * I)),
                                (api.MAT_UP, om.up, slice(e * I, (e + 1) * I)),
                                (api.MAT_DOWN, om.down, slice(e * H, (e + 1) * H))):
            codes, scales = api.focr_moe_export_quantized(packed, mat, e)
            q = omat.q[rows]
            ref = oracle.nibble_pack(q) if omat.wtype == W4 else q.reshape(-1).view(np.uint8)
            assert np.array_equal(codes, ref), (name, mat, e)
            assert np.array_equal(scales.view(np.uint32), omat.s[rows].reshape(-1).view(np.uint32)), (name, mat, e)
    for mat, omat in ((api.MAT_SHARED_GATE, om.sgate), (api.MAT_SHARED_UP, om.sup), (api.MAT_SHARED_DOWN, om.sdown)):
        codes, scales = api.focr_moe_export_quantized(packed, mat)
        if omat.wtype == WB:
            assert np.array_equal(codes.view(np.uint16), (omat.f.view(np.uint32) >> 16).astype(np.uint16).reshape(-1))
            assert scales.size == 0
        else:
            assert np.array_equal(codes, omat.q.reshape(-1).view(np.uint8))
            assert np.array_equal(scales.view(np.uint32), omat.s.reshape(-1).view(np.uint32))
    codes, _ = api.focr_moe_export_quantized(packed, api.MAT_ROUTER)
    assert np.array_equal(codes.view(np.uint16), om.router.reshape(-1))


# ------------------------------------------------------------------ forward parity

@pytest.mark.parametrize("name", ["int8_g128", "int4_g32", "int4_g64", "int4_g128"])
def test_decode_single_token(name):
    seed = LAYERS[name][0]
    om, packed = moe_case(*LAYERS[name])
    x = synth.hidden(seed, 1)
    assert_parity(run_gpu(packed, x), om.forward(x))


@pytest.mark.parametrize("T", [8, 32, 64])
def test_batched_decode_skewed_routing(T):
    om, packed = moe_case(*LAYERS["int4_g64_skew"])
    x = synth.hidden(2, T, skew=True)
    r = om.forward(x, nthreads=NTHREADS)
    assert_parity(run_gpu(packed, x), r)
    # the skew concentrates load on low-index experts
    assert r["counts"][:8].sum() > r["counts"][-32:].sum()


def test_prefill_289_tokens():
    om, packed = moe_case(*LAYERS["int4_g64_prefill"])
    x = synth.prefill_hidden(3)
    r = om.forward(x, nthreads=NTHREADS)
    g = run_gpu(packed, x)
    assert_parity(g, r)
    assert (r["counts"] > 0).all()


@pytest.mark.parametrize("T", [2, 3, 5, 7, 9, 13, 17, 65, 97, 130])
def test_ragged_token_counts(T):
    om, packed = moe_case(*LAYERS["int4_g64"])
    x = synth.hidden(40 + T, T)
    assert_parity(run_gpu(packed, x), om.forward(x, nthreads=NTHREADS))


def test_int8_layer_batched():
    om, packed = moe_case(*LAYERS["int8_g128"])
    x = synth.hidden(41, 11)
    assert_parity(run_gpu(packed, x), om.forward(x, nthreads=NTHREADS))


def test_repeated_calls_reuse_workspace():
    torch = _torch()
    om, packed = moe_case(*LAYERS["int4_g64"])
    ws = api.new_workspace(64)
    x1 = synth.hidden(42, 5)
    x2 = synth.hidden(43, 64)
    g1 = run_gpu(packed, x1, ws)
    g2 = run_gpu(packed, x2, ws)
    g3 = run_gpu(packed, x1, ws)
    np.testing.assert_array_equal(g1["topk_idx"], g3["topk_idx"])
    np.testing.assert_array_equal(g1["perm"], g3["perm"])
    assert per_token_rel_err(g3["out"], g1["out"]).max() < 1e-5
    assert_parity(g2, om.forward(x2, nthreads=NTHREADS))
    # control words, k-split sums and counters back to zero after every forward
    zb = api.focr_moe_workspace_zero_bytes()
    assert int(ws[:zb].count_nonzero()) == 0
    # decode-size calls of different T on the same workspace
    for T in (1, 8, 3):
        x = synth.hidden(45 + T, T)
        assert_parity(run_gpu(packed, x, ws), om.forward(x, nthreads=NTHREADS))
        assert int(ws[:zb].count_nonzero()) == 0


# every weight-type pairing the kernels instantiate beyond the ones above, on the
# decode path (T <= 8: gate/up kernel + down kernel) and the grouped path (T > 8)
MIXED = [
    (W4, W4, 64), (W4, W4, 32), (W4, W8, 128), (W8, WB, 128), (W8, W4, 128),
    (WB, WB, 128), (WB, W4, 32), (WB, W8, 128),
]


@functools.lru_cache(maxsize=1)   # one mixed layer alive at a time (T varies fastest below)
def mixed_case(routed, shared, group):
    return moe_case.__wrapped__(5, routed, shared, group)


@pytest.mark.parametrize("T", [3, 12, 80])
@pytest.mark.parametrize("routed,shared,group", MIXED)
def test_mixed_weight_types(routed, shared, group, T):
    om, packed = mixed_case(routed, shared, group)
    x = synth.hidden(50 + T, T)
    assert_parity(run_gpu(packed, x), om.forward(x, nthreads=NTHREADS))


def test_uniform_router_ties_pick_lowest_experts():
    # zero input: every logit is 0, so the top-6 must be experts 0..5 with weight 1/64
    om, packed = moe_case(*LAYERS["int4_g64"])
    x = np.zeros((3, 1280), np.float32)
    g = run_gpu(packed, x)
    assert (g["topk_idx"] == np.arange(6)).all()
    np.testing.assert_allclose(g["topk_w"], 1 / 64, rtol=1e-6)
    assert np.abs(g["out"]).max() == 0.0


def test_large_batch_sampled_tokens():
    om, packed = moe_case(*LAYERS["int4_g64"])
    T = 1024
    x = synth.hidden(44, T)
    g = run_gpu(packed, x)
    lg = oracle.router_logits(x, om.router)
    idx, w, _ = oracle.softmax_topk(lg, 6)
    counts, offsets, perm = oracle.dispatch(idx, 64)
    np.testing.assert_array_equal(g["topk_idx"], idx)
    np.testing.assert_array_equal(g["perm"], perm)
    np.testing.assert_array_equal(g["offsets"], offsets)
    sample = np.random.default_rng(0).choice(T, 12, replace=False)
    sample = np.concatenate([[0, T - 1], sample])
    r = om.forward(x[sample], nthreads=NTHREADS)
    err = per_token_rel_err(g["out"][sample], r["out"])
    assert err.max() <= TOL_TC


def test_forward_rejects_bad_arguments_on_device():
    torch = _torch()
    om, packed = moe_case(*LAYERS["int4_g64"])
    x = torch.zeros(4, 1280, device="cuda")
    out = torch.empty_like(x)
    ws = api.new_workspace(4)
    small = api.new_workspace(1)
    with pytest.raises(api.FocrError, match="INVALID_ARG"):
        api.focr_moe_layer_forward(packed, x, out, small)
    with pytest.raises(api.FocrError, match="INVALID_ARG"):
        api.focr_moe_layer_forward(packed, x, x, ws)            # overlap
    with pytest.raises(api.FocrError, match="INVALID_ARG"):
        api.focr_moe_layer_forward(packed, x.view(-1)[1:1281].view(1, 1280), out, ws)  # misaligned
    L = api.lib()
    st = L.focr_moe_layer_forward(api.ctypes.c_void_p(packed.handle), x.data_ptr(), 0, out.data_ptr(),
                                  ws.data_ptr(), ws.numel(), None, None)
    assert st == 1
    st = L.focr_moe_layer_forward(api.ctypes.c_void_p(packed.handle), x.data_ptr(), 8193, out.data_ptr(),
                                  ws.data_ptr(), ws.numel(), None, None)
    assert st == 1
    torch.cuda.synchronize()
