"""Parity of the decode-step companions against the CPU oracle, through the C ABI:
the int8 lm_head GEMV + argmax, the final RMSNorm, the dense layer-0 SwiGLU MLP, the
residual form of the MoE forward, and a short decode stack built from them.

Bit-exact: exported codes and scales, argmax wherever the oracle's top two logits differ
by more than the fp32 accumulation bound (elsewhere the GPU's pick must be within that
bound of the maximum).  Floating point: logits within 1e-5 of the largest |logit|, the
dense layer within the 2e-3 per-token relative error of the layer tests.
"""
import functools
import os

import numpy as np
import pytest

import oracle
from conftest import moe_case, per_token_rel_err
from weight_quantized_expert_b200 import api, synth

pytestmark = pytest.mark.gpu
NTHREADS = max(1, os.cpu_count() or 1)


def _torch():
    import torch
    return torch


@functools.lru_cache(maxsize=None)
def lm_case():
    w = synth.lm_head(4)
    head = api.focr_lm_head_pack(w)
    ref = oracle.OracleLMHead(w)
    del w
    return ref, head


@functools.lru_cache(maxsize=None)
def dense_case():
    d = synth.dense_mlp(4)
    mlp = api.focr_dense_mlp_pack(d.gate, d.up, d.down, synth.W_INT8, 128)
    ref = oracle.OracleDense(d.gate, d.up, d.down, oracle.W_INT8, 128)
    del d
    return ref, mlp


# ------------------------------------------------------------------ lm_head

def test_lm_head_export_is_bit_exact():
    ref, head = lm_case()
    codes, scales = api.focr_lm_head_export(head)
    assert np.array_equal(codes, ref.q)
    assert np.array_equal(scales.view(np.uint32), ref.s.view(np.uint32))


def _check_argmax(got_idx, ref_logits, bound):
    for t in range(ref_logits.shape[0]):
        lg = ref_logits[t].astype(np.float64)
        top = np.argsort(-lg, kind="stable")[:2]
        assert lg[got_idx[t]] >= lg[top[0]] - bound
        if lg[top[0]] - lg[top[1]] > bound:
            assert got_idx[t] == top[0]


@pytest.mark.parametrize("T", [1, 5, 8, 9, 32, 40])
def test_lm_head_logits_and_argmax(T):
    torch = _torch()
    ref, head = lm_case()
    x = synth.normal_f32(60 + T, 1, (T, 1280))
    r_idx, r_logits = ref.forward(x, want_logits=True, nthreads=NTHREADS)
    xd = torch.from_numpy(x).cuda()
    logits = torch.empty(T, 129280, device="cuda")
    am = api.focr_lm_head_gemv(head, xd, logits=logits)
    torch.cuda.synchronize()
    g_logits = logits.cpu().numpy()
    scale = np.abs(r_logits).max()
    np.testing.assert_allclose(g_logits, r_logits, rtol=0, atol=1e-5 * scale)
    _check_argmax(am.cpu().numpy(), r_logits, 1e-5 * scale)
    # argmax without the logits buffer is the same
    am2 = api.focr_lm_head_gemv(head, xd)
    torch.cuda.synchronize()
    assert np.array_equal(am2.cpu().numpy(), am.cpu().numpy())


def test_lm_head_ring_kernel_agrees_with_the_streaming_kernel():
    # T <= 8 runs the bulk-copy ring kernel, T > 8 the streaming kernel: the same fragments and
    # MMAs, the ring kernel summing each tile as two halves, so the first 8 tokens' logits agree to
    # fp32 rounding of the partial sums
    torch = _torch()
    _, head = lm_case()
    x = torch.from_numpy(synth.normal_f32(71, 1, (9, 1280))).cuda()
    out = []
    for T in (8, 9):
        ws = torch.zeros(api.focr_lm_head_workspace_bytes(T), dtype=torch.uint8, device="cuda")
        logits = torch.empty(T, 129280, device="cuda")
        am = api.focr_lm_head_gemv(head, x[:T].contiguous(), logits=logits, workspace=ws)
        api.focr_lm_head_check(ws)
        out.append((logits[:8].cpu().numpy(), am[:8].cpu().numpy()))
    scale = np.abs(out[1][0]).max()
    np.testing.assert_allclose(out[0][0], out[1][0], rtol=0, atol=2e-6 * scale)
    _check_argmax(out[0][1], out[1][0].astype(np.float64), 4e-6 * scale)


def test_lm_head_tie_goes_to_the_lower_row():
    torch = _torch()
    ref, head = lm_case()
    # a token equal to a multiple of one row's codes makes that row the clear winner
    x = np.zeros((2, 1280), np.float32)
    x[0] = ref.q[77].astype(np.float32)
    x[1] = ref.q[129279].astype(np.float32)
    r_idx, r_logits = ref.forward(x, want_logits=True)
    am = api.focr_lm_head_gemv(head, torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    assert am.cpu().numpy().tolist() == r_idx.tolist()


# ------------------------------------------------------------------ RMSNorm

@pytest.mark.parametrize("with_gamma", [False, True])
def test_rmsnorm_matches_oracle(with_gamma):
    torch = _torch()
    x = synth.normal_f32(70, 1, (7, 1280)) * np.float32(3.0)
    gamma = synth.normal_f32(70, 2, (1280,)) if with_gamma else None
    ref = oracle.rmsnorm(x, gamma, eps=1e-6)
    g = api.focr_rmsnorm(torch.from_numpy(x).cuda(), None if gamma is None else torch.from_numpy(gamma).cuda(),
                         eps=1e-6)
    torch.cuda.synchronize()
    np.testing.assert_allclose(g.cpu().numpy(), ref, rtol=2e-6, atol=1e-6)


# ------------------------------------------------------------------ dense layer 0

def test_dense_export_is_bit_exact_including_the_short_tail_group():
    ref, mlp = dense_case()
    for m, om in enumerate((ref.G, ref.U, ref.D)):
        codes, scales = api.focr_dense_mlp_export_quantized(mlp, m)
        assert np.array_equal(codes, om.q.reshape(-1).view(np.uint8)), m
        assert np.array_equal(scales.view(np.uint32), om.s.reshape(-1).view(np.uint32)), m
    assert ref.D.s.shape == (1280, 54)   # 6848 = 53 x 128 + 64


@pytest.mark.parametrize("T", [1, 3, 32])
def test_dense_forward_matches_oracle(T):
    torch = _torch()
    ref, mlp = dense_case()
    x = synth.normal_f32(80 + T, 1, (T, 1280))
    r = ref.forward(x, nthreads=NTHREADS)
    xd = torch.from_numpy(x).cuda()
    g = api.focr_dense_mlp_forward(mlp, xd)
    gr = api.focr_dense_mlp_forward(mlp, xd, flags=api.FWD_RESIDUAL)
    torch.cuda.synchronize()
    g, gr = g.cpu().numpy(), gr.cpu().numpy()
    tol = 2e-3 if T <= 8 else 1e-2   # decode kernels / tensor-core kernel (the dense layer takes it for T > 8)
    assert per_token_rel_err(g, r).max() <= tol
    # residual form: x + layer(x), against the oracle
    assert per_token_rel_err(gr - x, r).max() <= tol


# ------------------------------------------------------------------ residual MoE forward and a short stack

def test_residual_moe_forward_adds_the_input():
    torch = _torch()
    om, packed = moe_case(1, synth.W_INT4, synth.W_BF16, 64)
    x = synth.hidden(90, 4)
    xd = torch.from_numpy(x).cuda()
    plain = api.focr_moe_layer_forward(packed, xd)
    resid = api.focr_moe_layer_forward(packed, xd, flags=api.FWD_RESIDUAL)
    torch.cuda.synchronize()
    plain, resid = plain.cpu().numpy(), resid.cpu().numpy()
    ref = om.forward(x)["out"]
    assert per_token_rel_err(plain, ref).max() <= 2e-3
    assert per_token_rel_err(resid - x, ref).max() <= 2e-3


@pytest.mark.parametrize("T", [1, 4])
def test_short_decode_stack(T):
    """h <- RMSNorm(h + FFN(h)) for the dense layer and two MoE layers, then argmax(lm_head(h))."""
    torch = _torch()
    dref, mlp = dense_case()
    om_a, la = moe_case(1, synth.W_INT4, synth.W_BF16, 64)
    om_b, lb = moe_case(3, synth.W_INT4, synth.W_BF16, 64)
    href, head = lm_case()
    x = synth.hidden(95, T)
    # oracle composition (fp32 residual adds, like the device path)
    h = oracle.rmsnorm(x + dref.forward(x), eps=1e-6)
    h = oracle.rmsnorm(h + om_a.forward(h)["out"], eps=1e-6)
    rn = oracle.rmsnorm(h + om_b.forward(h)["out"], eps=1e-6)
    r_idx, r_logits = href.forward(rn, want_logits=True, nthreads=NTHREADS)
    # device path
    ws = api.new_workspace(T)
    h0 = torch.from_numpy(x).cuda()
    g = api.focr_rmsnorm(api.focr_dense_mlp_forward(mlp, h0, workspace=ws, flags=api.FWD_RESIDUAL), eps=1e-6)
    g = api.focr_rmsnorm(api.focr_moe_layer_forward(la, g, workspace=ws, flags=api.FWD_RESIDUAL), eps=1e-6)
    rg = api.focr_rmsnorm(api.focr_moe_layer_forward(lb, g, workspace=ws, flags=api.FWD_RESIDUAL), eps=1e-6)
    am = api.focr_lm_head_gemv(head, rg)
    torch.cuda.synchronize()
    assert per_token_rel_err(rg.cpu().numpy(), rn).max() <= 5e-3
    scale = np.abs(r_logits).max()
    _check_argmax(am.cpu().numpy(), r_logits, 2e-2 * scale)


def test_router_survives_non_finite_tokens():
    """A token with NaN entries still routes to six distinct in-range experts (its outputs are NaN); the
    finite tokens of the batch are unaffected."""
    torch = _torch()
    om, packed = moe_case(1, synth.W_INT4, synth.W_BF16, 64)
    x = synth.hidden(96, 3)
    x[1, 5] = np.nan
    xd = torch.from_numpy(x).cuda()
    idx = torch.empty(3, 6, dtype=torch.int32, device="cuda")
    ws = api.new_workspace(3)
    out = api.focr_moe_layer_forward(packed, xd, workspace=ws, debug={"topk_idx": idx})
    torch.cuda.synchronize()
    api.focr_moe_check(ws)
    assert int(ws[:api.focr_moe_workspace_zero_bytes()].count_nonzero()) == 0
    got = idx.cpu().numpy()
    for t in range(3):
        assert len(set(got[t].tolist())) == 6 and got[t].min() >= 0 and got[t].max() < 64
    ref = om.forward(x[[0, 2]])
    g = out.cpu().numpy()[[0, 2]]
    assert np.array_equal(got[[0, 2]], ref["idx"])
    assert per_token_rel_err(g, ref["out"]).max() <= 2e-3
