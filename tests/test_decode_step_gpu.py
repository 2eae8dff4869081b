"""The whole decode step through the C ABI (focr_decode_step) against the oracle composition:
the dense layer 0, eleven MoE layers with residual adds and RMSNorms, the lm_head and the
greedy argmax (frankenocr.pages.dev, "One forward pass": layer 0 dense SwiGLU, layers 1-11
mixture-of-experts, final norm, lm_head, argmax).

The eleven MoE layers alternate two independently drawn layers.  Argmax bar: let err be the
largest |logit_gpu - logit_oracle| measured over the batch; a token whose oracle top-two gap
exceeds 2 * err cannot change its winner under that error, so there the GPU's argmax must be
the oracle's exactly; elsewhere the GPU's pick must be within 2 * err of the oracle maximum.
"""
import functools
import os

import numpy as np
import pytest

import oracle
from conftest import moe_case, per_token_rel_err
from test_companions_gpu import dense_case, lm_case
from weight_quantized_expert_b200 import api, synth

pytestmark = pytest.mark.gpu
NTHREADS = max(1, os.cpu_count() or 1)
N_MOE = 11
EPS = 1e-6
# final hidden state, per-token relative error after 12 residual layers: the per-layer bars of
# the layer tests (2e-3 on the decode kernels, 1e-2 on the bf16 tensor-core path) times a margin
# for their accumulation through the stack
HIDDEN_TOL = {1: 2e-2, 32: 6e-2}


@functools.lru_cache(maxsize=None)
def stack_case():
    om_a, la = moe_case(1, synth.W_INT4, synth.W_BF16, 64)
    om_b, lb = moe_case(3, synth.W_INT4, synth.W_BF16, 64)
    refs, layers = [], []
    for l in range(N_MOE):
        src, om = (la, om_a) if l % 2 == 0 else (lb, om_b)
        layers.append(src if l < 2 else api.focr_moe_layer_clone(src))
        refs.append(om)
    dref, mlp = dense_case()
    href, head = lm_case()
    model = api.DecodeModel(mlp, layers, head, eps=EPS)
    return model, dref, refs, href


def oracle_step(dref, refs, href, x):
    h = oracle.rmsnorm(x + dref.forward(x, nthreads=NTHREADS), eps=EPS)
    for om in refs:
        h = oracle.rmsnorm(h + om.forward(h, nthreads=NTHREADS)["out"], eps=EPS)
    am, logits = href.forward(h, want_logits=True, nthreads=NTHREADS)
    return h, am, logits


@pytest.mark.parametrize("T", [1, 32])
def test_decode_step_eleven_moe_layers_against_oracle(T):
    import torch
    model, dref, refs, href = stack_case()
    x = synth.hidden(120 + T, T)
    r_h, r_am, r_logits = oracle_step(dref, refs, href, x)
    xd = torch.from_numpy(x).cuda()
    logits = torch.empty(T, api.VOCAB, device="cuda")
    hid = torch.empty(T, 1280, device="cuda")
    ws = api.new_decode_step_workspace(T)
    am = api.focr_decode_step(model, xd, logits=logits, hidden_out=hid, workspace=ws)
    torch.cuda.synchronize()
    api.focr_moe_check(ws[256:])
    g_h, g_am, g_logits = hid.cpu().numpy(), am.cpu().numpy(), logits.cpu().numpy()

    herr = per_token_rel_err(g_h, r_h).max()
    assert herr <= HIDDEN_TOL[T], herr
    err = float(np.abs(g_logits.astype(np.float64) - r_logits).max())
    assert err <= 5e-2 * float(np.abs(r_logits).max()), (err, np.abs(r_logits).max())
    top2 = np.sort(r_logits, axis=1)[:, -2:]
    decided = (top2[:, 1] - top2[:, 0]) > 2 * err
    np.testing.assert_array_equal(g_am[decided], r_am[decided])
    picked = r_logits[np.arange(T), g_am]
    assert (r_logits.max(axis=1) - picked <= 2 * err + 1e-6).all()


def test_decode_step_repeats_bit_for_bit_and_accepts_a_shared_workspace():
    # the same workspace serves T = 80 then T = 1 then T = 80 again; at T = 80 every layer runs on the
    # tensor-core kernel, which sums in a fixed order, so the two T = 80 calls agree bit for bit
    import torch
    model, _, _, _ = stack_case()
    ws = api.new_decode_step_workspace(80)
    x80 = torch.from_numpy(synth.hidden(133, 80)).cuda()
    x1 = torch.from_numpy(synth.hidden(134, 1)).cuda()
    outs = []
    for x in (x80, x1, x80):
        hid = torch.empty_like(x)
        am = api.focr_decode_step(model, x, hidden_out=hid, workspace=ws)
        torch.cuda.synchronize()
        outs.append((am.cpu().numpy(), hid.cpu().numpy()))
    api.focr_moe_check(ws[256:])
    np.testing.assert_array_equal(outs[0][0], outs[2][0])
    np.testing.assert_array_equal(outs[0][1], outs[2][1])


def test_decode_step_rejects_bad_arguments():
    import ctypes
    import torch
    model, _, _, _ = stack_case()
    L = api.lib()
    x = torch.zeros(2, 1280, device="cuda")
    am = torch.empty(2, dtype=torch.int32, device="cuda")
    ws = api.new_decode_step_workspace(1)   # too small for T = 2
    st = L.focr_decode_step(ctypes.byref(model.desc), x.data_ptr(), 2, None, am.data_ptr(), None, ws.data_ptr(),
                            ws.numel(), None)
    assert st == 1 and "workspace" in api.focr_last_error()
    st = L.focr_decode_step(None, x.data_ptr(), 2, None, am.data_ptr(), None, ws.data_ptr(), ws.numel(), None)
    assert st == 1
