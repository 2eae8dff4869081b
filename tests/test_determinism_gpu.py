"""Repeated calls give bit-identical outputs.

T <= 8 with FOCR_FWD_DETERMINISTIC: the small-batch kernels add their parts as 64-bit fixed-point
integers and convert each output once (the order in which parts arrive cannot change a bit).
T > 64: the tensor-core kernel always sums each token's parts in a fixed order.  (9 to 64 tokens
take the grouped mma.sync kernel, which adds into the output with fp32 atomics; not covered.)
"""
import numpy as np
import pytest

from conftest import moe_case
from weight_quantized_expert_b200 import api, synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [1, 3, 8, 80, 289])
@pytest.mark.parametrize("shared", [synth.W_BF16, synth.W_INT8])
def test_repeated_forwards_are_bit_identical(T, shared):
    import torch
    group = 128 if shared == synth.W_INT8 else 64
    _, packed = moe_case(11, synth.W_INT4, shared, group)
    x = torch.from_numpy(synth.hidden(500 + T, T)).cuda()
    outs = []
    for rep in range(3):
        ws = api.new_workspace(T)   # a fresh workspace each time, and the same one twice below
        o = api.focr_moe_layer_forward(packed, x, workspace=ws, flags=api.FWD_DETERMINISTIC)
        if rep == 2:
            o = api.focr_moe_layer_forward(packed, x, workspace=ws, flags=api.FWD_DETERMINISTIC)
        torch.cuda.synchronize()
        api.focr_moe_check(ws)
        outs.append(o.cpu().numpy())
    np.testing.assert_array_equal(outs[0], outs[1])
    np.testing.assert_array_equal(outs[0], outs[2])


def test_dense_layer_repeats_bit_for_bit_at_one_token():
    import torch
    from test_companions_gpu import dense_case
    _, mlp = dense_case()
    x = torch.from_numpy(synth.hidden(510, 1)).cuda()
    ws = api.new_workspace(1)
    a = api.focr_dense_mlp_forward(mlp, x, workspace=ws, flags=api.FWD_DETERMINISTIC).cpu().numpy()
    b = api.focr_dense_mlp_forward(mlp, x, workspace=ws, flags=api.FWD_DETERMINISTIC).cpu().numpy()
    np.testing.assert_array_equal(a, b)


def test_deterministic_mode_keeps_parity():
    import os
    from conftest import per_token_rel_err
    import torch
    om, packed = moe_case(11, synth.W_INT4, synth.W_BF16, 64)
    for T in (1, 5):
        x = synth.hidden(520 + T, T)
        ws = api.new_workspace(T)
        o = api.focr_moe_layer_forward(packed, torch.from_numpy(x).cuda(), workspace=ws, flags=api.FWD_DETERMINISTIC)
        torch.cuda.synchronize()
        api.focr_moe_check(ws)
        assert int(ws[:api.focr_moe_workspace_zero_bytes()].count_nonzero()) == 0   # sums and counters cleared
        r = om.forward(x, nthreads=max(1, os.cpu_count() or 1))
        assert per_token_rel_err(o.cpu().numpy(), r["out"]).max() <= 2e-3
