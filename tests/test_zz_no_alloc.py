"""The allocation-free forward (focr_moe_layer_forward_noalloc) against the regular one.

Some callers cannot allocate device memory where they run the layer (a plug-in inside
an application that owns the device memory budget, or latency-critical code that must
not call cudaMalloc).  The allocation-free entry point serves them with a fixed scratch
array inside the library.  This file is collected last on purpose; it must pass alone
in a fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest

from conftest import moe_case, per_token_rel_err
from weight_quantized_expert_b200 import api, synth

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _forward_both(packed, x):
    import torch
    T = x.shape[0]
    xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    idx_a = torch.empty(T, 6, dtype=torch.int32, device="cuda")
    idx_b = torch.empty(T, 6, dtype=torch.int32, device="cuda")
    ref = api.focr_moe_layer_forward(packed, xd, workspace=api.new_workspace(T), debug={"topk_idx": idx_a})
    got = api.focr_moe_layer_forward_noalloc(packed, xd, debug={"topk_idx": idx_b})
    torch.cuda.synchronize()
    return got.cpu().numpy(), ref.cpu().numpy(), idx_b.cpu().numpy(), idx_a.cpu().numpy()


def test_noalloc_forward_matches_regular_forward_on_two_calls_in_a_row():
    _, packed = moe_case(1, synth.W_INT4, synth.W_BF16, 64)
    for x in (synth.hidden(61, 7), synth.hidden(62, 1)):   # second call reuses the dirty array
        got, ref, idx_g, idx_r = _forward_both(packed, x)
        np.testing.assert_array_equal(idx_g, idx_r)
        assert per_token_rel_err(got, ref).max() <= TOL


def test_noalloc_rejects_tokens_beyond_the_scratch_limit():
    import torch
    _, packed = moe_case(1, synth.W_INT4, synth.W_BF16, 64)
    L = api.lib()
    x = torch.zeros(api.NOALLOC_T_MAX + 1, 1280, device="cuda")
    out = torch.empty_like(x)
    st = L.focr_moe_layer_forward_noalloc(ctypes.c_void_p(packed.handle), x.data_ptr(), api.NOALLOC_T_MAX + 1,
                                          out.data_ptr(), None, None)
    assert st == 1 and "scratch limit" in api.focr_last_error()
