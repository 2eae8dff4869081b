"""The allocation-free forward (focr_moe_layer_forward_noalloc) against the oracle.

Some callers cannot allocate device memory where they run the layer (a plug-in inside
an application that owns the device memory budget, or latency-critical code that must
not call cudaMalloc).  The allocation-free entry point serves them with a fixed scratch
array inside the library (T <= NOALLOC_T_MAX tokens).  Nothing in that array is cleared
per call: every forward that completes leaves its control words zero, and
focr_moe_check_noalloc reports (and repairs) a forward whose device wait ran out.

The calls below are chained through the one array in a large - small - large order, so a
forward that left anything behind would spoil the next one.  This file is collected last
on purpose; it must pass alone in a fresh process and after the rest of the suite.
"""
import ctypes
import os

import numpy as np
import pytest

from conftest import moe_case, per_token_rel_err
from weight_quantized_expert_b200 import api, synth

pytestmark = pytest.mark.gpu
NTHREADS = max(1, (os.cpu_count() or 1))
TOL_DECODE = 2e-3   # T <= 64: mma.sync kernels, f16 activations, fp32 accumulation
TOL_TC = 1e-2       # T > 64: tensor-core kernel, f16 gate/up and bf16 down operands


def _noalloc(packed, x):
    import torch
    T = x.shape[0]
    xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    dbg = dict(topk_idx=torch.empty(T, 6, dtype=torch.int32, device="cuda"),
               counts=torch.empty(64, dtype=torch.int32, device="cuda"),
               perm=torch.empty(T * 6, dtype=torch.int32, device="cuda"))
    out = api.focr_moe_layer_forward_noalloc(packed, xd, debug=dbg)
    torch.cuda.synchronize()
    api.focr_moe_check_noalloc()   # raises if a device wait of this forward ran out
    return out.cpu().numpy(), {k: v.cpu().numpy() for k, v in dbg.items()}


@pytest.mark.parametrize("chain", [(289, 7, 33, 1, 289), (33, 320, 9, 8, 64)])
def test_noalloc_chained_large_small_large_against_oracle(chain):
    om, packed = moe_case(3, synth.W_INT4, synth.W_BF16, 64)
    for i, T in enumerate(chain):
        x = synth.hidden(70 + 10 * i + T, T)
        got, dbg = _noalloc(packed, x)
        r = om.forward(x, nthreads=NTHREADS)
        np.testing.assert_array_equal(dbg["topk_idx"], r["idx"])
        np.testing.assert_array_equal(dbg["counts"], r["counts"])
        np.testing.assert_array_equal(dbg["perm"], r["perm"])
        tol = TOL_DECODE if T <= 64 else TOL_TC
        assert per_token_rel_err(got, r["out"]).max() <= tol, (T, per_token_rel_err(got, r["out"]).max())


def test_noalloc_matches_the_regular_forward():
    # same kernels, same inputs: bit for bit where the kernels sum in a fixed order
    import torch
    _, packed = moe_case(1, synth.W_INT4, synth.W_BF16, 64)
    for T in (7, 80):
        x = synth.hidden(61 + T, T)
        xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
        ref = api.focr_moe_layer_forward(packed, xd, workspace=api.new_workspace(T))
        got = api.focr_moe_layer_forward_noalloc(packed, xd)
        torch.cuda.synchronize()
        api.focr_moe_check_noalloc()
        if T > 64:   # the tensor-core path sums in a fixed order
            np.testing.assert_array_equal(got.cpu().numpy(), ref.cpu().numpy())
        else:   # the small-batch kernels add their parts with fp32 atomics, in arrival order
            assert per_token_rel_err(got.cpu().numpy(), ref.cpu().numpy()).max() <= 1e-5


def test_noalloc_rejects_tokens_beyond_the_scratch_limit():
    import torch
    _, packed = moe_case(1, synth.W_INT4, synth.W_BF16, 64)
    L = api.lib()
    x = torch.zeros(api.NOALLOC_T_MAX + 1, 1280, device="cuda")
    out = torch.empty_like(x)
    st = L.focr_moe_layer_forward_noalloc(ctypes.c_void_p(packed.handle), x.data_ptr(), api.NOALLOC_T_MAX + 1,
                                          out.data_ptr(), None, None)
    assert st == 1 and "scratch limit" in api.focr_last_error()
    api.focr_moe_check_noalloc()   # a rejected call leaves nothing to report
