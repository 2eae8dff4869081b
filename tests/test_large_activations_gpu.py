"""Inputs with large-magnitude outlier channels (1e3 to 3e4 in a few hidden channels, the rest
~N(0, 1)) against the oracle.

The tensor-core path (T > 64) takes x as f16 operands (finite up to 65504) and the SwiGLU
output a as bf16, so such inputs keep their parity.  The mma.sync kernels (T <= 64) take a
as f16 as well; where an outlier drives |a| past 65504 the forward reports FOCR_ERR_RANGE
through focr_moe_check instead of returning unflagged garbage.  A finite |x| above 65504 is
reported the same way on both paths.
"""
import os

import numpy as np
import pytest

from conftest import moe_case, per_token_rel_err
from weight_quantized_expert_b200 import api, synth

pytestmark = pytest.mark.gpu
NTHREADS = max(1, os.cpu_count() or 1)


def outlier_hidden(seed: int, T: int, magnitude: float, n_channels: int = 4) -> np.ndarray:
    x = synth.hidden(seed, T)
    rng = np.random.default_rng(seed)
    ch = rng.choice(1280, n_channels, replace=False)
    sign = rng.choice(np.array([-1.0, 1.0], np.float32), size=(T, n_channels))
    x[:, ch] = (sign * magnitude * rng.uniform(0.5, 1.0, size=(T, n_channels))).astype(np.float32)
    return x


def _forward(packed, x):
    import torch
    T = x.shape[0]
    ws = api.new_workspace(T)
    idx = torch.empty(T, 6, dtype=torch.int32, device="cuda")
    out = api.focr_moe_layer_forward(packed, torch.from_numpy(x).cuda(), workspace=ws, debug={"topk_idx": idx})
    torch.cuda.synchronize()
    return out, idx, ws


@pytest.mark.parametrize("magnitude", [1e3, 3e4])
def test_tensor_core_path_keeps_parity_with_outlier_channels(magnitude):
    om, packed = moe_case(3, synth.W_INT4, synth.W_BF16, 64)
    x = outlier_hidden(200 + int(magnitude) % 97, 80, magnitude)
    r = om.forward(x, nthreads=NTHREADS)
    out, idx, ws = _forward(packed, x)
    api.focr_moe_check(ws)   # no range error: every |x| <= 65504
    np.testing.assert_array_equal(idx.cpu().numpy(), r["idx"])
    assert per_token_rel_err(out.cpu().numpy(), r["out"]).max() <= 1e-2


@pytest.mark.parametrize("magnitude", [1e3, 3e4])
def test_small_batch_path_keeps_parity_or_reports_the_range(magnitude):
    om, packed = moe_case(3, synth.W_INT4, synth.W_BF16, 64)
    x = outlier_hidden(300 + int(magnitude) % 89, 3, magnitude)
    r = om.forward(x, nthreads=NTHREADS)
    out, idx, ws = _forward(packed, x)
    np.testing.assert_array_equal(idx.cpu().numpy(), r["idx"])
    try:
        api.focr_moe_check(ws)
    except api.FocrError as e:
        assert e.status == 6, e   # FOCR_ERR_RANGE: the explicit rejection
        assert magnitude > 1e3    # moderate outliers must not be rejected
        return
    assert per_token_rel_err(out.cpu().numpy(), r["out"]).max() <= 2e-3


@pytest.mark.parametrize("T", [3, 33, 80])
def test_inputs_beyond_the_f16_range_are_reported(T):
    _, packed = moe_case(3, synth.W_INT4, synth.W_BF16, 64)
    x = synth.hidden(400 + T, T)
    x[T // 2, 17] = 1e5
    _, _, ws = _forward(packed, x)
    with pytest.raises(api.FocrError) as ei:
        api.focr_moe_check(ws)
    assert ei.value.status == 6
    api.focr_moe_check(ws)   # the word was cleared by the report
