"""R-SWA decode attention through the C ABI against the oracle.

franken_ocr README, "Design Philosophy" / "Architecture" (R-SWA: every reference row plus the
last 128 generated tokens through a ring) and frankenocr.pages.dev, "One forward pass", step 6
(10 heads x 128).  Tolerance: the output is a convex combination of value rows, computed in fp32
(dot products of 128 terms, online softmax, split-key merge) against the oracle's fp64; per
(sequence, head) the bar is 3e-5 x max |v| over the attended rows, about 250 fp32 ulps of the
largest value.  The ring update is a copy and must match exactly.
"""
import numpy as np
import pytest

import oracle
from weight_quantized_expert_b200 import api, synth

pytestmark = pytest.mark.gpu
TOL = 3e-5


def _dev(a):
    import torch
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda() for k, v in a.items()}


def _run(a, ref_len, n_gen):
    import torch
    d = _dev(a)
    rl = torch.tensor(ref_len, dtype=torch.int32, device="cuda")
    ng = torch.tensor(n_gen, dtype=torch.int32, device="cuda")
    out = api.focr_rswa_decode(d["q"], d["k_new"], d["v_new"], d["k_ref"], d["v_ref"], rl, d["k_ring"], d["v_ring"], ng)
    torch.cuda.synchronize()
    return out.cpu().numpy(), d["k_ring"].cpu().numpy(), d["v_ring"].cpu().numpy()


def _ref(a, ref_len, n_gen):
    return oracle.rswa_decode(a["q"], a["k_new"], a["v_new"], a["k_ref"], a["v_ref"], ref_len, a["k_ring"],
                              a["v_ring"], n_gen)


def _compare(a, ref_len, n_gen):
    out, kg, vg = _run(a, ref_len, n_gen)
    r_out, r_kg, r_vg = _ref(a, ref_len, n_gen)
    np.testing.assert_array_equal(kg, r_kg)
    np.testing.assert_array_equal(vg, r_vg)
    for b in range(len(ref_len)):
        vmax = max(np.abs(a["v_ref"][b, :, :ref_len[b]]).max(initial=0.0), np.abs(a["v_ring"][b]).max(),
                   np.abs(a["v_new"][b]).max())
        err = np.abs(out[b].astype(np.float64) - r_out[b]).max()
        assert err <= TOL * vmax, (b, err, vmax)
    return out


@pytest.mark.parametrize("n", [1, 2, 77, 127, 128, 129, 600])
def test_single_sequence_with_the_prefill_reference_block(n):
    a = synth.rswa_inputs(10 + n, 1, synth.RSWA_REF)
    _compare(a, [synth.RSWA_REF], [n])


def test_ragged_batch():
    a = synth.rswa_inputs(21, 5, 300)
    _compare(a, [0, 17, 300, 289, 1], [1, 500, 128, 600, 3])


def test_batch_of_eight_at_the_bench_shape():
    a = synth.rswa_inputs(22, 8, synth.RSWA_REF)
    _compare(a, [synth.RSWA_REF] * 8, [600, 1, 64, 128, 129, 255, 256, 1000])


def test_long_reference_block():
    a = synth.rswa_inputs(23, 2, 4096)
    _compare(a, [4096, 2500], [900, 40])


def test_dominant_key_with_large_scores():
    a = synth.rswa_inputs(24, 1, 32)
    a["q"] *= 8.0
    a["k_ref"][0, :, 5] = a["q"][0] * 0.5   # scores near 180 for one reference row
    out = _compare(a, [32], [300])
    np.testing.assert_allclose(out[0], a["v_ref"][0, :, 5], rtol=0, atol=1e-4)


def test_consecutive_steps_update_the_ring_in_place():
    import torch
    a = synth.rswa_inputs(25, 2, 64)
    d = _dev(a)
    rl = torch.tensor([64, 10], dtype=torch.int32, device="cuda")
    r_kg, r_vg = a["k_ring"], a["v_ring"]
    rng = np.random.default_rng(25)
    for step, n0 in enumerate((126, 127, 128, 129, 130)):
        kn = rng.standard_normal(a["k_new"].shape).astype(np.float32)
        vn = rng.standard_normal(a["v_new"].shape).astype(np.float32)
        q = rng.standard_normal(a["q"].shape).astype(np.float32)
        n = [n0, n0 + 100]
        ng = torch.tensor(n, dtype=torch.int32, device="cuda")
        out = api.focr_rswa_decode(torch.from_numpy(q).cuda(), torch.from_numpy(kn).cuda(), torch.from_numpy(vn).cuda(),
                                   d["k_ref"], d["v_ref"], rl, d["k_ring"], d["v_ring"], ng)
        r_out, r_kg, r_vg = oracle.rswa_decode(q, kn, vn, a["k_ref"], a["v_ref"], [64, 10], r_kg, r_vg, n)
        torch.cuda.synchronize()
        assert np.abs(out.cpu().numpy() - r_out).max() <= TOL * 5.0, step
        np.testing.assert_array_equal(d["k_ring"].cpu().numpy(), r_kg)
        np.testing.assert_array_equal(d["v_ring"].cpu().numpy(), r_vg)


def test_invalid_lengths_give_nan_and_keep_the_ring():
    a = synth.rswa_inputs(26, 3, 16)
    out, kg, vg = _run(a, [17, -1, 16], [1, 5, 0])
    assert np.isnan(out).all()
    np.testing.assert_array_equal(kg, a["k_ring"])
    np.testing.assert_array_equal(vg, a["v_ring"])


def test_rejects_bad_arguments():
    import ctypes
    import torch
    L = api.lib()
    x = torch.zeros(16, device="cuda")
    p = x.data_ptr()
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    assert L.focr_rswa_decode(p, p, p, p, p, p, 1, p, p, p, 0, p, ws.data_ptr(), 256, None) == 1
    assert L.focr_rswa_decode(p, p, p, p, p, p, 40000, p, p, p, 1, p, ws.data_ptr(), 256, None) == 1
    assert L.focr_rswa_decode(p + 4, p, p, p, p, p, 1, p, p, p, 1, p, ws.data_ptr(), 1 << 20, None) == 1
    assert L.focr_rswa_decode(p, p, p, p, p, p, 16, p, p, p, 1, p, ws.data_ptr(), 16, None) == 1
    assert "workspace" in api.focr_last_error()
    assert L.focr_rswa_decode(None, p, p, p, p, p, 1, p, p, p, 1, p, ws.data_ptr(), 1 << 20, None) == 1
