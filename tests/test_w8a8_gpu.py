"""W8A8 GEMV through the C ABI against the oracle, bit for bit.

franken_ocr README, "CPU Backend and Optimizations": the int8 decode linears quantise the
activation per token and run an integer GEMV with exact i32 accumulation; "Command Reference",
`focr robot`: K = 6848 is the accumulation's worst case.  Every step of the formula is exact
integer arithmetic or one correctly rounded IEEE operation (the fp32 divisions that decide the
codes are taken in fp32 on both sides), so codes, scales and outputs must match exactly.

Shapes: the dense layer's 6848 x 1280 and 1280 x 6848 (split and unsplit K), the lm_head's
129280 x 1280, and ragged N and K (tails of a 16-row tile and of a 32-column k-step).
"""
import numpy as np
import pytest

import oracle
from weight_quantized_expert_b200 import api

pytestmark = pytest.mark.gpu


def _w(seed, N, K):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal((N, K)).astype(np.float32) * 0.02
    w[rng.integers(0, N, max(1, N // 50)), rng.integers(0, K, max(1, N // 50))] *= 40.0   # outlier weights
    return w


def _x(seed, T, K):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, K)).astype(np.float32)
    x[:, rng.integers(0, K, 3)] *= 30.0   # outlier channels, as activations of a trained model have
    return x


_PACKED = {}


def _packed(seed, N, K):
    key = (seed, N, K)
    if key not in _PACKED:
        w = _w(seed, N, K)
        _PACKED.clear()
        _PACKED[key] = (oracle.OracleW8A8(w), api.focr_w8a8_pack(w))
    return _PACKED[key]


def _gemv(m, x):
    import torch
    ws = torch.zeros(api.focr_w8a8_workspace_bytes(m, x.shape[0]), dtype=torch.uint8, device="cuda")
    y = api.focr_w8a8_gemv(m, torch.from_numpy(x).cuda(), workspace=ws)
    api.focr_w8a8_check(ws)
    return y.cpu().numpy()


@pytest.mark.parametrize("N,K", [(6848, 1280), (1280, 6848), (37, 100), (1, 1), (16, 33)])
def test_pack_export_matches_the_oracle_codes(N, K):
    om, m = _packed(1, N, K)
    q, s = api.focr_w8a8_export(m)
    np.testing.assert_array_equal(q, om.q)
    np.testing.assert_array_equal(s, om.s)


@pytest.mark.parametrize("T,K", [(1, 1280), (3, 6848), (64, 1280), (100, 100), (5, 1), (2, 33)])
def test_activation_quantiser_matches_the_oracle(T, K):
    import torch
    x = _x(10 + T, T, K)
    if T >= 3:
        x[1] = 0.0                                            # all-zero token: s = 0, q = 0
        x[2, : min(K, 7)] = np.array([127, -63.5, 31.75, 0.5, -0.5, 1.5, 2.5], np.float32)[: min(K, 7)]
        x[2, 7:] = 0.0                                        # half-way codes (s = 1)
    qx, sx = api.focr_w8a8_quantize_x(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    rq, rs = oracle.w8a8_quantize_x(x)
    np.testing.assert_array_equal(sx.cpu().numpy(), rs)
    np.testing.assert_array_equal(qx.cpu().numpy(), rq)


@pytest.mark.parametrize("N,K", [(6848, 1280), (1280, 6848), (37, 100), (16, 33)])
@pytest.mark.parametrize("T", [1, 3, 8, 9, 64])
def test_gemv_is_bit_exact(N, K, T):
    om, m = _packed(1, N, K)
    x = _x(100 + T, T, K)
    y_ref, _, _ = om.forward(x)
    np.testing.assert_array_equal(_gemv(m, x), y_ref)


@pytest.mark.parametrize("T", [1, 8])
def test_gemv_is_bit_exact_at_lm_head_size(T):
    om, m = _packed(2, api.VOCAB, api.H)
    x = _x(200 + T, T, api.H)
    y_ref, _, _ = om.forward(x)
    np.testing.assert_array_equal(_gemv(m, x), y_ref)


@pytest.mark.parametrize("K", [6848, api.W8A8_K_MAX])
def test_worst_case_accumulation_is_exact(K):
    # every code at +-127: |acc| reaches K * 127^2 (110,451,392 at K = 6848; 2,147,463,447 at the
    # largest K, just under 2^31), summed over many split-K warps
    w = np.full((19, K), 1.0, np.float32)
    w[1] = -1.0
    w[2, 1::2] = -1.0
    w[3] = 0.0
    x = np.full((3, K), 2.0, np.float32)
    x[1] = -2.0
    x[2] = 0.0
    om = oracle.OracleW8A8(w)
    y_ref, _, _, acc = om.forward(x, want_acc=True)
    assert acc[0, 0] == K * 127 * 127 < 2 ** 31 and acc[1, 0] == -K * 127 * 127
    m = api.focr_w8a8_pack(w)
    np.testing.assert_array_equal(_gemv(m, x), y_ref)


def test_workspace_is_shared_across_token_counts_and_left_zero():
    import torch
    om, m = _packed(1, 1280, 6848)   # split K: the sums and counters are used
    ws = torch.zeros(api.focr_w8a8_workspace_bytes(m, api.W8A8_T_MAX), dtype=torch.uint8, device="cuda")
    outs = []
    for T in (64, 1, 9, 64):
        x = torch.from_numpy(_x(300, 64, 6848)[:T].copy()).cuda()
        outs.append(api.focr_w8a8_gemv(m, x, workspace=ws).cpu().numpy())
    torch.cuda.synchronize()
    np.testing.assert_array_equal(outs[0], outs[3])
    np.testing.assert_array_equal(outs[1], outs[0][:1])
    np.testing.assert_array_equal(outs[2], outs[0][:9])
    api.focr_w8a8_check(ws)                          # no bounded wait ran out
    tiles = (1280 + 15) // 16
    assert int(ws[: 256 + 4 * tiles].sum()) == 0     # error word and per-tile counters back at zero
    np.testing.assert_array_equal(outs[0], om.forward(_x(300, 64, 6848))[0])


def test_gemv_rejects_bad_arguments():
    import ctypes
    import torch
    _, m = _packed(1, 37, 100)
    L = api.lib()
    x = torch.zeros(65, 100, device="cuda")
    y = torch.empty(65, 37, device="cuda")
    ws = torch.zeros(api.focr_w8a8_workspace_bytes(m, 64), dtype=torch.uint8, device="cuda")
    h = ctypes.c_void_p(m.handle)
    assert L.focr_w8a8_gemv(h, x.data_ptr(), 0, y.data_ptr(), ws.data_ptr(), ws.numel(), None) == 1
    assert L.focr_w8a8_gemv(h, x.data_ptr(), 65, y.data_ptr(), ws.data_ptr(), ws.numel(), None) == 1
    assert L.focr_w8a8_gemv(h, x.data_ptr(), 8, y.data_ptr(), ws.data_ptr(), 256, None) == 1
    assert "workspace" in api.focr_last_error()
