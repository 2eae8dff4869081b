"""Pins for the CPU oracle: each check ties it to something other than itself.

Hand values from the pages' definitions (tests/golden), closed forms,
brute force on tiny inputs, and independent numpy routines (matmul, sort).
A plausible slip anywhere in the oracle (a dropped term, a wrong sign, a
swapped nibble, a transposed operand, a renormalised weight, a wrong tie
rule) fails at least one of these.
"""
import os

import numpy as np
import pytest

import oracle
from weight_quantized_expert_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ nibbles
# frankenocr.pages.dev, "Four bits, one shared scale": a two's-complement nibble.

def test_nibble_roundtrip_all_16_values():
    q = np.arange(-8, 8, dtype=np.int8)
    for a in q:
        for b in q:
            packed = oracle.nibble_pack(np.array([a, b], np.int8))
            assert packed.shape == (1,)
            # element 2j -> bits 0-3, element 2j+1 -> bits 4-7, two's complement
            assert packed[0] == ((int(a) & 0xF) | ((int(b) & 0xF) << 4))
            back = oracle.nibble_unpack(packed, 2)
            assert back.tolist() == [a, b]


def test_nibble_codes_are_twos_complement():
    codes = {-8: 0x8, -7: 0x9, -2: 0xE, -1: 0xF, 0: 0x0, 1: 0x1, 7: 0x7}
    for v, nib in codes.items():
        assert oracle.nibble_pack(np.array([v, 0], np.int8))[0] == nib
        assert oracle.nibble_pack(np.array([0, v], np.int8))[0] == nib << 4


def test_byte_unpack_all_256():
    packed = np.arange(256, dtype=np.uint8)
    q = oracle.nibble_unpack(packed, 512).reshape(256, 2)
    for b in range(256):
        lo, hi = b & 0xF, b >> 4
        assert q[b, 0] == (lo - 16 if lo >= 8 else lo)
        assert q[b, 1] == (hi - 16 if hi >= 8 else hi)
    assert np.array_equal(oracle.nibble_pack(q.reshape(-1)), packed)


# ------------------------------------------------------------------ quantiser

def _golden_cases():
    out = []
    with open(os.path.join(GOLDEN, "quantizer_cases.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            head, w, s, q = [p.strip() for p in line.split("|")]
            bits, group = map(int, head.split())
            out.append((bits, group, np.array(w.split(), np.float32),
                        np.array(s.split(), np.float32), np.array(q.split(), np.int8)))
    return out


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: f"int{c[0]}-g{c[1]}-{c[2].size}")
def test_quantizer_golden(case):
    bits, group, w, s_exp, q_exp = case
    q, s = oracle.quantize_rows(w[None, :], group, bits)
    assert np.array_equal(s[0], s_exp)
    assert np.array_equal(q[0], q_exp)


def test_quantizer_outlier_takes_the_extreme_code():
    # ~N(0, 0.02) weights with one x20 outlier: the outlier lands exactly on +-7 and
    # the ordinary weights of its group collapse toward 0 (coarse scale).
    rng = np.random.default_rng(0)
    for sign in (1.0, -1.0):
        w = (rng.standard_normal(64) * 0.02).astype(np.float32)
        w[17] = np.float32(sign * 20 * 0.05)
        q, s = oracle.quantize_rows(w[None, :], 64, 4)
        assert q[0, 17] == (7 if sign > 0 else -7)
        assert np.abs(q[0]).max() == 7
        assert np.count_nonzero(q[0]) < 32


@pytest.mark.parametrize("bits,group", [(4, 32), (4, 64), (4, 128), (8, 128), (8, 1280)])
def test_quantizer_error_bound_and_extremes(bits, group):
    Q = 7 if bits == 4 else 127
    w = synth.weights_f32(7, 1, (32, 1280))
    q, s = oracle.quantize_rows(w, group, bits)
    assert s.shape == (32, 1280 // group)
    sc = np.repeat(s.astype(np.float64), group, axis=1)
    err = np.abs(w.astype(np.float64) - q.astype(np.float64) * sc)
    # round-to-nearest: each weight within half a step (plus fp32 division slop)
    assert np.all(err <= 0.5 * sc * (1 + 1e-5) + 1e-30)
    assert q.min() >= -Q and q.max() <= Q
    # the largest magnitude of each group maps to +-Q
    wg = np.abs(w).reshape(32, -1, group)
    qg = np.abs(q.astype(np.int32)).reshape(32, -1, group)
    am = wg.argmax(axis=2)
    assert np.all(np.take_along_axis(qg, am[..., None], 2) == Q)


def test_quantizer_short_tail_group_like_k6848():
    # 6848 = 53 * 128 + 64: the last group of a dense-down row has 64 elements
    w = synth.weights_f32(3, 2, (2, 6848))
    q, s = oracle.quantize_rows(w, 128, 8)
    assert s.shape == (2, 54)
    tail = np.abs(w[:, 6784:]).max(axis=1)
    assert np.array_equal(s[:, 53], (tail / np.float32(127)).astype(np.float32))
    assert np.abs(q[:, 6784:]).max() == 127


# ------------------------------------------------------------------ router
# frankenocr.pages.dev, "One forward pass" step 6: softmax router, top 6 picked
# greedily, no renormalisation.

def test_router_logits_match_numpy_matmul():
    x = synth.normal_f32(5, 1, (7, 1280))
    wr = synth.f32_to_bf16_bits(synth.normal_f32(5, 2, (64, 1280), 0.02))
    lg = oracle.router_logits(x, wr)
    ref = x.astype(np.float64) @ synth.bf16_bits_to_f32(wr).astype(np.float64).T
    np.testing.assert_allclose(lg, ref.astype(np.float32), rtol=2e-7, atol=1e-9)


def test_zero_input_gives_uniform_router_and_lowest_indices():
    T = 3
    x = np.zeros((T, 1280), np.float32)
    wr = synth.f32_to_bf16_bits(synth.normal_f32(5, 2, (64, 1280), 0.02))
    idx, w, p = oracle.softmax_topk(oracle.router_logits(x, wr), 6)
    assert np.array_equal(idx, np.tile(np.arange(6), (T, 1)))      # ties -> lower index
    np.testing.assert_allclose(w, 1.0 / 64, rtol=1e-15)
    np.testing.assert_allclose(w.sum(axis=1), 0.09375, rtol=1e-15)  # not renormalised
    np.testing.assert_allclose(p, 1.0 / 64, rtol=1e-15)


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(1)
    logits = rng.integers(-3, 4, size=(200, 64)).astype(np.float32) * np.float32(0.5)
    for k in (1, 6, 64):
        idx, w, p = oracle.softmax_topk(logits, k)
        for t in range(logits.shape[0]):
            order = np.lexsort((np.arange(64), -logits[t].astype(np.float64)))
            assert idx[t].tolist() == order[:k].tolist()


def test_topk_weights_are_raw_softmax_probabilities():
    x = synth.normal_f32(6, 1, (16, 1280))
    wr = synth.f32_to_bf16_bits(synth.normal_f32(6, 2, (64, 1280), 0.02))
    lg = oracle.router_logits(x, wr)
    idx, w, p = oracle.softmax_topk(lg, 6)
    l64 = lg.astype(np.float64)
    ref = np.exp(l64 - l64.max(axis=1, keepdims=True))
    ref /= ref.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(p, ref, rtol=1e-13)
    np.testing.assert_allclose(w, np.take_along_axis(ref, idx, 1), rtol=1e-13)
    assert np.all(w.sum(axis=1) < 1.0)            # no renormalisation
    assert np.all(np.diff(w, axis=1) <= 0)        # greedy order


def test_one_hot_logits_put_weight_one_on_the_winner():
    lg = np.zeros((2, 64), np.float32)
    lg[0, 41] = 60.0
    lg[1, 3] = 60.0
    idx, w, _ = oracle.softmax_topk(lg, 6)
    assert idx[0, 0] == 41 and idx[1, 0] == 3
    assert idx[0, 1:].tolist() == [0, 1, 2, 3, 4]
    np.testing.assert_allclose(w[:, 0], 1.0, rtol=1e-20, atol=1e-24)
    assert np.all(w[:, 1:] < 1e-25)


# ------------------------------------------------------------------ dispatch

@pytest.mark.parametrize("T", [1, 5, 64, 289])
def test_dispatch_invariants_and_stable_sort(T):
    rng = np.random.default_rng(T)
    idx = np.stack([rng.permutation(64)[:6] for _ in range(T)]).astype(np.int32)
    counts, offsets, perm = oracle.dispatch(idx, 64)
    flat = idx.reshape(-1)
    assert counts.sum() == 6 * T
    assert np.array_equal(counts, np.bincount(flat, minlength=64))
    assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(np.sort(perm), np.arange(6 * T))              # bijection
    assert np.array_equal(perm, np.argsort(flat, kind="stable"))        # library stable sort
    for e in range(64):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e)
        assert np.all(np.diff(seg // 6) > 0)                            # token ascending


# ------------------------------------------------------------------ expert math
# franken_ocr README, "Architecture": each expert 1280 -> 896, SiLU-gated.

def _silu(v):
    return v / (1.0 + np.exp(-v))


def _np_swiglu(G, U, D, x):
    return D @ (_silu(G @ x) * (U @ x))


@pytest.mark.parametrize("wtype,group", [(oracle.W_INT4, 16), (oracle.W_INT8, 32), (oracle.W_BF16, 0)])
def test_swiglu_equals_dense_numpy_on_dequantised_weights(wtype, group):
    G = oracle.OMat(synth.weights_f32(9, 1, (48, 64)), wtype, group)
    U = oracle.OMat(synth.weights_f32(9, 2, (48, 64)), wtype, group)
    D = oracle.OMat(synth.weights_f32(9, 3, (64, 48)), wtype, group)
    x = synth.normal_f32(9, 4, (64,)).astype(np.float64)
    y = oracle.swiglu(G, U, D, x)
    ref = _np_swiglu(G.dequant(), U.dequant(), D.dequant(), x)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(oracle.gemv(G, x), G.dequant() @ x, rtol=1e-12, atol=1e-15)


def test_dequant_of_int4_codes_is_q_times_group_scale():
    w = synth.weights_f32(9, 5, (4, 64))
    m = oracle.OMat(w, oracle.W_INT4, 16)
    d = m.dequant()
    for r in range(4):
        for c in range(64):
            assert d[r, c] == float(m.q[r, c]) * float(m.s[r, c // 16])


def _tiny_layer(seed, E=8, H=64, I=32, Is=64, rt=oracle.W_INT4, st=oracle.W_BF16, g=16,
                same_experts=False, zero_routed=False, zero_shared=False):
    def w(tid, shape):
        return synth.weights_f32(seed, tid, shape)
    gate, up, down = w(2, (E, I, H)), w(3, (E, I, H)), w(4, (E, H, I))
    if same_experts:
        gate[:], up[:], down[:] = gate[0], up[0], down[0]
    if zero_routed:
        gate[:] = 0
        up[:] = 0
        down[:] = 0
    sg, su, sd = w(5, (Is, H)), w(6, (Is, H)), w(7, (H, Is))
    if zero_shared:
        sg[:] = 0
        su[:] = 0
        sd[:] = 0
    return synth.MoELayerInputs(
        router_bf16=synth.f32_to_bf16_bits(synth.normal_f32(seed, 1, (E, H), 0.3)),
        gate=gate, up=up, down=down, sgate=sg, sup=su, sdown=sd,
        routed_type=rt, shared_type=st, group=g)


def _np_layer(om, x, k):
    """Independent numpy restatement of the layer on the oracle's quantised weights."""
    E, I, H = om.E, om.I, om.H
    G = om.gate.dequant().reshape(E, I, H)
    U = om.up.dequant().reshape(E, I, H)
    D = om.down.dequant().reshape(E, H, I)
    wr = synth.bf16_bits_to_f32(om.router).astype(np.float64)
    out = np.zeros((x.shape[0], H))
    for t in range(x.shape[0]):
        xt = x[t].astype(np.float64)
        lg = (wr @ xt).astype(np.float32).astype(np.float64)
        p = np.exp(lg - lg.max())
        p /= p.sum()
        sel = np.lexsort((np.arange(E), -lg))[:k]
        for e in sel:
            out[t] += p[e] * _np_swiglu(G[e], U[e], D[e], xt)
        out[t] += _np_swiglu(om.sgate.dequant(), om.sup.dequant(), om.sdown.dequant(), xt)
    return out


@pytest.mark.parametrize("rt,st", [(oracle.W_INT4, oracle.W_BF16), (oracle.W_INT8, oracle.W_INT8)])
def test_moe_layer_matches_numpy_restatement(rt, st):
    om = oracle.OracleMoE(_tiny_layer(11, rt=rt, st=st), topk=3)
    x = synth.normal_f32(11, 50, (5, 64))
    r = om.forward(x)
    ref = _np_layer(om, x, 3)
    np.testing.assert_allclose(r["out"], ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())


def test_identical_experts_scale_by_sum_of_weights():
    om = oracle.OracleMoE(_tiny_layer(12, same_experts=True), topk=3)
    x = synth.normal_f32(12, 50, (4, 64))
    r = om.forward(x)
    G = om.gate.dequant()[:om.I]
    U = om.up.dequant()[:om.I]
    D = om.down.dequant()[:om.H]
    for t in range(4):
        xt = x[t].astype(np.float64)
        e_out = _np_swiglu(G, U, D, xt)
        s_out = _np_swiglu(om.sgate.dequant(), om.sup.dequant(), om.sdown.dequant(), xt)
        ref = r["w"][t].sum() * e_out + s_out
        np.testing.assert_allclose(r["out"][t], ref, rtol=1e-6, atol=1e-7 * np.abs(ref).max())


def test_zero_routed_experts_leave_only_the_shared_expert():
    om = oracle.OracleMoE(_tiny_layer(13, zero_routed=True), topk=3)
    x = synth.normal_f32(13, 50, (3, 64))
    r = om.forward(x)
    for t in range(3):
        ref = _np_swiglu(om.sgate.dequant(), om.sup.dequant(), om.sdown.dequant(), x[t].astype(np.float64))
        np.testing.assert_allclose(r["out"][t], ref, rtol=1e-6, atol=1e-7 * np.abs(ref).max())


def test_zero_shared_expert_leaves_only_the_routed_sum():
    om = oracle.OracleMoE(_tiny_layer(14, zero_shared=True), topk=3)
    x = synth.normal_f32(14, 50, (3, 64))
    r = om.forward(x)
    E, I, H = om.E, om.I, om.H
    G = om.gate.dequant().reshape(E, I, H)
    U = om.up.dequant().reshape(E, I, H)
    D = om.down.dequant().reshape(E, H, I)
    for t in range(3):
        xt = x[t].astype(np.float64)
        ref = sum(r["w"][t, j] * _np_swiglu(G[e], U[e], D[e], xt) for j, e in enumerate(r["idx"][t]))
        np.testing.assert_allclose(r["out"][t], ref, rtol=1e-6, atol=1e-7 * np.abs(ref).max())


def test_fused_shared_expert_is_the_sum_of_its_two_halves():
    # "2 fused shared experts" = one SwiGLU of width 2*I; groups never straddle the halves.
    H, Ih = 64, 32
    for wtype, g in ((oracle.W_BF16, 0), (oracle.W_INT8, 16), (oracle.W_INT4, 16)):
        sg = synth.weights_f32(15, 5, (2 * Ih, H))
        su = synth.weights_f32(15, 6, (2 * Ih, H))
        sd = synth.weights_f32(15, 7, (H, 2 * Ih))
        x = synth.normal_f32(15, 8, (H,)).astype(np.float64)
        fused = oracle.swiglu(oracle.OMat(sg, wtype, g), oracle.OMat(su, wtype, g), oracle.OMat(sd, wtype, g), x)
        halves = sum(oracle.swiglu(oracle.OMat(sg[h * Ih:(h + 1) * Ih], wtype, g),
                                   oracle.OMat(su[h * Ih:(h + 1) * Ih], wtype, g),
                                   oracle.OMat(np.ascontiguousarray(sd[:, h * Ih:(h + 1) * Ih]), wtype, g), x)
                     for h in range(2))
        np.testing.assert_allclose(fused, halves, rtol=1e-12, atol=1e-15)


def test_routing_debug_outputs_agree_with_the_standalone_steps():
    om = oracle.OracleMoE(_tiny_layer(16, E=16), topk=4)
    x = synth.normal_f32(16, 50, (9, 64))
    r = om.forward(x)
    lg = oracle.router_logits(x, om.router)
    idx, w, _ = oracle.softmax_topk(lg, 4)
    counts, offsets, perm = oracle.dispatch(idx, 16)
    assert np.array_equal(r["logits"], lg) and np.array_equal(r["idx"], idx)
    assert np.array_equal(r["w"], w) and np.array_equal(r["perm"], perm)
    assert np.array_equal(r["counts"], counts) and np.array_equal(r["offsets"], offsets)


# ------------------------------------------------------------------ companions
# frankenocr.pages.dev, "One forward pass" step 7: final RMSNorm, lm_head GEMV, greedy.

def test_rmsnorm_closed_forms():
    c = np.float32(2.5)
    x = np.full((1, 1280), c, np.float32)
    y = oracle.rmsnorm(x, eps=1e-6)
    np.testing.assert_allclose(y, c / np.sqrt(c * c + 1e-6), rtol=1e-7)
    x = synth.normal_f32(17, 1, (4, 1280))
    y = oracle.rmsnorm(x, eps=0.0)
    np.testing.assert_allclose((y.astype(np.float64) ** 2).mean(axis=1), 1.0, rtol=1e-6)
    np.testing.assert_allclose(oracle.rmsnorm(3 * x, eps=0.0), y, rtol=1e-6)
    gamma = synth.normal_f32(17, 2, (1280,))
    np.testing.assert_allclose(oracle.rmsnorm(x, gamma, eps=0.0), y * gamma, rtol=1e-6, atol=1e-6)


def test_lm_head_scale_and_argmax_brute_force():
    w = synth.weights_f32(18, 1, (300, 1280))
    w[100] = w[37]                     # exact tie: the lower row wins
    w[37] *= np.float32(1.0)
    head = oracle.OracleLMHead(w)
    np.testing.assert_array_equal(head.s, (np.abs(w).max(axis=1) / np.float32(127)).astype(np.float32))
    x = synth.normal_f32(18, 2, (6, 1280))
    x[5] = np.sign(w[37]) * np.float32(5.0)   # token 5 points at row 37 (and its twin 100)
    am, logits = head.forward(x, want_logits=True)
    ref = (x.astype(np.float64) @ head.q.astype(np.float64).T) * head.s.astype(np.float64)[None, :]
    np.testing.assert_allclose(logits, ref.astype(np.float32), rtol=1e-6, atol=1e-6)
    for t in range(6):
        lg = logits[t]
        assert am[t] == int(np.flatnonzero(lg == lg.max())[0])
    assert am[5] == 37


def test_dense_mlp_matches_numpy():
    d = synth.dense_mlp(19, inter=200)
    od = oracle.OracleDense(d.gate, d.up, d.down, oracle.W_INT8, 128)   # 200 = 128 + 72 tail
    x = synth.normal_f32(19, 4, (3, 1280))
    out = od.forward(x)
    for t in range(3):
        ref = _np_swiglu(od.G.dequant(), od.U.dequant(), od.D.dequant(), x[t].astype(np.float64))
        np.testing.assert_allclose(out[t], ref, rtol=1e-6, atol=1e-7 * np.abs(ref).max())


# ------------------------------------------------------------------ dimensions

def _dims():
    d = {}
    with open(os.path.join(GOLDEN, "model_dims.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                k, v = line.split()
                d[k] = int(v)
    return d


def test_page_dimensions_and_matrix_counts():
    d = _dims()
    assert (synth.H, synth.E, synth.TOPK, synth.I, synth.VOCAB) == (
        d["hidden"], d["routed_experts"], d["topk"], d["moe_intermediate"], d["vocab"])
    # the shared pair is fused: width 2 x 896
    assert synth.IS == d["shared_experts"] * d["moe_intermediate"]
    # 2,148 quantised FFN matrices = dense layer 0 (3) + 11 MoE layers x (64 x 3 routed + 3 shared):
    # only a single fused gate/up/down triple per layer for the shared pair fits the count.
    assert d["quantized_ffn_matrices"] == 3 + d["moe_layers"] * (d["routed_experts"] * 3 + 3)
    assert d["quantized_ffn_matrices"] != 3 + d["moe_layers"] * (d["routed_experts"] * 3 + 3 * d["shared_experts"])
    assert d["attention_projections"] == d["decoder_layers"] * 4
    assert d["hidden"] == d["heads"] * d["head_dim"]
    assert synth.DENSE_I == d["int8_selftest_worst_k"]


def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: the even neighbour (1) wins;
    # 1 + 3*2^-8 lies halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even).
    vals = np.array([1.0, 1.00390625, 1.01171875, 1.0078125, -1.00390625, 1.005], np.float32)
    exp = np.array([1.0, 1.0, 1.015625, 1.0078125, -1.0, 1.0078125], np.float32)
    np.testing.assert_array_equal(oracle.round_bf16(vals), exp)
    np.testing.assert_array_equal(oracle.f32_to_bf16(vals), synth.f32_to_bf16_bits(vals))


# ------------------------------------------------------------------ W8A8 GEMV
# franken_ocr README, "CPU Backend and Optimizations": the int8 decode linears quantise the
# activation per token and run an integer GEMV with exact i32 accumulation; "Command Reference",
# `focr robot`: the worst case is K = 6848.

def _w8a8_golden():
    out = []
    with open(os.path.join(GOLDEN, "w8a8_activation_cases.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                x, s, q = [p.strip() for p in line.split("|")]
                out.append((np.array(x.split(), np.float32), np.float32(s), np.array(q.split(), np.int8)))
    return out


@pytest.mark.parametrize("case", _w8a8_golden(), ids=lambda c: f"K{c[0].size}-s{c[1]}")
def test_w8a8_activation_golden(case):
    x, s_exp, q_exp = case
    qx, sx = oracle.w8a8_quantize_x(x[None, :])
    assert sx[0] == s_exp
    np.testing.assert_array_equal(qx[0], q_exp)


def test_w8a8_activation_error_bound_and_extreme_code():
    rng = np.random.default_rng(81)
    x = (rng.standard_normal((9, 333)) * rng.uniform(1e-3, 1e3, (9, 1))).astype(np.float32)
    x[2, 5] = -50.0 * np.abs(x[2]).max()    # a negative outlier owns the scale
    qx, sx = oracle.w8a8_quantize_x(x)
    amax = np.abs(x).max(axis=1)
    np.testing.assert_array_equal(np.abs(qx).max(axis=1), 127)
    np.testing.assert_array_equal(qx[np.arange(9), np.abs(x).argmax(axis=1)],
                                  (127 * np.sign(x[np.arange(9), np.abs(x).argmax(axis=1)])).astype(np.int8))
    assert np.all(np.abs(sx.astype(np.float64) * 127 - amax) <= 1e-6 * amax)
    err = np.abs(qx.astype(np.float64) * sx[:, None] - x)
    assert np.all(err <= 0.5 * sx[:, None].astype(np.float64) * (1 + 1e-5))


def test_w8a8_power_of_two_scales_give_the_exact_product():
    # every max is 127 * 2^e and every entry a multiple of 2^e: both quantisers are exact, and
    # K * 127^2 < 2^24 keeps the fp32 result exact, so y must equal the plain integer dot product
    rng = np.random.default_rng(82)
    N, K, T = 37, 64, 3
    iw = rng.integers(-127, 128, (N, K)); iw[:, 7] = 127
    ix = rng.integers(-127, 128, (T, K)); ix[:, 11] = -127
    ew, ex = rng.integers(-6, 4, N), np.array([-3, 0, 5])
    w = (iw * 2.0 ** ew[:, None]).astype(np.float32)
    x = (ix * 2.0 ** ex[:, None]).astype(np.float32)
    y, qx, sx = oracle.OracleW8A8(w).forward(x)
    np.testing.assert_array_equal(qx, ix.astype(np.int8))
    np.testing.assert_array_equal(sx, (2.0 ** ex).astype(np.float32))
    exact = (ix.astype(np.int64) @ iw.T.astype(np.int64)) * 2.0 ** (ex[:, None] + ew[None, :])
    np.testing.assert_array_equal(y, exact.astype(np.float32))


def test_w8a8_worst_case_accumulator_fits_i32_at_k6848():
    K = synth.DENSE_I
    assert K == 6848
    w = np.full((2, K), 127.0, np.float32)
    w[1, 1::2] = -127.0
    x = np.full((1, K), 127.0, np.float32)
    y, _, _, acc = oracle.OracleW8A8(w).forward(x, want_acc=True)
    assert acc[0, 0] == K * 127 * 127 == 110_451_392 < 2 ** 31 - 1
    assert acc[0, 1] == 0
    # s_w = s_x = 1, and 110,451,392 is a multiple of 8 (the fp32 spacing there): y is acc exactly
    assert y[0, 0] == 110_451_392.0 and y[0, 1] == 0.0


def test_w8a8_gemv_brute_force_integer_dot():
    rng = np.random.default_rng(83)
    N, K, T = 5, 29, 4
    w = rng.standard_normal((N, K)).astype(np.float32)
    x = rng.standard_normal((T, K)).astype(np.float32)
    om = oracle.OracleW8A8(w)
    y, qx, sx, acc = om.forward(x, want_acc=True)
    for t in range(T):
        for n in range(N):
            a = sum(int(om.q[n, k]) * int(qx[t, k]) for k in range(K))
            assert acc[t, n] == a
            assert y[t, n] == np.float32((float(om.s[n]) * float(sx[t])) * a)
    # against the unquantised product: the error of symmetric 8-bit codes on both sides
    ref = x.astype(np.float64) @ w.T.astype(np.float64)
    assert np.abs(y - ref).max() <= 0.05 * np.abs(ref).max()


# ------------------------------------------------------------------ R-SWA decode attention
# franken_ocr README, "Design Philosophy" (bounded generated-token KV) and "Architecture" (R-SWA):
# a generated token attends to every reference row plus the last 128 generated tokens, which a
# 128-slot ring holds; frankenocr.pages.dev, "One forward pass", step 6: 10 heads of dimension 128.

RH, RD, RW = oracle.RSWA_HEADS, oracle.RSWA_DIM, oracle.RSWA_RING


def _rswa_inputs(seed, B, Rcap, fill=0.0):
    rng = np.random.default_rng(seed)
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    return dict(q=f(B, RH, RD), k_new=f(B, RH, RD), v_new=f(B, RH, RD), k_ref=f(B, RH, Rcap, RD),
                v_ref=f(B, RH, Rcap, RD), k_ring=f(B, RH, RW, RD) + fill, v_ring=f(B, RH, RW, RD) + fill)


def _rswa(a, ref_len, n_gen):
    return oracle.rswa_decode(a["q"], a["k_new"], a["v_new"], a["k_ref"], a["v_ref"], ref_len, a["k_ring"],
                              a["v_ring"], n_gen)


def test_rswa_single_key_returns_its_value():
    a = _rswa_inputs(91, 2, 4)
    out, kg, vg = _rswa(a, [0, 0], [1, 1])
    np.testing.assert_array_equal(out, a["v_new"])                  # one key: weight exactly 1
    np.testing.assert_array_equal(kg[:, :, 0], a["k_new"])         # token 0 goes to slot 0
    np.testing.assert_array_equal(vg[:, :, 1:], a["v_ring"][:, :, 1:])


def test_rswa_two_keys_take_hand_computed_weights():
    # q . k_ref / sqrt(128) = ln 3 and q . k_new = 0: softmax weights 3/4 and 1/4
    a = _rswa_inputs(92, 1, 3)
    a["q"][:] = 0.0
    a["q"][0, :, 5] = 2.0
    a["k_ref"][:] = 0.0
    a["k_ref"][0, :, 0, 5] = np.float32(np.sqrt(128.0) * np.log(3.0) / 2.0)
    a["k_new"][:] = 0.0
    out, _, _ = _rswa(a, [1], [1])
    exp = 0.75 * a["v_ref"][:, :, 0].astype(np.float64) + 0.25 * a["v_new"].astype(np.float64)
    np.testing.assert_allclose(out, exp, rtol=0, atol=1e-6)


def test_rswa_zero_query_averages_the_window():
    # q = 0 gives equal weights: the output is the mean of the attended values
    a = _rswa_inputs(93, 1, 40)
    a["q"][:] = 0.0
    R, n = 17, 300
    out, _, _ = _rswa(a, [R], [n])
    cur = (n - 1) % RW
    ring = a["v_ring"][0].astype(np.float64).copy()
    ring[:, cur] = a["v_new"][0]
    vals = np.concatenate([a["v_ref"][0, :, :R].astype(np.float64), ring], axis=1)
    np.testing.assert_allclose(out[0], vals.mean(axis=1), rtol=0, atol=1e-6)


@pytest.mark.parametrize("n", [5, 128, 129, 300])
def test_rswa_window_is_the_last_128_generated_tokens(n):
    # slots outside the window, and the current slot's stale token (n - 129), must not matter
    a = _rswa_inputs(94, 1, 8)
    base, kg, vg = _rswa(a, [6], [n])
    b = {k: v.copy() for k, v in a.items()}
    cur = (n - 1) % RW
    outside = [s for s in range(RW) if s >= n] + [cur]
    b["k_ring"][:, :, outside] = 1e4
    b["v_ring"][:, :, outside] = -7e3
    other, kg2, vg2 = _rswa(b, [6], [n])
    np.testing.assert_array_equal(other, base)
    np.testing.assert_array_equal(kg2[:, :, cur], a["k_new"])     # the current token is stored at (n - 1) mod 128
    np.testing.assert_array_equal(vg2[:, :, cur], a["v_new"])
    keep = [s for s in range(RW) if s != cur]
    np.testing.assert_array_equal(vg2[:, :, keep], b["v_ring"][:, :, keep])
    # a slot inside the window does matter
    if n > 1:
        c = {k: v.copy() for k, v in a.items()}
        c["v_ring"][:, :, (n - 2) % RW] += 1.0
        assert not np.array_equal(_rswa(c, [6], [n])[0], base)


def test_rswa_reference_rows_are_attended():
    a = _rswa_inputs(95, 1, 10)
    base, _, _ = _rswa(a, [7], [3])
    b = {k: v.copy() for k, v in a.items()}
    b["v_ref"][:, :, 6] += 1.0                   # the last reference row counts
    assert not np.array_equal(_rswa(b, [7], [3])[0], base)
    c = {k: v.copy() for k, v in a.items()}
    c["k_ref"][:, :, 7:] = 1e4                   # rows beyond ref_len do not
    c["v_ref"][:, :, 7:] = 1e6
    np.testing.assert_array_equal(_rswa(c, [7], [3])[0], base)


def test_rswa_one_dominant_key_with_huge_scores():
    # scores near 1e4: the largest key takes all the weight and nothing overflows
    a = _rswa_inputs(96, 1, 5)
    a["q"][:] = 0.0
    a["q"][0, :, 0] = 100.0
    a["k_ref"][:] = 0.0
    a["k_ref"][0, :, :, 0] = np.array([10, 12, 20, 11, 9], np.float32)[None, :] * 100.0
    a["k_new"][:] = 0.0
    out, _, _ = _rswa(a, [5], [1])
    assert np.isfinite(out).all()
    np.testing.assert_allclose(out[0], a["v_ref"][0, :, 2], rtol=0, atol=1e-6)


def test_rswa_sequences_are_independent_and_bad_lengths_give_nan():
    a = _rswa_inputs(97, 3, 12)
    lens, gens = [12, 0, 5], [1, 200, 64]
    out, kg, vg = _rswa(a, lens, gens)
    for b in range(3):
        one = {k: v[b:b + 1] for k, v in a.items()}
        o1, k1, v1 = _rswa(one, [lens[b]], [gens[b]])
        np.testing.assert_array_equal(out[b], o1[0])
        np.testing.assert_array_equal(kg[b], k1[0])
    bad, kgb, _ = _rswa(a, [13, -1, 5], [1, 5, 0])
    assert np.isnan(bad).all()
    np.testing.assert_array_equal(kgb, a["k_ring"])   # rings unchanged
