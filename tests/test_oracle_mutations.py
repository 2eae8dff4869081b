"""The oracle's pins must catch plausible mistakes.

Each case copies the oracle's C source, plants one slip (in the copy only, on
the CPU), builds it, and runs the pin suite against it in a child process:
the suite has to fail.  The real oracle is never modified.
"""
import os
import subprocess
import sys
import tempfile

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "focr_oracle.c")

MUTATIONS = {
    "nibble_order_swapped": ("out[j] = (uint8_t)(lo | (hi << 4));", "out[j] = (uint8_t)(hi | (lo << 4));"),
    "silu_sign_flipped": ("return v / (1.0 + exp(-v));", "return v / (1.0 + exp(v));"),
    "topk_ties_to_higher_index": ("if (best < 0 || l[e] > l[best]) best = e;", "if (best < 0 || l[e] >= l[best]) best = e;"),
    "softmax_not_normalised": ("for (int e = 0; e < E; ++e) p[e] /= den;", ";"),
    "shared_expert_dropped": ("out[(int64_t)t * H + c] = (float)(acc[c] + y[c]);", "out[(int64_t)t * H + c] = (float)(acc[c]);"),
    "scale_index_wrong": ("(double)m->s[r * ng + c / m->group]", "(double)m->s[r * ng + c % ng]"),
    "scale_divisor_off_by_one": ("const float sc = m / (float)qmax;", "const float sc = m / (float)(qmax + 1);"),
    "round_half_away": ("float rn = nearbyintf(ratio);", "float rn = roundf(ratio);"),
    "gate_up_swapped": ("for (int64_t i = 0; i < inter; ++i) g[i] = silu(g[i]) * u[i];", "for (int64_t i = 0; i < inter; ++i) g[i] = silu(u[i]) * g[i];"),
    "dispatch_unstable": ("for (int64_t i = 0; i < (int64_t)T * k; ++i) perm[cursor[idx[i]]++] = (int32_t)i;",
                          "for (int64_t i = (int64_t)T * k - 1; i >= 0; --i) perm[cursor[idx[i]]++] = (int32_t)i;"),
    "rmsnorm_sum_not_mean": ("1.0 / sqrt(ss / (double)H + eps)", "1.0 / sqrt(ss + eps)"),
    "lm_head_ties_to_last": ("if (bi < 0 || lg > best) { best = lg; bi = n; }", "if (bi < 0 || lg >= best) { best = lg; bi = n; }"),
    "router_weight_transposed": ("(double)orc_bf16_to_f32(wr[(int64_t)e * H + k])", "(double)orc_bf16_to_f32(wr[(int64_t)k * E + e])"),
    "routed_weight_renormalised": ("acc[c] += wj * y[c];", "acc[c] += (wj / w[(int64_t)t * L->topk]) * y[c];"),
    "w8a8_x_divisor_128": ("const float sc = m / 127.0f;", "const float sc = m / 128.0f;"),
    "w8a8_x_round_half_away": ("float rn = nearbyintf(xt[k] / sc);", "float rn = roundf(xt[k] / sc);"),
    "w8a8_activation_scale_dropped": ("(float)(((double)sw[n] * (double)sx[t]) * (double)acc)",
                                      "(float)((double)sw[n] * (double)acc)"),
    "rswa_scale_dropped": ("const double inv = 1.0 / sqrt((double)D);", "const double inv = 1.0;"),
    "rswa_window_129": ("const int p0 = n > W ? n - W : 0;", "const int p0 = n > W ? n - W - 1 : 0;"),
    "rswa_reference_ignored": ("for (int r = 0; r < R; ++r) {\n                double acc = 0.0;",
                               "for (int r = 0; r < 0; ++r) {\n                double acc = 0.0;"),
    "rswa_no_max_subtraction": ("for (int j = 1; j < nk; ++j)\n                if (sc[j] > m) m = sc[j];", "m = 0.0;"),
    "rswa_ring_slot_off_by_one": ("const int slot = (n - 1) % W;", "const int slot = n % W;"),
    "w8a8_activation_transposed": ("(int64_t)qw[n * K + k] * (int64_t)qx[(int64_t)t * K + k]",
                                   "(int64_t)qw[n * K + k] * (int64_t)qx[(int64_t)k * T + t]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "mut.c"
    mutated.write_text(src.replace(old, new))
    so = oracle.compile_to(str(mutated), str(tmp_path / "libmut.so"))
    env = dict(os.environ, FOCR_ORACLE_SO=so)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"planted mistake '{name}' was not caught by any pin"
