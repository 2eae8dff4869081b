"""The byte counts the benchmark divides by, checked against figures worked out by hand
from the layer's shapes (6 experts x (2 x 896x1280 + 1280x896) weights, shared 1792,
router 64x1280 bf16, fp32 activations in and out)."""
from weight_quantized_expert_b200 import roofline as rf


def test_int8_g128_single_token():
    # int8 expert: 3 x 1,146,880 codes + 3 x 8,960 groups x 4 B = 3,548,160 B
    assert rf.swiglu_bytes(896, rf.W_INT8, 128) == 3_548_160
    assert rf.swiglu_bytes(1792, rf.W_INT8, 128) == 7_096_320
    assert rf.moe_layer_bytes(1, rf.W_INT8, rf.W_INT8, 128, 6) == 28_559_360


def test_int4_single_token_group_sweep():
    # int4 expert: 1,720,320 nibble bytes + scales (g64: 53,760 groups x 4 B = 215,040 B)
    assert rf.swiglu_bytes(896, rf.W_INT4, 64) == 1_935_360
    assert rf.swiglu_bytes(1792, rf.W_BF16, 0) == 13_762_560
    assert rf.moe_layer_bytes(1, rf.W_INT4, rf.W_BF16, 32, 6) == 26_839_040
    assert rf.moe_layer_bytes(1, rf.W_INT4, rf.W_BF16, 64, 6) == 25_548_800
    assert rf.moe_layer_bytes(1, rf.W_INT4, rf.W_BF16, 128, 6) == 24_903_680


def test_prefill_all_experts():
    assert rf.moe_layer_bytes(289, rf.W_INT4, rf.W_BF16, 64, 64) == 140_748_800
    assert abs(rf.moe_layer_flops(289) - 15.96e9) / 15.96e9 < 0.01


def test_decode_step_companions():
    # dense layer 0, int8 g128: gate/up 6848 x 1280 codes + 6848 x 10 scales; down 1280 x 6848 codes
    # + 1280 x 54 scales (the 54th group of each down row is the short 64-wide tail)
    assert rf.swiglu_bytes(6848, rf.W_INT8, 128) == 2 * (8_765_440 + 273_920) + (8_765_440 + 276_480)
    assert rf.swiglu_bytes(6848, rf.W_INT8, 128) == 27_120_640


def test_decode_step_bench_bytes():
    import bench
    from weight_quantized_expert_b200 import synth
    lm = 129_280 * 1_280 + 129_280 * 4          # int8 codes + one f32 scale per row
    assert bench.step_bytes_companion(synth.STEP_WORKLOADS["lm_head_t1"]) == lm + 1_280 * 4 + 4
    assert bench.step_bytes_companion(synth.STEP_WORKLOADS["dense_t1"]) == 27_120_640 + 2 * 1_280 * 4
    # T = 1 stack: dense + 11 MoE layers of 25,548,800 B + 12 RMSNorms (in + out) + lm_head
    got = bench.step_bytes_companion(synth.STEP_WORKLOADS["stack_t1"], [6] * 11)
    assert got == (27_120_640 + 2 * 5_120) + 11 * 25_548_800 + 12 * 2 * 5_120 + (lm + 5_120 + 4)


def test_profile_identity_ignores_comments_only(tmp_path, monkeypatch):
    import shutil
    import bench
    src = tmp_path / "weight_quantized_expert_b200" / "csrc"
    shutil.copytree(bench.os.path.join(bench.ROOT, "weight_quantized_expert_b200", "csrc"), src)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench.sources_hash()
    f = src / "rmsnorm.cu"
    f.write_text("// an extra comment line\n" + f.read_text().replace("{", "{ /* inline */", 1))
    assert bench.sources_hash() == h0
    f.write_text(f.read_text().replace("1e-6", "2e-6") + "\nstatic int focr_extra_symbol = 1;\n")
    assert bench.sources_hash() != h0


def test_w8a8_and_rswa_bench_bytes():
    import bench
    from weight_quantized_expert_b200 import synth
    # W8A8 at the lm_head's shape, T = 1: 165,478,400 codes + 517,120 scale bytes + 5,120 B of x + 517,120 B of y
    assert bench.step_bytes_companion(synth.STEP_WORKLOADS["w8a8_lm_head_t1"]) == 166_517_760
    # R-SWA, one sequence, 289 reference rows + a full 128-slot window: 417 keys x (k + v) x 10 heads x 512 B,
    # plus q, k_new, v_new, out and the two ring-slot rows (6 x 5,120 B)
    assert bench.rswa_step_bytes(synth.STEP_WORKLOADS["rswa_t1"]) == 417 * 2 * 5_120 + 6 * 5_120 == 4_300_800
    assert bench.rswa_step_bytes(synth.STEP_WORKLOADS["rswa_b8"]) == 8 * 4_300_800
    # a window that has not filled yet counts only the generated tokens so far
    assert bench.rswa_step_bytes(dict(T=1, R=10, n_gen=5)) == (10 + 5) * 2 * 5_120 + 6 * 5_120
