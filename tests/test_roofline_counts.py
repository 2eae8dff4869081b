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
