"""Seeded synthetic inputs for the MoE layer (and its decode-stack companions).

This module only *creates inputs*: hidden states, fp32 expert weights, a bf16
router matrix, the dense layer-0 weights and the lm_head matrix.  It holds none
of the method's arithmetic (no quantisation, routing or expert math), so both
the CPU oracle and the CUDA path can take their inputs from here.

Shapes follow the Unlimited-OCR decoder as described by the pages
("frankenocr.pages.dev", section "One forward pass", step 6 for the MoE layer;
"franken_ocr" README, section "Design Philosophy", for the fixed dimensions):
hidden 1280, 64 routed experts, top-6, expert intermediate 896, two fused shared
experts (one SwiGLU of width 1792), vocab 129280, dense layer-0 intermediate 6848.

Recipe (stated once, used by every config):
  * normal draws: Box-Muller in fp64 from two uniform draws of a PCG64 stream,
    then rounded to fp32;
  * expert / shared / dense / lm_head weights ~ N(0, 0.02), then a Bernoulli(0.001)
    mask of positions multiplied by 20 (outliers);
  * router weights ~ N(0, 0.02) rounded to bf16 (round-to-nearest-even bits);
  * hidden states ~ N(0, 1);
  * skewed routing (batched-decode config): a seeded unit vector u; router row e
    gets + (alpha / (e + 1)) * u with alpha = 0.5, token t gets + beta * u with
    beta = 8, so low-index experts win far more often (a Zipf-like load).
Every tensor has its own sub-stream: SeedSequence([seed, tensor_id]).
"""
from __future__ import annotations

import dataclasses
import numpy as np

H = 1280          # hidden size
E = 64            # routed experts
TOPK = 6          # experts per token
I = 896           # routed expert intermediate
IS = 1792         # fused shared-expert intermediate (2 x 896)
VOCAB = 129280    # lm_head rows
DENSE_I = 6848    # dense layer-0 intermediate

W_STD = 0.02
OUTLIER_P = 0.001
OUTLIER_MUL = 20.0
SKEW_ALPHA = 0.5
SKEW_BETA = 8.0

# weight type tags shared with the C ABI (focr_wtype)
W_BF16, W_INT8, W_INT4 = 0, 1, 2

_CHUNK = 1 << 22


def _stream(seed: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor_id])))


def normal_f32(seed: int, tensor_id: int, shape, std: float = 1.0) -> np.ndarray:
    """N(0, std^2) draws by Box-Muller in fp64, rounded to fp32."""
    rng = _stream(seed, tensor_id)
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    pos = 0
    while pos < n:
        m = min(_CHUNK, n - pos)
        half = (m + 1) // 2
        u1 = rng.random(half)
        u2 = rng.random(half)
        r = np.sqrt(-2.0 * np.log1p(-u1))       # 1 - u1 lies in (0, 1]
        ang = 2.0 * np.pi * u2
        z = np.empty(2 * half, dtype=np.float64)
        z[0::2] = r * np.cos(ang)
        z[1::2] = r * np.sin(ang)
        out[pos:pos + m] = (z[:m] * std).astype(np.float32)
        pos += m
    return out.reshape(shape)


def weights_f32(seed: int, tensor_id: int, shape, std: float = W_STD,
                outliers: bool = True) -> np.ndarray:
    """N(0, std^2) weights with Bernoulli(0.001) positions scaled by 20."""
    w = normal_f32(seed, tensor_id, shape, std)
    if outliers:
        rng = _stream(seed, 10_000 + tensor_id)
        flat = w.reshape(-1)
        pos = 0
        n = flat.size
        while pos < n:
            m = min(_CHUNK, n - pos)
            mask = rng.random(m) < OUTLIER_P
            flat[pos:pos + m][mask] *= np.float32(OUTLIER_MUL)
            pos += m
    return w


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the 16-bit patterns.
    Input synthesis only: the router is *given* as a bf16 tensor."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = ((u >> 16) & 1) + 0x7FFF
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class MoELayerInputs:
    """fp32 weights in nn.Linear orientation [out, in]; router as bf16 bits."""
    router_bf16: np.ndarray   # [E, H] uint16
    gate: np.ndarray          # [E, I, H] f32
    up: np.ndarray            # [E, I, H] f32
    down: np.ndarray          # [E, H, I] f32
    sgate: np.ndarray         # [IS, H] f32
    sup: np.ndarray           # [IS, H] f32
    sdown: np.ndarray         # [H, IS] f32
    routed_type: int
    shared_type: int
    group: int


def moe_layer(seed: int, routed_type: int, shared_type: int, group: int,
              skew: bool = False, layer_id: int = 0) -> MoELayerInputs:
    base = 100 * layer_id
    router = normal_f32(seed, base + 1, (E, H), W_STD)
    if skew:
        u = _skew_direction(seed)
        router = router + (SKEW_ALPHA / (np.arange(E, dtype=np.float32) + 1.0))[:, None] * u[None, :]
        router = router.astype(np.float32)
    return MoELayerInputs(
        router_bf16=f32_to_bf16_bits(router),
        gate=weights_f32(seed, base + 2, (E, I, H)),
        up=weights_f32(seed, base + 3, (E, I, H)),
        down=weights_f32(seed, base + 4, (E, H, I)),
        sgate=weights_f32(seed, base + 5, (IS, H)),
        sup=weights_f32(seed, base + 6, (IS, H)),
        sdown=weights_f32(seed, base + 7, (H, IS)),
        routed_type=routed_type, shared_type=shared_type, group=group)


def _skew_direction(seed: int) -> np.ndarray:
    v = normal_f32(seed, 99, (H,), 1.0).astype(np.float64)
    return (v / np.linalg.norm(v)).astype(np.float32)


def hidden(seed: int, T: int, skew: bool = False, stream_id: int = 50) -> np.ndarray:
    x = normal_f32(seed, stream_id, (T, H), 1.0)
    if skew:
        x = (x + SKEW_BETA * _skew_direction(seed)[None, :]).astype(np.float32)
    return x


def prefill_hidden(seed: int) -> np.ndarray:
    """289 rows: 273 'visual' rows (BOS + 16 x (16 patches + newline) + separator)
    followed by 16 prompt rows, all ~N(0, 1)."""
    vis = normal_f32(seed, 51, (273, H), 1.0)
    prompt = normal_f32(seed, 52, (16, H), 1.0)
    return np.concatenate([vis, prompt], axis=0)


@dataclasses.dataclass
class DenseMLPInputs:
    gate: np.ndarray   # [DENSE_I, H]
    up: np.ndarray     # [DENSE_I, H]
    down: np.ndarray   # [H, DENSE_I]


def dense_mlp(seed: int, inter: int = DENSE_I) -> DenseMLPInputs:
    return DenseMLPInputs(gate=weights_f32(seed, 2001, (inter, H)),
                          up=weights_f32(seed, 2002, (inter, H)),
                          down=weights_f32(seed, 2003, (H, inter)))


def lm_head(seed: int, vocab: int = VOCAB) -> np.ndarray:
    return weights_f32(seed, 3001, (vocab, H))


RSWA_HEADS, RSWA_DIM, RSWA_RING = 10, 128, 128
RSWA_REF = 289   # reference block of the prefill workload: 273 visual rows + 16 prompt rows


def rswa_inputs(seed: int, B: int, Rcap: int) -> dict:
    """One R-SWA decode step's tensors for B sequences, all ~N(0, 1) (so q . k / sqrt(128) ~ N(0, 1)):
    q, k_new, v_new [B, 10, 128]; k_ref, v_ref [B, 10, Rcap, 128]; k_ring, v_ring [B, 10, 128, 128]."""
    sh, sr, sg = (B, RSWA_HEADS, RSWA_DIM), (B, RSWA_HEADS, Rcap, RSWA_DIM), (B, RSWA_HEADS, RSWA_RING, RSWA_DIM)
    return dict(q=normal_f32(seed, 4001, sh), k_new=normal_f32(seed, 4002, sh), v_new=normal_f32(seed, 4003, sh),
                k_ref=normal_f32(seed, 4004, sr), v_ref=normal_f32(seed, 4005, sr),
                k_ring=normal_f32(seed, 4006, sg), v_ring=normal_f32(seed, 4007, sg))


# ---------------------------------------------------------------- workloads
# The five measured workloads of the method (one MoE layer at hidden 1280).
WORKLOADS = {
    "t1_int8_g128": dict(seed=0, T=1, routed=W_INT8, shared=W_INT8, group=128),
    "t1_int4_g32": dict(seed=1, T=1, routed=W_INT4, shared=W_BF16, group=32),
    "t1_int4_g64": dict(seed=1, T=1, routed=W_INT4, shared=W_BF16, group=64),
    "t1_int4_g128": dict(seed=1, T=1, routed=W_INT4, shared=W_BF16, group=128),
    "batch8_int4_g64_skew": dict(seed=2, T=8, routed=W_INT4, shared=W_BF16, group=64, skew=True),
    "batch32_int4_g64_skew": dict(seed=2, T=32, routed=W_INT4, shared=W_BF16, group=64, skew=True),
    "batch64_int4_g64_skew": dict(seed=2, T=64, routed=W_INT4, shared=W_BF16, group=64, skew=True),
    "prefill289_int4_g64": dict(seed=3, T=289, routed=W_INT4, shared=W_BF16, group=64, prefill=True),
}


# The decode-step companions and the stack of one decode step: dense SwiGLU layer 0 (int8 g128),
# 11 MoE layers (int4 g64, bf16 router and shared expert), final RMSNorm, int8 lm_head + argmax.
STEP_WORKLOADS = {
    "lm_head_t1": dict(kind="lm_head", seed=4, T=1),
    "dense_t1": dict(kind="dense", seed=4, T=1),
    "stack_t1": dict(kind="stack", seed=4, T=1, moe_layers=11),
    "stack_t32": dict(kind="stack", seed=4, T=32, moe_layers=11),
    # W8A8 GEMV on the lm_head's shape (129280 x 1280 int8, one scale per row; 165 MB > L2)
    "w8a8_lm_head_t1": dict(kind="w8a8", seed=4, T=1),
    "w8a8_lm_head_t8": dict(kind="w8a8", seed=4, T=8),
    # R-SWA decode attention: T sequences, a 289-row reference block, 600 tokens generated (ring wrapped)
    "rswa_t1": dict(kind="rswa", seed=5, T=1, R=289, n_gen=600),
    "rswa_b8": dict(kind="rswa", seed=5, T=8, R=289, n_gen=600),
}


def workload(name: str):
    """Return (x [T,H] f32, MoELayerInputs) for a named workload."""
    w = WORKLOADS[name]
    layer = moe_layer(w["seed"], w["routed"], w["shared"], w["group"], skew=w.get("skew", False))
    if w.get("prefill"):
        x = prefill_hidden(w["seed"])
    else:
        x = hidden(w["seed"], w["T"], skew=w.get("skew", False))
    return x, layer
