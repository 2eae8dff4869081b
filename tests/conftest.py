import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this environment")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


# ---------------------------------------------------------------- shared GPU fixtures
import functools  # noqa: E402

import numpy as np  # noqa: E402


@functools.lru_cache(maxsize=None)
def moe_case(seed: int, routed: int, shared: int, group: int, skew: bool = False):
    """(OracleMoE, packed device layer) for one synthetic layer; fp32 inputs are dropped."""
    import oracle
    from weight_quantized_expert_b200 import api, synth
    layer = synth.moe_layer(seed, routed, shared, group, skew=skew)
    om = oracle.OracleMoE(layer)
    packed = api.focr_moe_pack_weights(layer)
    del layer
    return om, packed


def per_token_rel_err(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return np.abs(got - ref).max(axis=1) / np.abs(ref).max(axis=1)
