"""The tcgen05 tile primitives (instruction and shared-memory descriptors, TMEM allocation,
tcgen05.st / tcgen05.ld, MMA with A from shared or tensor memory) against an fp64 host GEMM,
through the C ABI's diagnostic entry focr_tc_selftest.  bf16 inputs are exact in fp64 and every
product is exact in fp32, so the only error is the fp32 accumulation order."""
import numpy as np
import pytest

from weight_quantized_expert_b200 import api

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("a_from_tmem", [False, True])
@pytest.mark.parametrize("n,k", [(16, 64), (32, 64), (112, 128), (256, 64), (48, 256)])
def test_tile_matches_host_gemm(a_from_tmem, n, k):
    import torch
    g = torch.Generator().manual_seed(1000 * n + k)
    a = torch.randn(128, k, generator=g).to(torch.bfloat16)
    b = torch.randn(n, k, generator=g).to(torch.bfloat16)
    d, err = api.focr_tc_selftest(a.cuda(), b.cuda(), a_from_tmem)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = a.double().numpy() @ b.double().numpy().T
    got = d.cpu().numpy()
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()
