"""Run in a fresh process by test_threads_gpu.py: the library's first forwards come from two
host threads at once, each with its own CUDA stream and workspace (one on the small-batch
decode kernels, one on the tensor-core kernel), and both results are checked against the
oracle."""
import os
import sys
import threading

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import oracle  # noqa: E402
from weight_quantized_expert_b200 import api, synth  # noqa: E402


def main():
    import torch
    layer = synth.moe_layer(5, synth.W_INT4, synth.W_BF16, 64)
    om = oracle.OracleMoE(layer)
    packed = api.focr_moe_pack_weights(layer)
    cases = [synth.hidden(81, 1), synth.hidden(82, 33)]
    xs = [torch.from_numpy(x).cuda() for x in cases]
    streams = [torch.cuda.Stream() for _ in cases]
    wss = [api.new_workspace(x.shape[0]) for x in cases]
    outs = [None, None]
    errs = []
    torch.cuda.synchronize()
    barrier = threading.Barrier(2)

    def run(i):
        try:
            barrier.wait()
            with torch.cuda.stream(streams[i]):
                outs[i] = api.focr_moe_layer_forward(packed, xs[i], workspace=wss[i], stream=streams[i])
            streams[i].synchronize()
            api.focr_moe_check(wss[i], stream=streams[i])
        except Exception as e:  # reported by the parent test
            errs.append(repr(e))

    th = [threading.Thread(target=run, args=(i,)) for i in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    if errs:
        print("FAIL", errs)
        return 1
    for i, x in enumerate(cases):
        ref = om.forward(x, nthreads=max(1, os.cpu_count() or 1))["out"]
        got = outs[i].cpu().numpy()
        err = (np.abs(got.astype(np.float64) - ref).max(axis=1) / np.abs(ref).max(axis=1)).max()
        tol = 2e-3 if x.shape[0] <= 8 else 1e-2
        if not err <= tol:
            print("FAIL", i, x.shape[0], err)
            return 1
    print("OK")
    return 0


if __name__ == "__main__":
    sys.exit(main())
