"""Parity of the configuration bench.py times: R rotated weight copies of a layer
captured as one CUDA graph with DBF_FWD_WEIGHTS_STATIC (programmatic dependent
launch chaining every forward), at the full sizes of the workloads.  The
output after a replay is checked against the fp64 oracle on every token."""
import numpy as np
import pytest
import torch

import dbf_inputs as gen
import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,batch", [("attn_1b", 1), ("attn_2b", 16), ("mlp_up", 1), ("mlp_up", 2048)])
def test_bench_launch_configuration(name, batch):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import bench
    from binary_factorized_weight_b200 import build

    build.build()
    import binary_factorized_weight_b200 as dbf

    dbf.load_library()
    shape = gen.CONFIGS[name]
    wl = bench.Workload(dbf, torch, shape, batch, torch.device("cuda", 0))
    g = wl.capture()
    wl.y.fill_(float("nan"))
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert dbf.dbf_workspace_status(wl.ws) == 0
    y = wl.y.float().cpu().numpy().astype(np.float64)
    ref = oracle.forward_staged(wl.host["x"], wl.host["A"], wl.host["B"], wl.host["a"], wl.host["mid"], wl.host["b"])
    got = y  # every token
    assert np.all(np.isfinite(got))
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert rel <= 2e-3, rel
    assert np.abs(got - ref).max() <= 1e-2 * np.sqrt(np.mean(ref * ref))
    del g, wl
    torch.cuda.empty_cache()
