"""bench.py times `value` through fp4_linear_fwd / fp4_linear_bwd and takes
its per-kernel split from a second region that issues the same kernels
through the primitive entry points.  The two must stay the same computation:
their outputs (Y, dX, dW and the saved context) are compared bit for bit for
every workload recipe the bench runs, on small shapes."""
import numpy as np
import pytest
import torch

import bench

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("config,M,K,N", [(1, 256, 512, 512), (2, 512, 256, 384), (3, 384, 256, 512),
                                          (4, 256, 512, 384)])
def test_primitive_sequence_equals_linear_entry_points(cuda_lib, config, M, K, N):
    cfg = dict(bench.CONFIGS[config], M=M, layers=(("linear", K, N),))
    host = bench.make_host_data(cfg)
    L = bench.Layers(cuda_lib, cfg, torch.device("cuda", 0), host)
    outs = ("Y", "dX", "dW") if cfg["bwd"] else ("Y",)
    L.linear_step(77)
    torch.cuda.synchronize()
    lay = L.layers[0]
    ref = {k: lay[k].clone() for k in outs}
    ctx_ref = [lay["ctx"].xq.codes.clone(), lay["ctx"].wq.codes.clone(), lay["ctx"].xq.scales_swz.clone()]
    for k in outs:
        lay[k].fill_(np.nan)
    rec = bench.Recorder()
    L.primitive_step(77, rec)
    torch.cuda.synchronize()
    for k in outs:
        assert torch.equal(lay[k].view(torch.int32), ref[k].view(torch.int32)), k
    assert torch.equal(lay["ctx"].xq.codes, ctx_ref[0])
    assert torch.equal(lay["ctx"].wq.codes, ctx_ref[1])
    assert torch.equal(lay["ctx"].xq.scales_swz, ctx_ref[2])
    st = rec.summary(cuda_lib)
    assert st["n_gemm"] == (3 if cfg["bwd"] else 1)
    assert st["gemm_flops"] == pytest.approx(bench.step_flops(cfg))
    assert cuda_lib.get_last_error() == 0
