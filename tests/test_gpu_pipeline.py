"""HostPipeline (copies overlapped with compute) returns, batch by batch, exactly what
MoELayer.forward returns for the same host inputs (needs a B200)."""
import pytest
import torch

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build
from load_balanced_dispatch_warp_b200 import inputs as I
from load_balanced_dispatch_warp_b200.pipeline import HostPipeline

pytestmark = pytest.mark.gpu


def test_pipeline_matches_forward():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    ws = [I.small_workload("p", 512, 32, 4, 8, 4, 256, 256, alpha=a, seed=s) for a, s in ((0.5, 1), (2.0, 2), (1.0, 3))]
    W = I.make_weights(ws[0], device="cuda")
    batches = [(I.make_logits(w).pin_memory(), I.make_x(w).pin_memory()) for w in ws]
    w = ws[0]
    ref_layer = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
    refs = []
    for lg, x in batches:
        refs.append(ref_layer.forward(lg.cuda(), x.cuda(), *W).clone())
    torch.cuda.synchronize()
    layer = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
    pipe = HostPipeline(layer, *W)
    outs = [torch.empty(w.T, w.d, dtype=torch.bfloat16).pin_memory() for _ in batches]
    pipe.run(batches + batches, outs + [torch.empty_like(o).pin_memory() for o in outs])
    torch.cuda.synchronize()
    assert int(layer.err.item()) == 0
    for o, r in zip(outs, refs):
        assert torch.equal(o, r.cpu())
