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


def test_first_forward_inside_graph_capture():
    """A layer whose very first forward is captured: replays equal an eager layer's output,
    and the forward (fused routing call) equals the seven separate calls run in order."""
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    w = I.small_workload("cap", 768, 64, 6, 8, 8, 256, 384, alpha=0.8, seed=31)
    W = I.make_weights(w, device="cuda")
    lg, x = I.make_logits(w).cuda(), I.make_x(w).cuda()
    eager = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
    ref = eager.forward(lg, x, *W).clone()
    seq = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
    seq.route(lg)
    seq.measure()
    seq.balance()
    seq.prefetch(*W)
    seq.dispatch(x)
    seq.expert_ffn(*W)
    seq.combine()
    torch.cuda.synchronize()
    assert torch.equal(seq.out, ref)
    L = M.MoELayer(w.T, w.E, w.k, w.R, w.S, w.d, w.F)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        L.forward(lg, x, *W)
    for _ in range(2):
        L.out.zero_()
        g.replay()
    torch.cuda.synchronize()
    assert int(L.err.item()) == 0
    assert torch.equal(L.out, ref)
    del g
