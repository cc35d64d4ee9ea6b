"""Grouped FFN at the group sizes where its tiling changes (needs a B200).

A group's last 128-row tile with at most 64 valid rows runs M = 64 tensor-core MMAs (a
64-row operand box, the accumulator's rows 16 per TMEM lane quadrant); every other tile
runs M = 128.  Uniform groups of cap rows (the fixed-capacity layout) put each size on
every expert: 1, 63, 64, 65, 127, 128, 129, 191, 192 rows.  Every element of h and y is
checked against the fp64 oracle within 1e-2 * max(1, |oracle|).
"""
import numpy as np
import pytest
import torch

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build
from oracle import moe_oracle as O

from harness import assert_close_scaled, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    M.lib()


@pytest.mark.parametrize("cap", [1, 63, 64, 65, 127, 128, 129, 191, 192])
@pytest.mark.parametrize("d,F", [(256, 256), (384, 128)])
def test_ffn_tile_edges(cap, d, F):
    E = 5
    g = torch.Generator().manual_seed(cap * 7 + d)
    rows = E * cap
    recv = torch.randn(rows, d, generator=g).to(torch.bfloat16).cuda()
    W1 = (torch.randn(E, F, d, generator=g) / d ** 0.5).to(torch.bfloat16).cuda()
    W3 = (torch.randn(E, F, d, generator=g) / d ** 0.5).to(torch.bfloat16).cuda()
    W2 = (torch.randn(E, d, F, generator=g) / d ** 0.5).to(torch.bfloat16).to(torch.float16).cuda()
    h = torch.full((rows, F), float("nan"), dtype=torch.float16, device="cuda")
    y = torch.full((rows, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_grouped_ffn_capacity(recv, W1, W3, W2, cap, h, y, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    X = to64(recv)
    h_ref = np.zeros((rows, F))
    y_ref = np.zeros((rows, d))
    for e in range(E):
        w1, w3, w2 = to64(W1[e]), to64(W3[e]), to64(W2[e])
        Xe = X[e * cap:(e + 1) * cap]
        h_ref[e * cap:(e + 1) * cap] = O.silu(Xe @ w1.T) * (Xe @ w3.T)
        y_ref[e * cap:(e + 1) * cap] = O.expert_ffn(Xe, w1, w3, w2)
    assert_close_scaled(to64(h), h_ref, f"h, cap {cap}")
    assert_close_scaled(to64(y), y_ref, f"y, cap {cap}")
