"""Router variants on the GPU against the oracle (needs a B200): bias-only selection and
the fixed-capacity ledger (including the pages' 16-token fixture)."""
import json
import os

import numpy as np
import pytest
import torch

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build
from load_balanced_dispatch_warp_b200 import inputs as I
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()


def _biased_gpu(logits, bias, k):
    T, E = logits.shape
    idx = torch.empty(T, k, dtype=torch.int32, device="cuda")
    gate = torch.empty(T, k, dtype=torch.float32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_topk_biased(logits.cuda(), bias.cuda(), k, idx, gate, err)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), gate.cpu().double().numpy(), int(err.item())


@pytest.mark.parametrize("T,E,k,seed", [(300, 8, 2, 0), (1000, 64, 6, 1), (4096, 256, 8, 2), (77, 700, 5, 3)])
def test_biased_topk_parity(T, E, k, seed):
    g = torch.Generator().manual_seed(seed)
    logits = torch.randn(T, E, generator=g)
    bias = torch.randn(E, generator=g) * 0.7
    idx, gate, err = _biased_gpu(logits, bias, k)
    ri, rg, rerr = O.topk_route_biased(logits.numpy(), bias.numpy(), k)
    assert err == rerr == 0
    assert np.array_equal(idx, ri)
    assert np.abs(gate - rg).max() <= 1e-6


def test_biased_topk_ties_in_fp32_sum():
    # logit + 100 rounds many distinct logits to one fp32 value: ties go to the lower id
    g = torch.Generator().manual_seed(5)
    logits = (torch.randn(512, 32, generator=g) * 1e-6).contiguous()
    bias = torch.full((32,), 100.0)
    idx, gate, err = _biased_gpu(logits, bias, 4)
    ri, rg, _ = O.topk_route_biased(logits.numpy(), bias.numpy(), 4)
    assert err == 0 and np.array_equal(idx, ri)
    assert np.abs(gate - rg).max() <= 1e-6


def test_biased_topk_balances_the_hot_workload():
    """A bias against the hot experts lowers maxvio on the DeepSeek-shaped logits."""
    w = I.WORKLOADS["deepseek"]
    logits = I.make_logits(w)
    hot = I.hot_experts(w)
    bias = torch.zeros(w.E)
    bias[hot] = -I.bias_param(w)  # cancel the hotspot's logit offset
    idx0 = torch.from_numpy(O.topk_route(logits.numpy(), w.k)[0])
    idx1, _, err = _biased_gpu(logits, bias, w.k)
    assert err == 0
    mv0 = O.expert_histogram(idx0.numpy(), w.E, w.R)["maxvio"]
    mv1 = O.expert_histogram(idx1, w.E, w.R)["maxvio"]
    assert mv1 < 0.5 * mv0


def _ledger_gpu(counts, T, k, num, den):
    E = len(counts)
    c = torch.tensor(counts, dtype=torch.int32, device="cuda")
    p, o, d = (torch.empty(E, dtype=torch.int32, device="cuda") for _ in range(3))
    tot = torch.empty(4, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_capacity_ledger(c, T, k, num, den, p, o, d, tot, err)
    torch.cuda.synchronize()
    return p.tolist(), o.tolist(), d.tolist(), tot.tolist()


def test_capacity_ledger_fixture():
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hotspot_fixture.json")))
    num, den = g["capacity_factor_num_den"]
    p, o, d, tot = _ledger_gpu(g["expert_demand"], g["tokens"], g["top_k"], num, den)
    assert tot == [g["capacity"], g["processed_sum"], g["overflow_sum"], g["padding_sum"]]
    assert p == g["processed"] and o == g["overflow"] and d == g["padding"]


@pytest.mark.parametrize("name", ["near_balanced", "deepseek", "mixtral"])
def test_capacity_ledger_parity(name):
    w = I.WORKLOADS[name]
    idx, _, _ = O.topk_route(I.make_logits(w).numpy(), w.k)
    counts = O.expert_histogram(idx, w.E, w.R)["counts"]
    for num, den in ((5, 4), (1, 1), (2, 1)):
        led = O.capacity_ledger(counts, w.A, w.E, num, den)
        p, o, d, tot = _ledger_gpu(counts.tolist(), w.T, w.k, num, den)
        assert tot == [led["cap"], int(led["processed"].sum()), int(led["overflow"].sum()), int(led["padding"].sum())]
        assert p == led["processed"].tolist() and o == led["overflow"].tolist() and d == led["padding"].tolist()


def test_w2_to_f16_matches_the_rounding_of_torch():
    """bf16 -> fp16 of the down projection: every value equal to torch's conversion (round to
    nearest even through fp32), including values that become fp16 subnormals or zeros, and
    the synthetic W2 of the workloads (bf16-rounded N(0, 1/d) values)."""
    g = torch.Generator().manual_seed(3)
    v = torch.randn(1 << 16, generator=g) * torch.exp2(torch.randint(-30, 10, (1 << 16,), generator=g).float())
    w = torch.cat([v, torch.tensor([0.0, -0.0, 65504.0, -65504.0, 2.0 ** -24, 2.0 ** -25, 1e5])])
    w = torch.cat([w, torch.zeros((-w.numel()) % 8)]).to(torch.bfloat16).cuda()
    out = M.w2_to_f16(w)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), w.float().to(torch.float16).view(torch.int16))
    wl = I.small_workload("w2conv", 64, 8, 2, 4, 2, 256, 384)
    W2 = I.make_weights(wl, device="cuda")[2]  # the fp16 images of bf16 values
    back = M.w2_to_f16(W2.to(torch.bfloat16))
    assert torch.equal(back, W2)
