"""moe_route_plan (needs a B200): routing, histogram and plan fused into one launch.

Every output must equal the three separate calls' (moe_topk or moe_topk_biased, then
moe_histogram_maxvio with the home map, then moe_plan_balanced) bit for bit, on the same
inputs, from the same pre-filled buffers -- including the error paths, where the fields
the separate calls leave untouched must stay untouched.  The layer's forward runs this
call, so every layer test also checks it against the oracle.
"""
import pytest
import torch

import load_balanced_dispatch_warp_b200 as M
from load_balanced_dispatch_warp_b200 import build
from load_balanced_dispatch_warp_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build.build()
    M.lib()


SENTINEL = dict(idx=-7, gate=-3.0, counts=11, loads=13, maxvio=-1.5, bal=-2.5, plan=17, err=99)


def buffers(T, E, k, R, S):
    """Output buffers pre-filled with sentinels (fields a call leaves untouched keep them)."""
    lay = M.plan_layout(E, R, S)
    i32, f32, f64 = torch.int32, torch.float32, torch.float64
    shapes = dict(idx=((T, k), i32), gate=((T, k), f32), counts=((E,), i32), loads=((R,), i32),
                  maxvio=((1,), f64), bal=((1,), f64), plan=((lay.words,), i32), err=((1,), i32))
    return {key: torch.full(shp, SENTINEL[key], dtype=dt, device="cuda")
            for key, (shp, dt) in shapes.items()}


def refill(b):
    for key in SENTINEL:
        b[key].fill_(SENTINEL[key])


def run_separate(logits, k, R, S, b, bias=None):
    T, E = logits.shape
    if bias is None:
        M.moe_topk(logits, k, b["idx"], b["gate"], b["err"])
    else:
        M.moe_topk_biased(logits, bias, k, b["idx"], b["gate"], b["err"])
    M.moe_histogram_maxvio(b["idx"], E, R, b["counts"], b["loads"], b["maxvio"], b["bal"], b["err"])
    M.moe_plan_balanced(b["counts"], T, k, R, S, b["plan"], b["err"])


def run_fused(logits, k, R, S, b, bias=None):
    E = logits.shape[1]
    if "_ws" not in b:  # scratch, not an output: any contents
        b["_ws"] = torch.full((M.route_plan_workspace_words(E),), 123, dtype=torch.int32,
                              device="cuda")
    M.moe_route_plan(logits, k, R, S, b["idx"], b["gate"], b["counts"], b["loads"], b["maxvio"],
                     b["bal"], b["plan"], b["_ws"], b["err"], bias=bias)


def assert_same(a, b):
    torch.cuda.synchronize()
    for key in SENTINEL:
        assert torch.equal(a[key], b[key]), key


def compare(logits, k, R, S, bias=None):
    T, E = logits.shape
    a, b = buffers(T, E, k, R, S), buffers(T, E, k, R, S)
    run_separate(logits, k, R, S, a, bias)
    run_fused(logits, k, R, S, b, bias)
    assert_same(a, b)
    return b


@pytest.mark.parametrize("name", ["tiny", "near_balanced", "qwen_mv1", "mixtral", "deepseek"])
def test_route_plan_equals_separate_calls(name):
    w = I.WORKLOADS[name]
    logits = I.make_logits(w).cuda()
    b = compare(logits, w.k, w.R, w.S)
    assert int(b["err"].item()) == 0
    assert int(b["counts"].sum().item()) == w.T * w.k


@pytest.mark.parametrize("T,E,k,R,S", [(1000, 64, 6, 8, 8), (96, 32, 1, 8, 2), (200, 512, 8, 16, 12),
                                       (333, 128, 3, 1, 0), (64, 16, 4, 1, 0),
                                       (1024, 1024, 32, 1024, 3), (40, 8, 8, 4, 2)])
def test_route_plan_shapes(T, E, k, R, S):
    if (T * k) % R:
        pytest.skip("T*k must divide by R")
    g = torch.Generator().manual_seed(T + E + k)
    logits = (torch.randn(T, E, generator=g) - 0.3 * torch.log(torch.arange(1, E + 1.0))).cuda()
    compare(logits, k, R, S)


def test_route_plan_ties_take_the_exact_path():
    """Logits on a coarse grid: many equal keys, so most warps take the ordered fallback."""
    g = torch.Generator().manual_seed(3)
    logits = torch.randint(-3, 4, (2048, 64), generator=g).float().cuda()
    compare(logits, 6, 8, 8)


def test_route_plan_biased():
    w = I.WORKLOADS["deepseek"]
    logits = I.make_logits(w).cuda()
    g = torch.Generator().manual_seed(8)
    bias = (0.1 * torch.randn(w.E, generator=g)).cuda()
    compare(logits, w.k, w.R, w.S, bias=bias)


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), float("-inf")])
def test_route_plan_nonfinite_leaves_what_the_separate_calls_leave(bad):
    w = I.WORKLOADS["near_balanced"]
    logits = I.make_logits(w).cuda()
    logits[1234, 17] = bad
    b = compare(logits, w.k, w.R, w.S)
    assert int(b["err"].item()) == M.DERR_NONFINITE
    assert int(b["counts"].abs().sum().item()) == 0
    assert int(b["loads"][0].item()) == 0 and bool((b["loads"][1:] == 13).all())
    assert float(b["maxvio"].item()) == -1.5 and bool((b["plan"] == 17).all())


def test_route_plan_slot_overflow():
    # all tokens on experts 0..3 (rank 0) and no prefetch slots: replicas are needed
    w = I.small_workload("noslots", 64, 16, 4, 4, 0, 128, 128, alpha=200.0, seed=10)
    logits = I.make_logits(w).cuda()
    b = compare(logits, w.k, w.R, w.S)
    assert int(b["err"].item()) == M.DERR_SLOTS


def test_route_plan_empty_batch():
    logits = torch.empty(0, 8, device="cuda")
    b = compare(logits, 2, 4, 2)
    assert int(b["err"].item()) == 0
    assert int(b["counts"].abs().sum().item()) == 0
    assert float(b["maxvio"].item()) == 0.0 and float(b["bal"].item()) == 1.0


def test_route_plan_repeated_calls_and_graph():
    """The ticket and the counts start from the launcher's memsets every call: repeated
    calls, and replays of a captured call, give the same outputs."""
    w = I.WORKLOADS["qwen_mv1"]
    logits = I.make_logits(w).cuda()
    ref = buffers(w.T, w.E, w.k, w.R, w.S)
    run_separate(logits, w.k, w.R, w.S, ref)
    b = buffers(w.T, w.E, w.k, w.R, w.S)
    for _ in range(3):
        run_fused(logits, w.k, w.R, w.S, b)
    assert_same(ref, b)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run_fused(logits, w.k, w.R, w.S, b)
    torch.cuda.synchronize()
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr, stream=s):
        run_fused(logits, w.k, w.R, w.S, b)
    refill(b)
    for _ in range(2):
        gr.replay()
    assert_same(ref, b)
    del gr
