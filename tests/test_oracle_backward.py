"""Pins of the oracle's backward pass (CPU only).

The backward is the chain rule through the oracle's forward; it is checked against
  - central finite differences of the oracle's own forward, O.layer (fp64, tiny shapes,
    logits far from top-k ties so the selection is locally constant);
  - torch.autograd in fp64 through a token-major formulation that has no plan, no
    dispatch, no replica slots and no combine buffer (each token runs its k experts
    directly), so the row placement and the reduction of replica gradients back to the
    home experts are checked against a computation without them;
  - invariance of every gradient under the number of prefetch slots S (replicas).
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O


def tiny_case(seed, T=12, E=4, k=2, R=2, S=2, d=5, F=3, skew=2.5):
    rng = np.random.default_rng(seed)
    # well-separated logits (no near-ties), skewed towards expert 0 so that the plan
    # streams rows of the hot expert to the other rank as a replica
    logits = rng.permuted(np.tile(np.arange(E, dtype=np.float64) * 0.7, (T, 1)), axis=1)
    logits[:, 0] += skew
    logits = logits.astype(np.float32)
    x = rng.standard_normal((T, d))
    W1 = rng.standard_normal((E, F, d)) / np.sqrt(d)
    W3 = rng.standard_normal((E, F, d)) / np.sqrt(d)
    W2 = rng.standard_normal((E, d, F)) / np.sqrt(F)
    dout = rng.standard_normal((T, d))
    return dict(logits=logits, x=x, W1=W1, W3=W3, W2=W2, dout=dout, k=k, R=R, S=S, E=E)


def loss(c, x=None, W1=None, W3=None, W2=None):
    f = O.layer(c["logits"], c["x"] if x is None else x, c["W1"] if W1 is None else W1,
                c["W3"] if W3 is None else W3, c["W2"] if W2 is None else W2,
                c["k"], c["R"], c["S"])
    assert f["err"] == 0
    return float((f["out"] * c["dout"]).sum()), f


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_backward_matches_finite_differences(seed):
    c = tiny_case(seed)
    _, f = loss(c)
    n_rep = sum(1 for e in f["plan"]["replica_expert"] if e >= 0)
    assert n_rep >= 1, "the case must exercise a replica slot"
    b = O.layer_backward(f, c["dout"], c["W1"], c["W3"], c["W2"], c["E"])
    rng = np.random.default_rng(100 + seed)
    eps = 1e-6
    for name, grad in (("x", b["dx"]), ("W1", b["dW1"]), ("W3", b["dW3"]), ("W2", b["dW2"])):
        base = c[name]
        for _ in range(12):
            i = tuple(int(rng.integers(0, n)) for n in base.shape)
            p = base.copy()
            m = base.copy()
            p[i] += eps
            m[i] -= eps
            num = (loss(c, **{name: p})[0] - loss(c, **{name: m})[0]) / (2 * eps)
            assert abs(num - grad[i]) <= 1e-6 * max(1.0, abs(num)), (name, i, num, grad[i])


def token_major_autograd(c):
    """Each token through its k chosen experts directly (no plan, no rows, no pool)."""
    f = O.layer(c["logits"], c["x"], c["W1"], c["W3"], c["W2"], c["k"], c["R"], c["S"])
    idx = torch.from_numpy(np.asarray(f["idx"]).astype(np.int64))
    lg = torch.tensor(np.asarray(c["logits"], dtype=np.float64), requires_grad=True)
    x = torch.tensor(c["x"], requires_grad=True)
    W1 = torch.tensor(c["W1"], requires_grad=True)
    W3 = torch.tensor(c["W3"], requires_grad=True)
    W2 = torch.tensor(c["W2"], requires_grad=True)
    chosen = torch.gather(lg, 1, idx)
    gate = torch.softmax(chosen, dim=1)
    T, k = idx.shape
    outs = []
    for t in range(T):
        acc = 0
        for j in range(k):
            e = int(idx[t, j])
            g = W1[e] @ x[t]
            u = W3[e] @ x[t]
            h = torch.nn.functional.silu(g) * u
            acc = acc + gate[t, j] * (W2[e] @ h)
        outs.append(acc)
    out = torch.stack(outs)
    (out * torch.from_numpy(c["dout"])).sum().backward()
    return f, dict(dx=x.grad.numpy(), dlogits=lg.grad.numpy(), dW1=W1.grad.numpy(),
                   dW3=W3.grad.numpy(), dW2=W2.grad.numpy(), out=out.detach().numpy())


@pytest.mark.parametrize("seed", [3, 4])
def test_backward_matches_token_major_autograd(seed):
    c = tiny_case(seed, T=16, E=6, k=3, R=3, S=2, d=6, F=4, skew=3.0)
    f, ref = token_major_autograd(c)
    assert np.allclose(f["out"], ref["out"], rtol=1e-12, atol=1e-12)
    b = O.layer_backward(f, c["dout"], c["W1"], c["W3"], c["W2"], c["E"])
    for key in ("dx", "dlogits", "dW1", "dW3", "dW2"):
        assert np.allclose(b[key], ref[key], rtol=1e-10, atol=1e-12), key


def test_weight_gradients_do_not_depend_on_replicas():
    """More slots move rows to replica copies; the gradients reduced home are the same."""
    grads = []
    for S in (1, 2, 4):
        c = tiny_case(7, T=24, E=4, k=2, R=4, S=S, d=5, F=3, skew=4.0)
        _, f = loss(c)
        b = O.layer_backward(f, c["dout"], c["W1"], c["W3"], c["W2"], c["E"])
        grads.append((sum(1 for e in f["plan"]["replica_expert"] if e >= 0), b))
    assert grads[0][0] >= 1
    for _, b in grads[1:]:
        for key in ("dx", "dlogits", "dW1", "dW3", "dW2"):
            assert np.allclose(b[key], grads[0][1][key], rtol=1e-12, atol=1e-12), key


def test_silu_grad_closed_forms():
    assert O.silu_grad(np.array([0.0]))[0] == 0.5
    z = np.linspace(-6, 6, 25)
    h = 1e-6
    num = (O.silu(z + h) - O.silu(z - h)) / (2 * h)
    assert np.allclose(O.silu_grad(z), num, rtol=1e-8, atol=1e-10)


def test_gate_backward_closed_form_k2():
    """k = 2: gate_0 = sigmoid(l0 - l1), so dL/dl0 = -dL/dl1 = g0 g1 (dg0 - dg1)."""
    gate = np.array([[0.3, 0.7]])
    dgate = np.array([[1.5, -0.5]])
    dl = O.topk_backward(gate, dgate, np.array([[2, 0]]), 3)
    v = 0.3 * 0.7 * (1.5 - (-0.5))
    assert np.allclose(dl, [[-v, 0.0, v]])


# ----------------------------------------------------------------- per-piece adjoint pins
# Each linear piece of the layer is pinned by the dot-product (adjoint) identity
# <A v, w> = <v, A^T w> with random v and w, which holds for the true transpose and fails
# for a dropped term, a wrong index or a transposed operand in either the forward or the
# backward; the nonlinear gate softmax is pinned by central differences.

def random_placement(rng, T, k, rows):
    """A bijection of the T*k assignments onto `rows` rows (perm) and its inverse (src)."""
    order = rng.permutation(rows)[: T * k]
    perm = order.reshape(T, k)
    src = np.full(rows, -1)
    for t in range(T):
        for j in range(k):
            src[perm[t, j]] = t
    return perm, src


def test_dispatch_backward_is_the_adjoint_of_dispatch():
    rng = np.random.default_rng(11)
    T, k, d = 9, 3, 5
    perm, src = random_placement(rng, T, k, T * k)
    x = rng.standard_normal((T, d))
    g = rng.standard_normal((T * k, d))
    lhs = float((O.dispatch(x, src) * g).sum())
    rhs = float((x * O.dispatch_backward(g, perm)).sum())
    assert abs(lhs - rhs) <= 1e-12 * max(1.0, abs(lhs))


def test_combine_backward_is_the_adjoint_in_rows_and_in_gates():
    rng = np.random.default_rng(12)
    T, k, d = 7, 4, 6
    perm, _ = random_placement(rng, T, k, T * k)
    y = rng.standard_normal((T * k, d))
    gate = rng.random((T, k))
    dout = rng.standard_normal((T, d))
    dy, dgate = O.combine_backward(dout, y, perm, gate)
    out = O.combine(y, perm, gate)
    # combine is linear in y for fixed gates, and linear in the gates for fixed y
    ip = float((out * dout).sum())
    assert abs(ip - float((y * dy).sum())) <= 1e-12 * max(1.0, abs(ip))
    assert abs(ip - float((gate * dgate).sum())) <= 1e-12 * max(1.0, abs(ip))


def test_topk_backward_matches_central_differences_of_the_gates():
    """Gates as a function of the chosen logits (selection held fixed by well-separated
    logits): <d gate, dgate> / eps against <v, dlogits> for random directions v.  The router
    computes on fp32 logits, so the logits sit on a 2^-8 grid below 8 in magnitude and move
    by 2^-16 along directions in {-1, 0, 1}: every perturbed logit is exact in fp32."""
    rng = np.random.default_rng(13)
    T, E, k = 5, 10, 3
    logits = rng.permuted(np.tile(np.arange(E, dtype=np.float64) * 0.7 - 3.0, (T, 1)), axis=1)
    logits = np.round(logits * 256) / 256
    idx, gate, err = O.topk_route(logits, k)
    assert err == 0
    dgate = rng.standard_normal((T, k))
    dl = O.topk_backward(gate, dgate, idx, E)
    eps = 2.0 ** -16
    for _ in range(4):
        v = rng.integers(-1, 2, size=(T, E)).astype(np.float64)
        assert np.array_equal((logits + eps * v).astype(np.float32), logits + eps * v)
        gp = O.topk_route(logits + eps * v, k)
        gm = O.topk_route(logits - eps * v, k)
        assert np.array_equal(gp[0], idx) and np.array_equal(gm[0], idx)
        num = float(((gp[1] - gm[1]) * dgate).sum()) / (2 * eps)
        assert abs(num - float((v * dl).sum())) <= 1e-7 * max(1.0, abs(num))


def test_expert_ffn_backward_matches_central_differences():
    rng = np.random.default_rng(14)
    n, d, F = 6, 5, 4
    X = rng.standard_normal((n, d))
    w1 = rng.standard_normal((F, d)) / np.sqrt(d)
    w3 = rng.standard_normal((F, d)) / np.sqrt(d)
    w2 = rng.standard_normal((d, F)) / np.sqrt(F)
    dy = rng.standard_normal((n, d))
    b = O.expert_ffn_backward(X, w1, w3, w2, dy)
    args = dict(X=X, w1=w1, w3=w3, w2=w2)
    grads = dict(X=b["dX"], w1=b["dw1"], w3=b["dw3"], w2=b["dw2"])

    def f(**kw):
        a = dict(args, **kw)
        return float((O.expert_ffn(a["X"], a["w1"], a["w3"], a["w2"]) * dy).sum())

    eps = 1e-6
    for name, grad in grads.items():
        v = rng.standard_normal(args[name].shape)
        num = (f(**{name: args[name] + eps * v}) - f(**{name: args[name] - eps * v})) / (2 * eps)
        assert abs(num - float((v * grad).sum())) <= 1e-7 * max(1.0, abs(num)), name
