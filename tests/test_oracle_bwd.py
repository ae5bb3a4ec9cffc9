"""Pins of the backward oracle against things other than itself:

* central finite differences of L = <g, out> (the definition of a gradient)
  along random directions and per entry, with the routing held fixed and
  checked to be locally constant;
* E = 1, k = 1 reduces the layer to a textbook RMSNorm + dense SwiGLU FFN
  with gate 1, differentiated by torch autograd in float64; the router then
  gets exactly zero gradient;
* softmax-backward rows sum to zero, so the bias gradient does too;
* planted mistakes in each piece of the chain rule fail the finite-difference
  check.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O
from oracle import moe_oracle_bwd as B

CASES = {
    # name: (T, d, E, k, widths, capacity_factor, renormalize)
    "dropless": (7, 6, 4, 2, [3, 5, 4, 2], 0.0, False),
    "capacity_renorm": (9, 5, 3, 2, [4, 2, 3], 0.5, True),
    "k_eq_E": (4, 6, 3, 3, [2, 3, 4], 0.0, False),
    "top1_capacity": (8, 4, 4, 1, [3, 3, 2, 5], 1.0, False),
}
PARAMS = ("x", "gamma", "Wr", "bias", "W1", "W3", "W2")
EPS = 1e-5


def make(name, seed=0):
    T, d, E, k, widths, cf, renorm = CASES[name]
    rng = np.random.default_rng(seed)
    F = sum(widths)
    P = {"x": rng.standard_normal((T, d)),
         "gamma": 1.0 + 0.3 * rng.standard_normal(d),
         "Wr": rng.standard_normal((d, E)),
         "bias": 0.5 * rng.standard_normal(E),
         "W1": rng.standard_normal((d, F)) / np.sqrt(d),
         "W3": rng.standard_normal((d, F)) / np.sqrt(d),
         "W2": rng.standard_normal((F, d)) / np.sqrt(F)}
    g = rng.standard_normal((T, d))
    return P, g, dict(widths=widths, k=k, eps=EPS, capacity_factor=cf, renormalize=renorm)


def fwd(P, kw, idx=None):
    return B.layer_forward(P["x"], P["gamma"], P["Wr"], P["bias"], P["W1"], P["W3"],
                           P["W2"], idx=idx, **kw)


def fd_check(P, g, kw, grads, rng, h=1e-5, rtol=1e-7):
    """Directional central differences for every parameter; returns the worst
    relative error.  Routing is replayed at the perturbed points (the function
    is then smooth) and the free routing is checked to stay the same there."""
    base = fwd(P, kw)
    idx = base["idx"]
    worst = 0.0
    for name in PARAMS:
        V = rng.standard_normal(P[name].shape)
        Pp = dict(P, **{name: P[name] + h * V})
        Pm = dict(P, **{name: P[name] - h * V})
        for Q in (Pp, Pm):
            assert np.array_equal(fwd(Q, kw)["idx"], idx), "routing not locally constant"
        fd = (B.loss(fwd(Pp, kw, idx), g) - B.loss(fwd(Pm, kw, idx), g)) / (2 * h)
        an = float((grads["d" + name] * V).sum())
        err = abs(fd - an) / max(abs(fd), 1e-3)
        worst = max(worst, err)
    return worst


@pytest.mark.parametrize("name", sorted(CASES))
def test_gradients_match_finite_differences(name):
    P, g, kw = make(name)
    grads = B.layer_backward(fwd(P, kw), g)
    assert fd_check(P, g, kw, grads, np.random.default_rng(1)) < 1e-7


@pytest.mark.parametrize("name", ["capacity_renorm", "dropless"])
def test_small_gradients_entrywise(name):
    """Every entry of dgamma and dbias, and a few of dx, by central differences."""
    P, g, kw = make(name)
    f = fwd(P, kw)
    grads = B.layer_backward(f, g)
    h = 1e-6
    probes = [("gamma", (i,)) for i in range(P["gamma"].size)]
    probes += [("bias", (e,)) for e in range(P["bias"].size)]
    probes += [("x", (t, 1)) for t in range(P["x"].shape[0])]
    for name_, at in probes:
        Pp = {kk: v.copy() for kk, v in P.items()}
        Pm = {kk: v.copy() for kk, v in P.items()}
        Pp[name_][at] += h
        Pm[name_][at] -= h
        fd = (B.loss(fwd(Pp, kw, f["idx"]), g) - B.loss(fwd(Pm, kw, f["idx"]), g)) / (2 * h)
        assert abs(fd - grads["d" + name_][at]) <= 1e-7 * max(1.0, abs(fd)), (name_, at)


def test_single_expert_equals_textbook_rmsnorm_swiglu_autograd():
    """E = 1, k = 1: gate = softmax over one logit = 1, so the layer is
    RMSNorm(x) * gamma followed by a dense SwiGLU FFN.  torch autograd of that
    textbook form (norm before the GEMM, not the statistic after it) gives
    the same gradients; the router gets exactly zero."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(3)
    T, d, f = 6, 8, 5
    P = {"x": rng.standard_normal((T, d)), "gamma": 1 + 0.2 * rng.standard_normal(d),
         "Wr": rng.standard_normal((d, 1)), "bias": np.array([0.3]),
         "W1": rng.standard_normal((d, f)), "W3": rng.standard_normal((d, f)),
         "W2": rng.standard_normal((f, d))}
    g = rng.standard_normal((T, d))
    kw = dict(widths=[f], k=1, eps=EPS, capacity_factor=0.0, renormalize=False)
    grads = B.layer_backward(fwd(P, kw), g)
    tt = {kk: torch.tensor(P[kk], dtype=torch.float64, requires_grad=True)
          for kk in ("x", "gamma", "W1", "W3", "W2")}
    x = tt["x"]
    n = x * torch.rsqrt((x * x).mean(dim=1, keepdim=True) + EPS) * tt["gamma"]
    out = (torch.nn.functional.silu(n @ tt["W1"]) * (n @ tt["W3"])) @ tt["W2"]
    (out * torch.tensor(g)).sum().backward()
    for kk in tt:
        np.testing.assert_allclose(grads["d" + kk], tt[kk].grad.numpy(), rtol=1e-10, atol=1e-12)
    assert np.all(grads["dWr"] == 0) and np.all(grads["dbias"] == 0)


@pytest.mark.parametrize("name", sorted(CASES))
def test_logit_gradient_rows_sum_to_zero(name):
    P, g, kw = make(name)
    grads = B.layer_backward(fwd(P, kw), g)
    np.testing.assert_allclose(grads["dl"].sum(axis=1), 0.0, atol=1e-13)
    assert abs(grads["dbias"].sum()) < 1e-12


def test_dropped_slots_get_no_gate_gradient():
    P, g, kw = make("capacity_renorm")
    f = fwd(P, kw)
    grads = B.layer_backward(f, g)
    dropped = ~f["kept"].reshape(grads["dgate"].shape)
    assert dropped.any()
    assert np.all(grads["dgate"][dropped] == 0)


def _sig(u):
    return 1.0 / (1.0 + np.exp(-u))


MUTANTS = {
    "silu_grad without the u(1-sigma) term": ("silu_grad", lambda u: _sig(u)),
    "softmax backward without <dp,p>": ("softmax_backward", lambda p, dp: p * dp),
    "rms backward with the wrong sign": (
        "rms_backward", lambda x, r, dr: -((dr * -(r ** 3) / x.shape[1])[:, None] * x)),
    "renormalised gates treated as plain": ("gate_backward", lambda dg, q, rn: dg.copy()),
    "router drops its dr term": (
        "router_backward",
        lambda dl, xg, z, r, Wr: (dl.sum(0), xg.T @ (r[:, None] * dl), (r[:, None] * dl) @ Wr.T,
                                  np.zeros(len(r)))),
    "router forgets r on its input gradient": (
        "router_backward",
        lambda dl, xg, z, r, Wr: (dl.sum(0), xg.T @ (r[:, None] * dl), dl @ Wr.T,
                                  (dl * z).sum(1))),
    "swiglu gradients swapped": (
        "swiglu_backward", lambda dh, u, v: (dh * O.silu(u), dh * v * B.silu_grad(u))),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistakes_fail_the_finite_difference_pin(mutant, monkeypatch):
    attr, bad = MUTANTS[mutant]
    monkeypatch.setattr(B, attr, bad)
    worst = 0.0
    for name in ("capacity_renorm", "dropless"):
        P, g, kw = make(name)
        grads = B.layer_backward(fwd(P, kw), g)
        worst = max(worst, fd_check(P, g, kw, grads, np.random.default_rng(1)))
    assert worst > 1e-4, mutant


def test_float64_forward_matches_the_pinned_forward():
    """The forward the backward differentiates is the forward oracle's layer
    (which rounds the logits to fp32 once; the routing is replayed so both
    sides take the same experts)."""
    import moe_workloads as mw
    w = mw.WORKLOADS["tiny"]
    x, gamma = mw.gen_x(w), mw.gen_gamma(w)
    Wr, bias = mw.gen_router_weight(w), mw.gen_router_bias(w)
    widths = O.expert_widths(w.expert_sizes)
    W1, W3, W2 = mw.gen_expert_weights(w, widths)
    ref = O.moe_layer(x, gamma, Wr, bias, W1, W3, W2, widths, w.k, w.eps, 0.0)
    f = B.layer_forward(O.widen_bf16(x), O.widen_bf16(gamma), O.widen_bf16(Wr), bias,
                        O.widen_bf16(W1), O.widen_bf16(W3), O.widen_bf16(W2), widths, w.k,
                        w.eps, idx=ref["idx"])
    np.testing.assert_allclose(f["out"], ref["out"], rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(f["r"], ref["r"], rtol=1e-15)
