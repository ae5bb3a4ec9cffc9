"""The plain-C oracle (oracle/moe_ref.c) against the numpy oracle and the pins.

The two oracles are separate float64 implementations of the same definition
(the C one in index-order loops, the numpy one with BLAS matrix products), so
agreement to float64 rounding on routing, dispatch and the layer output is a
check of each against the other.  The C oracle is also pinned directly
against closed forms and brute force: E = 1, k = 1 equals a dense SwiGLU FFN;
k = E equals the full softmax mixture; the dispatch of random ids equals a
brute-force per-expert scan; a capacity of zero drops everything.
"""
import itertools
import math

import numpy as np
import pytest

import moe_workloads as mw
from oracle import moe_oracle as O
from oracle import ref_c as C

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

W = mw.Workload
CASES = {
    "tiny": mw.WORKLOADS["tiny"],
    "ragged_mixed_widths": W("ragged_mixed_widths", T=200, d_model=256, E=4, k=2,
                             expert_sizes=((1, 128), (1, 384), (1, 256), (1, 100))),
    "single_expert": W("single_expert", T=130, d_model=128, E=1, k=1, expert_sizes=((1, 256),)),
    "all_experts": W("all_experts", T=96, d_model=128, E=4, k=4, expert_sizes=((4, 128),)),
    "capacity_one": W("capacity_one", T=256, d_model=128, E=8, k=2, expert_sizes=((8, 128),),
                      capacity_factor=1.0 / 64, bias="zipf"),
    "switch_small": W("switch_small", T=300, d_model=128, E=16, k=1, expert_sizes=((16, 128),),
                      capacity_factor=1.25, bias="zipf"),
    "fine_small": W("fine_small", T=128, d_model=128, E=16, k=4, expert_sizes=((16, 128),), bias="normal"),
}


def _inputs(w):
    widths = O.expert_widths(w.expert_sizes)
    W1, W3, W2 = mw.gen_expert_weights(w, widths)
    b = mw.gen_router_bias(w)
    cf = float(np.float32(w.capacity_factor)) if w.capacity_factor else 0.0
    return mw.gen_x(w), mw.gen_gamma(w), mw.gen_router_weight(w), b, W1, W3, W2, widths, cf


@pytest.mark.parametrize("name", sorted(CASES))
@pytest.mark.parametrize("renormalize", [False, True])
def test_c_oracle_matches_numpy_oracle(name, renormalize):
    w = CASES[name]
    x, g, Wr, b, W1, W3, W2, widths, cf = _inputs(w)
    R = O.moe_layer(x, g, Wr, b, W1, W3, W2, widths, w.k, w.eps, capacity_factor=cf, renormalize=renormalize)
    Q = C.layer(x, g, Wr, b, W1, W3, W2, widths, w.k, w.eps, capacity_factor=cf, renormalize=renormalize)
    np.testing.assert_allclose(Q["r"], R["r"], rtol=1e-14, atol=0)
    # fp32 logits from fp64 sums in two summation orders: equal, or one fp32 ulp apart
    ulp = np.spacing(np.abs(R["logits"]).astype(np.float32))
    assert np.all(np.abs(Q["logits"].astype(np.float64) - R["logits"].astype(np.float64)) <= ulp)
    # these seeded inputs have no near-ties, so the routing agrees everywhere
    assert np.array_equal(Q["idx"], R["idx"])
    np.testing.assert_allclose(Q["gate"], R["gate"], rtol=1e-12, atol=1e-15)
    for key in ("counts", "offsets", "perm", "inv_perm"):
        assert np.array_equal(Q[key], R[key]), key
    scale = np.maximum(np.linalg.norm(R["out"], axis=1), 1e-30)
    rel = np.linalg.norm(Q["out"] - R["out"], axis=1) / scale
    assert rel.max() <= 1e-12, rel.max()


def test_c_oracle_replays_given_ids():
    w = CASES["ragged_mixed_widths"]
    x, g, Wr, b, W1, W3, W2, widths, cf = _inputs(w)
    ids = np.random.default_rng(5).integers(0, w.E, size=(w.T, w.k)).astype(np.int32)
    R = O.moe_layer(x, g, Wr, b, W1, W3, W2, widths, w.k, w.eps, idx_override=ids)
    Q = C.layer(x, g, Wr, b, W1, W3, W2, widths, w.k, w.eps, idx_override=ids)
    assert np.array_equal(Q["idx"], ids)
    for key in ("counts", "offsets", "perm", "inv_perm"):
        assert np.array_equal(Q[key], R[key]), key
    scale = np.maximum(np.linalg.norm(R["out"], axis=1), 1e-30)
    assert (np.linalg.norm(Q["out"] - R["out"], axis=1) / scale).max() <= 1e-12


def test_c_oracle_rejects_bad_ids():
    w = CASES["tiny"]
    x, g, Wr, b, W1, W3, W2, widths, cf = _inputs(w)
    ids = np.zeros((w.T, w.k), dtype=np.int32)
    ids[3, 1] = w.E
    with pytest.raises(ValueError):
        C.layer(x, g, Wr, b, W1, W3, W2, widths, w.k, w.eps, idx_override=ids)


def _rng_problem(T, d, E, k, widths, seed):
    rng = np.random.default_rng(seed)
    F_ = sum(widths)
    bits = lambda a: mw.f32_to_bf16_bits(np.asarray(a, dtype=np.float32))
    x = bits(rng.standard_normal((T, d)))
    g = bits(1 + 0.1 * rng.standard_normal(d))
    Wr = bits(rng.standard_normal((d, E)) / math.sqrt(d))
    W1 = bits(rng.standard_normal((d, F_)) / math.sqrt(d))
    W3 = bits(rng.standard_normal((d, F_)) / math.sqrt(d))
    W2 = bits(rng.standard_normal((F_, d)) / math.sqrt(F_ / E))
    return x, g, Wr, W1, W3, W2


def _swiglu_dense(x, g, W1, W3, W2, eps):
    """Textbook RMSNorm then SwiGLU, float64 (the E = 1, k = 1 closed form)."""
    xf, gf = O.widen_bf16(x), O.widen_bf16(g)
    xn = xf / np.sqrt(np.mean(xf * xf, axis=1, keepdims=True) + eps) * gf[None, :]
    u, v = xn @ O.widen_bf16(W1), xn @ O.widen_bf16(W3)
    return (u / (1 + np.exp(-u)) * v) @ O.widen_bf16(W2)


def test_c_oracle_single_expert_is_dense_swiglu():
    x, g, Wr, W1, W3, W2 = _rng_problem(40, 64, 1, 1, [128], 11)
    Q = C.layer(x, g, Wr, None, W1, W3, W2, [128], 1, 1e-5)
    ref = _swiglu_dense(x, g, W1, W3, W2, 1e-5)
    np.testing.assert_allclose(Q["gate"], 1.0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(Q["out"], ref, rtol=1e-10, atol=1e-12)


def test_c_oracle_all_experts_is_softmax_mixture():
    E, widths = 3, [128, 256, 128]
    x, g, Wr, W1, W3, W2 = _rng_problem(24, 64, E, E, widths, 12)
    Q = C.layer(x, g, Wr, None, W1, W3, W2, widths, E, 1e-5)
    offs = O.expert_offsets(widths)
    xf, gf = O.widen_bf16(x), O.widen_bf16(g)
    xn = xf / np.sqrt(np.mean(xf * xf, axis=1, keepdims=True) + 1e-5) * gf[None, :]
    logits = (xn @ O.widen_bf16(Wr)).astype(np.float32).astype(np.float64)
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ref = np.zeros_like(xf)
    for e in range(E):
        o0, o1 = offs[e], offs[e + 1]
        u, v = xn @ O.widen_bf16(W1[:, o0:o1]), xn @ O.widen_bf16(W3[:, o0:o1])
        ref += p[:, e:e + 1] * ((u / (1 + np.exp(-u)) * v) @ O.widen_bf16(W2[o0:o1]))
    np.testing.assert_allclose(Q["out"], ref, rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("cap", [0.0, 0.5, 1.0])
def test_c_oracle_dispatch_bruteforce(cap):
    T, E, k = 37, 5, 3
    x, g, Wr, W1, W3, W2 = _rng_problem(T, 64, E, k, [128] * E, 13)
    rng = np.random.default_rng(14)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    Q = C.layer(x, g, Wr, None, W1, W3, W2, [128] * E, k, 1e-5, capacity_factor=cap, idx_override=ids)
    Cap = math.floor(T * k / E * cap) if cap > 0 else T * k
    flat = ids.reshape(-1)
    pos, nxt = {}, 0
    for e in range(E):                       # expert-major, assignment order inside
        kept_e = [a for a in range(T * k) if flat[a] == e][:Cap]
        for a in kept_e:
            pos[a] = nxt
            nxt += 1
    for a in range(T * k):
        assert Q["inv_perm"][a] == pos.get(a, -1)
    assert Q["n_kept"] == nxt
    assert np.array_equal(Q["perm"], np.array(sorted(pos, key=pos.get), dtype=np.int64))
    assert np.array_equal(Q["counts"], np.bincount(flat, minlength=E))


def test_c_oracle_capacity_zero_drops_everything():
    T, E, k = 16, 4, 1
    x, g, Wr, W1, W3, W2 = _rng_problem(T, 64, E, k, [128] * E, 15)
    Q = C.layer(x, g, Wr, None, W1, W3, W2, [128] * E, k, 1e-5, capacity_factor=1e-3)
    assert Q["n_kept"] == 0 and np.all(Q["inv_perm"] == -1)
    assert np.all(Q["out"] == 0.0)


def test_c_oracle_topk_bruteforce():
    T, E, k = 30, 6, 3
    x, g, Wr, W1, W3, W2 = _rng_problem(T, 64, E, k, [128] * E, 16)
    Q = C.layer(x, g, Wr, None, W1, W3, W2, [128] * E, k, 1e-5)
    for t in range(T):
        lt = Q["logits"][t].astype(np.float64)
        best = max(itertools.combinations(range(E), k), key=lambda s: (sum(lt[list(s)]), [-i for i in s]))
        assert set(Q["idx"][t].tolist()) == set(best)
        assert all(lt[Q["idx"][t][j]] >= lt[Q["idx"][t][j + 1]] for j in range(k - 1))
