"""Pins of the CPU oracle against what the sources and the mathematics fix.

None of these tests compares the oracle with itself: each one checks it
against a printed value (tests/golden), a closed form, a library routine that
computes the same quantity another way (torch's rms_norm / silu / softmax,
Python's sorted(), itertools subsets), or an invariant.  The mutation tests at
the end plant plausible mistakes in the oracle (on the CPU) and check that a
pin catches each one.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import moe_workloads as mw
from oracle import moe_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _small_problem(T=40, d=64, E=4, k=2, widths=None, bias=True, seed=3):
    rng = np.random.default_rng(seed)
    widths = widths or [128] * E
    F_ = sum(widths)
    x = mw.f32_to_bf16_bits(rng.standard_normal((T, d)).astype(np.float32))
    gamma = mw.f32_to_bf16_bits((1 + 0.1 * rng.standard_normal(d)).astype(np.float32))
    Wr = mw.f32_to_bf16_bits((rng.standard_normal((d, E)) / math.sqrt(d)).astype(np.float32))
    b = (0.3 * rng.standard_normal(E)).astype(np.float32) if bias else None
    W1 = mw.f32_to_bf16_bits((rng.standard_normal((d, F_)) / math.sqrt(d)).astype(np.float32))
    W3 = mw.f32_to_bf16_bits((rng.standard_normal((d, F_)) / math.sqrt(d)).astype(np.float32))
    W2 = np.concatenate([
        mw.f32_to_bf16_bits((rng.standard_normal((f, d)) / math.sqrt(f)).astype(np.float32))
        for f in widths], axis=0)
    return x, gamma, Wr, b, W1, W3, W2, widths


def _t(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


# ---------------------------------------------------------------- widths
def test_widths_and_offsets_printed_example(golden_dir):
    g = _load(golden_dir, "nanomoe_variable_experts.json")
    sizes = [tuple(p) for p in g["expert_sizes"]]
    widths = O.expert_widths(sizes, g["block_size"])
    offs = O.expert_offsets(widths)
    assert widths == g["expert_widths"]
    assert offs == g["expert_offsets"]
    assert offs[-1] == g["total_expert_width"]
    assert [g["n_embd"], offs[-1]] == g["w1_shape"]
    assert [offs[-1], g["n_embd"]] == g["w2_shape"]
    blocks = [w // g["block_size"] for w in widths]
    block_offs = [o // g["block_size"] for o in offs]
    assert blocks[:3] == g["expert_size_blocks_prefix"]
    assert block_offs[:3] == g["expert_block_offsets_prefix"]
    assert [offs[1], offs[2]] == g["expert1_w1_columns"]


def test_widths_round_up_to_block():
    assert O.expert_widths([(2, 100), (1, 129), (1, 128)]) == [128, 128, 256, 128]
    assert O.expert_widths([(3, 1)], block=64) == [64, 64, 64]


def test_offsets_running_sum_bugfix_example(golden_dir):
    g = _load(golden_dir, "bugfix_offsets.json")
    widths = O.expert_widths([tuple(p) for p in g["expert_sizes"]])
    offs = O.expert_offsets(widths)
    e = g["large_expert"]
    assert offs[e] == g["large_expert_offset"]
    assert offs[e] != e * widths[e] == g["wrong_index_times_width_offset"]
    assert offs[-1] == g["total_expert_width"]
    # the printed wrong output offset is token blocks times the large expert's blocks
    assert g["token_blocks_on_large_expert"] * (widths[e] // 128) == g["wrong_output_offset_printed"]


# ---------------------------------------------------------------- capacity
def test_capacity_printed_formula(golden_dir):
    g = _load(golden_dir, "expert_capacity.json")
    for c in g["cases"]:
        assert O.capacity(c["T"], c["k"], c["E"], c["capacity_factor"]) == c["capacity"]
    assert O.capacity(4096, 1, 16, 0.0) is None
    assert O.capacity(4096, 1, 16, -1.0) is None


def test_capacity_rounds_down_reading():
    # the formula has no rounding; the reading taken is floor
    assert O.capacity(1000, 2, 3, 1.0) == 666
    assert O.capacity(10, 1, 4, 0.01) == 0


# ---------------------------------------------------------------- RMS statistic
def test_rms_stat_closed_forms():
    d = 64
    for c in (0.5, 1.0, 3.0):
        x = np.full((1, d), c)
        assert O.rms_stat(x, 1e-5)[0] == pytest.approx(1 / math.sqrt(c * c + 1e-5), rel=1e-15)
    x = np.zeros((1, d)); x[0, 7] = 2.0
    assert O.rms_stat(x, 1e-5)[0] == pytest.approx(1 / math.sqrt(4.0 / d + 1e-5), rel=1e-15)
    assert O.rms_stat(np.zeros((1, d)), 1e-5)[0] == pytest.approx(1 / math.sqrt(1e-5))


def test_rms_stat_matches_torch_rms_norm():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((33, 96)) * 3
    gamma = 1 + 0.1 * rng.standard_normal(96)
    ref = F.rms_norm(_t(x), (96,), _t(gamma), eps=1e-5).numpy()
    np.testing.assert_allclose(O.rmsnorm(x, gamma, 1e-5), ref, rtol=1e-13, atol=1e-14)


def test_norm_then_gemm_equals_gemm_then_rowscale():
    """CODA thread: the statistic commutes across the GEMM into an epilogue."""
    x, gamma, Wr, _, W1, _, _, _ = _small_problem()
    xf, gf, Wrf = O.widen_bf16(x), O.widen_bf16(gamma), O.widen_bf16(Wr)
    xn = F.rms_norm(_t(xf), (xf.shape[1],), _t(gf), eps=1e-5)
    plain = (xn @ _t(Wrf)).numpy()
    r = O.rms_stat(xf, 1e-5)
    commuted = r[:, None] * ((xf * gf[None, :]) @ Wrf)
    np.testing.assert_allclose(commuted, plain, rtol=1e-12, atol=1e-13)
    # the oracle's fp32 router logits equal the plain form rounded once to fp32
    lg = O.router_logits(x=xf, gamma=gf, Wr=Wrf, bias=None, r=r)
    np.testing.assert_array_equal(lg, plain.astype(np.float32))


# ---------------------------------------------------------------- top-k
def test_topk_bruteforce_subsets():
    rng = np.random.default_rng(1)
    for E in range(1, 8):
        for k in range(1, E + 1):
            lg = rng.standard_normal((20, E)).astype(np.float32)
            idx = O.topk_experts(lg, k)
            for t in range(lg.shape[0]):
                best = max(itertools.combinations(range(E), k),
                           key=lambda s: sum(float(lg[t, e]) for e in s))
                assert set(idx[t].tolist()) == set(best)
                vals = lg[t, idx[t]]
                assert np.all(vals[:-1] >= vals[1:])
                rest = [e for e in range(E) if e not in best]
                if rest:
                    assert min(lg[t, list(best)]) >= max(lg[t, rest])


def test_topk_exact_ties_go_to_lower_index():
    lg = np.array([[1, 3, 3, 0, 3],
                   [2, 2, 2, 2, 2],
                   [0, 5, 1, 5, -1]], dtype=np.float32)
    assert O.topk_experts(lg, 2).tolist() == [[1, 2], [0, 1], [1, 3]]
    assert O.topk_experts(lg, 3).tolist() == [[1, 2, 4], [0, 1, 2], [1, 3, 2]]
    assert O.topk_experts(np.array([[-0.0, 0.0]], dtype=np.float32), 1).tolist() == [[0]]
    assert O.topk_experts(np.array([[0.0, -0.0]], dtype=np.float32), 1).tolist() == [[0]]


def test_topk_margin():
    lg = np.array([[3, 1, 2, 0], [1, 1, 1, 1]], dtype=np.float32)
    np.testing.assert_array_equal(O.topk_margin(lg, 2), [1.0, 0.0])
    assert np.isinf(O.topk_margin(lg, 4)).all()


def test_gates_match_torch_softmax():
    rng = np.random.default_rng(2)
    lg = (2 * rng.standard_normal((50, 9))).astype(np.float32)
    idx = O.topk_experts(lg, 3)
    p = torch.softmax(_t(lg), dim=1).numpy()
    np.testing.assert_allclose(O.gates(lg, idx), np.take_along_axis(p, idx, 1), rtol=1e-14)
    g1 = O.gates(lg, O.topk_experts(lg, 1))
    np.testing.assert_allclose(g1[:, 0], p.max(1), rtol=1e-14)      # Switch: top prob, not 1
    assert (g1 < 1).all()
    gr = O.gates(lg, idx, renormalize=True)
    np.testing.assert_allclose(gr.sum(1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(gr, p[np.arange(50)[:, None], idx] / p[np.arange(50)[:, None], idx].sum(1, keepdims=True), rtol=1e-14)


# ---------------------------------------------------------------- dispatch
def _dispatch_bruteforce(idx, E, C):
    """Kept flags by counting earlier assignments; order by Python's sorted()."""
    flat = [int(e) for e in np.asarray(idx).reshape(-1)]
    kept = []
    for a, e in enumerate(flat):
        earlier = sum(1 for b in range(a) if flat[b] == e)
        kept.append(C is None or earlier < C)
    order = sorted((flat[a], a) for a in range(len(flat)) if kept[a])
    return [a for _, a in order], kept


@pytest.mark.parametrize("C", [None, 0, 1, 3, 7, 1000])
def test_dispatch_bruteforce(C):
    idx = mw.random_routing(37, 6, 3, seed=5, skew=1.2)
    D = O.dispatch(idx, 6, C)
    perm, kept = _dispatch_bruteforce(idx, 6, C)
    assert D["perm"].tolist() == perm
    assert D["kept"].tolist() == kept


@pytest.mark.parametrize("C", [None, 0, 1, 40, 100])
def test_dispatch_invariants(C):
    T, E, k = 500, 8, 2
    idx = mw.random_routing(T, E, k, seed=11, skew=1.5)
    D = O.dispatch(idx, E, C)
    counts, kc, offs = D["counts"], D["kept_counts"], D["offsets"]
    assert counts.sum() == T * k
    assert np.array_equal(counts, np.bincount(idx.reshape(-1), minlength=E))
    assert np.array_equal(kc, counts if C is None else np.minimum(counts, C))
    assert offs[0] == 0 and np.array_equal(np.diff(offs), kc)
    perm, inv = D["perm"], D["inv_perm"]
    assert perm.size == D["n_kept"] == offs[-1]
    assert np.array_equal(inv[perm], np.arange(perm.size))           # perm then inv_perm
    kept_a = np.nonzero(inv >= 0)[0]
    assert np.array_equal(perm[inv[kept_a]], kept_a)                  # inv_perm then perm
    flat = idx.reshape(-1)
    for e in range(E):
        seg = perm[offs[e]:offs[e + 1]]
        assert (flat[seg] == e).all()
        assert np.all(np.diff(seg // k) > 0)                          # token order inside a group
    if C is not None:
        assert D["n_kept"] <= E * C


def test_dispatch_rejects_bad_ids():
    with pytest.raises(ValueError):
        O.dispatch(np.array([[0, 9]]), 4, None)


# ---------------------------------------------------------------- whole layer
def _torch_ffn(xn, W1, W3, W2):
    return (F.silu(xn @ W1) * (xn @ W3)) @ W2


def test_single_expert_top1_is_dense_swiglu():
    """E=1, k=1: the layer is a textbook RMSNorm followed by a dense SwiGLU FFN."""
    x, gamma, Wr, _, W1, W3, W2, widths = _small_problem(T=30, d=64, E=1, k=1, widths=[256], bias=False)
    R = O.moe_layer(x, gamma, Wr, None, W1, W3, W2, widths, k=1, eps=1e-5)
    assert np.all(R["gate"] == 1.0)
    xn = F.rms_norm(_t(O.widen_bf16(x)), (64,), _t(O.widen_bf16(gamma)), eps=1e-5)
    ref = _torch_ffn(xn, _t(O.widen_bf16(W1)), _t(O.widen_bf16(W3)), _t(O.widen_bf16(W2))).numpy()
    np.testing.assert_allclose(R["out"], ref, rtol=1e-11, atol=1e-12)


def test_all_experts_is_full_softmax_mixture():
    """k=E: the layer is the softmax-weighted sum of every expert's FFN."""
    E = 4
    widths = [128, 256, 128, 384]
    x, gamma, Wr, b, W1, W3, W2, _ = _small_problem(T=25, d=64, E=E, k=E, widths=widths)
    R = O.moe_layer(x, gamma, Wr, b, W1, W3, W2, widths, k=E, eps=1e-5)
    np.testing.assert_allclose(R["gate"].sum(1), 1.0, rtol=1e-13)
    xn = F.rms_norm(_t(O.widen_bf16(x)), (64,), _t(O.widen_bf16(gamma)), eps=1e-5)
    logits = (xn @ _t(O.widen_bf16(Wr)) + _t(b)).float().double()
    p = torch.softmax(logits, dim=1)
    offs = np.concatenate([[0], np.cumsum(widths)])
    w1, w3, w2 = (_t(O.widen_bf16(a)) for a in (W1, W3, W2))
    ref = sum(p[:, e:e + 1] * _torch_ffn(xn, w1[:, offs[e]:offs[e + 1]], w3[:, offs[e]:offs[e + 1]],
                                          w2[offs[e]:offs[e + 1]]) for e in range(E)).numpy()
    np.testing.assert_allclose(R["out"], ref, rtol=1e-6, atol=1e-9)


def test_topk_layer_matches_masked_mixture():
    """k<E: the output equals the mixture restricted to each token's chosen experts."""
    E, k = 5, 2
    widths = [128, 256, 128, 128, 256]
    x, gamma, Wr, b, W1, W3, W2, _ = _small_problem(T=31, d=64, E=E, k=k, widths=widths, seed=9)
    R = O.moe_layer(x, gamma, Wr, b, W1, W3, W2, widths, k=k, eps=1e-5)
    xn = F.rms_norm(_t(O.widen_bf16(x)), (64,), _t(O.widen_bf16(gamma)), eps=1e-5)
    logits = (xn @ _t(O.widen_bf16(Wr)) + _t(b)).float().double()
    p = torch.softmax(logits, dim=1)
    top = torch.topk(logits, k, dim=1).indices
    mask = torch.zeros_like(p).scatter_(1, top, 1.0)
    offs = np.concatenate([[0], np.cumsum(widths)])
    w1, w3, w2 = (_t(O.widen_bf16(a)) for a in (W1, W3, W2))
    ref = sum((p * mask)[:, e:e + 1] * _torch_ffn(xn, w1[:, offs[e]:offs[e + 1]], w3[:, offs[e]:offs[e + 1]],
                                                   w2[offs[e]:offs[e + 1]]) for e in range(E)).numpy()
    np.testing.assert_allclose(R["out"], ref, rtol=1e-6, atol=1e-9)


def test_capacity_zero_drops_everything():
    x, gamma, Wr, b, W1, W3, W2, widths = _small_problem(T=20, E=4, k=2)
    R = O.moe_layer(x, gamma, Wr, b, W1, W3, W2, widths, k=2, eps=1e-5, capacity_factor=1e-6)
    assert R["capacity"] == 0
    assert np.all(R["out"] == 0) and np.all(R["inv_perm"] == -1)


def test_dropped_slot_contributes_zero():
    x, gamma, Wr, b, W1, W3, W2, widths = _small_problem(T=64, E=4, k=2, seed=4)
    R = O.moe_layer(x, gamma, Wr, b, W1, W3, W2, widths, k=2, eps=1e-5, capacity_factor=0.5)
    full = O.moe_layer(x, gamma, Wr, b, W1, W3, W2, widths, k=2, eps=1e-5)
    kept = R["kept"].reshape(-1, 2)
    assert (~kept).any() and kept.any()
    for t in range(64):
        exp = sum(full["gate"][t, j] * full["y"][2 * t + j] for j in range(2) if kept[t, j])
        np.testing.assert_allclose(R["out"][t], exp if np.ndim(exp) else np.zeros(64), rtol=1e-12, atol=1e-15)


def test_sampled_tokens_equal_full_layer():
    w = mw.WORKLOADS["tiny"]
    widths = O.expert_widths(w.expert_sizes)
    x = mw.gen_x(w); g = mw.gen_gamma(w); Wr = mw.gen_router_weight(w)
    W1, W3, W2 = mw.gen_expert_weights(w, widths)
    R = O.moe_layer(x, g, Wr, None, W1, W3, W2, widths, w.k, w.eps)
    toks = mw.sample_tokens(w, 17)
    out = O.moe_layer_tokens(mw.gen_x(w, toks), toks, g, W1, W3, W2, widths,
                             R["idx"], R["gate"], R["kept"], w.eps)
    np.testing.assert_allclose(out, R["out"][toks], rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- router metrics
def test_router_stats_uniform_closed_form():
    # equal logits: every expert gets probability 1/E; balanced counts
    E, T, k = 8, 64, 2
    lg = np.zeros((T, E), dtype=np.float32)
    counts = np.full(E, T * k // E)
    st = O.router_stats(lg, counts, n_kept=T * k, k=k)
    np.testing.assert_allclose(st["prob_mean"], 1.0 / E, rtol=1e-15)
    assert st["aux_loss"] == pytest.approx(1.0, rel=1e-15)
    assert st["cv2_prob"] == pytest.approx(0.0, abs=1e-30) and st["cv2_load"] == 0.0
    assert st["dropped_frac"] == 0.0


def test_router_stats_one_hot_closed_form():
    # one expert takes everything (huge logit): P -> e_j, f = e_j
    E, T = 6, 50
    lg = np.zeros((T, E), dtype=np.float32); lg[:, 2] = 200.0
    counts = np.zeros(E, dtype=np.int64); counts[2] = T
    st = O.router_stats(lg, counts, n_kept=10, k=1)
    assert st["aux_loss"] == pytest.approx(E, rel=1e-12)
    assert st["cv2_prob"] == pytest.approx(E - 1, rel=1e-12)      # CV^2 of a one-hot vector
    assert st["cv2_load"] == pytest.approx(E - 1, rel=1e-12)
    assert st["dropped_frac"] == pytest.approx(0.8)


def test_router_stats_matches_torch_definitions():
    rng = np.random.default_rng(8)
    lg = (1.5 * rng.standard_normal((300, 10))).astype(np.float32)
    idx = O.topk_experts(lg, 3)
    counts = np.bincount(idx.reshape(-1), minlength=10)
    st = O.router_stats(lg, counts, n_kept=900, k=3)
    P = torch.softmax(_t(lg), dim=1).mean(0)
    np.testing.assert_allclose(st["prob_mean"], P.numpy(), rtol=1e-13)
    assert st["cv2_prob"] == pytest.approx(float(P.var(unbiased=False) / P.mean() ** 2), rel=1e-10)
    assert st["aux_loss"] == pytest.approx(float(10 * (torch.from_numpy(counts / 900.0) * P).sum()), rel=1e-12)
    assert np.isclose(st["prob_mean"].sum(), 1.0)


# ---------------------------------------------------------------- generator
def test_generator_is_seeded_and_sliceable():
    w = mw.WORKLOADS["tiny"]
    a, b = mw.gen_x(w), mw.gen_x(w)
    assert np.array_equal(a, b)
    rows = np.array([0, 5, 255, 100])
    assert np.array_equal(mw.gen_x(w, rows), a[rows])
    widths = [256] * 8
    W1, W3, W2 = mw.gen_expert_weights(w, widths)
    V1, V3, V2 = mw.gen_expert_weights(w, widths, experts=[3])
    assert np.array_equal(V1[:, 768:1024], W1[:, 768:1024]) and not V1[:, :768].any()
    s = O.widen_bf16(W2[:256]).std()
    assert abs(s - 1 / 16) < 0.01
    assert abs(O.widen_bf16(a).std() - 1) < 0.02


def test_bf16_rounding_is_nearest_even():
    v = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e-3], dtype=np.float32)
    bits = mw.f32_to_bf16_bits(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, ref)


# ---------------------------------------------------------------- planted mistakes
MUTANTS = {
    "rms_without_eps": ("rms_stat", lambda x, eps: 1.0 / np.sqrt(np.mean(np.asarray(x, float) ** 2, axis=1))),
    "rms_sum_not_mean": ("rms_stat", lambda x, eps: 1.0 / np.sqrt(np.sum(np.asarray(x, float) ** 2, axis=1) + eps)),
    "router_drops_r": ("router_logits", lambda x, gamma, Wr, bias, r: (
        (np.asarray(x, float) * np.asarray(gamma, float)) @ np.asarray(Wr, float)
        + (0 if bias is None else bias)).astype(np.float32)),
    "topk_ascending": ("topk_experts", lambda lg, k: np.argsort(np.asarray(lg, float), axis=1, kind="stable")[:, :k]),
    "swiglu_swapped": ("expert_ffn", lambda xg, r, W1e, W3e, W2e: (
        O.silu(r[:, None] * (xg @ W3e)) * (r[:, None] * (xg @ W1e))) @ W2e),
    "ffn_without_r": ("expert_ffn", lambda xg, r, W1e, W3e, W2e: (O.silu(xg @ W1e) * (xg @ W3e)) @ W2e),
    "offsets_index_times_width": ("expert_offsets", lambda widths: [e * int(widths[min(e, len(widths) - 1)]) for e in range(len(widths) + 1)]),
}

PINS = [
    lambda gd: test_widths_and_offsets_printed_example(gd),
    lambda gd: test_offsets_running_sum_bugfix_example(gd),
    lambda gd: test_rms_stat_matches_torch_rms_norm(),
    lambda gd: test_norm_then_gemm_equals_gemm_then_rowscale(),
    lambda gd: test_topk_bruteforce_subsets(),
    lambda gd: test_single_expert_top1_is_dense_swiglu(),
    lambda gd: test_all_experts_is_full_softmax_mixture(),
    lambda gd: test_topk_layer_matches_masked_mixture(),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, monkeypatch, golden_dir):
    fn_name, mutant = MUTANTS[name]
    monkeypatch.setattr(O, fn_name, mutant)
    caught = 0
    for pin in PINS:
        try:
            pin(golden_dir)
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught > 0, f"no pin caught mutant {name}"
