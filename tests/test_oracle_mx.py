"""Pins of the MXFP8 oracle against things other than itself: the E4M3 value
set enumerated from its bit layout, torch's own float8_e4m3fn conversion,
closed forms of the shared exponent, the blocking axis, and the reduction of
the MX layer to the pinned forward oracle when quantisation is the identity."""
import numpy as np
import pytest

import moe_workloads as mw
from oracle import moe_oracle as O
from oracle import moe_oracle_mx as M


def e4m3_values():
    """All finite E4M3 (fn) values from the bit layout: 1 sign, 4 exponent
    (bias 7), 3 fraction bits; exponent field 0 is subnormal; 0x7F/0xFF NaN."""
    vals = []
    for code in range(128):
        if code == 0x7F:
            continue
        e, f = code >> 3, code & 7
        v = (f / 8.0) * 2.0 ** -6 if e == 0 else (1 + f / 8.0) * 2.0 ** (e - 7)
        vals.append((code, v))
    return vals


def test_every_e4m3_value_is_a_fixed_point():
    vals = np.array([v for _, v in e4m3_values()])
    assert vals.max() == 448.0 and sorted(vals)[1] == 2.0 ** -9
    np.testing.assert_array_equal(M.e4m3_round(vals), vals)
    np.testing.assert_array_equal(M.e4m3_round(-vals), -vals)


def test_midpoints_round_to_the_even_code():
    vals = sorted(e4m3_values(), key=lambda cv: cv[1])
    for (c0, v0), (c1, v1) in zip(vals, vals[1:]):
        mid = 0.5 * (v0 + v1)
        want = v0 if c0 % 2 == 0 else v1
        assert M.e4m3_round(np.array([mid]))[0] == want, (v0, v1)


def test_saturation_above_the_largest_normal():
    np.testing.assert_array_equal(M.e4m3_round(np.array([449.0, 464.0, 500.0, 1e9, -1e9])),
                                  [448.0, 448.0, 448.0, 448.0, -448.0])


def test_rounding_matches_torch_float8_e4m3fn():
    torch = pytest.importorskip("torch")
    if not hasattr(torch, "float8_e4m3fn"):
        pytest.skip("torch without float8")
    v = np.random.default_rng(0).uniform(-440.0, 440.0, 20000)
    v = np.concatenate([v, v * 1e-3, v * 1e-5])
    ref = torch.tensor(v, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(M.e4m3_round(v.astype(np.float32).astype(np.float64)), ref)


def test_shared_exponent_closed_forms():
    # amax in [2^e, 2^(e+1)) -> e - 8; zero block -> -127
    assert list(M.mx_scale_exp(np.array([1.0, 1.99, 2.0, 0.75, 448.0, 0.0]))) == [-8, -8, -7, -9, 0, -127]
    b = np.zeros((1, 32))
    b[0, 3] = 1.9            # scaled: 1.9 * 256 = 486.4 -> saturates to 448 -> 1.75
    b[0, 5] = -0.5           # -128 exactly
    c, s = M.mx_quantize(b)
    assert s[0, 0] == -8
    assert c[0, 3] == 448.0 and c[0, 5] == -128.0
    np.testing.assert_array_equal(M.mx_value(b)[0, [3, 5]], [1.75, -0.5])
    c, s = M.mx_quantize(np.zeros((2, 64)))
    assert (s == -127).all() and (c == 0).all()


def test_relative_error_bound_of_unsaturated_values():
    v = np.random.default_rng(1).standard_normal((64, 256))
    q = M.mx_value(v, axis=1)
    # every block's largest element scales into [256, 512); elements that do
    # not saturate are rounded with relative error <= 2^-4
    a = np.abs(v)
    blk = a.reshape(64, 8, 32).max(axis=2).repeat(32, axis=1)
    ok = (a / np.exp2(np.floor(np.log2(blk)) - 8) <= 448.0) & (a >= blk * 2.0 ** -8)
    assert ok.mean() > 0.9
    assert np.all(np.abs(q - v)[ok] <= a[ok] * 2.0 ** -4 + 1e-300)


def test_blocks_run_along_the_requested_axis():
    # a 2^20 spike sets its block's scale to 2^12, so the block's ones fall
    # below E4M3's smallest step (2^-9 after scaling) and vanish; every other
    # block is untouched
    W = np.ones((64, 8))
    W[0, 3] = 2.0 ** 20      # one block of column 3 along axis 0: rows 0..31
    q = M.mx_value(W, axis=0)
    assert np.all(q[:, [0, 1, 2, 4, 5, 6, 7]] == 1.0)
    assert np.all(q[32:, 3] == 1.0)
    assert q[0, 3] == 2.0 ** 20 and np.all(q[1:32, 3] == 0.0)
    x = np.ones((4, 64))
    x[2, 40] = 2.0 ** 20     # token 2's second block along d
    q = M.mx_value(x, axis=1)
    assert np.all(q[[0, 1, 3]] == 1.0) and np.all(q[2, :32] == 1.0)
    assert q[2, 40] == 2.0 ** 20 and np.count_nonzero(q[2, 32:]) == 1


def test_mx_layer_with_identity_quantisation_is_the_forward_oracle(monkeypatch):
    w = mw.WORKLOADS["tiny"]
    x, g = mw.gen_x(w), mw.gen_gamma(w)
    Wr, b = mw.gen_router_weight(w), mw.gen_router_bias(w)
    widths = O.expert_widths(w.expert_sizes)
    W1, W3, W2 = mw.gen_expert_weights(w, widths)
    ref = O.moe_layer(x, g, Wr, b, W1, W3, W2, widths, w.k, w.eps)
    monkeypatch.setattr(M, "mx_value", lambda v, axis=-1: np.asarray(v, dtype=np.float64))
    got = M.moe_layer_mx(x, g, Wr, b, W1, W3, W2, widths, w.k, w.eps)
    np.testing.assert_allclose(got["out"], ref["out"], rtol=1e-12, atol=1e-14)


def test_mx_layer_is_close_to_the_exact_layer():
    w = mw.WORKLOADS["tiny"]
    x, g = mw.gen_x(w), mw.gen_gamma(w)
    Wr, b = mw.gen_router_weight(w), mw.gen_router_bias(w)
    widths = O.expert_widths(w.expert_sizes)
    W1, W3, W2 = mw.gen_expert_weights(w, widths)
    ref = O.moe_layer(x, g, Wr, b, W1, W3, W2, widths, w.k, w.eps)
    got = M.moe_layer_mx(x, g, Wr, b, W1, W3, W2, widths, w.k, w.eps)
    rel = np.linalg.norm(got["out"] - ref["out"]) / np.linalg.norm(ref["out"])
    assert 1e-3 < rel < 0.08, rel        # E4M3 carries 3 fraction bits


MUTANTS = {
    "round half away from zero": lambda v: np.copysign(
        np.minimum(np.floor(np.abs(v) / (s := np.exp2(np.maximum(np.floor(np.log2(np.where(np.abs(v) > 0, np.abs(v), 1.0))), -6) - 3)) + 0.5) * s, 448.0), v),
    "no saturation": lambda v: np.copysign(
        np.round(np.abs(v) / (s := np.exp2(np.maximum(np.floor(np.log2(np.where(np.abs(v) > 0, np.abs(v), 1.0))), -6) - 3))) * s, v),
    "no subnormals": lambda v: np.copysign(
        np.minimum(np.round(np.abs(v) / (s := np.exp2(np.floor(np.log2(np.where(np.abs(v) > 0, np.abs(v), 1.0))) - 3))) * s, 448.0), v),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_rounding_mistakes_are_caught(mutant, monkeypatch):
    monkeypatch.setattr(M, "e4m3_round", MUTANTS[mutant])
    failures = 0
    for t in (test_every_e4m3_value_is_a_fixed_point, test_midpoints_round_to_the_even_code,
              test_saturation_above_the_largest_normal):
        try:
            t()
        except AssertionError:
            failures += 1
    assert failures > 0, mutant


def test_lazy_per_expert_quantisation_equals_the_whole_matrix():
    w = mw.WORKLOADS["variable_size"]
    widths = O.expert_widths(w.expert_sizes)
    W1, W3, W2 = mw.gen_expert_weights(w, widths, experts=[0, 3])
    full = M.quantized_weights(W1, W3, W2)
    offs = O.expert_offsets(widths)
    lazy = M.LazyExpertWeights(W1, W3, W2, offs)
    for e in (0, 3):
        o0, o1 = offs[e], offs[e + 1]
        for got, ref in zip(lazy.expert(e), (full["W1"][:, o0:o1], full["W3"][:, o0:o1], full["W2"][o0:o1, :])):
            np.testing.assert_array_equal(got, ref)
