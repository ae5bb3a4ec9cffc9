"""The element-wise gradient checks of the GPU backward tests, exercised on
the CPU: the oracle's own gradients, perturbed at the GPU path's rounding
level (bf16, 2^-9 relative per element), pass; a mistake confined to one
expert's weight slice, one token's dx, one router column or one element of a
cancelling sum fails -- mistakes a whole-tensor norm would dilute."""
import numpy as np
import pytest

import moe_workloads as mw
from oracle import moe_oracle as O
from oracle import moe_oracle_bwd as B
from tests import _harness as H


@pytest.fixture(scope="module")
def case():
    w = mw.Workload("grad_checks", T=96, d_model=128, E=8, k=2, expert_sizes=((8, 128),), bias="normal")
    p = H.make_problem(w)
    f = B.layer_forward(O.widen_bf16(p.x), O.widen_bf16(p.gamma), O.widen_bf16(p.Wr), p.bias,
                        O.widen_bf16(p.W1), O.widen_bf16(p.W3), O.widen_bf16(p.W2), p.widths, w.k, w.eps)
    g = O.widen_bf16(mw.f32_to_bf16_bits(np.random.default_rng(5).standard_normal((w.T, w.d_model))
                                         .astype(np.float32)))
    ref = B.layer_backward(f, g)
    return w, f, g, ref


def _noisy(a, seed):
    """a with an independent relative error of 2^-9 per element (one bf16 rounding)."""
    rng = np.random.default_rng(seed)
    return a * (1.0 + 2.0 ** -9 * rng.uniform(-1.0, 1.0, size=np.shape(a)))


def test_rounding_level_errors_pass(case):
    w, f, g, ref = case
    H.check_grad_rows(_noisy(ref["dx"], 1), ref["dx"], "dx")
    o = f["offs"]
    for e in range(w.E):
        H.check_grad_slice(_noisy(ref["dW1"][:, o[e]:o[e + 1]], 2), ref["dW1"][:, o[e]:o[e + 1]], "dW1")
        H.check_grad_slice(_noisy(ref["dW2"][o[e]:o[e + 1]], 3), ref["dW2"][o[e]:o[e + 1]], "dW2")
    rss = H.grad_term_rss(f, g, ref)
    H.check_sum_elems(_noisy(ref["dWr"], 4), ref["dWr"], rss["dWr"], "dWr")
    H.check_sum_elems(_noisy(ref["dgamma"], 5), ref["dgamma"], rss["dgamma"], "dgamma")
    H.check_sum_elems(_noisy(ref["dbias"], 6), ref["dbias"], rss["dbias"], "dbias")
    H.check_sum_elems(_noisy(ref["dr"], 7), ref["dr"], rss["dr"], "dr")
    # an error the size of one term's rounding, on a sum that cancels to ~0, passes
    H.check_sum_elems(ref["dbias"] + 2.0 ** -9 * rss["dbias"], ref["dbias"], rss["dbias"], "dbias")


def test_one_expert_slice_wrong_by_four_percent_fails(case):
    w, f, g, ref = case
    o = f["offs"]
    bad = ref["dW1"].copy()
    bad[:, o[3]:o[4]] *= 1.04
    # diluted over the whole tensor it stays under the bar ...
    whole = np.linalg.norm(bad - ref["dW1"]) / np.linalg.norm(ref["dW1"])
    assert whole < H.GRAD_REL
    # ... but the slice check catches it
    with pytest.raises(AssertionError):
        for e in range(w.E):
            H.check_grad_slice(bad[:, o[e]:o[e + 1]], ref["dW1"][:, o[e]:o[e + 1]], "dW1")


def test_one_token_and_one_column_fail(case):
    w, f, g, ref = case
    dx = ref["dx"].copy()
    dx[17] *= 1.05
    with pytest.raises(AssertionError):
        H.check_grad_rows(dx, ref["dx"], "dx")
    dWr = ref["dWr"].copy()
    dWr[:, 2] = -dWr[:, 2]  # a sign error in one expert's router column
    rss = H.grad_term_rss(f, g, ref)
    with pytest.raises(AssertionError):
        H.check_sum_elems(dWr, ref["dWr"], rss["dWr"], "dWr")


def test_renormalised_unchosen_expert_has_a_zero_router_gradient_floor():
    """With renormalised gates <dp, p> = 0, so an expert no token chose has an
    exactly zero router gradient in exact arithmetic; the bound of its dbias
    and dWr entries comes from the size of the softmax backward's terms, so
    fp32 residue of that size passes and a gross error still fails."""
    w = mw.Workload("grad_checks_renorm", T=64, d_model=128, E=16, k=2, expert_sizes=((16, 128),), bias="normal")
    p = H.make_problem(w)
    p.bias = p.bias.copy()
    p.bias[5] = -30.0   # expert 5 is never chosen
    f = B.layer_forward(O.widen_bf16(p.x), O.widen_bf16(p.gamma), O.widen_bf16(p.Wr), p.bias,
                        O.widen_bf16(p.W1), O.widen_bf16(p.W3), O.widen_bf16(p.W2), p.widths, w.k, w.eps,
                        renormalize=True)
    assert not (f["idx"] == 5).any()
    g = np.random.default_rng(2).standard_normal((w.T, w.d_model))
    ref = B.layer_backward(f, g)
    rss = H.grad_term_rss(f, g, ref)
    assert abs(ref["dbias"][5]) < 1e-6 * rss["dbias"][5] + 1e-300
    noisy = ref["dbias"].copy()
    noisy[5] += 1e-3 * rss["dbias"][5]          # fp32-level residue on an exact zero
    H.check_sum_elems(noisy, ref["dbias"], rss["dbias"], "dbias")
    noisy[5] += 0.1 * rss["dbias"][5]           # a real error
    with pytest.raises(AssertionError):
        H.check_sum_elems(noisy, ref["dbias"], rss["dbias"], "dbias")


def test_one_element_of_a_cancelling_sum_fails(case):
    w, f, g, ref = case
    rss = H.grad_term_rss(f, g, ref)
    db = ref["dbias"].copy()
    db[4] += 0.1 * rss["dbias"][4]  # ten percent of the terms' size: far above rounding
    with pytest.raises(AssertionError):
        H.check_sum_elems(db, ref["dbias"], rss["dbias"], "dbias")
    dr = ref["dr"].copy()
    dr[5] = -dr[5] if abs(dr[5]) > 0.05 * rss["dr"][5] else dr[5] + 0.1 * rss["dr"][5]
    with pytest.raises(AssertionError):
        H.check_sum_elems(dr, ref["dr"], rss["dr"], "dr")
