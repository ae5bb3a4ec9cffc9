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
        H.check_grad_rows(_noisy(ref["dW1"][:, o[e]:o[e + 1]], 2), ref["dW1"][:, o[e]:o[e + 1]], "dW1")
        H.check_grad_rows(_noisy(ref["dW2"][o[e]:o[e + 1]], 3), ref["dW2"][o[e]:o[e + 1]], "dW2")
    H.check_grad_rows(_noisy(ref["dWr"], 4).T, ref["dWr"].T, "dWr")
    rss = H.grad_term_rss(f, g, ref)
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
            H.check_grad_rows(bad[:, o[e]:o[e + 1]], ref["dW1"][:, o[e]:o[e + 1]], "dW1")


def test_one_token_and_one_column_fail(case):
    w, f, g, ref = case
    dx = ref["dx"].copy()
    dx[17] *= 1.05
    with pytest.raises(AssertionError):
        H.check_grad_rows(dx, ref["dx"], "dx")
    dWr = ref["dWr"].copy()
    dWr[:, 2] = -dWr[:, 2]  # a sign error in one expert's router column
    with pytest.raises(AssertionError):
        H.check_grad_rows(dWr.T, ref["dWr"].T, "dWr")


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
