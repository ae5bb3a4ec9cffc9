"""GPU parity of the layer backward (training forward + moe_layer_bwd) against
the float64 backward oracle, on the GPU's own routing (replayed into the
oracle, whose routing parity the forward tests establish).

Every gradient is compared piece by piece, at the forward's bar
(``tests/_harness.py``): dx per token row; dW1, dW3, dW2 per expert slice;
dWr, dgamma, dbias and dr per element, within 2e-2 of |ref| plus the
root-sum-square of the terms they sum (those sums can cancel); dgate
per assignment against the dot product of dout with the GPU's own saved
expert output (replay), and as a vector against the oracle.  A mistake
confined to one expert's slice therefore fails even when the other slices
are right.  The GPU path rounds x*gamma, U, V, H, gate*dout,
dS and dS3 to bf16 (each 2^-9 relative) and accumulates in fp32; the
measured errors are printed.
"""
import numpy as np
import pytest
import torch

import moe_workloads as mw
import sparse_mixture_experts_rms_b200 as moe
from oracle import moe_oracle as O
from oracle import moe_oracle_bwd as B
from tests import _harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_rms_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _upstream(T, d, seed=7):
    g = np.random.default_rng(seed).standard_normal((T, d)).astype(np.float32)
    return mw.f32_to_bf16_bits(g)


def _rel(a, b):
    n = float(np.linalg.norm(b))
    return float(np.linalg.norm(a - b)) / (n if n > 0 else 1.0)


def run_case(w, renormalize=False, bias_override=None, problem=None):
    p = H.make_problem(w) if problem is None else problem
    if bias_override is not None:
        p.bias = np.asarray(bias_override, dtype=np.float32)
    cfg = H.make_cfg(p, renormalize=renormalize)
    d = H.Dev(p, cfg)
    T, dm, E, F = cfg.T, cfg.d_model, cfg.E, cfg.F
    tws = moe.alloc_train_workspace(cfg)
    out = torch.empty((T, dm), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_fwd_train(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out, tws)
    ref_out = torch.empty_like(out)
    moe.moe_layer_fwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, ref_out, d.ws)
    g_bits = _upstream(T, dm)
    dout = H.bits_to_dev(g_bits)
    f32 = dict(dtype=torch.float32, device="cuda")
    G = {"dx": torch.full((T, dm), float("nan"), **f32), "dgamma": torch.full((dm,), float("nan"), **f32),
         "dWr": torch.full((dm, E), float("nan"), **f32), "dbias": torch.full((E,), float("nan"), **f32),
         "dW1": torch.full((dm, F), float("nan"), **f32), "dW3": torch.full((dm, F), float("nan"), **f32),
         "dW2": torch.full((F, dm), float("nan"), **f32)}
    moe.moe_layer_bwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, dout, G["dx"], G["dgamma"],
                      G["dWr"], G["dbias"], G["dW1"], G["dW3"], G["dW2"], tws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(tws, raise_on_error=False) == 0
    assert torch.equal(out, ref_out), "training forward differs from the inference forward"
    idx = moe.train_saved_view(cfg, tws, "idx").cpu().numpy()
    f = B.layer_forward(O.widen_bf16(p.x), O.widen_bf16(p.gamma), O.widen_bf16(p.Wr), p.bias,
                        O.widen_bf16(p.W1), O.widen_bf16(p.W3), O.widen_bf16(p.W2), p.widths, w.k,
                        w.eps, w.capacity_factor, renormalize, idx=idx)
    ref = B.layer_backward(f, O.widen_bf16(g_bits))
    got = {name: t.cpu().numpy().astype(np.float64) for name, t in G.items()}
    errs = {}
    errs["dx"] = H.check_grad_rows(got["dx"], ref["dx"], "dx per token")[0]
    offs = f["offs"]
    kept_e = np.bincount(idx.reshape(-1)[f["kept"]], minlength=E)
    slices = (("dW1", lambda o0, o1: np.s_[:, o0:o1]), ("dW3", lambda o0, o1: np.s_[:, o0:o1]),
              ("dW2", lambda o0, o1: np.s_[o0:o1, :]))
    for e in range(E):
        o0, o1 = offs[e], offs[e + 1]
        for name, sl in slices:
            if kept_e[e] == 0:  # an expert with no rows gets exactly zero weight gradients
                assert np.count_nonzero(got[name][sl(o0, o1)]) == 0, (name, e)
            else:
                errs[f"{name}[{e}]"] = H.check_grad_slice(got[name][sl(o0, o1)], ref[name][sl(o0, o1)],
                                                          f"{name} expert {e} slice")
    rss = H.grad_term_rss(f, O.widen_bf16(g_bits), ref)
    errs["dWr"] = H.check_sum_elems(got["dWr"], ref["dWr"], rss["dWr"], "dWr")
    errs["dgamma"] = H.check_sum_elems(got["dgamma"], ref["dgamma"], rss["dgamma"], "dgamma")
    errs["dbias"] = H.check_sum_elems(got["dbias"], ref["dbias"], rss["dbias"], "dbias")
    kept = f["kept"]
    dg = moe.train_saved_view(cfg, tws, "dgate").cpu().numpy().astype(np.float64)
    # dgate: per assignment against the dot product with the GPU's own saved y (replay;
    # fp32 accumulation of d products), and as a vector against the oracle (the chain)
    rep, rep_rss = H.dgate_replay(cfg, tws, g_bits)
    H.check_sum_elems(dg[kept], rep.reshape(-1)[kept], rep_rss.reshape(-1)[kept], "dgate replay",
                      rel=H.DGATE_REPLAY_REL)
    errs["dgate"] = _rel(dg[kept], ref["dgate"].reshape(-1)[kept])
    assert errs["dgate"] <= H.GRAD_REL, ("dgate", errs["dgate"])
    dr = moe.train_saved_view(cfg, tws, "dr").cpu().numpy().astype(np.float64)
    errs["dr"] = H.check_sum_elems(dr, ref["dr"], rss["dr"], "dr")
    worst_slice = max((v for k_, v in errs.items() if "[" in k_), default=0.0)
    print(w.name, {k_: f"{v:.2e}" for k_, v in errs.items() if "[" not in k_},
          f"worst weight slice {worst_slice:.2e}")
    return p, f, G


def test_tiny_backward():
    run_case(mw.WORKLOADS["tiny"])


def test_variable_widths_renormalized_backward():
    """Widths that are odd multiples of 128 (N tile 128 in the dS GEMM), a
    ragged row count and renormalised gates."""
    w = mw.Workload("bwd_var", T=300, d_model=256, E=4, k=2,
                    expert_sizes=((1, 128), (1, 384), (1, 256), (1, 512)))
    run_case(w, renormalize=True)


def test_capacity_and_empty_expert_backward():
    """Top-1 with capacity drops; expert 2 never chosen (large negative bias):
    its weight gradients are exactly zero."""
    w = mw.Workload("bwd_cap", T=512, d_model=256, E=4, k=1, expert_sizes=((4, 256),),
                    capacity_factor=1.0)
    p, f, G = run_case(w, bias_override=[0.5, 0.0, -60.0, 0.2])
    o = O.expert_offsets(p.widths)
    assert not (f["idx"] == 2).any()
    assert torch.count_nonzero(G["dW1"][:, o[2]:o[3]]).item() == 0
    assert torch.count_nonzero(G["dW3"][:, o[2]:o[3]]).item() == 0
    assert torch.count_nonzero(G["dW2"][o[2]:o[3], :]).item() == 0
    assert not f["kept"].all()


def test_several_tiles_backward():
    """Several 256-row M tiles and 64-row K blocks per expert."""
    w = mw.Workload("bwd_tiles", T=1000, d_model=256, E=4, k=2, expert_sizes=((4, 512),), bias="normal")
    run_case(w)


def test_autograd_layer_gives_the_direct_gradients():
    """MoETrainLayer under torch autograd returns what moe_layer_bwd returns
    (cast to the parameters' dtypes) and the forward's output."""
    w = mw.WORKLOADS["tiny"]
    p = H.make_problem(w)
    cfg = H.make_cfg(p)
    d = H.Dev(p, cfg)
    params = [t.clone().requires_grad_(True) for t in (d.gamma, d.Wr, d.W1, d.W3, d.W2)]
    x = d.x.clone().requires_grad_(True)
    layer = moe.MoETrainLayer(cfg, params[0], params[1], None, params[2], params[3], params[4])
    out = layer(x)
    dout = H.bits_to_dev(_upstream(w.T, w.d_model))
    out.backward(dout)
    torch.cuda.synchronize()
    ref_out = torch.empty_like(out)
    moe.moe_layer_fwd(cfg, d.x, d.gamma, d.Wr, None, d.W1, d.W3, d.W2, ref_out, d.ws)
    assert torch.equal(out.detach(), ref_out)
    tws = moe.alloc_train_workspace(cfg)
    moe.moe_layer_fwd_train(cfg, d.x, d.gamma, d.Wr, None, d.W1, d.W3, d.W2, torch.empty_like(out), tws)
    f32 = dict(dtype=torch.float32, device="cuda")
    T, dm, E, F = cfg.T, cfg.d_model, cfg.E, cfg.F
    G = [torch.empty((T, dm), **f32), torch.empty((dm,), **f32), torch.empty((dm, E), **f32),
         torch.empty((E,), **f32), torch.empty((dm, F), **f32), torch.empty((dm, F), **f32),
         torch.empty((F, dm), **f32)]
    moe.moe_layer_bwd(cfg, d.x, d.gamma, d.Wr, None, d.W1, d.W3, d.W2, dout, *G, tws)
    torch.cuda.synchronize()
    for got, ref in zip([x.grad] + [t.grad for t in params], [G[0], G[1], G[2], G[4], G[5], G[6]]):
        assert torch.equal(got, ref.to(got.dtype))


def test_fine_grained_backward():
    """E = 64, top-8 with renormalised gates and a normal logit bias: the
    E <= 64 variant of the norm backward and the router backward over 8 slots."""
    w = mw.Workload("bwd_fine", T=300, d_model=256, E=64, k=8, expert_sizes=((64, 128),), bias="normal")
    run_case(w, renormalize=True)


def test_degenerate_rows_backward():
    """Zero rows (r = 1/sqrt(eps), all logits tied at 0), rows scaled by 2^12 and
    2^-12, and two identical router columns: every gradient within the bar.
    A zero row has U = V = 0, so H, y, dS, dS3, dgate and the router gradient
    of that token vanish, and its dx is exactly zero."""
    w = mw.Workload("bwd_degenerate", T=256, d_model=256, E=8, k=2, expert_sizes=((8, 128),))
    _, _, G = run_case(w, problem=H.degenerate_problem(w))
    assert torch.count_nonzero(G["dx"][0:16]).item() == 0
