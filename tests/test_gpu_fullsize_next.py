"""Full-size parity of the backward and the MXFP8 path on sampled tokens.

The GPU runs the whole layer at the workload's full size (the configuration
the bench times); the oracle recomputes a sample of tokens.  Without a
capacity limit a token's output, and its dx / dr / gate gradients, depend on
that token alone (given the routing, replayed from the GPU as in the other
full-size tests), so the sample is computed exactly.  Samples are drawn among
tokens whose experts lie in a few experts, so that the oracle widens or
quantises only those experts' weight slices.  Gradients are compared element
by element: dx per token row, dr per token, dgate per assignment against the
GPU's own saved expert outputs and as a vector against the oracle (see
``tests/_harness.py`` for the bars).
"""
import numpy as np
import pytest
import torch

import moe_workloads as mw
import sparse_mixture_experts_rms_b200 as moe
from oracle import moe_oracle as O
from oracle import moe_oracle_bwd as B
from oracle import moe_oracle_mx as M
from tests import _harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_rms_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _sample(idx, allowed, n, seed=3):
    ok = np.all(np.isin(idx, allowed), axis=1)
    cand = np.nonzero(ok)[0]
    assert cand.size > 0
    rng = np.random.default_rng(seed)
    return np.sort(rng.choice(cand, size=min(n, cand.size), replace=False))


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


@pytest.mark.parametrize("name,allowed,n", [("mixtral", [0, 1, 2], 24), ("fine_grained", list(range(64)), 96)])
def test_mx_layer_full_size_sampled(name, allowed, n):
    w = mw.WORKLOADS[name]
    p = H.make_problem(w)
    cfg = H.make_cfg(p)
    d = H.Dev(p, cfg)
    wq = moe.alloc_mx_weights(cfg, d.W1, d.W3, d.W2)
    ws = moe.alloc_mx_workspace(cfg)
    out = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_fwd_mx(cfg, d.x, d.gamma, d.Wr, d.bias, wq, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws, raise_on_error=False) == 0
    g_idx = moe.mx_part_view(cfg, wq, ws, "IDX").cpu().numpy()
    toks = _sample(g_idx, allowed, n)
    x = O.widen_bf16(p.x[toks])
    logits = O.router_logits(x, O.widen_bf16(p.gamma), O.widen_bf16(p.Wr), p.bias, O.rms_stat(x, w.eps))
    gate = np.zeros((w.T, w.k))
    gate[toks] = O.gates(logits, g_idx[toks])
    lazy = M.LazyExpertWeights(p.W1, p.W3, p.W2, O.expert_offsets(p.widths))
    ref = M.moe_layer_mx_tokens(p.x[toks], toks, p.gamma, lazy, p.widths, g_idx, gate,
                                np.ones(w.T * w.k, dtype=bool), w.eps)
    got = H.bf16_dev_to_f64(out[torch.from_numpy(toks).cuda()])
    H.check_rows(got, ref, f"{name} mx out")
    print(name, f"MX full size, {toks.size} tokens: normwise {_rel(got, ref):.2e}")


@pytest.mark.parametrize("name,allowed,n", [("mixtral", [0, 1], 8), ("fine_grained", list(range(64)), 48)])
def test_backward_full_size_sampled(name, allowed, n):
    w = mw.WORKLOADS[name]
    p = H.make_problem(w)
    cfg = H.make_cfg(p)
    d = H.Dev(p, cfg)
    T, dm, E, F = cfg.T, cfg.d_model, cfg.E, cfg.F
    tws = moe.alloc_train_workspace(cfg)
    out = torch.empty((T, dm), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_fwd_train(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out, tws)
    g_bits = mw.f32_to_bf16_bits(np.random.default_rng(7).standard_normal((T, dm)).astype(np.float32))
    f32 = dict(dtype=torch.float32, device="cuda")
    G = [torch.empty((T, dm), **f32), torch.empty((dm,), **f32), torch.empty((dm, E), **f32),
         torch.empty((E,), **f32), torch.empty((dm, F), **f32), torch.empty((dm, F), **f32),
         torch.empty((F, dm), **f32)]
    moe.moe_layer_bwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, H.bits_to_dev(g_bits), *G, tws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(tws, raise_on_error=False) == 0
    g_idx = moe.train_saved_view(cfg, tws, "idx").cpu().numpy()
    toks = _sample(g_idx, allowed, n)
    f = B.layer_forward(O.widen_bf16(p.x[toks]), O.widen_bf16(p.gamma), O.widen_bf16(p.Wr), p.bias,
                        p.W1, p.W3, p.W2, p.widths, w.k, w.eps, idx=g_idx[toks])
    ref = B.layer_backward(f, O.widen_bf16(g_bits[toks]), weight_grads=False)
    dx = G[0][torch.from_numpy(toks).cuda()].cpu().numpy().astype(np.float64)
    dr = moe.train_saved_view(cfg, tws, "dr").cpu().numpy()[toks].astype(np.float64)
    dgate = moe.train_saved_view(cfg, tws, "dgate").cpu().numpy().reshape(T, w.k)[toks].astype(np.float64)
    rss = H.grad_term_rss(f, O.widen_bf16(g_bits[toks]), ref)
    kept = f["kept"].reshape(-1)
    rep, rep_rss = H.dgate_replay(cfg, tws, g_bits, toks)
    H.check_sum_elems(dgate.reshape(-1)[kept], rep.reshape(-1)[kept], rep_rss.reshape(-1)[kept],
                      f"{name} dgate replay", rel=H.DGATE_REPLAY_REL)
    errs = {"dx": H.check_grad_rows(dx, ref["dx"], f"{name} dx per token")[0],
            "dr": H.check_sum_elems(dr, ref["dr"], rss["dr"], f"{name} dr"),
            "dgate": _rel(dgate.reshape(-1)[kept], ref["dgate"].reshape(-1)[kept])}
    assert errs["dgate"] <= H.GRAD_REL, ("dgate", errs["dgate"])
    print(name, f"backward full size, {toks.size} tokens (dx: worst row error; dr: worst error / bound; "
                "dgate: normwise):", {k: f"{v:.2e}" for k, v in errs.items()})
