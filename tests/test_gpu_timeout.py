"""The bounded-wait failure path, made to run on purpose.

Every pipeline wait of the router and the expert GEMMs gives up after a
limit (4 s by default), sets MOE_DEVERR_TIMEOUT, stops its kernel (both CTAs
of a tensor-core pair), lets the copies and matrix operations already in
flight finish and returns.  Here the limit is set to 1 ns through the
workspace header (moe_set_wait_limit), so nearly every wait that does not
complete at once gives up, on an otherwise normal call.  Each case checks
that the call returns, that the error word says TIMEOUT, and that the next
call on the same workspace with the default limit gives exactly the result
of a call before the failure -- which itself matches the oracle.
No GPU fault is involved: the waits are on barriers whose copies and MMAs
are all legitimately in flight and complete.
"""
import numpy as np
import pytest
import torch

import moe_workloads as mw
import sparse_mixture_experts_rms_b200 as moe
from oracle import moe_oracle as O
from tests import _harness as H

pytestmark = pytest.mark.gpu
SHORT_NS = 1


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_rms_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _problem():
    # several 256-row tiles per expert and 32 K blocks per tile, so every kernel
    # has waits that cannot complete at once
    w = mw.Workload("timeout_case", T=2048, d_model=2048, E=4, k=2, expert_sizes=((4, 512),))
    p = H.make_problem(w)
    return w, p, H.make_cfg(p), H.Dev(p, H.make_cfg(p))


def _expect_timeout(ws):
    code = moe.moe_get_device_error(ws, raise_on_error=False)
    assert code & moe.MOE_DEVERR_TIMEOUT, f"device error word 0x{code:x}: no wait ran out"


def test_forward_waits_run_out_then_recover():
    w, p, cfg, d = _problem()
    run = lambda out: moe.moe_layer_fwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out, d.ws,
                                        expert_idx=idx)
    idx = torch.empty((w.T, w.k), dtype=torch.int32, device="cuda")
    ref = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    run(ref)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(d.ws, raise_on_error=False) == 0
    # the result before the failure matches the oracle
    R = O.moe_layer(p.x, p.gamma, p.Wr, p.bias, p.W1, p.W3, p.W2, p.widths, w.k, w.eps,
                    idx_override=idx.cpu().numpy())
    H.check_rows(H.bf16_dev_to_f64(ref), R["out"], "out before the failure")

    moe.moe_set_wait_limit(d.ws, SHORT_NS)
    bad = torch.zeros_like(ref)
    run(bad)
    torch.cuda.synchronize()          # the call returns
    _expect_timeout(d.ws)

    moe.moe_set_wait_limit(d.ws, 0)   # back to the default limit
    again = torch.empty_like(ref)
    run(again)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(d.ws, raise_on_error=False) == 0
    assert torch.equal(again, ref), "the call after the failure differs"


def test_each_forward_gemm_alone_times_out():
    """The staged up and down GEMMs, each with the short limit on its own."""
    w, p, cfg, d = _problem()
    o = H.run_staged(d)
    y_ref = o["y"].clone()
    for stage in ("up", "down"):
        moe.moe_set_wait_limit(d.ws, SHORT_NS)
        if stage == "up":
            moe.moe_experts_up(cfg, o["x_perm"], o["r"], o["perm"], o["offsets"], d.W1, d.W3, d.ws)
        else:
            moe.moe_experts_down(cfg, o["gate"], o["perm"], o["offsets"], d.W2, o["y"], d.ws)
        torch.cuda.synchronize()
        _expect_timeout(d.ws)
        moe.moe_set_wait_limit(d.ws, 0)
    moe.moe_experts_fwd(cfg, o["x_perm"], o["r"], o["gate"], o["perm"], o["offsets"], d.W1, d.W3, d.W2,
                        o["y"], d.ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(d.ws, raise_on_error=False) == 0
    n = int(o["offsets"][-1].item())
    assert torch.equal(o["y"][:n], y_ref[:n])


def test_mx_forward_waits_run_out_then_recover():
    w, p, cfg, d = _problem()
    wq = moe.alloc_mx_weights(cfg, d.W1, d.W3, d.W2)
    ws = moe.alloc_mx_workspace(cfg)
    run = lambda out: moe.moe_layer_fwd_mx(cfg, d.x, d.gamma, d.Wr, d.bias, wq, out, ws)
    ref = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    run(ref)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws, raise_on_error=False) == 0
    moe.moe_set_wait_limit(ws, SHORT_NS)
    run(torch.zeros_like(ref))
    torch.cuda.synchronize()
    _expect_timeout(ws)
    moe.moe_set_wait_limit(ws, 0)
    again = torch.empty_like(ref)
    run(again)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws, raise_on_error=False) == 0
    assert torch.equal(again, ref)


def test_backward_waits_run_out_then_recover():
    """The four backward contractions (including the dS GEMM, whose epilogue
    waits for its own loads of the saved U, V)."""
    w, p, cfg, d = _problem()
    T, dm, E, F = cfg.T, cfg.d_model, cfg.E, cfg.F
    tws = moe.alloc_train_workspace(cfg)
    out = torch.empty((T, dm), dtype=torch.bfloat16, device="cuda")
    dout = H.bits_to_dev(mw.f32_to_bf16_bits(
        np.random.default_rng(3).standard_normal((T, dm)).astype(np.float32)))
    f32 = dict(dtype=torch.float32, device="cuda")

    def grads():
        return [torch.empty((T, dm), **f32), torch.empty((dm,), **f32), torch.empty((dm, E), **f32),
                torch.empty((E,), **f32), torch.empty((dm, F), **f32), torch.empty((dm, F), **f32),
                torch.empty((F, dm), **f32)]

    moe.moe_layer_fwd_train(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out, tws)
    G_ref = grads()
    moe.moe_layer_bwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, dout, *G_ref, tws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(tws, raise_on_error=False) == 0
    moe.moe_set_wait_limit(tws, SHORT_NS)
    moe.moe_layer_bwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, dout, *grads(), tws)
    torch.cuda.synchronize()
    _expect_timeout(tws)
    moe.moe_set_wait_limit(tws, 0)
    G = grads()
    moe.moe_layer_bwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, dout, *G, tws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(tws, raise_on_error=False) == 0
    for a, b in zip(G, G_ref):
        assert torch.equal(a, b)
