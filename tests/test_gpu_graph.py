"""The layer is stream-ordered with no host synchronisation, so it can be
captured into a CUDA graph and replayed; and more tile-boundary cases of the
2-CTA grouped GEMM (expert row counts just below / at / above the 256-row pair
tile, empty experts between full ones)."""
import numpy as np
import pytest
import torch

import moe_workloads as mw
import sparse_mixture_experts_rms_b200 as moe
from oracle import moe_oracle as O
from tests import _harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_rms_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def test_layer_captures_into_cuda_graph_and_replays_bit_exactly():
    w = mw.WORKLOADS["variable_size"].with_tokens(1500, name="var_graph")
    p = H.make_problem(w)
    cfg = H.make_cfg(p)
    d = H.Dev(p, cfg)
    out_eager = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    stats_eager = torch.empty(4, dtype=torch.float32, device="cuda")
    moe.moe_layer_fwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out_eager, d.ws,
                      stats=stats_eager)   # first call: per-device set-up happens outside capture
    torch.cuda.synchronize()
    out_g = torch.zeros_like(out_eager)
    stats_g = torch.zeros_like(stats_eager)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_layer_fwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out_g, d.ws,
                          stats=stats_g)
    for _ in range(3):
        out_g.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_g, out_eager)
        assert torch.equal(stats_g, stats_eager)
    assert moe.moe_get_device_error(d.ws, raise_on_error=False) == 0
    del g


@pytest.mark.parametrize("rows", [[255, 0, 256, 257], [1, 511, 0, 512], [0, 0, 1000, 3]])
def test_pair_tile_boundaries(rows):
    """Expert row counts chosen around the 256-row pair tile (k=1), through the
    staged calls with a replayed routing."""
    E = len(rows)
    T = sum(rows)
    w = mw.Workload("tiles", T=T, d_model=256, E=E, k=1, expert_sizes=((E, 256),))
    p = H.make_problem(w)
    # the routing is given (replayed): token t goes to expert want[t]
    idx = np.repeat(np.arange(E), rows).reshape(T, 1).astype(np.int32)
    x = O.widen_bf16(p.x)
    cfg = H.make_cfg(p)
    d = H.Dev(p, cfg)
    mk = moe.moe_max_kept(cfg)
    o = {"counts": torch.empty(E, dtype=torch.int32, device="cuda"),
         "offsets": torch.empty(E + 1, dtype=torch.int32, device="cuda"),
         "perm": torch.empty(mk, dtype=torch.int32, device="cuda"),
         "inv_perm": torch.empty(T, dtype=torch.int32, device="cuda"),
         "x_perm": torch.empty(mk, w.d_model, dtype=torch.bfloat16, device="cuda"),
         "y": torch.zeros(mk, w.d_model, dtype=torch.bfloat16, device="cuda"),
         "out": torch.empty(T, w.d_model, dtype=torch.bfloat16, device="cuda")}
    gate = torch.rand(T, 1, generator=torch.Generator().manual_seed(1)).float().cuda()
    r = torch.from_numpy(O.rms_stat(x, w.eps).astype(np.float32)).cuda()
    moe.moe_dispatch(cfg, torch.from_numpy(idx).cuda(), d.x, d.gamma, o["counts"], o["offsets"],
                     o["perm"], o["inv_perm"], o["x_perm"], d.ws)
    moe.moe_experts_fwd(cfg, o["x_perm"], r, gate, o["perm"], o["offsets"], d.W1, d.W3, d.W2,
                        o["y"], d.ws)
    moe.moe_combine(cfg, o["y"], o["inv_perm"], o["out"])
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(d.ws, raise_on_error=False) == 0
    assert o["counts"].cpu().tolist() == rows
    D = O.dispatch(idx, E, None)
    y = O.experts_forward(p.x, p.gamma, r.cpu().numpy().astype(np.float64), idx, D["kept"], p.W1, p.W3,
                          p.W2, O.expert_offsets(p.widths))
    ref = O.combine(y, gate.cpu().numpy().astype(np.float64), D["kept"])
    H.check_rows(H.bf16_dev_to_f64(o["out"]), ref, "out")


def test_training_step_and_mx_forward_capture_into_cuda_graphs():
    """The training forward + backward and the MXFP8 forward are stream-ordered
    too: captured once, replayed, they reproduce the eager results bit for bit."""
    w = mw.WORKLOADS["variable_size"].with_tokens(700, name="var_graph_train")
    p = H.make_problem(w)
    cfg = H.make_cfg(p)
    d = H.Dev(p, cfg)
    T, dm, E, F = cfg.T, cfg.d_model, cfg.E, cfg.F
    dout = torch.randn((T, dm), generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).cuda()
    f32 = dict(dtype=torch.float32, device="cuda")

    def grads():
        return [torch.zeros((T, dm), **f32), torch.zeros((dm,), **f32), torch.zeros((dm, E), **f32),
                torch.zeros((E,), **f32), torch.zeros((dm, F), **f32), torch.zeros((dm, F), **f32),
                torch.zeros((F, dm), **f32)]

    tws = moe.alloc_train_workspace(cfg)
    out_e, G_e = torch.empty((T, dm), dtype=torch.bfloat16, device="cuda"), grads()
    moe.moe_layer_fwd_train(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out_e, tws)
    moe.moe_layer_bwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, dout, *G_e, tws)
    wq = moe.alloc_mx_weights(cfg, d.W1, d.W3, d.W2)
    mws = moe.alloc_mx_workspace(cfg)
    mx_e = torch.empty((T, dm), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_fwd_mx(cfg, d.x, d.gamma, d.Wr, d.bias, wq, mx_e, mws)
    torch.cuda.synchronize()
    out_g, G_g = torch.zeros_like(out_e), grads()
    mx_g = torch.zeros_like(mx_e)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.moe_layer_fwd_train(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out_g, tws)
        moe.moe_layer_bwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, dout, *G_g, tws)
        moe.moe_layer_fwd_mx(cfg, d.x, d.gamma, d.Wr, d.bias, wq, mx_g, mws)
    for _ in range(2):
        for t in [out_g, mx_g] + G_g:
            t.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out_g, out_e) and torch.equal(mx_g, mx_e)
        for a, b in zip(G_g, G_e):
            assert torch.equal(a, b)
    assert moe.moe_get_device_error(tws, raise_on_error=False) == 0
    assert moe.moe_get_device_error(mws, raise_on_error=False) == 0
    del g


def test_empty_batch_for_training_mx_and_host_calls():
    """T = 0: nothing is launched except the zeroing of every parameter
    gradient; the MX and host-buffer calls are no-ops."""
    w = mw.WORKLOADS["tiny"].with_tokens(0, name="tiny0")
    widths = moe.ffn_offsets_from_sizes(w.expert_sizes)
    cfg = moe.MoEConfig(T=0, d_model=w.d_model, E=w.E, k=w.k, ffn_offsets=widths, eps=w.eps)
    dm, E, F = cfg.d_model, cfg.E, cfg.F
    bf = dict(dtype=torch.bfloat16, device="cuda")
    x = torch.empty((0, dm), **bf)
    gamma, Wr = torch.ones((dm,), **bf), torch.zeros((dm, E), **bf)
    W1, W3, W2 = torch.zeros((dm, F), **bf), torch.zeros((dm, F), **bf), torch.zeros((F, dm), **bf)
    f32 = dict(dtype=torch.float32, device="cuda")
    G = [torch.empty((0, dm), **f32), torch.full((dm,), 7.0, **f32), torch.full((dm, E), 7.0, **f32),
         torch.full((E,), 7.0, **f32), torch.full((dm, F), 7.0, **f32), torch.full((dm, F), 7.0, **f32),
         torch.full((F, dm), 7.0, **f32)]
    tws = moe.alloc_train_workspace(cfg)
    moe.moe_layer_fwd_train(cfg, x, gamma, Wr, None, W1, W3, W2, torch.empty((0, dm), **bf), tws)
    moe.moe_layer_bwd(cfg, x, gamma, Wr, None, W1, W3, W2, torch.empty((0, dm), **bf), *G, tws)
    wq = moe.alloc_mx_weights(cfg, W1, W3, W2)
    moe.moe_layer_fwd_mx(cfg, x, gamma, Wr, None, wq, torch.empty((0, dm), **bf), moe.alloc_mx_workspace(cfg))
    moe.moe_layer_fwd_host(cfg, torch.empty((0, dm), dtype=torch.bfloat16), gamma, Wr, None, W1, W3, W2,
                           torch.empty((0, dm), dtype=torch.bfloat16), moe.alloc_host_workspace(cfg))
    torch.cuda.synchronize()
    for t in G[1:]:
        assert int(torch.count_nonzero(t).item()) == 0
