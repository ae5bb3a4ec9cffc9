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
