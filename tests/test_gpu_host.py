"""The host-buffer layer (copies pipelined with the compute over token
chunks) gives moe_layer_fwd's output bit for bit: per-token routing, per-row
GEMM sums independent of the tile's other rows, per-token combine."""
import pytest
import torch

import moe_workloads as mw
import sparse_mixture_experts_rms_b200 as moe
from tests import _harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_rms_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _run(w, n_chunks):
    p = H.make_problem(w)
    cfg = H.make_cfg(p)
    d = H.Dev(p, cfg)
    ref = torch.empty((w.T, w.d_model), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_fwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, ref, d.ws)
    x_h = d.x.cpu().pin_memory()
    out_h = torch.full((w.T, w.d_model), float("nan"), dtype=torch.bfloat16).pin_memory()
    ws = moe.alloc_host_workspace(cfg, n_chunks)
    moe.moe_layer_fwd_host(cfg, x_h, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out_h, ws, n_chunks=n_chunks)
    torch.cuda.current_stream().synchronize()
    assert moe.moe_get_device_error(ws, raise_on_error=False) == 0
    assert torch.equal(out_h, ref.cpu()), (w.name, n_chunks)


@pytest.mark.parametrize("n_chunks", [1, 3, 4, 7])
def test_host_layer_matches_device_layer_dropless(n_chunks):
    _run(mw.WORKLOADS["variable_size"].with_tokens(1500, name="var_host"), n_chunks)


def test_host_layer_with_capacity_is_one_chunk():
    w = mw.WORKLOADS["switch_capacity"].with_tokens(1000, name="cap_host")
    assert moe.moe_host_chunks(H.make_cfg(H.make_problem(w)), 4) == 1
    _run(w, 4)


def test_host_layer_repeated_calls_reuse_the_pipeline():
    w = mw.WORKLOADS["tiny"]
    for _ in range(3):
        _run(w, 2)


def test_host_layer_tiny_batch_more_chunks_than_ramp_allows():
    _run(mw.WORKLOADS["tiny"].with_tokens(5, name="tiny5"), 4)
