"""Stream ordering of the layer's launches.

Consecutive kernels of the layer are launched with programmatic stream
serialization: a kernel may start while the one before drains, and waits
(griddepcontrol.wait) before it touches global memory.  These tests put a
torch kernel that rewrites a stage's input immediately before the stage on
the same stream, so a stage that read its input before the kernel before it
had finished would see the old contents.  They also check the top-1 path,
which writes kept rows straight into the output after a memset clears the
rows of dropped tokens, over an output buffer full of a non-zero pattern.
"""
import numpy as np
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


def _problem(w):
    p = H.make_problem(w)
    cfg = H.make_cfg(p)
    return p, cfg, H.Dev(p, cfg)


def test_top1_capacity_clears_dropped_rows_over_a_filled_output():
    # Switch-like: top-1, capacity 1.25, Zipf-skewed router, so many tokens are dropped
    w = mw.Workload("top1_fill", T=700, d_model=256, E=16, k=1, expert_sizes=((16, 256),),
                    capacity_factor=1.25, bias="zipf")
    p, cfg, d = _problem(w)
    staged = H.run_staged(d)                      # combine path: dropped tokens' rows are zero
    kept_tok = staged["inv_perm"].view(w.T, w.k).cpu().numpy().max(axis=1) >= 0
    assert (~kept_tok).sum() > 0, "the case must drop tokens"
    out = torch.full((w.T, w.d_model), 1.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_fwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out, d.ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(d.ws, raise_on_error=False) == 0
    assert torch.equal(out, staged["out"]), "direct top-1 write differs from the combine path"
    dropped = torch.from_numpy(~kept_tok).cuda()
    assert int(out[dropped].abs().max().item()) == 0


def test_each_stage_sees_the_kernel_just_before_it():
    w = mw.Workload("ordering", T=1000, d_model=384, E=3, k=2, expert_sizes=((1, 512), (2, 256)))
    p, cfg, d = _problem(w)
    ref = H.run_staged(d)
    s = torch.cuda.current_stream()
    n = int(ref["offsets"][-1].item())

    # up + down: x_perm rewritten by a torch kernel right before the expert GEMMs
    xp = torch.zeros_like(ref["x_perm"])
    y = torch.zeros_like(ref["y"])
    for _ in range(3):
        xp.zero_()
        xp.add_(ref["x_perm"])                    # the kernel just before the up GEMM
        moe.moe_experts_fwd(cfg, xp, ref["r"], ref["gate"], ref["perm"], ref["offsets"], d.W1, d.W3, d.W2,
                            y, d.ws, stream=s)
        torch.cuda.synchronize()
        assert torch.equal(y[:n], ref["y"][:n]), "the up GEMM read x_perm before it was written"
        y.fill_(3.0)

    # combine: y rewritten by a torch kernel right before the combine
    yb = torch.zeros_like(ref["y"])
    out = torch.empty_like(ref["out"])
    for _ in range(3):
        yb.zero_()
        yb.add_(ref["y"])
        moe.moe_combine(cfg, yb, ref["inv_perm"], out, stream=s)
        torch.cuda.synchronize()
        assert torch.equal(out, ref["out"]), "the combine read y before it was written"

    # the whole layer, twice in a row on one stream with x changed in between
    x2 = d.x.clone()
    out_a = torch.empty_like(ref["out"])
    moe.moe_layer_fwd(cfg, x2, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out_a, d.ws, stream=s)
    x2.mul_(-1.0)                                 # exact in bf16: the next layer call sees -x
    out_b = torch.empty_like(out_a)
    moe.moe_layer_fwd(cfg, x2, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out_b, d.ws, stream=s)
    x3 = -d.x
    out_c = torch.empty_like(out_a)
    torch.cuda.synchronize()
    moe.moe_layer_fwd(cfg, x3, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, out_c, d.ws, stream=s)
    torch.cuda.synchronize()
    assert torch.equal(out_a, ref["out"])
    assert torch.equal(out_b, out_c), "a layer call read x before the kernel before it rewrote it"
    assert moe.moe_get_device_error(d.ws, raise_on_error=False) == 0
