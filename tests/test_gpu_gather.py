"""moe_layer_fwd_gather: the row gather fused into GEMM 1's A-operand load.

The router writes xg = bf16(x * gamma) in token order and GEMM 1 gathers its A
rows from it by the permutation with four-row TMA gathers, instead of reading
the permuted copy the dispatch writes for moe_layer_fwd.  The rows are the
same bf16 values and the MMAs run in the same order, so the output must be
bit-identical to moe_layer_fwd (whose own parity with the oracle is checked
in test_gpu_layer.py); routing outputs too.  Small ragged cases (T not a
multiple of 128, mixed widths, tiles past the last kept row, capacity drops,
k = 1 and k = E) and the full-size workloads.
"""
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


W = mw.Workload
CASES = {
    "tiny": mw.WORKLOADS["tiny"],
    "ragged_mixed_widths": W("ragged_mixed_widths", T=200, d_model=256, E=4, k=2,
                             expert_sizes=((1, 128), (1, 384), (1, 256), (1, 100))),
    "single_expert": W("single_expert", T=130, d_model=128, E=1, k=1, expert_sizes=((1, 256),)),
    "all_experts": W("all_experts", T=96, d_model=128, E=4, k=4, expert_sizes=((4, 128),)),
    "capacity_one": W("capacity_one", T=256, d_model=128, E=8, k=2, expert_sizes=((8, 128),),
                      capacity_factor=1.0 / 64, bias="zipf"),
    "multi_tile": W("multi_tile", T=1000, d_model=384, E=3, k=2, expert_sizes=((1, 512), (2, 256)),
                    bias="normal"),
    "switch_small": W("switch_small", T=700, d_model=256, E=16, k=1, expert_sizes=((16, 256),),
                      capacity_factor=1.25, bias="zipf"),
    "wide_d": W("wide_d", T=384, d_model=1024, E=4, k=2, expert_sizes=((4, 256),)),
}


def _both(w):
    p = H.make_problem(w)
    cfg = H.make_cfg(p)
    d = H.Dev(p, cfg)
    res = []
    for gather in (False, True):
        o = {"out": torch.full((w.T, w.d_model), 7.0, dtype=torch.bfloat16, device="cuda"),
             "idx": torch.empty((w.T, w.k), dtype=torch.int32, device="cuda"),
             "gate": torch.empty((w.T, w.k), dtype=torch.float32, device="cuda"),
             "r": torch.empty((w.T,), dtype=torch.float32, device="cuda"),
             "counts": torch.empty((w.E,), dtype=torch.int32, device="cuda")}
        moe.moe_layer_fwd(cfg, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, o["out"], d.ws,
                          expert_idx=o["idx"], gate=o["gate"], r=o["r"], counts=o["counts"], gather=gather)
        torch.cuda.synchronize()
        assert moe.moe_get_device_error(d.ws, raise_on_error=False) == 0
        res.append(o)
    return res


@pytest.mark.parametrize("name", sorted(CASES))
def test_gather_layer_is_bit_identical_small(name):
    a, b = _both(CASES[name])
    for key in ("idx", "gate", "r", "counts"):
        assert torch.equal(a[key], b[key]), key
    assert torch.equal(a["out"], b["out"]), "gathered A rows give a different layer output"


@pytest.mark.parametrize("name", ["switch_capacity", "variable_size", "fine_grained", "mixtral"])
def test_gather_layer_is_bit_identical_full_size(name):
    a, b = _both(mw.WORKLOADS[name])
    assert torch.equal(a["counts"], b["counts"])
    assert torch.equal(a["out"], b["out"]), "gathered A rows give a different layer output"
