"""moe_dispatch_noalloc agrees with moe_dispatch, call after call.

Some callers of this library cannot allocate device memory: an inference
engine that hands a plugin only its input and output buffers, or a runtime
that forbids cudaMalloc once it is serving (the call synchronises the device
and can fail under memory pressure).  They cannot supply the workspace that
moe_dispatch uses for its per-tile count vectors, so moe_dispatch_noalloc keeps
that scratch in a fixed array inside the library.  This test calls it through
the C ABI twice in a row, on two different problems (so the second call finds
the first call's counts still in the array), and compares every output with
moe_dispatch's on the same inputs.  Dispatch results are integers and an
exact copy of bf16(x * gamma), so the comparison is bit-exact, as in the
other dispatch tests.
"""
import numpy as np
import pytest
import torch

import moe_workloads as mw
import sparse_mixture_experts_rms_b200 as moe

pytestmark = pytest.mark.gpu


def _outputs(cfg):
    mk = max(moe.moe_max_kept(cfg), 1)
    return {"counts": torch.full((cfg.E,), -1, dtype=torch.int32, device="cuda"),
            "offsets": torch.full((cfg.E + 1,), -1, dtype=torch.int32, device="cuda"),
            "perm": torch.full((mk,), -1, dtype=torch.int32, device="cuda"),
            "inv_perm": torch.full((cfg.T * cfg.k,), -2, dtype=torch.int32, device="cuda"),
            "x_perm": torch.zeros((mk, cfg.d_model), dtype=torch.bfloat16, device="cuda")}


@pytest.mark.parametrize("dummy", [0])
def test_noalloc_dispatch_matches_workspace_dispatch(dummy):
    from sparse_mixture_experts_rms_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    problems = [  # (T, d, E, k, capacity or None, skew, seed)
        (3001, 256, 64, 8, None, 1.5, 11),
        (1200, 128, 16, 1, 40, 2.0, 12),
    ]
    for T, d, E, k, C, skew, seed in problems:
        idx = torch.from_numpy(mw.random_routing(T, E, k, seed=seed, skew=skew)).cuda()
        cf = 0.0 if C is None else (C + 0.5) * E / (T * k)
        cfg = moe.MoEConfig(T=T, d_model=d, E=E, k=k, ffn_offsets=[128 * i for i in range(E + 1)],
                            capacity_factor=cf)
        g = torch.Generator().manual_seed(seed)
        x = torch.randn(T, d, generator=g).to(torch.bfloat16).cuda()
        gamma = (1 + 0.1 * torch.randn(d, generator=g)).to(torch.bfloat16).cuda()

        ref = _outputs(cfg)
        ws = moe.alloc_workspace(cfg)
        moe.moe_dispatch(cfg, idx, x, gamma, ref["counts"], ref["offsets"], ref["perm"],
                         ref["inv_perm"], ref["x_perm"], ws)
        got = _outputs(cfg)
        moe.moe_dispatch_noalloc(cfg, idx, x, gamma, got["counts"], got["offsets"], got["perm"],
                                 got["inv_perm"], got["x_perm"])
        torch.cuda.synchronize()
        assert moe.moe_get_device_error(ws, raise_on_error=False) == 0
        n = int(ref["offsets"][-1].item())
        assert int(got["counts"].sum().item()) == T * k
        for key in ("counts", "offsets", "inv_perm"):
            assert torch.equal(got[key], ref[key]), key
        assert torch.equal(got["perm"][:n], ref["perm"][:n])
        assert torch.equal(got["x_perm"][:n], ref["x_perm"][:n])
