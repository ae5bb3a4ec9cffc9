"""moe_dispatch_noalloc against the oracle and against moe_dispatch, call after call.

Some callers of this library cannot allocate device memory: an inference
engine that hands a plugin only its input and output buffers, or a runtime
that forbids cudaMalloc once it is serving (the call synchronises the device
and can fail under memory pressure).  They cannot supply the workspace that
moe_dispatch uses for its per-tile count vectors, so moe_dispatch_noalloc keeps
that scratch in a fixed array inside the library.  This test calls it through
the C ABI several times in a row on different problems (so each call finds the
previous call's counts still in the array): the counts, offsets, perm and
inv_perm must equal the oracle's dispatch of the same expert ids bit for bit
(OmniMoE summary, section 2.2 ordering; MoE glossary, "Expert Capacity"),
x_perm must equal bf16(x * gamma) of the permuted tokens exactly, and every
output must equal moe_dispatch's.  A call with expert ids outside [0, E) drops
exactly those assignments, and the valid call after it is exact again.
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


def _outputs(cfg):
    mk = max(moe.moe_max_kept(cfg), 1)
    return {"counts": torch.full((cfg.E,), -1, dtype=torch.int32, device="cuda"),
            "offsets": torch.full((cfg.E + 1,), -1, dtype=torch.int32, device="cuda"),
            "perm": torch.full((mk,), -1, dtype=torch.int32, device="cuda"),
            "inv_perm": torch.full((cfg.T * cfg.k,), -2, dtype=torch.int32, device="cuda"),
            "x_perm": torch.zeros((mk, cfg.d_model), dtype=torch.bfloat16, device="cuda")}


def _problem(T, d, E, k, C, skew, seed):
    idx = mw.random_routing(T, E, k, seed=seed, skew=skew)
    cf = 0.0 if C is None else (C + 0.5) * E / (T * k)   # floor gives C
    cfg = moe.MoEConfig(T=T, d_model=d, E=E, k=k, ffn_offsets=[128 * i for i in range(E + 1)],
                        capacity_factor=cf)
    assert moe.moe_capacity(cfg) == (-1 if C is None else C)
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g).to(torch.bfloat16)
    gamma = (1 + 0.1 * torch.randn(d, generator=g)).to(torch.bfloat16)
    return idx, cfg, x, gamma


def _noalloc(cfg, idx, x, gamma):
    got = _outputs(cfg)
    moe.moe_dispatch_noalloc(cfg, torch.from_numpy(idx).cuda(), x.cuda(), gamma.cuda(), got["counts"],
                             got["offsets"], got["perm"], got["inv_perm"], got["x_perm"])
    torch.cuda.synchronize()
    return got


def _check_against_oracle(cfg, idx, x, gamma, C, got):
    g = {k_: v.cpu().numpy() for k_, v in got.items() if v.dtype != torch.bfloat16}
    D = H.check_dispatch(idx, cfg.E, C, g)   # the oracle's dispatch of the same ids, bit-exact
    n = D["n_kept"]
    xg = (x.float() * gamma.float()).to(torch.bfloat16)   # on the host: bf16 x bf16 is exact in fp32
    ref = xg[torch.from_numpy(D["perm"] // cfg.k)]
    assert torch.equal(got["x_perm"][:n].cpu(), ref)
    return n


@pytest.mark.parametrize("dummy", [0])
def test_noalloc_dispatch_matches_oracle_and_workspace_dispatch(dummy):
    problems = [  # (T, d, E, k, capacity or None, skew, seed)
        (3001, 256, 64, 8, None, 1.5, 11),
        (1200, 128, 16, 1, 40, 2.0, 12),
        (2048, 128, 8, 2, None, 0.0, 13),
    ]
    for T, d, E, k, C, skew, seed in problems:
        idx, cfg, x, gamma = _problem(T, d, E, k, C, skew, seed)
        got = _noalloc(cfg, idx, x, gamma)
        n = _check_against_oracle(cfg, idx, x, gamma, C, got)
        assert int(got["counts"].sum().item()) == T * k
        # the workspace dispatch gives the same bits
        ref = _outputs(cfg)
        ws = moe.alloc_workspace(cfg)
        moe.moe_dispatch(cfg, torch.from_numpy(idx).cuda(), x.cuda(), gamma.cuda(), ref["counts"],
                         ref["offsets"], ref["perm"], ref["inv_perm"], ref["x_perm"], ws)
        torch.cuda.synchronize()
        assert moe.moe_get_device_error(ws, raise_on_error=False) == 0
        for key in ("counts", "offsets", "inv_perm"):
            assert torch.equal(got[key], ref[key]), key
        assert torch.equal(got["perm"][:n], ref["perm"][:n])
        assert torch.equal(got["x_perm"][:n], ref["x_perm"][:n])


def test_noalloc_dispatch_drops_out_of_range_ids_then_recovers():
    T, d, E, k = 700, 128, 8, 2
    idx, cfg, x, gamma = _problem(T, d, E, k, None, 0.5, 21)
    bad = idx.copy()
    bad[123, 1] = E       # one past the last expert
    bad[400, 0] = -1
    got = _noalloc(cfg, bad, x, gamma)
    inv = got["inv_perm"].cpu().numpy()
    assert inv[123 * k + 1] == -1 and inv[400 * k + 0] == -1
    assert int(got["counts"].sum().item()) == T * k - 2
    # the valid assignments are dispatched as the oracle dispatches them without the two bad ones
    valid = np.ones(T * k, dtype=bool)
    valid[[123 * k + 1, 400 * k]] = False
    assert np.all(inv[valid] >= 0)
    assert np.array_equal(np.sort(inv[valid]), np.arange(T * k - 2))
    # the next valid call on the same array is exact again
    got = _noalloc(cfg, idx, x, gamma)
    _check_against_oracle(cfg, idx, x, gamma, None, got)
    assert int(got["counts"].sum().item()) == T * k
