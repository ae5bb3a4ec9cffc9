"""GPU parity of every stage of the layer against the CPU oracle, through the C ABI.

Routing is compared token by token (expert ids bit-exact outside near ties of
the fp32 logits, gates to 1e-5); dispatch is compared bit-exactly in replay
mode (the oracle dispatches the GPU's own expert ids); expert outputs and the
layer output per token, normwise, against the oracle replaying the GPU's
routing.  Small cases compare every output; the full-size workloads compare
all routing and dispatch results and the outputs of a seeded token sample.
"""
import dataclasses

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


W = mw.Workload
SMALL_CASES = {
    "tiny": mw.WORKLOADS["tiny"],
    # T not a multiple of 128, mixed widths, ragged M tiles in every expert
    "ragged_mixed_widths": W("ragged_mixed_widths", T=200, d_model=256, E=4, k=2,
                             expert_sizes=((1, 128), (1, 384), (1, 256), (1, 100))),
    # E = 1, k = 1: a dense SwiGLU FFN with gate 1
    "single_expert": W("single_expert", T=130, d_model=128, E=1, k=1, expert_sizes=((1, 256),)),
    # k = E: the full softmax mixture
    "all_experts": W("all_experts", T=96, d_model=128, E=4, k=4, expert_sizes=((4, 128),)),
    # capacity 1 and a Zipf-skewed router: almost everything dropped
    "capacity_one": W("capacity_one", T=256, d_model=128, E=8, k=2, expert_sizes=((8, 128),),
                      capacity_factor=1.0 / 64, bias="zipf"),
    # capacity 0: every slot dropped, output exactly zero
    "capacity_zero": W("capacity_zero", T=64, d_model=128, E=8, k=1, expert_sizes=((8, 128),),
                       capacity_factor=1e-3),
    # several M tiles per expert, K loop longer than the smem ring, d % 256 != 0
    "multi_tile": W("multi_tile", T=1000, d_model=384, E=3, k=2, expert_sizes=((1, 512), (2, 256)),
                    bias="normal"),
    "switch_small": W("switch_small", T=700, d_model=256, E=16, k=1, expert_sizes=((16, 256),),
                      capacity_factor=1.25, bias="zipf"),
}


def _full_check(p: H.Problem, renormalize=False, fused_too=True):
    cfg = H.make_cfg(p, renormalize)
    d = H.Dev(p, cfg)
    o = H.run_staged(d)
    code = moe.moe_get_device_error(d.ws, raise_on_error=False)
    assert code == 0, f"device error word 0x{code:x}"
    g = {k: v.cpu().numpy() for k, v in o.items() if v.dtype != torch.bfloat16}
    R = H.oracle_route(p, renormalize)
    H.check_route(p, R, g["idx"], g["gate"], g["r"], g["logits"])
    C = O.capacity(p.w.T, p.w.k, p.w.E, p.cf32)
    D = H.check_dispatch(g["idx"], p.w.E, C, g)
    n = D["n_kept"]
    # x_perm rows: bf16(x * gamma) in expert-centric order (torch's RNE cast)
    xg = (O.widen_bf16(p.x) * O.widen_bf16(p.gamma)[None, :]).astype(np.float32)
    exp_xp = torch.from_numpy(xg[D["perm"] // p.w.k]).to(torch.bfloat16)
    assert torch.equal(o["x_perm"][:n].cpu(), exp_xp)
    # expert outputs, replaying the GPU routing
    gate_o = O.gates(R["logits"], g["idx"], renormalize)
    y = O.experts_forward(p.x, p.gamma, R["r"], g["idx"], D["kept"], p.W1, p.W3, p.W2,
                          O.expert_offsets(p.widths))
    if n:
        exp_y = gate_o.reshape(-1)[D["perm"]][:, None] * y[D["perm"]]
        H.check_rows(H.bf16_dev_to_f64(o["y"][:n]), exp_y, "y")
    out_ref = O.combine(y, gate_o, D["kept"])
    H.check_rows(H.bf16_dev_to_f64(o["out"]), out_ref, "out")
    H.check_stats(R, g["counts"], n, p.w.k, g["prob_mean"], g["stats"])
    if fused_too:
        f = H.run_fused(d)
        assert torch.equal(f["out"], o["out"]), "fused layer differs from the staged calls"
        assert torch.equal(f["idx"], o["idx"]) and torch.equal(f["counts"], o["counts"])
        assert torch.equal(f["stats"], o["stats"]), "fused router metrics differ from the staged ones"
        assert moe.moe_get_device_error(d.ws, raise_on_error=False) == 0
    return o, R, D


@pytest.mark.parametrize("name", sorted(SMALL_CASES))
def test_layer_small_all_outputs(name):
    _full_check(H.make_problem(SMALL_CASES[name]))


def test_layer_renormalized_gates():
    _full_check(H.make_problem(SMALL_CASES["ragged_mixed_widths"]), renormalize=True)


def test_every_token_to_one_expert():
    w = W("one_hot", T=300, d_model=128, E=6, k=1, expert_sizes=((6, 128),))
    p = H.make_problem(w)
    p = dataclasses.replace(p, bias=np.array([0, 0, 50.0, 0, 0, 0], dtype=np.float32))
    o, R, D = _full_check(p)
    assert D["counts"].tolist() == [0, 0, 300, 0, 0, 0]


def test_capacity_zero_output_is_exactly_zero():
    p = H.make_problem(SMALL_CASES["capacity_zero"])
    cfg = H.make_cfg(p)
    assert moe.moe_capacity(cfg) == 0
    o = H.run_fused(H.Dev(p, cfg))
    assert int(o["out"].abs().max().item()) == 0


@pytest.mark.parametrize("name", ["switch_capacity", "variable_size", "fine_grained", "mixtral"])
def test_layer_full_size_sampled(name):
    w = mw.WORKLOADS[name]
    p = H.make_problem(w)
    cfg = H.make_cfg(p)
    d = H.Dev(p, cfg)
    o = H.run_fused(d)
    assert moe.moe_get_device_error(d.ws, raise_on_error=False) == 0
    g_idx, g_gate, g_r = (o[k].cpu().numpy() for k in ("idx", "gate", "r"))
    R = H.oracle_route(p)
    H.check_route(p, R, g_idx, g_gate, g_r)
    C = O.capacity(w.T, w.k, w.E, p.cf32)
    D = O.dispatch(g_idx, w.E, C)
    assert np.array_equal(o["counts"].cpu().numpy(), D["counts"])
    H.check_stats(R, D["counts"], D["n_kept"], w.k, None, o["stats"].cpu().numpy())
    toks = mw.sample_tokens(w, 192)
    gate_o = O.gates(R["logits"], g_idx)
    ref = O.moe_layer_tokens(p.x[toks], toks, p.gamma, p.W1, p.W3, p.W2, p.widths,
                             g_idx, gate_o, D["kept"], w.eps)
    H.check_rows(H.bf16_dev_to_f64(o["out"][torch.from_numpy(toks).cuda()]), ref, f"{name} out")


@pytest.mark.parametrize("E,k,C,skew", [(8, 2, None, 0.0), (64, 8, None, 1.5), (16, 1, 320, 1.0),
                                        (16, 1, 1, 2.0), (64, 8, 0, 0.5), (5, 5, None, 0.0),
                                        (1, 1, None, 0.0), (64, 1, 3, 1.0)])
def test_dispatch_random_routing(E, k, C, skew):
    T, dm = 3001, 128
    idx = mw.random_routing(T, E, k, seed=E * 100 + k, skew=skew)
    cf = 0.0 if C is None else (C + 0.5) * E / (T * k)   # floor gives C
    cfg = moe.MoEConfig(T=T, d_model=dm, E=E, k=k, ffn_offsets=[128 * i for i in range(E + 1)],
                        capacity_factor=cf)
    assert moe.moe_capacity(cfg) == (-1 if C is None else C)
    rng = np.random.default_rng(1)
    x = torch.randn(T, dm).to(torch.bfloat16).cuda()
    gamma = (1 + 0.1 * torch.randn(dm)).to(torch.bfloat16).cuda()
    mk = max(moe.moe_max_kept(cfg), 1)
    ws = moe.alloc_workspace(cfg)
    o = {"counts": torch.empty(E, dtype=torch.int32, device="cuda"),
         "offsets": torch.empty(E + 1, dtype=torch.int32, device="cuda"),
         "perm": torch.empty(mk, dtype=torch.int32, device="cuda"),
         "inv_perm": torch.empty(T * k, dtype=torch.int32, device="cuda"),
         "x_perm": torch.empty(mk, dm, dtype=torch.bfloat16, device="cuda")}
    moe.moe_dispatch(cfg, torch.from_numpy(idx).cuda(), x, gamma, o["counts"], o["offsets"], o["perm"],
                     o["inv_perm"], o["x_perm"], ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws, raise_on_error=False) == 0
    g = {k_: v.cpu().numpy() for k_, v in o.items() if v.dtype != torch.bfloat16}
    D = H.check_dispatch(idx, E, C, g)
    n = D["n_kept"]
    ref = (x.float() * gamma.float()).to(torch.bfloat16)[torch.from_numpy(D["perm"] // k).cuda()]
    assert torch.equal(o["x_perm"][:n], ref)


def test_dispatch_reports_bad_expert_id():
    T, E, k, dm = 100, 4, 2, 128
    idx = mw.random_routing(T, E, k, seed=3)
    idx[17, 1] = 7   # out of range
    idx[50, 0] = -2
    cfg = moe.MoEConfig(T=T, d_model=dm, E=E, k=k, ffn_offsets=[128 * i for i in range(E + 1)])
    ws = moe.alloc_workspace(cfg)
    mk = moe.moe_max_kept(cfg)
    inv = torch.empty(T * k, dtype=torch.int32, device="cuda")
    moe.moe_dispatch(cfg, torch.from_numpy(idx).cuda(), torch.zeros(T, dm, dtype=torch.bfloat16, device="cuda"),
                     torch.ones(dm, dtype=torch.bfloat16, device="cuda"),
                     torch.empty(E, dtype=torch.int32, device="cuda"),
                     torch.empty(E + 1, dtype=torch.int32, device="cuda"),
                     torch.empty(mk, dtype=torch.int32, device="cuda"), inv,
                     torch.empty(mk, dm, dtype=torch.bfloat16, device="cuda"), ws)
    code = moe.moe_get_device_error(ws, raise_on_error=False)
    assert code & moe.MOE_DEVERR_EXPERT_ID
    inv = inv.cpu().numpy()
    assert inv[17 * k + 1] == -1 and inv[50 * k + 0] == -1
    assert moe.moe_get_device_error(ws, raise_on_error=False) == 0   # cleared by the read


def test_zero_tokens_is_a_no_op():
    cfg = moe.MoEConfig(T=0, d_model=128, E=4, k=2, ffn_offsets=[0, 128, 256, 384, 512])
    ws = moe.alloc_workspace(cfg)
    e = torch.empty(0, dtype=torch.bfloat16, device="cuda")
    out = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros(128, 512, dtype=torch.bfloat16, device="cuda")
    counts = torch.full((4,), 7, dtype=torch.int32, device="cuda")
    moe.moe_layer_fwd(cfg, e.view(0, 128), torch.ones(128, dtype=torch.bfloat16, device="cuda"),
                      torch.zeros(128, 4, dtype=torch.bfloat16, device="cuda"), None, W, W,
                      torch.zeros(512, 128, dtype=torch.bfloat16, device="cuda"), out, ws,
                      counts=counts)
    assert moe.moe_get_device_error(ws, raise_on_error=False) == 0
    assert counts.cpu().tolist() == [0, 0, 0, 0]


def test_degenerate_rows_and_tied_router_columns():
    """Inputs the method has special cases for:
    - all-zero rows: r = 1/sqrt(eps), every logit is exactly 0, so the tie rule
      picks experts 0..k-1 with gates 1/E, and the output row is exactly zero;
    - rows scaled by 2^12 and by 2^-12 (for the latter eps dominates the mean
      square, so r is close to 1/sqrt(eps) rather than the row's own scale);
    - two identical router columns (3 and 5): their logits tie bit-exactly for
      every token, and expert 5 is never taken ahead of expert 3.
    """
    w = W("degenerate", T=256, d_model=256, E=8, k=2, expert_sizes=((8, 128),))
    p = H.degenerate_problem(w)
    o, R, D = _full_check(p)
    idx, gate = o["idx"].cpu().numpy(), o["gate"].cpu().numpy()
    logits = o["logits"].cpu().numpy()
    assert np.array_equal(idx[0:16], np.tile([0, 1], (16, 1)))
    assert np.all(np.abs(gate[0:16] - 1.0 / w.E) <= 1e-7)
    assert np.all(logits[0:16] == 0.0)
    assert int(o["out"][0:16].abs().max().item()) == 0
    assert np.array_equal(logits[:, 3].view(np.uint32), logits[:, 5].view(np.uint32))
    has3, has5 = np.any(idx == 3, axis=1), np.any(idx == 5, axis=1)
    assert not np.any(has5 & ~has3), "expert 5 chosen over the tied expert 3"
    both = has3 & has5
    assert both.any() and np.all(np.argmax(idx[both] == 3, axis=1) < np.argmax(idx[both] == 5, axis=1))
    eps_rows = O.rms_stat(O.widen_bf16(p.x[32:48]), w.eps)
    assert np.all(eps_rows > 0.5 / np.sqrt(w.eps))  # the eps term dominates these rows' statistic
