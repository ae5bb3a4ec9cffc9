"""GPU parity of the MXFP8 expert path against the MX oracle.

Bit-exact where both sides quantise the same values: the weights (bf16 in)
and x*gamma (the product of two bf16 values is exact in fp32), codes and
scales.  The layer output is compared with the MX oracle on the GPU's own
routing; H is requantised from fp32 (GPU) vs fp64 (oracle) accumulators, so
an element near a rounding boundary can land one E4M3 step apart: the bar is
the forward's per-token normwise 2e-2 and mean-absolute 1e-3.
"""
import numpy as np
import pytest
import torch

import moe_workloads as mw
import sparse_mixture_experts_rms_b200 as moe
from oracle import moe_oracle as O
from oracle import moe_oracle_mx as M
from tests import _harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from sparse_mixture_experts_rms_b200 import build
    build.build()
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def e4m3(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.float64)


def sf_offset(r, k, K):
    r, k = np.asarray(r, dtype=np.int64), np.asarray(k, dtype=np.int64)
    return ((r // 128) * (K // 128) + k // 128) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + (k % 128) // 32


def run_mx(w, bias=None, problem=None):
    p = H.make_problem(w) if problem is None else problem
    if bias is not None:
        p.bias = np.asarray(bias, dtype=np.float32)
    cfg = H.make_cfg(p)
    d = H.Dev(p, cfg)
    wq = moe.alloc_mx_weights(cfg, d.W1, d.W3, d.W2)
    ws = moe.alloc_mx_workspace(cfg)
    out = torch.full((w.T, w.d_model), float("nan"), dtype=torch.bfloat16, device="cuda")
    moe.moe_layer_fwd_mx(cfg, d.x, d.gamma, d.Wr, d.bias, wq, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_device_error(ws, raise_on_error=False) == 0
    return p, cfg, d, wq, ws, out


SMALL = mw.Workload("mx_var", T=700, d_model=256, E=4, k=2,
                    expert_sizes=((1, 128), (1, 384), (1, 256), (1, 512)))
SMALL8 = mw.Workload("mx_degenerate", T=300, d_model=256, E=8, k=2, expert_sizes=((8, 128),))


def test_weight_codes_and_scales_are_bit_exact():
    p, cfg, d, wq, ws, out = run_mx(SMALL)
    dm, F = cfg.d_model, cfg.F
    c1, s1 = M.mx_quantize(O.widen_bf16(p.W1), axis=0)      # [d, F], [d/32, F]
    c3, s3 = M.mx_quantize(O.widen_bf16(p.W3), axis=0)
    c2, s2 = M.mx_quantize(O.widen_bf16(p.W2), axis=0)      # [F, d], [F/32, d]
    np.testing.assert_array_equal(e4m3(moe.mx_part_view(cfg, wq, None, "W1")).T, c1)
    np.testing.assert_array_equal(e4m3(moe.mx_part_view(cfg, wq, None, "W3")).T, c3)
    np.testing.assert_array_equal(e4m3(moe.mx_part_view(cfg, wq, None, "W2")).T, c2)
    n = np.arange(F)[:, None]
    k = (np.arange(dm // 32) * 32)[None, :]
    for name, s in (("SF1", s1), ("SF3", s3)):
        sf = moe.mx_part_view(cfg, wq, None, name).cpu().numpy().astype(np.int64) - 127
        np.testing.assert_array_equal(sf[sf_offset(n, k, dm)], s.T)
    sf2 = moe.mx_part_view(cfg, wq, None, "SF2").cpu().numpy().astype(np.int64) - 127
    c = np.arange(dm)[:, None]
    f = (np.arange(F // 32) * 32)[None, :]
    np.testing.assert_array_equal(sf2[sf_offset(c, f, F)], s2.T)


@pytest.mark.parametrize("degenerate", [False, True], ids=["random", "degenerate_rows"])
def test_activation_codes_and_scales_are_bit_exact(degenerate):
    """With degenerate rows, zero blocks get scale byte 0 (2^-127) and zero codes."""
    p, cfg, d, wq, ws, out = run_mx(SMALL8, problem=H.degenerate_problem(SMALL8)) if degenerate else run_mx(SMALL)
    perm = moe.mx_part_view(cfg, wq, ws, "PERM").cpu().numpy()
    offs = moe.mx_part_view(cfg, wq, ws, "OFFSETS").cpu().numpy()
    assert np.all(offs % 128 == 0)
    rows = np.arange(offs[-1])
    x8 = e4m3(moe.mx_part_view(cfg, wq, ws, "X8"))[: offs[-1]]
    xsf = moe.mx_part_view(cfg, wq, ws, "XSF").cpu().numpy().astype(np.int64)
    live = perm[: offs[-1]] >= 0
    t = perm[: offs[-1]][live] // cfg.k
    xg = O.widen_bf16(p.x)[t] * O.widen_bf16(p.gamma)[None, :]
    codes, se = M.mx_quantize(xg, axis=1)
    np.testing.assert_array_equal(x8[live], codes)
    assert np.all(x8[~live] == 0)
    r = rows[live][:, None]
    kk = (np.arange(cfg.d_model // 32) * 32)[None, :]
    np.testing.assert_array_equal(xsf[sf_offset(r, kk, cfg.d_model)] - 127, se)


def _check_layer(p, cfg, d, wq, ws, out):
    idx = moe.mx_part_view(cfg, wq, ws, "IDX").cpu().numpy()
    w = p.w
    ref = M.moe_layer_mx(p.x, p.gamma, p.Wr, p.bias, p.W1, p.W3, p.W2, p.widths, w.k, w.eps,
                         w.capacity_factor, idx_override=idx)
    got = H.bf16_dev_to_f64(out)
    H.check_rows(got, ref["out"], "mx out")
    exact = O.moe_layer(p.x, p.gamma, p.Wr, p.bias, p.W1, p.W3, p.W2, p.widths, w.k, w.eps,
                        w.capacity_factor, idx_override=idx)["out"]
    rel_mx = np.linalg.norm(got - ref["out"]) / np.linalg.norm(ref["out"])
    rel_exact = np.linalg.norm(got - exact) / np.linalg.norm(exact)
    print(w.name, f"vs MX oracle {rel_mx:.2e}  vs exact layer {rel_exact:.2e}")


@pytest.mark.parametrize("w", [mw.WORKLOADS["tiny"], SMALL,
                               mw.WORKLOADS["variable_size"].with_tokens(1500, name="mx_var1500")],
                         ids=lambda w: w.name)
def test_layer_matches_mx_oracle(w):
    _check_layer(*run_mx(w))


def test_layer_with_capacity_and_an_empty_expert():
    w = mw.Workload("mx_cap", T=600, d_model=256, E=4, k=1, expert_sizes=((4, 512),), capacity_factor=1.0)
    p, cfg, d, wq, ws, out = run_mx(w, bias=[0.5, 0.0, -60.0, 0.2])
    _check_layer(p, cfg, d, wq, ws, out)


def test_layer_fine_grained_many_experts():
    """E = 64 experts of width 128, top-8: 64 row segments padded to 128 rows."""
    w = mw.Workload("mx_fine", T=512, d_model=256, E=64, k=8, expert_sizes=((64, 128),), bias="normal")
    _check_layer(*run_mx(w))


def test_layer_every_expert_chosen():
    """k = E: every token visits every expert."""
    w = mw.Workload("mx_kE", T=200, d_model=128, E=4, k=4, expert_sizes=((4, 256),))
    _check_layer(*run_mx(w))


def test_layer_degenerate_rows():
    """Zero rows, rows scaled by 2^12 and 2^-12, tied router columns: the layer
    against the MX oracle, zero rows exactly zero."""
    p, cfg, d, wq, ws, out = run_mx(SMALL8, problem=H.degenerate_problem(SMALL8))
    _check_layer(p, cfg, d, wq, ws, out)
    assert int(out[0:16].abs().max().item()) == 0
