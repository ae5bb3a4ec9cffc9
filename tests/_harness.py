"""Helpers for the GPU parity tests: seeded inputs on the device, calls through
the C ABI (staged or fused), and the comparisons against the CPU oracle."""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Dict, Optional

import numpy as np
import torch

import moe_workloads as mw
import sparse_mixture_experts_rms_b200 as moe
from oracle import moe_oracle as O

# Tolerances.  Gates and logits come from fp32 logits on both sides (the GPU
# sums exact bf16 products in fp64 chunks and rounds once), so they agree to
# a few fp32 ulps; tokens whose k-th and (k+1)-th oracle logits are closer
# than TIE_MARGIN may take the other expert and are left out of the routing
# comparison.  The layer output passes through bf16 operands and a bf16 H on
# the GPU, so it is compared normwise per token and by its mean absolute error.
GATE_ATOL = 1e-5          # gates: absolute
LOGIT_ATOL = 1e-5         # router logits: absolute (also the near-tie margin)
TIE_MARGIN = 1e-5         # k-th vs (k+1)-th oracle fp32 logit
ROW_REL = 2e-2            # per-token normwise relative error of the layer output
MEAN_ABS = 1e-3           # mean absolute error of the layer output
# The 1e-3 mean-absolute bound is stated for the five reference workloads,
# whose outputs have mean magnitude 0.05-0.21.  bf16 quantisation error
# (inputs x*gamma and H of the tensor-core GEMMs, stored outputs) grows in
# proportion to the magnitude, so cases with larger outputs (k = E mixtures)
# get the bound scaled by mean|out| / MAG_REF when that exceeds 1.
MAG_REF = 0.25
R_RTOL = 2e-6             # RMS statistic, relative


def bits_to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_dev_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


@dataclass
class Problem:
    w: mw.Workload
    widths: list
    x: np.ndarray
    gamma: np.ndarray
    Wr: np.ndarray
    bias: Optional[np.ndarray]
    W1: np.ndarray
    W3: np.ndarray
    W2: np.ndarray

    @property
    def cf32(self) -> float:
        return float(np.float32(self.w.capacity_factor))


def make_problem(w: mw.Workload) -> Problem:
    widths = O.expert_widths(w.expert_sizes)
    W1, W3, W2 = mw.gen_expert_weights(w, widths)
    return Problem(w, widths, mw.gen_x(w), mw.gen_gamma(w), mw.gen_router_weight(w),
                   mw.gen_router_bias(w), W1, W3, W2)


def degenerate_problem(w: mw.Workload) -> Problem:
    """The workload's problem with rows 0-15 of x zero, rows 16-31 scaled by
    2^12 and rows 32-47 by 2^-12 (exact in bf16), and router column 5 a copy
    of column 3 (needs T >= 48, E >= 6)."""
    p = make_problem(w)
    xf = O.widen_bf16(p.x).astype(np.float32)
    xf[0:16] = 0.0
    xf[16:32] *= np.float32(2.0 ** 12)
    xf[32:48] *= np.float32(2.0 ** -12)
    Wr = p.Wr.copy()
    Wr[:, 5] = Wr[:, 3]
    x = mw.f32_to_bf16_bits(xf)
    assert np.array_equal(O.widen_bf16(x).astype(np.float32), xf)
    return dataclasses.replace(p, x=x, Wr=Wr)


def make_cfg(p: Problem, renormalize: bool = False) -> moe.MoEConfig:
    w = p.w
    return moe.MoEConfig(T=w.T, d_model=w.d_model, E=w.E, k=w.k,
                         ffn_offsets=moe.ffn_offsets_from_sizes(w.expert_sizes),
                         capacity_factor=w.capacity_factor, eps=w.eps, renormalize=renormalize)


class Dev:
    """The problem's tensors on the device plus a workspace."""

    def __init__(self, p: Problem, cfg: moe.MoEConfig):
        self.p, self.cfg = p, cfg
        self.x = bits_to_dev(p.x)
        self.gamma = bits_to_dev(p.gamma)
        self.Wr = bits_to_dev(p.Wr)
        self.bias = None if p.bias is None else torch.from_numpy(p.bias).cuda()
        self.W1 = bits_to_dev(p.W1)
        self.W3 = bits_to_dev(p.W3)
        self.W2 = bits_to_dev(p.W2)
        self.ws = moe.alloc_workspace(cfg)


def run_staged(d: Dev) -> Dict[str, torch.Tensor]:
    c = d.cfg
    T, dm, E, k = c.T, c.d_model, c.E, c.k
    mk = max(moe.moe_max_kept(c), 1)
    o = {
        "idx": torch.empty((T, k), dtype=torch.int32, device="cuda"),
        "gate": torch.empty((T, k), dtype=torch.float32, device="cuda"),
        "r": torch.empty((T,), dtype=torch.float32, device="cuda"),
        "logits": torch.empty((T, E), dtype=torch.float32, device="cuda"),
        "counts": torch.empty((E,), dtype=torch.int32, device="cuda"),
        "offsets": torch.empty((E + 1,), dtype=torch.int32, device="cuda"),
        "perm": torch.full((mk,), -7, dtype=torch.int32, device="cuda"),
        "inv_perm": torch.empty((T * k,), dtype=torch.int32, device="cuda"),
        "x_perm": torch.zeros((mk, dm), dtype=torch.bfloat16, device="cuda"),
        "y": torch.zeros((mk, dm), dtype=torch.bfloat16, device="cuda"),
        "out": torch.empty((T, dm), dtype=torch.bfloat16, device="cuda"),
        "prob_mean": torch.empty((E,), dtype=torch.float32, device="cuda"),
        "stats": torch.empty((4,), dtype=torch.float32, device="cuda"),
    }
    moe.moe_route(c, d.x, d.gamma, d.Wr, d.bias, o["idx"], o["gate"], o["r"], o["logits"], d.ws,
                  prob_mean=o["prob_mean"])
    moe.moe_dispatch(c, o["idx"], d.x, d.gamma, o["counts"], o["offsets"], o["perm"], o["inv_perm"],
                     o["x_perm"], d.ws)
    moe.moe_experts_fwd(c, o["x_perm"], o["r"], o["gate"], o["perm"], o["offsets"], d.W1, d.W3, d.W2,
                        o["y"], d.ws)
    moe.moe_combine(c, o["y"], o["inv_perm"], o["out"])
    moe.moe_router_stats(c, o["prob_mean"], o["counts"], o["offsets"], o["stats"])
    torch.cuda.synchronize()
    return o


def run_fused(d: Dev) -> Dict[str, torch.Tensor]:
    c = d.cfg
    o = {
        "idx": torch.empty((c.T, c.k), dtype=torch.int32, device="cuda"),
        "gate": torch.empty((c.T, c.k), dtype=torch.float32, device="cuda"),
        "r": torch.empty((c.T,), dtype=torch.float32, device="cuda"),
        "counts": torch.empty((c.E,), dtype=torch.int32, device="cuda"),
        "out": torch.empty((c.T, c.d_model), dtype=torch.bfloat16, device="cuda"),
        "stats": torch.empty((4,), dtype=torch.float32, device="cuda"),
    }
    moe.moe_layer_fwd(c, d.x, d.gamma, d.Wr, d.bias, d.W1, d.W3, d.W2, o["out"], d.ws,
                      expert_idx=o["idx"], gate=o["gate"], r=o["r"], counts=o["counts"],
                      stats=o["stats"])
    torch.cuda.synchronize()
    return o


def oracle_route(p: Problem, renormalize: bool = False) -> Dict[str, np.ndarray]:
    x = O.widen_bf16(p.x)
    return O.route(x, O.widen_bf16(p.gamma), O.widen_bf16(p.Wr), p.bias, p.w.k, p.w.eps, renormalize)


def check_route(p: Problem, R: Dict[str, np.ndarray], g_idx, g_gate, g_r, g_logits=None):
    """idx bit-exact outside near ties; gates, r, logits within tolerance."""
    k = p.w.k
    margin = O.topk_margin(R["logits"], k)
    ok_tok = margin >= TIE_MARGIN
    np.testing.assert_allclose(g_r, R["r"], rtol=R_RTOL, atol=0)
    if g_logits is not None:
        np.testing.assert_allclose(g_logits, R["logits"].astype(np.float64), rtol=0, atol=LOGIT_ATOL)
    bad = np.nonzero(ok_tok & np.any(g_idx != R["idx"], axis=1))[0]
    assert bad.size == 0, f"{bad.size} tokens routed differently (margin >= {TIE_MARGIN}): {bad[:10]}"
    np.testing.assert_allclose(g_gate[ok_tok], R["gate"][ok_tok], rtol=0, atol=GATE_ATOL)
    return np.nonzero(~ok_tok)[0]


STATS_RTOL = 1e-5         # router metrics (fp32 probabilities, fp64 reductions)


def check_stats(R: Dict[str, np.ndarray], counts: np.ndarray, n_kept: int, k: int,
                g_prob_mean: Optional[np.ndarray], g_stats: np.ndarray):
    """Router metrics against the oracle on the same routing (the GPU's counts)."""
    S = O.router_stats(R["logits"], counts, n_kept, k)
    if g_prob_mean is not None:
        np.testing.assert_allclose(g_prob_mean, S["prob_mean"], rtol=STATS_RTOL, atol=1e-7)
    exp = np.array([S["aux_loss"], S["cv2_prob"], S["cv2_load"], S["dropped_frac"]])
    np.testing.assert_allclose(g_stats, exp, rtol=STATS_RTOL, atol=1e-6)


def check_dispatch(g_idx: np.ndarray, E: int, C: Optional[int], o: Dict[str, np.ndarray]):
    """Replay: the oracle's dispatch of the GPU's own routing, bit-exact."""
    D = O.dispatch(g_idx, E, C)
    assert np.array_equal(o["counts"], D["counts"])
    assert np.array_equal(o["offsets"], D["offsets"])
    n = D["n_kept"]
    assert np.array_equal(o["perm"][:n], D["perm"])
    assert np.array_equal(o["inv_perm"], D["inv_perm"])
    return D


def check_rows(g_out: np.ndarray, ref: np.ndarray, what: str = "out"):
    """Per-row normwise relative error and mean absolute error."""
    err = g_out - ref
    nref = np.linalg.norm(ref, axis=1)
    nerr = np.linalg.norm(err, axis=1)
    zero = nref == 0
    assert np.all(nerr[zero] == 0), f"{what}: rows that must be exactly zero are not"
    rel = nerr[~zero] / nref[~zero]
    worst = float(rel.max()) if rel.size else 0.0
    mae = float(np.abs(err).mean()) if err.size else 0.0
    bound = MEAN_ABS * max(1.0, float(np.abs(ref).mean()) / MAG_REF) if ref.size else MEAN_ABS
    assert worst <= ROW_REL, f"{what}: max row relative error {worst:.3e} > {ROW_REL}"
    assert mae <= bound, f"{what}: mean abs error {mae:.3e} > {bound:.3e}"
    return worst, mae


# ---- gradients (training path), compared element by element
#
# GRAD_REL is the forward's per-row normwise bar.  Mean absolute error:
# the forward's 1e-3 sits at 0.5-2 % of its workloads' mean output magnitude
# (0.05-0.21); gradients have no fixed scale, so their bar is relative:
# mean|err| <= GRAD_MEAN_REL * mean|ref| (measured normwise errors ~3.5e-3).
# dx is compared per token row; dW1, dW3, dW2 per expert slice.  Quantities
# that are sums whose terms may cancel (dbias, dWr and dgamma over tokens, dr
# over a token's assignments) are compared element by element against GRAD_REL * (|ref| + rss), rss = the root-sum-square of the
# sum's terms: the GPU's bf16 roundings of the terms' operands are
# independent from term to term, so their effect on the sum grows with the
# terms' rss, not with the (possibly cancelled) value of the sum.  Where a
# term is itself a product with a sum that may cancel (dr's terms contain
# dh = W2_e dy, a sum over d; dbias and dWr contain the softmax backward's
# dl), that factor enters the rss at the size of its own terms.
GRAD_REL = 2e-2
GRAD_MEAN_REL = 1e-2


def check_grad_rows(got: np.ndarray, ref: np.ndarray, what: str):
    """Per-row normwise relative error <= GRAD_REL (rows whose reference is
    exactly zero must be exactly zero) and mean|err| <= GRAD_MEAN_REL *
    mean|ref|.  Returns (worst row error, relative mean absolute error)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    err = got - ref
    nref = np.linalg.norm(ref, axis=1)
    nerr = np.linalg.norm(err, axis=1)
    zero = nref == 0
    assert np.all(nerr[zero] == 0), f"{what}: rows that must be exactly zero are not"
    rel = nerr[~zero] / nref[~zero]
    worst = float(rel.max()) if rel.size else 0.0
    mref = float(np.abs(ref).mean()) if ref.size else 0.0
    mae = float(np.abs(err).mean()) if err.size else 0.0
    rmae = mae / mref if mref > 0 else 0.0
    assert worst <= GRAD_REL, f"{what}: row {int(np.argmax(rel))} relative error {worst:.3e} > {GRAD_REL}"
    assert mae <= GRAD_MEAN_REL * mref, f"{what}: mean abs error {mae:.3e} > {GRAD_MEAN_REL} x {mref:.3e}"
    return worst, rmae


def check_grad_slice(got: np.ndarray, ref: np.ndarray, what: str):
    """One block (an expert's slice of a weight gradient) as a whole:
    normwise relative error <= GRAD_REL and mean|err| <= GRAD_MEAN_REL *
    mean|ref|.  Returns the normwise error."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    n = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(got - ref)) / (n if n > 0 else 1.0)
    mref = float(np.abs(ref).mean()) if ref.size else 0.0
    mae = float(np.abs(got - ref).mean()) if ref.size else 0.0
    assert rel <= GRAD_REL, f"{what}: normwise relative error {rel:.3e} > {GRAD_REL}"
    assert mae <= GRAD_MEAN_REL * mref, f"{what}: mean abs error {mae:.3e} > {GRAD_MEAN_REL} x {mref:.3e}"
    return rel


def check_sum_elems(got: np.ndarray, ref: np.ndarray, rss: np.ndarray, what: str, rel: float = GRAD_REL):
    """|got - ref| <= rel * (|ref| + rss) element by element, for sums whose
    terms have root-sum-square rss.  Returns the worst ratio of the error to
    its bound."""
    got = np.asarray(got, dtype=np.float64).reshape(-1)
    ref = np.asarray(ref, dtype=np.float64).reshape(-1)
    rss = np.asarray(rss, dtype=np.float64).reshape(-1)
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    bound = rel * (np.abs(ref) + rss)
    err = np.abs(got - ref)
    bad = np.nonzero(err > bound)[0]
    assert bad.size == 0, (f"{what}: {bad.size} elements outside the bound, first {bad[:5]}: "
                           f"got {got[bad[:3]]}, ref {ref[bad[:3]]}, bound {bound[bad[:3]]}")
    nz = bound > 0
    return float((err[nz] / bound[nz]).max()) if nz.any() else 0.0


def grad_term_rss(f: Dict[str, object], g: np.ndarray, ref: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """Root-sum-square of the terms of the backward's reductions, from the
    oracle's forward state ``f`` (moe_oracle_bwd.layer_forward), the upstream
    gradient g and the oracle's gradients ``ref``:
      dgamma_i = sum_t dxg_ti x_ti          dbias_e = sum_t dl_te
      dWr_ie = sum_t xg_ti r_t dl_te        (dl_te entering at its terms' size)
      dr_t = sum_a <du_a, s_a> + <dv_a, s3_a> + <dl_t, z_t>
    with du = dh v silu'(u), dv = dh silu(u), dh = W2_e (gate g_t) for the
    kept assignment a; dh's entries enter at |dh| plus the rss of their own d
    terms."""
    from oracle import moe_oracle_bwd as B
    g = np.asarray(g, dtype=np.float64)
    x, r, idx, gate, kept, k = f["x"], f["r"], f["idx"], f["gate"], f["kept"], f["k"]
    T = x.shape[0]
    # the router's dl_te = p_te (dp_te - <dp_t, p_t>) is itself a sum that can
    # cancel (with renormalised gates <dp, p> = 0 exactly, so an expert no token
    # chose has dl = 0 in exact arithmetic): its terms' size is
    # m_te = p_te (|dp_te| + sum_j |dp_tj| p_tj)
    dq = B.gate_backward(ref["dgate"], f["q"], f["renormalize"])
    dp = np.zeros_like(f["p"])
    np.put_along_axis(dp, idx, dq, axis=1)
    p = f["p"]
    m = p * (np.abs(dp) + (np.abs(dp) * p).sum(axis=1, keepdims=True))
    rm = r[:, None] * m
    out = {"dgamma": np.sqrt(((ref["dxg"] * x) ** 2).sum(axis=0)),
           "dbias": np.sqrt((m ** 2).sum(axis=0)),
           # dWr_ie = sum_t xg_ti r_t dl_te
           "dWr": np.sqrt((f["xg"] ** 2).T @ (rm ** 2))}
    dr2 = ((ref["dl"] * f["z"]) ** 2).sum(axis=1)
    for a in range(T * k):
        if not kept[a]:
            continue
        t, j = a // k, a % k
        e = int(idx[t, j])
        W1e, W3e, W2e = f["slices"][e]
        dy = gate[t, j] * g[t]
        dh = W2e @ dy
        dh_mag = np.abs(dh) + np.sqrt((W2e ** 2) @ (dy ** 2))
        u, v = r[t] * f["s"][a], r[t] * f["s3"][a]
        du1, dv1 = B.swiglu_backward(np.ones_like(dh), u, v)   # du, dv per unit dh
        dr2[t] += ((dh_mag * du1 * f["s"][a]) ** 2).sum() + ((dh_mag * dv1 * f["s3"][a]) ** 2).sum()
    out["dr"] = np.sqrt(dr2)
    return out


def dgate_replay(cfg, tws, g_bits: np.ndarray, toks: Optional[np.ndarray] = None):
    """dgate_a = <g_t, y_a> recomputed in float64 from the GPU's own saved
    ungated y (training workspace), for every assignment (0 where dropped),
    with the root-sum-square of each dot product's terms: checks the
    backward's dot product on the forward's stored rows.  Returns
    (values [n, k], rss [n, k])."""
    T, k, d = cfg.T, cfg.k, cfg.d_model
    inv = moe.train_saved_view(cfg, tws, "inv_perm").cpu().numpy().reshape(T, k)
    y = moe.train_saved_view(cfg, tws, "y")
    toks = np.arange(T) if toks is None else np.asarray(toks)
    g = O.widen_bf16(g_bits[toks])
    out = np.zeros((toks.size, k))
    rss = np.zeros((toks.size, k))
    for j in range(k):
        pos = inv[toks, j]
        ok = pos >= 0
        if ok.any():
            rows = y[torch.from_numpy(pos[ok].astype(np.int64)).cuda()].float().cpu().numpy().astype(np.float64)
            out[ok, j] = (g[ok] * rows).sum(axis=1)
            rss[ok, j] = np.sqrt(((g[ok] * rows) ** 2).sum(axis=1))
    return out, rss


# dgate against its replay: fp32 accumulation of d products, err ~ sqrt(d) *
# 2^-24 * rss (4e-6 at d = 4096); the bar leaves 25x.
DGATE_REPLAY_REL = 1e-4
