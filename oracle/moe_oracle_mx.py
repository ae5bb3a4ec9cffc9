"""CPU oracle of the MXFP8 expert path -- TEST INFRASTRUCTURE ONLY.

Same rules as ``moe_oracle``: only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it; the library never does.

The CODA sparse-MoE thread (digg.com) notes that when the expert GEMMs run in
low precision, the conversions they need can sit in the epilogues of the
kernels that produce their inputs.  The format taken here is the OCP
Microscaling (MX) v1.0 MXFP8: blocks of 32 consecutive values along the GEMM's
reduction dimension share one power-of-two scale (E8M0) and each value is an
FP8 E4M3 number.  The conversion of a block V (the MX specification's
quantisation, with the element format's largest normal exponent emax = 8 for
E4M3) is:

    shared_exp = floor(log2(max_i |V_i|)) - 8        (all-zero block: -127)
    X          = 2^shared_exp                        (stored as the byte shared_exp + 127)
    P_i        = E4M3(V_i / X), round to nearest even, magnitudes above the
                 largest normal 448 clamped to 448

and the block's value is X * P_i.  The layer is the forward oracle's layer with
every expert-GEMM operand replaced by its MX value: x*gamma and W1/W3 blocked
along d, the SwiGLU output H and W2 blocked along the expert width; products
are summed exactly (float64).  The gate, r and combine are as in
``moe_oracle``.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np

from oracle import moe_oracle as O

E4M3_MAX = 448.0
E4M3_EMAX = 8           # exponent of the largest normal, 448 = 1.75 * 2^8
E4M3_MIN_NORMAL_EXP = -6
E4M3_MANTISSA_BITS = 3
MX_BLOCK = 32


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Nearest E4M3 value of each float64 in v (ties to even), saturating at
    +-448.  Normal numbers have 3 fraction bits; below 2^-6 the spacing is the
    subnormal step 2^-9."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, E4M3_MIN_NORMAL_EXP)
    step = np.exp2(e - E4M3_MANTISSA_BITS)
    q = np.round(a / step) * step           # numpy rounds halves to even
    q = np.minimum(q, E4M3_MAX)
    return np.copysign(q, v)


def mx_scale_exp(amax: np.ndarray) -> np.ndarray:
    """Shared exponent of blocks with largest magnitude amax (int64);
    -127 for an all-zero block."""
    amax = np.asarray(amax, dtype=np.float64)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(amax > 0, amax, 1.0))).astype(np.int64) - E4M3_EMAX
    e = np.where(amax > 0, e, -127)
    return np.clip(e, -127, 127)


def mx_quantize(v: np.ndarray, axis: int = -1):
    """MXFP8 quantisation along ``axis`` (its length a multiple of 32).

    Returns (codes, scale_exp): codes are the E4M3 values P_i as float64 (so a
    code compares exactly), scale_exp the int64 shared exponents with that
    axis divided by 32.
    """
    v = np.moveaxis(np.asarray(v, dtype=np.float64), axis, -1)
    n = v.shape[-1]
    if n % MX_BLOCK:
        raise ValueError("length along the blocked axis must be a multiple of 32")
    b = v.reshape(v.shape[:-1] + (n // MX_BLOCK, MX_BLOCK))
    se = mx_scale_exp(np.abs(b).max(axis=-1))
    p = e4m3_round(b / np.exp2(se)[..., None])
    codes = np.moveaxis(p.reshape(v.shape), -1, axis)
    return codes, np.moveaxis(se, -1, axis)


def mx_dequantize(codes: np.ndarray, scale_exp: np.ndarray, axis: int = -1) -> np.ndarray:
    """X * P_i: the value an MX block represents."""
    c = np.moveaxis(np.asarray(codes, dtype=np.float64), axis, -1)
    s = np.repeat(np.exp2(np.moveaxis(np.asarray(scale_exp, dtype=np.float64), axis, -1)), MX_BLOCK, axis=-1)
    return np.moveaxis(c * s, -1, axis)


def mx_value(v: np.ndarray, axis: int = -1) -> np.ndarray:
    """The MX value of v (quantise, then dequantise)."""
    c, s = mx_quantize(v, axis)
    return mx_dequantize(c, s, axis)


# --------------------------------------------------------------------------
# the layer with MXFP8 expert GEMMs
# --------------------------------------------------------------------------
def quantized_weights(W1_bits, W3_bits, W2_bits) -> Dict[str, np.ndarray]:
    """MX values of the expert weights: W1, W3 [d, F] blocked along d (their
    GEMM's reduction), W2 [F, d] blocked along F (blocks never cross experts:
    every expert width is a multiple of 128)."""
    return {"W1": mx_value(O.as_f64(W1_bits), axis=0), "W3": mx_value(O.as_f64(W3_bits), axis=0),
            "W2": mx_value(O.as_f64(W2_bits), axis=0)}


class LazyExpertWeights:
    """MX values of one expert's weight slices, quantised when first used:
    W1/W3 columns o_e..o_e+1 blocked along d, W2 rows o_e..o_e+1 blocked along
    F.  Blocks never cross an expert (every width is a multiple of 128), so a
    slice's MX value equals the slice of the whole matrix's."""

    def __init__(self, W1_bits, W3_bits, W2_bits, offs):
        self.W, self.offs, self.cache = (W1_bits, W3_bits, W2_bits), offs, {}

    def expert(self, e):
        if e not in self.cache:
            W1, W3, W2 = self.W
            o0, o1 = int(self.offs[e]), int(self.offs[e + 1])
            self.cache[e] = (mx_value(O.as_f64(W1[:, o0:o1]), axis=0), mx_value(O.as_f64(W3[:, o0:o1]), axis=0),
                             mx_value(O.as_f64(W2[o0:o1, :]), axis=0))
        return self.cache[e]


def _expert_mx(Wq, offs, e):
    if isinstance(Wq, LazyExpertWeights):
        return Wq.expert(e)
    o0, o1 = int(offs[e]), int(offs[e + 1])
    return Wq["W1"][:, o0:o1], Wq["W3"][:, o0:o1], Wq["W2"][o0:o1, :]


def experts_forward_mx(x_rows: np.ndarray, gamma: np.ndarray, r: np.ndarray, idx: np.ndarray,
                       kept: np.ndarray, Wq: Dict[str, np.ndarray], offs: Sequence[int],
                       tokens: np.ndarray) -> np.ndarray:
    """y [T*k, d] for the kept assignments of ``tokens`` (rows of x_rows in
    that order): u = r (MX(x*gamma) MX(W1_e)), v likewise with W3, h = silu(u) v,
    y = MX(h) MX(W2_e), the MX blocks of h running along the expert width.
    ``Wq``: ``quantized_weights``' dict or a ``LazyExpertWeights``."""
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    d = x_rows.shape[1]
    xq = mx_value(x_rows * gamma[None, :], axis=1)
    y = np.zeros((T * k, d))
    a_all = (tokens[:, None] * k + np.arange(k)[None, :]).reshape(-1)
    row_all = np.repeat(np.arange(tokens.size), k)
    e_all = idx[tokens].reshape(-1)
    kept_all = np.asarray(kept, dtype=bool)[a_all]
    for e in range(len(offs) - 1):
        m = (e_all == e) & kept_all
        if not m.any():
            continue
        sel, rows = a_all[m], row_all[m]
        W1e, W3e, W2e = _expert_mx(Wq, offs, e)
        rr = np.asarray(r, dtype=np.float64)[sel // k][:, None]
        u = rr * (xq[rows] @ W1e)
        v = rr * (xq[rows] @ W3e)
        h = O.silu(u) * v
        y[sel] = mx_value(h, axis=1) @ W2e
    return y


def moe_layer_mx(x_bits, gamma_bits, Wr_bits, bias, W1_bits, W3_bits, W2_bits,
                 widths: Sequence[int], k: int, eps: float = 1e-5, capacity_factor: float = 0.0,
                 renormalize: bool = False, idx_override: Optional[np.ndarray] = None,
                 Wq: Optional[Dict[str, np.ndarray]] = None) -> Dict[str, np.ndarray]:
    """Steps 1-7 with MXFP8 expert GEMMs (router, dispatch and combine as in
    ``moe_oracle.moe_layer``)."""
    x = O.widen_bf16(x_bits)
    gamma = O.widen_bf16(gamma_bits)
    T, E = x.shape[0], Wr_bits.shape[1]
    R = O.route(x, gamma, O.widen_bf16(Wr_bits), bias, k, eps, renormalize)
    if idx_override is not None:
        R["idx"] = np.asarray(idx_override, dtype=np.int64)
        R["gate"] = O.gates(R["logits"], R["idx"], renormalize)
    D = O.dispatch(R["idx"], E, O.capacity(T, k, E, capacity_factor))
    if Wq is None:
        Wq = quantized_weights(W1_bits, W3_bits, W2_bits)
    y = experts_forward_mx(x, gamma, R["r"], R["idx"], D["kept"], Wq, O.expert_offsets(widths),
                           np.arange(T))
    res = dict(R)
    res.update(D)
    res.update({"y": y, "out": O.combine(y, R["gate"], D["kept"])})
    return res


def moe_layer_mx_tokens(x_rows_bits, tokens, gamma_bits, Wq: Dict[str, np.ndarray],
                        widths: Sequence[int], idx: np.ndarray, gate: np.ndarray, kept: np.ndarray,
                        eps: float = 1e-5) -> np.ndarray:
    """MX layer output for a subset of tokens given the routing (full-size
    sampled checks): out [n, d]."""
    tokens = np.asarray(tokens, dtype=np.int64)
    x_rows = O.widen_bf16(x_rows_bits)
    T = np.asarray(idx).shape[0]
    r_full = np.zeros(T)
    r_full[tokens] = O.rms_stat(x_rows, eps)
    y = experts_forward_mx(x_rows, O.widen_bf16(gamma_bits), r_full, idx, kept, Wq,
                           O.expert_offsets(widths), tokens)
    return O.combine(y, gate, kept)[tokens]
