"""CPU oracle of the sparse MoE FFN layer forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The library in
``sparse_mixture_experts_rms_b200`` never imports it and shares no code with
it; the only common input is the seeded generator in ``moe_workloads``.

What it computes, in the order the sources give it:

1. RMS statistic r_t = 1 / sqrt(mean_i x_ti^2 + eps) (CODA sparse-MoE thread,
   the RMSNorm paragraph: the scale by the statistic commutes across the GEMM
   that follows the norm, so it can be applied in that GEMM's epilogue).
2. Router: a plain linear layer on the normalised token,
   l_te = r_t * sum_i x_ti gamma_i Wr_ie + b_e, with r applied after the GEMM
   and before the top-k (CODA thread: the router is a plain GEMM that follows
   the RMSNorm, so its epilogue applies the r-scale just ahead of the top-k;
   MoE glossary, "gating network").
3. Top-k gating: the k experts with the largest logits (MoE glossary,
   "Top-k Gating" / "Switch Routing"); ties go to the lower expert index and
   the k slots are in descending logit order (the sources are silent; this is
   the reading taken).  gate = softmax over all E logits at the chosen
   experts, optionally renormalised over the k chosen.
4. Expert capacity C = (T * k) / E * capacity_factor, rounded down; an
   expert keeps its first C assignments in token order and drops the rest
   (MoE glossary, "Expert Capacity").
5. Expert-centric schedule: routing decisions flattened to a task list,
   grouped by expert and ordered by token id inside each group (OmniMoE
   summary, section 2.2 "Expert-Centric Scheduling").  ``perm`` lists the
   kept assignment ids a = t*k + j in that order; ``inv_perm`` maps back.
6. Experts: SwiGLU FFN per expert on the normalised token, with r applied
   after the first expert GEMM (CODA thread: the r-scale is carried with the
   dispatched token to the first expert linear).  Expert widths come from a
   ``[(count, size), ...]`` list rounded up to a multiple of 128, with
   cumulative column offsets into the concatenated W1 [d, F] / W2 [F, d]
   (nanoMOE variable-size-experts notes, "Configuration Changes", "Offset
   Calculation", "Weight Allocation").
7. Combine: out_t = sum over kept slots j of gate_tj * y_(t,j); dropped slots
   contribute zero (MoE glossary, "Top-k Gating": outputs combined by a
   weighted sum of the scores).

Precision: bf16 inputs are widened exactly; every sum and product is float64.
The router logits are rounded once to float32, and the top-k decision is taken
on those float32 values, because the layer decides its routing on fp32 logits.
Softmax is float64 on the float32 logits.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

DEFAULT_BLOCK = 128


# --------------------------------------------------------------------------
# helpers for inputs
# --------------------------------------------------------------------------
def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def as_f64(a: np.ndarray) -> np.ndarray:
    """Values of ``a`` as float64: bf16 bit patterns (uint16) are widened
    exactly; float arrays (weights widened once by the caller) pass through."""
    if a.dtype == np.uint16:
        return widen_bf16(a)
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------
# variable-width experts (nanoMOE variable-size-experts notes)
# --------------------------------------------------------------------------
def expert_widths(expert_sizes: Sequence[Tuple[int, int]], block: int = DEFAULT_BLOCK) -> List[int]:
    """Per-expert FFN widths from ``[(count, size), ...]``.

    nanoMOE notes, "1. Configuration Changes" / "Expert Size Computation":
    each size is rounded up to a multiple of the block size, then repeated
    ``count`` times, in list order.
    """
    widths: List[int] = []
    for count, size in expert_sizes:
        rounded = ((int(size) + block - 1) // block) * block
        widths.extend([rounded] * int(count))
    return widths


def expert_offsets(widths: Sequence[int]) -> List[int]:
    """Cumulative column offsets [E+1] of the experts in W1/W3 (rows of W2).

    nanoMOE notes, "Offset Calculation": offsets start at 0 and each expert
    adds its own width (a running sum, never index * width).
    """
    offs = [0]
    for w in widths:
        offs.append(offs[-1] + int(w))
    return offs


# --------------------------------------------------------------------------
# 1. RMS statistic and the textbook RMSNorm
# --------------------------------------------------------------------------
def rms_stat(x: np.ndarray, eps: float) -> np.ndarray:
    """r_t = 1 / sqrt((1/d) * sum_i x_ti^2 + eps), float64 [T]."""
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / np.sqrt(np.mean(x * x, axis=1) + eps)


def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """Textbook RMSNorm: (x_t * r_t) * gamma, float64 [T, d]."""
    x = np.asarray(x, dtype=np.float64)
    return (x * rms_stat(x, eps)[:, None]) * np.asarray(gamma, dtype=np.float64)[None, :]


# --------------------------------------------------------------------------
# 2./3. router, top-k, softmax gates
# --------------------------------------------------------------------------
def router_logits(x: np.ndarray, gamma: np.ndarray, Wr: np.ndarray,
                  bias: Optional[np.ndarray], r: np.ndarray) -> np.ndarray:
    """Router logits as float32 [T, E].

    CODA placement: the GEMM runs on x * gamma (no statistic), and r_t scales
    the GEMM result row-wise before the bias and the top-k.
    """
    xg = np.asarray(x, dtype=np.float64) * np.asarray(gamma, dtype=np.float64)[None, :]
    s = xg @ np.asarray(Wr, dtype=np.float64)
    logits = np.asarray(r, dtype=np.float64)[:, None] * s
    if bias is not None:
        logits = logits + np.asarray(bias, dtype=np.float64)[None, :]
    return logits.astype(np.float32)


def topk_experts(logits32: np.ndarray, k: int) -> np.ndarray:
    """Indices [T, k] of the k largest logits per row, largest first.

    Ties are broken toward the lower expert index: a stable sort of the
    negated logits keeps equal values in index order.
    """
    neg = -np.asarray(logits32, dtype=np.float64)
    order = np.argsort(neg, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def softmax(logits32: np.ndarray) -> np.ndarray:
    """Row softmax over all experts, float64."""
    z = np.asarray(logits32, dtype=np.float64)
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=1, keepdims=True)


def gates(logits32: np.ndarray, idx: np.ndarray, renormalize: bool = False) -> np.ndarray:
    """gate_tj = softmax(l_t)[idx_tj]; optionally renormalised over the k chosen."""
    p = softmax(logits32)
    g = np.take_along_axis(p, np.asarray(idx, dtype=np.int64), axis=1)
    if renormalize:
        g = g / g.sum(axis=1, keepdims=True)
    return g


def topk_margin(logits32: np.ndarray, k: int) -> np.ndarray:
    """l_(k) - l_(k+1) per token (k-th minus (k+1)-th largest fp32 logit).

    +inf when k equals the number of experts (every expert is chosen).
    """
    T, E = logits32.shape
    if k >= E:
        return np.full(T, np.inf)
    srt = -np.sort(-np.asarray(logits32, dtype=np.float64), axis=1)
    return srt[:, k - 1] - srt[:, k]


def route(x, gamma, Wr, bias, k: int, eps: float, renormalize: bool = False) -> Dict[str, np.ndarray]:
    """Steps 1-3: r, fp32 logits, top-k expert ids and gates."""
    r = rms_stat(x, eps)
    logits = router_logits(x, gamma, Wr, bias, r)
    idx = topk_experts(logits, k)
    g = gates(logits, idx, renormalize)
    return {"r": r, "logits": logits, "idx": idx, "gate": g}


# --------------------------------------------------------------------------
# 4./5. capacity and dispatch
# --------------------------------------------------------------------------
def capacity(T: int, k: int, E: int, capacity_factor: float) -> Optional[int]:
    """Expert capacity C = (T * k) / E * capacity_factor, rounded down.

    MoE glossary, "Expert Capacity".  ``capacity_factor <= 0`` means no
    capacity limit (dropless); returns None then.
    """
    if capacity_factor is None or capacity_factor <= 0:
        return None
    return int(math.floor(T * k / E * capacity_factor))


def dispatch(idx: np.ndarray, E: int, C: Optional[int]) -> Dict[str, np.ndarray]:
    """Histogram, stable per-expert rank, capacity and the expert-centric order.

    Assignments a = t*k + j are taken in token order.  rank_a counts the
    earlier assignments to the same expert; a is kept iff rank_a < C.
    ``offsets`` is the exclusive running sum of the kept counts; perm lists
    kept assignments grouped by expert, token order inside a group (OmniMoE
    summary, "Expert-Centric Scheduling"); inv_perm[a] is a's position in
    perm, or -1 when a was dropped.
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    flat = idx.reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert id out of range")
    counts = np.bincount(flat, minlength=E).astype(np.int64)
    rank = np.empty(flat.size, dtype=np.int64)
    for e in range(E):
        where = np.nonzero(flat == e)[0]          # ascending assignment ids
        rank[where] = np.arange(where.size)
    kept = np.ones(flat.size, dtype=bool) if C is None else rank < C
    kept_counts = counts.copy() if C is None else np.minimum(counts, C)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept_counts)
    perm = np.empty(int(offsets[-1]), dtype=np.int64)
    inv_perm = np.full(flat.size, -1, dtype=np.int64)
    a_kept = np.nonzero(kept)[0]
    pos = offsets[flat[a_kept]] + rank[a_kept]
    perm[pos] = a_kept
    inv_perm[a_kept] = pos
    return {"counts": counts, "kept_counts": kept_counts, "offsets": offsets,
            "perm": perm, "inv_perm": inv_perm, "rank": rank, "kept": kept,
            "n_kept": int(offsets[-1])}


# --------------------------------------------------------------------------
# 6./7. experts and combine
# --------------------------------------------------------------------------
def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z / (1 + exp(-z))."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def expert_ffn(xg_rows: np.ndarray, r_rows: np.ndarray, W1e: np.ndarray,
               W3e: np.ndarray, W2e: np.ndarray) -> np.ndarray:
    """SwiGLU expert on rows of x*gamma with the statistic applied after GEMM 1.

    u = r * ((x*gamma) W1_e), v = r * ((x*gamma) W3_e), h = silu(u) * v,
    y = h W2_e.  All float64.
    """
    u = r_rows[:, None] * (xg_rows @ W1e)
    v = r_rows[:, None] * (xg_rows @ W3e)
    return (silu(u) * v) @ W2e


def experts_forward(x_bits: np.ndarray, gamma_bits: np.ndarray, r: np.ndarray,
                    idx: np.ndarray, kept: np.ndarray, W1_bits: np.ndarray,
                    W3_bits: np.ndarray, W2_bits: np.ndarray, offs: Sequence[int],
                    tokens: Optional[np.ndarray] = None) -> np.ndarray:
    """y [T*k, d] float64: each kept assignment's expert output (0 if dropped).

    If ``tokens`` is given, only those tokens' assignments are computed (rows
    of the other tokens stay 0); ``x_bits`` then holds just those tokens' rows
    in the same order.  Expert weight slices are widened one expert at a time
    (or used as given when the caller passes them already as float64).
    """
    idx = np.asarray(idx, dtype=np.int64)
    T, k = idx.shape
    d = W1_bits.shape[0]
    gamma = widen_bf16(gamma_bits)
    if tokens is None:
        tokens = np.arange(T)
    tokens = np.asarray(tokens, dtype=np.int64)
    xg = widen_bf16(x_bits) * gamma[None, :]
    y = np.zeros((T * k, d), dtype=np.float64)
    # every (token, slot) of the requested tokens, with the row of x_bits it uses
    a_all = (tokens[:, None] * k + np.arange(k)[None, :]).reshape(-1)
    row_all = np.repeat(np.arange(tokens.size), k)
    e_all = idx[tokens].reshape(-1)
    kept_all = np.asarray(kept, dtype=bool)[a_all]
    E = len(offs) - 1
    for e in range(E):
        m = (e_all == e) & kept_all
        if not m.any():
            continue
        sel_a = a_all[m]
        rows = row_all[m]
        t_of = sel_a // k
        o0, o1 = int(offs[e]), int(offs[e + 1])
        W1e = as_f64(W1_bits[:, o0:o1])
        W3e = as_f64(W3_bits[:, o0:o1])
        W2e = as_f64(W2_bits[o0:o1, :])
        y[sel_a] = expert_ffn(xg[rows], np.asarray(r, dtype=np.float64)[t_of], W1e, W3e, W2e)
    return y


def combine(y: np.ndarray, gate: np.ndarray, kept: np.ndarray) -> np.ndarray:
    """out_t = sum_j [kept] gate_tj * y_(t*k+j), summed in slot order j = 0..k-1."""
    gate = np.asarray(gate, dtype=np.float64)
    T, k = gate.shape
    d = y.shape[1]
    w = gate.reshape(-1) * np.asarray(kept, dtype=np.float64)
    out = np.zeros((T, d), dtype=np.float64)
    for j in range(k):
        out += w[j::k][:, None] * y[j::k]
    return out


# --------------------------------------------------------------------------
# router metrics (MoE glossary, "Load Balancing" / "Auxiliary Loss")
# --------------------------------------------------------------------------
def router_stats(logits32: np.ndarray, counts: np.ndarray, n_kept: int, k: int) -> Dict[str, object]:
    """Load-balance metrics of one routing pass, float64.

    prob_mean[e] = (1/T) sum_t softmax(l_t)[e]  (the routing probability mass
    each expert receives); the glossary's auxiliary loss is the squared
    coefficient of variation of that distribution across experts,
    cv2_prob = Var_e(prob_mean) / Mean_e(prob_mean)^2 (population variance);
    the Switch-style form E * sum_e f_e * prob_mean_e with f_e = counts_e/(T*k)
    is reported too, with cv2_load (the same CV^2 of the counts) and the
    fraction of assignments dropped by the capacity limit.
    """
    p = softmax(logits32)
    T, E = p.shape
    prob_mean = p.mean(axis=0)
    counts = np.asarray(counts, dtype=np.float64)
    f = counts / float(T * k)

    def cv2(v):
        m = v.mean()
        return float(((v - m) ** 2).mean() / (m * m)) if m != 0 else 0.0

    return {"prob_mean": prob_mean,
            "aux_loss": float(E * np.sum(f * prob_mean)),
            "cv2_prob": cv2(prob_mean),
            "cv2_load": cv2(counts),
            "dropped_frac": float(1.0 - n_kept / float(T * k))}


# --------------------------------------------------------------------------
# the whole layer
# --------------------------------------------------------------------------
def moe_layer(x_bits, gamma_bits, Wr_bits, bias, W1_bits, W3_bits, W2_bits,
              widths: Sequence[int], k: int, eps: float = 1e-5,
              capacity_factor: float = 0.0, renormalize: bool = False,
              idx_override: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Steps 1-7 on all tokens.  ``idx_override`` replays another router's ids."""
    x = widen_bf16(x_bits)
    gamma = widen_bf16(gamma_bits)
    Wr = widen_bf16(Wr_bits)
    T = x.shape[0]
    E = Wr.shape[1]
    R = route(x, gamma, Wr, bias, k, eps, renormalize)
    if idx_override is not None:
        R["idx"] = np.asarray(idx_override, dtype=np.int64)
        R["gate"] = gates(R["logits"], R["idx"], renormalize)
    C = capacity(T, k, E, capacity_factor)
    D = dispatch(R["idx"], E, C)
    offs = expert_offsets(widths)
    y = experts_forward(x_bits, gamma_bits, R["r"], R["idx"], D["kept"],
                        W1_bits, W3_bits, W2_bits, offs)
    out = combine(y, R["gate"], D["kept"])
    res = dict(R)
    res.update(D)
    res.update({"capacity": C, "y": y, "out": out})
    return res


def moe_layer_tokens(x_rows_bits, tokens, gamma_bits, W1_bits, W3_bits, W2_bits,
                     widths: Sequence[int], idx: np.ndarray, gate: np.ndarray,
                     kept: np.ndarray, eps: float = 1e-5) -> np.ndarray:
    """Layer output for a subset of tokens, given routing and kept flags.

    Used at full problem sizes: routing and dispatch are computed for every
    token, the expert FFNs only for the sampled ones.  Returns out [n, d].
    """
    tokens = np.asarray(tokens, dtype=np.int64)
    x_rows = widen_bf16(x_rows_bits)
    r_rows = rms_stat(x_rows, eps)
    T, k = np.asarray(idx).shape
    r_full = np.zeros(T)
    r_full[tokens] = r_rows
    offs = expert_offsets(widths)
    y = experts_forward(x_rows_bits, gamma_bits, r_full, idx, kept, W1_bits,
                        W3_bits, W2_bits, offs, tokens=tokens)
    out = combine(y, gate, kept)
    return out[tokens]
