"""CPU oracle of the sparse MoE FFN layer backward -- TEST INFRASTRUCTURE ONLY.

Same rules as ``moe_oracle``: only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import it; the library never does.

The CODA sparse-MoE thread (digg.com) fixes two things about the backward:
the RMSNorm backward is fused into the backward of the first expert linear
(and, by the same commuting argument, of the router), and that fusion needs
the statistic r of each token, which is why r travels with the dispatched
token.  The thread gives no formulas; the gradient is the plain derivative
of the forward defined in ``moe_oracle`` (steps 1-7), written out here by the
chain rule in float64.  Routing (top-k ids, capacity drops) is piecewise
constant, so it carries no gradient: the gradient reaches the router only
through the gates.

Forward quantities per kept assignment a = (t, j) of expert e
(xg_t = x_t * gamma, float64 throughout):

    s_a  = xg_t W1_e          s3_a = xg_t W3_e          (pre-statistic)
    u_a  = r_t s_a            v_a  = r_t s3_a           (statistic in GEMM 1's epilogue)
    h_a  = silu(u_a) * v_a    y_a  = h_a W2_e
    out_t = sum_j kept_a gate_tj y_a
    z_t  = xg_t Wr            l_t = r_t z_t + b         p_t = softmax(l_t)

Backward, for an upstream gradient g = dL/dout:

    dy_a    = gate_a g_t                    dgate_a = <g_t, y_a>   (0 if dropped)
    dh_a    = dy_a W2_e^T                   dW2_e  += h_a^T dy_a
    du_a    = dh_a * v_a * silu'(u_a)       dv_a    = dh_a * silu(u_a)
    dS_a    = r_t du_a, dS3_a = r_t dv_a    (gradient w.r.t. s_a, s3_a)
    dW1_e  += xg_t^T dS_a                   dW3_e  += xg_t^T dS3_a
    dxg_t  += dS_a W1_e^T + dS3_a W3_e^T    dr_t   += <du_a, s_a> + <dv_a, s3_a>
    router: dl_t from dgate through the gate map and the softmax,
            db += dl_t, dWr += xg_t^T (r_t dl_t), dxg_t += r_t dl_t Wr^T,
            dr_t += <dl_t, z_t>
    norm:   dgamma += dxg_t * x_t,
            dx_t = dxg_t * gamma + dr_t * dr_t/dx_t,  dr_t/dx_t = -r_t^3 x_t / d

The dr terms are exactly what fusing the RMSNorm backward into the two
linears' backward epilogues computes: a per-row dot product of the
epilogue's gradient with the pre-statistic GEMM output.
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence

import numpy as np

from oracle import moe_oracle as O


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


class _ExpertSlices:
    """Expert e's (W1[:, o_e:o_e+1], W3[...], W2[o_e:o_e+1, :]) as float64,
    widened on first use and kept."""

    def __init__(self, W1, W3, W2, offs):
        self.W, self.offs, self.cache = (W1, W3, W2), offs, {}

    def __getitem__(self, e):
        if e not in self.cache:
            W1, W3, W2 = self.W
            o0, o1 = self.offs[e], self.offs[e + 1]
            self.cache[e] = (O.as_f64(W1[:, o0:o1]), O.as_f64(W3[:, o0:o1]), O.as_f64(W2[o0:o1, :]))
        return self.cache[e]


# --------------------------------------------------------------------------
# forward in float64 with everything the backward reads
# --------------------------------------------------------------------------
def layer_forward(x, gamma, Wr, bias, W1, W3, W2, widths: Sequence[int], k: int,
                  eps: float = 1e-5, capacity_factor: float = 0.0,
                  renormalize: bool = False, idx: Optional[np.ndarray] = None) -> Dict[str, object]:
    """Steps 1-7 on float64 values (no fp32 rounding of the logits), keeping
    the per-assignment intermediates.  ``idx`` replays a given routing.  The
    expert weights may be float64 or bf16 bit patterns (uint16); their expert
    slices are widened where used, one expert at a time."""
    x, gamma, Wr = (_f64(v) for v in (x, gamma, Wr))
    T, d = x.shape
    E = Wr.shape[1]
    r = O.rms_stat(x, eps)
    xg = x * gamma[None, :]
    z = xg @ Wr
    logits = r[:, None] * z
    if bias is not None:
        logits = logits + _f64(bias)[None, :]
    if idx is None:
        idx = O.topk_experts(logits, k)
    idx = np.asarray(idx, dtype=np.int64)
    p = O.softmax(logits)
    q = np.take_along_axis(p, idx, axis=1)
    gate = q / q.sum(axis=1, keepdims=True) if renormalize else q
    D = O.dispatch(idx, E, O.capacity(T, k, E, capacity_factor))
    offs = O.expert_offsets(widths)
    n_a = T * k
    s = [None] * n_a
    s3 = [None] * n_a
    h = [None] * n_a
    y = np.zeros((n_a, d))
    slices = _ExpertSlices(W1, W3, W2, offs)
    for a in range(n_a):
        if not D["kept"][a]:
            continue
        t, e = a // k, int(idx[a // k, a % k])
        W1e, W3e, W2e = slices[e]
        s[a] = xg[t] @ W1e
        s3[a] = xg[t] @ W3e
        h[a] = O.silu(r[t] * s[a]) * (r[t] * s3[a])
        y[a] = h[a] @ W2e
    out = np.zeros((T, d))
    for t in range(T):
        for j in range(k):
            a = t * k + j
            if D["kept"][a]:
                out[t] += gate[t, j] * y[a]
    return {"x": x, "gamma": gamma, "Wr": Wr, "W1": W1, "W3": W3, "W2": W2, "slices": slices,
            "r": r, "xg": xg, "z": z, "logits": logits, "p": p, "q": q,
            "idx": idx, "gate": gate, "kept": D["kept"], "offs": offs,
            "s": s, "s3": s3, "h": h, "y": y, "out": out, "k": k,
            "renormalize": bool(renormalize)}


# --------------------------------------------------------------------------
# the pieces of the chain rule (kept separate so tests can plant mistakes)
# --------------------------------------------------------------------------
def silu_grad(u: np.ndarray) -> np.ndarray:
    """d silu / du = sigma(u) * (1 + u * (1 - sigma(u)))."""
    with np.errstate(over="ignore"):
        sg = 1.0 / (1.0 + np.exp(-u))
    return sg * (1.0 + u * (1.0 - sg))


def gate_backward(dgate: np.ndarray, q: np.ndarray, renormalize: bool) -> np.ndarray:
    """Gradient w.r.t. q = p[idx] from the gradient w.r.t. the gates.

    Without renormalisation gate = q.  With it, gate_j = q_j / S, S = sum q,
    so dq_j = (dgate_j - sum_i dgate_i gate_i) / S.
    """
    if not renormalize:
        return dgate.copy()
    S = q.sum(axis=1, keepdims=True)
    gate = q / S
    return (dgate - (dgate * gate).sum(axis=1, keepdims=True)) / S


def softmax_backward(p: np.ndarray, dp: np.ndarray) -> np.ndarray:
    """dl = p * (dp - <dp, p>) for p = softmax(l), row-wise."""
    return p * (dp - (dp * p).sum(axis=1, keepdims=True))


def rms_backward(x: np.ndarray, r: np.ndarray, dr: np.ndarray) -> np.ndarray:
    """Contribution of dL/dr_t to dL/dx_t: dr_t * (-r_t^3 x_t / d)."""
    d = x.shape[1]
    return (dr * -(r ** 3) / d)[:, None] * x


def router_backward(dl: np.ndarray, xg: np.ndarray, z: np.ndarray, r: np.ndarray, Wr: np.ndarray):
    """Backward of l = r * (xg Wr) + b: (dbias, dWr, dxg part, dr part)."""
    rdl = r[:, None] * dl
    return dl.sum(axis=0), xg.T @ rdl, rdl @ Wr.T, (dl * z).sum(axis=1)


def swiglu_backward(dh: np.ndarray, u: np.ndarray, v: np.ndarray):
    """(du, dv) for h = silu(u) * v."""
    return dh * v * silu_grad(u), dh * O.silu(u)


# --------------------------------------------------------------------------
# the whole backward
# --------------------------------------------------------------------------
def layer_backward(f: Dict[str, object], g, weight_grads: bool = True) -> Dict[str, np.ndarray]:
    """Gradients of L = <g, out> w.r.t. x, gamma, Wr, bias, W1, W3, W2.

    ``f`` is ``layer_forward``'s result.  Also returns the per-assignment
    dgate and the per-token dr (split into its expert and router parts) so
    that each stage of another implementation can be checked on its own.
    ``weight_grads=False`` skips dW1, dW3, dW2 (returned as None): the other
    gradients of a token then depend on that token alone (without a capacity
    limit), so a subset of tokens can be checked at full size.
    """
    g = _f64(g)
    x, gamma, Wr = f["x"], f["gamma"], f["Wr"]
    slices = f["slices"]
    r, xg, z, p, q = f["r"], f["xg"], f["z"], f["p"], f["q"]
    idx, gate, kept, offs, k = f["idx"], f["gate"], f["kept"], f["offs"], f["k"]
    T, d = x.shape
    E = Wr.shape[1]
    F = int(offs[-1])
    dW1 = np.zeros((d, F)) if weight_grads else None
    dW3 = np.zeros((d, F)) if weight_grads else None
    dW2 = np.zeros((F, d)) if weight_grads else None
    dxg = np.zeros((T, d))
    dr_exp = np.zeros(T)
    dgate = np.zeros((T, k))
    for a in range(T * k):
        if not kept[a]:
            continue                     # a dropped slot does not reach out
        t, j = a // k, a % k
        e = int(idx[t, j])
        o0, o1 = offs[e], offs[e + 1]
        W1e, W3e, W2e = slices[e]
        dgate[t, j] = g[t] @ f["y"][a]
        dy = gate[t, j] * g[t]
        dh = W2e @ dy
        u, v = r[t] * f["s"][a], r[t] * f["s3"][a]
        du, dv = swiglu_backward(dh, u, v)
        dS, dS3 = r[t] * du, r[t] * dv
        if weight_grads:
            dW2[o0:o1, :] += np.outer(f["h"][a], dy)
            dW1[:, o0:o1] += np.outer(xg[t], dS)
            dW3[:, o0:o1] += np.outer(xg[t], dS3)
        dxg[t] += W1e @ dS + W3e @ dS3
        dr_exp[t] += du @ f["s"][a] + dv @ f["s3"][a]
    # router: gates -> q -> p (scattered to the chosen experts) -> logits
    dq = gate_backward(dgate, q, f["renormalize"])
    dp = np.zeros((T, E))
    np.put_along_axis(dp, idx, dq, axis=1)   # top-k ids of a token are distinct
    dl = softmax_backward(p, dp)
    dbias, dWr, dxg_router, dr_router = router_backward(dl, xg, z, r, Wr)
    dxg += dxg_router
    dr = dr_exp + dr_router
    dgamma = (dxg * x).sum(axis=0)
    dx = dxg * gamma[None, :] + rms_backward(x, r, dr)
    return {"dx": dx, "dgamma": dgamma, "dWr": dWr, "dbias": dbias,
            "dW1": dW1, "dW3": dW3, "dW2": dW2, "dgate": dgate, "dl": dl,
            "dr": dr, "dr_exp": dr_exp, "dr_router": dr_router, "dxg": dxg}


def loss(f: Dict[str, object], g) -> float:
    """L = <g, out>, the scalar the gradients above belong to."""
    return float((_f64(g) * f["out"]).sum())
