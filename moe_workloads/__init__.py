"""Seeded synthetic workloads for the sparse MoE FFN layer forward.

This module is shared by the CPU oracle and by the CUDA path's tests and
benchmark. It holds only shapes, value distributions and a counter-based
random generator: none of the layer's arithmetic (no normalisation, routing,
capacity rule, width rounding or expert math) lives here, so that the two
implementations it feeds stay independent.

Every tensor is drawn from numpy's Philox-4x64 counter-based generator keyed
by ``(seed, stream)``; each tensor (and each expert's slice of a weight) has
its own stream, so slices can be generated in parallel threads and any subset
can be regenerated without drawing the rest.  Floating-point tensors are drawn
in float32 and rounded to bfloat16 with round-to-nearest-even; they are handed
out as ``numpy.uint16`` arrays of bf16 bit patterns, which both sides widen
exactly.

The five workloads are the layer shapes of the MoE literature the layer is
meant for: a tiny layer that a plain CPU implementation finishes instantly, a
Switch-style top-1 layer with an expert capacity and a skewed router, a layer
with variable-width experts in the ``[(count, size), ...]`` notation of the
nanoMOE variable-size-experts notes, a fine-grained 64-expert top-8 layer and a
Mixtral-8x7B-shaped layer.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

# Stream ids of the tensors.  Expert weight slices use stream = id * 4096 + e.
_STREAM_X = 1
_STREAM_GAMMA = 2
_STREAM_WR = 3
_STREAM_BIAS = 4
_STREAM_W1 = 5
_STREAM_W3 = 6
_STREAM_W2 = 7


@dataclass(frozen=True)
class Workload:
    """Shape and distribution recipe of one synthetic MoE layer problem.

    ``expert_sizes`` uses the ``[(count, size), ...]`` notation; the sizes
    listed here are the raw sizes (each side applies its own width rule).
    ``bias`` names the router logit-bias recipe: ``"none"``, ``"zipf"``
    (b_e = 1.5 * ln(1/(e+1))) or ``"normal"`` (b_e ~ N(0, variance 0.5)).
    ``capacity_factor <= 0`` means dropless.
    """

    name: str
    T: int
    d_model: int
    E: int
    k: int
    expert_sizes: Tuple[Tuple[int, int], ...]
    capacity_factor: float = 0.0
    bias: str = "none"
    eps: float = 1e-5
    seed: int = 0
    description: str = ""

    def with_tokens(self, T: int, name: Optional[str] = None) -> "Workload":
        return Workload(name or f"{self.name}_T{T}", T, self.d_model, self.E, self.k,
                        self.expert_sizes, self.capacity_factor, self.bias, self.eps,
                        self.seed, self.description)

    def raw_sizes(self) -> List[int]:
        out: List[int] = []
        for count, size in self.expert_sizes:
            out.extend([int(size)] * int(count))
        return out


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny", T=256, d_model=128, E=8, k=2, expert_sizes=((8, 256),),
                 description="tiny layer: T=256, d=128, E=8, top-2, d_ffn=256, dropless"),
        Workload("switch_capacity", T=4096, d_model=1024, E=16, k=1,
                 expert_sizes=((16, 4096),), capacity_factor=1.25, bias="zipf",
                 description="Switch top-1: T=4096, d=1024, E=16, d_ffn=4096, "
                             "capacity factor 1.25, Zipf-like logit bias"),
        Workload("variable_size", T=8192, d_model=768, E=8, k=2,
                 expert_sizes=((1, 2048), (7, 1024)),
                 description="variable-size experts [(1,2048),(7,1024)]: T=8192, "
                             "d=768, E=8, top-2, dropless"),
        Workload("fine_grained", T=16384, d_model=2048, E=64, k=8,
                 expert_sizes=((64, 512),), bias="normal",
                 description="fine-grained: T=16384, d=2048, E=64, top-8, "
                             "d_ffn=512, logit bias N(0, 0.5), dropless"),
        Workload("mixtral", T=16384, d_model=4096, E=8, k=2,
                 expert_sizes=((8, 14336),),
                 description="Mixtral-8x7B-shaped: T=16384 (8 x 2048), d=4096, "
                             "E=8, top-2, d_ffn=14336, dropless"),
    ]
}

WORKLOAD_ORDER = ["tiny", "switch_capacity", "variable_size", "fine_grained", "mixtral"]

# Small cases for profiler captures: the per-tile work of a full-size
# workload (same d and expert width) with few experts, so that a multi-pass
# capture holds a few GB on the device.
PROFILE_WORKLOADS: Dict[str, Workload] = {
    "mixtral_2e": Workload("mixtral_2e", T=4096, d_model=4096, E=2, k=1,
                           expert_sizes=((2, 14336),),
                           description="two Mixtral-shaped experts: T=4096, d=4096, E=2, "
                                       "top-1, d_ffn=14336 (profiling case)"),
}
WORKLOADS.update(PROFILE_WORKLOADS)


def _philox(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=[int(seed), int(stream)]))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round-to-nearest-even), as uint16 bits.

    The inputs are finite normal draws; NaN handling is not needed here.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal_bf16(seed: int, stream: int, shape: Sequence[int], std: float,
                 mean: float = 0.0) -> np.ndarray:
    g = _philox(seed, stream)
    a = g.standard_normal(int(np.prod(shape)), dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    if mean != 0.0:
        a += np.float32(mean)
    return f32_to_bf16_bits(a).reshape(shape)


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def gen_x(w: Workload, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """Activations x [T, d] ~ N(0, 1) as bf16 bits.

    Drawn in blocks of 256 tokens (one Philox stream per block) so that a subset
    of rows can be regenerated without drawing the whole tensor.
    """
    blk = 256
    nblk = (w.T + blk - 1) // blk

    def block(b: int) -> np.ndarray:
        n = min(blk, w.T - b * blk)
        return _normal_bf16(w.seed, (_STREAM_X << 32) + b, (n, w.d_model), 1.0)

    if rows is None:
        out = np.empty((w.T, w.d_model), dtype=np.uint16)
        with ThreadPoolExecutor(_threads()) as ex:
            for b, arr in enumerate(ex.map(block, range(nblk))):
                out[b * blk: b * blk + arr.shape[0]] = arr
        return out
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), w.d_model), dtype=np.uint16)
    cache: Dict[int, np.ndarray] = {}
    for i, t in enumerate(rows):
        b = int(t) // blk
        if b not in cache:
            cache[b] = block(b)
        out[i] = cache[b][int(t) - b * blk]
    return out


def gen_gamma(w: Workload) -> np.ndarray:
    """RMSNorm weight gamma [d] = 1 + 0.1 * N(0, 1), as bf16 bits."""
    g = _philox(w.seed, _STREAM_GAMMA)
    a = g.standard_normal(w.d_model, dtype=np.float32) * np.float32(0.1) + np.float32(1.0)
    return f32_to_bf16_bits(a)


def gen_router_weight(w: Workload) -> np.ndarray:
    """Router weight Wr [d, E] ~ N(0, 1/d) (fan_in = d), as bf16 bits."""
    return _normal_bf16(w.seed, _STREAM_WR, (w.d_model, w.E), 1.0 / math.sqrt(w.d_model))


def gen_router_bias(w: Workload) -> Optional[np.ndarray]:
    """Per-expert router logit bias [E] float32, or None for an unbiased router."""
    if w.bias == "none":
        return None
    if w.bias == "zipf":
        return np.array([1.5 * math.log(1.0 / (e + 1)) for e in range(w.E)], dtype=np.float32)
    if w.bias == "normal":
        g = _philox(w.seed, _STREAM_BIAS)
        return (g.standard_normal(w.E) * math.sqrt(0.5)).astype(np.float32)
    raise ValueError(f"unknown bias recipe {w.bias!r}")


def gen_expert_weights(w: Workload, widths: Sequence[int],
                       experts: Optional[Sequence[int]] = None
                       ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Expert weights in the concatenated layout, as bf16 bits.

    ``widths`` are the per-expert FFN widths f_e the caller has settled on.
    W1, W3 are [d, F] with expert e in columns [o_e, o_e + f_e); W2 is [F, d]
    with expert e in rows [o_e, o_e + f_e), where o_e = f_0 + ... + f_{e-1}.
    W1_e, W3_e ~ N(0, 1/d); W2_e ~ N(0, 1/f_e) (fan_in of each linear map).
    If ``experts`` is given, only those experts' slices are drawn (the rest
    stay zero).
    """
    d = w.d_model
    widths = [int(f) for f in widths]
    offs = np.concatenate([[0], np.cumsum(widths)]).astype(np.int64)
    F = int(offs[-1])
    W1 = np.zeros((d, F), dtype=np.uint16)
    W3 = np.zeros((d, F), dtype=np.uint16)
    W2 = np.zeros((F, d), dtype=np.uint16)
    sel = range(w.E) if experts is None else [int(e) for e in experts]

    def job(item):
        which, e = item
        f = widths[e]
        if which == 2:
            return item, _normal_bf16(w.seed, (_STREAM_W2 << 12) + e, (f, d), 1.0 / math.sqrt(f))
        stream = ((_STREAM_W1 if which == 1 else _STREAM_W3) << 12) + e
        return item, _normal_bf16(w.seed, stream, (d, f), 1.0 / math.sqrt(d))

    items = [(which, e) for e in sel for which in (1, 3, 2)]
    with ThreadPoolExecutor(_threads()) as ex:
        for (which, e), arr in ex.map(job, items):
            o, f = int(offs[e]), widths[e]
            if which == 1:
                W1[:, o:o + f] = arr
            elif which == 3:
                W3[:, o:o + f] = arr
            else:
                W2[o:o + f, :] = arr
    return W1, W3, W2


def sample_tokens(w: Workload, n: int, salt: int = 99) -> np.ndarray:
    """A seeded, sorted sample of n distinct token ids of the workload."""
    g = _philox(w.seed, (salt << 40) + 1)
    n = min(n, w.T)
    return np.sort(g.choice(w.T, size=n, replace=False)).astype(np.int64)


def random_routing(T: int, E: int, k: int, seed: int, skew: float = 0.0) -> np.ndarray:
    """Seeded expert ids [T, k] (distinct per row) for dispatch-only tests.

    ``skew > 0`` draws experts with Zipf-like weights (e+1)^-skew.
    """
    g = _philox(seed, 0xD15)
    p = (np.arange(E) + 1.0) ** (-skew)
    p /= p.sum()
    out = np.empty((T, k), dtype=np.int32)
    for t in range(T):
        out[t] = g.choice(E, size=k, replace=False, p=p)
    return out
