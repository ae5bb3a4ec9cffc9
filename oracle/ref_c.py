"""ctypes loader of ``moe_ref.c``, the plain-C float64 oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` use it (``__graft_entry__.build()`` compiles it).  It computes
the same definition as ``moe_oracle.py`` in plain C loops, written separately
from the sources, so the two oracles check each other; neither shares code
with the library.
"""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess
from typing import Dict, Optional, Sequence

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_ref.c")
LIB = os.path.join(HERE, "libmoe_ref.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile moe_ref.c into oracle/libmoe_ref.so with the host C compiler."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        raise RuntimeError("no C compiler found for the C oracle")
    cmd = [cc, "-O2", "-std=c99", "-shared", "-fPIC", "-o", LIB, SRC, "-lm"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"C oracle build failed:\n{res.stdout}\n{res.stderr}")
    return LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32, f64 = ctypes.c_int32, ctypes.c_double
        lib.moe_ref_layer.restype = ctypes.c_int
        lib.moe_ref_layer.argtypes = [P, P, P, P, P, P, P, P, i32, i32, i32, i32, f64, f64, i32, P,
                                      P, P, P, P, P, P, P, P, P]
        _lib = lib
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def layer(x_bits, gamma_bits, Wr_bits, bias, W1_bits, W3_bits, W2_bits, widths: Sequence[int], k: int,
          eps: float = 1e-5, capacity_factor: float = 0.0, renormalize: bool = False,
          idx_override: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """The layer forward (steps 1-7) in C; the same keys as moe_oracle.moe_layer."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    T, d = x.shape
    Wr = np.ascontiguousarray(Wr_bits, dtype=np.uint16)
    E = Wr.shape[1]
    offs = np.zeros(E + 1, dtype=np.int32)
    offs[1:] = np.cumsum(np.asarray(widths, dtype=np.int64))
    gamma = np.ascontiguousarray(gamma_bits, dtype=np.uint16)
    W1 = np.ascontiguousarray(W1_bits, dtype=np.uint16)
    W3 = np.ascontiguousarray(W3_bits, dtype=np.uint16)
    W2 = np.ascontiguousarray(W2_bits, dtype=np.uint16)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float64)
    io = None if idx_override is None else np.ascontiguousarray(idx_override, dtype=np.int32)
    r = np.empty(T, dtype=np.float64)
    logits = np.empty((T, E), dtype=np.float32)
    idx = np.empty((T, k), dtype=np.int32)
    gate = np.empty((T, k), dtype=np.float64)
    counts = np.empty(E, dtype=np.int32)
    offsets = np.empty(E + 1, dtype=np.int32)
    perm = np.empty(max(T * k, 1), dtype=np.int32)
    inv_perm = np.empty(max(T * k, 1), dtype=np.int32)
    out = np.empty((T, d), dtype=np.float64)
    st = _load().moe_ref_layer(_p(x), _p(gamma), _p(Wr), _p(b), _p(W1), _p(W3), _p(W2), _p(offs),
                               T, d, E, k, float(eps), float(capacity_factor or 0.0), int(bool(renormalize)),
                               _p(io), _p(r), _p(logits), _p(idx), _p(gate), _p(counts), _p(offsets), _p(perm),
                               _p(inv_perm), _p(out))
    if st == 1:
        raise ValueError("expert id out of range")
    if st != 0:
        raise RuntimeError(f"C oracle failed ({st})")
    n = int(offsets[-1])
    return {"r": r, "logits": logits, "idx": idx.astype(np.int64), "gate": gate, "counts": counts.astype(np.int64),
            "offsets": offsets.astype(np.int64), "perm": perm[:n].astype(np.int64),
            "inv_perm": inv_perm[:T * k].astype(np.int64), "out": out, "n_kept": n}
