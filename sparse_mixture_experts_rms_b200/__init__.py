"""Python binding of ``libmoe_b200.so``: the B200 sparse MoE FFN layer forward.

The functions here have the names of the C ABI in ``include/moe.h`` and only
marshal arguments: they check torch tensors (device, dtype, shape,
contiguity), pass raw pointers and the current CUDA stream, and raise
``MoEError`` on a non-OK status.  Every step of the layer runs in the
library's sm_100a kernels; there is no fallback path.  If the library has not
been built, importing works but every call raises.

Layer (forward only): RMS statistic -> router GEMM with the statistic applied
before the top-k (CODA) -> softmax/top-k gating -> dispatch (histogram,
capacity, expert-centric permutation) -> grouped SwiGLU expert GEMMs with
variable widths, r applied after GEMM 1, gate after GEMM 2 -> combine.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libmoe_b200.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_ALIGNMENT = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_UNSUPPORTED = 4
MOE_ERR_CUDA = 5
MOE_ERR_DEVICE = 6
MOE_ERR_NO_DEVICE = 7

MOE_DEVERR_EXPERT_ID = 0x1
MOE_DEVERR_TIMEOUT = 0x2
MOE_DEVERR_TILE_TABLE = 0x4

EXPORTED = ["moe_status_string", "moe_capacity", "moe_max_kept", "moe_expert_offsets", "moe_workspace_size",
            "moe_workspace_init", "moe_get_device_error", "moe_set_wait_limit", "moe_route", "moe_dispatch",
            "moe_dispatch_noalloc",
            "moe_experts_fwd", "moe_experts_up", "moe_experts_down", "moe_combine",
            "moe_layer_fwd", "moe_layer_fwd_gather", "moe_router_stats", "moe_train_workspace_size", "moe_train_rows",
            "moe_train_saved", "moe_layer_fwd_train", "moe_layer_bwd",
            "moe_host_workspace_size", "moe_host_chunks", "moe_layer_fwd_host",
            "moe_mx_weights_size", "moe_quantize_weights_mx", "moe_mx_workspace_size", "moe_mx_rows",
            "moe_layer_fwd_mx", "moe_mx_part"]

# ids of moe_mx_part
MOE_MX = {"W1": 0, "W3": 1, "W2": 2, "SF1": 3, "SF3": 4, "SF2": 5, "X8": 6, "XSF": 7, "H8": 8, "HSF": 9,
          "PERM": 10, "OFFSETS": 11, "IDX": 12, "GATE": 13, "R": 14}

# ids of moe_train_saved
MOE_SAVED = {"r": 0, "idx": 1, "gate": 2, "logits": 3, "offsets": 4, "perm": 5, "inv_perm": 6,
             "U": 7, "V": 8, "H": 9, "y": 10, "dgate": 11, "dr": 12, "counts": 13}


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str = "", code: int = 0):
        self.status = status
        self.code = code
        msg = _status_text(status)
        if what:
            msg = f"{what}: {msg}"
        if code:
            msg += f" (device error word 0x{code:x})"
        super().__init__(msg)


class _Config(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d_model", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("ffn_offsets", ctypes.POINTER(ctypes.c_int32)),
                ("capacity_factor", ctypes.c_float), ("eps", ctypes.c_float),
                ("renormalize", ctypes.c_int32)]


_lib_handle = None


def library_available() -> bool:
    return os.path.exists(LIB_PATH)


def _lib():
    global _lib_handle
    if _lib_handle is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m sparse_mixture_experts_rms_b200.build` "
                "(nvcc, sm_100a). There is no non-CUDA path.")
        lib = ctypes.CDLL(LIB_PATH)
        P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        cfgp = ctypes.POINTER(_Config)
        lib.moe_status_string.restype = ctypes.c_char_p
        lib.moe_status_string.argtypes = [ctypes.c_int]
        lib.moe_capacity.restype = ctypes.c_int64
        lib.moe_capacity.argtypes = [cfgp]
        lib.moe_expert_offsets.restype = ctypes.c_int32
        lib.moe_expert_offsets.argtypes = [P, P, ctypes.c_int32, P, ctypes.c_int32]
        lib.moe_max_kept.restype = ctypes.c_int64
        lib.moe_max_kept.argtypes = [cfgp]
        lib.moe_workspace_size.restype = SZ
        lib.moe_workspace_size.argtypes = [cfgp]
        lib.moe_workspace_init.restype = ctypes.c_int
        lib.moe_workspace_init.argtypes = [P, SZ, P]
        lib.moe_get_device_error.restype = ctypes.c_int
        lib.moe_get_device_error.argtypes = [P, SZ, P, ctypes.POINTER(ctypes.c_uint32)]
        lib.moe_set_wait_limit.restype = ctypes.c_int
        lib.moe_set_wait_limit.argtypes = [P, SZ, ctypes.c_uint32, P]
        lib.moe_route.restype = ctypes.c_int
        lib.moe_route.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, SZ, P]
        lib.moe_router_stats.restype = ctypes.c_int
        lib.moe_router_stats.argtypes = [cfgp, P, P, P, P, P]
        lib.moe_dispatch.restype = ctypes.c_int
        lib.moe_dispatch.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, SZ, P]
        lib.moe_dispatch_noalloc.restype = ctypes.c_int
        lib.moe_dispatch_noalloc.argtypes = [cfgp, P, P, P, P, P, P, P, P, P]
        lib.moe_experts_fwd.restype = ctypes.c_int
        lib.moe_experts_fwd.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, SZ, P]
        lib.moe_experts_up.restype = ctypes.c_int
        lib.moe_experts_up.argtypes = [cfgp, P, P, P, P, P, P, P, SZ, P]
        lib.moe_experts_down.restype = ctypes.c_int
        lib.moe_experts_down.argtypes = [cfgp, P, P, P, P, P, P, SZ, P]
        lib.moe_combine.restype = ctypes.c_int
        lib.moe_combine.argtypes = [cfgp, P, P, P, P]
        lib.moe_layer_fwd.restype = ctypes.c_int
        lib.moe_layer_fwd.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
        lib.moe_layer_fwd_gather.restype = ctypes.c_int
        lib.moe_layer_fwd_gather.argtypes = lib.moe_layer_fwd.argtypes
        lib.moe_mx_weights_size.restype = SZ
        lib.moe_mx_weights_size.argtypes = [cfgp]
        lib.moe_quantize_weights_mx.restype = ctypes.c_int
        lib.moe_quantize_weights_mx.argtypes = [cfgp, P, P, P, P, SZ, P]
        lib.moe_mx_workspace_size.restype = SZ
        lib.moe_mx_workspace_size.argtypes = [cfgp]
        lib.moe_mx_rows.restype = ctypes.c_int64
        lib.moe_mx_rows.argtypes = [cfgp]
        lib.moe_layer_fwd_mx.restype = ctypes.c_int
        lib.moe_layer_fwd_mx.argtypes = [cfgp, P, P, P, P, P, SZ, P, P, SZ, P]
        lib.moe_mx_part.restype = ctypes.c_int
        lib.moe_mx_part.argtypes = [cfgp, P, P, SZ, ctypes.c_int32, ctypes.POINTER(ctypes.c_void_p)]
        lib.moe_host_workspace_size.restype = SZ
        lib.moe_host_workspace_size.argtypes = [cfgp, ctypes.c_int32]
        lib.moe_host_chunks.restype = ctypes.c_int32
        lib.moe_host_chunks.argtypes = [cfgp, ctypes.c_int32]
        lib.moe_layer_fwd_host.restype = ctypes.c_int
        lib.moe_layer_fwd_host.argtypes = [cfgp, P, P, P, P, P, P, P, P, ctypes.c_int32, P, SZ, P]
        lib.moe_train_workspace_size.restype = SZ
        lib.moe_train_workspace_size.argtypes = [cfgp]
        lib.moe_train_rows.restype = ctypes.c_int64
        lib.moe_train_rows.argtypes = [cfgp]
        lib.moe_train_saved.restype = ctypes.c_int
        lib.moe_train_saved.argtypes = [cfgp, P, SZ, ctypes.c_int32, ctypes.POINTER(ctypes.c_void_p)]
        lib.moe_layer_fwd_train.restype = ctypes.c_int
        lib.moe_layer_fwd_train.argtypes = [cfgp, P, P, P, P, P, P, P, P, P, SZ, P]
        lib.moe_layer_bwd.restype = ctypes.c_int
        lib.moe_layer_bwd.argtypes = [cfgp] + [P] * 15 + [P, SZ, P]
        _lib_handle = lib
    return _lib_handle


def _status_text(status: int) -> str:
    try:
        return _lib().moe_status_string(int(status)).decode()
    except Exception:  # library missing: still describe the code
        return f"status {status}"


def ffn_offsets_from_sizes(expert_sizes: Sequence[Tuple[int, int]], max_experts: int = 64) -> List[int]:
    """Cumulative expert column offsets [E+1] from ``[(count, size), ...]``,
    computed by the library (moe_expert_offsets: sizes rounded up to 128,
    repeated count times, running sums)."""
    n = len(expert_sizes)
    counts = (ctypes.c_int32 * max(n, 1))(*[int(c) for c, _ in expert_sizes])
    sizes = (ctypes.c_int32 * max(n, 1))(*[int(s) for _, s in expert_sizes])
    offs = (ctypes.c_int32 * (max_experts + 1))()
    E = _lib().moe_expert_offsets(counts, sizes, n, offs, max_experts)
    if E < 0:
        raise ValueError(f"invalid expert sizes {list(expert_sizes)} (counts >= 0, sizes >= 1, "
                         f"at most {max_experts} experts)")
    return [int(offs[i]) for i in range(E + 1)]


@dataclass
class MoEConfig:
    """Layer configuration (mirrors ``moe_config_t``)."""

    T: int
    d_model: int
    E: int
    k: int
    ffn_offsets: List[int]
    capacity_factor: float = 0.0
    eps: float = 1e-5
    renormalize: bool = False
    _c: Optional[_Config] = field(default=None, repr=False, compare=False)
    _offs: Optional[ctypes.Array] = field(default=None, repr=False, compare=False)

    def c(self) -> _Config:
        self._offs = (ctypes.c_int32 * len(self.ffn_offsets))(*[int(v) for v in self.ffn_offsets])
        self._c = _Config(int(self.T), int(self.d_model), int(self.E), int(self.k),
                          ctypes.cast(self._offs, ctypes.POINTER(ctypes.c_int32)),
                          float(self.capacity_factor), float(self.eps), int(bool(self.renormalize)))
        return self._c

    @property
    def F(self) -> int:
        return int(self.ffn_offsets[-1])


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, shape=None) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(0)
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(int(s.cuda_stream))


def _check(status: int, what: str):
    if status != MOE_OK:
        raise MoEError(status, what)


# ------------------------------------------------------------------ C ABI
def moe_status_string(status: int) -> str:
    return _lib().moe_status_string(int(status)).decode()


def moe_capacity(cfg: MoEConfig) -> int:
    return int(_lib().moe_capacity(ctypes.byref(cfg.c())))


def moe_max_kept(cfg: MoEConfig) -> int:
    return int(_lib().moe_max_kept(ctypes.byref(cfg.c())))


def moe_workspace_size(cfg: MoEConfig) -> int:
    return int(_lib().moe_workspace_size(ctypes.byref(cfg.c())))


def alloc_workspace(cfg: MoEConfig, device=None, stream=None) -> torch.Tensor:
    """A zero-initialised workspace of ``moe_workspace_size(cfg)`` bytes (torch-owned)."""
    n = moe_workspace_size(cfg)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    moe_workspace_init(ws, stream)
    return ws


def moe_workspace_init(ws: torch.Tensor, stream=None) -> None:
    _check(_lib().moe_workspace_init(_ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream)),
           "moe_workspace_init")


def moe_get_device_error(ws: torch.Tensor, stream=None, raise_on_error: bool = True) -> int:
    code = ctypes.c_uint32(0)
    st = _lib().moe_get_device_error(_ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream),
                                     ctypes.byref(code))
    if st == MOE_ERR_DEVICE:
        if raise_on_error:
            raise MoEError(st, "moe_get_device_error", int(code.value))
        return int(code.value)
    _check(st, "moe_get_device_error")
    return int(code.value)


def moe_set_wait_limit(ws: torch.Tensor, limit_ns: int, stream=None) -> None:
    """Limit (ns) of the bounded pipeline waits of the kernels that later run on
    ``ws``; 0 restores the default (4 s).  For tests of the timeout path."""
    _check(_lib().moe_set_wait_limit(_ptr(ws, "ws", torch.uint8), ws.numel(), int(limit_ns), _stream(stream)),
           "moe_set_wait_limit")


def moe_route(cfg: MoEConfig, x, gamma, Wr, bias, expert_idx, gate, r, logits,
              ws: torch.Tensor, prob_mean=None, stream=None) -> None:
    T, d, E, k = cfg.T, cfg.d_model, cfg.E, cfg.k
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    st = _lib().moe_route(
        ctypes.byref(cfg.c()), _ptr(x, "x", bf, (T, d)), _ptr(gamma, "gamma", bf, (d,)),
        _ptr(Wr, "Wr", bf, (d, E)), _ptr(bias, "bias", f32, (E,)),
        _ptr(expert_idx, "expert_idx", i32, (T, k)), _ptr(gate, "gate", f32, (T, k)),
        _ptr(r, "r", f32, (T,)), _ptr(logits, "logits", f32, (T, E)),
        _ptr(prob_mean, "prob_mean", f32, (E,)),
        _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream))
    _check(st, "moe_route")


def moe_router_stats(cfg: MoEConfig, prob_mean, counts, expert_offsets, stats, stream=None) -> None:
    """stats[4] = {E*sum f_e*P_e, CV^2(P), CV^2(counts), dropped fraction} on the device."""
    E = cfg.E
    st = _lib().moe_router_stats(
        ctypes.byref(cfg.c()), _ptr(prob_mean, "prob_mean", torch.float32, (E,)),
        _ptr(counts, "counts", torch.int32, (E,)),
        _ptr(expert_offsets, "expert_offsets", torch.int32, (E + 1,)),
        _ptr(stats, "stats", torch.float32, (4,)), _stream(stream))
    _check(st, "moe_router_stats")


def moe_dispatch(cfg: MoEConfig, expert_idx, x, gamma, counts, expert_offsets, perm, inv_perm,
                 x_perm, ws: torch.Tensor, stream=None) -> None:
    T, d, E, k = cfg.T, cfg.d_model, cfg.E, cfg.k
    i32, bf = torch.int32, torch.bfloat16
    if x_perm is not None and (x_perm.dim() != 2 or x_perm.shape[1] != d
                               or x_perm.shape[0] < moe_max_kept(cfg)):
        raise ValueError("x_perm must be [>= moe_max_kept(cfg), d]")
    if perm is not None and perm.numel() < moe_max_kept(cfg):
        raise ValueError("perm must hold >= moe_max_kept(cfg) entries")
    st = _lib().moe_dispatch(
        ctypes.byref(cfg.c()), _ptr(expert_idx, "expert_idx", i32, (T, k)), _ptr(x, "x", bf, (T, d)),
        _ptr(gamma, "gamma", bf, (d,)), _ptr(counts, "counts", i32, (E,)),
        _ptr(expert_offsets, "expert_offsets", i32, (E + 1,)), _ptr(perm, "perm", i32),
        _ptr(inv_perm, "inv_perm", i32, (T * k,)), _ptr(x_perm, "x_perm", bf),
        _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream))
    _check(st, "moe_dispatch")


def moe_dispatch_noalloc(cfg: MoEConfig, expert_idx, x, gamma, counts, expert_offsets, perm,
                         inv_perm, x_perm, stream=None) -> None:
    """moe_dispatch without a workspace, for callers that cannot allocate device
    memory: the scratch is a fixed array inside the library (T*k <= 2^20)."""
    T, d, E, k = cfg.T, cfg.d_model, cfg.E, cfg.k
    i32, bf = torch.int32, torch.bfloat16
    if x_perm is not None and (x_perm.dim() != 2 or x_perm.shape[1] != d
                               or x_perm.shape[0] < moe_max_kept(cfg)):
        raise ValueError("x_perm must be [>= moe_max_kept(cfg), d]")
    if perm is not None and perm.numel() < moe_max_kept(cfg):
        raise ValueError("perm must hold >= moe_max_kept(cfg) entries")
    st = _lib().moe_dispatch_noalloc(
        ctypes.byref(cfg.c()), _ptr(expert_idx, "expert_idx", i32, (T, k)), _ptr(x, "x", bf, (T, d)),
        _ptr(gamma, "gamma", bf, (d,)), _ptr(counts, "counts", i32, (E,)),
        _ptr(expert_offsets, "expert_offsets", i32, (E + 1,)), _ptr(perm, "perm", i32),
        _ptr(inv_perm, "inv_perm", i32, (T * k,)), _ptr(x_perm, "x_perm", bf), _stream(stream))
    _check(st, "moe_dispatch_noalloc")


def moe_experts_fwd(cfg: MoEConfig, x_perm, r, gate, perm, expert_offsets, W1, W3, W2, y,
                    ws: torch.Tensor, stream=None) -> None:
    T, d, E, k, F = cfg.T, cfg.d_model, cfg.E, cfg.k, cfg.F
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    mk = moe_max_kept(cfg)
    for name, t in (("x_perm", x_perm), ("y", y)):
        if t.dim() != 2 or t.shape[1] != d or t.shape[0] < mk:
            raise ValueError(f"{name} must be [>= moe_max_kept(cfg), d]")
    if perm.numel() < mk:
        raise ValueError("perm must hold >= moe_max_kept(cfg) entries")
    st = _lib().moe_experts_fwd(
        ctypes.byref(cfg.c()), _ptr(x_perm, "x_perm", bf), _ptr(r, "r", f32, (T,)),
        _ptr(gate, "gate", f32, (T, k)), _ptr(perm, "perm", i32),
        _ptr(expert_offsets, "expert_offsets", i32, (E + 1,)), _ptr(W1, "W1", bf, (d, F)),
        _ptr(W3, "W3", bf, (d, F)), _ptr(W2, "W2", bf, (F, d)), _ptr(y, "y", bf),
        _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream))
    _check(st, "moe_experts_fwd")


def moe_experts_up(cfg: MoEConfig, x_perm, r, perm, expert_offsets, W1, W3, ws: torch.Tensor,
                   stream=None) -> None:
    T, d, E, F = cfg.T, cfg.d_model, cfg.E, cfg.F
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    mk = moe_max_kept(cfg)
    if x_perm.dim() != 2 or x_perm.shape[1] != d or x_perm.shape[0] < mk:
        raise ValueError("x_perm must be [>= moe_max_kept(cfg), d]")
    if perm.numel() < mk:
        raise ValueError("perm must hold >= moe_max_kept(cfg) entries")
    st = _lib().moe_experts_up(
        ctypes.byref(cfg.c()), _ptr(x_perm, "x_perm", bf), _ptr(r, "r", f32, (T,)),
        _ptr(perm, "perm", i32), _ptr(expert_offsets, "expert_offsets", i32, (E + 1,)),
        _ptr(W1, "W1", bf, (d, F)), _ptr(W3, "W3", bf, (d, F)),
        _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream))
    _check(st, "moe_experts_up")


def moe_experts_down(cfg: MoEConfig, gate, perm, expert_offsets, W2, y, ws: torch.Tensor,
                     stream=None) -> None:
    T, d, E, k, F = cfg.T, cfg.d_model, cfg.E, cfg.k, cfg.F
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    mk = moe_max_kept(cfg)
    if y.dim() != 2 or y.shape[1] != d or y.shape[0] < mk:
        raise ValueError("y must be [>= moe_max_kept(cfg), d]")
    if perm.numel() < mk:
        raise ValueError("perm must hold >= moe_max_kept(cfg) entries")
    st = _lib().moe_experts_down(
        ctypes.byref(cfg.c()), _ptr(gate, "gate", f32, (T, k)), _ptr(perm, "perm", i32),
        _ptr(expert_offsets, "expert_offsets", i32, (E + 1,)), _ptr(W2, "W2", bf, (F, d)),
        _ptr(y, "y", bf), _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream))
    _check(st, "moe_experts_down")


def moe_combine(cfg: MoEConfig, y, inv_perm, out, stream=None) -> None:
    T, d, k = cfg.T, cfg.d_model, cfg.k
    if y.dim() != 2 or y.shape[1] != d:
        raise ValueError("y must be [rows, d]")
    st = _lib().moe_combine(ctypes.byref(cfg.c()), _ptr(y, "y", torch.bfloat16),
                            _ptr(inv_perm, "inv_perm", torch.int32, (T * k,)),
                            _ptr(out, "out", torch.bfloat16, (T, d)), _stream(stream))
    _check(st, "moe_combine")


def moe_layer_fwd(cfg: MoEConfig, x, gamma, Wr, bias, W1, W3, W2, out, ws: torch.Tensor,
                  expert_idx=None, gate=None, r=None, counts=None, prob_mean=None, stats=None,
                  stream=None, gather: bool = False) -> None:
    """The layer; with `gather`, through moe_layer_fwd_gather (the row gather in
    GEMM 1's A load instead of a permuted copy of x)."""
    T, d, E, k, F = cfg.T, cfg.d_model, cfg.E, cfg.k, cfg.F
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    name = "moe_layer_fwd_gather" if gather else "moe_layer_fwd"
    st = getattr(_lib(), name)(
        ctypes.byref(cfg.c()), _ptr(x, "x", bf, (T, d)), _ptr(gamma, "gamma", bf, (d,)),
        _ptr(Wr, "Wr", bf, (d, E)), _ptr(bias, "bias", f32, (E,)), _ptr(W1, "W1", bf, (d, F)),
        _ptr(W3, "W3", bf, (d, F)), _ptr(W2, "W2", bf, (F, d)), _ptr(out, "out", bf, (T, d)),
        _ptr(expert_idx, "expert_idx", i32, (T, k)), _ptr(gate, "gate", f32, (T, k)),
        _ptr(r, "r", f32, (T,)), _ptr(counts, "counts", i32, (E,)),
        _ptr(prob_mean, "prob_mean", f32, (E,)), _ptr(stats, "stats", f32, (4,)),
        _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream))
    _check(st, name)


# ------------------------------------------------------------------ MXFP8 expert GEMMs
def moe_mx_weights_size(cfg: MoEConfig) -> int:
    return int(_lib().moe_mx_weights_size(ctypes.byref(cfg.c())))


def moe_mx_workspace_size(cfg: MoEConfig) -> int:
    return int(_lib().moe_mx_workspace_size(ctypes.byref(cfg.c())))


def moe_mx_rows(cfg: MoEConfig) -> int:
    return int(_lib().moe_mx_rows(ctypes.byref(cfg.c())))


def moe_quantize_weights_mx(cfg: MoEConfig, W1, W3, W2, wq: torch.Tensor, stream=None) -> None:
    d, F = cfg.d_model, cfg.F
    bf = torch.bfloat16
    st = _lib().moe_quantize_weights_mx(
        ctypes.byref(cfg.c()), _ptr(W1, "W1", bf, (d, F)), _ptr(W3, "W3", bf, (d, F)), _ptr(W2, "W2", bf, (F, d)),
        _ptr(wq, "wq", torch.uint8), wq.numel(), _stream(stream))
    _check(st, "moe_quantize_weights_mx")


def alloc_mx_weights(cfg: MoEConfig, W1, W3, W2, stream=None) -> torch.Tensor:
    """The MXFP8 copies of W1, W3, W2 (torch-owned device buffer)."""
    n = moe_mx_weights_size(cfg)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_mx_weights_size")
    wq = torch.empty(n, dtype=torch.uint8, device=W1.device)
    moe_quantize_weights_mx(cfg, W1, W3, W2, wq, stream)
    return wq


def alloc_mx_workspace(cfg: MoEConfig, device=None, stream=None) -> torch.Tensor:
    n = moe_mx_workspace_size(cfg)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_mx_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    moe_workspace_init(ws, stream)
    return ws


def moe_layer_fwd_mx(cfg: MoEConfig, x, gamma, Wr, bias, wq: torch.Tensor, out, ws: torch.Tensor,
                     stream=None) -> None:
    T, d, E = cfg.T, cfg.d_model, cfg.E
    bf, f32 = torch.bfloat16, torch.float32
    st = _lib().moe_layer_fwd_mx(
        ctypes.byref(cfg.c()), _ptr(x, "x", bf, (T, d)), _ptr(gamma, "gamma", bf, (d,)),
        _ptr(Wr, "Wr", bf, (d, E)), _ptr(bias, "bias", f32, (E,)), _ptr(wq, "wq", torch.uint8), wq.numel(),
        _ptr(out, "out", bf, (T, d)), _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream))
    _check(st, "moe_layer_fwd_mx")


def mx_part_view(cfg: MoEConfig, wq: torch.Tensor, ws: Optional[torch.Tensor], name: str) -> torch.Tensor:
    """A view of one MX buffer (weights parts from wq, the rest from ws)."""
    T, d, E, k, F = cfg.T, cfg.d_model, cfg.E, cfg.k, cfg.F
    fmax = max(b - a for a, b in zip(cfg.ffn_offsets[:-1], cfg.ffn_offsets[1:]))
    rows = moe_mx_rows(cfg)
    u8, i32, f32 = torch.uint8, torch.int32, torch.float32
    spec = {"W1": (u8, (F, d)), "W3": (u8, (F, d)), "W2": (u8, (d, F)),
            "SF1": (u8, ((F // 128) * (d // 128) * 512,)), "SF3": (u8, ((F // 128) * (d // 128) * 512,)),
            "SF2": (u8, ((d // 128) * (F // 128) * 512,)),
            "X8": (u8, (rows, d)), "XSF": (u8, ((rows // 128) * (d // 128) * 512,)),
            "H8": (u8, (rows, fmax)), "HSF": (u8, ((rows // 128) * (fmax // 128) * 512,)),
            "PERM": (i32, (rows,)), "OFFSETS": (i32, (E + 1,)), "IDX": (i32, (T, k)),
            "GATE": (f32, (T, k)), "R": (f32, (T,))}[name]
    out = ctypes.c_void_p(0)
    base = wq if MOE_MX[name] <= MOE_MX["SF2"] else ws
    st = _lib().moe_mx_part(ctypes.byref(cfg.c()), _ptr(wq, "wq", torch.uint8),
                            _ptr(ws, "ws", torch.uint8) if ws is not None else ctypes.c_void_p(0),
                            ws.numel() if ws is not None else 0, MOE_MX[name], ctypes.byref(out))
    _check(st, "moe_mx_part")
    dtype, shape = spec
    off = int(out.value) - base.data_ptr()
    n = 1
    for v in shape:
        n *= v
    return base[off:off + n * torch.empty(0, dtype=dtype).element_size()].view(dtype).view(shape)


# ------------------------------------------------------------------ host buffers
def _host_ptr(t: torch.Tensor, name: str, dtype, shape) -> ctypes.c_void_p:
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")
    return ctypes.c_void_p(t.data_ptr())


def moe_host_workspace_size(cfg: MoEConfig, n_chunks: int = 0) -> int:
    return int(_lib().moe_host_workspace_size(ctypes.byref(cfg.c()), int(n_chunks)))


def moe_host_chunks(cfg: MoEConfig, n_chunks: int = 0) -> int:
    return int(_lib().moe_host_chunks(ctypes.byref(cfg.c()), int(n_chunks)))


def alloc_host_workspace(cfg: MoEConfig, n_chunks: int = 0, device=None, stream=None) -> torch.Tensor:
    n = moe_host_workspace_size(cfg, n_chunks)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_host_workspace_size")
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    moe_workspace_init(ws, stream)
    return ws


def moe_layer_fwd_host(cfg: MoEConfig, x_host, gamma, Wr, bias, W1, W3, W2, out_host,
                       ws: torch.Tensor, n_chunks: int = 0, stream=None) -> None:
    """The layer on host x/out (pin them for overlapped copies); see moe.h."""
    T, d, E, F = cfg.T, cfg.d_model, cfg.E, cfg.F
    bf, f32 = torch.bfloat16, torch.float32
    st = _lib().moe_layer_fwd_host(
        ctypes.byref(cfg.c()), _host_ptr(x_host, "x_host", bf, (T, d)), _ptr(gamma, "gamma", bf, (d,)),
        _ptr(Wr, "Wr", bf, (d, E)), _ptr(bias, "bias", f32, (E,)), _ptr(W1, "W1", bf, (d, F)),
        _ptr(W3, "W3", bf, (d, F)), _ptr(W2, "W2", bf, (F, d)), _host_ptr(out_host, "out_host", bf, (T, d)),
        int(n_chunks), _ptr(ws, "ws", torch.uint8), ws.numel(), _stream(stream))
    _check(st, "moe_layer_fwd_host")


# ------------------------------------------------------------------ training
def moe_train_workspace_size(cfg: MoEConfig) -> int:
    return int(_lib().moe_train_workspace_size(ctypes.byref(cfg.c())))


def moe_train_rows(cfg: MoEConfig) -> int:
    return int(_lib().moe_train_rows(ctypes.byref(cfg.c())))


def alloc_train_workspace(cfg: MoEConfig, device=None, stream=None) -> torch.Tensor:
    """A training workspace of ``moe_train_workspace_size(cfg)`` bytes (torch-owned)."""
    n = moe_train_workspace_size(cfg)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_train_workspace_size")
    tws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    moe_workspace_init(tws, stream)
    return tws


def moe_train_saved(cfg: MoEConfig, tws: torch.Tensor, name: str) -> int:
    """Device address of a saved tensor inside the training workspace."""
    out = ctypes.c_void_p(0)
    st = _lib().moe_train_saved(ctypes.byref(cfg.c()), _ptr(tws, "tws", torch.uint8), tws.numel(),
                                MOE_SAVED[name], ctypes.byref(out))
    _check(st, "moe_train_saved")
    return int(out.value)


def train_saved_view(cfg: MoEConfig, tws: torch.Tensor, name: str) -> torch.Tensor:
    """A view of a saved tensor (shares the workspace's memory)."""
    T, d, E, k = cfg.T, cfg.d_model, cfg.E, cfg.k
    rows = moe_train_rows(cfg)
    fmax = max(b - a for a, b in zip(cfg.ffn_offsets[:-1], cfg.ffn_offsets[1:]))
    spec = {"r": (torch.float32, (T,)), "idx": (torch.int32, (T, k)), "gate": (torch.float32, (T, k)),
            "logits": (torch.float32, (T, E)), "offsets": (torch.int32, (E + 1,)),
            "perm": (torch.int32, (rows,)), "inv_perm": (torch.int32, (T * k,)),
            "U": (torch.bfloat16, (rows, fmax)), "V": (torch.bfloat16, (rows, fmax)),
            "H": (torch.bfloat16, (rows, fmax)), "y": (torch.bfloat16, (rows, d)),
            "dgate": (torch.float32, (T * k,)), "dr": (torch.float32, (T,)),
            "counts": (torch.int32, (E,))}[name]
    dtype, shape = spec
    off = moe_train_saved(cfg, tws, name) - tws.data_ptr()
    n = 1
    for v in shape:
        n *= v
    return tws[off:off + n * torch.empty(0, dtype=dtype).element_size()].view(dtype).view(shape)


def moe_layer_fwd_train(cfg: MoEConfig, x, gamma, Wr, bias, W1, W3, W2, out, tws: torch.Tensor,
                        stream=None) -> None:
    T, d, E, F = cfg.T, cfg.d_model, cfg.E, cfg.F
    bf, f32 = torch.bfloat16, torch.float32
    st = _lib().moe_layer_fwd_train(
        ctypes.byref(cfg.c()), _ptr(x, "x", bf, (T, d)), _ptr(gamma, "gamma", bf, (d,)),
        _ptr(Wr, "Wr", bf, (d, E)), _ptr(bias, "bias", f32, (E,)), _ptr(W1, "W1", bf, (d, F)),
        _ptr(W3, "W3", bf, (d, F)), _ptr(W2, "W2", bf, (F, d)), _ptr(out, "out", bf, (T, d)),
        _ptr(tws, "tws", torch.uint8), tws.numel(), _stream(stream))
    _check(st, "moe_layer_fwd_train")


def moe_layer_bwd(cfg: MoEConfig, x, gamma, Wr, bias, W1, W3, W2, dout, dx, dgamma, dWr, dbias,
                  dW1, dW3, dW2, tws: torch.Tensor, stream=None) -> None:
    T, d, E, F = cfg.T, cfg.d_model, cfg.E, cfg.F
    bf, f32 = torch.bfloat16, torch.float32
    st = _lib().moe_layer_bwd(
        ctypes.byref(cfg.c()), _ptr(x, "x", bf, (T, d)), _ptr(gamma, "gamma", bf, (d,)),
        _ptr(Wr, "Wr", bf, (d, E)), _ptr(bias, "bias", f32, (E,)), _ptr(W1, "W1", bf, (d, F)),
        _ptr(W3, "W3", bf, (d, F)), _ptr(W2, "W2", bf, (F, d)), _ptr(dout, "dout", bf, (T, d)),
        _ptr(dx, "dx", f32, (T, d)), _ptr(dgamma, "dgamma", f32, (d,)), _ptr(dWr, "dWr", f32, (d, E)),
        _ptr(dbias, "dbias", f32, (E,)), _ptr(dW1, "dW1", f32, (d, F)), _ptr(dW3, "dW3", f32, (d, F)),
        _ptr(dW2, "dW2", f32, (F, d)), _ptr(tws, "tws", torch.uint8), tws.numel(), _stream(stream))
    _check(st, "moe_layer_bwd")


class MoELayer:
    """Holds a layer's weights and workspace; ``forward(x)`` calls moe_layer_fwd."""

    def __init__(self, cfg: MoEConfig, gamma, Wr, bias, W1, W3, W2):
        self.cfg = cfg
        self.gamma, self.Wr, self.bias = gamma, Wr, bias
        self.W1, self.W3, self.W2 = W1, W3, W2
        self.ws = alloc_workspace(cfg, device=gamma.device)

    def forward(self, x, out=None, expert_idx=None, gate=None, r=None, counts=None, prob_mean=None,
                stats=None, stream=None):
        c = self.cfg
        if out is None:
            out = torch.empty((c.T, c.d_model), dtype=torch.bfloat16, device=x.device)
        moe_layer_fwd(c, x, self.gamma, self.Wr, self.bias, self.W1, self.W3, self.W2, out, self.ws,
                      expert_idx=expert_idx, gate=gate, r=r, counts=counts, prob_mean=prob_mean,
                      stats=stats, stream=stream)
        return out

    __call__ = forward


class _MoETrainFn(torch.autograd.Function):
    """autograd glue: forward = moe_layer_fwd_train, backward = moe_layer_bwd.
    Gradients come back in fp32 and are cast to each input's dtype."""

    @staticmethod
    def forward(ctx, cfg, tws, x, gamma, Wr, bias, W1, W3, W2):
        out = torch.empty((cfg.T, cfg.d_model), dtype=torch.bfloat16, device=x.device)
        moe_layer_fwd_train(cfg, x, gamma, Wr, bias, W1, W3, W2, out, tws)
        ctx.cfg, ctx.tws = cfg, tws
        ctx.save_for_backward(x, gamma, Wr, bias if bias is not None else torch.empty(0), W1, W3, W2)
        ctx.has_bias = bias is not None
        return out

    @staticmethod
    def backward(ctx, dout):
        cfg, tws = ctx.cfg, ctx.tws
        x, gamma, Wr, bias, W1, W3, W2 = ctx.saved_tensors
        bias = bias if ctx.has_bias else None
        T, d, E, F = cfg.T, cfg.d_model, cfg.E, cfg.F
        f32 = dict(dtype=torch.float32, device=x.device)
        g = [torch.empty((T, d), **f32), torch.empty((d,), **f32), torch.empty((d, E), **f32),
             torch.empty((E,), **f32), torch.empty((d, F), **f32), torch.empty((d, F), **f32),
             torch.empty((F, d), **f32)]
        moe_layer_bwd(cfg, x, gamma, Wr, bias, W1, W3, W2, dout.to(torch.bfloat16).contiguous(), *g, tws)
        dx, dgamma, dWr, dbias, dW1, dW3, dW2 = g
        return (None, None, dx.to(x.dtype), dgamma.to(gamma.dtype), dWr.to(Wr.dtype),
                dbias if ctx.has_bias else None, dW1.to(W1.dtype), dW3.to(W3.dtype), dW2.to(W2.dtype))


class MoETrainLayer:
    """A layer for training: ``forward(x)`` runs the training forward and
    returns an output whose backward runs moe_layer_bwd (one forward in flight
    per layer: the training workspace holds one forward's saved state)."""

    def __init__(self, cfg: MoEConfig, gamma, Wr, bias, W1, W3, W2):
        self.cfg = cfg
        self.gamma, self.Wr, self.bias = gamma, Wr, bias
        self.W1, self.W3, self.W2 = W1, W3, W2
        self.tws = alloc_train_workspace(cfg, device=gamma.device)

    def forward(self, x):
        return _MoETrainFn.apply(self.cfg, self.tws, x, self.gamma, self.Wr, self.bias, self.W1, self.W3, self.W2)

    __call__ = forward
