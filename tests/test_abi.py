"""The C ABI library loads, exports every declared symbol, and validates its
arguments on the host before touching a device (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import sparse_mixture_experts_rms_b200 as moe
from sparse_mixture_experts_rms_b200 import build as moe_build
from oracle import moe_oracle as O
import moe_workloads as mw

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe._lib()


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", src)))


def test_header_declares_every_binding_name():
    assert _declared_symbols() == sorted(moe.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_symbols():
        assert hasattr(lib, name), name


def _cfg(w: mw.Workload, **kw):
    offs = moe.ffn_offsets_from_sizes(w.expert_sizes)
    c = moe.MoEConfig(T=w.T, d_model=w.d_model, E=w.E, k=w.k, ffn_offsets=offs,
                      capacity_factor=w.capacity_factor, eps=w.eps)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("name", mw.WORKLOAD_ORDER)
def test_capacity_and_sizes_match_oracle(lib, name):
    w = mw.WORKLOADS[name]
    c = _cfg(w)
    C = O.capacity(w.T, w.k, w.E, float(np.float32(w.capacity_factor)))
    assert moe.moe_capacity(c) == (-1 if C is None else C)
    mk = w.T * w.k if C is None else min(w.T * w.k, w.E * C)
    assert moe.moe_max_kept(c) == mk
    ws = moe.moe_workspace_size(c)
    widths = O.expert_widths(w.expert_sizes)
    assert c.ffn_offsets == O.expert_offsets(widths)
    # at least the expert intermediates: x_perm, H (max width), y
    assert ws >= mk * (2 * w.d_model + max(widths)) * 2


def test_switch_capacity_is_320(lib):
    assert moe.moe_capacity(_cfg(mw.WORKLOADS["switch_capacity"])) == 320


def test_capacity_rounding_on_fp32_factor(lib):
    w = mw.WORKLOADS["tiny"]
    for cf in (0.3, 1.1, 1.25, 2.0, 0.01):
        c = _cfg(w, capacity_factor=cf)
        assert moe.moe_capacity(c) == O.capacity(w.T, w.k, w.E, float(np.float32(cf)))


@pytest.mark.parametrize("bad", [
    dict(k=0), dict(k=9), dict(E=0), dict(d_model=100), dict(d_model=0), dict(T=-1),
    dict(eps=float("nan")), dict(eps=-1.0), dict(capacity_factor=float("inf")),
])
def test_invalid_config_rejected(lib, bad):
    c = _cfg(mw.WORKLOADS["tiny"], **bad)
    assert moe.moe_workspace_size(c) == 0
    assert moe.moe_capacity(c) == -1


def test_invalid_widths_rejected(lib):
    base = mw.WORKLOADS["tiny"]
    for offs in ([0, 256, 300, 512, 768, 1024, 1280, 1536, 1792],   # width 44
                 [1, 257, 513, 769, 1025, 1281, 1537, 1793, 2049],  # offsets[0] != 0
                 [0, 256, 256, 512, 768, 1024, 1280, 1536, 1792]):  # zero width
        c = _cfg(base, ffn_offsets=offs)
        assert moe.moe_workspace_size(c) == 0


def test_too_many_experts_unsupported(lib):
    c = moe.MoEConfig(T=16, d_model=128, E=65, k=2, ffn_offsets=[128 * i for i in range(66)])
    assert moe.moe_workspace_size(c) == 0


def _call_layer(lib, cfg, ptrs, ws_ptr, ws_bytes, entry="moe_layer_fwd"):
    P = ctypes.c_void_p
    return getattr(lib, entry)(ctypes.byref(cfg.c()), *[P(p) for p in ptrs], P(0), P(0), P(0), P(0),
                               P(0), P(0), P(ws_ptr), ws_bytes, P(0))


@pytest.mark.parametrize("entry", ["moe_layer_fwd", "moe_layer_fwd_gather"])
def test_layer_argument_errors_before_any_device_work(lib, entry):
    _call = lambda *a: _call_layer(*a, entry=entry)
    c = _cfg(mw.WORKLOADS["tiny"])
    good = [4096 * (i + 1) for i in range(8)]   # fake, aligned, never dereferenced
    wsz = moe.moe_workspace_size(c)
    # null tensor
    bad = list(good); bad[0] = 0
    assert _call(lib, c, bad, 1 << 20, wsz) == moe.MOE_ERR_INVALID_ARG
    # misaligned bf16 matrix
    bad = list(good); bad[4] += 8
    assert _call(lib, c, bad, 1 << 20, wsz) == moe.MOE_ERR_ALIGNMENT
    # workspace too small / missing / misaligned
    assert _call(lib, c, good, 1 << 20, wsz - 1) == moe.MOE_ERR_WORKSPACE
    assert _call(lib, c, good, 0, wsz) == moe.MOE_ERR_WORKSPACE
    assert _call(lib, c, good, (1 << 20) + 16, wsz) == moe.MOE_ERR_ALIGNMENT
    # k > E
    ck = _cfg(mw.WORKLOADS["tiny"], k=9)
    assert _call(lib, ck, good, 1 << 20, wsz) == moe.MOE_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
@pytest.mark.parametrize("entry", ["moe_layer_fwd", "moe_layer_fwd_gather"])
def test_valid_call_without_device_reports_no_device(lib, entry):
    c = _cfg(mw.WORKLOADS["tiny"])
    good = [4096 * (i + 1) for i in range(8)]
    wsz = moe.moe_workspace_size(c)
    assert _call_layer(lib, c, good, 1 << 20, wsz, entry=entry) == moe.MOE_ERR_NO_DEVICE


def test_wait_limit_rejects_bad_workspace_before_device_work(lib):
    P = ctypes.c_void_p
    assert lib.moe_set_wait_limit(P(0), 1 << 20, 5, P(0)) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_set_wait_limit(P(1 << 20), 255, 5, P(0)) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_set_wait_limit(P((1 << 20) + 16), 1 << 20, 5, P(0)) == moe.MOE_ERR_ALIGNMENT


def test_status_strings(lib):
    for s in range(8):
        assert moe.moe_status_string(s).startswith("MOE_")
    assert "UNKNOWN" in moe.moe_status_string(99)


def test_product_does_not_import_oracle():
    pkg = os.path.join(ROOT, "sparse_mixture_experts_rms_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+(oracle|moe_workloads)\b", src, re.M), f
                assert "moe_oracle" not in src and "moe_workloads" not in src, f


def test_noalloc_dispatch_rejects_oversize_before_device_work(lib):
    # T*k above the fixed scratch limit (2^20 assignments) is refused on the host
    c = moe.MoEConfig(T=(1 << 19) + 1, d_model=128, E=8, k=2, ffn_offsets=[128 * i for i in range(9)])
    P = ctypes.c_void_p
    st = lib.moe_dispatch_noalloc(ctypes.byref(c.c()), *[P(4096 * (i + 1)) for i in range(8)], P(0))
    assert st == moe.MOE_ERR_UNSUPPORTED


@pytest.mark.parametrize("name", mw.WORKLOAD_ORDER)
def test_training_sizes_and_saved_tensors(lib, name):
    """The training layout pads every expert segment to 64 rows and holds the
    saved tensors inside the workspace; both are host-side arithmetic."""
    w = mw.WORKLOADS[name]
    c = _cfg(w)
    rows = moe.moe_train_rows(c)
    assert rows == moe.moe_max_kept(c) + w.E * 63
    n = moe.moe_train_workspace_size(c)
    fmax = max(O.expert_widths(w.expert_sizes))
    # U, V, H, dS, dS3 (bf16) + y, dY (bf16) + dX (fp32) per padded row
    assert n >= rows * (5 * fmax * 2 + 2 * w.d_model * 2 + w.d_model * 4)
    base = 1 << 20
    seen = []
    for sid in range(14):
        out = ctypes.c_void_p(0)
        assert lib.moe_train_saved(ctypes.byref(c.c()), ctypes.c_void_p(base), n, sid, ctypes.byref(out)) == 0
        assert base <= out.value < base + n
        seen.append(out.value)
    assert len(set(seen)) == 14
    out = ctypes.c_void_p(0)
    assert lib.moe_train_saved(ctypes.byref(c.c()), ctypes.c_void_p(base), n, 99, ctypes.byref(out)) == \
        moe.MOE_ERR_INVALID_ARG
    assert lib.moe_train_saved(ctypes.byref(c.c()), ctypes.c_void_p(base), n - 1, 0, ctypes.byref(out)) == \
        moe.MOE_ERR_WORKSPACE


def test_backward_rejects_bad_arguments_before_device_work(lib):
    c = _cfg(mw.WORKLOADS["tiny"])
    P = ctypes.c_void_p
    ok = [P(1 << 20)] * 15   # x .. dW2
    n = moe.moe_train_workspace_size(c)
    # a missing weight-gradient output
    args = list(ok)
    args[12] = P(0)         # dW1
    assert lib.moe_layer_bwd(ctypes.byref(c.c()), *args, P(1 << 20), n, P(0)) == moe.MOE_ERR_INVALID_ARG
    # a misaligned dW2
    args = list(ok)
    args[14] = P((1 << 20) + 4)   # dW2
    assert lib.moe_layer_bwd(ctypes.byref(c.c()), *args, P(1 << 20), n, P(0)) == moe.MOE_ERR_ALIGNMENT
    # a workspace one byte short
    assert lib.moe_layer_bwd(ctypes.byref(c.c()), *ok, P(1 << 20), n - 1, P(0)) == moe.MOE_ERR_WORKSPACE


def test_host_pipeline_chunking(lib):
    """Dropless batches are cut into ceil(T/n)-token chunks with no empty
    chunk; a capacity limit keeps the batch whole."""
    mix = _cfg(mw.WORKLOADS["mixtral"])
    assert moe.moe_host_chunks(mix, 0) == 3
    assert moe.moe_host_chunks(mix, 3) == 3
    small = _cfg(mw.WORKLOADS["tiny"].with_tokens(5))
    assert moe.moe_host_chunks(small, 4) == 4          # 5 tokens, no chunk empty
    assert moe.moe_host_chunks(small, 99) == 5
    cap = _cfg(mw.WORKLOADS["switch_capacity"])
    assert moe.moe_host_chunks(cap, 4) == 1
    for c, n in ((mix, 4), (small, 4), (cap, 4)):
        m = moe.moe_host_chunks(c, n)
        w = [1] * m if m <= 2 else [1] + [4] * (m - 2) + [1]
        bounds = [c.T * sum(w[:i]) // sum(w) for i in range(m + 1)]
        for i in range(1, m):
            bounds[i] = min(max(bounds[i], bounds[i - 1] + 1), c.T - (m - i))
        assert all(b1 > b0 for b0, b1 in zip(bounds, bounds[1:])), bounds
        T_c = max(b1 - b0 for b0, b1 in zip(bounds, bounds[1:]))
        sub = _cfg(mw.WORKLOADS["tiny"])
        sub.__dict__.update(c.__dict__)
        sub.T = T_c
        staging = 4 * T_c * c.d_model * 2
        assert moe.moe_host_workspace_size(c, n) >= moe.moe_workspace_size(sub) + staging


@pytest.mark.parametrize("name", ["mixtral", "variable_size", "fine_grained"])
def test_mx_weights_layout(lib, name):
    """The MX weights buffer holds the K-major E4M3 copies, the standard scale
    blocks (the parts moe_mx_part names, in order, none overlapping) and one
    more copy of the scales, four times over, that the GEMM loads: at least
    4x the scale bytes of W1 + W3 + W2 beyond the parts.  Pure host
    arithmetic: the part pointers are offsets from a fake base."""
    import ctypes
    w = mw.WORKLOADS[name]
    cfg = moe.MoEConfig(T=w.T, d_model=w.d_model, E=w.E, k=w.k,
                        ffn_offsets=moe.ffn_offsets_from_sizes(w.expert_sizes))
    d, F = cfg.d_model, cfg.F
    total = moe.moe_mx_weights_size(cfg)
    base = 1 << 40
    out = ctypes.c_void_p()
    sizes = {"W1": d * F, "W3": d * F, "W2": d * F, "SF1": d * F // 32, "SF3": d * F // 32, "SF2": d * F // 32}
    end = 0
    for part in ("W1", "W3", "W2", "SF1", "SF3", "SF2"):
        st = lib.moe_mx_part(ctypes.byref(cfg.c()), ctypes.c_void_p(base), ctypes.c_void_p(0), ctypes.c_size_t(0),
                             moe.MOE_MX[part], ctypes.byref(out))
        assert st == 0
        off = out.value - base
        assert off >= end and off % 256 == 0, part
        end = off + sizes[part]
    assert total - end >= 4 * 3 * d * F // 32


def test_expert_offsets_printed_example(golden_dir):
    """moe_expert_offsets against the nanoMOE notes' printed widths and offsets."""
    import json
    import os
    with open(os.path.join(golden_dir, "nanomoe_variable_experts.json")) as f:
        g = json.load(f)
    assert moe.ffn_offsets_from_sizes([tuple(p) for p in g["expert_sizes"]]) == g["expert_offsets"]


@pytest.mark.parametrize("sizes", [((8, 14336),), ((16, 4096),), ((64, 512),), ((1, 1), (2, 127), (0, 9), (3, 129)),
                                   ((1, 2048), (7, 1024))])
def test_expert_offsets_follow_the_rounding_rule(sizes):
    widths = [-(-s // 128) * 128 for c, s in sizes for _ in range(c)]
    assert moe.ffn_offsets_from_sizes(sizes) == [0] + list(np.cumsum(widths).astype(int))


@pytest.mark.parametrize("bad", [((65, 128),), ((1, 0),), ((-1, 128),), ((2, 2 ** 30),)])
def test_expert_offsets_reject_bad_lists(lib, bad):
    n = len(bad)
    counts = (ctypes.c_int32 * n)(*[c for c, _ in bad])
    sizes = (ctypes.c_int32 * n)(*[s for _, s in bad])
    offs = (ctypes.c_int32 * 65)(*([-7] * 65))
    assert lib.moe_expert_offsets(counts, sizes, n, offs, 64) == -1
    assert offs[0] == -7  # nothing written
    assert lib.moe_expert_offsets(None, sizes, n, offs, 64) == -1
