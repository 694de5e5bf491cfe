"""The C-ABI library loads, exports every entry point that include/ress.h
declares, and rejects bad arguments on the host before any CUDA call (these
cases need no GPU)."""

import ctypes
import os
import re
import subprocess

import pytest
import torch

from block_sparse_global_mean_b200 import build as ress_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ress.h")


@pytest.fixture(scope="module")
def ress():
    ress_build.build()
    from block_sparse_global_mean_b200 import ress as mod
    return mod


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ress_[a-z_]+)\s*\(", text)))


def test_header_declares_the_three_stage_entry_points():
    names = _declared_functions()
    for n in ("ress_select_blocks", "ress_block_sparse_attn", "ress_block_drift"):
        assert n in names


def test_library_exports_every_declared_symbol(ress):
    names = _declared_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", ress.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(\w+)$", out, flags=re.M))
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(ress.lib, n)


def test_library_is_built_for_sm100a(ress):
    out = subprocess.run(["strings", ress.LIB_PATH], capture_output=True, text=True).stdout
    assert "sm_100a" in out


def test_status_strings(ress):
    assert ress.lib.ress_status_string(0) == b"ok"
    assert ress.lib.ress_status_string(3) == b"workspace too small"
    assert ress.lib.ress_status_string(99) == b"unknown status"
    assert ress.lib.ress_version() >> 16 == 1


def _shape(ress, n=512, heads=2, d=64, block=64, dtype=0):
    return ress.ress_shape(n, heads, d, block, dtype)


FAKE = 0x10000          # 16-byte aligned, never dereferenced: every case fails validation
FAKE_WS = 0x20000       # 256-byte aligned

# The cases below pass placeholder addresses that every host check must reject
# before a CUDA call.  They run where no GPU is visible, so that even a
# regressed check could only produce a CUDA error, never a launch on a bad
# address.
no_gpu_only = pytest.mark.skipif(torch.cuda.is_available(),
                                 reason="placeholder-pointer cases run only without a GPU")


def _select(ress, shape, q=FAKE, k=FAKE, v=None, budget=4, lam=0.0, idx=FAKE, ws=FAKE_WS,
            ws_bytes=1 << 30):
    return ress.lib.ress_select_blocks(ctypes.byref(shape) if shape is not None else None, q, k, v,
                                       budget, ctypes.c_float(lam), idx, ws, ws_bytes, None)


@no_gpu_only
def test_select_rejects_bad_arguments_on_the_host(ress):
    E = ress
    assert _select(ress, None) == E.RESS_ERR_INVALID_ARG
    assert _select(ress, _shape(ress, d=32)) == E.RESS_ERR_UNSUPPORTED
    assert _select(ress, _shape(ress, block=96)) == E.RESS_ERR_UNSUPPORTED
    assert _select(ress, _shape(ress, n=500)) == E.RESS_ERR_INVALID_ARG      # not a multiple of B
    assert _select(ress, _shape(ress, heads=0)) == E.RESS_ERR_INVALID_ARG
    assert _select(ress, _shape(ress, heads=65)) == E.RESS_ERR_UNSUPPORTED
    assert _select(ress, _shape(ress, dtype=7)) == E.RESS_ERR_INVALID_ARG
    assert _select(ress, _shape(ress), budget=0) == E.RESS_ERR_INVALID_ARG
    assert _select(ress, _shape(ress), budget=9) == E.RESS_ERR_INVALID_ARG   # nb = 8
    assert _select(ress, _shape(ress), lam=-1.0) == E.RESS_ERR_INVALID_ARG
    assert _select(ress, _shape(ress), lam=float("nan")) == E.RESS_ERR_INVALID_ARG
    assert _select(ress, _shape(ress), lam=0.5, v=None) == E.RESS_ERR_INVALID_ARG
    assert _select(ress, _shape(ress), q=None) == E.RESS_ERR_INVALID_ARG
    assert _select(ress, _shape(ress), q=FAKE + 8) == E.RESS_ERR_INVALID_ARG  # misaligned
    assert _select(ress, _shape(ress), ws=FAKE_WS + 16) == E.RESS_ERR_INVALID_ARG
    assert _select(ress, _shape(ress), ws_bytes=16) == E.RESS_ERR_WORKSPACE
    big = _shape(ress, n=64 * 4097)
    assert _select(ress, big, budget=1) == E.RESS_ERR_UNSUPPORTED               # nb > 4096


@no_gpu_only
def test_empty_input_is_a_no_op(ress):
    sh = _shape(ress, n=0)
    assert _select(ress, sh, budget=0) == ress.RESS_OK
    assert ress.lib.ress_block_sparse_attn(ctypes.byref(sh), FAKE, FAKE, FAKE, 0, FAKE, FAKE, 0,
                                           None, None, 0, None) == ress.RESS_OK
    assert ress.lib.ress_block_drift(ctypes.byref(sh), FAKE, FAKE, FAKE, 0, FAKE, FAKE, FAKE,
                                     None, None, 0, None) == ress.RESS_OK


@no_gpu_only
def test_attention_and_drift_reject_bad_arguments_on_the_host(ress):
    sh = _shape(ress)
    lib = ress.lib
    assert lib.ress_block_sparse_attn(ctypes.byref(sh), FAKE, FAKE, FAKE, 0, FAKE, FAKE, 0,
                                      None, None, 0, None) == ress.RESS_ERR_INVALID_ARG
    assert lib.ress_block_sparse_attn(ctypes.byref(sh), FAKE, FAKE, None, 4, FAKE, FAKE, 0,
                                      None, None, 0, None) == ress.RESS_ERR_INVALID_ARG
    assert lib.ress_block_sparse_attn(ctypes.byref(sh), FAKE, FAKE, FAKE, 4, FAKE + 2, FAKE, 0,
                                      None, None, 0, None) == ress.RESS_ERR_INVALID_ARG
    assert lib.ress_block_sparse_attn(ctypes.byref(sh), FAKE, FAKE, FAKE, 4, FAKE, FAKE, 5,
                                      None, None, 0, None) == ress.RESS_ERR_INVALID_ARG  # out dtype
    f32 = _shape(ress, dtype=1)
    assert lib.ress_block_sparse_attn(ctypes.byref(f32), FAKE, FAKE, FAKE, 4, FAKE, FAKE, 0,
                                      None, None, 0, None) == ress.RESS_ERR_WORKSPACE
    assert lib.ress_block_drift(ctypes.byref(sh), FAKE, FAKE, FAKE, 4, FAKE, None, FAKE, None,
                                None, 0, None) == ress.RESS_ERR_INVALID_ARG     # lse NULL
    assert lib.ress_block_drift(ctypes.byref(sh), FAKE, FAKE, FAKE, 4, FAKE, FAKE, None, None,
                                None, 0, None) == ress.RESS_ERR_INVALID_ARG     # drift NULL
    assert lib.ress_block_drift(ctypes.byref(sh), FAKE, FAKE, FAKE, 9, FAKE, FAKE, FAKE, None,
                                None, 0, None) == ress.RESS_ERR_INVALID_ARG     # budget > nb


def test_workspace_queries(ress):
    import torch
    # bf16, 100 views x 1,408 tokens, H=16, B=64 (nb_pad 2304).  lambda=0: Qbar,
    # then the larger of Kbar^T and the tensor-core arrays (Khi, Klo, 128
    # sample keys, key norms, a count slot, a row list).
    n, h, nb = 140800, 16, 2200
    got = ress.select_workspace_bytes(n, h, 64, torch.bfloat16, 0.0)
    qbar = 4 * h * nb * 64
    tc = 2 * 4 * h * 2304 * 64 + 4 * h * 128 * 64 + 4 * h * nb + 256 + 4 * h * nb
    assert got == qbar + max(4 * h * 64 * 2304, tc)
    # lambda > 0: Qbar + Kbar^T + Vbar + contrast
    with_v = ress.select_workspace_bytes(n, h, 64, torch.bfloat16, 0.5)
    assert with_v == qbar + 4 * h * 64 * 2304 + 4 * h * nb * 64 + 4 * h * nb
    assert ress.attn_workspace_bytes(n, h, 64, torch.bfloat16) == 0
    assert ress.attn_workspace_bytes(512, 2, 64, torch.float32) == 3 * 512 * 2 * 64 * 2
    assert ress.lib.ress_select_workspace_bytes(None, ctypes.c_float(0.0)) == 0


def _cdf(ress, shape, q=FAKE, k=FAKE, tau=0.9, cap=4, counts=FAKE, idx=FAKE, ws=FAKE_WS,
         ws_bytes=1 << 30):
    return ress.lib.ress_select_blocks_cdf(ctypes.byref(shape) if shape is not None else None, q,
                                           k, ctypes.c_float(tau), cap, counts, idx, ws, ws_bytes,
                                           None)


def test_cdf_select_rejects_bad_arguments_on_the_host(ress):
    E = ress
    assert _cdf(ress, None) == E.RESS_ERR_INVALID_ARG
    assert _cdf(ress, _shape(ress, d=32)) == E.RESS_ERR_UNSUPPORTED
    for tau in (0.0, -0.5, 1.5, float("nan"), float("inf")):
        assert _cdf(ress, _shape(ress), tau=tau) == E.RESS_ERR_INVALID_ARG, tau
    assert _cdf(ress, _shape(ress), cap=0) == E.RESS_ERR_INVALID_ARG
    assert _cdf(ress, _shape(ress), cap=9) == E.RESS_ERR_INVALID_ARG      # nb = 8
    assert _cdf(ress, _shape(ress), counts=None) == E.RESS_ERR_INVALID_ARG
    assert _cdf(ress, _shape(ress), counts=FAKE + 2) == E.RESS_ERR_INVALID_ARG
    assert _cdf(ress, _shape(ress), idx=None) == E.RESS_ERR_INVALID_ARG
    assert _cdf(ress, _shape(ress), q=FAKE + 8) == E.RESS_ERR_INVALID_ARG
    assert _cdf(ress, _shape(ress), ws_bytes=16) == E.RESS_ERR_WORKSPACE
    assert _cdf(ress, _shape(ress, n=64 * 4097), cap=1) == E.RESS_ERR_UNSUPPORTED
    assert _cdf(ress, _shape(ress, n=0), cap=0) == E.RESS_OK               # empty: no launch


def test_binding_rejects_mismatched_tensors_before_any_library_call(ress):
    """Shapes, dtypes and devices that the kernels would read or write out of
    bounds are refused by the binding (these checks need no GPU)."""
    import torch
    bf = torch.bfloat16
    H, B, nb = 2, 64, 4
    q = torch.zeros(nb * B, H, 64, dtype=bf)
    k_short = torch.zeros((nb - 1) * B, H, 64, dtype=bf)
    with pytest.raises(ValueError, match="k has shape"):
        ress.ress_select_blocks(q, k_short, None, 2, 0.0, B)
    with pytest.raises(TypeError, match="v is"):
        ress.ress_block_sparse_attn(q, q, q.float(), torch.zeros(H, nb, 2, dtype=torch.int32), B)
    with pytest.raises(TypeError, match="idx must be"):
        ress.ress_block_sparse_attn(q, q, q, torch.zeros(H, nb, 2, dtype=torch.int64), B)
    with pytest.raises(ValueError, match="idx must have shape"):
        ress.ress_block_sparse_attn(q, q, q, torch.zeros(H + 1, nb, 2, dtype=torch.int32), B)
    with pytest.raises(ValueError, match="out must have shape"):
        ress.ress_block_sparse_attn(q, q, q, torch.zeros(H, nb, 2, dtype=torch.int32), B,
                                    out=torch.zeros(nb * B, H, 32, dtype=bf))
    with pytest.raises(TypeError, match="lse must be"):
        ress.ress_block_sparse_attn(q, q, q, torch.zeros(H, nb, 2, dtype=torch.int32), B,
                                    lse=torch.zeros(H, nb * B, dtype=torch.float64))
    idx = torch.zeros(H, nb, 2, dtype=torch.int32)
    lse = torch.zeros(H, nb * B)
    with pytest.raises(ValueError, match="drift must have shape"):
        ress.ress_block_drift(q, q, q, idx, lse, B, drift=torch.zeros(H, nb, nb))
    with pytest.raises(ValueError, match="lse must have shape"):
        ress.ress_block_drift(q, q, q, idx, torch.zeros(H, nb), B)
    with pytest.raises(TypeError, match="counts must be"):
        ress.ress_select_blocks_cdf(q, q, 0.9, B, counts=torch.zeros(H, nb, dtype=torch.int64))
    with pytest.raises(TypeError, match="workspace must be"):
        ress.ress_select_blocks(q, q, None, 2, 0.0, B, workspace=torch.zeros(64))
    with pytest.raises(ValueError, match="idx must have shape"):
        ress.ress_select_blocks(q, q, None, 2, 0.0, B, idx=torch.zeros(H, nb, 3, dtype=torch.int32))
    # Consistent host tensors pass every check and stop at the device check.
    with pytest.raises(ValueError, match="CUDA device"):
        ress.ress_select_blocks(q, q, None, 2, 0.0, B)


@no_gpu_only
def test_validate_idx_rejects_bad_arguments_on_the_host(ress):
    sh = _shape(ress)
    lib = ress.lib
    assert lib.ress_validate_idx(None, 4, FAKE, None) == ress.RESS_ERR_INVALID_ARG
    assert lib.ress_validate_idx(ctypes.byref(sh), 0, FAKE, None) == ress.RESS_ERR_INVALID_ARG
    assert lib.ress_validate_idx(ctypes.byref(sh), 9, FAKE, None) == ress.RESS_ERR_INVALID_ARG
    assert lib.ress_validate_idx(ctypes.byref(sh), 4, None, None) == ress.RESS_ERR_INVALID_ARG
    assert lib.ress_validate_idx(ctypes.byref(sh), 4, FAKE + 2, None) == ress.RESS_ERR_INVALID_ARG
    empty = _shape(ress, n=0)
    assert lib.ress_validate_idx(ctypes.byref(empty), 0, FAKE, None) == ress.RESS_OK


@no_gpu_only
def test_noalloc_rejects_problems_beyond_its_fixed_scratch(ress):
    # H = 64, nb = 4,096: about 134 MB of scratch, more than the fixed 32 MiB.
    big = _shape(ress, n=64 * 4096, heads=64)
    assert ress.lib.ress_select_blocks_noalloc(ctypes.byref(big), FAKE, FAKE, None, 8,
                                               ctypes.c_float(0.0), FAKE, None) \
        == ress.RESS_ERR_WORKSPACE
    # and argument errors come first, as for the workspace entry point
    assert ress.lib.ress_select_blocks_noalloc(ctypes.byref(big), FAKE, FAKE, None, 0,
                                               ctypes.c_float(0.0), FAKE, None) \
        == ress.RESS_ERR_INVALID_ARG


@no_gpu_only
def test_layout_entry_points_reject_bad_layouts_on_the_host(ress):
    lib = ress.lib
    sh = _shape(ress, n=1024, heads=2, block=64)                  # 1,024 tokens
    bad = [ress.ress_layout(0, 1, 0), ress.ress_layout(96, 90, 5),  # not a multiple of the block
           ress.ress_layout(384, 300, 5),                          # does not divide N
           ress.ress_layout(256, 0, 0), ress.ress_layout(256, 257, 0),
           ress.ress_layout(256, 200, 201), ress.ress_layout(256, 200, -1)]
    for lay in bad:
        assert lib.ress_select_blocks_layout(ctypes.byref(sh), ctypes.byref(lay), FAKE, FAKE, 4,
                                             FAKE, FAKE_WS, 1 << 30, None) == ress.RESS_ERR_INVALID_ARG
        assert lib.ress_block_sparse_attn_layout(ctypes.byref(sh), ctypes.byref(lay), FAKE, FAKE,
                                                 FAKE, 4, FAKE, FAKE, 0, None, FAKE_WS, 1 << 30,
                                                 None) == ress.RESS_ERR_INVALID_ARG
        assert lib.ress_block_drift_layout(ctypes.byref(sh), ctypes.byref(lay), FAKE, FAKE, FAKE,
                                           4, FAKE, FAKE, FAKE, None, None, 0,
                                           None) == ress.RESS_ERR_INVALID_ARG
        assert lib.ress_attn_layout_workspace_bytes(ctypes.byref(sh), ctypes.byref(lay), 0) == 0
    assert lib.ress_select_blocks_layout(ctypes.byref(sh), None, FAKE, FAKE, 4, FAKE, FAKE_WS,
                                         1 << 30, None) == ress.RESS_ERR_INVALID_ARG
    good = ress.ress_layout(256, 200, 5)
    # 4 views x 5 special rows -> 128 gathered rows: bf16 queries and output, float32 lse
    assert lib.ress_attn_layout_workspace_bytes(ctypes.byref(sh), ctypes.byref(good), 0) == \
        128 * 2 * 64 * 2 * 2 + 128 * 2 * 4
    none = ress.ress_layout(256, 200, 0)
    assert lib.ress_attn_layout_workspace_bytes(ctypes.byref(sh), ctypes.byref(none), 0) == 0
    assert lib.ress_select_blocks_layout(ctypes.byref(sh), ctypes.byref(good), FAKE, FAKE, 4,
                                         FAKE, FAKE_WS, 16, None) == ress.RESS_ERR_WORKSPACE


@no_gpu_only
def test_restore_rejects_bad_arguments_on_the_host(ress):
    lib = ress.lib
    sh = _shape(ress)                                              # nb = 8

    def call(budget=4, rounds=4, cand=8, q=FAKE, v=FAKE, ws_bytes=1 << 30):
        return lib.ress_select_blocks_restore(ctypes.byref(sh), q, FAKE, v, budget, rounds, cand,
                                              FAKE, None, None, FAKE_WS, ws_bytes, None)
    assert call(budget=0) == ress.RESS_ERR_INVALID_ARG
    assert call(budget=9) == ress.RESS_ERR_INVALID_ARG
    assert call(rounds=-1) == ress.RESS_ERR_INVALID_ARG
    assert call(rounds=65) == ress.RESS_ERR_INVALID_ARG
    assert call(cand=0) == ress.RESS_ERR_INVALID_ARG
    assert call(cand=17) == ress.RESS_ERR_INVALID_ARG
    assert call(v=None) == ress.RESS_ERR_INVALID_ARG
    assert call(q=FAKE + 4) == ress.RESS_ERR_INVALID_ARG
    assert call(ws_bytes=16) == ress.RESS_ERR_WORKSPACE
    # Qbar, Kbar^T and Vbar^T (nb_pad = 256)
    assert lib.ress_restore_workspace_bytes(ctypes.byref(sh)) == 4 * 2 * 8 * 64 + 2 * 4 * 2 * 64 * 256


@no_gpu_only
def test_vasc_rejects_bad_arguments_on_the_host(ress):
    lib = ress.lib
    sh = _shape(ress)                                              # H = 2, nb = 8

    def call(budgets=(2, 3), cap=4, va=1, reset=0, q=FAKE, v=FAKE, mem=FAKE, dem=None,
             ws_bytes=1 << 30):
        arr = None if budgets is None else (ctypes.c_int32 * len(budgets))(*budgets)
        return lib.ress_select_blocks_vasc(ctypes.byref(sh), q, FAKE, v,
                                           None if arr is None else ctypes.cast(arr, ctypes.c_void_p),
                                           cap, va, reset, mem, FAKE, dem, None, FAKE_WS, ws_bytes,
                                           None)
    assert call(budgets=None) == ress.RESS_ERR_INVALID_ARG
    assert call(budgets=(0, 3)) == ress.RESS_ERR_INVALID_ARG
    assert call(budgets=(2, 5)) == ress.RESS_ERR_INVALID_ARG      # above the capacity
    assert call(cap=0) == ress.RESS_ERR_INVALID_ARG
    assert call(cap=9) == ress.RESS_ERR_INVALID_ARG               # above nb
    assert call(va=2) == ress.RESS_ERR_INVALID_ARG
    assert call(reset=-1) == ress.RESS_ERR_INVALID_ARG
    assert call(v=None) == ress.RESS_ERR_INVALID_ARG              # the contrast needs V
    assert call(mem=None) == ress.RESS_ERR_INVALID_ARG
    assert call(q=FAKE + 4) == ress.RESS_ERR_INVALID_ARG
    assert call(mem=FAKE + 2) == ress.RESS_ERR_INVALID_ARG
    assert call(dem=FAKE + 2) == ress.RESS_ERR_INVALID_ARG
    assert call(ws_bytes=16) == ress.RESS_ERR_WORKSPACE
    assert lib.ress_select_blocks_vasc(None, FAKE, FAKE, FAKE, None, 4, 1, 0, FAKE, FAKE, None,
                                       None, FAKE_WS, 1 << 30, None) == ress.RESS_ERR_INVALID_ARG
    # Qbar; Kbar^T and Vbar^T (nb_pad = 256); rho, mhat, demand sums and
    # service counts for 2 x 4 pairs, each padded to 256 bytes.
    assert lib.ress_vasc_workspace_bytes(ctypes.byref(sh)) == \
        4 * 2 * 8 * 64 + 2 * 4 * 2 * 64 * 256 + 4 * 256


def test_vasc_binding_checks_its_buffers_before_the_library(ress):
    q = torch.zeros(512, 2, 64)
    with pytest.raises(ValueError):
        ress.ress_select_blocks_vasc(q, q, None, [2, 3], 64)      # contrast without V
    with pytest.raises(ValueError):
        ress.ress_select_blocks_vasc(q, q, q, [2, 3, 4], 64)      # one budget per head
    assert ress.vasc_pairs(8) == 4 and ress.vasc_pairs(9) == 5
