"""Python binding of the C ABI in ``include/ress.h`` (ctypes).

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libress.so``.  PyTorch supplies device memory and the current stream.  If
the library is missing, importing this module raises ImportError; there is no
fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG_DIR, "libress.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m block_sparse_global_mean_b200.build` "
        "(this package has no CPU fallback)")

lib = ctypes.CDLL(LIB_PATH)

RESS_OK = 0
RESS_ERR_INVALID_ARG = 1
RESS_ERR_UNSUPPORTED = 2
RESS_ERR_WORKSPACE = 3
RESS_ERR_CUDA = 4
RESS_ERR_TIMEOUT = 5
RESS_ERR_BAD_INDEX = 6

RESS_BF16 = 0
RESS_F32 = 1


class ress_shape(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int64), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block", ctypes.c_int32), ("dtype", ctypes.c_int32)]


class ress_layout(ctypes.Structure):
    _fields_ = [("tokens_per_view", ctypes.c_int32), ("real_tokens", ctypes.c_int32),
                ("special_tokens", ctypes.c_int32)]


_P = ctypes.c_void_p
_SHAPE = ctypes.POINTER(ress_shape)

lib.ress_version.restype = ctypes.c_int
lib.ress_version.argtypes = []
lib.ress_status_string.restype = ctypes.c_char_p
lib.ress_status_string.argtypes = [ctypes.c_int]
lib.ress_select_workspace_bytes.restype = ctypes.c_size_t
lib.ress_select_workspace_bytes.argtypes = [_SHAPE, ctypes.c_float]
lib.ress_select_blocks.restype = ctypes.c_int
lib.ress_select_blocks.argtypes = [_SHAPE, _P, _P, _P, ctypes.c_int32, ctypes.c_float, _P, _P,
                                   ctypes.c_size_t, _P]
lib.ress_attn_workspace_bytes.restype = ctypes.c_size_t
lib.ress_attn_workspace_bytes.argtypes = [_SHAPE]
lib.ress_block_sparse_attn.restype = ctypes.c_int
lib.ress_block_sparse_attn.argtypes = [_SHAPE, _P, _P, _P, ctypes.c_int32, _P, _P, ctypes.c_int32,
                                       _P, _P, ctypes.c_size_t, _P]
lib.ress_block_drift.restype = ctypes.c_int
lib.ress_block_drift.argtypes = [_SHAPE, _P, _P, _P, ctypes.c_int32, _P, _P, _P, _P, _P,
                                 ctypes.c_size_t, _P]
lib.ress_select_blocks_noalloc.restype = ctypes.c_int
lib.ress_select_blocks_noalloc.argtypes = [_SHAPE, _P, _P, _P, ctypes.c_int32, ctypes.c_float, _P, _P]
lib.ress_select_blocks_cdf.restype = ctypes.c_int
lib.ress_select_blocks_cdf.argtypes = [_SHAPE, _P, _P, ctypes.c_float, ctypes.c_int32, _P, _P, _P,
                                         ctypes.c_size_t, _P]
lib.ress_last_cuda_error.restype = ctypes.c_char_p
lib.ress_last_cuda_error.argtypes = []
lib.ress_test_exp2.restype = ctypes.c_int
lib.ress_test_exp2.argtypes = [_P, _P, ctypes.c_int32, _P]
_LAYOUT = ctypes.POINTER(ress_layout)
lib.ress_select_blocks_layout.restype = ctypes.c_int
lib.ress_select_blocks_layout.argtypes = [_SHAPE, _LAYOUT, _P, _P, ctypes.c_int32, _P, _P,
                                          ctypes.c_size_t, _P]
lib.ress_attn_layout_workspace_bytes.restype = ctypes.c_size_t
lib.ress_attn_layout_workspace_bytes.argtypes = [_SHAPE, _LAYOUT, ctypes.c_int32]
lib.ress_block_sparse_attn_layout.restype = ctypes.c_int
lib.ress_block_sparse_attn_layout.argtypes = [_SHAPE, _LAYOUT, _P, _P, _P, ctypes.c_int32, _P, _P,
                                              ctypes.c_int32, _P, _P, ctypes.c_size_t, _P]
lib.ress_block_drift_layout.restype = ctypes.c_int
lib.ress_block_drift_layout.argtypes = [_SHAPE, _LAYOUT, _P, _P, _P, ctypes.c_int32, _P, _P, _P,
                                        _P, _P, ctypes.c_size_t, _P]
lib.ress_restore_workspace_bytes.restype = ctypes.c_size_t
lib.ress_restore_workspace_bytes.argtypes = [_SHAPE]
lib.ress_select_blocks_restore.restype = ctypes.c_int
lib.ress_select_blocks_restore.argtypes = [_SHAPE, _P, _P, _P, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_int32, _P, _P, _P, _P, ctypes.c_size_t, _P]
lib.ress_vasc_workspace_bytes.restype = ctypes.c_size_t
lib.ress_vasc_workspace_bytes.argtypes = [_SHAPE]
lib.ress_select_blocks_vasc.restype = ctypes.c_int
lib.ress_select_blocks_vasc.argtypes = [_SHAPE, _P, _P, _P, _P, ctypes.c_int32, ctypes.c_int32,
                                        ctypes.c_int32, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]
lib.ress_validate_idx.restype = ctypes.c_int
lib.ress_validate_idx.argtypes = [_SHAPE, ctypes.c_int32, _P, _P]
lib.ress_check_device_errors.restype = ctypes.c_int
lib.ress_check_device_errors.argtypes = [_P, ctypes.POINTER(ctypes.c_int32)]


class RessError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.ress_status_string(status).decode()
        if status == RESS_ERR_CUDA:
            msg += f" [{lib.ress_last_cuda_error().decode()}]"
        super().__init__(f"{where}: {msg} (status {status})")


def _check(status: int, where: str) -> None:
    if status != RESS_OK:
        raise RessError(status, where)


def _on(device: torch.device, fn, *args) -> int:
    """Calls ``fn(*args)`` with ``device`` current: the library looks up its
    per-device state (error flag, fixed scratch) on the current device."""
    with torch.cuda.device(device):
        return fn(*args)


def make_shape(n: int, heads: int, block: int, dtype: torch.dtype, head_dim: int = 64) -> ress_shape:
    if dtype == torch.bfloat16:
        code = RESS_BF16
    elif dtype == torch.float32:
        code = RESS_F32
    else:
        raise TypeError(f"unsupported dtype {dtype}")
    return ress_shape(n, heads, head_dim, block, code)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream_ptr(stream: Optional[torch.cuda.Stream], device: torch.device) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _shape_of(q: torch.Tensor, block: int) -> ress_shape:
    if q.dim() != 3:
        raise ValueError("q, k, v must be [N, H, d]")
    n, h, d = q.shape
    return make_shape(n, h, block, q.dtype, d)


def _check_inputs(q: torch.Tensor, k: torch.Tensor, v: Optional[torch.Tensor] = None) -> None:
    """k and v must match q in shape, dtype and device (the library reads all
    three with q's shape)."""
    if q.dim() != 3:
        raise ValueError("q, k, v must be [N, H, d]")
    for name, t in (("k", k), ("v", v)):
        if t is None:
            continue
        if tuple(t.shape) != tuple(q.shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, q has {tuple(q.shape)}")
        if t.dtype != q.dtype:
            raise TypeError(f"{name} is {t.dtype}, q is {q.dtype}")
        if t.device != q.device:
            raise ValueError(f"{name} is on {t.device}, q on {q.device}")


def _check_buffer(t: torch.Tensor, shape, dtype: torch.dtype, device: torch.device,
                  name: str) -> None:
    """A caller-provided buffer must have exactly the shape, dtype and device
    the library writes or reads."""
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def _check_workspace(ws: Optional[torch.Tensor], device: torch.device) -> None:
    if ws is not None:
        _check_buffer(ws, (ws.numel(),), torch.uint8, device, "workspace")


def _check_idx(idx: torch.Tensor, h: int, nb: int, device: torch.device) -> int:
    """idx must be int32 [H, nb, budget]; returns budget."""
    if idx.dim() != 3:
        raise ValueError(f"idx must be [H, nb, budget], got {tuple(idx.shape)}")
    _check_buffer(idx, (h, nb, idx.shape[2]), torch.int32, device, "idx")
    return int(idx.shape[2])


def select_workspace_bytes(n: int, heads: int, block: int, dtype: torch.dtype, lam: float) -> int:
    sh = make_shape(n, heads, block, dtype)
    return int(lib.ress_select_workspace_bytes(ctypes.byref(sh), ctypes.c_float(lam)))


def vasc_workspace_bytes(n: int, heads: int, block: int, dtype: torch.dtype) -> int:
    sh = make_shape(n, heads, block, dtype)
    return int(lib.ress_vasc_workspace_bytes(ctypes.byref(sh)))


def attn_workspace_bytes(n: int, heads: int, block: int, dtype: torch.dtype) -> int:
    sh = make_shape(n, heads, block, dtype)
    return int(lib.ress_attn_workspace_bytes(ctypes.byref(sh)))


def ress_select_blocks(q: torch.Tensor, k: torch.Tensor, v: Optional[torch.Tensor], budget: int,
                       lam: float, block: int, idx: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None,
                       stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Stage 1: returns idx [H, nb, budget] int32 (ascending kept blocks per row)."""
    _check_inputs(q, k, v if lam else None)
    sh = _shape_of(q, block)
    n, h = q.shape[0], q.shape[1]
    nb = n // block
    if idx is None:
        idx = torch.empty((h, nb, budget), dtype=torch.int32, device=q.device)
    _check_buffer(idx, (h, nb, budget), torch.int32, q.device, "idx")
    _check_workspace(workspace, q.device)
    need = int(lib.ress_select_workspace_bytes(ctypes.byref(sh), ctypes.c_float(lam)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    status = _on(q.device, lib.ress_select_blocks, ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), int(budget),
                                    ctypes.c_float(lam), _ptr(idx), _ptr(workspace),
                                    workspace.numel(), _stream_ptr(stream, q.device))
    _check(status, "ress_select_blocks")
    return idx


def ress_select_blocks_cdf(q: torch.Tensor, k: torch.Tensor, tau: float, block: int,
                           capacity: Optional[int] = None, counts: Optional[torch.Tensor] = None,
                           idx: Optional[torch.Tensor] = None,
                           workspace: Optional[torch.Tensor] = None,
                           stream: Optional[torch.cuda.Stream] = None
                           ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Stage 1 with the cumulative (CDF) threshold: returns (counts [H, nb]
    int32, idx [H, nb, capacity] int32); capacity defaults to nb."""
    _check_inputs(q, k)
    sh = _shape_of(q, block)
    n, h = q.shape[0], q.shape[1]
    nb = n // block
    cap = nb if capacity is None else int(capacity)
    if counts is None:
        counts = torch.empty((h, nb), dtype=torch.int32, device=q.device)
    if idx is None:
        idx = torch.empty((h, nb, max(cap, 1)), dtype=torch.int32, device=q.device)
    _check_buffer(counts, (h, nb), torch.int32, q.device, "counts")
    _check_buffer(idx, (h, nb, max(cap, 1)), torch.int32, q.device, "idx")
    _check_workspace(workspace, q.device)
    need = int(lib.ress_select_workspace_bytes(ctypes.byref(sh), ctypes.c_float(0.0)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    status = _on(q.device, lib.ress_select_blocks_cdf, ctypes.byref(sh), _ptr(q), _ptr(k), ctypes.c_float(tau),
                                        cap, _ptr(counts), _ptr(idx), _ptr(workspace),
                                        workspace.numel(), _stream_ptr(stream, q.device))
    _check(status, "ress_select_blocks_cdf")
    return counts, idx


def ress_select_blocks_noalloc(q: torch.Tensor, k: torch.Tensor, v: Optional[torch.Tensor],
                               budget: int, lam: float, block: int,
                               idx: Optional[torch.Tensor] = None,
                               stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Stage 1 with the library's fixed scratch array instead of a workspace
    (for callers that cannot allocate device memory); see include/ress.h."""
    _check_inputs(q, k, v if lam else None)
    sh = _shape_of(q, block)
    n, h = q.shape[0], q.shape[1]
    if idx is None:
        idx = torch.empty((h, n // block, budget), dtype=torch.int32, device=q.device)
    _check_buffer(idx, (h, n // block, budget), torch.int32, q.device, "idx")
    status = _on(q.device, lib.ress_select_blocks_noalloc, ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), int(budget),
                                            ctypes.c_float(lam), _ptr(idx),
                                            _stream_ptr(stream, q.device))
    _check(status, "ress_select_blocks_noalloc")
    return idx


def ress_block_sparse_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor,
                           block: int, out: Optional[torch.Tensor] = None,
                           lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                           workspace: Optional[torch.Tensor] = None,
                           stream: Optional[torch.cuda.Stream] = None,
                           out_dtype: Optional[torch.dtype] = None
                           ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Stage 2: returns (out [N, H, 64], lse [H, N] float32 or None).

    The output dtype is ``out.dtype`` if ``out`` is given, else ``out_dtype``,
    else the input dtype."""
    _check_inputs(q, k, v)
    sh = _shape_of(q, block)
    n, h = q.shape[0], q.shape[1]
    budget = _check_idx(idx, h, n // block, q.device)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    out_code = RESS_F32 if out.dtype == torch.float32 else (
        RESS_BF16 if out.dtype == torch.bfloat16 else None)
    if out_code is None:
        raise TypeError(f"unsupported output dtype {out.dtype}")
    _check_buffer(out, q.shape, out.dtype, q.device, "out")
    if lse is None and want_lse:
        lse = torch.empty((h, n), dtype=torch.float32, device=q.device)
    if lse is not None:
        _check_buffer(lse, (h, n), torch.float32, q.device, "lse")
    _check_workspace(workspace, q.device)
    need = int(lib.ress_attn_workspace_bytes(ctypes.byref(sh)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    status = _on(q.device, lib.ress_block_sparse_attn, ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), int(budget),
                                        _ptr(idx), _ptr(out), out_code, _ptr(lse), _ptr(workspace),
                                        0 if workspace is None else workspace.numel(),
                                        _stream_ptr(stream, q.device))
    _check(status, "ress_block_sparse_attn")
    return out, lse


def ress_block_drift(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor,
                     lse: torch.Tensor, block: int, drift: Optional[torch.Tensor] = None,
                     set_drift: Optional[torch.Tensor] = None,
                     workspace: Optional[torch.Tensor] = None,
                     stream: Optional[torch.cuda.Stream] = None
                     ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Stage 3: returns (drift [H, nb, nb - budget], set_drift [H, nb]) float32."""
    _check_inputs(q, k, v)
    sh = _shape_of(q, block)
    n, h = q.shape[0], q.shape[1]
    nb = n // block
    budget = _check_idx(idx, h, nb, q.device)
    _check_buffer(lse, (h, n), torch.float32, q.device, "lse")
    if drift is None:
        drift = torch.empty((h, nb, max(nb - budget, 0)), dtype=torch.float32, device=q.device)
    if set_drift is None:
        set_drift = torch.empty((h, nb), dtype=torch.float32, device=q.device)
    _check_buffer(drift, (h, nb, max(nb - budget, 0)), torch.float32, q.device, "drift")
    _check_buffer(set_drift, (h, nb), torch.float32, q.device, "set_drift")
    _check_workspace(workspace, q.device)
    need = int(lib.ress_attn_workspace_bytes(ctypes.byref(sh)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    status = _on(q.device, lib.ress_block_drift, ctypes.byref(sh), _ptr(q), _ptr(k), _ptr(v), int(budget),
                                  _ptr(idx), _ptr(lse), _ptr(drift) if drift.numel() else None,
                                  _ptr(set_drift), _ptr(workspace),
                                  0 if workspace is None else workspace.numel(),
                                  _stream_ptr(stream, q.device))
    _check(status, "ress_block_drift")
    return drift, set_drift


def _layout(layout) -> ress_layout:
    """(tokens_per_view, real_tokens, special_tokens) -> ress_layout."""
    t, r, sp = (int(x) for x in layout)
    return ress_layout(t, r, sp)


def ress_select_blocks_layout(q: torch.Tensor, k: torch.Tensor, budget: int, block: int, layout,
                              idx: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None,
                              stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """Stage 1 with a per-view layout (tokens_per_view, real_tokens,
    special_tokens): returns idx [H, nb, budget] int32."""
    _check_inputs(q, k)
    sh = _shape_of(q, block)
    lay = _layout(layout)
    n, h = q.shape[0], q.shape[1]
    nb = n // block
    if idx is None:
        idx = torch.empty((h, nb, budget), dtype=torch.int32, device=q.device)
    _check_buffer(idx, (h, nb, budget), torch.int32, q.device, "idx")
    _check_workspace(workspace, q.device)
    need = int(lib.ress_select_workspace_bytes(ctypes.byref(sh), ctypes.c_float(0.0)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    status = _on(q.device, lib.ress_select_blocks_layout, ctypes.byref(sh), ctypes.byref(lay),
                 _ptr(q), _ptr(k), int(budget), _ptr(idx), _ptr(workspace), workspace.numel(),
                 _stream_ptr(stream, q.device))
    _check(status, "ress_select_blocks_layout")
    return idx


def ress_block_sparse_attn_layout(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                  idx: torch.Tensor, block: int, layout,
                                  out: Optional[torch.Tensor] = None,
                                  lse: Optional[torch.Tensor] = None, want_lse: bool = True,
                                  workspace: Optional[torch.Tensor] = None,
                                  stream: Optional[torch.cuda.Stream] = None,
                                  out_dtype: Optional[torch.dtype] = None
                                  ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Stage 2 with a per-view layout: returns (out [N, H, 64], lse [H, N])."""
    _check_inputs(q, k, v)
    sh = _shape_of(q, block)
    lay = _layout(layout)
    n, h = q.shape[0], q.shape[1]
    budget = _check_idx(idx, h, n // block, q.device)
    if out is None:
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    out_code = RESS_F32 if out.dtype == torch.float32 else (
        RESS_BF16 if out.dtype == torch.bfloat16 else None)
    if out_code is None:
        raise TypeError(f"unsupported output dtype {out.dtype}")
    _check_buffer(out, q.shape, out.dtype, q.device, "out")
    if lse is None and want_lse:
        lse = torch.empty((h, n), dtype=torch.float32, device=q.device)
    if lse is not None:
        _check_buffer(lse, (h, n), torch.float32, q.device, "lse")
    _check_workspace(workspace, q.device)
    need = int(lib.ress_attn_layout_workspace_bytes(ctypes.byref(sh), ctypes.byref(lay), out_code))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    status = _on(q.device, lib.ress_block_sparse_attn_layout, ctypes.byref(sh), ctypes.byref(lay),
                 _ptr(q), _ptr(k), _ptr(v), int(budget), _ptr(idx), _ptr(out), out_code,
                 _ptr(lse), _ptr(workspace), 0 if workspace is None else workspace.numel(),
                 _stream_ptr(stream, q.device))
    _check(status, "ress_block_sparse_attn_layout")
    return out, lse


def ress_block_drift_layout(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, idx: torch.Tensor,
                            lse: torch.Tensor, block: int, layout,
                            drift: Optional[torch.Tensor] = None,
                            set_drift: Optional[torch.Tensor] = None,
                            workspace: Optional[torch.Tensor] = None,
                            stream: Optional[torch.cuda.Stream] = None
                            ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Stage 3 with a per-view layout: returns (drift [H, nb, nb - budget], set_drift [H, nb])."""
    _check_inputs(q, k, v)
    sh = _shape_of(q, block)
    lay = _layout(layout)
    n, h = q.shape[0], q.shape[1]
    nb = n // block
    budget = _check_idx(idx, h, nb, q.device)
    _check_buffer(lse, (h, n), torch.float32, q.device, "lse")
    if drift is None:
        drift = torch.empty((h, nb, max(nb - budget, 0)), dtype=torch.float32, device=q.device)
    if set_drift is None:
        set_drift = torch.empty((h, nb), dtype=torch.float32, device=q.device)
    _check_buffer(drift, (h, nb, max(nb - budget, 0)), torch.float32, q.device, "drift")
    _check_buffer(set_drift, (h, nb), torch.float32, q.device, "set_drift")
    _check_workspace(workspace, q.device)
    need = int(lib.ress_attn_workspace_bytes(ctypes.byref(sh)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    status = _on(q.device, lib.ress_block_drift_layout, ctypes.byref(sh), ctypes.byref(lay),
                 _ptr(q), _ptr(k), _ptr(v), int(budget), _ptr(idx), _ptr(lse),
                 _ptr(drift) if drift.numel() else None, _ptr(set_drift), _ptr(workspace),
                 0 if workspace is None else workspace.numel(), _stream_ptr(stream, q.device))
    _check(status, "ress_block_drift_layout")
    return drift, set_drift


def ress_select_blocks_restore(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, budget: int,
                               block: int, rounds: int = 4, candidates: int = 8,
                               idx: Optional[torch.Tensor] = None,
                               drift_init: Optional[torch.Tensor] = None,
                               drift_final: Optional[torch.Tensor] = None,
                               workspace: Optional[torch.Tensor] = None,
                               stream: Optional[torch.cuda.Stream] = None
                               ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Stage 1 by drift with restoration: returns (idx [H, nb, budget] int32,
    drift of the initial drop set [H, nb], drift of the result [H, nb])."""
    _check_inputs(q, k, v)
    sh = _shape_of(q, block)
    n, h = q.shape[0], q.shape[1]
    nb = n // block
    if idx is None:
        idx = torch.empty((h, nb, budget), dtype=torch.int32, device=q.device)
    if drift_init is None:
        drift_init = torch.empty((h, nb), dtype=torch.float32, device=q.device)
    if drift_final is None:
        drift_final = torch.empty((h, nb), dtype=torch.float32, device=q.device)
    _check_buffer(idx, (h, nb, budget), torch.int32, q.device, "idx")
    _check_buffer(drift_init, (h, nb), torch.float32, q.device, "drift_init")
    _check_buffer(drift_final, (h, nb), torch.float32, q.device, "drift_final")
    _check_workspace(workspace, q.device)
    need = int(lib.ress_restore_workspace_bytes(ctypes.byref(sh)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    status = _on(q.device, lib.ress_select_blocks_restore, ctypes.byref(sh), _ptr(q), _ptr(k),
                 _ptr(v), int(budget), int(rounds), int(candidates), _ptr(idx), _ptr(drift_init),
                 _ptr(drift_final), _ptr(workspace), workspace.numel(),
                 _stream_ptr(stream, q.device))
    _check(status, "ress_select_blocks_restore")
    return idx, drift_init, drift_final


def vasc_pairs(nb: int) -> int:
    """Memory entries per head of the VASC selection: one per fixed pair of
    neighbouring key blocks, the last a singleton when nb is odd."""
    return (nb + 1) // 2


def ress_select_blocks_vasc(q: torch.Tensor, k: torch.Tensor, v: Optional[torch.Tensor],
                            budgets, block: int, capacity: Optional[int] = None,
                            memory: Optional[torch.Tensor] = None, value_aware: bool = True,
                            reset: Optional[bool] = None, idx: Optional[torch.Tensor] = None,
                            demand: Optional[torch.Tensor] = None,
                            service: Optional[torch.Tensor] = None,
                            workspace: Optional[torch.Tensor] = None,
                            stream: Optional[torch.cuda.Stream] = None
                            ) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor],
                                       Optional[torch.Tensor]]:
    """VASC selection of one global layer: returns (idx [H, nb, capacity]
    int32, memory [H, pairs] float32 settled in place, demand, service).

    ``budgets`` holds c_h for every head (an int applies to all); capacity
    defaults to the largest.  Without ``memory`` a zeroed one is made and
    ``reset`` defaults to True (the first global layer); with one, ``reset``
    defaults to False.  ``demand`` / ``service`` ([H, pairs] float32) are
    filled when given.
    """
    _check_inputs(q, k, v)
    if value_aware and v is None:
        raise ValueError("the value contrast needs v (or value_aware=False)")
    sh = _shape_of(q, block)
    n, h = q.shape[0], q.shape[1]
    nb = n // block
    pairs = vasc_pairs(nb)
    per_head = [int(budgets)] * h if isinstance(budgets, int) else [int(b) for b in budgets]
    if len(per_head) != h:
        raise ValueError(f"budgets needs {h} entries, got {len(per_head)}")
    cap = max(per_head) if capacity is None else int(capacity)
    if memory is None:
        memory = torch.zeros((h, pairs), dtype=torch.float32, device=q.device)
        reset = True if reset is None else reset
    reset = False if reset is None else reset
    if idx is None:
        idx = torch.empty((h, nb, max(cap, 1)), dtype=torch.int32, device=q.device)
    _check_buffer(memory, (h, pairs), torch.float32, q.device, "memory")
    _check_buffer(idx, (h, nb, max(cap, 1)), torch.int32, q.device, "idx")
    for name, t in (("demand", demand), ("service", service)):
        if t is not None:
            _check_buffer(t, (h, pairs), torch.float32, q.device, name)
    _check_workspace(workspace, q.device)
    need = int(lib.ress_vasc_workspace_bytes(ctypes.byref(sh)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    host_budgets = (ctypes.c_int32 * h)(*per_head)
    status = _on(q.device, lib.ress_select_blocks_vasc, ctypes.byref(sh), _ptr(q), _ptr(k),
                 _ptr(v), ctypes.cast(host_budgets, _P), cap, int(bool(value_aware)),
                 int(bool(reset)), _ptr(memory), _ptr(idx), _ptr(demand), _ptr(service),
                 _ptr(workspace), workspace.numel(), _stream_ptr(stream, q.device))
    _check(status, "ress_select_blocks_vasc")
    return idx, memory, demand, service


def ress_validate_idx(idx: torch.Tensor, n: int, block: int,
                      stream: Optional[torch.cuda.Stream] = None) -> None:
    """Checks idx [H, nb, budget] on the device (in range, strictly ascending
    rows); a bad row shows up in ress_check_device_errors (RESS_ERR_BAD_INDEX,
    detail 80 out of range, 81 repeated block, 82 not ascending)."""
    if idx.dim() != 3:
        raise ValueError(f"idx must be [H, nb, budget], got {tuple(idx.shape)}")
    h = idx.shape[0]
    _check_idx(idx, h, n // block, idx.device)
    sh = make_shape(n, h, block, torch.bfloat16)
    status = _on(idx.device, lib.ress_validate_idx, ctypes.byref(sh), int(idx.shape[2]), _ptr(idx),
                 _stream_ptr(stream, idx.device))
    _check(status, "ress_validate_idx")


def ress_check_device_errors(stream: Optional[torch.cuda.Stream] = None,
                             device: Optional[torch.device] = None) -> Tuple[int, int]:
    """Synchronise and return (status, detail) of the device error flag (cleared)."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    detail = ctypes.c_int32(0)
    status = _on(dev, lib.ress_check_device_errors, _stream_ptr(stream, dev), ctypes.byref(detail))
    return int(status), int(detail.value)
