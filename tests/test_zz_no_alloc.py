"""The allocation-free selection entry point, called through the C ABI,
returns the same kept-block masks as the workspace entry point, on two calls
in a row (the fixed scratch array keeps the previous call's contents).

Some callers cannot allocate device memory (a plugin inside another
framework's allocator, or a loop where an allocation is not allowed); they
use ress_select_blocks_noalloc.  This file is collected last so that a run
that stops at the first failure has already run every other test.  The
oversized-problem rejection, which needs no GPU, is in test_abi_cpu.py."""

import ctypes

import pytest
import torch

from block_sparse_global_mean_b200 import workloads
from tests.parity import poison

pytestmark = pytest.mark.gpu


def _call_noalloc(ress, w, q, k, v, idx):
    sh = ress.make_shape(w.n_tokens, w.heads, w.block, q.dtype)
    stream = torch.cuda.current_stream().cuda_stream
    status = ress.lib.ress_select_blocks_noalloc(
        ctypes.byref(sh), q.data_ptr(), k.data_ptr(), v.data_ptr() if w.lam else None,
        w.budget, ctypes.c_float(w.lam), idx.data_ptr(), stream)
    return status


def _reference(ress, w, q, k, v):
    ref = ress.ress_select_blocks(q, k, v if w.lam else None, w.budget, w.lam, w.block,
                                  idx=poison((w.heads, w.n_blocks, w.budget), torch.int32))
    assert ress.ress_check_device_errors()[0] == 0
    return ref


@pytest.mark.parametrize("name", ["tiny", "vggt8", "views32"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(name, ress_gpu):
    w = workloads.WORKLOADS[name]
    q, k, v = workloads.generate(w, device="cuda")
    ref = _reference(ress_gpu, w, q, k, v)
    for _ in range(2):
        idx = torch.full_like(ref, -1)
        assert _call_noalloc(ress_gpu, w, q, k, v, idx) == ress_gpu.RESS_OK
        assert ress_gpu.ress_check_device_errors()[0] == 0
        # Masks are integer outputs: the tolerance is bit-exact.
        assert torch.equal(idx, ref)


def test_a_smaller_call_after_a_larger_one(ress_gpu):
    """Calls of different sizes share the array: the 32-view call with the
    value contrast fills more of it than the 8-view call that follows, which
    must read only what it wrote itself."""
    for name in ["views32", "vggt8", "tiny", "views32"]:
        w = workloads.WORKLOADS[name]
        q, k, v = workloads.generate(w, device="cuda")
        ref = _reference(ress_gpu, w, q, k, v)
        idx = torch.full_like(ref, -1)
        assert _call_noalloc(ress_gpu, w, q, k, v, idx) == ress_gpu.RESS_OK
        assert ress_gpu.ress_check_device_errors()[0] == 0
        assert torch.equal(idx, ref), name
