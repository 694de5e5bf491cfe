"""The allocation-free selection entry point, called through the C ABI,
returns the same kept-block masks as the workspace entry point, on two calls
in a row (the fixed scratch array keeps the previous call's contents).

Some callers cannot allocate device memory (a plugin inside another
framework's allocator, or a loop where an allocation is not allowed); they
use ress_select_blocks_noalloc.  This file is collected last so that a run
that stops at the first failure has already run every other test."""

import ctypes

import pytest
import torch

from block_sparse_global_mean_b200 import workloads

pytestmark = pytest.mark.gpu


def _call_noalloc(ress, w, q, k, v, idx):
    sh = ress.make_shape(w.n_tokens, w.heads, w.block, q.dtype)
    stream = torch.cuda.current_stream().cuda_stream
    status = ress.lib.ress_select_blocks_noalloc(
        ctypes.byref(sh), q.data_ptr(), k.data_ptr(), v.data_ptr() if w.lam else None,
        w.budget, ctypes.c_float(w.lam), idx.data_ptr(), stream)
    return status


@pytest.mark.parametrize("name", ["vggt8", "views32"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(name, ress_gpu):
    w = workloads.WORKLOADS[name]
    q, k, v = workloads.generate(w, device="cuda")
    ref = ress_gpu.ress_select_blocks(q, k, v if w.lam else None, w.budget, w.lam, w.block)
    assert ress_gpu.ress_check_device_errors()[0] == 0
    for _ in range(2):
        idx = torch.full_like(ref, -1)
        assert _call_noalloc(ress_gpu, w, q, k, v, idx) == ress_gpu.RESS_OK
        assert ress_gpu.ress_check_device_errors()[0] == 0
        # Masks are integer outputs: the tolerance is bit-exact.
        assert torch.equal(idx, ref)


def test_noalloc_rejects_problems_beyond_its_fixed_scratch(ress_gpu):
    # H = 64, nb = 4,096: about 134 MB of scratch, more than the fixed 32 MiB.
    w = workloads.Workload("big", 1, 64 * 4096, 64 * 4096, 64, 64, "bf16", 64, 8, 0.0, 0, "iid")
    sh = ress_gpu.make_shape(w.n_tokens, w.heads, w.block, torch.bfloat16)
    fake = 1 << 20     # aligned, never dereferenced: the call returns before any launch
    status = ress_gpu.lib.ress_select_blocks_noalloc(ctypes.byref(sh), fake, fake, None, 8,
                                                     ctypes.c_float(0.0), fake, None)
    assert status == ress_gpu.RESS_ERR_WORKSPACE
