"""ress_validate_idx on the GPU: a selection's own output passes; planted bad
rows (made on the host, read only by the bounded validation kernel) are
flagged with their detail code, and the flag clears once read."""

import numpy as np
import pytest
import torch

from tests.parity import poison

pytestmark = pytest.mark.gpu


def _validate(ress, idx_np, n, block):
    idx = torch.from_numpy(np.ascontiguousarray(idx_np, dtype=np.int32)).cuda()
    ress.ress_validate_idx(idx, n, block)
    return ress.ress_check_device_errors()


def test_selection_output_passes(ress_gpu):
    g = torch.Generator().manual_seed(8)
    nb, H, B, budget = 40, 3, 64, 9
    q, k = (torch.randn(nb * B, H, 64, generator=g).to(torch.bfloat16).cuda() for _ in range(2))
    idx = ress_gpu.ress_select_blocks(q, k, None, budget, 0.0, B,
                                      idx=poison((H, nb, budget), torch.int32))
    ress_gpu.ress_validate_idx(idx, nb * B, B)
    assert ress_gpu.ress_check_device_errors() == (0, 0)


@pytest.mark.parametrize("row,detail", [([0, 3, 40], 80), ([-1, 3, 7], 80), ([2, 2, 7], 81),
                                        ([5, 3, 7], 82), ([0, 1, 39], 0)])
def test_planted_rows_are_flagged(row, detail, ress_gpu):
    nb, H, B = 40, 2, 128
    idx = np.tile(np.array([1, 4, 9], dtype=np.int32), (H, nb, 1))
    idx[1, 17] = row
    status, got = _validate(ress_gpu, idx, nb * B, B)
    if detail == 0:
        assert (status, got) == (0, 0)
    else:
        assert status == ress_gpu.RESS_ERR_BAD_INDEX and got == detail
        assert ress_gpu.ress_check_device_errors() == (0, 0)       # cleared


def test_budget_one_and_full_budget(ress_gpu):
    nb, B = 33, 64
    assert _validate(ress_gpu, np.arange(nb).reshape(1, nb, 1), nb * B, B) == (0, 0)
    full = np.tile(np.arange(nb), (2, nb, 1))
    assert _validate(ress_gpu, full, nb * B, B) == (0, 0)
    full[0, 32, 31:] = [32, 31]
    status, detail = _validate(ress_gpu, full, nb * B, B)
    assert status == ress_gpu.RESS_ERR_BAD_INDEX and detail == 82
