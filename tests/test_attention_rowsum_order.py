"""The fused-attention tests' emulation of the call's row-sum order, pinned on the host: with every score
equal to the row maximum each allowed numerator is exp(0) = 1 exactly, so every row sum must be the
row's number of allowed keys, whatever the split count (the ranges, tiles and column blocks of the
emulation then have to cover each allowed key exactly once and no masked one)."""
import numpy as np
import pytest

from tests.test_gpu_attention_fused import _row_sums_in_call_order


@pytest.mark.parametrize("causal,q_offset", [(True, 100), (True, 0), (True, -60), (False, 0)])
@pytest.mark.parametrize("splits", [1, 2, 3, 5])
def test_row_sum_emulation_counts_allowed_keys(causal, q_offset, splits):
    H, Tq, Tk = 2, 256, 320
    s = np.zeros((H, Tq, Tk), np.float32)
    m = np.zeros((H, Tq), np.float32)
    got = _row_sums_in_call_order(s, m, causal, q_offset, splits)
    q = np.arange(Tq)
    want = np.clip(q + q_offset + 1, 0, Tk) if causal else np.full(Tq, Tk)
    assert np.array_equal(got, np.broadcast_to(want.astype(np.float32), (H, Tq)))
