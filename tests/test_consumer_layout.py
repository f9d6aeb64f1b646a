"""The tensor-core product reads block scales where the oracle's tile layout puts them (host only: the
library evaluates the consumer's own scale layout without touching a GPU)."""
import numpy as np
import pytest

import nvfp4_block_scaled_11_b200 as nv
from oracle import oracle as O


@pytest.mark.parametrize("rows,K,batch", [(128, 64, 1), (200, 128, 2), (1, 32, 3), (300, 96, 1),
                                          (129, 8192, 1), (64, 256, 4)])
def test_consumer_reads_scales_at_oracle_offsets(rows, K, batch):
    bpr = K // 16
    per = O.sf_mma_bytes(rows, bpr)
    want = np.array([l * per + O.sf_mma_offset(r, c, bpr) for l in range(batch) for r in range(rows)
                     for c in range(bpr)], np.int64)
    assert np.array_equal(nv.gemm_sf_offsets(rows, K, batch), want)
    assert nv.sf_mma_bytes(rows, K, batch) == batch * per


def test_sf_mma_bytes_rejects_bad_sizes():
    with pytest.raises(nv.NVFP4Error):
        nv.sf_mma_bytes(10, 24)
    with pytest.raises(nv.NVFP4Error):
        nv.sf_mma_bytes(-1, 32)
    assert nv.sf_mma_bytes(0, 32) == 0
