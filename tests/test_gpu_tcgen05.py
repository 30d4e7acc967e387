"""The tensor-memory MMA building block (mkv_selftest_tc_logits): 128 token rows written to TMEM
by their threads, Q read from shared memory by tcgen05.mma, the fp32 result read back from TMEM.
Inputs on exact grids (codes c - 3.5, queries in 1/16 steps) make the float64 reference exact."""
import numpy as np
import pytest
import torch

from mixed_format_paged_mkv_b200 import Pool

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seed", [1, 2])
def test_tensor_memory_mma_is_exact(seed):
    rng = np.random.default_rng(seed)
    a = rng.integers(0, 8, size=(128, 256)) - 3.5
    q = (rng.integers(-32, 32, size=(8, 256)) / 16.0)
    pool = Pool(1, 64, 1, 1, 1, 1)
    d = pool.selftest_tc_logits(torch.tensor(a, dtype=torch.float16, device="cuda"),
                                torch.tensor(q, dtype=torch.float16, device="cuda"))
    torch.cuda.synchronize()
    pool.device_status()
    assert np.array_equal(d.cpu().numpy().astype(np.float64), a @ q.T)
