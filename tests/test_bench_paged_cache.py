"""Host logic of the benchmark's paged-cache workload (bench.paged_cache):
the shuffled page pool and its block table describe the original cache
exactly, for both pool layouts (checked on the CPU through the oracle's
page gather)."""
import numpy as np
import pytest
import torch

import bench
from oracle import gather_pages


@pytest.mark.parametrize("layout", ["head_major", "token_major"])
def test_paged_cache_reproduces_the_contiguous_cache(layout):
    B, Hkv, S, E, ps = 3, 2, 64, 8, 16
    g = torch.Generator().manual_seed(0)
    k = torch.randn(B, Hkv, S, E, generator=g)
    v = torch.randn(B, Hkv, S, E + 8, generator=g)
    kp, vp, table = bench.paged_cache(k, v, ps, layout, seed=7)
    assert table.dtype == torch.int32 and table.shape == (B, S // ps)
    assert sorted(table.flatten().tolist()) == list(range(B * S // ps))  # every page used once
    if layout == "head_major":  # the oracle gathers token-major pools
        kp, vp = kp.transpose(1, 2), vp.transpose(1, 2)
    lens = np.full(B, S)
    for b in range(B):
        np.testing.assert_array_equal(gather_pages(kp, table.numpy(), lens, b), k[b].double().numpy())
        np.testing.assert_array_equal(gather_pages(vp, table.numpy(), lens, b), v[b].double().numpy())
    assert not torch.equal(table.flatten(), torch.arange(B * S // ps, dtype=torch.int32))  # shuffled
