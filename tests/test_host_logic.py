"""Host-side logic of the test and bench harness, on the CPU."""
import numpy as np
import torch

import oracle
from gpu_cases import sampled_oracle


def test_sampled_oracle_matches_full_oracle():
    rng = np.random.default_rng(3)
    B, F, N, D, L = 37, 3, 50, 8, 5
    weights = [torch.from_numpy(rng.normal(0, 0.1, (N, D)).astype(np.float32)) for _ in range(F)]
    idx = rng.integers(0, N, (F, B * L)).astype(np.int32)
    # ragged offsets with some empty bags
    offs = np.sort(rng.integers(0, B * L + 1, (F, B)), axis=1).astype(np.int32)
    offs[:, 0] = 0
    dense = torch.from_numpy(rng.normal(0, 1, (B, D)).astype(np.float32))
    ws = [w.numpy() for w in weights]
    pooled = oracle.embbag_sum_multi(ws, idx, offs, B, L)
    inter = oracle.interact_lower_tri(dense.numpy(), pooled, concat_dense=True)
    samples = np.array([0, 5, 17, 36])
    sp, si, sb = sampled_oracle(weights, idx, offs, dense, B, L, samples, True)
    assert np.array_equal(sp.view(np.uint32), pooled[samples].view(np.uint32))
    assert np.array_equal(si.view(np.uint32), inter[samples].view(np.uint32))
    assert sb.shape == (4, F * (F + 1) // 2)
