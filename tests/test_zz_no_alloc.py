"""GPU test of dlrm_sparse_interact_host_static, the host-buffer stage whose
device staging is a fixed array inside the library.

It exists for callers that cannot allocate device memory: a plugin run by a
framework that owns the device's memory, code running while a CUDA graph is
captured on the device, or a loop that must not synchronise the device with
cudaMalloc/cudaFree. The test calls it through the C ABI (ctypes) and checks
each result against dlrm_sparse_interact_host, the entry point that stages in
caller-allocated buffers, on two calls in a row with different inputs: the
second call must not see what the first left in the shared array. Pooled
vectors and the dense part of concatenated rows must match bit for bit, dots
within 1e-5 * sum_d |v_i[d] v_j[d]|, as in the other parity tests.

The file is named so that pytest collects it last.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from dlrm_embedding_bag_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def ops():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from dlrm_embedding_bag_b200 import ops as _ops

    return _ops


def _batch(w: syn.Workload, replica: int):
    """Pinned host inputs of one batch of the workload."""
    idx = torch.from_numpy(syn.make_indices(w, replica=replica).reshape(-1)).pin_memory()
    off = torch.from_numpy(syn.make_offsets(w)).pin_memory()
    g = torch.Generator()
    g.manual_seed(3000 + replica)
    dense = torch.randn((w.B, w.D), generator=g).pin_memory()
    return idx, off, dense


def _static_call(ops, weights, idx, off, dense, w, concat, pooled_host, inter_host):
    """One call of the entry point through the C ABI, on the current stream."""
    F = len(weights)
    arr = (ctypes.c_void_p * F)(*[t.data_ptr() for t in weights])
    return ops._lib.dlrm_sparse_interact_host_static(
        arr, idx.data_ptr(), off.data_ptr(), dense.data_ptr(), w.B, F, w.L, w.D,
        1 if concat else 0, pooled_host.data_ptr() if pooled_host is not None else None,
        inter_host.data_ptr(), torch.cuda.current_stream().cuda_stream)


def _dot_bound(dense: np.ndarray, pooled: np.ndarray) -> np.ndarray:
    """S_ij = sum_d |v_i[d] v_j[d]| over the pairs of the strict lower triangle."""
    v = np.concatenate([dense[:, None, :], pooled], axis=1).astype(np.float64)
    i, j = np.tril_indices(v.shape[1], -1)
    return np.einsum("bpd,bpd->bp", np.abs(v[:, i, :]), np.abs(v[:, j, :]))


def _compare(got_inter, got_pooled, ref_inter, ref_pooled, dense, D, concat, what):
    assert np.array_equal(got_pooled.numpy().view(np.uint32), ref_pooled.numpy().view(np.uint32)), \
        f"{what}: pooled vectors differ"
    gi, ri = got_inter.numpy(), ref_inter.numpy()
    if concat:
        assert np.array_equal(gi[:, :D].view(np.uint32), ri[:, :D].view(np.uint32)), \
            f"{what}: dense part differs"
        gi, ri = gi[:, D:], ri[:, D:]
    bound = _dot_bound(dense.numpy(), ref_pooled.numpy())
    err = np.abs(gi.astype(np.float64) - ri.astype(np.float64))
    assert np.all(err <= 1e-5 * bound + 1e-30), f"{what}: dots differ by up to {err.max()}"


def test_static_staging_matches_caller_staging_on_two_calls(ops):
    w1 = syn.C2_CONCAT.scaled(B=300)   # F=8, 1e5 x 64 tables, L=32, rows [dense | dots]
    w2 = syn.C2_CONCAT.scaled(B=123, L=20)
    weights = syn.make_weights(w1, DEV)
    cases = [(w1, True, 11), (w2, False, 12)]
    results = []
    for w, concat, replica in cases:
        idx, off, dense = _batch(w, replica)
        row = w.D + w.P if concat else w.P
        inter = torch.full((w.B, row), float("nan")).pin_memory()
        pooled = torch.full((w.B, w.F, w.D), float("nan")).pin_memory()
        ref_inter = torch.empty((w.B, row)).pin_memory()
        ref_pooled = torch.empty((w.B, w.F, w.D)).pin_memory()
        stage = ops.HostStage(weights, w.B, w.L, concat_dense=concat, want_pooled=True)
        results.append((w, concat, idx, off, dense, inter, pooled, ref_inter, ref_pooled, stage))
    torch.cuda.synchronize()

    for n, (w, concat, idx, off, dense, inter, pooled, ref_inter, ref_pooled, stage) in \
            enumerate(results):
        free_before = torch.cuda.mem_get_info()[0]
        rc = _static_call(ops, weights, idx, off, dense, w, concat, pooled, inter)
        assert rc == 0, ops.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        if n > 0:  # after the first call's set-up, a call allocates nothing
            assert torch.cuda.mem_get_info()[0] == free_before
        stage(idx, off, dense, ref_inter, ref_pooled)
        torch.cuda.synchronize()
        _compare(inter, pooled, ref_inter, ref_pooled, dense, w.D, concat,
                 f"call {n + 1} ({w.name}, concat={concat})")


def test_static_staging_rejects_oversized_calls(ops):
    w = syn.C2_CONCAT.scaled(B=1 << 16)  # 64 MiB of indices: more than the array holds
    weights = syn.make_weights(w.scaled(N=16), DEV)
    F = len(weights)
    arr = (ctypes.c_void_p * F)(*[t.data_ptr() for t in weights])
    fake = 0x10000  # never dereferenced: the size check fails first
    rc = ops._lib.dlrm_sparse_interact_host_static(arr, fake, fake, fake, w.B, F, w.L, w.D, 1,
                                                   None, fake, None)
    assert rc == -10
    assert ops.STATUS[rc] == "DLRM_ERR_SCRATCH"
