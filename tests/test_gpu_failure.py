"""Failure detection on the GPU without a fault: a bounded wait that runs out
reports DLRM_FLAG_TIMEOUT through the status word, the kernel returns, and the
context stays usable for the next calls."""
import pytest
import torch

from dlrm_embedding_bag_b200 import ops

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def test_bounded_wait_times_out_and_context_survives():
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    ops.probe_bounded_wait(status, limit_cycles=2_000_000)  # about a millisecond
    torch.cuda.synchronize()
    assert int(status.item()) == ops.FLAG_TIMEOUT
    assert ops._lib.dlrm_status_from_flags(int(status.item())) == -8
    # the context is intact: an ordinary call runs and is correct
    w = [torch.arange(12, dtype=torch.float32, device=DEV).reshape(3, 4)]
    idx = torch.tensor([[0, 2]], dtype=torch.int32, device=DEV)
    off = torch.tensor([[0]], dtype=torch.int32, device=DEV)
    pooled = ops.embbag_sum_multi(w, idx, off, 2)
    torch.cuda.synchronize()
    assert pooled.flatten().tolist() == [8.0, 10.0, 12.0, 14.0]


def test_bounded_wait_limit_is_clamped():
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    ops.probe_bounded_wait(status, limit_cycles=0)  # raised to the minimum
    torch.cuda.synchronize()
    assert int(status.item()) == ops.FLAG_TIMEOUT
