"""Failure detection on the GPU without a fault: a bounded wait on an
mbarrier that nothing arrives at runs out after about a second, reports
SALA_ERR_TIMEOUT through the device status word, and leaves the context
usable."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out(cuda_device):
    from hybrid_sparse_linear_lightning_b200 import sala
    assert sala.sala_get_device_status() == sala.SALA_OK
    assert sala.sala_selftest_bounded_wait() == sala.SALA_ERR_TIMEOUT
    # the status word was cleared by the read, and the context still works
    assert sala.sala_get_device_status() == sala.SALA_OK
    x = torch.arange(4096, device=cuda_device, dtype=torch.float32)
    assert float(x.sum()) == 4095 * 4096 / 2
