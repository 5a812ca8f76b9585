"""Bounded device-side waits: a wait nobody satisfies ends with
MMSP_ETIMEOUT from mmsp_device_status(), no trap, no hang, and the context
stays usable."""
import pytest
import torch

from gpu_util import lib, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]


def test_bounded_wait_reports_timeout_then_clears():
    m = lib()
    m.mmsp_device_status()  # clean start
    m.mmsp_selftest_bounded_wait(200000)
    with pytest.raises(m.MmspError) as e:
        m.mmsp_device_status()
    assert e.value.status == 4
    m.mmsp_device_status()  # cleared
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0  # context still usable
