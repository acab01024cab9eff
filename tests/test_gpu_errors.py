"""Bounded device waits: a wait that runs out latches an error the host reads,
and the context stays usable afterwards."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_cleared():
    import streaming_frame_causal_b200 as swa
    assert swa.swa_device_error_check() == 0
    swa.swa_debug_wait_timeout(2000)     # 2 ms on a flag nothing sets
    assert swa.swa_device_error_check() == -6
    assert swa.swa_device_error_check() == 0
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0
