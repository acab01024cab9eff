"""Bounded device waits: a wait that runs out latches an error the host reads,
every later call on the device returns it without launching until it is
cleared, and the context stays usable afterwards."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_cleared():
    import streaming_frame_causal_b200 as swa
    assert swa.swa_device_error_check() == 0
    swa.swa_debug_wait_timeout(2000)     # 2 ms on a flag nothing sets
    assert swa.swa_device_error_check() == -6
    assert swa.swa_device_error_check() == 0
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0


def test_latched_error_is_returned_by_the_next_calls():
    import streaming_frame_causal_b200 as swa
    lib = swa._lib
    assert swa.swa_device_error_check() == 0
    q, k, v = (t.cuda() for t in synth.tiny_qkv(seed=0))
    out = torch.empty_like(q)
    st = torch.cuda.current_stream().cuda_stream
    B, N, H, D = q.shape

    def prefill():
        return lib.swa_prefill(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), B, 8, 21, H * D, H, D,
                               3, 1, 2, 0, st)

    assert prefill() == 0
    torch.cuda.synchronize()
    swa.swa_debug_wait_timeout(1000)
    torch.cuda.synchronize()             # the wait has run out on the device
    n0 = swa.swa_launch_count()
    # no synchronizing check in between: the calls themselves report the error
    assert prefill() == -6
    assert prefill() == -6
    dq, dkn, dvn, dkc, dvc = (t.cuda() for t in synth.decode_inputs(seed=3, B=2, W=256, Hq=8, Hkv=2, D=64))
    dout = torch.empty_like(dq)
    assert lib.swa_decode_noalloc(dq.data_ptr(), dkn.data_ptr(), dvn.data_ptr(), dkc.data_ptr(), dvc.data_ptr(),
                                  100, 256, 2, 8, 2, 64, dout.data_ptr(), 1, st) == -6
    assert swa.swa_launch_count() == n0  # nothing was launched
    assert swa.swa_device_error_check() == -6
    assert prefill() == 0
    torch.cuda.synchronize()
    assert swa.swa_device_error_check() == 0
