"""Token-band GQA prefill and rolling-buffer GQA decode against the oracle."""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as orc
from tol import check_bf16, check_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def swa():
    import streaming_frame_causal_b200 as m
    return m


@pytest.mark.parametrize("N,Hq,Hkv,D,W,dtype", [
    (700, 4, 2, 64, 200, torch.bfloat16),
    (520, 3, 1, 64, 130, torch.bfloat16),     # odd group size: single-head items
    (300, 4, 4, 64, 1000, torch.bfloat16),    # window wider than the sequence
    (640, 8, 2, 128, 256, torch.bfloat16),    # head_dim 128, two query-head pairs per group
    (333, 2, 2, 128, 64, torch.bfloat16),     # ragged last query tile, no grouping
    (200, 4, 2, 128, 50, torch.float32),
    (90, 2, 1, 32, 7, torch.float32),
])
def test_band_parity(swa, N, Hq, Hkv, D, W, dtype):
    q = synth.normal((1, N, Hq, D), 11, dtype)
    k = synth.normal((1, N, Hkv, D), 12, dtype)
    v = synth.normal((1, N, Hkv, D), 13, dtype)
    out = torch.empty(q.shape, dtype=dtype, device="cuda")
    swa.swa_band_prefill(q.cuda(), k.cuda(), v.cuda(), out, window=W)
    torch.cuda.synchronize()
    assert swa.swa_device_error_check() == 0
    ref = orc.band_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), W)
    got = out.float().cpu().numpy()
    (check_bf16 if dtype == torch.bfloat16 else check_f32)(got, ref, "band")


@pytest.mark.parametrize("B,W,pos,Hq,Hkv,D,dtype", [
    (3, 64, 200, 8, 2, 128, torch.bfloat16),
    (2, 64, 10, 8, 2, 128, torch.bfloat16),     # buffer not yet full
    (2, 96, 95, 4, 1, 64, torch.bfloat16),      # exactly full
    (2, 32, 40, 4, 2, 64, torch.float32),
    # head_dim 128 on the tensor cores: one to eight query heads per KV head,
    # a ragged last key tile, a partly filled window over several tiles, and a
    # single KV head whose keys are cut into five pieces
    (2, 300, 1000, 16, 16, 128, torch.bfloat16),
    (4, 1024, 500, 16, 8, 128, torch.bfloat16),
    (3, 256, 700, 64, 8, 128, torch.bfloat16),
    (1, 640, 639, 8, 1, 128, torch.bfloat16),
    (2, 130, 129, 4, 1, 128, torch.bfloat16),
    # head_dim 64 on the same kernel (one 64-column sub-tile per key tile)
    (2, 700, 699, 8, 4, 64, torch.bfloat16),
    (3, 300, 1000, 8, 8, 64, torch.bfloat16),
    # group sizes that are not powers of two: 3, 5, 6 and 7 query heads per KV head
    (2, 512, 2000, 12, 4, 128, torch.bfloat16),
    (2, 260, 259, 10, 2, 64, torch.bfloat16),
    (1, 384, 5000, 24, 4, 128, torch.bfloat16),
    (2, 200, 150, 14, 2, 64, torch.bfloat16),
])
def test_decode_parity(swa, B, W, pos, Hq, Hkv, D, dtype):
    q, kn, vn, kc, vc = synth.decode_inputs(seed=pos, B=B, W=W, Hq=Hq, Hkv=Hkv, D=D, dtype=dtype)
    kcd, vcd = kc.cuda(), vc.cuda()
    out = torch.empty(q.shape, dtype=dtype, device="cuda")
    swa.swa_decode(q.cuda(), kn.cuda(), vn.cuda(), kcd, vcd, pos, out)
    torch.cuda.synchronize()
    assert swa.swa_device_error_check() == 0
    ref, kref, vref = orc.decode(q.float().numpy(), kn.float().numpy(), vn.float().numpy(),
                                 kc.float().numpy(), vc.float().numpy(), pos, W)
    got = out.float().cpu().numpy()
    (check_bf16 if dtype == torch.bfloat16 else check_f32)(got, ref, "decode")
    np.testing.assert_array_equal(kcd.float().cpu().numpy(), kref)
    np.testing.assert_array_equal(vcd.float().cpu().numpy(), vref)


def test_decode_full_workload(swa):
    """Batch 64 at position 200000 (slot 3392) against a 4096-slot cache, GQA 32/8, D=128."""
    q, kn, vn, kc, vc = synth.decode_inputs(seed=1)
    kcd, vcd = kc.cuda(), vc.cuda()
    out = torch.empty(q.shape, dtype=q.dtype, device="cuda")
    swa.swa_decode(q.cuda(), kn.cuda(), vn.cuda(), kcd, vcd, 200000, out)
    torch.cuda.synchronize()
    ref, _, _ = orc.decode(q.float().numpy(), kn.float().numpy(), vn.float().numpy(),
                           kc.float().numpy(), vc.float().numpy(), 200000, 4096)
    check_bf16(out.float().cpu().numpy(), ref, "decode full")
    assert torch.equal(kcd[:, 3392].cpu(), kn)
    assert torch.equal(vcd[:, 3392].cpu(), vn)


def test_band_full_workload_sampled_rows(swa):
    """32768 tokens, GQA 32/8, D=128, window 4096: rows near the start (partial
    windows), at the window edge and at the end, on heads of different groups."""
    q, k, v = synth.band_qkv(seed=1)
    out = torch.empty(q.shape, dtype=q.dtype, device="cuda")
    swa.swa_band_prefill(q.cuda(), k.cuda(), v.cuda(), out, window=4096)
    torch.cuda.synchronize()
    assert swa.swa_device_error_check() == 0
    rows = np.array([0, 1, 127, 128, 4094, 4095, 4096, 4097, 8191, 8192, 20000, 32640, 32767])
    heads = [0, 3, 4, 17, 31]
    ref = orc.band_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), 4096,
                             rows=rows, heads=heads)
    check_bf16(out.float().cpu().numpy()[:, rows][:, :, heads], ref, "band full")
