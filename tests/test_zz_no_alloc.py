"""swa_decode_noalloc -- the decode entry point for callers that cannot allocate
device memory (its split-K scratch is a fixed array inside the library) --
checked through the C ABI against swa_decode with a caller-provided workspace.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test; it also passes on its own."""
import ctypes as C

import numpy as np
import pytest
import torch

import synth
from tol import check_bf16

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, q, kn, vn, kc, vc, pos, out):
    B, Hq, D = q.shape
    W, Hkv = kc.shape[1], kc.shape[2]
    return lib.swa_decode_noalloc(q.data_ptr(), kn.data_ptr(), vn.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                  C.c_longlong(pos), W, B, Hq, Hkv, D, out.data_ptr(), 1,
                                  torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("B,W,pos,Hq,Hkv,D", [(8, 1024, 5000, 32, 8, 128), (4, 256, 100, 8, 2, 64)])
def test_noalloc_decode_matches_workspace_decode_twice(B, W, pos, Hq, Hkv, D):
    import streaming_frame_causal_b200 as swa
    lib = swa._lib
    q, kn, vn, kc, vc = (t.cuda() for t in synth.decode_inputs(seed=pos, B=B, W=W, Hq=Hq, Hkv=Hkv, D=D))
    kc_ref, vc_ref = kc.clone(), vc.clone()
    ref = torch.empty_like(q)
    swa.swa_decode(q, kn, vn, kc_ref, vc_ref, pos, ref)
    torch.cuda.synchronize()
    ref_np = ref.float().cpu().numpy()
    for call in range(2):
        kc2, vc2 = kc.clone(), vc.clone()
        out = torch.full_like(q, float("nan"))
        assert _call_noalloc(lib, q, kn, vn, kc2, vc2, pos, out) == 0
        torch.cuda.synchronize()
        check_bf16(out.float().cpu().numpy(), ref_np, f"no-alloc decode, call {call}")
        assert torch.equal(kc2, kc_ref) and torch.equal(vc2, vc_ref)
    assert swa.swa_device_error_check() == 0


def test_noalloc_decode_rejects_oversize_and_f32():
    import streaming_frame_causal_b200 as swa
    lib = swa._lib
    # 1024 sequences x 8 KV heads x 4 query heads of 128 need more than the fixed scratch
    need = swa.swa_decode_workspace_bytes(1024, 32, 8, 128, 4096)
    assert need > lib_scratch_bytes()
    dummy = 256
    assert lib.swa_decode_noalloc(dummy, dummy, dummy, dummy, dummy, C.c_longlong(10), 4096, 1024, 32, 8,
                                  128, dummy, 1, None) == -4
    assert lib.swa_decode_noalloc(dummy, dummy, dummy, dummy, dummy, C.c_longlong(10), 64, 2, 8, 2,
                                  128, dummy, 0, None) == -7


def lib_scratch_bytes():
    return 16 * 1024 * 1024
