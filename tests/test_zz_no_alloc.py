"""swa_decode_noalloc -- the decode entry point for callers that cannot allocate
device memory (its split-K scratch is a fixed array inside the library) --
checked through the C ABI against swa_decode with a caller-provided workspace
and against the float64 oracle.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test; it also passes on its own."""
import ctypes as C
import os
import re

import numpy as np
import pytest
import torch

import synth
from oracle import attention as orc
from tol import check_bf16

pytestmark = pytest.mark.gpu

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "swa.h")


def scratch_bytes_from_header():
    """SWA_DECODE_NOALLOC_SCRATCH_BYTES as include/swa.h defines it."""
    with open(HEADER) as f:
        m = re.search(r"#define\s+SWA_DECODE_NOALLOC_SCRATCH_BYTES\s+\(([^)]*)\)", f.read())
    expr = m.group(1).replace("u", "")
    assert re.fullmatch(r"[\d\s*+]+", expr), expr
    return int(eval(expr))


def _call_noalloc(lib, q, kn, vn, kc, vc, pos, out, dtype=1):
    B, Hq, D = q.shape
    W, Hkv = kc.shape[1], kc.shape[2]
    return lib.swa_decode_noalloc(q.data_ptr(), kn.data_ptr(), vn.data_ptr(), kc.data_ptr(), vc.data_ptr(),
                                  C.c_longlong(pos), W, B, Hq, Hkv, D, out.data_ptr(), dtype,
                                  torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("B,W,pos,Hq,Hkv,D", [(8, 1024, 5000, 32, 8, 128), (4, 256, 100, 8, 2, 64)])
def test_noalloc_decode_matches_workspace_decode_twice(B, W, pos, Hq, Hkv, D):
    import streaming_frame_causal_b200 as swa
    lib = swa._lib
    inputs = synth.decode_inputs(seed=pos, B=B, W=W, Hq=Hq, Hkv=Hkv, D=D)
    q, kn, vn, kc, vc = (t.cuda() for t in inputs)
    kc_ref, vc_ref = kc.clone(), vc.clone()
    ref = torch.empty_like(q)
    swa.swa_decode(q, kn, vn, kc_ref, vc_ref, pos, ref)
    torch.cuda.synchronize()
    ref_np = ref.float().cpu().numpy()
    want, _, _ = orc.decode(*(t.float().numpy() for t in inputs), pos, W)
    for call in range(2):
        kc2, vc2 = kc.clone(), vc.clone()
        out = torch.full_like(q, float("nan"))
        assert _call_noalloc(lib, q, kn, vn, kc2, vc2, pos, out) == 0
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        check_bf16(got, ref_np, f"no-alloc decode vs swa_decode, call {call}")
        check_bf16(got, want, f"no-alloc decode vs oracle, call {call}")
        assert torch.equal(kc2, kc_ref) and torch.equal(vc2, vc_ref)
    assert swa.swa_device_error_check() == 0


@pytest.mark.parametrize("D", [64, 128])
def test_slots_past_the_position_may_hold_nan(D):
    # a partly filled rolling cache: slots pos+1..W-1 were never written (NaN
    # here); neither decode may let them reach the output
    import streaming_frame_causal_b200 as swa
    lib = swa._lib
    B, W, Hq, Hkv, pos = 3, 512, 8, 2, 200
    q, kn, vn, kc, vc = synth.decode_inputs(seed=5 + D, B=B, W=W, Hq=Hq, Hkv=Hkv, D=D)
    kc[:, pos + 1:] = float("nan")
    vc[:, pos + 1:] = float("nan")
    want, _, _ = orc.decode(q.float().numpy(), kn.float().numpy(), vn.float().numpy(), kc.float().numpy(),
                            vc.float().numpy(), pos, W)
    for which in ("swa_decode", "swa_decode_noalloc"):
        kcd, vcd = kc.cuda(), vc.cuda()
        out = torch.full((B, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        if which == "swa_decode":
            swa.swa_decode(q.cuda(), kn.cuda(), vn.cuda(), kcd, vcd, pos, out)
        else:
            assert _call_noalloc(lib, q.cuda(), kn.cuda(), vn.cuda(), kcd, vcd, pos, out) == 0
        torch.cuda.synchronize()
        check_bf16(out.float().cpu().numpy(), want, which)
    assert swa.swa_device_error_check() == 0


def test_noalloc_capacity_boundary():
    # 64 query / 8 KV heads of 128, 4096 slots: 63 sequences fit the fixed
    # scratch, 64 do not (the partial count jumps with the batch)
    import streaming_frame_causal_b200 as swa
    lib = swa._lib
    cap = scratch_bytes_from_header()
    Hq, Hkv, D, W, pos = 64, 8, 128, 4096, 9000
    assert swa.swa_decode_workspace_bytes(63, Hq, Hkv, D, W) <= cap < swa.swa_decode_workspace_bytes(64, Hq, Hkv,
                                                                                                    D, W)
    dummy = 256
    assert lib.swa_decode_noalloc(dummy, dummy, dummy, dummy, dummy, C.c_longlong(pos), W, 64, Hq, Hkv, D, dummy,
                                  1, None) == -4
    q, kn, vn, kc, vc = (t.cuda() for t in synth.decode_inputs(seed=11, B=63, W=W, Hq=Hq, Hkv=Hkv, D=D))
    ref = torch.empty_like(q)
    kr, vr = kc.clone(), vc.clone()
    swa.swa_decode(q, kn, vn, kr, vr, pos, ref)
    out = torch.empty_like(q)
    assert _call_noalloc(lib, q, kn, vn, kc, vc, pos, out) == 0
    torch.cuda.synchronize()
    check_bf16(out.float().cpu().numpy(), ref.float().cpu().numpy(), "no-alloc decode at capacity")
    assert swa.swa_device_error_check() == 0


def test_noalloc_decode_rejects_oversize_and_f32():
    import streaming_frame_causal_b200 as swa
    lib = swa._lib
    # 1024 sequences x 8 KV heads x 4 query heads of 128 need more than the fixed scratch
    need = swa.swa_decode_workspace_bytes(1024, 32, 8, 128, 4096)
    assert need > scratch_bytes_from_header()
    dummy = 256
    assert lib.swa_decode_noalloc(dummy, dummy, dummy, dummy, dummy, C.c_longlong(10), 4096, 1024, 32, 8,
                                  128, dummy, 1, None) == -4
    assert lib.swa_decode_noalloc(dummy, dummy, dummy, dummy, dummy, C.c_longlong(10), 64, 2, 8, 2,
                                  128, dummy, 0, None) == -7
