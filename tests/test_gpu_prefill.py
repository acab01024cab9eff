"""Parity of the frame-causal prefill (tensor-core bf16 path and f32 path)
against the float64 oracle on identical seeded inputs."""
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


def _run(swa, q, k, v, F, P, sws, S, nfpb=1):
    dev = "cuda"
    out = torch.empty(q.shape, dtype=q.dtype, device=dev)
    swa.swa_prefill(q.to(dev), k.to(dev), v.to(dev), out, S=F, P=P, sliding_window_size=sws,
                    num_frame_per_block=nfpb, num_frame_for_scale=S)
    torch.cuda.synchronize()
    assert swa.swa_device_error_check() == 0
    return out.float().cpu().numpy()


def _ref(q, k, v, P, S, sws, nfpb=1, rows=None, heads=None):
    return orc.prefill(q.float().numpy(), k.float().numpy(), v.float().numpy(), P=P, scale_frames=S,
                       sliding_window_size=sws, num_frame_per_block=nfpb, rows=rows, heads=heads)


def test_tiny_config_f32(swa):
    """8 frames x 21 tokens, 2 heads x 32, window 3, 2 scale frames, float32."""
    q, k, v = synth.tiny_qkv(seed=0)
    got = _run(swa, q, k, v, 8, 21, 3, 2)
    check_f32(got, _ref(q, k, v, 21, 2, 3), "tiny f32")


@pytest.mark.parametrize("F,P,H,sws,S,nfpb", [
    (6, 200, 2, 2, 1, 1),      # two query tiles per frame (128 + 72), one pair
    (4, 1004, 2, 2, 1, 1),     # eight tiles per frame, ragged last tile of 108 rows
    (5, 100, 3, -1, 0, 1),     # single ragged tile per frame, full causal
    (3, 128, 1, 1, 0, 1),      # exact tile, window of one frame (block diagonal)
    (4, 129, 2, 5, 2, 1),      # one row past a tile; window wider than the clip
    (7, 60, 2, 1, 2, 2),       # window in blocks of two frames
    (1, 300, 2, 3, 0, 1),      # a single frame
    (9, 50, 2, 2, 12, 1),      # more scale frames than frames
])
def test_bf16_parity_small(swa, F, P, H, sws, S, nfpb):
    q, k, v = synth.tiny_qkv(seed=F * 1000 + P, F=F, P=P, H=H, D=64, dtype=torch.bfloat16)
    got = _run(swa, q, k, v, F, P, sws, S, nfpb)
    check_bf16(got, _ref(q, k, v, P, S, sws, nfpb), f"bf16 F{F} P{P}")


@pytest.mark.parametrize("D", [64, 128])
def test_bf16_growing_scores(swa, D):
    """Row maxima that climb by ~2^10 from key tile to key tile, with one jump of
    ~2^100, on alternate rows only: exercises the rescale of O and the row sum
    when the running max grows, the exact re-run of a tile whose scores jump too
    far, and warps whose lanes take different branches."""
    q, k, v = synth.growing_scores_qkv(D=D)
    got = _run(swa, q, k, v, 1, 1000, -1, 0)
    check_bf16(got, _ref(q, k, v, 1000, 0, -1), f"growing scores D{D}")


def test_bf16_head_dim_128(swa):
    q, k, v = synth.tiny_qkv(seed=128, F=5, P=260, H=2, D=128, dtype=torch.bfloat16)
    got = _run(swa, q, k, v, 5, 260, 2, 1)
    check_bf16(got, _ref(q, k, v, 260, 1, 2), "bf16 D128")


def test_f32_head_dims(swa):
    for D in (64, 128):
        q, k, v = synth.tiny_qkv(seed=D, F=5, P=17, H=2, D=D)
        got = _run(swa, q, k, v, 5, 17, 2, 1)
        check_f32(got, _ref(q, k, v, 17, 1, 2), f"f32 D{D}")


def test_batch_two(swa):
    q, k, v = synth.tiny_qkv(seed=7, B=2, F=4, P=150, H=2, D=64, dtype=torch.bfloat16)
    got = _run(swa, q, k, v, 4, 150, 2, 1)
    check_bf16(got, _ref(q, k, v, 150, 1, 2), "batch 2")


def test_empty_clip_is_noop(swa):
    q = torch.zeros(1, 0, 2, 64, dtype=torch.bfloat16, device="cuda")
    swa.swa_prefill(q, q, q, q, S=0, P=10, sliding_window_size=2)


def test_projected_workload_sampled_rows(swa):
    """The 32-frame, 1004-token, 16x64 workload (LayerNorm(x) @ W inputs,
    window 6, 8 scale frames) at full size, checked on sampled rows of every
    frame for several heads."""
    F, P = 32, 1004
    q, k, v = synth.projected_qkv(seed=0, F=F, P=P)
    got = _run(swa, q, k, v, F, P, 6, 8)
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[f * P + r for f in range(F) for r in (0, 127, 128, P - 1)],
                                     rng.integers(0, F * P, 64)]))
    heads = [0, 5, 15]
    ref = _ref(q, k, v, P, 8, 6, rows=rows, heads=heads)
    check_bf16(got[:, rows][:, :, heads], ref, "projected workload")
