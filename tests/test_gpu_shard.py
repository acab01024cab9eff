"""Head sharding on one GPU: the head-sliced prefill / append / attend run one
shard after another, each writing its heads of the shared output in place, and
together equal the unsliced call (bit for bit where the two launch the same
kernels on the same work) and the float64 oracle."""
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


@pytest.mark.parametrize("F,P,H,D,world,dtype", [
    (6, 1004, 16, 64, 2, torch.bfloat16),
    (4, 300, 8, 128, 4, torch.bfloat16),
    (5, 60, 4, 32, 2, torch.float32),
])
def test_prefill_head_shards_equal_the_whole(swa, F, P, H, D, world, dtype):
    q, k, v = (t.cuda() for t in synth.tiny_qkv(seed=17 + H, F=F, P=P, H=H, D=D, dtype=dtype))
    whole = torch.empty_like(q)
    swa.swa_prefill(q, k, v, whole, S=F, P=P, sliding_window_size=2, num_frame_for_scale=1)
    out = torch.full_like(q, float("nan"))
    for r in range(world):
        h0, hr = swa.head_shard(r, world, H)
        swa.swa_prefill_heads(q, k, v, out, S=F, P=P, head0=h0, heads=hr, sliding_window_size=2,
                              num_frame_for_scale=1)
    torch.cuda.synchronize()
    assert swa.swa_device_error_check() == 0
    assert torch.equal(out, whole)
    rows = np.arange(0, F * P, 7)
    ref = orc.prefill(q.float().cpu().numpy(), k.float().cpu().numpy(), v.float().cpu().numpy(), P=P,
                      scale_frames=1, sliding_window_size=2, rows=rows)
    (check_bf16 if dtype == torch.bfloat16 else check_f32)(out.float().cpu().numpy()[:, rows], ref, "sharded")


@pytest.mark.parametrize("max_splits", [1, 12])
def test_stream_head_shards(swa, max_splits):
    """Two caches of 8 heads each serve a 16-head stream (8 scale + 4 window
    frames, 20 frames of 1004 tokens): with one split both shards run exactly
    the unsliced kernels' per-head work (bit-exact); with split-KV the split
    count follows each launch's own size, so the shards are checked against
    the oracle within the bf16 tolerance."""
    P, H, D, S, Wc, F, world = 1004, 16, 64, 2, 4, 12, 2
    kw = dict(num_layers=1, head_dim=D, P=P, scale_frames=S, window_frames=Wc, max_frames=F,
              dtype=torch.bfloat16, max_splits=max_splits)
    whole = swa.SwaStream(heads=H, **kw)
    shards = [swa.SwaStream(heads=swa.head_shard(r, world, H)[1], **kw) for r in range(world)]
    oc = orc.StreamCache(heads=H, head_dim=D, P=P, scale_frames=S, window_frames=Wc, page_tokens=16)
    for i in range(F):
        fq, fk, fv = synth.stream_frame(i, P=P, H=H, D=D)
        q, k, v = fq.cuda(), fk.cuda(), fv.cuda()
        ref_out = torch.empty_like(q)
        whole.swa_stream_append_evict(0, i, k, v)
        whole.swa_stream_attend(0, i, q, ref_out)
        out = torch.full_like(q, float("nan"))
        for r, c in enumerate(shards):
            h0, _ = swa.head_shard(r, world, H)
            c.swa_stream_append_evict_heads(0, i, k, v, head0=h0)
            c.swa_stream_attend_heads(0, i, q, out, head0=h0)
        torch.cuda.synchronize()
        oc.append_evict(0, i, fk.float().numpy(), fv.float().numpy())
        if max_splits == 1:
            assert torch.equal(out, ref_out), i
        if i in (0, 5, F - 1):
            rows = np.arange(0, P, 13)
            want = oc.attend(0, fq.float().numpy())[rows]
            check_bf16(out.float().cpu().numpy()[rows], want, f"sharded stream frame {i}")
        for c in shards:
            m = c.swa_stream_get_meta(0)
            assert m["n_frames"] == i + 1 and m["n_evicted"] == whole.swa_stream_get_meta(0)["n_evicted"]
    assert swa.swa_device_error_check() == 0

