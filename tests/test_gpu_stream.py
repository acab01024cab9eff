"""Streaming rolling paged cache on the GPU: bookkeeping bit-exact against the
oracle's host model, stored K/V bit-exact, attention outputs within tolerance."""
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


def _compare_meta(meta, oc, layer, i):
    assert meta["n_frames"] == i + 1
    assert meta["last_evicted"] == oc.layers[layer].last_evicted, i
    assert meta["n_evicted"] == oc.layers[layer].n_evicted
    assert meta["n_special"] == oc.n_special_tokens(layer)
    np.testing.assert_array_equal(meta["slot_frame"], oc.slot_frames(layer))
    np.testing.assert_array_equal(meta["page_table"], oc.page_table(layer))


def _stream(swa, F, P, H, D, S, Wc, special, dtype, frames_to_check, max_frames=None, layers=1,
            check_rows=None, num_special=5, check_heads=None):
    max_frames = max_frames or F
    dev = "cuda"
    cache = swa.SwaStream(num_layers=layers, heads=H, head_dim=D, P=P, scale_frames=S, window_frames=Wc,
                          cross_frame_special=special, num_special=num_special, max_frames=max_frames,
                          dtype=dtype)
    oc = orc.StreamCache(heads=H, head_dim=D, P=P, scale_frames=S, window_frames=Wc, page_tokens=16,
                         cross_frame_special=special, num_special=num_special, max_frames=max_frames,
                         num_layers=layers)
    for i in range(F):
        for layer in range(layers):
            q, k, v = synth.stream_frame(i, P=P, H=H, D=D, dtype=dtype, base_seed=layer)
            cache.swa_stream_append_evict(layer, i, k.to(dev), v.to(dev))
            oc.append_evict(layer, i, k.float().numpy(), v.float().numpy())
            _compare_meta(cache.swa_stream_get_meta(layer), oc, layer, i)
            if i in frames_to_check:
                out = torch.empty(q.shape, dtype=dtype, device=dev)
                cache.swa_stream_attend(layer, i, q.to(dev), out)
                torch.cuda.synchronize()
                got = out.float().cpu().numpy()
                if check_heads is not None:
                    # every query row of the listed heads
                    kc, vc = oc.gather(layer)
                    qq = q.float().numpy()
                    ref = np.stack([orc.softmax_attention(qq[:, h], kc[:, h], vc[:, h]) for h in check_heads], 1)
                    got = got[:, check_heads]
                elif check_rows is None:
                    ref = oc.attend(layer, q.float().numpy())
                else:
                    kc, vc = oc.gather(layer)
                    qq = q.float().numpy()[check_rows]
                    ref = np.stack([orc.softmax_attention(qq[:, h], kc[:, h], vc[:, h]) for h in range(H)], 1)
                    got = got[check_rows]
                if dtype == torch.float32:
                    check_f32(got, ref, f"frame {i}")
                else:
                    check_bf16(got, ref, f"frame {i}")
    assert swa.swa_device_error_check() == 0
    return cache, oc


def test_tiny_config_stream_equals_prefill(swa):
    """8 frames x 21 tokens, 2 x 32, f32: streaming through a 2+3-frame rolling
    cache matches the oracle's prefill with window 3 and 2 scale frames."""
    F, P, H, D = 8, 21, 2, 32
    q, k, v = synth.tiny_qkv(seed=0)
    full = orc.prefill(q.numpy(), k.numpy(), v.numpy(), P=P, scale_frames=2, sliding_window_size=3)[0]
    cache = swa.SwaStream(num_layers=1, heads=H, head_dim=D, P=P, scale_frames=2, window_frames=3,
                          max_frames=F, dtype=torch.float32)
    gpu_prefill = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    swa.swa_prefill(q.cuda(), k.cuda(), v.cuda(), gpu_prefill, S=F, P=P, sliding_window_size=3,
                    num_frame_for_scale=2)
    for i in range(F):
        sl = slice(i * P, (i + 1) * P)
        cache.swa_stream_append_evict(0, i, k[0, sl].contiguous().cuda(), v[0, sl].contiguous().cuda())
        out = torch.empty(P, H, D, device="cuda")
        cache.swa_stream_attend(0, i, q[0, sl].contiguous().cuda(), out)
        torch.cuda.synchronize()
        check_f32(out.cpu().numpy(), full[sl], f"stream frame {i}")
        check_f32(out.cpu().numpy(), gpu_prefill[0, sl].cpu().numpy(), f"stream vs prefill {i}")


@pytest.mark.parametrize("special", [False, True])
def test_bf16_small_stream(swa, special):
    _stream(swa, F=12, P=300, H=2, D=64, S=2, Wc=3, special=special, dtype=torch.bfloat16,
            frames_to_check=set(range(12)))


def test_two_layers_are_independent(swa):
    _stream(swa, F=7, P=130, H=2, D=64, S=1, Wc=2, special=True, dtype=torch.bfloat16,
            frames_to_check={0, 3, 6}, layers=2)


def test_stored_pages_bit_exact(swa):
    F, P, H, D, S, Wc = 9, 40, 2, 64, 2, 3
    cache, oc = _stream(swa, F=F, P=P, H=H, D=D, S=S, Wc=Wc, special=True, dtype=torch.bfloat16,
                        frames_to_check=set())
    kst = cache.storage(0, "k").cpu()
    ppf = -(-P // 16)
    for j in sorted(oc.layers[0].frames):
        s = oc.slot_of(j)
        _, k, _ = synth.stream_frame(j, P=P, H=H, D=D)
        assert torch.equal(kst[s * ppf * 16: s * ppf * 16 + P], k)
    for e, j in enumerate(oc.layers[0].special_from):
        _, k, _ = synth.stream_frame(j, P=P, H=H, D=D)
        for r in range(5):
            page, off = oc.special_location(e * 5 + r)
            assert torch.equal(kst[page * 16 + off], k[r])


def test_out_of_order_and_bounds(swa):
    cache = swa.SwaStream(num_layers=2, heads=2, head_dim=64, P=20, scale_frames=1, window_frames=2,
                          max_frames=4)
    q, k, v = synth.stream_frame(0, P=20, H=2, D=64)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    out = torch.empty_like(q)
    with pytest.raises(swa.SwaError) as e:
        cache.swa_stream_attend(0, 0, q, out)          # attend before append
    assert e.value.status == -3
    with pytest.raises(swa.SwaError) as e:
        cache.swa_stream_append_evict(0, 1, k, v)      # skips frame 0
    assert e.value.status == -3
    with pytest.raises(swa.SwaError) as e:
        cache.swa_stream_append_evict(2, 0, k, v)      # no such layer
    assert e.value.status == -4
    for i in range(4):
        cache.swa_stream_append_evict(0, i, k, v)
    with pytest.raises(swa.SwaError) as e:
        cache.swa_stream_append_evict(0, 4, k, v)      # beyond max_frames
    assert e.value.status == -4
    cache.swa_stream_reset()
    cache.swa_stream_append_evict(0, 0, k, v)
    assert cache.swa_stream_get_meta(0)["n_frames"] == 1


def test_300_frame_stream(swa):
    """8 scale + 64 window frames, 1004 tokens, 16 x 64, page 16, 300 frames:
    bookkeeping of every frame bit-exact; every query row of heads 0 and 9 at the
    first frame, the last scale frame, the first window frame, the frame that
    fills the cache, the first evictions, mid-stream and the last frame."""
    _stream(swa, F=300, P=1004, H=16, D=64, S=8, Wc=64, special=False, dtype=torch.bfloat16,
            frames_to_check={0, 7, 8, 71, 72, 73, 150, 299}, check_heads=[0, 9])


def test_1000_frame_stream_with_specials(swa):
    """Same cache, 1000 frames, evicted frames keep 5 special tokens each.  Every
    query row of heads 0 and 15 is checked where the special run changes shape:
    frame 72 (the first eviction, 5 specials), 73, 75 (20 specials: the run
    first spills onto a second 16-token page), 87 (80 specials: the run first
    ends exactly on a page boundary), 500 and 999 (4640 specials, 76,928 keys)."""
    _stream(swa, F=1000, P=1004, H=16, D=64, S=8, Wc=64, special=True, dtype=torch.bfloat16,
            frames_to_check={72, 73, 75, 87, 500, 999}, check_heads=[0, 15])


# ---------------------------------------------------------------- non-keyframe attend
def _raw_meta(cache, layer=0):
    m = cache.swa_stream_get_meta(layer)
    return {k: (v.tolist() if hasattr(v, "tolist") else v) for k, v in m.items()}


def _transient_stream(swa, F, P, H, D, S, Wc, special, dtype, at, check_rows=None, keyframes=None):
    """Keyframes 0..F-1; before each keyframe listed in ``at`` (F: after the
    last) a non-keyframe with its own seeded Q/K/V attends through the cache
    without persisting.  Its output matches the oracle, the metadata is
    bit-identical before and after it, and the keyframes listed in
    ``keyframes`` (default: all) still match the oracle.  With ``check_rows``
    the oracle is evaluated on those query rows only."""
    dev = "cuda"
    cache = swa.SwaStream(num_layers=1, heads=H, head_dim=D, P=P, scale_frames=S, window_frames=Wc,
                          cross_frame_special=special, num_special=5, max_frames=F, dtype=dtype)
    oc = orc.StreamCache(heads=H, head_dim=D, P=P, scale_frames=S, window_frames=Wc, page_tokens=16,
                         cross_frame_special=special, num_special=5, max_frames=F)
    check = check_f32 if dtype == torch.float32 else check_bf16
    rows = np.arange(P) if check_rows is None else np.asarray(check_rows)

    def ref_rows(q, extra=None):
        # oracle attention of the sampled query rows against the cache (+ extra K/V)
        if oc.layers[0].frames or oc.layers[0].specials_k:
            kc, vc = oc.gather(0)
            if extra is not None:
                kc, vc = np.concatenate([kc, extra[0]]), np.concatenate([vc, extra[1]])
        else:
            kc, vc = extra
        qq = q[rows]
        return np.stack([orc.softmax_attention(qq[:, h], kc[:, h], vc[:, h]) for h in range(H)], 1)

    for i in range(F + 1):
        if i in at:
            tq, tk, tv = synth.stream_frame(10_000 + i, P=P, H=H, D=D, dtype=dtype, base_seed=7)
            before = _raw_meta(cache) if i > 0 else None
            out = torch.empty(tq.shape, dtype=dtype, device=dev)
            cache.swa_stream_attend_transient(0, tq.to(dev), tk.to(dev), tv.to(dev), out)
            torch.cuda.synchronize()
            got = out.float().cpu().numpy()[rows]
            if check_rows is None:
                ref = oc.attend_transient(0, tq.float().numpy(), tk.float().numpy(), tv.float().numpy())
            else:
                ref = ref_rows(tq.float().numpy(), (tk.float().numpy(), tv.float().numpy()))
            check(got, ref, f"non-keyframe before keyframe {i}")
            if before is not None:
                assert _raw_meta(cache) == before
        if i == F:
            break
        q, k, v = synth.stream_frame(i, P=P, H=H, D=D, dtype=dtype)
        cache.swa_stream_append_evict(0, i, k.to(dev), v.to(dev))
        oc.append_evict(0, i, k.float().numpy(), v.float().numpy())
        _compare_meta(cache.swa_stream_get_meta(0), oc, 0, i)
        if keyframes is not None and i not in keyframes:
            continue
        out = torch.empty(q.shape, dtype=dtype, device=dev)
        cache.swa_stream_attend(0, i, q.to(dev), out)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()[rows]
        ref = oc.attend(0, q.float().numpy()) if check_rows is None else ref_rows(q.float().numpy())
        check(got, ref, f"keyframe {i}")
    assert swa.swa_device_error_check() == 0


@pytest.mark.parametrize("special", [False, True])
def test_transient_attend_bf16(swa, special):
    """2 scale + 3 window frames of 200 tokens (two query tiles), 2 x 64: the
    non-keyframe on an empty cache, while the window fills, once it is full
    (the frame a keyframe would evict is still visible), and late in the stream."""
    _transient_stream(swa, F=10, P=200, H=2, D=64, S=2, Wc=3, special=special, dtype=torch.bfloat16,
                      at={0, 1, 4, 5, 6, 9, 10})


def test_transient_attend_head_dim_128_and_f32(swa):
    _transient_stream(swa, F=7, P=130, H=2, D=128, S=1, Wc=2, special=True, dtype=torch.bfloat16,
                      at={0, 3, 5, 7})
    _transient_stream(swa, F=6, P=21, H=2, D=32, S=1, Wc=2, special=True, dtype=torch.float32,
                      at={0, 2, 4, 6})


def test_transient_attend_full_size(swa):
    """8 scale + 64 window frames of 1004 tokens, 16 x 64: a non-keyframe after
    80 keyframes (73 frames of keys), checked on sampled rows."""
    rows = np.unique(np.concatenate([np.arange(0, 1004, 61), [127, 128, 1003]]))
    _transient_stream(swa, F=80, P=1004, H=16, D=64, S=8, Wc=64, special=False, dtype=torch.bfloat16,
                      at={79, 80}, check_rows=rows, keyframes={79})


def test_more_key_runs_than_the_shared_prefix_holds(swa):
    """No window (every frame retained) over 1030 frames of 16 tokens, 2 x 64:
    from frame 1023 on the attend sees 1024 or more key runs, more than a CTA
    keeps the tile prefix of in shared memory, so it walks the runs in the device
    metadata instead; each pair has a single query tile, and the frame's keys are
    cut into as many splits as the handle allows.  Bookkeeping bit-exact on every
    frame; attention against the oracle at frame 0, at frame 1022 (the last whose
    runs fit the prefix), 1023 and 1029."""
    _stream(swa, F=1030, P=16, H=2, D=64, S=0, Wc=0, special=False, dtype=torch.bfloat16,
            frames_to_check={0, 1022, 1023, 1029})


def test_camera_only_retention(swa):
    """Evicted frames keep only their camera token (num_special = 1, the reading
    taken for kv_cache_camera_only): bookkeeping bit-exact, attention matches."""
    _stream(swa, F=12, P=300, H=2, D=64, S=2, Wc=3, special=True, dtype=torch.bfloat16,
            frames_to_check=set(range(12)), num_special=1)


def test_no_scale_frames(swa):
    """No protected scale frames (scale_frames = 0, the reading taken for
    kv_cache_include_scale_frames=False): a pure window of frames."""
    _stream(swa, F=10, P=300, H=2, D=64, S=0, Wc=3, special=False, dtype=torch.bfloat16,
            frames_to_check=set(range(10)))
    _stream(swa, F=10, P=300, H=2, D=64, S=0, Wc=3, special=True, dtype=torch.bfloat16,
            frames_to_check={3, 6, 9})


def test_split_attend_equals_one_split_over_a_long_stream(swa):
    """Full size (8 scale + 64 window frames of 1004 tokens, 16 x 64), 30
    keyframe attends in steady state and two non-keyframes, each through a cache
    whose attend is split into pieces (partials merged by the CTA that finishes
    an item last) and through one that runs every item whole: every (query row,
    head) agrees within bf16 rounding, so no piece's partial is lost, merged
    twice or read before it was written (a block of 32 rows from one softmax warp
    is the failure this looks for)."""
    P, H, D, S, Wc = 1004, 16, 64, 8, 64
    kw = dict(num_layers=1, heads=H, head_dim=D, P=P, scale_frames=S, window_frames=Wc, max_frames=120,
              dtype=torch.bfloat16)
    split, whole = swa.SwaStream(max_splits=12, **kw), swa.SwaStream(max_splits=1, **kw)
    frames = [tuple(t.cuda() for t in synth.stream_frame(i, P=P, H=H, D=D)) for i in range(8)]
    extra = tuple(t.cuda() for t in synth.stream_frame(5_000, P=P, H=H, D=D, base_seed=3))

    def agree(a, b, what):
        a, b = a.float(), b.float()
        assert torch.isfinite(a).all(), what
        num = (a - b).norm(dim=2)
        den = b.norm(dim=2).clamp_min(1e-6)
        worst = float((num / den).max())
        assert worst <= 2e-2, f"{what}: worst (row, head) relative error {worst:.3e}"

    for i in range(100):
        q, k, v = frames[i % 8]
        if i in (80, 95):
            oa = torch.full((P, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
            ob = torch.full_like(oa, float("nan"))
            split.swa_stream_attend_transient(0, *extra, oa)
            whole.swa_stream_attend_transient(0, *extra, ob)
            agree(oa, ob, f"non-keyframe before keyframe {i}")
        split.swa_stream_append_evict(0, i, k, v)
        whole.swa_stream_append_evict(0, i, k, v)
        if i >= 70:
            oa = torch.full((P, H, D), float("nan"), dtype=torch.bfloat16, device="cuda")
            ob = torch.full_like(oa, float("nan"))
            split.swa_stream_attend(0, i, q, oa)
            whole.swa_stream_attend(0, i, q, ob)
            agree(oa, ob, f"keyframe {i}")
    assert swa.swa_device_error_check() == 0
