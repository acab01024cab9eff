"""Pins for the float64 oracle: each check ties it to something other than itself.

The pages print no worked numeric example, so the pins are hand-worked
visible sets and cache bookkeeping (tests/golden/), the pages' own mask
snippet, closed forms, library special cases (torch SDPA in float64 on CPU),
brute-force enumeration on tiny inputs, the stream == prefill identity and
receptive-field reachability.
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _parse_visible_sets():
    cases = []
    with open(os.path.join(GOLDEN, "visible_sets.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, body = line.split("|")
            F, S, sws, nfpb = (int(x) for x in head.split())
            sets = {}
            for item in body.split(";"):
                i, js = item.strip().split(":")
                sets[int(i)] = sorted(int(j) for j in js.split(","))
            cases.append((F, S, sws, nfpb, sets))
    return cases


VISIBLE_CASES = _parse_visible_sets()


# --------------------------------------------------------------------- masks
@pytest.mark.parametrize("case", VISIBLE_CASES, ids=lambda c: f"F{c[0]}S{c[1]}w{c[2]}b{c[3]}")
def test_visible_sets_match_hand_worked(case):
    F, S, sws, nfpb, sets = case
    for i in range(F):
        got = [j for j in range(F) if orc.frame_visible(i, j, S, sws, nfpb)]
        assert got == sets[i], (i, got, sets[i])


@pytest.mark.parametrize("case", VISIBLE_CASES, ids=lambda c: f"F{c[0]}S{c[1]}w{c[2]}b{c[3]}")
def test_token_mask_expands_frames(case):
    F, S, sws, nfpb, sets = case
    P = 3
    m = orc.frame_mask(F, P, S, sws, nfpb)
    for t in range(F * P):
        expect = np.zeros(F * P, dtype=bool)
        for j in sets[t // P]:
            expect[j * P:(j + 1) * P] = True
        assert np.array_equal(m[t], expect)


def _page_snippet_mask_rows(num_frames, frame_seqlen, num_frame_per_block, sliding_window_size, rows):
    """The window mask as the AggregatorStream guide's "Manual Sliding-Window
    Mask Construction" example builds it: per query frame, a slice from the
    window start frame to the end of the current frame is set True.  Restated
    here for the selected rows only."""
    N = num_frames * frame_seqlen
    out = np.zeros((len(rows), N), dtype=bool)
    win = sliding_window_size * num_frame_per_block
    for r_i, t in enumerate(rows):
        i = t // frame_seqlen
        lo = max(0, i - win + 1) * frame_seqlen
        hi = (i + 1) * frame_seqlen
        out[r_i, lo:hi] = True
    return out


@pytest.mark.parametrize("F,P,nfpb,sws", [(10, 1560, 1, 4), (7, 5, 1, 3), (9, 4, 2, 2), (6, 3, 1, 1)])
def test_window_part_equals_page_snippet(F, P, nfpb, sws):
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, P - 1, P, F * P - 1], rng.integers(0, F * P, 40)]))
    ref = _page_snippet_mask_rows(F, P, nfpb, sws, rows)
    got = orc.frame_mask(F, P, 0, sws, nfpb, rows)
    assert np.array_equal(got, ref)


def test_minus_one_and_wide_window_are_full_causal():
    F, P = 6, 4
    causal = np.zeros((F * P, F * P), dtype=bool)
    for t in range(F * P):
        causal[t, : (t // P + 1) * P] = True
    for sws in (-1, 0, F, F + 3):
        assert np.array_equal(orc.frame_mask(F, P, 0, sws, 1), causal)
        assert np.array_equal(orc.frame_mask(F, P, 2, sws, 1), causal)


# ------------------------------------------------------------ attention values
def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_single_frame_is_textbook_attention():
    q, k, v = (_rand((1, 9, 2, 8), s) for s in (1, 2, 3))
    got = orc.prefill(q, k, v, P=9, scale_frames=0, sliding_window_size=3)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(got, ref, atol=1e-13, rtol=0)


def test_window_one_is_per_frame_attention():
    F, P, H, D = 4, 5, 2, 6
    q, k, v = (_rand((1, F * P, H, D), s) for s in (4, 5, 6))
    got = orc.prefill(q, k, v, P=P, scale_frames=0, sliding_window_size=1)
    for f in range(F):
        sl = slice(f * P, (f + 1) * P)
        tq, tk, tv = (torch.from_numpy(x[:, sl]).permute(0, 2, 1, 3) for x in (q, k, v))
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3).numpy()
        np.testing.assert_allclose(got[:, sl], ref, atol=1e-13, rtol=0)


def test_full_causal_matches_sdpa_with_frame_block_mask():
    F, P, H, D = 5, 3, 2, 4
    q, k, v = (_rand((1, F * P, H, D), s) for s in (7, 8, 9))
    got = orc.prefill(q, k, v, P=P, scale_frames=0, sliding_window_size=-1)
    blk = torch.zeros(F * P, F * P, dtype=torch.bool)
    for t in range(F * P):
        blk[t, : (t // P + 1) * P] = True
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=blk)
    np.testing.assert_allclose(got, ref.permute(0, 2, 1, 3).numpy(), atol=1e-13, rtol=0)


def test_constant_values_pass_through():
    F, P, H, D = 6, 4, 2, 5
    q, k = _rand((1, F * P, H, D), 10), _rand((1, F * P, H, D), 11)
    c = _rand((H, D), 12)
    v = np.broadcast_to(c, (1, F * P, H, D)).copy()
    got = orc.prefill(q, k, v, P=P, scale_frames=2, sliding_window_size=2)
    np.testing.assert_allclose(got, v, atol=1e-14, rtol=0)


@pytest.mark.parametrize("case", VISIBLE_CASES, ids=lambda c: f"F{c[0]}S{c[1]}w{c[2]}b{c[3]}")
def test_zero_queries_give_visible_token_fractions(case):
    """Q = 0 makes the softmax uniform over the visible keys; with V one-hot in
    the key's frame, output column f equals (#visible tokens of f)/(#visible)."""
    F, S, sws, nfpb, sets = case
    P = 3
    q = np.zeros((1, F * P, 1, 4))
    k = _rand((1, F * P, 1, 4), 13)
    v = np.zeros((1, F * P, 1, F))
    for t in range(F * P):
        v[0, t, 0, t // P] = 1.0
    got = orc.prefill(q, k, v, P=P, scale_frames=S, sliding_window_size=sws, num_frame_per_block=nfpb)
    for t in range(F * P):
        vis = sets[t // P]
        expect = np.zeros(F)
        expect[vis] = 1.0 / len(vis)
        np.testing.assert_allclose(got[0, t, 0], expect, atol=1e-15, rtol=0)


def test_softmax_scale_is_inverse_sqrt_head_dim():
    q, k, v = (_rand((5, 16), s) for s in (14, 15, 16))
    got = orc.softmax_attention(q, k, v)
    z = q @ k.T / 4.0
    e = np.exp(z - z.max(1, keepdims=True))
    np.testing.assert_allclose(got, (e / e.sum(1, keepdims=True)) @ v, atol=1e-14)
    with pytest.raises(AssertionError):
        np.testing.assert_allclose(orc.softmax_attention(q, k, v, scale=1.0), got, atol=1e-6)


# ---------------------------------------------------------------- streaming
def _parse_bookkeeping():
    rows = []
    with open(os.path.join(GOLDEN, "stream_bookkeeping.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            parts = [p.strip() for p in line.split("|")]
            rows.append(dict(frame=int(parts[0]), evicted=int(parts[1]),
                             slots=[int(x) for x in parts[2].split()],
                             pages=[int(x) for x in parts[3].split()],
                             n_special=int(parts[4])))
    return rows


def test_bookkeeping_matches_hand_worked():
    cache = orc.StreamCache(heads=1, head_dim=2, P=21, scale_frames=2, window_frames=3,
                            page_tokens=16, cross_frame_special=True, num_special=5)
    for row in _parse_bookkeeping():
        k = _rand((21, 1, 2), row["frame"])
        ev = cache.append_evict(0, row["frame"], k, k)
        assert ev == ([] if row["evicted"] < 0 else [row["evicted"]])
        assert cache.layers[0].last_evicted == row["evicted"]
        assert cache.slot_frames(0).tolist() == row["slots"]
        assert cache.page_table(0).tolist() == row["pages"]
        assert cache.n_special_tokens(0) == row["n_special"]


@pytest.mark.parametrize("S,W,F", [(2, 3, 8), (8, 64, 300), (0, 1, 5), (8, 6, 32), (3, 5, 40)])
def test_slots_collision_free_and_window_equals_mask(S, W, F):
    cache = orc.StreamCache(heads=1, head_dim=1, P=1, scale_frames=S, window_frames=W)
    slot_of = {}
    for i in range(F):
        ev = cache.append_evict(0, i, np.zeros((1, 1, 1)), np.zeros((1, 1, 1)))
        if i >= S + W:
            assert ev == [i - W]
            assert cache.slot_of(i) == slot_of[i - W]
        else:
            assert ev == []
        slot_of[i] = cache.slot_of(i)
        retained = sorted(cache.layers[0].frames)
        assert retained == [j for j in range(i + 1) if orc.frame_visible(i, j, S, W, 1)]
        slots = [slot_of[j] for j in retained]
        assert len(set(slots)) == len(slots) and max(slots) < S + W


def _tiny_stream(S, W, F, P, H, D, special, ns, seed):
    q, k, v = (_rand((F * P, H, D), seed + s) for s in range(3))
    cache = orc.StreamCache(heads=H, head_dim=D, P=P, scale_frames=S, window_frames=W,
                            page_tokens=4, cross_frame_special=special, num_special=ns)
    outs = []
    for i in range(F):
        sl = slice(i * P, (i + 1) * P)
        cache.append_evict(0, i, k[sl], v[sl])
        outs.append(cache.attend(0, q[sl]))
    return q, k, v, np.concatenate(outs, axis=0)


@pytest.mark.parametrize("S", [2, 0])
def test_stream_equals_prefill_tiny_config(S):
    """The 8-frame, 21-token, 2x32 check case: frame-by-frame streaming through
    the rolling cache reproduces the full-sequence masked attention.  S = 0 is
    the cache without protected scale frames (the reading taken for
    kv_cache_include_scale_frames=False): a pure frame window."""
    W, F, P, H, D = 3, 8, 21, 2, 32
    q, k, v, streamed = _tiny_stream(S, W, F, P, H, D, False, 5, 100)
    full = orc.prefill(q[None], k[None], v[None], P=P, scale_frames=S, sliding_window_size=W)[0]
    np.testing.assert_allclose(streamed, full, atol=1e-12, rtol=0)


@pytest.mark.parametrize("ns", [2, 1])
def test_special_retention_equals_extended_mask(ns):
    """Evicted frames keep their first ns tokens.  ns = 1 keeps the camera token
    only (the reading taken for kv_cache_camera_only)."""
    S, W, F, P, H, D = 1, 2, 7, 7, 2, 4
    q, k, v, streamed = _tiny_stream(S, W, F, P, H, D, True, ns, 200)
    N = F * P
    for i in range(F):
        mask = np.zeros((P, N), dtype=bool)
        for j in range(i + 1):
            if j < S or j >= i - W + 1:
                mask[:, j * P:(j + 1) * P] = True
            else:  # evicted frame: its first ns tokens stay
                mask[:, j * P:j * P + ns] = True
        for h in range(H):
            ref = orc.softmax_attention(q[i * P:(i + 1) * P, h], k[:, h], v[:, h], mask)
            np.testing.assert_allclose(streamed[i * P:(i + 1) * P, h], ref, atol=1e-12, rtol=0)


def test_key_order_does_not_matter():
    q, k, v = (_rand((6, 8), s) for s in (20, 21, 22))
    perm = np.random.default_rng(3).permutation(6)
    np.testing.assert_allclose(orc.softmax_attention(q, k, v), orc.softmax_attention(q, k[perm], v[perm]),
                               atol=1e-12)


def test_streaming_rejects_out_of_order():
    cache = orc.StreamCache(heads=1, head_dim=1, P=1, scale_frames=0, window_frames=2)
    cache.append_evict(0, 0, np.zeros((1, 1, 1)), np.zeros((1, 1, 1)))
    with pytest.raises(ValueError):
        cache.append_evict(0, 2, np.zeros((1, 1, 1)), np.zeros((1, 1, 1)))


def test_special_locations():
    cache = orc.StreamCache(heads=1, head_dim=1, P=1004, scale_frames=8, window_frames=64,
                            page_tokens=16, cross_frame_special=True, num_special=5)
    assert cache.ppf == 63
    assert cache.special_location(0) == (72 * 63, 0)
    assert cache.special_location(16) == (72 * 63 + 1, 0)
    assert cache.special_location(4639) == (72 * 63 + 289, 15)


# ----------------------------------------------------- token band and decode
def test_rolling_buffer_six_slot_toy():
    # the explainer's widget: tokens written at slot i mod 6, never more than 6 slots
    slots = [orc.decode_slot(i, 6) for i in range(12)]
    assert slots == [0, 1, 2, 3, 4, 5, 0, 1, 2, 3, 4, 5]
    assert orc.decode_slot(200000, 4096) == 3392


def test_band_wide_window_is_causal_sdpa():
    q, k, v = (_rand((1, 11, 2, 8), s) for s in (30, 31, 32))
    got = orc.band_attention(q, k, v, W=64)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    np.testing.assert_allclose(got, ref.permute(0, 2, 1, 3).numpy(), atol=1e-13, rtol=0)


def test_band_window_one_returns_values():
    q, k, v = _rand((1, 9, 4, 8), 33), _rand((1, 9, 2, 8), 34), _rand((1, 9, 2, 8), 35)
    got = orc.band_attention(q, k, v, W=1)
    np.testing.assert_allclose(got, np.repeat(v, 2, axis=2), atol=1e-15, rtol=0)


def test_band_gqa_matches_sdpa_enable_gqa():
    N, W = 20, 6
    q, k, v = _rand((1, N, 8, 8), 36), _rand((1, N, 2, 8), 37), _rand((1, N, 2, 8), 38)
    got = orc.band_attention(q, k, v, W=W)
    tq, tk, tv = (torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v))
    band = torch.from_numpy(orc.band_mask(N, W))
    t = torch.arange(N)
    assert torch.equal(band, (t[None] <= t[:, None]) & (t[None] > t[:, None] - W))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=band, enable_gqa=True)
    np.testing.assert_allclose(got, ref.permute(0, 2, 1, 3).numpy(), atol=1e-13, rtol=0)


@pytest.mark.parametrize("pos", [3, 7, 8, 29])
def test_decode_equals_band_row(pos):
    """Writing positions 0..pos into a W-slot rolling buffer (slot p mod W) and
    attending over it equals band attention at row pos of the full sequence."""
    W, B, Hq, Hkv, D = 8, 2, 4, 2, 8
    n = pos + 1
    q = _rand((B, n, Hq, D), 40)
    k = _rand((B, n, Hkv, D), 41)
    v = _rand((B, n, Hkv, D), 42)
    kc = np.full((B, W, Hkv, D), np.nan)
    vc = np.full((B, W, Hkv, D), np.nan)
    for p in range(pos):
        kc[:, p % W] = k[:, p]
        vc[:, p % W] = v[:, p]
    kc = np.nan_to_num(kc)
    vc = np.nan_to_num(vc)
    out, kc2, _ = orc.decode(q[:, pos], k[:, pos], v[:, pos], kc, vc, pos, W)
    ref = orc.band_attention(q, k, v, W=W, rows=[pos])[:, 0]
    np.testing.assert_allclose(out, ref, atol=1e-13, rtol=0)
    np.testing.assert_array_equal(kc2[:, pos % W], k[:, pos])


# -------------------------------------------------------------- reachability
def _stack_band(x, ws, W):
    for wq, wk, wv in ws:
        q, k, v = (x @ w for w in (wq, wk, wv))
        x = x + orc.band_attention(q[None, :, None], k[None, :, None], v[None, :, None], W)[0, :, 0]
    return x


@pytest.mark.parametrize("L,W", [(1, 4), (2, 4), (3, 3)])
def test_band_receptive_field_is_L_times_W_minus_1(L, W):
    """Stacking L band layers: output i depends on input j iff 0 <= i-j <= L(W-1).
    The explainer rounds this reach to L*W (32 layers x 4096 ~ 131k tokens)."""
    N, C = 16, 6
    rng = np.random.default_rng(50)
    ws = [tuple(rng.standard_normal((C, C)) * 0.5 for _ in range(3)) for _ in range(L)]
    x = rng.standard_normal((N, C))
    base = _stack_band(x, ws, W)
    reach = L * (W - 1)
    for j in range(N):
        xp = x.copy()
        xp[j] += 1.0
        out = _stack_band(xp, ws, W)
        for i in range(N):
            changed = not np.array_equal(out[i], base[i])
            assert changed == (0 <= i - j <= reach), (i, j)
    assert 32 * 4096 == 131072


def _stack_frames(x, ws, P, S, Wf):
    for wq, wk, wv in ws:
        q, k, v = (x @ w for w in (wq, wk, wv))
        x = x + orc.prefill(q[None, :, None], k[None, :, None], v[None, :, None], P=P,
                            scale_frames=S, sliding_window_size=Wf)[0, :, 0]
    return x


def test_frame_receptive_field_with_scale_frames():
    """Frames: reach L(Wf-1) frames back, and the scale frames reach every later frame."""
    L, Wf, S, F, P, C = 2, 2, 1, 7, 2, 4
    rng = np.random.default_rng(51)
    ws = [tuple(rng.standard_normal((C, C)) * 0.5 for _ in range(3)) for _ in range(L)]
    x = rng.standard_normal((F * P, C))
    base = _stack_frames(x, ws, P, S, Wf)
    for jf in range(F):
        xp = x.copy()
        xp[jf * P] += 1.0
        out = _stack_frames(xp, ws, P, S, Wf)
        for i in range(F * P):
            fi = i // P
            reachable = fi >= jf and (jf < S or fi - jf <= L * (Wf - 1))
            assert (not np.array_equal(out[i], base[i])) == reachable, (i, jf)


# ---------------------------------------------------------------- non-keyframe attend
def _frame(P, H, D, seed):
    g = np.random.default_rng(seed)
    return tuple(g.standard_normal((P, H, D)) for _ in range(3))


def _state(cache, layer=0):
    st = cache.layers[layer]
    return (list(st.cached), sorted(st.frames), st.n_frames, st.n_evicted, st.last_evicted,
            len(st.specials_k), cache.slot_frames(layer).tolist(), cache.page_table(layer).tolist())


@pytest.mark.parametrize("special", [False, True])
def test_transient_attend_equals_append_then_attend_before_any_eviction(special):
    """While no eviction is due (fewer than S + W_c frames cached), appending a
    frame and attending is exactly attending to the cache plus the frame."""
    import copy
    S, W, P, H, D = 2, 3, 7, 2, 4
    cache = orc.StreamCache(H, D, P, S, W, page_tokens=4, cross_frame_special=special, num_special=2,
                            max_frames=20)
    for i in range(S + W):
        q, k, v = _frame(P, H, D, 100 + i)
        twin = copy.deepcopy(cache)
        twin.append_evict(0, i, k, v)
        assert twin.layers[0].last_evicted == -1
        np.testing.assert_allclose(cache.attend_transient(0, q, k, v), twin.attend(0, q), atol=1e-12, rtol=0)
        cache.append_evict(0, i, k, v)


@pytest.mark.parametrize("special", [False, True])
def test_transient_attend_leaves_cache_unchanged(special):
    S, W, P, H, D = 1, 2, 6, 2, 4
    cache = orc.StreamCache(H, D, P, S, W, page_tokens=4, cross_frame_special=special, num_special=2,
                            max_frames=30)
    for i in range(9):
        q, k, v = _frame(P, H, D, 200 + i)
        before = _state(cache)
        cache.attend_transient(0, q, k, v)
        assert _state(cache) == before
        cache.append_evict(0, i, k, v)


def test_transient_attend_sees_the_frame_a_keyframe_would_evict():
    """Q = 0 gives uniform weights; V = one-hot of the key's frame id makes each
    output column the fraction of keys from that frame.  A non-keyframe after
    frame i sees scale frames, the window [i - W_c + 1, i] (eviction deferred:
    frame i - W_c + 1 stays) and itself; the keyframe i + 1 sees one frame
    fewer (i + 1 - W_c is evicted)."""
    S, W, P, H = 1, 3, 5, 1
    F = 8
    D = F + 1  # one-hot over frame ids 0..F (id F: the non-keyframe)
    cache = orc.StreamCache(H, D, P, S, W, page_tokens=4, max_frames=20)
    z = np.zeros((P, H, D))
    for i in range(F):
        v = np.zeros((P, H, D))
        v[:, :, i] = 1.0
        cache.append_evict(0, i, z, v)
    i = F - 1
    vt = np.zeros((P, H, D))
    vt[:, :, F] = 1.0
    got = cache.attend_transient(0, z, z, vt)[0, 0]
    frames = list(range(S)) + list(range(i - W + 1, i + 1)) + [F]
    want = np.zeros(D)
    want[frames] = 1.0 / len(frames)
    np.testing.assert_allclose(got, want, atol=1e-15, rtol=0)
    assert 1.0 / len(frames) == pytest.approx(1.0 / (S + W + 1))


# ---------------------------------------------------------------- attn_pre prologue
def _prologue_inputs(P=6, H=2, D=8, seed=5):
    g = np.random.default_rng(seed)
    C = H * D
    x = g.standard_normal((P, C)) * 3 + 1
    w = dict(ln_w=1 + 0.1 * g.standard_normal(C), ln_b=0.1 * g.standard_normal(C),
             w_qkv=g.standard_normal((3 * C, C)) / np.sqrt(C), b_qkv=0.1 * g.standard_normal(3 * C),
             qn_w=1 + 0.1 * g.standard_normal(D), qn_b=0.1 * g.standard_normal(D),
             kn_w=1 + 0.1 * g.standard_normal(D), kn_b=0.1 * g.standard_normal(D))
    ang = g.uniform(-np.pi, np.pi, (P, D // 2))
    rot = np.stack([np.cos(ang), np.sin(ang)], axis=-1)
    return x, w, rot, ang


def test_layer_norm_matches_torch_and_row_statistics():
    x, w, _, _ = _prologue_inputs()
    eps = 1e-6
    got = orc.layer_norm(x, w["ln_w"], w["ln_b"], eps)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x), (x.shape[1],), torch.from_numpy(w["ln_w"]),
                                         torch.from_numpy(w["ln_b"]), eps).numpy()
    np.testing.assert_allclose(got, ref, atol=1e-12, rtol=0)
    plain = orc.layer_norm(x, np.ones(x.shape[1]), np.zeros(x.shape[1]), eps)
    var = x.var(axis=1)
    np.testing.assert_allclose(plain.mean(axis=1), 0, atol=1e-13)
    np.testing.assert_allclose((plain ** 2).mean(axis=1), var / (var + eps), rtol=1e-12)


def test_rope_complex_matches_torch_complex_product():
    g = np.random.default_rng(8)
    P, H, D = 5, 3, 8
    x = g.standard_normal((P, H, D))
    ang = g.uniform(-3, 3, (P, D // 2))
    rot = np.stack([np.cos(ang), np.sin(ang)], axis=-1)
    xt = torch.view_as_complex(torch.from_numpy(x).reshape(P, H, D // 2, 2).contiguous())
    ref = torch.view_as_real(xt * torch.polar(torch.ones(P, 1, D // 2, dtype=torch.float64),
                                              torch.from_numpy(ang)[:, None, :])).reshape(P, H, D).numpy()
    np.testing.assert_allclose(orc.rope_complex(x, rot), ref, atol=1e-12, rtol=0)


def test_rope_identity_norms_and_relative_positions():
    g = np.random.default_rng(9)
    P, H, D = 7, 2, 8
    x = g.standard_normal((P, H, D))
    ident = np.stack([np.ones((P, D // 2)), np.zeros((P, D // 2))], axis=-1)
    np.testing.assert_array_equal(orc.rope_complex(x, ident), x)
    # a frequency per pair, position p -> angle p * omega: rotated q_m . k_n depends on n - m only
    omega = 10.0 ** (-np.arange(D // 2) / (D // 2))
    def table(pos):
        a = np.outer(pos, omega)
        return np.stack([np.cos(a), np.sin(a)], axis=-1)
    q, k = g.standard_normal((1, H, D)), g.standard_normal((1, H, D))
    def dot(m, n):
        return np.sum(orc.rope_complex(q, table([m])) * orc.rope_complex(k, table([n])))
    for m, n, t in [(0, 3, 5), (2, -4, 11), (7, 7, -3)]:
        assert dot(m, n) == pytest.approx(dot(m + t, n + t), abs=1e-12)
    r = orc.rope_complex(x, table(np.arange(P)))
    np.testing.assert_allclose(np.linalg.norm(r, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-12)


def test_attn_pre_matches_torch_restatement():
    x, w, rot, ang = _prologue_inputs()
    P, C = x.shape
    H, D = 2, C // 2
    eps = 1e-6
    q, k, v = orc.attn_pre(x, w["ln_w"], w["ln_b"], w["w_qkv"], w["b_qkv"], w["qn_w"], w["qn_b"],
                           w["kn_w"], w["kn_b"], rot, heads=H, eps=eps)
    T = {n: torch.from_numpy(a) for n, a in w.items()}
    F = torch.nn.functional
    xn = F.layer_norm(torch.from_numpy(x), (C,), T["ln_w"], T["ln_b"], eps)
    qkv = F.linear(xn, T["w_qkv"], T["b_qkv"]).reshape(P, 3, H, D)
    tq = F.layer_norm(qkv[:, 0], (D,), T["qn_w"], T["qn_b"], eps)
    tk = F.layer_norm(qkv[:, 1], (D,), T["kn_w"], T["kn_b"], eps)
    rotc = torch.polar(torch.ones(P, 1, D // 2, dtype=torch.float64), torch.from_numpy(ang)[:, None, :])
    def rope(t):
        return torch.view_as_real(torch.view_as_complex(t.reshape(P, H, D // 2, 2).contiguous()) * rotc
                                  ).reshape(P, H, D)
    np.testing.assert_allclose(q, rope(tq).numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(k, rope(tk).numpy(), atol=1e-12, rtol=0)
    np.testing.assert_allclose(v, qkv[:, 2].numpy(), atol=1e-12, rtol=0)


def test_attn_pre_head_norms_closed_form():
    """Unit norm weights, zero norm biases: each rotated q/k head vector has squared
    norm D * s2 / (s2 + eps), s2 the variance of that head of the linear output."""
    x, w, rot, _ = _prologue_inputs(seed=11)
    P, C = x.shape
    H, D = 2, C // 2
    eps = 1e-6
    one, zero = np.ones(D), np.zeros(D)
    q, k, _ = orc.attn_pre(x, w["ln_w"], w["ln_b"], w["w_qkv"], w["b_qkv"], one, zero, one, zero, rot,
                           heads=H, eps=eps)
    lin = (orc.layer_norm(x, w["ln_w"], w["ln_b"], eps) @ w["w_qkv"].T + w["b_qkv"]).reshape(P, 3, H, D)
    for t, out in ((0, q), (1, k)):
        s2 = lin[:, t].var(axis=-1)
        np.testing.assert_allclose((out ** 2).sum(axis=-1), D * s2 / (s2 + eps), rtol=1e-12)


# ---------------------------------------------------------------- 3-D RoPE table
def test_rope3d_bands_split_head_dim():
    assert orc.rope3d_bands(64) == (12, 10, 10)
    assert orc.rope3d_bands(128) == (22, 21, 21)
    assert orc.rope3d_bands(12) == (2, 2, 2)


def test_rope3d_table_hand_worked_entry():
    """head_dim 12: bands of 2 pairs each, frequencies 1 and theta^(-1/2) = 0.01.
    Patch token 5 + 7 of a grid 3 wide sits at (t, h, w) = (4, 2, 1)."""
    tab = orc.rope3d_table(frame_idx=4, P=20, num_special=5, grid_w=3, head_dim=12, theta=10000.0)
    want_ang = [4.0, 0.04, 2.0, 0.02, 1.0, 0.01]
    np.testing.assert_allclose(tab[12, :, 0], np.cos(want_ang), atol=1e-15)
    np.testing.assert_allclose(tab[12, :, 1], np.sin(want_ang), atol=1e-15)


def test_rope3d_table_structure():
    D, P, s, gw = 64, 5 + 37 * 27, 5, 27
    tab = orc.rope3d_table(frame_idx=9, P=P, num_special=s, grid_w=gw, head_dim=D)
    np.testing.assert_allclose(np.hypot(tab[..., 0], tab[..., 1]), 1.0, atol=1e-14)
    n_t, n_h, n_w = orc.rope3d_bands(D)
    # special tokens: only the temporal band rotates
    np.testing.assert_array_equal(tab[:s, n_t:, 0], 1.0)
    np.testing.assert_array_equal(tab[:s, n_t:, 1], 0.0)
    # every token of a frame shares the temporal band
    np.testing.assert_array_equal(tab[:, :n_t], np.broadcast_to(tab[:1, :n_t], tab[:, :n_t].shape))


def test_rope3d_rotated_dot_depends_on_displacement_only():
    """q at token a of frame f1 and k at token b of frame f2: the rotated dot
    product depends on (f2 - f1, h_b - h_a, w_b - w_a) only."""
    D, s, gw = 64, 5, 27
    g = np.random.default_rng(4)
    q, k = g.standard_normal((1, 1, D)), g.standard_normal((1, 1, D))
    def dot(f1, a, f2, b):
        t1 = orc.rope3d_table(f1, a + 1, s, gw, D)[a:a + 1]
        t2 = orc.rope3d_table(f2, b + 1, s, gw, D)[b:b + 1]
        return np.sum(orc.rope_complex(q, t1) * orc.rope_complex(k, t2))
    # token s + 28 is at (h, w) = (1, 1); s + 56 at (2, 2); s + 0 at (0, 0); s + 28 + 1 at (1, 2)
    assert dot(3, s + 0, 5, s + 28) == pytest.approx(dot(10, s + 28, 12, s + 56), abs=1e-10)
    assert dot(0, s + 1, 0, s + 29) == pytest.approx(dot(7, s + 28, 7, s + 56), abs=1e-10)
