"""The attention prologue (norm1, qkv linear, per-head q/k LayerNorm, RoPE) on the
tensor cores against the float64 oracle, and its fused form in the streaming
append (K/V written straight into the cache slot)."""
import numpy as np
import pytest
import torch

import synth
from oracle import attention as orc
from tol import check_bf16

pytestmark = pytest.mark.gpu

EPS = 1e-6
ORDER = ("ln_w", "ln_b", "w_qkv", "b_qkv", "qn_w", "qn_b", "kn_w", "kn_b", "rot")


@pytest.fixture(scope="module")
def swa():
    import streaming_frame_causal_b200 as m
    return m


def _oracle(inp, heads):
    a = {k: v.double().numpy() for k, v in inp.items()}
    return orc.attn_pre(a["x"], a["ln_w"], a["ln_b"], a["w_qkv"], a["b_qkv"], a["qn_w"], a["qn_b"], a["kn_w"],
                        a["kn_b"], a["rot"], heads=heads, eps=EPS)


@pytest.mark.parametrize("P,C,H", [
    (1004, 1024, 16),   # the streaming frame: 1004 tokens, 16 heads x 64 (8 token tiles, ragged last)
    (200, 1024, 8),     # head_dim 128, two token tiles
    (37, 512, 8),       # one ragged token tile, two feature tiles per section
])
def test_attn_pre_matches_oracle(swa, P, C, H):
    inp = synth.prologue_inputs(seed=P + C + H, P=P, C=C, heads=H)
    d = {k: v.cuda() for k, v in inp.items()}
    q, k, v = swa.swa_attn_pre(d["x"], *(d[n] for n in ORDER), heads=H, eps=EPS)
    torch.cuda.synchronize()
    assert swa.swa_device_error_check() == 0
    rq, rk, rv = _oracle(inp, H)
    # bf16 tolerance: norm1's output is rounded to bf16 before the GEMM (relative
    # 2^-9 per element, averaging down over the C-term sums), the outputs to bf16
    for got, ref, name in ((q, rq, "q"), (k, rk, "k"), (v, rv, "v")):
        check_bf16(got.float().cpu().numpy(), ref, f"{name} P{P} C{C} H{H}")


def test_attn_pre_rejects_bad_shapes(swa):
    inp = synth.prologue_inputs(seed=1, P=16, C=512, heads=8)
    d = {k: v.cuda() for k, v in inp.items()}
    with pytest.raises(RuntimeError):
        swa.swa_attn_pre(d["x"][:, :320].contiguous(), *(d[n] for n in ORDER), heads=5)   # head_dim 64, C 320
    with pytest.raises(RuntimeError):
        swa.swa_attn_pre(d["x"], *(d[n] for n in ORDER), heads=16)                        # head_dim 32


@pytest.mark.parametrize("special", [False, True])
def test_fused_append_writes_the_prologue_into_the_slot(swa, special):
    """Frames appended from their tokens: the page storage of each frame's slot
    holds exactly the K/V swa_attn_pre produces for those tokens, Q matches too,
    the bookkeeping is the oracle's, and evicted frames' specials were moved
    before the slot was overwritten."""
    P, C, H, S, Wc, F = 300, 1024, 16, 1, 2, 6
    D = C // H
    cache = swa.SwaStream(num_layers=1, heads=H, head_dim=D, P=P, scale_frames=S, window_frames=Wc,
                          cross_frame_special=special, num_special=5, max_frames=F, dtype=torch.bfloat16)
    oc = orc.StreamCache(heads=H, head_dim=D, P=P, scale_frames=S, window_frames=Wc, page_tokens=16,
                         cross_frame_special=special, num_special=5, max_frames=F)
    ks = cache.storage(0, "k")
    vs = cache.storage(0, "v")
    ppf = -(-P // 16)
    frames_k = {}
    for i in range(F):
        inp = synth.prologue_inputs(seed=50 + i, P=P, C=C, heads=H)
        d = {k: v.cuda() for k, v in inp.items()}
        q_ref, k_ref, v_ref = swa.swa_attn_pre(d["x"], *(d[n] for n in ORDER), heads=H, eps=EPS)
        q_out = torch.empty_like(q_ref)
        cache.swa_stream_append_evict_pre(0, i, d["x"], *(d[n] for n in ORDER), q_out=q_out, eps=EPS)
        torch.cuda.synchronize()
        assert torch.equal(q_out, q_ref)
        slot = oc.slot_of(i)
        r0 = slot * ppf * 16
        assert torch.equal(ks[r0:r0 + P], k_ref) and torch.equal(vs[r0:r0 + P], v_ref)
        oc.append_evict(0, i, np.zeros((P, H, D)), np.zeros((P, H, D)))
        frames_k[i] = k_ref.clone()
        meta = cache.swa_stream_get_meta(0)
        assert meta["n_frames"] == i + 1 and meta["n_evicted"] == oc.layers[0].n_evicted
        np.testing.assert_array_equal(meta["slot_frame"], oc.slot_frames(0))
        np.testing.assert_array_equal(meta["page_table"], oc.page_table(0))
        if special and oc.layers[0].last_evicted >= 0:
            j = oc.layers[0].last_evicted
            sp0 = cache.layout.n_slots * ppf * 16 + (j - S) * 5
            assert torch.equal(ks[sp0:sp0 + 5], frames_k[j][:5])
    assert swa.swa_device_error_check() == 0


@pytest.mark.parametrize("D", [64, 128])
def test_rope3d_table_matches_oracle(swa, D):
    """The lingbot-map frame (5 special tokens + a 37 x 27 patch grid) at frames
    0, 7 and 999: angles in double on the device, stored as f32."""
    P, s, gw = 5 + 37 * 27, 5, 27
    for f in (0, 7, 999):
        got = swa.swa_rope3d_table(f, P, s, gw, D).cpu().numpy()
        ref = orc.rope3d_table(f, P, s, gw, D)
        np.testing.assert_allclose(got, ref, atol=2e-7, rtol=0)


def test_prologue_with_3d_rope_table(swa):
    P, C, H = 5 + 37 * 27, 1024, 16
    inp = synth.prologue_inputs(seed=77, P=P, C=C, heads=H)
    d = {k: v.cuda() for k, v in inp.items()}
    rot = swa.swa_rope3d_table(42, P, 5, 27, C // H)
    q, k, v = swa.swa_attn_pre(d["x"], *(d[n] for n in ORDER[:-1]), rot, heads=H, eps=EPS)
    torch.cuda.synchronize()
    a = {n: t.double().numpy() for n, t in inp.items()}
    a["rot"] = orc.rope3d_table(42, P, 5, 27, C // H)
    rq, rk, rv = orc.attn_pre(a["x"], *(a[n] for n in ORDER), heads=H, eps=EPS)
    for got, ref, name in ((q, rq, "q"), (k, rk, "k"), (v, rv, "v")):
        check_bf16(got.float().cpu().numpy(), ref, f"{name} with the 3-D table")


def test_rope3d_table_rejects_bad_arguments(swa):
    lib = swa._lib
    buf = torch.empty(16, 32, 2, device="cuda")
    assert lib.swa_rope3d_table(-1, 16, 5, 3, 64, 10000.0, buf.data_ptr(), None) == -1
    assert lib.swa_rope3d_table(0, 16, 17, 3, 64, 10000.0, buf.data_ptr(), None) == -1
    assert lib.swa_rope3d_table(0, 16, 5, 0, 64, 10000.0, buf.data_ptr(), None) == -1
    assert lib.swa_rope3d_table(0, 16, 5, 3, 63, 10000.0, buf.data_ptr(), None) == -1
    assert lib.swa_rope3d_table(0, 16, 5, 3, 64, 1.0, buf.data_ptr(), None) == -1
    assert lib.swa_rope3d_table(0, 16, 5, 3, 64, 10000.0, None, None) == -1


@pytest.mark.parametrize("frame,H", [(0, 16), (7, 16), (999, 16), (999, 8)])
def test_prologue_generates_3d_rope(swa, frame, H):
    """The lingbot-map frame (5 special tokens + a 37 x 27 grid) with the 3-D RoPE
    generated inside the prologue: q/k against the oracle's prologue with its
    float64 table, v unchanged; head_dim 64 and 128."""
    P, C = 5 + 37 * 27, 1024
    inp = synth.prologue_inputs(seed=900 + frame + H, P=P, C=C, heads=H)
    d = {k: v.cuda() for k, v in inp.items()}
    q, k, v = swa.swa_attn_pre_rope3d(d["x"], *(d[n] for n in ORDER[:-1]), heads=H, frame_idx=frame,
                                      num_special=5, grid_w=27, eps=EPS)
    torch.cuda.synchronize()
    assert swa.swa_device_error_check() == 0
    a = {n: t.double().numpy() for n, t in inp.items()}
    a["rot"] = orc.rope3d_table(frame, P, 5, 27, C // H)
    rq, rk, rv = orc.attn_pre(a["x"], *(a[n] for n in ORDER), heads=H, eps=EPS)
    for got, ref, name in ((q, rq, "q"), (k, rk, "k"), (v, rv, "v")):
        check_bf16(got.float().cpu().numpy(), ref, f"{name}, generated 3-D RoPE, frame {frame}")


def test_fused_append_with_generated_rope(swa):
    """The streaming append with the generated 3-D RoPE writes into the slot
    exactly what swa_attn_pre_rope3d computes for the frame's index."""
    P, C, H, S, Wc, F = 5 + 37 * 27, 1024, 16, 1, 2, 4
    D = C // H
    cache = swa.SwaStream(num_layers=1, heads=H, head_dim=D, P=P, scale_frames=S, window_frames=Wc,
                          max_frames=F, dtype=torch.bfloat16)
    ks, vs = cache.storage(0, "k"), cache.storage(0, "v")
    ppf = -(-P // 16)
    oc = orc.StreamCache(heads=H, head_dim=D, P=P, scale_frames=S, window_frames=Wc, page_tokens=16,
                         max_frames=F)
    for i in range(F):
        inp = synth.prologue_inputs(seed=70 + i, P=P, C=C, heads=H)
        d = {k: v.cuda() for k, v in inp.items()}
        q_ref, k_ref, v_ref = swa.swa_attn_pre_rope3d(d["x"], *(d[n] for n in ORDER[:-1]), heads=H, frame_idx=i,
                                                      num_special=5, grid_w=27, eps=EPS)
        q_out = torch.empty_like(q_ref)
        cache.swa_stream_append_evict_pre_rope3d(0, i, d["x"], *(d[n] for n in ORDER[:-1]), q_out=q_out,
                                                 num_special=5, grid_w=27, eps=EPS)
        torch.cuda.synchronize()
        assert torch.equal(q_out, q_ref)
        r0 = oc.slot_of(i) * ppf * 16
        oc.append_evict(0, i, np.zeros((P, H, D)), np.zeros((P, H, D)))
        assert torch.equal(ks[r0:r0 + P], k_ref) and torch.equal(vs[r0:r0 + P], v_ref)
    assert swa.swa_device_error_check() == 0
