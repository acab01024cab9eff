"""Host-side checks of the C ABI (no GPU): the library loads, exports every
function the header declares, rejects bad arguments before touching the GPU,
and its tile scheduler covers exactly the oracle's visible set."""
import ctypes as C

import numpy as np
import pytest

from oracle import attention as orc


@pytest.fixture(scope="module")
def swa():
    import __graft_entry__
    __graft_entry__._builder().build()
    import streaming_frame_causal_b200 as m
    return m


def test_every_header_function_is_exported(swa):
    names = swa.header_functions()
    assert len(names) >= 20
    lib = C.CDLL(swa.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


# the C ABI the hot path's scope names (prefill, stream cache, decode), by name
SECTION_B_NAMES = ("swa_prefill", "swa_stream_cache_bytes", "swa_stream_init", "swa_stream_reset",
                   "swa_stream_append_evict", "swa_stream_attend", "swa_stream_get_meta", "swa_decode",
                   "swa_status_str")


def test_boundary_names_are_exported(swa):
    lib = C.CDLL(swa.LIB_PATH)
    assert all(hasattr(lib, n) for n in SECTION_B_NAMES)
    declared = set(swa.header_functions())
    assert set(SECTION_B_NAMES) <= declared
    # the earlier names stay as aliases of the same calls
    assert {"swa_stream_bytes", "swa_stream_create", "swa_stream_get_meta_raw"} <= declared


def test_meta_host_struct_matches_header(swa):
    # field order and types of swa_meta_host as include/swa.h declares them
    with open(swa.HEADER_PATH) as f:
        text = f.read()
    body = text[text.index("typedef struct swa_meta_host {"):text.index("} swa_meta_host;")]
    import re
    fields = re.findall(r"^\s*(int32_t\*|int)\s+(\w+);", body, re.M)
    assert [n for _, n in fields] == [n for n, _ in swa.swa_meta_host._fields_]
    for (ctype, name), (_, ftype) in zip(fields, swa.swa_meta_host._fields_):
        assert (ctype == "int") == (ftype is C.c_int), name


def test_meta_and_cache_bytes_reject_bad_args(swa):
    lib = swa._lib
    m = swa.swa_meta_host()
    assert lib.swa_stream_get_meta(None, 0, C.byref(m), None) == -1
    assert lib.swa_stream_get_meta_raw(None, 0, None, 0, None) == -1
    cfg = swa._make_cfg(1, 16, 64, 1004, 8, 64, 16, False, 5, 300, __import__("torch").bfloat16, 12)
    assert lib.swa_stream_cache_bytes(C.byref(cfg)) == lib.swa_stream_bytes(C.byref(cfg)) > 0
    h = C.c_void_p()
    assert lib.swa_stream_init(C.byref(h), C.byref(cfg), None, 0, None) == -1


def test_status_strings(swa):
    assert swa.swa_status_str(0) == "ok"
    assert swa.swa_status_str(-3) == "frame out of order"
    assert swa.swa_version() >= 100


def _visible_from_intervals(swa, i, sws, nfpb, S):
    out = []
    for lo, hi in swa.swa_sched_frame_intervals(i, sws, nfpb, S):
        out.extend(range(lo, hi))
    return out


@pytest.mark.parametrize("sws,nfpb,S", [(3, 1, 2), (6, 1, 8), (-1, 1, 0), (1, 1, 0), (2, 2, 1),
                                        (4, 1, 0), (1, 1, 5), (100, 1, 3), (0, 1, 2)])
def test_intervals_equal_oracle_visible_set(swa, sws, nfpb, S):
    for i in range(40):
        ivs = swa.swa_sched_frame_intervals(i, sws, nfpb, S)
        assert 1 <= len(ivs) <= 2
        # disjoint, ascending, not touching (touching runs are merged)
        for (a, b), (c, d) in zip(ivs, ivs[1:]):
            assert b < c
        got = _visible_from_intervals(swa, i, sws, nfpb, S)
        want = [j for j in range(i + 1) if orc.frame_visible(i, j, S, sws, nfpb)]
        assert got == want, (i, got, want)


@pytest.mark.parametrize("F,P,H,sws,S", [(32, 1004, 16, 6, 8), (8, 21, 2, 3, 2), (5, 128, 1, 2, 0),
                                         (7, 129, 3, -1, 1), (3, 300, 2, 1, 0)])
def test_prefill_schedule_covers_visible_pairs_once(swa, F, P, H, sws, S):
    B = 2
    items = swa.swa_sched_prefill(B, F, P, H, sws, 1, S)
    n_pairs = -(-(-(-P // 128)) // 2)
    assert len(items) == F * B * H * n_pairs
    # longest first (non-increasing key tiles), nothing empty
    assert np.all(np.diff(items[:, 6]) <= 0)
    assert np.all(items[:, 6] > 0)
    seen = {}
    for b, h, f, row0, ra, rb, tiles, toks in items:
        vis = [j for j in range(F) if orc.frame_visible(f, j, S, sws, 1)]
        assert toks == len(vis) * P
        # one tile per started 128 keys of each visible run, never a fully masked tile
        runs = swa.swa_sched_frame_intervals(int(f), sws, 1, S)
        assert tiles == sum(-(-((hi - lo) * P) // 128) for lo, hi in runs)
        assert tiles * 128 - toks < 128 * len(runs)
        t0 = (row0 - f * P) // 128
        for t, rows in ((t0, ra), (t0 + 1, rb)):
            if rows:
                key = (b, h, f, t)
                assert key not in seen
                seen[key] = rows
    # every query row of every (b, h, frame) is in exactly one tile
    for b in range(B):
        for h in range(H):
            for f in range(F):
                rows = sum(seen.get((b, h, f, t), 0) for t in range(-(-P // 128)))
                assert rows == P


def test_prefill_rejects_bad_shapes_before_launch(swa):
    lib = swa._lib
    # C != heads * head_dim
    assert lib.swa_prefill(16, 16, 16, 16, 1, 2, 4, 100, 2, 64, 2, 1, 0, 1, None) == -2
    # null pointers
    assert lib.swa_prefill(None, None, None, None, 1, 2, 4, 128, 2, 64, 2, 1, 0, 1, None) == -1
    # bad dtype
    assert lib.swa_prefill(16, 16, 16, 16, 1, 2, 4, 128, 2, 64, 2, 1, 0, 7, None) == -1
    # empty input is a no-op
    assert lib.swa_prefill(None, None, None, None, 1, 0, 4, 128, 2, 64, 2, 1, 0, 1, None) == 0
    # band: Hq not a multiple of Hkv
    assert lib.swa_band_prefill(16, 16, 16, 16, 1, 64, 6, 4, 64, 16, 1, None) == -2
    # decode: negative position
    assert lib.swa_decode(16, 16, 16, 16, 16, -1, 8, 1, 4, 2, 64, 16, None, 0, 1, None) == -1


def test_stream_geometry_sizes(swa):
    # 8 scale + 64 window frames of 1004 tokens, 16 heads x 64, bf16: 72 slots x 63 pages
    n = swa.swa_stream_bytes(num_layers=1, heads=16, head_dim=64, P=1004, scale_frames=8,
                             window_frames=64, page_tokens=16, cross_frame_special=False, num_special=5,
                             max_frames=300, dtype=__import__("torch").bfloat16, max_splits=16)
    rows = 72 * 63 * 16
    assert n >= 2 * rows * 16 * 64 * 2
    n2 = swa.swa_stream_bytes(num_layers=1, heads=16, head_dim=64, P=1004, scale_frames=8,
                              window_frames=64, page_tokens=16, cross_frame_special=True, num_special=5,
                              max_frames=1000, dtype=__import__("torch").bfloat16, max_splits=16)
    # special region: 928 evicted frames x 5 tokens = 4640 tokens = 290 pages
    assert n2 - n >= 2 * 290 * 16 * 16 * 64 * 2
    bad = swa._make_cfg(1, 16, 64, 1004, 8, 64, 16, False, 2000, 300, __import__("torch").bfloat16, 16)
    assert swa._lib.swa_stream_bytes(C.byref(bad)) == 0


@pytest.mark.parametrize("B,Hkv,W,pos", [(64, 8, 4096, 200000), (8, 8, 1024, 5000), (1, 1, 640, 639),
                                         (2, 16, 300, 1000), (4, 8, 1024, 500), (3, 8, 256, 700),
                                         (2, 1, 130, 129), (1, 8, 4096, 10), (1, 1, 5000, 4998),
                                         (200, 8, 4096, 10**6), (3, 2, 64, 200), (2, 2, 64, 10)])
def test_decode_plan_covers_the_valid_window(swa, B, Hkv, W, pos):
    pl = swa.swa_sched_decode(B, Hkv, W, pos)
    n_valid = min(pos + 1, W)
    assert pl["n_valid"] == n_valid
    # pieces fit the workspace's partial slots and are whole 128-key tiles
    assert 1 <= pl["pieces"] <= pl["slots"]
    assert pl["piece_len"] % 128 == 0 and pl["piece_len"] > 0
    # the pieces [k*len, min((k+1)*len, n_valid)) cover the valid slots exactly once
    covered = []
    for k in range(pl["pieces"]):
        lo, hi = k * pl["piece_len"], min((k + 1) * pl["piece_len"], n_valid)
        if hi > lo:
            covered.append((lo, hi))
    assert covered[0][0] == 0 and covered[-1][1] == n_valid
    assert all(a[1] == b[0] for a, b in zip(covered, covered[1:]))
    # one CTA per SM at most, none idle when units run short
    assert pl["grid"] == min(B * Hkv * pl["pieces"], 148)
    # the workspace the caller sizes holds every partial the plan writes
    G = 4
    need = swa.swa_decode_workspace_bytes(B, Hkv * G, Hkv, 128, W)
    assert need >= B * Hkv * pl["pieces"] * G * (128 + 2) * 4


def test_decode_plan_bench_shape_and_bad_args(swa):
    # batch 64, 8 KV heads, 4096 slots: two halves per (batch, KV head), 1024 units on 148 CTAs
    assert swa.swa_sched_decode(64, 8, 4096, 200000) == {"pieces": 2, "piece_len": 2048, "grid": 148,
                                                          "slots": 8, "n_valid": 4096}
    for bad in ((0, 8, 4096, 1), (1, 0, 4096, 1), (1, 8, 0, 1), (1, 8, 4096, -1)):
        with pytest.raises(swa.SwaError):
            swa.swa_sched_decode(*bad)


@pytest.mark.parametrize("T,H,P,max_splits", [(576, 16, 1004, 12), (601, 16, 1004, 12), (576, 8, 1004, 12),
                                               (576, 16, 1004, 32), (8, 2, 200, 12), (3, 2, 130, 12),
                                               (1, 1, 21, 12), (576, 16, 1004, 1)])
def test_stream_plan_splits_every_item_into_nonempty_ranges(swa, T, H, P, max_splits):
    """The streaming attend's split count stays within the handle's partial
    buffers, never exceeds the key tiles (no split is empty, so the combine never
    reads an unwritten partial), and the ranges differ by at most one tile."""
    pl = swa.swa_sched_stream(T, H, P, max_splits)
    n_pairs = -(-(-(-P // 128)) // 2)
    assert 1 <= pl["splits"] <= min(max_splits, T)
    assert pl["ctas"] == H * n_pairs * pl["splits"]
    assert pl["min_tiles"] >= 1 and pl["max_tiles"] - pl["min_tiles"] <= 1


def test_stream_plan_bench_shape_and_bad_args(swa):
    # 8 scale + 64 window frames of 1004 tokens, 16 heads: nine splits of 64 key tiles
    # (576 CTAs, 3.9 waves on 148 SMs), also with room for 32 (4 and 16 ran slower)
    assert swa.swa_sched_stream(576, 16, 1004, 12) == {"splits": 9, "ctas": 576, "min_tiles": 64, "max_tiles": 64}
    assert swa.swa_sched_stream(576, 16, 1004, 32)["splits"] == 9
    for bad in ((0, 16, 1004, 12), (576, 0, 1004, 12), (576, 16, 0, 12), (576, 16, 1004, 0), (576, 16, 1004, 33)):
        with pytest.raises(swa.SwaError):
            swa.swa_sched_stream(*bad)


def test_head_slices_and_generated_rope_are_validated(swa):
    lib = swa._lib
    # row stride shorter than head0 + heads: rejected before anything runs
    assert lib.swa_prefill_heads(256, 256, 256, 256, 1, 2, 16, 512, 4, 8, 64, 2, 1, 0, 1, None) == -2
    # row stride not a multiple of 16 bytes
    assert lib.swa_prefill_heads(256, 256, 256, 256, 1, 2, 16, 1028, 0, 8, 64, 2, 1, 0, 1, None) == -1
    # negative head offset
    assert lib.swa_prefill_heads(256, 256, 256, 256, 1, 2, 16, 1024, -1, 8, 64, 2, 1, 0, 1, None) == -1
    # generated RoPE: grid width 0, negative frame, theta <= 1, specials beyond P
    args = [256] * 9
    for fr, ns, gw, th in ((0, 5, 0, 1e4), (-1, 5, 27, 1e4), (0, 5, 27, 1.0), (0, 2000, 27, 1e4)):
        assert lib.swa_attn_pre_rope3d(*args, fr, ns, gw, th, 1004, 1024, 16, 1e-6, 256, 256, 256, 256,
                                       None) == -1


def test_binding_argument_counts_match_the_header(swa):
    """Every ctypes signature the binding declares takes as many arguments as
    the header's declaration of that function."""
    import re
    with open(swa.HEADER_PATH) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    decls = dict((m.group(1), m.group(2)) for m in re.finditer(r"\b(swa_[a-z0-9_]+)\s*\(([^;{]*?)\)\s*;", text))
    checked = 0
    for name, (_, args) in swa._sigs.items():
        params = decls[name].strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert n == len(args), (name, n, len(args))
        checked += 1
    assert checked == len(decls)
