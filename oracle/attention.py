"""Float64 CPU oracle for frame-causal sliding-window attention (TEST INFRASTRUCTURE).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The CUDA library never calls it and shares
no code with it: everything here is written straight from the method's
definition, slowly and explicitly, in float64 with explicit boolean masks.

Sources (page title, section):
  [AGG]  "Sliding Window Attention Mechanism in AggregatorStream: Implementation
         and Configuration Guide" -- sections "Configuring the Sliding Window",
         "Mask Generation in CausalAttention", "KV Cache Eviction Strategy",
         "Manual Sliding-Window Mask Construction", FAQ "What happens when
         sliding_window_size is set to -1?", FAQ "Can special tokens persist
         outside the sliding window?".
  [IO]   "Stream.py Aggregator Input and Output Formats" -- "Input Tensor
         Specifications" (tokens are [B*S, P, C]) and "Scalar Parameters".
  [BLK]  "Method forward" (lingbot_map/layers/block.py, FlashInferBlock.forward):
         append_frame -> evict_frames -> compute_attention, q/k/v in [tpf, H, D].
  [SWA]  sliding-window attention explainer (Mistral 7B): band i-W+1..i,
         rolling buffer slot i mod W, grouped-query attention, L*W reach.
  [PRE]  "Method forward" (block forward listing): the compiled attn_pre step
         "norm1 + qkv linear + reshape + q_norm + k_norm + RoPE + format", and
         the I/O page's 3-D RoPE format: a complex-valued table
         [.., S_global*P, head_dim/2] (WanRotaryPosEmbed).

Readings where the pages are silent:
  * causality is frame-granular: a query frame sees all of its own frame
    ([AGG] snippet ends the window at the end of the current frame);
  * the first ``S = num_frame_for_scale`` frames are always visible to later
    frames (they are never evicted from the cache, [AGG] eviction pseudocode);
  * ``sliding_window_size <= 0`` disables the window ([AGG] FAQ on -1);
  * the softmax scale is 1/sqrt(head_dim) (the default of the SDPA call named
    in [AGG] "Mask Generation");
  * the special tokens of a frame are its first ``num_special`` tokens
    (camera, then registers), and evicted frames keep them in cache order of
    eviction;
  * attn_pre: norm1 is a LayerNorm over C with weight and bias, the qkv linear
    has a bias, q_norm / k_norm are LayerNorms over head_dim with weight and
    bias, and RoPE multiplies the (2i, 2i+1) pairs of q and k by the caller's
    complex table (cos, sin) per token and pair.

Parity status: every function here is pinned by ``tests/test_oracle.py``
(closed forms, library special cases, brute force on tiny inputs, the pages'
own mask snippet, stream == prefill identity, reachability).  None is
"parity unpinned".
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

NEG_INF = -np.inf


# ----------------------------------------------------------------------------
# Visible set  ([AGG] "Mask Generation in CausalAttention")
# ----------------------------------------------------------------------------
def window_frames(sliding_window_size: int, num_frame_per_block: int) -> int:
    """Width of the frame window, in frames; 0 means "no window" (full causal).

    [AGG]: window_start_frame = max(0, i - sliding_window_size*num_frame_per_block + 1);
    sliding_window_size = -1 disables the window.
    """
    if sliding_window_size is None or sliding_window_size <= 0:
        return 0
    return int(sliding_window_size) * int(num_frame_per_block)


def frame_visible(i: int, j: int, scale_frames: int, sliding_window_size: int,
                  num_frame_per_block: int = 1) -> bool:
    """True iff query frame ``i`` may attend to key frame ``j``.

    Causal AND window ([AGG] "mask = mask & sliding_mask"), OR j is one of the
    retained scale frames (j < scale_frames, still causal).
    """
    if j > i:
        return False
    if j < scale_frames:
        return True
    wf = window_frames(sliding_window_size, num_frame_per_block)
    if wf == 0:
        return True
    window_start = max(0, i - wf + 1)
    return j >= window_start


def frame_mask(num_frames: int, P: int, scale_frames: int, sliding_window_size: int,
               num_frame_per_block: int = 1, rows=None) -> np.ndarray:
    """Explicit boolean mask [len(rows), N] over tokens, N = num_frames * P.

    Built element by element from :func:`frame_visible` applied to the frames
    of the query and key tokens (``num_frames = N // frame_seqlen`` in [AGG]).
    """
    N = num_frames * P
    if rows is None:
        rows = np.arange(N)
    rows = np.asarray(rows)
    key_frame = np.arange(N) // P
    m = np.zeros((len(rows), N), dtype=bool)
    for r_i, t in enumerate(rows):
        qi = int(t) // P
        vis = np.array([frame_visible(qi, int(j), scale_frames, sliding_window_size,
                                      num_frame_per_block) for j in range(num_frames)])
        m[r_i] = vis[key_frame]
    return m


# ----------------------------------------------------------------------------
# Masked softmax attention, one head
# ----------------------------------------------------------------------------
def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray,
                      mask: np.ndarray | None = None, scale: float | None = None) -> np.ndarray:
    """O = softmax(mask(q k^T * scale)) v in float64 for one head.

    q [nq, D], k [nk, D], v [nk, Dv]; mask [nq, nk] (True = visible).  Masked
    logits are -inf; the softmax subtracts the row maximum before exponentiating.
    Every row must see at least one key.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    logits = (q @ k.T) * scale
    if mask is not None:
        if not np.all(mask.any(axis=1)):
            raise ValueError("a query row sees no key")
        logits = np.where(mask, logits, NEG_INF)
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    return (e / e.sum(axis=1, keepdims=True)) @ v


# ----------------------------------------------------------------------------
# Full-sequence prefill  ([AGG] "Mask Generation"; [IO] tokens [B*S, P, C])
# ----------------------------------------------------------------------------
def prefill(q, k, v, P: int, scale_frames: int, sliding_window_size: int,
            num_frame_per_block: int = 1, rows=None, heads=None) -> np.ndarray:
    """Frame-causal sliding-window attention over a whole clip.

    q, k, v: [B, N, H, D] with N = num_frames * P (the pages' [B*S, P, C] with
    C = H*D split into heads).  Returns float64 [B, len(rows), len(heads), D].
    ``rows`` / ``heads`` select a sample of query rows / heads (default all).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, H, D = q.shape
    if N % P:
        raise ValueError("N must be a multiple of P")
    F = N // P
    rows = np.arange(N) if rows is None else np.asarray(rows)
    heads = list(range(H)) if heads is None else list(heads)
    mask = frame_mask(F, P, scale_frames, sliding_window_size, num_frame_per_block, rows)
    out = np.zeros((B, len(rows), len(heads), v.shape[-1]))
    for b in range(B):
        for hi, h in enumerate(heads):
            out[b, :, hi] = softmax_attention(q[b, rows, h], k[b, :, h], v[b, :, h], mask)
    return out


# ----------------------------------------------------------------------------
# Streaming rolling / paged cache  ([AGG] "KV Cache Eviction Strategy";
# [BLK] append_frame / evict_frames / compute_attention; [SWA] slot i mod W)
# ----------------------------------------------------------------------------
@dataclass
class _LayerState:
    cached: list = field(default_factory=list)      # frame indices, cache order
    frames: dict = field(default_factory=dict)      # frame index -> (k [P,H,D], v)
    specials_k: list = field(default_factory=list)  # per evicted frame: [ns, H, D]
    specials_v: list = field(default_factory=list)
    special_from: list = field(default_factory=list)  # frame index of each special block
    n_frames: int = 0
    n_evicted: int = 0
    last_evicted: int = -1


class StreamCache:
    """Host model of the per-layer rolling paged KV cache.

    Per layer (``global_idx`` selects the layer's cache, [BLK] ``block_idx=global_idx``):

    * appending frame i stores its K/V ([BLK] ``append_frame``);
    * then, while the number of cached full frames exceeds
      ``window_frames + scale_frames``, the frames in cache positions
      [scale_frames, num_cached - window_frames) are removed ([AGG] eviction
      pseudocode) -- at most one frame per step, the oldest non-scale frame;
    * with ``cross_frame_special`` an evicted frame leaves its first
      ``num_special`` tokens (camera + registers) in the cache ([AGG] FAQ on
      special tokens);
    * the frame's queries then attend to everything the cache holds, with no
      mask ([BLK] ``compute_attention`` after eviction; eviction happens before
      attention, [AGG]).

    Bookkeeping (pure functions of the frame index, exported for bit-exact
    comparison):

    * slots: frame i < S -> slot i; frame i >= S -> slot S + (i mod W_c)
      ([SWA] rolling buffer slot i mod W, applied to frames);
      ``window_frames <= 0`` keeps every frame, frame i -> slot i;
    * pages of ``page_tokens`` tokens; slot s owns physical pages
      s*ppf .. s*ppf+ppf-1 with ppf = ceil(P / page_tokens);
    * the special region starts at physical page n_slots*ppf; special token u
      (u = e*num_special + r for the e-th evicted frame) lives at page
      base + u // page_tokens, offset u % page_tokens;
    * the page table lists, for the retained full frames in ascending frame
      order, their ppf pages, then the special pages in order.
    """

    def __init__(self, heads: int, head_dim: int, P: int, scale_frames: int,
                 window_frames: int, page_tokens: int = 16, cross_frame_special: bool = False,
                 num_special: int = 5, max_frames: int | None = None, num_layers: int = 1):
        self.H, self.D, self.P = heads, head_dim, P
        self.S = int(scale_frames)
        self.W = int(window_frames)
        self.page_tokens = int(page_tokens)
        self.cross_frame_special = bool(cross_frame_special)
        self.num_special = int(num_special)
        self.ppf = -(-P // page_tokens)
        if self.W > 0:
            self.n_slots = self.S + self.W
        else:
            if max_frames is None:
                raise ValueError("an unbounded cache needs max_frames")
            self.n_slots = int(max_frames)
        self.max_frames = max_frames
        self.layers = [_LayerState() for _ in range(num_layers)]

    # --- pure bookkeeping ---------------------------------------------------
    def slot_of(self, i: int) -> int:
        if self.W <= 0 or i < self.S:
            return i
        return self.S + (i % self.W)

    # --- operations -----------------------------------------------------------
    def append_evict(self, layer: int, frame_idx: int, k, v) -> list:
        """Append frame ``frame_idx`` to the layer's cache, then apply the
        eviction rule literally on the ordered list of cached frames:
        if num_cached > W + S, drop cache positions [S, num_cached - W).
        Returns the evicted frame indices (ascending)."""
        st = self.layers[layer]
        if frame_idx != st.n_frames:
            raise ValueError("frames must be appended in order")
        if self.W <= 0 and frame_idx >= self.n_slots:
            raise ValueError("cache capacity exceeded")
        st.frames[frame_idx] = (np.asarray(k, dtype=np.float64), np.asarray(v, dtype=np.float64))
        st.cached.append(frame_idx)
        st.n_frames += 1
        evicted = []
        n = len(st.cached)
        if self.W > 0 and n > self.W + self.S:
            evicted = st.cached[self.S:n - self.W]
            st.cached = st.cached[:self.S] + st.cached[n - self.W:]
        for j in evicted:
            kj, vj = st.frames.pop(j)
            if self.cross_frame_special:
                st.specials_k.append(kj[: self.num_special])
                st.specials_v.append(vj[: self.num_special])
                st.special_from.append(j)
            st.n_evicted += 1
        st.last_evicted = evicted[-1] if evicted else -1
        return list(evicted)

    def gather(self, layer: int):
        """All cached keys/values, [n, H, D], full frames ascending then specials."""
        st = self.layers[layer]
        ks = [st.frames[j][0] for j in sorted(st.frames)] + list(st.specials_k)
        vs = [st.frames[j][1] for j in sorted(st.frames)] + list(st.specials_v)
        return np.concatenate(ks, axis=0), np.concatenate(vs, axis=0)

    def attend(self, layer: int, q) -> np.ndarray:
        """The current frame's queries [P, H, D] against the whole cache."""
        q = np.asarray(q, dtype=np.float64)
        kc, vc = self.gather(layer)
        out = np.zeros((q.shape[0], self.H, vc.shape[-1]))
        for h in range(self.H):
            out[:, h] = softmax_attention(q[:, h], kc[:, h], vc[:, h])
        return out

    def attend_transient(self, layer: int, q, k, v) -> np.ndarray:
        """Non-keyframe attend: the frame's queries [P, H, D] against everything
        the layer's cache holds plus the frame's own keys/values [P, H, D], with
        the cache left exactly as it was.

        Follows the "Non-keyframe path" of the streaming branch in the pages'
        block forward listing (lingbot-map AggregatorStream guide): the frame is
        appended with eviction deferred, attended to, and the append is rolled
        back.  So no frame is evicted (the oldest window frame is still visible),
        no special token moves, and the frame counter does not advance."""
        st = self.layers[layer]
        k = np.asarray(k, dtype=np.float64)
        v = np.asarray(v, dtype=np.float64)
        q = np.asarray(q, dtype=np.float64)
        if st.frames or st.specials_k:
            kc, vc = self.gather(layer)
            kc = np.concatenate([kc, k], axis=0)
            vc = np.concatenate([vc, v], axis=0)
        else:
            kc, vc = k, v
        out = np.zeros((q.shape[0], self.H, vc.shape[-1]))
        for h in range(self.H):
            out[:, h] = softmax_attention(q[:, h], kc[:, h], vc[:, h])
        return out

    # --- exported bookkeeping ---------------------------------------------------
    def n_special_tokens(self, layer: int) -> int:
        return len(self.layers[layer].specials_k) * self.num_special

    def slot_frames(self, layer: int) -> np.ndarray:
        s = -np.ones(self.n_slots, dtype=np.int32)
        for j in self.layers[layer].frames:
            s[self.slot_of(j)] = j
        return s

    def page_table(self, layer: int) -> np.ndarray:
        st = self.layers[layer]
        pages = []
        for j in sorted(st.frames):
            s = self.slot_of(j)
            pages.extend(range(s * self.ppf, s * self.ppf + self.ppf))
        base = self.n_slots * self.ppf
        nsp = self.n_special_tokens(layer)
        pages.extend(range(base, base + -(-nsp // self.page_tokens)))
        return np.asarray(pages, dtype=np.int32)

    def special_location(self, u: int):
        """(physical page, offset) of special token u."""
        base = self.n_slots * self.ppf
        return base + u // self.page_tokens, u % self.page_tokens


# ----------------------------------------------------------------------------
# Token-level band attention with grouped-query heads  ([SWA])
# ----------------------------------------------------------------------------
def band_mask(N: int, W: int, rows=None) -> np.ndarray:
    """Explicit mask: token t sees s iff t - W + 1 <= s <= t ([SWA])."""
    rows = np.arange(N) if rows is None else np.asarray(rows)
    s = np.arange(N)[None, :]
    t = rows[:, None]
    return (s <= t) & (s >= t - W + 1)


def band_attention(q, k, v, W: int, rows=None, heads=None) -> np.ndarray:
    """Mistral-style sliding-window attention with grouped-query heads.

    q [B, N, Hq, D], k/v [B, N, Hkv, D]; query head h reads KV head
    h // (Hq // Hkv).  Returns float64 [B, len(rows), len(heads), D].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    group = Hq // Hkv
    rows = np.arange(N) if rows is None else np.asarray(rows)
    heads = list(range(Hq)) if heads is None else list(heads)
    mask = band_mask(N, W, rows)
    out = np.zeros((B, len(rows), len(heads), v.shape[-1]))
    for b in range(B):
        for hi, h in enumerate(heads):
            out[b, :, hi] = softmax_attention(q[b, rows, h], k[b, :, h // group],
                                              v[b, :, h // group], mask)
    return out


# ----------------------------------------------------------------------------
# Single-token decode against a rolling buffer  ([SWA] slot i mod W)
# ----------------------------------------------------------------------------
def decode_slot(pos: int, W: int) -> int:
    """Rolling-buffer slot of position ``pos``: pos mod W ([SWA])."""
    return int(pos) % int(W)


def decode(q, k_new, v_new, k_cache, v_cache, pos: int, W: int):
    """Write the new token's K/V at slot pos mod W, then attend over the buffer.

    q [B, Hq, D], k_new/v_new [B, Hkv, D], caches [B, W, Hkv, D] holding
    positions pos-W+1 .. pos-1 (slot p mod W).  Valid slots are all W once
    pos >= W-1, else slots 0..pos.  Returns (out float64 [B, Hq, D],
    updated k_cache, updated v_cache) -- the caches as float64 copies.
    """
    q = np.asarray(q, dtype=np.float64)
    kc = np.array(k_cache, dtype=np.float64, copy=True)
    vc = np.array(v_cache, dtype=np.float64, copy=True)
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    group = Hq // Hkv
    s = decode_slot(pos, W)
    kc[:, s] = np.asarray(k_new, dtype=np.float64)
    vc[:, s] = np.asarray(v_new, dtype=np.float64)
    n_valid = W if pos >= W - 1 else pos + 1
    out = np.zeros((B, Hq, vc.shape[-1]))
    for b in range(B):
        for h in range(Hq):
            g = h // group
            out[b, h] = softmax_attention(q[b, h][None, :], kc[b, :n_valid, g],
                                          vc[b, :n_valid, g])[0]
    return out, kc, vc


# ----------------------------------------------------------------------------
# attn_pre prologue  ([PRE]: norm1 + qkv linear + reshape + q_norm + k_norm + RoPE)
# ----------------------------------------------------------------------------
def layer_norm(x, weight, bias, eps: float):
    """LayerNorm over the last axis: (x - mean) / sqrt(var + eps) * weight + bias
    (biased variance), in float64."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(weight, np.float64) + np.asarray(bias, np.float64)


def rope_complex(x, rot):
    """Rotate the (2i, 2i+1) pairs of x [..., P, H, D] by the complex numbers
    rot [P, D/2, 2] = (cos, sin) of each token and pair: the complex-valued
    position format of the I/O page's 3-D RoPE (x viewed as D/2 complex
    numbers, multiplied elementwise)."""
    x = np.asarray(x, dtype=np.float64)
    rot = np.asarray(rot, dtype=np.float64)
    re, im = x[..., 0::2], x[..., 1::2]
    c = rot[:, None, :, 0]  # broadcast over heads
    s = rot[:, None, :, 1]
    out = np.empty_like(x)
    out[..., 0::2] = re * c - im * s
    out[..., 1::2] = re * s + im * c
    return out


def attn_pre(x, ln_w, ln_b, w_qkv, b_qkv, qn_w, qn_b, kn_w, kn_b, rot, heads: int, eps: float = 1e-6):
    """One frame's attention prologue ([PRE]): x [P, C] -> q, k, v [P, H, D].

    norm1 (LayerNorm over C) -> qkv linear (x_n @ w_qkv.T + b_qkv, w_qkv
    [3C, C]) -> reshape to [P, 3, H, D] -> q_norm, k_norm (LayerNorm over D) ->
    RoPE on q and k (complex pairs, table rot [P, D/2, 2]); v is passed on."""
    x = np.asarray(x, dtype=np.float64)
    P, C = x.shape
    D = C // heads
    xn = layer_norm(x, ln_w, ln_b, eps)
    qkv = xn @ np.asarray(w_qkv, np.float64).T + np.asarray(b_qkv, np.float64)
    qkv = qkv.reshape(P, 3, heads, D)
    q = layer_norm(qkv[:, 0], qn_w, qn_b, eps)
    k = layer_norm(qkv[:, 1], kn_w, kn_b, eps)
    v = qkv[:, 2]
    return rope_complex(q, rot), rope_complex(k, rot), v.copy()


# ----------------------------------------------------------------------------
# 3-D RoPE table of a streaming frame ([IO] 3-D RoPE: complex-valued positions
# [1, 1, S_global*P, head_dim/2] from WanRotaryPosEmbed, built internally when
# enable_3d_rope=True)
# ----------------------------------------------------------------------------
def rope3d_bands(head_dim: int):
    """Complex pairs per axis (t, h, w): the head's D/2 pairs split as
    h = w = floor(D/6) pairs each and t = the rest (the Wan-style split of
    head_dim into temporal, height and width parts)."""
    d6 = head_dim // 6
    n_h = n_w = d6
    n_t = head_dim // 2 - n_h - n_w
    return n_t, n_h, n_w


def rope3d_table(frame_idx: int, P: int, num_special: int, grid_w: int, head_dim: int,
                 theta: float = 10000.0) -> np.ndarray:
    """(cos, sin) table [P, D/2, 2] of one frame.  Token k of the frame sits at
    (t, h, w) = (frame_idx, (k - s) // grid_w, (k - s) % grid_w) for patch tokens
    (k >= s = num_special) and at (frame_idx, 0, 0) for special tokens.  Pair j of
    an axis band with n pairs rotates by pos * theta^(-j / n)."""
    n_t, n_h, n_w = rope3d_bands(head_dim)
    ang = np.zeros((P, head_dim // 2), dtype=np.float64)
    for k in range(P):
        if k < num_special:
            t, h, w = frame_idx, 0, 0
        else:
            t, h, w = frame_idx, (k - num_special) // grid_w, (k - num_special) % grid_w
        off = 0
        for pos, n in ((t, n_t), (h, n_h), (w, n_w)):
            for j in range(n):
                ang[k, off + j] = pos * theta ** (-j / n)
            off += n
    return np.stack([np.cos(ang), np.sin(ang)], axis=-1)
