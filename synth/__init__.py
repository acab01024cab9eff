"""Seeded synthetic inputs shared by the oracle tests, the GPU parity tests and bench.py.

This module only draws numbers.  It holds none of the attention arithmetic: no
masks, no softmax, no cache bookkeeping.  Both sides of every parity check (the
float64 oracle under ``oracle/`` and the CUDA library) read the tensors returned
here, so they see bit-identical inputs.

Workload shapes follow the pages' examples:
  * lingbot-map frames are 518x378 images at patch 14 -> 37*27 = 999 patch tokens
    plus 1 camera and 4 register tokens, P = 1004 tokens per frame, C = 1024,
    16 heads of 64 (AggregatorStream guide; FlashInferBlock.forward signature,
    ``num_register_tokens=4``);
  * the Mistral-style token window is W = 4096 with grouped-query attention
    (sliding-window attention explainer, Mistral 7B paragraph).

All generators use ``torch.Generator('cpu')`` so the values do not depend on the
GPU.  bf16 tensors are produced by rounding a float32 draw to bfloat16 (round to
nearest even, torch's ``.to``).
"""
from __future__ import annotations

import torch

# ---------------------------------------------------------------- constants
P_FRAME = 1004          # 1 camera + 4 register + 37*27 patch tokens
NUM_SPECIAL = 5         # camera + 4 register tokens lead every frame
C_MODEL = 1024
HEADS = 16
HEAD_DIM = 64


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def normal(shape, seed: int, dtype=torch.float32) -> torch.Tensor:
    """i.i.d. N(0,1) draw, rounded to ``dtype``."""
    x = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    return x.to(dtype)


def tiny_qkv(seed: int = 0, B: int = 1, F: int = 8, P: int = 21, H: int = 2, D: int = 32,
             dtype=torch.float32):
    """Tiny check workload: q, k, v ~ N(0,1) of shape [B, F*P, H, D].

    Default shape: 8 frames of 21 tokens (1 camera + 4 register + 16 patch),
    2 heads of 32, float32.
    """
    g = _gen(seed)
    shape = (B, F * P, H, D)
    q = torch.randn(*shape, generator=g, dtype=torch.float32).to(dtype)
    k = torch.randn(*shape, generator=g, dtype=torch.float32).to(dtype)
    v = torch.randn(*shape, generator=g, dtype=torch.float32).to(dtype)
    return q, k, v


def projected_qkv(seed: int = 0, F: int = 32, P: int = P_FRAME, C: int = C_MODEL,
                  H: int = HEADS, std: float = 0.02, dtype=torch.bfloat16):
    """Prefill workload: Q/K/V = LayerNorm(x) @ W_{q,k,v}, x ~ N(0,1) [F*P, C],
    W ~ N(0, std^2) [C, C]; LayerNorm without affine parameters, eps 1e-5.

    Returns q, k, v of shape [1, F*P, H, C//H] in ``dtype``.  The projection is
    input synthesis (it shapes the value distribution like a real layer's),
    not part of the attention path.
    """
    g = _gen(seed)
    N = F * P
    x = torch.randn(N, C, generator=g, dtype=torch.float32)
    w = [torch.randn(C, C, generator=g, dtype=torch.float32) * std for _ in range(3)]
    x = torch.nn.functional.layer_norm(x, (C,), eps=1e-5)
    out = []
    for wi in w:
        y = (x @ wi).reshape(1, N, H, C // H).to(dtype)
        out.append(y.contiguous())
    return tuple(out)


def stream_frame(frame_idx: int, P: int = P_FRAME, H: int = HEADS, D: int = HEAD_DIM,
                 dtype=torch.bfloat16, base_seed: int = 0):
    """One streaming frame: q, k, v ~ N(0,1) of shape [P, H, D], seeded by the
    frame index (plus ``base_seed`` so layers can differ)."""
    g = _gen(base_seed * 1_000_003 + frame_idx)
    q = torch.randn(P, H, D, generator=g, dtype=torch.float32).to(dtype)
    k = torch.randn(P, H, D, generator=g, dtype=torch.float32).to(dtype)
    v = torch.randn(P, H, D, generator=g, dtype=torch.float32).to(dtype)
    return q, k, v


def band_qkv(seed: int = 1, N: int = 32768, Hq: int = 32, Hkv: int = 8, D: int = 128,
             dtype=torch.bfloat16):
    """Token-window GQA prefill workload: Q [1,N,Hq,D], K,V [1,N,Hkv,D] ~ N(0,1)."""
    g = _gen(seed)
    q = torch.randn(1, N, Hq, D, generator=g, dtype=torch.float32).to(dtype)
    k = torch.randn(1, N, Hkv, D, generator=g, dtype=torch.float32).to(dtype)
    v = torch.randn(1, N, Hkv, D, generator=g, dtype=torch.float32).to(dtype)
    return q, k, v


def decode_inputs(seed: int = 1, B: int = 64, W: int = 4096, Hq: int = 32, Hkv: int = 8,
                  D: int = 128, dtype=torch.bfloat16):
    """Single-token GQA decode workload against a fully populated rolling cache.

    Returns q [B,Hq,D], k_new, v_new [B,Hkv,D], k_cache, v_cache [B,W,Hkv,D].
    """
    g = _gen(seed)
    k_cache = torch.randn(B, W, Hkv, D, generator=g, dtype=torch.float32).to(dtype)
    v_cache = torch.randn(B, W, Hkv, D, generator=g, dtype=torch.float32).to(dtype)
    q = torch.randn(B, Hq, D, generator=g, dtype=torch.float32).to(dtype)
    k_new = torch.randn(B, Hkv, D, generator=g, dtype=torch.float32).to(dtype)
    v_new = torch.randn(B, Hkv, D, generator=g, dtype=torch.float32).to(dtype)
    return q, k_new, v_new, k_cache, v_cache


def growing_scores_qkv(seed: int = 7, P: int = 1000, H: int = 2, D: int = 64, steps=None,
                       q_scale: float = 4.0, noise: float = 0.05, dtype=torch.bfloat16):
    """One frame of P tokens whose key tiles (128 keys each) carry a rising common
    component, so a query row's largest score moves up from key tile to key tile.

    Every query row is ``q_scale`` times the all-ones vector, with the sign
    alternating between rows (even rows +, odd rows -).  Key rows are
    ``beta[t] / sqrt(D)`` times the all-ones vector plus ``noise`` times a normal
    draw, where t is the key's 128-token tile and ``beta`` the running sum of
    ``steps`` (default: eleven steps of 10 and one of 100, in units of
    log2(e)-scaled scores, converted here to raw values).  Values are normal.
    The tensors are [1, P, H, D].
    """
    if steps is None:
        steps = [10.0] * 5 + [100.0] + [10.0] * 6
    g = _gen(seed)
    # raw score of a +row against tile t is q_scale * sqrt(D) * beta[t]; choose beta so
    # that score * log2(e) / sqrt(D) rises by steps[t] from tile t-1 to tile t
    log2e = 1.4426950408889634
    unit = q_scale * log2e  # log2-scaled score per unit of beta
    beta = []
    acc = 0.0
    n_tiles = (P + 127) // 128
    for t in range(n_tiles):
        if t > 0:
            acc += steps[(t - 1) % len(steps)] / unit
        beta.append(acc)
    sign = torch.where(torch.arange(P) % 2 == 0, 1.0, -1.0).view(1, P, 1, 1)
    q = (q_scale * sign * torch.ones(1, P, H, D))
    tile_beta = torch.tensor([beta[i // 128] for i in range(P)], dtype=torch.float32).view(1, P, 1, 1)
    k = tile_beta / (D ** 0.5) * torch.ones(1, P, H, D) + noise * torch.randn(1, P, H, D, generator=g)
    v = torch.randn(1, P, H, D, generator=g)
    return q.to(dtype), k.to(dtype), v.to(dtype)


def prologue_inputs(seed: int = 3, P: int = P_FRAME, C: int = C_MODEL, heads: int = HEADS,
                    x_dtype=torch.bfloat16):
    """Inputs of one frame's attention prologue: tokens x [P, C] ~ N(0, 1) (bf16),
    norm weights ~ 1 + N(0, 0.1^2) and biases ~ N(0, 0.1^2) (f32), w_qkv [3C, C] ~
    N(0, 1/C) (bf16), b_qkv ~ N(0, 0.02^2) (f32), and a rotation table rot
    [P, D/2, 2] = (cos, sin) of angle p * 100^(-i/(D/2)) for token p and pair i
    (f32).  Returns a dict of CPU tensors."""
    g = _gen(seed)
    D = C // heads
    r = lambda *s: torch.randn(*s, generator=g, dtype=torch.float32)
    ang = torch.arange(P, dtype=torch.float64)[:, None] * (100.0 ** (-torch.arange(D // 2, dtype=torch.float64)
                                                                     / (D // 2)))[None, :]
    rot = torch.stack([torch.cos(ang), torch.sin(ang)], dim=-1).to(torch.float32)
    return {
        "x": r(P, C).to(x_dtype),
        "ln_w": 1 + 0.1 * r(C), "ln_b": 0.1 * r(C),
        "w_qkv": (r(3 * C, C) / C ** 0.5).to(torch.bfloat16), "b_qkv": 0.02 * r(3 * C),
        "qn_w": 1 + 0.1 * r(D), "qn_b": 0.1 * r(D),
        "kn_w": 1 + 0.1 * r(D), "kn_b": 0.1 * r(D),
        "rot": rot.contiguous(),
    }
