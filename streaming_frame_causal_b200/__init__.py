"""Python binding of libswa_b200.so (frame-causal sliding-window attention on B200).

Argument marshalling only: every function forwards tensor data pointers, sizes
and the current CUDA stream to the C ABI of ``include/swa.h`` under the same
name, and raises :class:`SwaError` on a non-zero status.  All arithmetic runs
in the library's CUDA kernels; there is no fallback.  Importing this module
fails if the library has not been built (``python
streaming_frame_causal_b200/build.py``).

Tensor layouts follow the pages' contracts: tokens [B, S*P, heads, head_dim]
(the [B*S, P, C] layout with C = heads*head_dim), streaming frames
[P, heads, head_dim], decode tensors [B, heads, head_dim] and caches
[B, W, Hkv, head_dim].
"""
from __future__ import annotations

import ctypes as C
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libswa_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "swa.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python streaming_frame_causal_b200/build.py`")
_lib = C.CDLL(LIB_PATH)

SWA_F32, SWA_BF16 = 0, 1
STATUS = {0: "SWA_OK", -1: "SWA_ERR_ARG", -2: "SWA_ERR_SHAPE", -3: "SWA_ERR_ORDER",
          -4: "SWA_ERR_CAPACITY", -5: "SWA_ERR_CUDA", -6: "SWA_ERR_TIMEOUT", -7: "SWA_ERR_UNSUPPORTED"}


class SwaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({_lib.swa_status_str(status).decode()})")


class swa_stream_cfg(C.Structure):
    _fields_ = [(n, C.c_int) for n in (
        "num_layers", "heads", "head_dim", "P", "scale_frames", "window_frames", "page_tokens",
        "cross_frame_special", "num_special", "max_frames", "dtype", "max_splits")]


class swa_meta_host(C.Structure):
    _fields_ = [(n, C.c_int) for n in (
        "n_frames", "n_evicted", "n_special_tokens", "n_pages", "n_segs", "n_retained", "n_slots",
        "n_last_evicted", "last_evicted")] + [
        ("slot_frame", C.POINTER(C.c_int32)), ("slot_cap", C.c_int),
        ("page_table", C.POINTER(C.c_int32)), ("page_cap", C.c_int),
        ("seg_row", C.POINTER(C.c_int32)), ("seg_len", C.POINTER(C.c_int32)), ("seg_cap", C.c_int)]


class swa_meta_layout(C.Structure):
    _fields_ = [(n, C.c_int) for n in (
        "n_ints", "n_slots", "pages_per_frame", "max_pages", "max_segs", "off_slot_frame",
        "off_page_table", "off_seg_row", "off_seg_len")]


_vp, _i, _i64, _sz = C.c_void_p, C.c_int, C.c_int64, C.c_size_t
_sigs = {
    "swa_status_str": (C.c_char_p, [_i]),
    "swa_version": (_i, []),
    "swa_sched_frame_intervals": (_i, [_i, _i, _i, _i, C.POINTER(_i), C.POINTER(_i)]),
    "swa_sched_prefill": (_i64, [_i, _i, _i, _i, _i, _i, _i, _vp, _i64]),
    "swa_sched_decode": (_i, [_i, _i, _i, C.c_longlong, _i, _vp]),
    "swa_sched_stream": (_i, [_i, _i, _i, _i, _i, _vp]),
    "swa_prefill": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "swa_prefill_heads": (_i, [_vp, _vp, _vp, _vp] + [_i] * 11 + [_vp]),
    "swa_stream_append_evict_heads": (_i, [_vp, _i, _i, _vp, _vp, _i, _i, _vp]),
    "swa_stream_attend_heads": (_i, [_vp, _i, _i, _vp, _vp, _i, _i, _vp]),
    "swa_stream_cache_bytes": (_sz, [C.POINTER(swa_stream_cfg)]),
    "swa_stream_init": (_i, [C.POINTER(_vp), C.POINTER(swa_stream_cfg), _vp, _sz, _vp]),
    "swa_stream_bytes": (_sz, [C.POINTER(swa_stream_cfg)]),
    "swa_stream_create": (_i, [C.POINTER(_vp), C.POINTER(swa_stream_cfg), _vp, _sz, _vp]),
    "swa_stream_destroy": (None, [_vp]),
    "swa_stream_reset": (_i, [_vp, _vp]),
    "swa_stream_append_evict": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
    "swa_stream_attend": (_i, [_vp, _i, _i, _vp, _vp, _vp]),
    "swa_stream_attend_transient": (_i, [_vp, _i, _vp, _vp, _vp, _vp, _vp]),
    "swa_attn_pre": (_i, [_vp] * 10 + [_i, _i, _i, C.c_float] + [_vp] * 5),
    "swa_stream_append_evict_pre": (_i, [_vp, _i, _i] + [_vp] * 10 + [C.c_float] + [_vp] * 3),
    "swa_rope3d_table": (_i, [_i, _i, _i, _i, _i, C.c_double, _vp, _vp]),
    "swa_attn_pre_rope3d": (_i, [_vp] * 9 + [_i, _i, _i, C.c_double, _i, _i, _i, C.c_float] + [_vp] * 5),
    "swa_stream_append_evict_pre_rope3d": (_i, [_vp, _i, _i] + [_vp] * 9 + [_i, _i, C.c_double, C.c_float]
                                           + [_vp] * 3),
    "swa_stream_meta_layout": (_i, [_vp, C.POINTER(swa_meta_layout)]),
    "swa_stream_get_meta": (_i, [_vp, _i, C.POINTER(swa_meta_host), _vp]),
    "swa_stream_get_meta_raw": (_i, [_vp, _i, _vp, _sz, _vp]),
    "swa_stream_k_storage": (_vp, [_vp, _i]),
    "swa_stream_v_storage": (_vp, [_vp, _i]),
    "swa_band_prefill": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "swa_decode_workspace_bytes": (_sz, [_i, _i, _i, _i, _i]),
    "swa_decode": (_i, [_vp, _vp, _vp, _vp, _vp, C.c_longlong, _i, _i, _i, _i, _i, _vp, _vp, _sz,
                        _i, _vp]),
    "swa_decode_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, C.c_longlong, _i, _i, _i, _i, _i, _vp, _i, _vp]),
    "swa_launch_count": (C.c_uint64, []),
    "swa_device_error_check": (_i, [_vp]),
    "swa_debug_wait_timeout": (_i, [_i, _vp]),
    "swa_debug_exp2_poly": (_i, [_vp, _vp, _i, _vp]),
}
for _name, (_res, _args) in _sigs.items():
    try:
        _f = getattr(_lib, _name)
    except AttributeError as _e:
        raise ImportError(f"{LIB_PATH} is stale (no {_name}); rebuild it") from _e
    _f.restype = _res
    _f.argtypes = _args


def header_functions() -> list[str]:
    """Names of every function include/swa.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(swa_[a-z0-9_]+)\s*\(", text)))


def _check(status: int, where: str) -> None:
    if status != 0:
        raise SwaError(status, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SWA_BF16
    if t.dtype == torch.float32:
        return SWA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


# --------------------------------------------------------------- scheduler
def swa_sched_frame_intervals(i: int, sliding_window_size: int, num_frame_per_block: int,
                              num_frame_for_scale: int) -> list[tuple[int, int]]:
    lo = (C.c_int * 2)()
    hi = (C.c_int * 2)()
    n = _lib.swa_sched_frame_intervals(i, sliding_window_size, num_frame_per_block, num_frame_for_scale,
                                       lo, hi)
    if n < 0:
        raise SwaError(n, "swa_sched_frame_intervals")
    return [(lo[j], hi[j]) for j in range(n)]


def swa_sched_prefill(B: int, S: int, P: int, heads: int, sliding_window_size: int,
                      num_frame_per_block: int, num_frame_for_scale: int):
    """Prefill work list as an int32 numpy array [items, 8] (see include/swa.h)."""
    import numpy as np
    n = _lib.swa_sched_prefill(B, S, P, heads, sliding_window_size, num_frame_per_block,
                               num_frame_for_scale, None, 0)
    if n < 0:
        raise SwaError(int(n), "swa_sched_prefill")
    out = np.zeros((n, 8), dtype=np.int32)
    _lib.swa_sched_prefill(B, S, P, heads, sliding_window_size, num_frame_per_block, num_frame_for_scale,
                           out.ctypes.data, n)
    return out


def swa_sched_decode(B: int, Hkv: int, W: int, pos: int, sms: int = 148) -> dict:
    """The decode's launch plan (see include/swa.h)."""
    out = (C.c_int * 5)()
    _check(_lib.swa_sched_decode(B, Hkv, W, pos, sms, out), "swa_sched_decode")
    return {"pieces": out[0], "piece_len": out[1], "grid": out[2], "slots": out[3], "n_valid": out[4]}


def swa_sched_stream(key_tiles: int, heads: int, P: int, max_splits: int = 12, sms: int = 148) -> dict:
    """The streaming attend's launch plan (see include/swa.h)."""
    out = (C.c_int * 4)()
    _check(_lib.swa_sched_stream(key_tiles, heads, P, max_splits, sms, out), "swa_sched_stream")
    return {"splits": out[0], "ctas": out[1], "min_tiles": out[2], "max_tiles": out[3]}


# ---------------------------------------------------------------- prefill
def swa_prefill(q, k, v, out, S: int, P: int, sliding_window_size: int, num_frame_per_block: int = 1,
                num_frame_for_scale: int = 0, stream=None) -> torch.Tensor:
    """Frame-causal sliding-window attention; q/k/v/out [B, S*P, heads, head_dim]."""
    B, N, H, D = q.shape
    _check(_lib.swa_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, S, P, H * D, H, D,
                            sliding_window_size, num_frame_per_block, num_frame_for_scale,
                            _dtype_code(q), _stream(stream)), "swa_prefill")
    return out


def head_shard(rank: int, world: int, heads: int) -> tuple[int, int]:
    """(head0, count) of rank ``rank``'s share when ``world`` GPUs split ``heads``
    attention heads (contiguous, as even as possible, lower ranks taking the
    extra head)."""
    if world < 1 or not 0 <= rank < world or heads < world:
        raise ValueError("need 0 <= rank < world <= heads")
    base, extra = divmod(heads, world)
    return rank * base + min(rank, extra), base + (1 if rank < extra else 0)


def swa_prefill_heads(q, k, v, out, S: int, P: int, head0: int, heads: int, sliding_window_size: int,
                      num_frame_per_block: int = 1, num_frame_for_scale: int = 0, stream=None) -> torch.Tensor:
    """swa_prefill on heads [head0, head0 + heads) of q/k/v/out [B, S*P, H, D], in place."""
    B, N, H, D = q.shape
    _check(_lib.swa_prefill_heads(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, S, P, H * D, head0, heads, D,
                                  sliding_window_size, num_frame_per_block, num_frame_for_scale,
                                  _dtype_code(q), _stream(stream)), "swa_prefill_heads")
    return out


def swa_attn_pre(x, ln_w, ln_b, w_qkv, b_qkv, qn_w, qn_b, kn_w, kn_b, rot, heads: int, eps: float = 1e-6,
                 q_out=None, k_out=None, v_out=None, xn_ws=None, stream=None):
    """Attention prologue of one frame: x [P, C] bf16 -> q, k, v [P, heads, C/heads]
    bf16 (norm1, qkv linear, q/k norms, RoPE by the complex table rot [P, D/2, 2];
    the steps and layouts are those of swa_attn_pre in include/swa.h)."""
    P, Cdim = x.shape
    D = Cdim // heads
    q_out = torch.empty(P, heads, D, dtype=x.dtype, device=x.device) if q_out is None else q_out
    k_out = torch.empty(P, heads, D, dtype=x.dtype, device=x.device) if k_out is None else k_out
    v_out = torch.empty(P, heads, D, dtype=x.dtype, device=x.device) if v_out is None else v_out
    xn_ws = torch.empty_like(x) if xn_ws is None else xn_ws
    _check(_lib.swa_attn_pre(_ptr(x), _ptr(ln_w), _ptr(ln_b), _ptr(w_qkv), _ptr(b_qkv), _ptr(qn_w), _ptr(qn_b),
                             _ptr(kn_w), _ptr(kn_b), _ptr(rot), P, Cdim, heads, float(eps), _ptr(xn_ws),
                             _ptr(q_out), _ptr(k_out), _ptr(v_out), _stream(stream)), "swa_attn_pre")
    return q_out, k_out, v_out


def swa_attn_pre_rope3d(x, ln_w, ln_b, w_qkv, b_qkv, qn_w, qn_b, kn_w, kn_b, heads: int, frame_idx: int,
                        num_special: int, grid_w: int, theta: float = 10000.0, eps: float = 1e-6, q_out=None,
                        k_out=None, v_out=None, xn_ws=None, stream=None):
    """swa_attn_pre with the frame's 3-D RoPE generated inside the prologue (no
    table; positions and bands as swa_rope3d_table, see include/swa.h)."""
    P, Cdim = x.shape
    D = Cdim // heads
    q_out = torch.empty(P, heads, D, dtype=x.dtype, device=x.device) if q_out is None else q_out
    k_out = torch.empty(P, heads, D, dtype=x.dtype, device=x.device) if k_out is None else k_out
    v_out = torch.empty(P, heads, D, dtype=x.dtype, device=x.device) if v_out is None else v_out
    xn_ws = torch.empty_like(x) if xn_ws is None else xn_ws
    _check(_lib.swa_attn_pre_rope3d(_ptr(x), _ptr(ln_w), _ptr(ln_b), _ptr(w_qkv), _ptr(b_qkv), _ptr(qn_w),
                                    _ptr(qn_b), _ptr(kn_w), _ptr(kn_b), int(frame_idx), int(num_special),
                                    int(grid_w), float(theta), P, Cdim, heads, float(eps), _ptr(xn_ws),
                                    _ptr(q_out), _ptr(k_out), _ptr(v_out), _stream(stream)),
           "swa_attn_pre_rope3d")
    return q_out, k_out, v_out


def swa_rope3d_table(frame_idx: int, P: int, num_special: int, grid_w: int, head_dim: int,
                     theta: float = 10000.0, out=None, device="cuda", stream=None) -> torch.Tensor:
    """3-D RoPE table [P, head_dim/2, 2] (cos, sin) of one streaming frame, the
    ``rot`` input of swa_attn_pre (layout and readings: include/swa.h)."""
    out = torch.empty(P, head_dim // 2, 2, dtype=torch.float32, device=device) if out is None else out
    _check(_lib.swa_rope3d_table(frame_idx, P, num_special, grid_w, head_dim, float(theta), _ptr(out),
                                 _stream(stream)), "swa_rope3d_table")
    return out


def swa_band_prefill(q, k, v, out, window: int, stream=None) -> torch.Tensor:
    """Token-band GQA attention; q/out [B, N, Hq, D], k/v [B, N, Hkv, D]."""
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    _check(_lib.swa_band_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, N, Hq, Hkv, D, window,
                                 _dtype_code(q), _stream(stream)), "swa_band_prefill")
    return out


# ----------------------------------------------------------------- decode
def swa_decode_workspace_bytes(B: int, Hq: int, Hkv: int, head_dim: int, W: int) -> int:
    return int(_lib.swa_decode_workspace_bytes(B, Hq, Hkv, head_dim, W))


def swa_decode(q, k_new, v_new, k_cache, v_cache, pos: int, out, workspace=None, stream=None):
    """One token per sequence at ``pos``; caches [B, W, Hkv, D] are updated in place."""
    B, Hq, D = q.shape
    W, Hkv = k_cache.shape[1], k_cache.shape[2]
    if workspace is None:
        n = swa_decode_workspace_bytes(B, Hq, Hkv, D, W)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)
    _check(_lib.swa_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), int(pos), W,
                           B, Hq, Hkv, D, _ptr(out), _ptr(workspace), workspace.numel(),
                           _dtype_code(q), _stream(stream)), "swa_decode")
    return out


def swa_decode_noalloc(q, k_new, v_new, k_cache, v_cache, pos: int, out, stream=None):
    """swa_decode for callers that cannot allocate: bf16 only, split-K scratch taken
    from a fixed array inside the library (calls must not overlap on the GPU)."""
    B, Hq, D = q.shape
    W, Hkv = k_cache.shape[1], k_cache.shape[2]
    _check(_lib.swa_decode_noalloc(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), int(pos),
                                   W, B, Hq, Hkv, D, _ptr(out), _dtype_code(q), _stream(stream)),
           "swa_decode_noalloc")
    return out


# ----------------------------------------------------------------- errors
def swa_device_error_check(stream=None) -> int:
    """Synchronizes and returns the status of the latched device error flag (0 = none)."""
    return int(_lib.swa_device_error_check(_stream(stream)))


def swa_debug_wait_timeout(timeout_us: int, stream=None) -> None:
    _check(_lib.swa_debug_wait_timeout(int(timeout_us), _stream(stream)), "swa_debug_wait_timeout")


def swa_launch_count() -> int:
    """Kernel launches the library has issued in this process."""
    return int(_lib.swa_launch_count())


def swa_debug_exp2_poly(x, y, stream=None):
    """y = 2^x through the kernels' FMA-pipe polynomial (float32 device tensors)."""
    _check(_lib.swa_debug_exp2_poly(_ptr(x), _ptr(y), x.numel(), _stream(stream)), "swa_debug_exp2_poly")
    return y


def swa_status_str(status: int) -> str:
    return _lib.swa_status_str(int(status)).decode()


def swa_version() -> int:
    return int(_lib.swa_version())


# -------------------------------------------------------------- streaming
def _make_cfg(num_layers, heads, head_dim, P, scale_frames, window_frames, page_tokens,
              cross_frame_special, num_special, max_frames, dtype, max_splits):
    return swa_stream_cfg(num_layers, heads, head_dim, P, scale_frames, window_frames, page_tokens,
                          int(bool(cross_frame_special)), num_special, max_frames,
                          SWA_BF16 if dtype == torch.bfloat16 else SWA_F32, max_splits)


def swa_stream_cache_bytes(**cfg) -> int:
    return int(_lib.swa_stream_cache_bytes(C.byref(_make_cfg(**cfg))))


swa_stream_bytes = swa_stream_cache_bytes  # earlier name, same call


class SwaStream:
    """Rolling paged KV cache over a torch-owned device buffer (one per model)."""

    def __init__(self, num_layers: int, heads: int, head_dim: int, P: int, scale_frames: int,
                 window_frames: int, page_tokens: int = 16, cross_frame_special: bool = False,
                 num_special: int = 5, max_frames: int = 1024, dtype=torch.bfloat16, max_splits: int = 12,
                 device="cuda", stream=None):
        self.cfg = _make_cfg(num_layers, heads, head_dim, P, scale_frames, window_frames, page_tokens,
                             cross_frame_special, num_special, max_frames, dtype, max_splits)
        self.nbytes = int(_lib.swa_stream_cache_bytes(C.byref(self.cfg)))
        if self.nbytes == 0:
            raise SwaError(-1, "swa_stream_cache_bytes")
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        h = C.c_void_p()
        _check(_lib.swa_stream_init(C.byref(h), C.byref(self.cfg), self.buf.data_ptr(), self.nbytes,
                                    _stream(stream)), "swa_stream_init")
        self.handle = h
        lay = swa_meta_layout()
        _check(_lib.swa_stream_meta_layout(self.handle, C.byref(lay)), "swa_stream_meta_layout")
        self.layout = lay

    def close(self) -> None:
        if getattr(self, "handle", None):
            _lib.swa_stream_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def swa_stream_reset(self, stream=None) -> None:
        _check(_lib.swa_stream_reset(self.handle, _stream(stream)), "swa_stream_reset")

    def swa_stream_append_evict(self, global_idx: int, frame_idx: int, k_frame, v_frame, stream=None):
        _check(_lib.swa_stream_append_evict(self.handle, global_idx, frame_idx, _ptr(k_frame),
                                            _ptr(v_frame), _stream(stream)), "swa_stream_append_evict")

    def swa_stream_append_evict_heads(self, global_idx: int, frame_idx: int, k_frame, v_frame, head0: int,
                                      stream=None):
        """Append heads [head0, head0 + cfg.heads) of k_frame / v_frame [P, H, D]."""
        P, H, D = k_frame.shape
        _check(_lib.swa_stream_append_evict_heads(self.handle, global_idx, frame_idx, _ptr(k_frame), _ptr(v_frame),
                                                  H * D, head0, _stream(stream)), "swa_stream_append_evict_heads")

    def swa_stream_attend_heads(self, global_idx: int, frame_idx: int, q_frame, out, head0: int, stream=None):
        """Attend heads [head0, head0 + cfg.heads) of q_frame [P, H, D] into the same heads of out."""
        P, H, D = q_frame.shape
        _check(_lib.swa_stream_attend_heads(self.handle, global_idx, frame_idx, _ptr(q_frame), _ptr(out), H * D,
                                            head0, _stream(stream)), "swa_stream_attend_heads")
        return out

    def swa_stream_attend(self, global_idx: int, frame_idx: int, q_frame, out, stream=None):
        _check(_lib.swa_stream_attend(self.handle, global_idx, frame_idx, _ptr(q_frame), _ptr(out),
                                      _stream(stream)), "swa_stream_attend")
        return out

    def swa_stream_append_evict_pre(self, global_idx: int, frame_idx: int, x, ln_w, ln_b, w_qkv, b_qkv, qn_w,
                                    qn_b, kn_w, kn_b, rot, q_out, eps: float = 1e-6, xn_ws=None, stream=None):
        """Append frame ``frame_idx`` from its tokens x [P, C]: eviction and
        metadata, then the attention prologue with K/V written into the frame's
        slot and Q to q_out [P, heads, head_dim] (see include/swa.h)."""
        xn_ws = torch.empty_like(x) if xn_ws is None else xn_ws
        _check(_lib.swa_stream_append_evict_pre(self.handle, global_idx, frame_idx, _ptr(x), _ptr(ln_w), _ptr(ln_b),
                                                _ptr(w_qkv), _ptr(b_qkv), _ptr(qn_w), _ptr(qn_b), _ptr(kn_w),
                                                _ptr(kn_b), _ptr(rot), float(eps), _ptr(xn_ws), _ptr(q_out),
                                                _stream(stream)), "swa_stream_append_evict_pre")
        return q_out

    def swa_stream_append_evict_pre_rope3d(self, global_idx: int, frame_idx: int, x, ln_w, ln_b, w_qkv, b_qkv,
                                           qn_w, qn_b, kn_w, kn_b, q_out, num_special: int, grid_w: int,
                                           theta: float = 10000.0, eps: float = 1e-6, xn_ws=None, stream=None):
        """swa_stream_append_evict_pre with the frame's 3-D RoPE generated inside
        the prologue (see include/swa.h)."""
        xn_ws = torch.empty_like(x) if xn_ws is None else xn_ws
        _check(_lib.swa_stream_append_evict_pre_rope3d(
            self.handle, global_idx, frame_idx, _ptr(x), _ptr(ln_w), _ptr(ln_b), _ptr(w_qkv), _ptr(b_qkv),
            _ptr(qn_w), _ptr(qn_b), _ptr(kn_w), _ptr(kn_b), int(num_special), int(grid_w), float(theta),
            float(eps), _ptr(xn_ws), _ptr(q_out), _stream(stream)), "swa_stream_append_evict_pre_rope3d")
        return q_out

    def swa_stream_attend_transient(self, global_idx: int, q_frame, k_frame, v_frame, out, stream=None):
        """Non-keyframe attend: q_frame against the cache plus this frame's own
        K/V, with nothing persisted (see include/swa.h)."""
        _check(_lib.swa_stream_attend_transient(self.handle, global_idx, _ptr(q_frame), _ptr(k_frame),
                                                _ptr(v_frame), _ptr(out), _stream(stream)),
               "swa_stream_attend_transient")
        return out

    def swa_stream_get_meta(self, global_idx: int, stream=None) -> dict:
        """Layer ``global_idx``'s bookkeeping through the swa_meta_host view."""
        import numpy as np
        lay = self.layout
        slot = np.zeros(lay.n_slots, dtype=np.int32)
        pages = np.zeros(lay.max_pages, dtype=np.int32)
        srow = np.zeros(lay.max_segs, dtype=np.int32)
        slen = np.zeros(lay.max_segs, dtype=np.int32)
        ip = C.POINTER(C.c_int32)
        m = swa_meta_host()
        m.slot_frame, m.slot_cap = slot.ctypes.data_as(ip), lay.n_slots
        m.page_table, m.page_cap = pages.ctypes.data_as(ip), lay.max_pages
        m.seg_row, m.seg_len, m.seg_cap = srow.ctypes.data_as(ip), slen.ctypes.data_as(ip), lay.max_segs
        _check(_lib.swa_stream_get_meta(self.handle, global_idx, C.byref(m), _stream(stream)),
               "swa_stream_get_meta")
        return {
            "n_frames": m.n_frames, "n_evicted": m.n_evicted, "n_special": m.n_special_tokens,
            "last_evicted": m.last_evicted, "n_last_evicted": m.n_last_evicted, "n_pages": m.n_pages,
            "n_segs": m.n_segs, "n_retained": m.n_retained, "slot_frame": slot[:m.n_slots].copy(),
            "page_table": pages[:m.n_pages].copy(), "seg_row": srow[:m.n_segs].copy(),
            "seg_len": slen[:m.n_segs].copy(),
        }

    def swa_stream_get_meta_raw(self, global_idx: int, stream=None):
        """Layer ``global_idx``'s raw int32 metadata block (layout: swa_stream_meta_layout)."""
        import numpy as np
        raw = np.zeros(self.layout.n_ints, dtype=np.int32)
        _check(_lib.swa_stream_get_meta_raw(self.handle, global_idx, raw.ctypes.data, self.layout.n_ints,
                                            _stream(stream)), "swa_stream_get_meta_raw")
        return raw

    def storage(self, global_idx: int, which: str = "k") -> torch.Tensor:
        """View of a layer's K or V page storage as [rows, heads, head_dim]."""
        fn = _lib.swa_stream_k_storage if which == "k" else _lib.swa_stream_v_storage
        addr = fn(self.handle, global_idx)
        if not addr:
            raise SwaError(-4, "swa_stream_storage")
        c = self.cfg
        esize = 2 if c.dtype == SWA_BF16 else 4
        rows = (self.layout.max_pages * c.page_tokens)
        off = addr - self.buf.data_ptr()
        view = self.buf[off:off + rows * c.heads * c.head_dim * esize]
        dt = torch.bfloat16 if c.dtype == SWA_BF16 else torch.float32
        return view.view(dt).view(rows, c.heads, c.head_dim)
