"""Float64 CPU oracle (test infrastructure only; see ``oracle.attention``).

Only tests, the smoke check and the CPU-baseline leg of the benchmark import it;
the CUDA library neither imports nor links anything here.
"""
from .attention import (  # noqa: F401
    band_attention, band_mask, decode, decode_slot, frame_mask, frame_visible,
    prefill, softmax_attention, StreamCache, window_frames,
)
