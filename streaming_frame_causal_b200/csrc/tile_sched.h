// tile_sched.h -- the block-sparse tile schedule, shared verbatim by the host (for the
// exported inspection functions and launch sizing) and the device (each CTA
// decodes its own work item from blockIdx with these functions).
//
// Visible set ("Sliding Window Attention Mechanism in AggregatorStream", section
// "Mask Generation in CausalAttention"): query frame i sees key frames
// [max(0, i - W_f + 1), i] with W_f = sliding_window_size * num_frame_per_block
// (no window when sliding_window_size <= 0), plus the retained scale frames
// [0, min(S, i+1)) ("KV Cache Eviction Strategy": those frames are never
// evicted).  Both pieces are contiguous runs of tokens, so a query frame's keys
// are at most two token intervals; they are cut into 128-token key tiles and no
// tile outside them is ever generated.
#pragma once
#include <cstdint>

#if defined(__CUDACC__)
#define SWA_HD __host__ __device__ __forceinline__
#else
#define SWA_HD inline
#endif

namespace swa {

constexpr int kTileRows = 128;  // query rows and key rows per tile

SWA_HD int imin(int a, int b) { return a < b ? a : b; }
SWA_HD int imax(int a, int b) { return a > b ? a : b; }
SWA_HD int cdiv(int a, int b) { return (a + b - 1) / b; }

SWA_HD int window_frames(int sliding_window_size, int num_frame_per_block) {
  return sliding_window_size <= 0 ? 0 : sliding_window_size * num_frame_per_block;
}

// Key-frame intervals [lo, hi) visible to query frame i; returns 1 or 2.
SWA_HD int frame_intervals(int i, int Wf, int S, int* lo, int* hi) {
  const int wlo = (Wf <= 0) ? 0 : imax(0, i - Wf + 1);
  const int send = imin(S, i + 1);
  if (send >= wlo) {
    lo[0] = 0;
    hi[0] = i + 1;
    return 1;
  }
  if (send <= 0) {
    lo[0] = wlo;
    hi[0] = i + 1;
    return 1;
  }
  lo[0] = 0;
  hi[0] = send;
  lo[1] = wlo;
  hi[1] = i + 1;
  return 2;
}

// Number of 128-row query tiles in a frame of P tokens, and tile pairs.
SWA_HD int qtiles_per_frame(int P) { return cdiv(P, kTileRows); }
SWA_HD int qpairs_per_frame(int P) { return cdiv(qtiles_per_frame(P), 2); }

// Prefill work item w (launch order = longest first: the visible key count is
// non-decreasing in the frame index, so frames go last to first; within a
// frame the tile pairs of one head are adjacent so they share K/V in L2).
struct PrefillItem {
  int b, h, f, pair;
};
SWA_HD PrefillItem prefill_item(int64_t w, int B, int H, int F, int n_pairs) {
  const int64_t per_f = static_cast<int64_t>(B) * H * n_pairs;
  PrefillItem it;
  it.f = F - 1 - static_cast<int>(w / per_f);
  int64_t rem = w % per_f;
  it.b = static_cast<int>(rem / (static_cast<int64_t>(H) * n_pairs));
  rem %= static_cast<int64_t>(H) * n_pairs;
  it.h = static_cast<int>(rem / n_pairs);
  it.pair = static_cast<int>(rem % n_pairs);
  return it;
}

// Query rows of tile t (0-based within the frame) of a frame of P tokens.
SWA_HD int qtile_rows(int P, int t) { return imax(0, imin(kTileRows, P - t * kTileRows)); }

// Token-band work item: a 128-row query tile and a pair of query heads of one
// KV group (or a single head when the group size is odd).  Longest first:
// later tiles see at least as many keys.
struct BandItem {
  int b, kvh, h0, h1, t;  // h1 < 0: single head
};
SWA_HD BandItem band_item(int64_t w, int B, int Hq, int Hkv, int n_qtiles) {
  const int G = Hq / Hkv;
  const int per_group = (G % 2 == 0) ? G / 2 : G;
  const int64_t per_t = static_cast<int64_t>(B) * Hkv * per_group;
  BandItem it;
  it.t = n_qtiles - 1 - static_cast<int>(w / per_t);
  int64_t rem = w % per_t;
  it.b = static_cast<int>(rem / (static_cast<int64_t>(Hkv) * per_group));
  rem %= static_cast<int64_t>(Hkv) * per_group;
  it.kvh = static_cast<int>(rem / per_group);
  const int j = static_cast<int>(rem % per_group);
  if (G % 2 == 0) {
    it.h0 = it.kvh * G + 2 * j;
    it.h1 = it.h0 + 1;
  } else {
    it.h0 = it.kvh * G + j;
    it.h1 = -1;
  }
  return it;
}

// Keys of a band query tile starting at token t0 with ``rows`` rows:
// [max(0, t0 - W + 1), t0 + rows).
SWA_HD void band_keys(int t0, int rows, int W, int* lo, int* hi) {
  *lo = imax(0, t0 - W + 1);
  *hi = t0 + rows;
}

// Streaming attend work item: (split, head, query-tile pair); pairs of a head
// are adjacent so they share the cache tiles in L2.
struct StreamItem {
  int split, h, pair;
};
SWA_HD StreamItem stream_item(int64_t w, int H, int n_pairs) {
  StreamItem it;
  const int64_t per = static_cast<int64_t>(H) * n_pairs;
  it.split = static_cast<int>(w / per);
  const int64_t rem = w % per;
  it.h = static_cast<int>(rem / n_pairs);
  it.pair = static_cast<int>(rem % n_pairs);
  return it;
}

// Balanced split of T key tiles into ``splits`` contiguous ranges.
SWA_HD void split_range(int T, int splits, int s, int* t0, int* t1) {
  *t0 = static_cast<int>((static_cast<int64_t>(T) * s) / splits);
  *t1 = static_cast<int>((static_cast<int64_t>(T) * (s + 1)) / splits);
}

// ---------------------------------------------------------------- streaming
// Pure bookkeeping of the rolling paged cache (the device writes it into the
// per-layer metadata block; the host uses it only to size launches).
SWA_HD int stream_slot(int i, int S, int Wc) {
  if (Wc <= 0 || i < S) return i;
  return S + (i % Wc);
}
// Frame evicted when frame i is appended, or -1.
SWA_HD int stream_evicted(int i, int S, int Wc) {
  if (Wc <= 0) return -1;
  return (i >= S + Wc) ? (i - Wc) : -1;
}
// Frames retained after appending frame i: [0, min(S, i+1)) and [wlo, i].
SWA_HD int stream_window_lo(int i, int S, int Wc) {
  if (Wc <= 0) return imin(S, i + 1);
  return imax(imin(S, i + 1), i - Wc + 1);
}
SWA_HD int stream_retained(int i, int S, int Wc) {
  return imin(S, i + 1) + (i + 1 - stream_window_lo(i, S, Wc));
}
// Evicted frames so far (after appending frame i).
SWA_HD int stream_n_evicted(int i, int S, int Wc) {
  if (Wc <= 0) return 0;
  return imax(0, i - (S + Wc) + 1);
}

}  // namespace swa
