// cache.cu -- device-side append + eviction for the rolling paged KV cache.
//
// Rule ("Sliding Window Attention Mechanism in AggregatorStream", section "KV
// Cache Eviction Strategy"): after frame i is appended, when more than
// window + scale frames are cached, cache positions [scale, n - window) leave,
// i.e. the single oldest non-scale frame i - window.  With
// kv_cache_cross_frame_special (same page, FAQ "Can special tokens persist
// outside the sliding window?") that frame's leading special tokens (camera,
// registers) move to a packed special region first.  Frame i lives in slot i
// (scale frame) or scale + (i mod window) -- the rolling-buffer rule "slot i
// modulo W" of the sliding-window explainer, applied to frames -- so the new
// frame lands exactly on the slot it frees.  Eviction happens before the
// attention kernel runs (same page: evict before attention).
//
// One launch does everything: each 16-byte chunk of the new frame is copied by
// one thread; the thread whose chunk overlaps the evicted frame's special
// tokens first moves the old chunk to the special region, so nothing races.
// Block 0 rewrites the layer's metadata (slot map, page table, key segments,
// counters) -- all pure functions of the frame index.
#include <cuda_runtime.h>
#include <cstdint>

#include "internal.h"
#include "exp2_poly.cuh"
#include "ptx.cuh"
#include "tile_sched.h"

namespace swa {
namespace {

__global__ void __launch_bounds__(256) append_evict_kernel(const AppendParams p) {
  const int i = p.frame;
  const int slot = stream_slot(i, p.S, p.Wc);
  const int ev = stream_evicted(i, p.S, p.Wc);
  const int chunks = p.row_bytes >> 4;
  const int64_t per_tensor = static_cast<int64_t>(p.P) * chunks;
  const int64_t slot_row0 = static_cast<int64_t>(slot) * p.ppf * p.page_tokens;
  const int64_t special_row0 = static_cast<int64_t>(p.n_slots) * p.ppf * p.page_tokens;
  const bool move_special = (ev >= 0) && p.cross_special;

  // 16-byte chunks, four per thread with their loads issued before the stores;
  // a frame is at most 2^31 chunks, so 32-bit indices
  const int n = static_cast<int>(2 * per_tensor);
  const int stride = static_cast<int>(gridDim.x * blockDim.x);
  for (int base = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x); base < n; base += 4 * stride) {
    uint4 v[4];
    uint4* dst[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int idx = base + k * stride;
      dst[k] = nullptr;
      if (idx >= n) continue;
      const int tsel = idx >= per_tensor;
      const int rem = idx - (tsel ? static_cast<int>(per_tensor) : 0);
      const int row = rem / chunks;
      const int ch = rem - row * chunks;
      uint8_t* store = tsel ? p.v_store : p.k_store;
      dst[k] = reinterpret_cast<uint4*>(store + (slot_row0 + row) * p.row_bytes) + ch;
      if (move_special && row < p.num_special) {
        const int64_t sp_row = special_row0 + static_cast<int64_t>(ev - p.S) * p.num_special + row;
        reinterpret_cast<uint4*>(store + sp_row * p.row_bytes)[ch] = *dst[k];
      }
      if (p.copy) {
        const uint8_t* src = tsel ? p.v_src : p.k_src;
        v[k] = reinterpret_cast<const uint4*>(src + p.src_off + static_cast<int64_t>(row) * p.src_row_bytes)[ch];
      }
    }
    if (p.copy) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (dst[k]) *dst[k] = v[k];
    }
  }

  // ---------------------------------------------------------------- metadata
  // every thread of the grid takes a share of the page table, the key runs and
  // the slot map (the table has ~4,500 entries at 72 frames of 63 pages), so no
  // single block is left with it after the copy
  int* hdr = p.meta;
  int* slot_frame = p.meta + p.off_slot_frame;
  int* pages = p.meta + p.off_page_table;
  int* seg_row = p.meta + p.off_seg_row;
  int* seg_len = p.meta + p.off_seg_len;
  const int n_scale = imin(p.S, i + 1);
  const int wlo = stream_window_lo(i, p.S, p.Wc);
  const int n_ret = stream_retained(i, p.S, p.Wc);
  const int n_ev = stream_n_evicted(i, p.S, p.Wc);
  const int n_special = p.cross_special ? n_ev * p.num_special : 0;
  const int sp_pages = cdiv(n_special, p.page_tokens);
  const int n_pages = n_ret * p.ppf + sp_pages;
  const int n_segs = n_ret + (n_special > 0 ? 1 : 0);
  if (n_pages > p.max_pages || n_segs > p.max_segs) {
    if (blockIdx.x == 0 && threadIdx.x == 0) latch_error(p.err, ERR_BAD_META);
    return;
  }
  const int gt = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x);
  const int gn = static_cast<int>(gridDim.x * blockDim.x);
  // retained frame with ordinal o (ascending frame index)
  auto ret_frame = [&](int o) { return o < n_scale ? o : wlo + (o - n_scale); };
  for (int e = gt; e < n_ret * p.ppf; e += gn) {
    const int o = e / p.ppf;
    const int pg = e - o * p.ppf;
    pages[e] = stream_slot(ret_frame(o), p.S, p.Wc) * p.ppf + pg;
  }
  for (int e = gt; e < sp_pages; e += gn) pages[n_ret * p.ppf + e] = p.n_slots * p.ppf + e;
  for (int o = gt; o < n_ret; o += gn) {
    seg_row[o] = stream_slot(ret_frame(o), p.S, p.Wc) * p.ppf * p.page_tokens;
    seg_len[o] = p.P;
  }
  if (gt == 0 && n_special > 0) {
    seg_row[n_ret] = p.n_slots * p.ppf * p.page_tokens;
    seg_len[n_ret] = n_special;
  }
  // slot map: which frame each slot holds after this append
  for (int s = gt; s < p.n_slots; s += gn) {
    int f = -1;
    if (p.Wc <= 0 || s < p.S) {
      f = (s <= i) ? s : -1;
    } else {
      const int r = s - p.S;  // residue of frames mapped here
      if (i >= r) {
        const int j = i - ((i - r) % p.Wc);  // latest frame <= i with j mod Wc == r
        f = (j >= wlo && j >= p.S) ? j : -1;
      }
    }
    slot_frame[s] = f;
  }
  if (gt == 0) {
    hdr[0] = i + 1;
    hdr[1] = n_ev;
    hdr[2] = n_special;
    hdr[3] = ev;
    hdr[4] = n_pages;
    hdr[5] = n_segs;
    hdr[6] = n_ret;
    hdr[7] = 0;
  }
}

// Non-keyframe attend ("Non-keyframe path" of the streaming block in the same
// guide: append with eviction deferred, attend, roll back): the frame's K/V are
// written to the scratch frame's pages, which no persistent page table lists,
// and the layer's non-keyframe area receives the persistent key runs followed by
// the scratch run.  Nothing persistent is written, so the roll-back is free.
__global__ void __launch_bounds__(256) transient_prepare_kernel(const TransientParams p) {
  const int chunks = p.row_bytes >> 4;
  const int per_tensor = p.P * chunks;  // the host keeps 2 * per_tensor below 2^31
  const int64_t row0 = static_cast<int64_t>(p.scratch_page) * p.page_tokens;
  // 16-byte chunks, four per thread with their loads issued before the stores
  const int n_chunks = 2 * per_tensor;
  const int stride = static_cast<int>(gridDim.x * blockDim.x);
  for (int base = static_cast<int>(blockIdx.x * blockDim.x + threadIdx.x); base < n_chunks; base += 4 * stride) {
    uint4 v[4];
    uint4* dst[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int idx = base + k * stride;
      dst[k] = nullptr;
      if (idx >= n_chunks) continue;
      const int tsel = idx >= per_tensor;
      const int rem = idx - (tsel ? per_tensor : 0);
      const int row = rem / chunks;
      const int ch = rem - row * chunks;
      dst[k] = reinterpret_cast<uint4*>((tsel ? p.v_store : p.k_store) + (row0 + row) * p.row_bytes) + ch;
      v[k] = reinterpret_cast<const uint4*>((tsel ? p.v_src : p.k_src) + static_cast<int64_t>(row) * p.row_bytes)[ch];
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (dst[k]) *dst[k] = v[k];
  }
  if (blockIdx.x != 0) return;
  const int* hdr = p.meta;
  int* th = p.meta + p.t_off;
  int* trow = th + 8;
  int* tlen = trow + (p.max_segs + 1);
  int n = hdr[5];
  if (n < 0 || n > p.max_segs) {
    if (threadIdx.x == 0) latch_error(p.err, ERR_BAD_META);
    n = 0;
  }
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    trow[e] = hdr[p.off_seg_row + e];
    tlen[e] = hdr[p.off_seg_len + e];
  }
  if (threadIdx.x == 0) {
    trow[n] = static_cast<int>(row0);
    tlen[n] = p.P;
    for (int e = 0; e < 8; ++e) th[e] = hdr[e];
    th[5] = n + 1;
  }
}

__global__ void debug_wait_kernel(int* err, long long timeout_ns) {
  // waits on a flag that nothing sets; gives up after timeout_ns and latches
  // the error -- the same bounded-wait contract every kernel follows
  __shared__ int flag;
  flag = 0;
  __syncthreads();
  const uint64_t t0 = global_timer_ns();
  while (*reinterpret_cast<volatile int*>(&flag) == 0) {
    if (global_timer_ns() - t0 > static_cast<uint64_t>(timeout_ns)) {
      latch_error(err, ERR_WAIT_DEBUG);
      return;
    }
  }
}

__global__ void exp2_poly_kernel(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], 0.f)).x;
  }
}

}  // namespace

cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t stream) {
  const int pairs = (n + 1) / 2;
  if (pairs == 0) return cudaSuccess;
  exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(x, y, n);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_append_evict(const AppendParams& p, cudaStream_t stream) {
  const int64_t work = 2LL * p.P * (p.row_bytes >> 4);
  if (work > 0x7fffffffLL) return cudaErrorInvalidValue;  // the kernel indexes chunks in 32 bits
  int64_t blocks = (work + 1023) / 1024;  // four chunks per thread
  if (blocks < 1) blocks = 1;
  if (blocks > 4096) blocks = 4096;
  append_evict_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_transient_prepare(const TransientParams& p, cudaStream_t stream) {
  const int64_t work = 2LL * p.P * (p.row_bytes >> 4);
  if (work > 0x7fffffffLL) return cudaErrorInvalidValue;  // the kernel indexes chunks in 32 bits
  int64_t blocks = (work + 1023) / 1024;  // four chunks per thread
  if (blocks < 1) blocks = 1;
  if (blocks > 4096) blocks = 4096;
  transient_prepare_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_debug_wait(int* err, long long timeout_ns, cudaStream_t stream) {
  debug_wait_kernel<<<1, 1, 0, stream>>>(err, timeout_ns);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swa
