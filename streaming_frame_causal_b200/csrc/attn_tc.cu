// attn_tc.cu -- tcgen05 / TMEM / TMA attention kernel for sm_100a (bf16 in,
// f32 accumulate, bf16 out), used by the frame-causal prefill, the streaming
// attend (split-KV; combine_kernel, launched behind it, merges the splits) and
// the token-band GQA prefill.
//
// What it computes: O = softmax(Q K^T / sqrt(D)) V over the keys the schedule
// lists for a 128-row query tile ("Sliding Window Attention Mechanism in
// AggregatorStream", "Mask Generation in CausalAttention": only in-window
// frames are visible; "KV Cache Eviction Strategy": only retained frames are in
// the cache; sliding-window explainer: token band t-W+1..t).
//
// CTA organisation (384 threads = 3 warpgroups, one CTA per SM):
//   warp 0      TMA producer: Q tiles once, then K key tiles into a ring (and
//               at head_dim 64 the V tile of the same key tile beside it)
//   warp 1      TMEM allocator; the whole warp runs the MMA issue loop and one
//               elected lane issues every tcgen05.mma and commit
//   warp 2      idle
//   warp 3      TMA producer at head_dim 128: V key tiles into a second ring
//   warps 4-7   softmax for query tile A (one thread per query row)
//   warps 8-11  softmax for query tile B
// After set-up, warpgroup 0 gives registers back (setmaxnreg.dec to 64) and the
// softmax warpgroups take them (setmaxnreg.inc to 216), so a thread can hold a
// whole 128-column row of S in registers.
// The two query tiles ping-pong: while softmax A turns S_A into P_A, the tensor
// core runs P_B V and Q_B K^T, and the other way round.  S (f32, 128 columns),
// P (bf16 pairs, 64 columns written over the front of S once it is read) and O
// (f32, D columns) of each tile live in tensor memory; P feeds the PV product
// straight from TMEM (A operand), so the shared-memory operands are Q, K and V,
// staged by TMA with 128-byte swizzle.  At head_dim 64 three S buffers form a
// ring shared by the two tiles: QK^T number n of the sequence A0 B0 A1 B1 ...
// writes buffer n mod 3 as soon as the PV of op n-3 (whose P sits there) is
// issued, so a tile's next scores are computed while its softmax still works on
// the current ones.  At head_dim 128 each tile has one S buffer.
// Online softmax uses exp2 with the scale folded in and skips rescaling O
// unless the running maximum grows by more than 2^8 (exact after the final
// division by the row sum).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cmath>
#include <cstdint>

#include "internal.h"
#include "exp2_poly.cuh"
#include "ptx.cuh"
#include "tile_sched.h"

// Build options, kept for same-box A/B timing against the layouts they replaced
// (SWA_NVCC_FLAGS="-DSWA_ISSUE_WARP=0" etc. with build.py):
//   SWA_ISSUE_WARP  1: the whole issuer warp runs the MMA loop, one elected lane
//                   issues; 0: lane 0 alone runs it
//   SWA_SRING       1: head_dim 64 uses three S buffers in a ring (below); 0: one
//                   S buffer per query tile and the row sums from the tensor core
#ifndef SWA_ISSUE_WARP
#define SWA_ISSUE_WARP 1
#endif
#ifndef SWA_SRING
#define SWA_SRING 1
#endif


namespace swa {

namespace {

constexpr int kThreads = 384;     // 3 warpgroups
constexpr int kRegsLaunch = 168;  // registers per thread at launch (384 x 168 = 64512 of 65536)
constexpr int kRegsCtl = 64;      // warpgroup 0 (TMA producer, MMA issuer) after setmaxnreg.dec
constexpr int kRegsSoftmax = 216; // warpgroups 1-2 (softmax) after setmaxnreg.inc
static_assert(4 * kRegsCtl + 8 * kRegsSoftmax <= 12 * kRegsLaunch,
              "register split must fit the pool the CTA was launched with");
constexpr int kRows = kTileRows;       // 128
constexpr int kMaxSegSmem = 1024;      // key runs whose tile prefix a CTA keeps in shared memory
constexpr int kSubBytes = 128 * 128;   // one 128-row x 64-column bf16 sub-tile (16 KB)

template <int D>
struct Plan {
  static_assert(D == 64 || D == 128, "tcgen05 path: head_dim 64 or 128");
  static constexpr int kSubs = D / 64;                 // 64-column sub-tiles per row
  static constexpr int kTileBytes = kRows * D * 2;     // Q, K or V tile
  static constexpr int kStages = (D == 64) ? 4 : 2;    // K/V ring depth
  // Row sums at D = 64 come out of the PV product: V is extended by a constant
  // 64-column block whose first column is 1, so O column D accumulates sum_k P
  // (in f32, from the same bf16 P the PV uses) and is rescaled with O.  The PV
  // then has N = D + 16.  At D = 128 that would not fit tensor memory; the
  // softmax threads add the row sums themselves.
  // D = 64 with SWA_SRING: three S buffers in a ring shared by the two query
  // tiles (the next QK^T of a tile runs while its softmax works on the
  // current one); the row sums then come from the softmax, O has D columns
  static constexpr bool kRing = (D == 64) && (SWA_SRING != 0);
  static constexpr bool kSumCol = (D == 64) && !kRing;
  // K and V stages with their own barriers (released after the QK^T and after
  // the PV respectively) for the two-stage ring at head_dim 128; one barrier per
  // stage for both at head_dim 64, where the four-stage ring has slack and the
  // single MMA-issuing thread saves a wait and a commit per key tile
  static constexpr bool kSplitKV = (D == 128);
  static constexpr int kON = kSumCol ? D + 16 : D;  // O columns written by the PV
  // Tensor-memory columns: S 2x128 | O 2x128 (D or D + 16 used).  P (64 columns
  // of bf16 pairs) reuses the first half of its own S once the softmax has read
  // S: the next QK^T that overwrites S is issued by the same thread after the PV
  // that reads P, and tcgen05.mma operations from one thread execute in issue order.
  SWA_DEV static uint32_t col_s(int g) { return g ? 128u : 0u; }
  SWA_DEV static uint32_t col_p(int g) { return col_s(g); }
  SWA_DEV static uint32_t col_o(int g) { return kRing ? 384u + 64u * g : (g ? 384u : 256u); }
  static constexpr uint32_t kTmemCols = 512;
  // shared-memory layout (offsets from a 1024-aligned base)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffOnes = kOffV + kStages * kTileBytes;  // the constant block (kSumCol)
  static constexpr int kOffBar = kOffOnes + (kSumCol ? kSubBytes : 0);
  static constexpr int kNumBars = 2 + 4 * kStages + 3 + 2 + 2 + 2 + 2 + 2;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;   // TMEM base (4 bytes)
  static constexpr int kOffSeg = kOffTmem + 16;              // stream mode: key tiles before each run
  static constexpr int kSmemBytes = kOffSeg + kMaxSegSmem * 4 + 1024;  // + alignment slack
};

struct Work {
  int b, kvh;
  int h0, h1;          // query heads of tiles A and B
  int qrow0, qrow1;    // first query row of tiles A and B (row index in the Q tensor, per batch)
  int rows0, rows1;    // valid query rows (0 = tile absent)
  int t_begin, t_end;  // key-tile range of this item
  int split;           // >= 0: write split-KV partials; -1: write the final output
  int nseg;
  int srow0, slen0, srow1, slen1;  // inline key runs (frame and band modes)
  const int* grow;                 // key runs in device metadata (stream mode)
  const int* glen;
  const int* tpre;                 // stream mode: key tiles before run s (shared memory), or null
  SWA_DEV int seg_row(int s) const { return grow ? __ldg(grow + s) : (s == 0 ? srow0 : srow1); }
  SWA_DEV int seg_len(int s) const { return glen ? __ldg(glen + s) : (s == 0 ? slen0 : slen1); }
};

struct Cursor {
  int s, off;
};

SWA_DEV bool cursor_seek(const Work& w, int t, Cursor& c) {
  c.s = 0;
  c.off = 0;
  if (w.tpre) {
    // run s holds key tiles tpre[s] .. tpre[s+1]-1: binary search, no walk over
    // the runs in global memory
    if (t < 0 || t >= w.tpre[w.nseg]) return false;
    int lo = 0, hi = w.nseg;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (w.tpre[mid] <= t) lo = mid;
      else hi = mid;
    }
    c.s = lo;
    c.off = (t - w.tpre[lo]) * kRows;
    return true;
  }
  while (c.s < w.nseg) {
    const int n = cdiv(w.seg_len(c.s), kRows);
    if (t < n) {
      c.off = t * kRows;
      return true;
    }
    t -= n;
    ++c.s;
  }
  return false;
}

SWA_DEV void cursor_tile(const Work& w, const Cursor& c, int* row0, int* valid) {
  const int len = w.seg_len(c.s);
  *row0 = w.seg_row(c.s) + c.off;
  *valid = imin(kRows, len - c.off);
}

SWA_DEV void cursor_next(const Work& w, Cursor& c) {
  c.off += kRows;
  if (c.off >= w.seg_len(c.s)) {
    ++c.s;
    c.off = 0;
  }
}

SWA_DEV int total_tiles(const Work& w) {
  int T = 0;
  for (int s = 0; s < w.nseg; ++s) T += cdiv(w.seg_len(s), kRows);
  return T;
}

SWA_DEV Work decode_work(const TcParams& p, const int* tpre) {
  Work w;
  w.grow = nullptr;
  w.glen = nullptr;
  w.tpre = nullptr;
  w.split = -1;
  w.nseg = 0;
  w.srow0 = w.slen0 = w.srow1 = w.slen1 = 0;
  const int64_t bid = blockIdx.x;
  if (p.mode == TC_FRAME) {
    const PrefillItem it = prefill_item(bid, p.B, p.Hq, p.F, p.n_pairs);
    w.b = it.b;
    w.kvh = it.h / (p.Hq / p.Hkv);
    w.h0 = w.h1 = it.h;
    const int t0 = 2 * it.pair;
    w.rows0 = qtile_rows(p.P, t0);
    w.rows1 = qtile_rows(p.P, t0 + 1);
    w.qrow0 = it.f * p.P + t0 * kRows;
    w.qrow1 = w.qrow0 + kRows;
    int lo[2], hi[2];
    w.nseg = frame_intervals(it.f, p.Wf, p.S, lo, hi);
    w.srow0 = lo[0] * p.P;
    w.slen0 = (hi[0] - lo[0]) * p.P;
    if (w.nseg > 1) {
      w.srow1 = lo[1] * p.P;
      w.slen1 = (hi[1] - lo[1]) * p.P;
    }
    w.t_begin = 0;
    w.t_end = total_tiles(w);
  } else if (p.mode == TC_BAND) {
    const BandItem it = band_item(bid, p.B, p.Hq, p.Hkv, p.n_qtiles);
    w.b = it.b;
    w.kvh = it.kvh;
    const int t0 = it.t * kRows;
    const int rows = imin(kRows, p.Nq - t0);
    w.h0 = it.h0;
    w.h1 = it.h1 < 0 ? it.h0 : it.h1;
    w.qrow0 = w.qrow1 = t0;
    w.rows0 = rows;
    w.rows1 = it.h1 < 0 ? 0 : rows;
    int lo, hi;
    band_keys(t0, rows, p.W, &lo, &hi);
    w.nseg = 1;
    w.srow0 = lo;
    w.slen0 = hi - lo;
    w.t_begin = 0;
    w.t_end = total_tiles(w);
  } else {  // TC_STREAM
    const StreamItem it = stream_item(bid, p.Hq, p.n_pairs);
    w.b = 0;
    w.kvh = it.h / (p.Hq / p.Hkv);
    w.h0 = w.h1 = it.h;
    const int t0 = 2 * it.pair;
    w.rows0 = qtile_rows(p.P, t0);
    w.rows1 = qtile_rows(p.P, t0 + 1);
    w.qrow0 = t0 * kRows;
    w.qrow1 = w.qrow0 + kRows;
    w.grow = p.seg_row;
    w.glen = p.seg_len;
    const int n = __ldg(p.meta_hdr + 5);
    w.nseg = (n >= 0 && n <= p.max_segs) ? n : 0;
    if (w.nseg < kMaxSegSmem) w.tpre = tpre;
    const int T = w.tpre ? w.tpre[w.nseg] : total_tiles(w);
    split_range(T, p.splits, it.split, &w.t_begin, &w.t_end);
    w.split = (p.splits > 1) ? it.split : -1;
  }
  return w;
}

// How the 64 exponential pairs of a 128-column row are split (per group of 8 pairs):
// the first kPolyPairs take 2^x on the FMA pipe (polynomial), the rest two f32
// MUFU exp2.  Measured on B200 with the warp issuer (same-box A/B): at head_dim
// 64, 3 beats 2 and 4 by 1-8 %; at head_dim 128, 1 beats 0 and 2 by 2-5 %.
// SWA_POLY_PAIRS_D64 / _D128 override them for tuning builds.
#ifndef SWA_POLY_PAIRS_D64
#define SWA_POLY_PAIRS_D64 3
#endif
#ifndef SWA_POLY_PAIRS_D128
#define SWA_POLY_PAIRS_D128 1
#endif
template <int D>
constexpr int kPolyPairs = (D == 64) ? SWA_POLY_PAIRS_D64 : SWA_POLY_PAIRS_D128;
static_assert(SWA_POLY_PAIRS_D64 <= 8 && SWA_POLY_PAIRS_D128 <= 8, "exp2 split");

SWA_DEV float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  using PL = Plan<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // a split stream attend's combine (programmatic launch) may launch now; it waits
  // for this grid before it reads a partial
  griddep_launch_dependents();

  // barriers
  const uint32_t bar0 = base + PL::kOffBar;
  auto q_full = [&](int g) { return bar0 + 8u * g; };
  // K and V stages have their own barriers: K_j is released once both tiles'
  // QK^T(j) are issued, V_j once both PV(j) are, so the K ring runs ahead
  auto k_full = [&](int s) { return bar0 + 8u * (2 + s); };
  auto v_full = [&](int s) { return bar0 + 8u * (2 + PL::kStages + s); };
  auto k_empty = [&](int s) { return bar0 + 8u * (2 + 2 * PL::kStages + s); };
  auto v_empty = [&](int s) { return bar0 + 8u * (2 + 3 * PL::kStages + s); };
  constexpr int kB = 2 + 4 * PL::kStages;
  auto s_full = [&](int i) { return bar0 + 8u * (kB + i); };      // per S buffer (3 in the ring)
  // P hand-off j of query tile g (128 arrivals, one per row) goes to barrier j mod 2, and
  // the issuer waits for it with parity (j / 2) mod 2.  One barrier per tile would not do:
  // the S of key tile j + 1 can be ready before every warp of the tile has handed off P_j
  // (the ring computes it early), so a warp running a whole key tile ahead of a slower one
  // would arrive for j + 1 while the other is still on j, and its arrivals would complete
  // hand-off j without the slower warp's rows of P
  auto p_full = [&](int g, int j) { return bar0 + 8u * ((j & 1) ? kB + 11 + g : kB + 3 + g); };
  auto p_parity = [](int j) { return static_cast<uint32_t>((j >> 1) & 1); };
  auto o_full = [&](int g) { return bar0 + 8u * (kB + 5 + g); };
  auto drain = [&](int g) { return bar0 + 8u * (kB + 7 + g); };
  auto o_done = [&](int g) { return bar0 + 8u * (kB + 9 + g); };  // ring: PV_g(j) complete
  const uint32_t tmem_slot = base + PL::kOffTmem;

  if (threadIdx.x == 0) {
    mbar_init(q_full(0), 1);
    mbar_init(q_full(1), 1);
    for (int s = 0; s < PL::kStages; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_empty(s), 1);
    }
    mbar_init(s_full(0), 1);
    mbar_init(s_full(1), 1);
    mbar_init(s_full(2), 1);
    mbar_init(o_done(0), 1);
    mbar_init(o_done(1), 1);
    for (int g = 0; g < 2; ++g) {
      mbar_init(p_full(g, 0), 128);
      mbar_init(p_full(g, 1), 128);
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(o_full(g), 1);
      mbar_init(drain(g), 1);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, PL::kTmemCols);
    tmem_relinquish();
  }
  if constexpr (PL::kSumCol) {
    // 128 keys x 64 columns of bf16 in the 128-byte-swizzled layout of a V
    // sub-tile: column 0 (logical 16-byte chunk 0 of key row k, stored at
    // physical chunk k mod 8) is 1.0, everything else 0
    uint4* ones = reinterpret_cast<uint4*>(gbase + PL::kOffOnes);
    for (int i = threadIdx.x; i < kSubBytes / 16; i += kThreads) {
      const int key = i >> 3, chunk = i & 7;
      ones[i] = make_uint4(chunk == (key & 7) ? 0x3F80u : 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  int* tpre = reinterpret_cast<int*>(gbase + PL::kOffSeg);
  if (p.mode == TC_STREAM && warp == 2) {
    // the tiles of the key runs, summed into a prefix in shared memory by one warp
    // (128 runs' lengths loaded at a time), so that no thread walks the runs in
    // global memory to find its split's first tile
    const int n = __ldg(p.meta_hdr + 5);
    const int nseg = (n >= 0 && n <= p.max_segs) ? n : 0;
    if (nseg < kMaxSegSmem) {
      if (lane == 0) tpre[0] = 0;
      int carry = 0;
      for (int c0 = 0; c0 < nseg; c0 += 128) {
        int v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int sg = c0 + 32 * k + lane;
          v[k] = sg < nseg ? cdiv(__ldg(p.seg_len + sg), kRows) : 0;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, v[k], off);
            if (lane >= off) v[k] += y;
          }
          const int sg = c0 + 32 * k + lane;
          if (sg < nseg) tpre[sg + 1] = carry + v[k];
          carry += __shfl_sync(0xffffffffu, v[k], 31);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + PL::kOffTmem);
  const Work w = decode_work(p, tpre);
  const int T = w.t_end - w.t_begin;
  const bool has_b = w.rows1 > 0;
  if (warp < 4) {
  reg_dealloc<kRegsCtl>();
  if (warp == 0 || warp == 3) {
    // ------------------------------------------------------------ producers
    // lane 0 of warp 0 loads the Q tiles and the K ring, lane 0 of warp 3 the V
    // ring (split K/V barriers); without the split warp 0 loads both
    const bool is_k = (warp == 0);
    if (lane == 0 && T > 0 && (PL::kSplitKV || is_k)) {
      const CUtensorMap* tm = is_k ? &p.tm_k : &p.tm_v;
      tma_prefetch_desc(tm);
      if (!PL::kSplitKV) tma_prefetch_desc(&p.tm_v);
      if (is_k) {
        tma_prefetch_desc(&p.tm_q);
        for (int g = 0; g < (has_b ? 2 : 1); ++g) {
          mbar_arrive_expect_tx(q_full(g), PL::kTileBytes);
          for (int sub = 0; sub < PL::kSubs; ++sub)
            tma_load_4d(base + PL::kOffQ + g * PL::kTileBytes + sub * kSubBytes, &p.tm_q, q_full(g),
                        sub * 64, g ? w.h1 : w.h0, g ? w.qrow1 : w.qrow0, w.b);
        }
      }
      const uint32_t ring = base + (is_k ? PL::kOffK : PL::kOffV);
      Cursor cur;
      bool ok = cursor_seek(w, w.t_begin, cur);
      if (!ok) latch_error(p.err, ERR_BAD_META);
      int issued = 0;
      for (int j = 0; j < T && ok; ++j) {
        const int st = j % PL::kStages;
        const uint32_t full = is_k ? k_full(st) : v_full(st);
        if (j >= PL::kStages && !mbar_wait(is_k ? k_empty(st) : v_empty(st), ((j / PL::kStages) - 1) & 1,
                                           p.err, ERR_WAIT_TMA)) {
          ok = false;
          break;
        }
        if (cur.s >= w.nseg) {
          latch_error(p.err, ERR_BAD_META);
          ok = false;
          break;
        }
        int krow, kvalid;
        cursor_tile(w, cur, &krow, &kvalid);
        mbar_arrive_expect_tx(full, PL::kSplitKV ? PL::kTileBytes : 2 * PL::kTileBytes);
        for (int sub = 0; sub < PL::kSubs; ++sub) {
          tma_load_4d(ring + st * PL::kTileBytes + sub * kSubBytes, tm, full, sub * 64, w.kvh, krow, w.b);
          if (!PL::kSplitKV)
            tma_load_4d(base + PL::kOffV + st * PL::kTileBytes + sub * kSubBytes, &p.tm_v, full, sub * 64, w.kvh,
                        krow, w.b);
        }
        cursor_next(w, cur);
        ++issued;
      }
      // drain: never leave the CTA with a bulk copy still writing its shared memory
      for (int j = issued - PL::kStages; j < issued; ++j) {
        if (j < 0) continue;
        mbar_wait(is_k ? k_full(j % PL::kStages) : v_full(j % PL::kStages), (j / PL::kStages) & 1, p.err,
                  ERR_WAIT_TMA);
      }
      if (is_k)
        for (int g = 0; g < (has_b ? 2 : 1); ++g) mbar_wait(q_full(g), 0, p.err, ERR_WAIT_TMA);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // One thread issues every tcgen05.mma and the commits that track them.
    // With SWA_ISSUE_WARP the whole warp runs the issue loop (uniform control
    // flow, the descriptors held alike by every lane) and the instructions are
    // predicated on one elected lane; otherwise lane 0 runs it alone.  The issue
    // path is kept short (a single thread's instruction latency bounds the MMA
    // rate for N <= 128): shared-memory descriptors are built once, and a K step
    // or a ring stage moves the start-address field by a constant (addresses
    // stay below 2^18, so the 14-bit field never carries).
#if SWA_ISSUE_WARP
    const bool run = T > 0;
    const uint32_t issue = elect_one();
    const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
    auto wait = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, p.err, ERR_WAIT_MMA));
    };
#else
    const bool run = lane == 0 && T > 0;
    const uint32_t issue = 1;
    const uint32_t tm = tmem;
    auto wait = [&](uint32_t bar, uint32_t parity) { return mbar_wait(bar, parity, p.err, ERR_WAIT_MMA); };
#endif
    if (run) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, PL::kON, 1);
      constexpr uint64_t kStageStep = PL::kTileBytes >> 4;
      const uint64_t dq0 = sdesc_sw128(base + PL::kOffQ, 16, 1024);
      const uint64_t dk0 = sdesc_sw128(base + PL::kOffK, 16, 1024);
      const uint64_t dv0 = sdesc_sw128(base + PL::kOffV, PL::kSumCol ? PL::kOffOnes - PL::kOffV : kSubBytes, 1024);
      auto issue_qk = [&](int g, int st) {
        const uint64_t dq = dq0 + g * kStageStep;  // Q tiles are kTileBytes apart too
        const uint64_t dk = dk0 + st * kStageStep;
        const uint32_t tS = tm + PL::col_s(g);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kSubBytes + (kk & 3) * 32) >> 4);
          mma_ss_if(issue, tS, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int g, int st, bool acc) {
        // kSumCol: the second 64-column block of B is the ones block, at a
        // leading-byte offset that shrinks as the stage moves up
        const uint64_t dv = PL::kSumCol ? dv0 + st * kStageStep - ((st * kStageStep) << 16)
                                        : dv0 + st * kStageStep;
        const uint32_t tP = tm + PL::col_p(g), tO = tm + PL::col_o(g);
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk)
          mma_ts_if(issue, tO, tP + kk * 8, dv + ((kk * 16 * 128) >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = wait(q_full(0), 0);
      if (ok && has_b) ok = wait(q_full(1), 0);
      if (ok) ok = wait(k_full(0), 0);
      if constexpr (PL::kRing) {
        // QK^T ops in the order A0 B0 A1 B1 A2 ...: op n of the sequence (n =
        // 2j + g, or j with one tile) writes S buffer n mod 3, whose previous
        // user, op n - 3, had its PV issued before it (P aliases its S)
        auto seq = [&](int g, int j) { return has_b ? 2 * j + g : j; };
        auto qk_ring = [&](int g, int j) {
          const int n = seq(g, j);
          const uint64_t dq = dq0 + g * kStageStep;
          const uint64_t dk = dk0 + (j % PL::kStages) * kStageStep;
          const uint32_t tS = tm + 128u * static_cast<uint32_t>(n % 3);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kSubBytes + (kk & 3) * 32) >> 4);
            mma_ss_if(issue, tS, dq + off, dk + off, idesc_qk, kk > 0 ? 1u : 0u);
          }
          mma_commit_if(issue, s_full(n % 3));
        };
        auto pv_ring = [&](int g, int j) {
          const int st = j % PL::kStages;
          const uint64_t dv = dv0 + st * kStageStep;
          const uint32_t tP = tm + 128u * static_cast<uint32_t>(seq(g, j) % 3), tO = tm + PL::col_o(g);
#pragma unroll
          for (int kk = 0; kk < kRows / 16; ++kk)
            mma_ts_if(issue, tO, tP + kk * 8, dv + ((kk * 16 * 128) >> 4), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit_if(issue, o_done(g));
          if (j == T - 1) mma_commit_if(issue, o_full(g));
        };
        if (ok) {
          tc_fence_after();
          qk_ring(0, 0);
          if (has_b) qk_ring(1, 0);
          if (T > 1) {
            ok = wait(k_full(1 % PL::kStages), (1 / PL::kStages) & 1);
            if (ok) qk_ring(0, 1);
          }
        }
        for (int j = 0; j < T && ok; ++j) {
          if (!wait(p_full(0, j), p_parity(j))) break;
          tc_fence_after();
          pv_ring(0, j);
          if (has_b) {
            if (j + 1 < T) qk_ring(1, j + 1);
            if (!wait(p_full(1, j), p_parity(j))) break;
            tc_fence_after();
            pv_ring(1, j);
          }
          mma_commit_if(issue, k_empty(j % PL::kStages));  // K_j and V_j leave after the last PV(j)
          if (j + 2 < T) {
            if (!wait(k_full((j + 2) % PL::kStages), ((j + 2) / PL::kStages) & 1)) break;
            qk_ring(0, j + 2);
          }
        }
        ok = false;  // the fixed-order loop below is for the other layouts
      }
      if (ok) {
        tc_fence_after();
        issue_qk(0, 0);
        mma_commit_if(issue, s_full(0));
        if (has_b) {
          issue_qk(1, 0);
          mma_commit_if(issue, s_full(1));
        }
        if (PL::kSplitKV) mma_commit_if(issue, k_empty(0));
      }
      const int ng = has_b ? 2 : 1;
      // Fixed order per key tile: PV_A(j) QK_A(j+1) | PV_B(j) QK_B(j+1), each
      // tile's MMAs back to back with its commit after them.  P_g aliases S_g:
      // QK_g(j+1) follows PV_g(j) in the issuing thread's order, which the
      // tensor core keeps.
      for (int j = 0; j < T && ok; ++j) {
        const int st = j % PL::kStages;
        const int st1 = (j + 1) % PL::kStages;
        const bool more = j + 1 < T;
        if (more && !wait(k_full(st1), ((j + 1) / PL::kStages) & 1)) break;
        if (PL::kSplitKV && !wait(v_full(st), (j / PL::kStages) & 1)) break;
#pragma unroll 1
        for (int g = 0; g < ng; ++g) {
          if (!wait(p_full(g, j), p_parity(j))) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(g, st, j > 0);
          if (more) {
            issue_qk(g, st1);
            mma_commit_if(issue, s_full(g));
          } else {
            mma_commit_if(issue, o_full(g));
          }
        }
        if (!ok) break;
        if (PL::kSplitKV) {
          mma_commit_if(issue, v_empty(st));
          if (more) mma_commit_if(issue, k_empty(st1));
        } else {
          mma_commit_if(issue, k_empty(st));  // K_j and V_j leave together after PV_B(j)
        }
      }
      // drain every MMA the issuing thread started before the CTA may free TMEM
      mma_commit_if(issue, drain(0));
      wait(drain(0), 0);
    }
  }
  } else {
    reg_alloc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    const int g = (warp - 4) >> 2;  // 0: tile A, 1: tile B
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS0 = tmem + lane_off + PL::col_s(g);
    const uint32_t tO = tmem + lane_off + PL::col_o(g);
    const float sl2 = p.scale_log2;
    const bool band = (p.mode == TC_BAND);
    const int my_h = g ? w.h1 : w.h0;
    const int my_row0 = g ? w.qrow1 : w.qrow0;
    const int my_rows = g ? w.rows1 : w.rows0;
    const int qrow = my_row0 + r;  // query token (band mode: absolute position)
    float m = -INFINITY;           // running reference max of raw scores
    float l = 0.f;                 // running row sum relative to m
    bool ok = (g == 0 || has_b) && T > 0;
    const bool active = ok;
    Cursor cur;
    if (ok) ok = cursor_seek(w, w.t_begin, cur);
    for (int j = 0; j < T && ok; ++j) {
      if (cur.s >= w.nseg) {
        ok = false;
        break;
      }
      int krow, kvalid;
      cursor_tile(w, cur, &krow, &kvalid);
      cursor_next(w, cur);
      // this key tile's S buffer and the phase of its barrier
      int sbuf = g;
      uint32_t sphase = j & 1;
      if constexpr (PL::kRing) {
        const int n = has_b ? 2 * j + g : j;
        sbuf = n % 3;
        sphase = (n / 3) & 1;
      }
      const uint32_t tS = PL::kRing ? tmem + lane_off + 128u * static_cast<uint32_t>(sbuf) : tS0;
      const uint32_t tP = tS;
      if (!__all_sync(0xffffffffu, mbar_wait(s_full(sbuf), sphase, p.err, ERR_WAIT_SOFTMAX))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s[128];
      tmem_ld32(tS + 0, s);
      tmem_ld32(tS + 32, s + 32);
      tmem_ld32(tS + 64, s + 64);
      tmem_ld32(tS + 96, s + 96);
      tmem_wait_ld();
      // ---- masks: unused tail of the last tile of a key run, band edges
      if (band) {
        const bool inside = (krow >= my_row0 + my_rows - 1 - p.W + 1) && (krow + kvalid - 1 <= my_row0) &&
                            kvalid == kRows;
        if (!inside) {
          const int lo = qrow - p.W + 1;
#pragma unroll
          for (int c = 0; c < 128; ++c) {
            const int key = krow + c;
            if (c >= kvalid || key < lo || key > qrow) s[c] = __float_as_uint(-INFINITY);
          }
        }
      } else if (kvalid < kRows) {
        // only the 32-column blocks that reach past the run's end (kvalid is
        // the same for every row, so the block test is warp-uniform)
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32)
          if (kvalid < c0 + 32) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c0 + c >= kvalid) s[c0 + c] = __float_as_uint(-INFINITY);
          }
      }
      // ---- row max: eight independent 3-input max chains
      float a[8];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        a[k] = max3f(__uint_as_float(s[k]), __uint_as_float(s[8 + k]), __uint_as_float(s[16 + k]));
#pragma unroll
      for (int c = 24; c < 120; c += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          a[k] = max3f(a[k], __uint_as_float(s[c + k]), __uint_as_float(s[c + 8 + k]));
#pragma unroll
      for (int k = 0; k < 8; ++k) a[k] = fmaxf(a[k], __uint_as_float(s[120 + k]));
      const float tmax = max3f(max3f(a[0], a[1], a[2]), max3f(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
      const float m_new = fmaxf(m, tmax);
      const bool grow = (m != -INFINITY) && ((m_new - m) * sl2 > 8.0f);
      float alpha = 1.f;
      if (m == -INFINITY) {
        m = m_new;
      } else if (grow) {
        alpha = ex2_approx((m - m_new) * sl2);
        m = m_new;
      }
      if (__any_sync(0xffffffffu, grow)) {
        // O of this tile must be complete up to key tile j-1 before it is
        // rescaled in place: the commit that signalled S_j covers the earlier
        // PV, except in the ring, where PV(j-1) may still run (wait for it)
        if (PL::kRing && j > 0) {
          if (!__all_sync(0xffffffffu, mbar_wait(o_done(g), (j - 1) & 1, p.err, ERR_WAIT_SOFTMAX))) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t orr[32];
          tmem_ld32(tO + c0, orr);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
          tmem_st32(tO + c0, orr);
        }
        if constexpr (PL::kSumCol) {
          uint32_t o16[16];
          tmem_ld16(tO + D, o16);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 16; ++c) o16[c] = __float_as_uint(__uint_as_float(o16[c]) * alpha);
          tmem_st16(tO + D, o16);
        }
        tmem_wait_st();
      }
      l *= alpha;
      // ---- P = 2^(s*scale - m*scale): MUFU for most column pairs, the
      // polynomial on the FMA pipe for kPolyPairs of every 8; packed bf16
      // pairs overwrite the front of s (pair pi reads s[2pi], s[2pi+1] >= pi)
      const float nb = (m == -INFINITY) ? 0.f : -m * sl2;
      const float2 c2 = make_float2(sl2, sl2);
      const float2 nb2 = make_float2(nb, nb);
      float2 acc[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int pi = 0; pi < 64; ++pi) {
        const float2 x =
            __ffma2_rn(make_float2(__uint_as_float(s[2 * pi]), __uint_as_float(s[2 * pi + 1])), c2, nb2);
        float2 pr;
        if ((pi & 7) < kPolyPairs<D>) {
          pr = exp2_poly2(x);
        } else {
          pr.x = ex2_approx(x.x);
          pr.y = ex2_approx(x.y);
        }
        if constexpr (!PL::kSumCol) acc[pi & 3] = __fadd2_rn(acc[pi & 3], pr);
        s[pi] = pack_bf16x2(pr.x, pr.y);
      }
      if constexpr (!PL::kSumCol)
        l += ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) + ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
      tmem_st32(tP + 0, s);
      tmem_st32(tP + 32, s + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(g, j));
    }
    // ---- epilogue
    if (active && ok) {
      if (__all_sync(0xffffffffu, mbar_wait(o_full(g), 0, p.err, ERR_WAIT_EPI))) {
        tc_fence_after();
        if constexpr (PL::kSumCol) {
          uint32_t o16[16];
          tmem_ld16(tO + D, o16);
          tmem_wait_ld();
          l = __uint_as_float(o16[0]);
        }
        const bool store = r < my_rows;
        const int row = my_row0 + r;
        const float inv = 1.f / l;
        const int64_t idx = (w.split < 0)
                                ? (static_cast<int64_t>(w.b) * p.Nq + row) * p.Hq + my_h
                                : (static_cast<int64_t>(w.split) * p.Nq + row) * p.Hq + my_h;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t orr[32];
          tmem_ld32(tO + c0, orr);
          tmem_wait_ld();
          if (!store) continue;
          if (w.split < 0) {
            const int64_t out_ld = p.out_ld ? p.out_ld : static_cast<int64_t>(p.Hq) * D;
            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) +
                                 (static_cast<int64_t>(w.b) * p.Nq + row) * out_ld +
                                 static_cast<int64_t>(p.out_h0 + my_h) * D + c0;
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(orr[c + 0]) * inv, __uint_as_float(orr[c + 1]) * inv);
              v.y = pack_bf16x2(__uint_as_float(orr[c + 2]) * inv, __uint_as_float(orr[c + 3]) * inv);
              v.z = pack_bf16x2(__uint_as_float(orr[c + 4]) * inv, __uint_as_float(orr[c + 5]) * inv);
              v.w = pack_bf16x2(__uint_as_float(orr[c + 6]) * inv, __uint_as_float(orr[c + 7]) * inv);
              *reinterpret_cast<uint4*>(dst + c) = v;
            }
          } else {
            float* dst = p.part_o + idx * D + c0;
#pragma unroll
            for (int c = 0; c < 32; c += 4)
              *reinterpret_cast<float4*>(dst + c) =
                  make_float4(__uint_as_float(orr[c]), __uint_as_float(orr[c + 1]),
                              __uint_as_float(orr[c + 2]), __uint_as_float(orr[c + 3]));
          }
        }
        if (store && w.split >= 0) {
          p.part_ml[idx * 2 + 0] = m * sl2;
          p.part_ml[idx * 2 + 1] = l;
        }
      }
    } else if (T == 0 && w.split >= 0 && (g == 0 || has_b) && r < my_rows) {
      // empty split: contributes nothing to the combine
      const int row = my_row0 + r;
      const int64_t idx = (static_cast<int64_t>(w.split) * p.Nq + row) * p.Hq + my_h;
      p.part_ml[idx * 2 + 0] = -INFINITY;
      p.part_ml[idx * 2 + 1] = 0.f;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, PL::kTmemCols);
  }
}

}  // namespace

// ---------------------------------------------------------------- combine
// O = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c  (m in log2 units), the
// log-sum-exp merge of split-KV partials.  One warp per (row, head): lane c
// holds split c's (m, l), the warp reduces M and the weighted sum, then every
// lane accumulates its slice of O over the splits with independent loads.
namespace {
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ part_o,
                                                      const float* __restrict__ part_ml,
                                                      __nv_bfloat16* __restrict__ out, int rows,
                                                      int H, int splits, int64_t out_ld, int out_h0) {
  griddep_wait();  // behind the attend (programmatic launch): its partials first
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= rows * H) return;
  const int64_t stride = static_cast<int64_t>(rows) * H;
  float mc = -INFINITY, lc = 0.f;
  if (lane < splits) {
    const float2 ml = *reinterpret_cast<const float2*>(part_ml + (lane * stride + gw) * 2);
    mc = ml.x;
    lc = ml.y;
  }
  float M = mc;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  const float wc = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
  float L = wc * lc;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  constexpr int E = D / 32;  // elements per lane: 2 (D = 64) or 4 (D = 128)
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  for (int c = 0; c < splits; ++c) {
    const float w = __shfl_sync(0xffffffffu, wc, c);
    if (w == 0.f) continue;  // a split without keys: its O was never written
    const float* src = part_o + (c * stride + gw) * D + lane * E;
    if constexpr (E == 2) {
      const float2 v = *reinterpret_cast<const float2*>(src);
      acc[0] = fmaf(w, v.x, acc[0]);
      acc[1] = fmaf(w, v.y, acc[1]);
    } else {
      const float4 v = *reinterpret_cast<const float4*>(src);
      acc[0] = fmaf(w, v.x, acc[0]);
      acc[1] = fmaf(w, v.y, acc[1]);
      acc[2] = fmaf(w, v.z, acc[2]);
      acc[3] = fmaf(w, v.w, acc[3]);
    }
  }
  const float inv = 1.f / L;
  const int row = gw / H, h = gw - row * H;
  __nv_bfloat16* dst = out + static_cast<int64_t>(row) * out_ld + static_cast<int64_t>(out_h0 + h) * D + lane * E;
  if constexpr (E == 2) {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
  } else {
    uint2 v;
    v.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    v.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2*>(dst) = v;
  }
}

}  // namespace

cudaError_t launch_combine(const float* part_o, const float* part_ml, void* out, int rows, int H, int splits,
                           int head_dim, int64_t out_ld, int out_h0, cudaStream_t stream) {
  if (splits < 1 || splits > 32) return cudaErrorInvalidValue;  // one split per lane
  const dim3 blocks(static_cast<unsigned>((static_cast<int64_t>(rows) * H + 7) / 8));
  __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out);
  cudaError_t e;
  if (head_dim == 64)
    e = launch_after(combine_kernel<64>, blocks, dim3(256), 0, stream, part_o, part_ml, o, rows, H, splits,
                     out_ld, out_h0);
  else if (head_dim == 128)
    e = launch_after(combine_kernel<128>, blocks, dim3(256), 0, stream, part_o, part_ml, o, rows, H, splits,
                     out_ld, out_h0);
  else
    return cudaErrorInvalidValue;
  count_launches(1);
  return e;
}

int tc_smem_bytes(int head_dim) {
  return head_dim == 64 ? Plan<64>::kSmemBytes : head_dim == 128 ? Plan<128>::kSmemBytes : -1;
}

namespace {
template <int D>
cudaError_t launch_tc_d(const TcParams& p, int64_t n_items, cudaStream_t stream) {
  static DeviceOnce attr_set;  // devices on which the smem opt-in was set
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (!attr_set.done(dev)) {
    // the setmaxnreg split moves registers inside the pool the CTA is launched
    // with; refuse to launch a build whose pool would be too small (the
    // increasing warpgroups would otherwise wait forever)
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_tc_kernel<D>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * 12 < 4 * kRegsCtl + 8 * kRegsSoftmax) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, Plan<D>::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set.mark(dev);
  }
  attn_tc_kernel<D><<<static_cast<unsigned>(n_items), kThreads, Plan<D>::kSmemBytes, stream>>>(p);
  count_launches(1);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_attn_tc(const TcParams& p, int head_dim, int64_t n_items, cudaStream_t stream) {
  if (n_items <= 0) return cudaSuccess;
  if (head_dim == 64) return launch_tc_d<64>(p, n_items, stream);
  if (head_dim == 128) return launch_tc_d<128>(p, n_items, stream);
  return cudaErrorInvalidValue;
}

}  // namespace swa
