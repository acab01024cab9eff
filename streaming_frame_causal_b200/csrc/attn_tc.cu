// attn_tc.cu -- tcgen05 / TMEM / TMA attention kernel for sm_100a (bf16 in,
// f32 accumulate, bf16 out), used by the frame-causal prefill, the streaming
// attend (split-KV, merged by the last CTA of each work item) and the
// token-band GQA prefill.
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
//   warp 1      TMEM allocator; lane 0 issues every tcgen05.mma
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
// (f32, D columns, plus the row-sum column at head_dim 64) of each tile live in
// tensor memory; P feeds the PV product straight from TMEM (A operand), so the
// shared-memory operands are Q, K and V, staged by TMA with 128-byte swizzle
// (and at head_dim 64 a constant block that turns one PV column into the row
// sum).
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

// Build-time variants of the kernel (A/B timing builds):
#ifndef SWA_ISSUE_WARP
#define SWA_ISSUE_WARP 1
#endif
#ifndef SWA_SRING
#define SWA_SRING 0
#endif
// SWA_KEY_HALVES: head_dim 64 runs attn_hs_kernel (two softmax warpgroups per
// query tile, one per 64-key half of every key tile)
#ifndef SWA_KEY_HALVES
#define SWA_KEY_HALVES 0
#endif
#ifndef SWA_PSTORE_SPLIT
#define SWA_PSTORE_SPLIT 0
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
  static constexpr int kNumBars = 2 + 4 * kStages + 3 + 2 + 2 + 2 + 2;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;   // TMEM base (4 bytes), then the merge flag
  static constexpr int kSmemBytes = kOffTmem + 16 + 1024;  // + alignment slack
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
  SWA_DEV int seg_row(int s) const { return grow ? __ldg(grow + s) : (s == 0 ? srow0 : srow1); }
  SWA_DEV int seg_len(int s) const { return glen ? __ldg(glen + s) : (s == 0 ? slen0 : slen1); }
};

struct Cursor {
  int s, off;
};

SWA_DEV bool cursor_seek(const Work& w, int t, Cursor& c) {
  c.s = 0;
  c.off = 0;
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

SWA_DEV Work decode_work(const TcParams& p) {
  Work w;
  w.grow = nullptr;
  w.glen = nullptr;
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
    const int T = total_tiles(w);
    split_range(T, p.splits, it.split, &w.t_begin, &w.t_end);
    w.split = (p.splits > 1) ? it.split : -1;
  }
  return w;
}

// How the 64 exponential pairs of a 128-column row are split (per group of 8 pairs):
// the first kPolyPairs take 2^x on the FMA pipe (polynomial), the rest two f32
// MUFU exp2 (packed f16x2/bf16x2 MUFU exp2 yields no more results per clock).
// Measured on B200 (same-box sweeps of 2, 3, 4): 3 is fastest at head_dim 64,
// where the row sums come from the tensor core and leave the FMA pipe room, and
// 2 at head_dim 128.  SWA_POLY_PAIRS_D64 / _D128 override them for tuning builds.
#ifndef SWA_POLY_PAIRS_D64
#define SWA_POLY_PAIRS_D64 3
#endif
#ifndef SWA_POLY_PAIRS_D128
#define SWA_POLY_PAIRS_D128 2
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

  const Work w = decode_work(p);
  const int T = w.t_end - w.t_begin;
  const bool has_b = w.rows1 > 0;

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
  auto p_full = [&](int g) { return bar0 + 8u * (kB + 3 + g); };
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
    mbar_init(p_full(0), 128);
    mbar_init(p_full(1), 128);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + PL::kOffTmem);
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
          if (!wait(p_full(0), j & 1)) break;
          tc_fence_after();
          pv_ring(0, j);
          if (has_b) {
            if (j + 1 < T) qk_ring(1, j + 1);
            if (!wait(p_full(1), j & 1)) break;
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
          if (!wait(p_full(g), j & 1)) {
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
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= kvalid) s[c] = __float_as_uint(-INFINITY);
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
        // SWA_PSTORE_SPLIT: the first 32 packed pairs go to TMEM while the
        // second half is computed (pairs 0..31 are final once pi reaches 32)
        if (SWA_PSTORE_SPLIT && pi == 32) tmem_st32(tP + 0, s);
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
      if (!SWA_PSTORE_SPLIT) tmem_st32(tP + 0, s);
      tmem_st32(tP + 32, s + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(g));
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
      // empty split: contributes nothing to the merge
      const int row = my_row0 + r;
      const int64_t idx = (static_cast<int64_t>(w.split) * p.Nq + row) * p.Hq + my_h;
      p.part_ml[idx * 2 + 0] = -INFINITY;
      p.part_ml[idx * 2 + 1] = 0.f;
    }
    if (w.split >= 0) {
      // ---- split-KV merge in the item's last CTA: every thread publishes its
      // partial stores (fence), the 256 softmax threads meet, one of them
      // counts this CTA in; the CTA that completes the count merges all of the
      // item's partials, O = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c (m
      // in log2 units), and puts the count back for the next launch
      volatile int* flag = reinterpret_cast<volatile int*>(gbase + PL::kOffTmem + 8);
      const int item = static_cast<int>(blockIdx.x % (static_cast<unsigned>(p.Hq) * p.n_pairs));
      __threadfence();
      __syncwarp();
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (warp == 4 && lane == 0) *flag = (atomicAdd(p.split_cnt + item, 1) == p.splits - 1) ? 1 : 0;
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (*flag) {
        __threadfence();
        if ((g == 0 || has_b) && r < my_rows) {
          const int row = my_row0 + r;
          const int64_t stride = static_cast<int64_t>(p.Nq) * p.Hq;
          const int64_t base_idx = static_cast<int64_t>(row) * p.Hq + my_h;
          float M = -INFINITY;
          for (int c = 0; c < p.splits; ++c) M = fmaxf(M, __ldcg(p.part_ml + (c * stride + base_idx) * 2));
          float L = 0.f;
          for (int c = 0; c < p.splits; ++c) {
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml + (c * stride + base_idx) * 2));
            L = fmaf((ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M), ml.y, L);
          }
          const float inv = 1.f / L;
          const int64_t out_ld = p.out_ld ? p.out_ld : static_cast<int64_t>(p.Hq) * D;
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * out_ld +
                               static_cast<int64_t>(p.out_h0 + my_h) * D;
          // 32 output columns at a time, each the weighted sum over the splits
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            float o[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0.f;
            for (int c = 0; c < p.splits; ++c) {
              const float m_c = __ldcg(p.part_ml + (c * stride + base_idx) * 2);
              const float wc = (m_c == -INFINITY) ? 0.f : exp2f(m_c - M);
              const float4* src = reinterpret_cast<const float4*>(p.part_o + (c * stride + base_idx) * D + c0);
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float4 v = __ldcg(src + e);
                o[4 * e] = fmaf(wc, v.x, o[4 * e]);
                o[4 * e + 1] = fmaf(wc, v.y, o[4 * e + 1]);
                o[4 * e + 2] = fmaf(wc, v.z, o[4 * e + 2]);
                o[4 * e + 3] = fmaf(wc, v.w, o[4 * e + 3]);
              }
            }
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 v;
              v.x = pack_bf16x2(o[e] * inv, o[e + 1] * inv);
              v.y = pack_bf16x2(o[e + 2] * inv, o[e + 3] * inv);
              v.z = pack_bf16x2(o[e + 4] * inv, o[e + 5] * inv);
              v.w = pack_bf16x2(o[e + 6] * inv, o[e + 7] * inv);
              *reinterpret_cast<uint4*>(dst + c0 + e) = v;
            }
          }
        }
        if (warp == 4 && lane == 0) p.split_cnt[item] = 0;
      }
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

// ---------------------------------------------------------------- head_dim 64, key halves
// The same attention at head_dim 64 with twice the softmax warps and no more
// tensor memory: every 128-key tile's scores are split between two
// warpgroups, one per 64-key half.  Each half keeps its own running maximum,
// row sum and O accumulator (the PV of a half multiplies that half's P by that
// half's 64 rows of V into its own O), so the two halves of a row never
// exchange anything per tile; the epilogue merges them like two split-KV
// partials.  640 threads = 5 warpgroups:
//   warpgroup 0   warp 0 TMA producer (Q once, K and V of a key tile under one
//                 barrier), warp 1 TMEM allocator and MMA issuer (whole warp,
//                 one elected lane), warps 2-3 idle
//   warpgroups 1-4  softmax of (tile A, keys 0-63), (A, 64-127), (B, 0-63),
//                 (B, 64-127): one thread per query row, 64 scores
// Tensor memory: S_A 0-127, S_B 128-255 (each half's P over the front of its
// own 64 columns), O_A0 256, O_A1 320, O_B0 384, O_B1 448 (64 columns each).
namespace hs {
constexpr int kThreads = 640;
constexpr int kRegsLaunch = 96;    // 640 x 96 = 61440 of 65536
constexpr int kRegsCtl = 64;       // warpgroup 0 after setmaxnreg.dec
constexpr int kRegsSoftmax = 104;  // warpgroups 1-4 after setmaxnreg.inc
static_assert(4 * kRegsCtl + 16 * kRegsSoftmax <= 20 * kRegsLaunch,
              "register split must fit the pool the CTA was launched with");
constexpr int kStages = 4;
constexpr int kTileBytes = kRows * 64 * 2;  // 16 KB: a Q, K or V tile
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + 2 * kTileBytes;
constexpr int kOffV = kOffK + kStages * kTileBytes;
constexpr int kOffX = kOffV + kStages * kTileBytes;  // epilogue exchange: [tile][half][row] (m, l)
constexpr int kOffBar = kOffX + 2 * 2 * kRows * 8;
// q_full 2, kv_full 4, kv_empty 4, s_full 2, p_full 4 (tile x half), o_full 2, drain 1
constexpr int kNumBars = 2 + 2 * kStages + 2 + 4 + 2 + 1;
constexpr int kOffTmem = kOffBar + kNumBars * 8;  // TMEM base (4 bytes), then the merge flag
constexpr int kSmemBytes = kOffTmem + 16 + 1024;
}  // namespace hs

__global__ void __launch_bounds__(hs::kThreads, 1) attn_hs_kernel(const __grid_constant__ TcParams p) {
  constexpr int D = 64;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const Work w = decode_work(p);
  const int T = w.t_end - w.t_begin;
  const bool has_b = w.rows1 > 0;

  const uint32_t bar0 = base + hs::kOffBar;
  auto q_full = [&](int g) { return bar0 + 8u * g; };
  auto kv_full = [&](int s) { return bar0 + 8u * (2 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (2 + hs::kStages + s); };
  constexpr int kB = 2 + 2 * hs::kStages;
  auto s_full = [&](int g) { return bar0 + 8u * (kB + g); };
  auto p_full = [&](int g, int h) { return bar0 + 8u * (kB + 2 + 2 * g + h); };
  auto o_full = [&](int g) { return bar0 + 8u * (kB + 6 + g); };
  const uint32_t drain = bar0 + 8u * (kB + 8);
  const uint32_t tmem_slot = base + hs::kOffTmem;

  if (threadIdx.x == 0) {
    for (int g = 0; g < 2; ++g) {
      mbar_init(q_full(g), 1);
      mbar_init(s_full(g), 1);
      mbar_init(o_full(g), 1);
      mbar_init(p_full(g, 0), 128);
      mbar_init(p_full(g, 1), 128);
    }
    for (int s = 0; s < hs::kStages; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + hs::kOffTmem);
  if (warp < 4) {
    reg_dealloc<hs::kRegsCtl>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0 && T > 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
        for (int g = 0; g < (has_b ? 2 : 1); ++g) {
          mbar_arrive_expect_tx(q_full(g), hs::kTileBytes);
          tma_load_4d(base + hs::kOffQ + g * hs::kTileBytes, &p.tm_q, q_full(g), 0, g ? w.h1 : w.h0,
                      g ? w.qrow1 : w.qrow0, w.b);
        }
        Cursor cur;
        bool ok = cursor_seek(w, w.t_begin, cur);
        if (!ok) latch_error(p.err, ERR_BAD_META);
        int issued = 0;
        for (int j = 0; j < T && ok; ++j) {
          const int st = j % hs::kStages;
          if (j >= hs::kStages &&
              !mbar_wait(kv_empty(st), ((j / hs::kStages) - 1) & 1, p.err, ERR_WAIT_TMA))
            break;
          if (cur.s >= w.nseg) {
            latch_error(p.err, ERR_BAD_META);
            break;
          }
          int krow, kvalid;
          cursor_tile(w, cur, &krow, &kvalid);
          mbar_arrive_expect_tx(kv_full(st), 2 * hs::kTileBytes);
          tma_load_4d(base + hs::kOffK + st * hs::kTileBytes, &p.tm_k, kv_full(st), 0, w.kvh, krow, w.b);
          tma_load_4d(base + hs::kOffV + st * hs::kTileBytes, &p.tm_v, kv_full(st), 0, w.kvh, krow, w.b);
          cursor_next(w, cur);
          ++issued;
        }
        // never leave the CTA with a bulk copy still writing its shared memory
        for (int j = issued - hs::kStages; j < issued; ++j)
          if (j >= 0) mbar_wait(kv_full(j % hs::kStages), (j / hs::kStages) & 1, p.err, ERR_WAIT_TMA);
        for (int g = 0; g < (has_b ? 2 : 1); ++g) mbar_wait(q_full(g), 0, p.err, ERR_WAIT_TMA);
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      // Per key tile j and query tile g: PV of key half 0 once its P is in, PV
      // of half 1 once its P is in, then QK^T(j+1) into S_g (after both PVs
      // that read P from S_g, in this thread's issue order).
      const uint32_t issue = elect_one();
      const uint32_t tm = __shfl_sync(0xffffffffu, tmem, 0);
      auto wait = [&](uint32_t bar, uint32_t parity) {
        return __all_sync(0xffffffffu, mbar_wait(bar, parity, p.err, ERR_WAIT_MMA));
      };
      if (T > 0) {
        constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0);
        constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 64, 1);
        constexpr uint64_t kStageStep = hs::kTileBytes >> 4;
        const uint64_t dq0 = sdesc_sw128(base + hs::kOffQ, 16, 1024);
        const uint64_t dk0 = sdesc_sw128(base + hs::kOffK, 16, 1024);
        const uint64_t dv0 = sdesc_sw128(base + hs::kOffV, kSubBytes, 1024);
        auto issue_qk = [&](int g, int st) {
          const uint64_t dq = dq0 + g * kStageStep;
          const uint64_t dk = dk0 + st * kStageStep;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss_if(issue, tm + 128u * g, dq + 2 * kk, dk + 2 * kk, idesc_qk, kk > 0 ? 1u : 0u);
        };
        auto issue_pv = [&](int g, int h, int st, bool acc) {
          const uint64_t dv = dv0 + st * kStageStep + ((64 * h * 128) >> 4);
          const uint32_t tP = tm + 128u * g + 64u * h, tO = tm + 256u + 128u * g + 64u * h;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ts_if(issue, tO, tP + kk * 8, dv + ((kk * 16 * 128) >> 4), idesc_pv, (acc || kk > 0) ? 1u : 0u);
        };
        const int ng = has_b ? 2 : 1;
        bool ok = wait(q_full(0), 0);
        if (ok && has_b) ok = wait(q_full(1), 0);
        if (ok) ok = wait(kv_full(0), 0);
        if (ok) {
          tc_fence_after();
          for (int g = 0; g < ng; ++g) {
            issue_qk(g, 0);
            mma_commit_if(issue, s_full(g));
          }
        }
        for (int j = 0; j < T && ok; ++j) {
          const int st = j % hs::kStages;
          const int st1 = (j + 1) % hs::kStages;
          const bool more = j + 1 < T;
          if (more && !wait(kv_full(st1), ((j + 1) / hs::kStages) & 1)) break;
#pragma unroll 1
          for (int g = 0; g < ng && ok; ++g) {
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
              if (!wait(p_full(g, h), j & 1)) {
                ok = false;
                break;
              }
              tc_fence_after();
              issue_pv(g, h, st, j > 0);
            }
            if (!ok) break;
            if (more) {
              issue_qk(g, st1);
              mma_commit_if(issue, s_full(g));
            } else {
              mma_commit_if(issue, o_full(g));
            }
          }
          if (!ok) break;
          mma_commit_if(issue, kv_empty(st));  // K_j and V_j leave after the last PV(j)
        }
        // drain every MMA the issuing thread started before the CTA may free TMEM
        mma_commit_if(issue, drain);
        wait(drain, 0);
      }
    }
  } else {
    reg_alloc<hs::kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    const int wg = (warp - 4) >> 2;  // 0..3
    const int g = wg >> 1;           // query tile
    const int hf = wg & 1;           // key half
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128u * g + 64u * hf;  // this half's scores; its P over their front
    const uint32_t tO = tmem + lane_off + 256u + 128u * g + 64u * hf;
    const float sl2 = p.scale_log2;
    const bool band = (p.mode == TC_BAND);
    const int my_h = g ? w.h1 : w.h0;
    const int my_row0 = g ? w.qrow1 : w.qrow0;
    const int my_rows = g ? w.rows1 : w.rows0;
    const int qrow = my_row0 + r;
    float m = -INFINITY;  // running reference max of this half's raw scores
    float l = 0.f;        // running row sum of this half relative to m
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
      if (!__all_sync(0xffffffffu, mbar_wait(s_full(g), j & 1, p.err, ERR_WAIT_SOFTMAX))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // ---- masks: unused tail of the last tile of a key run, band edges.  The
      // scores are read from TMEM twice, 32 columns at a time (for the row max,
      // then for the exponentials), so a thread holds 32 of them at once
      const int kbase = krow + 64 * hf;  // key of this half's column 0
      const int hvalid = kvalid - 64 * hf;
      bool full_cols = hvalid >= 64;
      int lo_key = -0x7fffffff, hi_key = 0x7fffffff;
      if (band) {
        const bool inside = (kbase >= my_row0 + my_rows - 1 - p.W + 1) && (kbase + 63 <= my_row0) && hvalid >= 64;
        if (!inside) {
          full_cols = false;
          lo_key = qrow - p.W + 1;
          hi_key = qrow;
        }
      }
      auto mask32 = [&](uint32_t* v, int c0) {
        if (full_cols) return;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int key = kbase + c0 + c;
          if (c0 + c >= hvalid || key < lo_key || key > hi_key) v[c] = __float_as_uint(-INFINITY);
        }
      };
      float a[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) a[k] = -INFINITY;
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tS + c0, v);
        tmem_wait_ld();
        mask32(v, c0);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          a[k] = max3f(a[k], max3f(__uint_as_float(v[k]), __uint_as_float(v[8 + k]), __uint_as_float(v[16 + k])),
                       __uint_as_float(v[24 + k]));
      }
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
        // this half's O is complete up to key tile j-1 (the commit that
        // signalled S_j covers both halves' earlier PVs): rescale in place
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t orr[32];
          tmem_ld32(tO + c0, orr);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
          tmem_st32(tO + c0, orr);
        }
        tmem_wait_st();
      }
      l *= alpha;
      // ---- P = 2^(s*scale - m*scale): 32 scores at a time, 16 packed bf16 pairs
      // stored over the front of this half's (already read) score columns
      const float nb = (m == -INFINITY) ? 0.f : -m * sl2;
      const float2 c2 = make_float2(sl2, sl2);
      const float2 nb2 = make_float2(nb, nb);
      float2 acc[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c0 = 0; c0 < 64; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tS + c0, v);
        tmem_wait_ld();
        mask32(v, c0);
        uint32_t pk[16];
#pragma unroll
        for (int pi = 0; pi < 16; ++pi) {
          const float2 x =
              __ffma2_rn(make_float2(__uint_as_float(v[2 * pi]), __uint_as_float(v[2 * pi + 1])), c2, nb2);
          float2 pr;
          if ((pi & 7) < kPolyPairs<64>) {
            pr = exp2_poly2(x);
          } else {
            pr.x = ex2_approx(x.x);
            pr.y = ex2_approx(x.y);
          }
          acc[pi & 3] = __fadd2_rn(acc[pi & 3], pr);
          pk[pi] = pack_bf16x2(pr.x, pr.y);
        }
        tmem_st16(tS + c0 / 2, pk);
      }
      l += ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) + ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full(g, hf));
    }
    // ---- epilogue: merge the two key halves of each row, then store
    float2* xch = reinterpret_cast<float2*>(gbase + hs::kOffX);  // [g][hf][row]
    float M = -INFINITY, a_self = 0.f, a_other = 0.f, L = 0.f;
    const bool have = active && ok &&
                      __all_sync(0xffffffffu, mbar_wait(o_full(g), 0, p.err, ERR_WAIT_EPI));
    if (have) xch[(g * 2 + hf) * kRows + r] = make_float2(m == -INFINITY ? -INFINITY : m * sl2, l);
    // the two warpgroups of this tile meet (named barrier 2 + g, 256 threads)
    __syncwarp();
    if (g == 0)
      asm volatile("bar.sync 2, 256;" ::: "memory");
    else
      asm volatile("bar.sync 3, 256;" ::: "memory");
    if (have) {
      const float2 mine = xch[(g * 2 + hf) * kRows + r];
      const float2 other = xch[(g * 2 + (hf ^ 1)) * kRows + r];
      M = fmaxf(mine.x, other.x);
      a_self = (mine.x == -INFINITY) ? 0.f : exp2f(mine.x - M);
      a_other = (other.x == -INFINITY) ? 0.f : exp2f(other.x - M);
      L = a_self * mine.y + a_other * other.y;
      tc_fence_after();
      // this half's thread writes output columns [32 hf, 32 hf + 32) of its row,
      // 16 at a time
      const uint32_t tO0 = tmem + lane_off + 256u + 128u * g;  // O of key half 0; half 1 at +64
      const float w0 = hf ? a_other : a_self;
      const float w1 = hf ? a_self : a_other;
      const bool store = r < my_rows;
      const int row = my_row0 + r;
      const float inv = 1.f / L;
      const int64_t out_ld = p.out_ld ? p.out_ld : static_cast<int64_t>(p.Hq) * D;
      const int64_t idx = (static_cast<int64_t>(w.split) * p.Nq + row) * p.Hq + my_h;
#pragma unroll 1
      for (int c0 = 32 * hf; c0 < 32 * hf + 32; c0 += 16) {
        uint32_t o0[16], o1[16];
        tmem_ld16(tO0 + c0, o0);
        tmem_ld16(tO0 + 64 + c0, o1);
        tmem_wait_ld();
        float f[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) f[e] = w0 * __uint_as_float(o0[e]) + w1 * __uint_as_float(o1[e]);
        if (store && w.split < 0) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) +
                               (static_cast<int64_t>(w.b) * p.Nq + row) * out_ld +
                               static_cast<int64_t>(p.out_h0 + my_h) * D + c0;
#pragma unroll
          for (int e = 0; e < 16; e += 8) {
            uint4 v;
            v.x = pack_bf16x2(f[e] * inv, f[e + 1] * inv);
            v.y = pack_bf16x2(f[e + 2] * inv, f[e + 3] * inv);
            v.z = pack_bf16x2(f[e + 4] * inv, f[e + 5] * inv);
            v.w = pack_bf16x2(f[e + 6] * inv, f[e + 7] * inv);
            *reinterpret_cast<uint4*>(dst + e) = v;
          }
        } else if (store) {
          // split-KV partial of the row: the merged numerator relative to M
          float* dst = p.part_o + idx * D + c0;
#pragma unroll
          for (int e = 0; e < 16; e += 4)
            *reinterpret_cast<float4*>(dst + e) = make_float4(f[e], f[e + 1], f[e + 2], f[e + 3]);
        }
      }
      if (store && w.split >= 0 && hf == 0) {
        p.part_ml[idx * 2 + 0] = M;
        p.part_ml[idx * 2 + 1] = L;
      }
    } else if (T == 0 && w.split >= 0 && (g == 0 || has_b) && r < my_rows && hf == 0) {
      // empty split: contributes nothing to the merge
      const int row = my_row0 + r;
      const int64_t idx = (static_cast<int64_t>(w.split) * p.Nq + row) * p.Hq + my_h;
      p.part_ml[idx * 2 + 0] = -INFINITY;
      p.part_ml[idx * 2 + 1] = 0.f;
    }
    if (w.split >= 0) {
      // ---- split-KV merge in the item's last CTA (as in attn_tc_kernel): the
      // 512 softmax threads meet, one counts this CTA in, and the CTA that
      // completes the count merges the item's partials; each half's threads
      // take 32 of the 64 output columns of their row
      volatile int* flag = reinterpret_cast<volatile int*>(gbase + hs::kOffTmem + 8);
      const int item = static_cast<int>(blockIdx.x % (static_cast<unsigned>(p.Hq) * p.n_pairs));
      __threadfence();
      __syncwarp();
      asm volatile("bar.sync 1, 512;" ::: "memory");
      if (warp == 4 && lane == 0) *flag = (atomicAdd(p.split_cnt + item, 1) == p.splits - 1) ? 1 : 0;
      asm volatile("bar.sync 1, 512;" ::: "memory");
      if (*flag) {
        __threadfence();
        if ((g == 0 || has_b) && r < my_rows) {
          const int row = my_row0 + r;
          const int64_t stride = static_cast<int64_t>(p.Nq) * p.Hq;
          const int64_t base_idx = static_cast<int64_t>(row) * p.Hq + my_h;
          float Mx = -INFINITY;
          for (int c = 0; c < p.splits; ++c) Mx = fmaxf(Mx, __ldcg(p.part_ml + (c * stride + base_idx) * 2));
          float Lx = 0.f;
          for (int c = 0; c < p.splits; ++c) {
            const float2 ml = __ldcg(reinterpret_cast<const float2*>(p.part_ml + (c * stride + base_idx) * 2));
            Lx = fmaf((ml.x == -INFINITY) ? 0.f : exp2f(ml.x - Mx), ml.y, Lx);
          }
          const float inv = 1.f / Lx;
          const int64_t out_ld = p.out_ld ? p.out_ld : static_cast<int64_t>(p.Hq) * D;
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(row) * out_ld +
                               static_cast<int64_t>(p.out_h0 + my_h) * D;
#pragma unroll 1
          for (int c0 = 32 * hf; c0 < 32 * hf + 32; c0 += 16) {
            float o[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) o[e] = 0.f;
            for (int c = 0; c < p.splits; ++c) {
              const float m_c = __ldcg(p.part_ml + (c * stride + base_idx) * 2);
              const float wc = (m_c == -INFINITY) ? 0.f : exp2f(m_c - Mx);
              const float4* src = reinterpret_cast<const float4*>(p.part_o + (c * stride + base_idx) * D + c0);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float4 v = __ldcg(src + e);
                o[4 * e] = fmaf(wc, v.x, o[4 * e]);
                o[4 * e + 1] = fmaf(wc, v.y, o[4 * e + 1]);
                o[4 * e + 2] = fmaf(wc, v.z, o[4 * e + 2]);
                o[4 * e + 3] = fmaf(wc, v.w, o[4 * e + 3]);
              }
            }
#pragma unroll
            for (int e = 0; e < 16; e += 8) {
              uint4 v;
              v.x = pack_bf16x2(o[e] * inv, o[e + 1] * inv);
              v.y = pack_bf16x2(o[e + 2] * inv, o[e + 3] * inv);
              v.z = pack_bf16x2(o[e + 4] * inv, o[e + 5] * inv);
              v.w = pack_bf16x2(o[e + 6] * inv, o[e + 7] * inv);
              *reinterpret_cast<uint4*>(dst + c0 + e) = v;
            }
          }
        }
        if (warp == 4 && lane == 0) p.split_cnt[item] = 0;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

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

cudaError_t launch_hs(const TcParams& p, int64_t n_items, cudaStream_t stream) {
  static DeviceOnce attr_set;  // devices on which the smem opt-in was set
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (!attr_set.done(dev)) {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_hs_kernel);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * 20 < 4 * hs::kRegsCtl + 16 * hs::kRegsSoftmax) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(attn_hs_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, hs::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set.mark(dev);
  }
  attn_hs_kernel<<<static_cast<unsigned>(n_items), hs::kThreads, hs::kSmemBytes, stream>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_attn_tc(const TcParams& p, int head_dim, int64_t n_items, cudaStream_t stream) {
  if (n_items <= 0) return cudaSuccess;
  if (head_dim == 64 && SWA_KEY_HALVES) return launch_hs(p, n_items, stream);
  if (head_dim == 64) return launch_tc_d<64>(p, n_items, stream);
  if (head_dim == 128) return launch_tc_d<128>(p, n_items, stream);
  return cudaErrorInvalidValue;
}

}  // namespace swa
