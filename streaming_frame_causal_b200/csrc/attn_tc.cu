// attn_tc.cu -- persistent tcgen05 / TMEM / TMA attention kernel for sm_100a
// (bf16 in, f32 accumulate, bf16 out), used by the frame-causal prefill, the
// streaming attend and the token-band GQA prefill.
//
// What it computes: O = softmax(Q K^T / sqrt(D)) V over the keys the schedule
// lists for a 128-row query tile ("Sliding Window Attention Mechanism in
// AggregatorStream", "Mask Generation in CausalAttention": only in-window
// frames are visible; "KV Cache Eviction Strategy": only retained frames are in
// the cache; sliding-window explainer: token band t-W+1..t).
//
// One CTA per SM (384 threads = 3 warpgroups) loops over work units:
//   warp 0      TMA producer: each unit's Q tiles, then its K/V key tiles into a ring
//   warp 1      TMEM allocator; lane 0 issues every tcgen05.mma
//   warps 2-3   idle
//   warps 4-7   softmax for query tile A (one thread per query row)
//   warps 8-11  softmax for query tile B
// A unit is a pair of 128-row query tiles (A, B) and a run of key tiles.  The
// prefill and band modes hand whole items to CTAs round-robin in longest-first
// order; the streaming mode cuts the flattened (item, key tile) space into one
// equal contiguous share per CTA, so a unit may cover part of an item and then
// writes a partial (max, sum, numerator) that the combine kernel merges.  The K/V
// ring, the S/P hand-offs and the Q reloads run straight across unit boundaries.
//
// After set-up, warpgroup 0 gives registers back (setmaxnreg.dec to 64) and the
// softmax warpgroups take them (setmaxnreg.inc to 216), so a thread can hold a
// whole 128-column row of S in registers.  The two query tiles ping-pong: while
// softmax A turns S_A into P_A, the tensor core runs P_B V and Q_B K^T, and the
// other way round.  S (f32, 128 columns), P (bf16 pairs, 64 columns) and O (f32,
// D columns) of each tile live in tensor memory; P feeds the PV product straight
// from TMEM (A operand), so the only shared-memory operands are Q, K and V,
// staged by TMA with 128-byte swizzle.  Online softmax uses exp2 with the scale
// folded in and skips rescaling O unless the running maximum grows by more than
// 2^8 (exact after the final division by the row sum).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cmath>
#include <cstdint>

#include "internal.h"
#include "exp2_poly.cuh"
#include "ptx.cuh"
#include "tile_sched.h"

namespace swa {

namespace {

constexpr int kThreads = 384;     // 3 warpgroups
constexpr int kRegsLaunch = 168;  // registers per thread at launch (384 x 168 = 64512 of 65536)
constexpr int kRegsCtl = 64;      // warpgroup 0 (TMA producer, MMA issuer) after setmaxnreg.dec
constexpr int kRegsSoftmax = 216; // warpgroups 1-2 (softmax) after setmaxnreg.inc
static_assert(4 * kRegsCtl + 8 * kRegsSoftmax <= 12 * kRegsLaunch,
              "register split must fit the pool the CTA was launched with");
constexpr int kRows = kTileRows;       // 128
constexpr int kMaxUnits = 256;         // work units one CTA may hold (host sizes the grid to fit)
constexpr int kSubBytes = 128 * 128;   // one 128-row x 64-column bf16 sub-tile (16 KB)

template <int D, bool kPersist>
struct Plan {
  static_assert(D == 64 || D == 128, "tcgen05 path: head_dim 64 or 128");
  static constexpr int kSubs = D / 64;                 // 64-column sub-tiles per row
  static constexpr int kTileBytes = kRows * D * 2;     // Q, K or V tile
  static constexpr int kStages = (D == 64) ? 4 : 2;    // K/V ring depth
  // Tensor-memory columns.  D = 64: S 2x128 | P 2x64 | O 2x64.  D = 128: S 2x128 |
  // O 2x128, and P (64 columns of bf16 pairs) reuses the first half of its own
  // S once the softmax has read S: the next QK^T that overwrites S is issued by
  // the same thread after the PV that reads P, and tcgen05.mma operations from
  // one thread execute in issue order.
  SWA_DEV static uint32_t col_s(int g) { return g ? 128u : 0u; }
  SWA_DEV static uint32_t col_p(int g) { return D == 64 ? (g ? 320u : 256u) : col_s(g); }
  SWA_DEV static uint32_t col_o(int g) { return D == 64 ? (g ? 448u : 384u) : (g ? 384u : 256u); }
  static constexpr uint32_t kTmemCols = 512;
  // shared-memory layout (offsets from a 1024-aligned base)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  // q_full[2] q_empty[2] kv_full[S] kv_empty[S] s_full[2] p_full[2] o_full[2] drain
  static constexpr int kNumBars = 4 + 2 * kStages + 6 + 1;
  static constexpr int kOffTmem = kOffBar + kNumBars * 8;
  static constexpr int kOffUnits = (kOffTmem + 16 + 127) / 128 * 128;  // unit descriptors (int4)
  static constexpr int kSmemBytes = kOffUnits + (kPersist ? kMaxUnits * 16 : 0) + 1024;  // + alignment slack
  static_assert(kOffQ % 1024 == 0 && kOffK % 1024 == 0 && kOffV % 1024 == 0 && kTileBytes % 1024 == 0,
                "swizzled operand tiles need 1024-byte alignment");
  static_assert(kOffBar % 8 == 0 && kOffUnits % 16 == 0, "barrier / descriptor alignment");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");
};

// One work unit: the query tiles, the key runs and the key-tile range.
struct Work {
  int b, kvh;
  int h0, h1;          // query heads of tiles A and B
  int qrow0, qrow1;    // first query row of tiles A and B (row index in the Q tensor, per batch)
  int rows0, rows1;    // valid query rows (0 = tile absent)
  int t_begin, t_end;  // key-tile range of this unit
  int item;            // work item the unit belongs to
  int slot;            // >= 0: partial slot of a split item; -1: write the final output
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

SWA_DEV int total_tiles_of(const int* glen, int nseg) {
  int T = 0;
  for (int s = 0; s < nseg; ++s) T += cdiv(__ldg(glen + s), kRows);
  return T;
}

SWA_DEV int64_t imin64(int64_t a, int64_t b) { return a < b ? a : b; }

// Unit descriptor as kept in shared memory: item, key-tile range, partial slot.
// Every role of the CTA walks the same list; the rest of a unit's description is
// recomputed from it when needed, so little per-unit state stays in registers.
struct UnitDesc {
  int item, t_begin, t_end, slot;
};

// Thread 0 fills the CTA's unit list; returns the count.
SWA_DEV int build_units(const TcParams& p, int4* list) {
  int n = 0;
  if (p.mode == TC_STREAM) {
    const int ns = __ldg(p.meta_hdr + 5);
    const int nseg = (ns >= 0 && ns <= p.max_segs) ? ns : 0;
    const int T = total_tiles_of(p.seg_len, nseg);
    if (T <= 0) return 0;
    const int64_t total = static_cast<int64_t>(p.n_items) * T;
    int64_t L = (total + gridDim.x - 1) / gridDim.x;
    if (L < 1) L = 1;
    int64_t pos = imin64(total, static_cast<int64_t>(blockIdx.x) * L);
    const int64_t end = imin64(total, pos + L);
    while (pos < end && n < kMaxUnits) {
      const int item = static_cast<int>(pos / T);
      const int t0 = static_cast<int>(pos - static_cast<int64_t>(item) * T);
      const int t1 = static_cast<int>(imin64(T, t0 + (end - pos)));
      int slot = -1;
      if (!(t0 == 0 && t1 == T)) slot = static_cast<int>(blockIdx.x - (static_cast<int64_t>(item) * T) / L);
      list[n++] = make_int4(item, t0, t1, slot);
      pos += t1 - t0;
    }
    return n;
  }
  for (int64_t item = blockIdx.x; item < p.n_items && n < kMaxUnits; item += gridDim.x)
    list[n++] = make_int4(static_cast<int>(item), 0, -1, -1);  // t_end filled on expansion
  return n;
}

SWA_DEV void expand_unit(const TcParams& p, int4 d, Work& w) {
  w.grow = nullptr;
  w.glen = nullptr;
  w.nseg = 0;
  w.srow0 = w.slen0 = w.srow1 = w.slen1 = 0;
  w.item = d.x;
  w.t_begin = d.y;
  w.t_end = d.z;
  w.slot = d.w;
  if (p.mode == TC_FRAME) {
    const PrefillItem pi = prefill_item(d.x, p.B, p.Hq, p.F, p.n_pairs);
    w.b = pi.b;
    w.kvh = pi.h / (p.Hq / p.Hkv);
    w.h0 = w.h1 = pi.h;
    const int t0 = 2 * pi.pair;
    w.rows0 = qtile_rows(p.P, t0);
    w.rows1 = qtile_rows(p.P, t0 + 1);
    w.qrow0 = pi.f * p.P + t0 * kRows;
    w.qrow1 = w.qrow0 + kRows;
    int lo[2], hi[2];
    w.nseg = frame_intervals(pi.f, p.Wf, p.S, lo, hi);
    w.srow0 = lo[0] * p.P;
    w.slen0 = (hi[0] - lo[0]) * p.P;
    if (w.nseg > 1) {
      w.srow1 = lo[1] * p.P;
      w.slen1 = (hi[1] - lo[1]) * p.P;
    }
    w.t_begin = 0;
    w.t_end = cdiv(w.slen0, kRows) + (w.nseg > 1 ? cdiv(w.slen1, kRows) : 0);
  } else if (p.mode == TC_BAND) {
    const BandItem bi = band_item(d.x, p.B, p.Hq, p.Hkv, p.n_qtiles);
    w.b = bi.b;
    w.kvh = bi.kvh;
    const int t0 = bi.t * kRows;
    const int rows = imin(kRows, p.Nq - t0);
    w.h0 = bi.h0;
    w.h1 = bi.h1 < 0 ? bi.h0 : bi.h1;
    w.qrow0 = w.qrow1 = t0;
    w.rows0 = rows;
    w.rows1 = bi.h1 < 0 ? 0 : rows;
    int lo, hi;
    band_keys(t0, rows, p.W, &lo, &hi);
    w.nseg = 1;
    w.srow0 = lo;
    w.slen0 = hi - lo;
    w.t_begin = 0;
    w.t_end = cdiv(w.slen0, kRows);
  } else {  // TC_STREAM
    w.b = 0;
    const int h = d.x / p.n_pairs;
    const int pair = d.x - h * p.n_pairs;
    w.kvh = h / (p.Hq / p.Hkv);
    w.h0 = w.h1 = h;
    w.rows0 = qtile_rows(p.P, 2 * pair);
    w.rows1 = qtile_rows(p.P, 2 * pair + 1);
    w.qrow0 = 2 * pair * kRows;
    w.qrow1 = w.qrow0 + kRows;
    w.grow = p.seg_row;
    w.glen = p.seg_len;
    const int ns = __ldg(p.meta_hdr + 5);
    w.nseg = (ns >= 0 && ns <= p.max_segs) ? ns : 0;
  }
}

#ifndef SWA_POLY_PAIRS
#define SWA_POLY_PAIRS 3  // of every 8 column pairs, how many take 2^x on the FMA pipe
#endif

SWA_DEV float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// kPersist = false: one unit per CTA (item = blockIdx.x, all its key tiles);
// true: the CTA walks the unit list it builds in shared memory.
template <int D, bool kPersist>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(const __grid_constant__ TcParams p) {
  using PL = Plan<D, kPersist>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // barriers
  const uint32_t bar0 = base + PL::kOffBar;
  auto q_full = [&](int g) { return bar0 + 8u * g; };
  auto q_empty = [&](int g) { return bar0 + 8u * (2 + g); };
  auto kv_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (4 + PL::kStages + s); };
  auto s_full = [&](int g) { return bar0 + 8u * (4 + 2 * PL::kStages + g); };
  auto p_full = [&](int g) { return bar0 + 8u * (6 + 2 * PL::kStages + g); };
  auto o_full = [&](int g) { return bar0 + 8u * (8 + 2 * PL::kStages + g); };
  const uint32_t drain = bar0 + 8u * (10 + 2 * PL::kStages);
  const uint32_t tmem_slot = base + PL::kOffTmem;

  int4* units = reinterpret_cast<int4*>(gbase + PL::kOffUnits);
  __shared__ int n_units_sh;
  if (threadIdx.x == 0) {
    if (kPersist) n_units_sh = build_units(p, units);
    for (int g = 0; g < 2; ++g) {
      mbar_init(q_full(g), 1);
      mbar_init(q_empty(g), 1);
      mbar_init(s_full(g), 1);
      mbar_init(p_full(g), 128);
      mbar_init(o_full(g), 1);
    }
    for (int s = 0; s < PL::kStages; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, PL::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + PL::kOffTmem);

  const int n_units = kPersist ? n_units_sh : 1;
  auto unit_desc = [&](int u) { return kPersist ? units[u] : make_int4(static_cast<int>(blockIdx.x), 0, -1, -1); };
  Work w;

  if (warp < 4) {
    reg_dealloc<kRegsCtl>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- producer
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      int qcnt[2] = {0, 0};
      int J = 0;  // K/V tiles issued so far (all units)
      bool ok = true;
      for (int u = 0; u < n_units && ok; ++u) {
        expand_unit(p, unit_desc(u), w);
        const bool has_b = w.rows1 > 0;
        for (int g = 0; g < (has_b ? 2 : 1) && ok; ++g) {
          // the previous unit's Q_g must no longer be read by the tensor core
          if (qcnt[g] > 0 && !mbar_wait(q_empty(g), (qcnt[g] - 1) & 1, p.err, ERR_WAIT_TMA)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(q_full(g), PL::kTileBytes);
          for (int sub = 0; sub < PL::kSubs; ++sub)
            tma_load_4d(base + PL::kOffQ + g * PL::kTileBytes + sub * kSubBytes, &p.tm_q, q_full(g), sub * 64,
                        g ? w.h1 : w.h0, g ? w.qrow1 : w.qrow0, w.b);
          ++qcnt[g];
        }
        Cursor cur;
        if (ok && !cursor_seek(w, w.t_begin, cur)) {
          atomicOr(p.err, ERR_BAD_META);
          ok = false;
        }
        for (int j = w.t_begin; j < w.t_end && ok; ++j, ++J) {
          const int st = J % PL::kStages;
          if (J >= PL::kStages && !mbar_wait(kv_empty(st), ((J / PL::kStages) - 1) & 1, p.err, ERR_WAIT_TMA)) {
            ok = false;
            break;
          }
          if (cur.s >= w.nseg) {
            atomicOr(p.err, ERR_BAD_META);
            ok = false;
            break;
          }
          int krow, kvalid;
          cursor_tile(w, cur, &krow, &kvalid);
          mbar_arrive_expect_tx(kv_full(st), 2 * PL::kTileBytes);
          for (int sub = 0; sub < PL::kSubs; ++sub) {
            tma_load_4d(base + PL::kOffK + st * PL::kTileBytes + sub * kSubBytes, &p.tm_k, kv_full(st), sub * 64,
                        w.kvh, krow, w.b);
            tma_load_4d(base + PL::kOffV + st * PL::kTileBytes + sub * kSubBytes, &p.tm_v, kv_full(st), sub * 64,
                        w.kvh, krow, w.b);
          }
          cursor_next(w, cur);
        }
      }
      // drain: never leave the CTA with a bulk copy still writing its shared memory
      for (int j = J - PL::kStages; j < J; ++j) {
        if (j < 0) continue;
        mbar_wait(kv_full(j % PL::kStages), (j / PL::kStages) & 1, p.err, ERR_WAIT_TMA);
      }
      for (int g = 0; g < 2; ++g)
        if (qcnt[g] > 0) mbar_wait(q_full(g), (qcnt[g] - 1) & 1, p.err, ERR_WAIT_TMA);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 1);
      auto issue_qk = [&](int g, int st) {
        const uint32_t qa = base + PL::kOffQ + g * PL::kTileBytes;
        const uint32_t kb = base + PL::kOffK + st * PL::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kSubBytes + (kk & 3) * 32;
          mma_ss(tmem + PL::col_s(g), sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), idesc_qk,
                 kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int g, int st, bool acc) {
        const uint32_t vb = base + PL::kOffV + st * PL::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kRows / 16; ++kk) {
          mma_ts(tmem + PL::col_o(g), tmem + PL::col_p(g) + kk * 8, sdesc_sw128(vb + kk * 16 * 128, kSubBytes, 1024),
                 idesc_pv, (acc || kk > 0) ? 1u : 0u);
        }
      };
      int qcnt[2] = {0, 0};  // units that used Q_g
      int pcnt[2] = {0, 0};  // key tiles whose P_g has been consumed
      int J = 0;
      bool ok = true;
      bool issued = false;
      for (int u = 0; u < n_units && ok; ++u) {
        expand_unit(p, unit_desc(u), w);
        const bool has_b = w.rows1 > 0;
        const int T = w.t_end - w.t_begin;
        if (T <= 0) continue;
        ok = mbar_wait(q_full(0), qcnt[0] & 1, p.err, ERR_WAIT_MMA);
        if (ok && has_b) ok = mbar_wait(q_full(1), qcnt[1] & 1, p.err, ERR_WAIT_MMA);
        if (ok) ok = mbar_wait(kv_full(J % PL::kStages), (J / PL::kStages) & 1, p.err, ERR_WAIT_MMA);
        if (!ok) break;
        tc_fence_after();
        issued = true;
        issue_qk(0, J % PL::kStages);
        mma_commit(s_full(0));
        if (kPersist && T == 1) mma_commit(q_empty(0));
        if (has_b) {
          issue_qk(1, J % PL::kStages);
          mma_commit(s_full(1));
          if (kPersist && T == 1) mma_commit(q_empty(1));
        }
        for (int j = 0; j < T && ok; ++j) {
          const int st = (J + j) % PL::kStages;
          const int st1 = (J + j + 1) % PL::kStages;
          const bool more = j + 1 < T;
          if (!mbar_wait(p_full(0), pcnt[0] & 1, p.err, ERR_WAIT_MMA)) {
            ok = false;
            break;
          }
          ++pcnt[0];
          tc_fence_after();
          issue_pv(0, st, j > 0);
          if (more) {
            if (!mbar_wait(kv_full(st1), ((J + j + 1) / PL::kStages) & 1, p.err, ERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_qk(0, st1);
            mma_commit(s_full(0));
            if (kPersist && j + 2 == T) mma_commit(q_empty(0));
          }
          if (has_b) {
            if (!mbar_wait(p_full(1), pcnt[1] & 1, p.err, ERR_WAIT_MMA)) {
              ok = false;
              break;
            }
            ++pcnt[1];
            tc_fence_after();
            issue_pv(1, st, j > 0);
          }
          mma_commit(kv_empty(st));
          if (has_b && more) {
            issue_qk(1, st1);
            mma_commit(s_full(1));
            if (kPersist && j + 2 == T) mma_commit(q_empty(1));
          }
          if (!more) {
            mma_commit(o_full(0));
            if (kPersist && has_b) mma_commit(o_full(1));
          }
        }
        J += T;
        ++qcnt[0];
        if (has_b) ++qcnt[1];
      }
      // drain every MMA this thread issued before the CTA may free TMEM
      if (issued) {
        mma_commit(drain);
        mbar_wait(drain, 0, p.err, ERR_WAIT_MMA);
      }
    }
  } else {
    reg_alloc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax
    const int g = (warp - 4) >> 2;  // 0: tile A, 1: tile B
    const int quarter = warp & 3;   // TMEM lane quarter this warp may access
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_off + PL::col_s(g);
    const uint32_t tP = tmem + lane_off + PL::col_p(g);
    const uint32_t tO = tmem + lane_off + PL::col_o(g);
    const float sl2 = p.scale_log2;
    const bool band = (p.mode == TC_BAND);
    int scnt = 0;  // key tiles this warpgroup has processed (all units)
    int ucnt = 0;  // units this warpgroup has finished
    bool ok = true;
    for (int u = 0; u < n_units && ok; ++u) {
      expand_unit(p, unit_desc(u), w);
      const bool has_b = w.rows1 > 0;
      if (g == 1 && !has_b) continue;
      const int T = w.t_end - w.t_begin;
      if (T <= 0) continue;
      const int my_row0 = g ? w.qrow1 : w.qrow0;
      const int my_rows = g ? w.rows1 : w.rows0;
      const int qrow = my_row0 + r;  // query token (band mode: absolute position)
      float m = -INFINITY;           // running reference max of raw scores
      float l = 0.f;                 // running row sum relative to m
      Cursor cur;
      if (!cursor_seek(w, w.t_begin, cur)) {
        ok = false;
        break;
      }
      for (int j = 0; j < T && ok; ++j, ++scnt) {
        if (cur.s >= w.nseg) {
          ok = false;
          break;
        }
        int krow, kvalid;
        cursor_tile(w, cur, &krow, &kvalid);
        cursor_next(w, cur);
        if (!__all_sync(0xffffffffu, mbar_wait(s_full(g), scnt & 1, p.err, ERR_WAIT_SOFTMAX))) {
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
          const bool inside =
              (krow >= my_row0 + my_rows - 1 - p.W + 1) && (krow + kvalid - 1 <= my_row0) && kvalid == kRows;
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
          for (int k = 0; k < 8; ++k) a[k] = max3f(a[k], __uint_as_float(s[c + k]), __uint_as_float(s[c + 8 + k]));
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
          // O of this tile is complete up to key tile j-1 (the commit that
          // signalled S_j covers the earlier PV), so it can be rescaled in place
#pragma unroll
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
        // ---- P = 2^(s*scale - m*scale): MUFU for most column pairs, the
        // polynomial on the FMA pipe for SWA_POLY_PAIRS of every 8; packed bf16
        // pairs overwrite the front of s (pair pi reads s[2pi], s[2pi+1] >= pi)
        const float nb = (m == -INFINITY) ? 0.f : -m * sl2;
        const float2 c2 = make_float2(sl2, sl2);
        const float2 nb2 = make_float2(nb, nb);
        float2 acc[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
        for (int pi = 0; pi < 64; ++pi) {
          const float2 x = __ffma2_rn(make_float2(__uint_as_float(s[2 * pi]), __uint_as_float(s[2 * pi + 1])), c2, nb2);
          float2 pr;
          if ((pi & 7) < SWA_POLY_PAIRS) {
            pr = exp2_poly2(x);
          } else {
            pr.x = ex2_approx(x.x);
            pr.y = ex2_approx(x.y);
          }
          acc[pi & 3] = __fadd2_rn(acc[pi & 3], pr);
          s[pi] = pack_bf16x2(pr.x, pr.y);
        }
        l += ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y)) + ((acc[2].x + acc[2].y) + (acc[3].x + acc[3].y));
        tmem_st32(tP + 0, s);
        tmem_st32(tP + 32, s + 32);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full(g));
      }
      if (!ok) break;
      // ---- epilogue of the unit: O / l as bf16, or the partial (max, sum, O)
      if (!__all_sync(0xffffffffu, mbar_wait(o_full(kPersist ? g : 0), ucnt & 1, p.err, ERR_WAIT_EPI))) {
        ok = false;
        break;
      }
      ++ucnt;
      tc_fence_after();
      if (kPersist) expand_unit(p, unit_desc(u), w);  // re-read: keeps unit fields out of the tile loop
      const int my_h = g ? w.h1 : w.h0;
      const bool store = r < my_rows;
      const int row = my_row0 + r;
      const float inv = 1.f / l;
      const int64_t fidx = (static_cast<int64_t>(w.b) * p.Nq + row) * p.Hq + my_h;
      const int64_t pidx =
          (static_cast<int64_t>(w.item) * p.max_units + (w.slot < 0 ? 0 : w.slot)) * 256 + g * kRows + r;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t orr[32];
        tmem_ld32(tO + c0, orr);
        tmem_wait_ld();
        if (!store) continue;
        if (w.slot < 0) {
          __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(p.out) + fidx * D + c0;
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
          float* dst = p.part_o + pidx * D + c0;
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            *reinterpret_cast<float4*>(dst + c) = make_float4(__uint_as_float(orr[c]), __uint_as_float(orr[c + 1]),
                                                              __uint_as_float(orr[c + 2]), __uint_as_float(orr[c + 3]));
        }
      }
      if (store && w.slot >= 0) {
        p.part_ml[pidx * 2 + 0] = m * sl2;
        p.part_ml[pidx * 2 + 1] = l;
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

// ---------------------------------------------------------------- combine
// Streaming attend: merge the partials of items that were split across CTAs,
// O = sum_u 2^(m_u - M) O_u / sum_u 2^(m_u - M) l_u (m in log2 units).  The
// split is recomputed from the same shares the attend kernel used.  One warp per
// (query row, head); items a single CTA finished were written directly.
template <int D>
__global__ void __launch_bounds__(256) combine_kernel(const TcParams p, int grid) {
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= p.P * p.Hq) return;
  const int row = gw / p.Hq, h = gw - row * p.Hq;
  const int item = h * p.n_pairs + row / 256;
  const int n = __ldg(p.meta_hdr + 5);
  const int nseg = (n >= 0 && n <= p.max_segs) ? n : 0;
  const int T = total_tiles_of(p.seg_len, nseg);
  if (T <= 0) return;
  const int64_t total = static_cast<int64_t>(p.n_items) * T;
  int64_t L = (total + grid - 1) / grid;
  if (L < 1) L = 1;
  const int64_t first = (static_cast<int64_t>(item) * T) / L;
  const int64_t last = (static_cast<int64_t>(item + 1) * T - 1) / L;
  const int units = static_cast<int>(last - first + 1);
  if (units <= 1) return;
  const int64_t base = static_cast<int64_t>(item) * p.max_units * 256 + row % 256;
  float M = -INFINITY;
  for (int u = 0; u < units; ++u) M = fmaxf(M, p.part_ml[(base + u * 256) * 2]);
  constexpr int E = D / 32;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float Lsum = 0.f;
  for (int u = 0; u < units; ++u) {
    const int64_t idx = base + u * 256;
    const float mu = p.part_ml[idx * 2];
    if (mu == -INFINITY) continue;
    const float wgt = exp2f(mu - M);
    Lsum += wgt * p.part_ml[idx * 2 + 1];
    const float* src = p.part_o + idx * D;
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] += wgt * src[lane + 32 * e];
  }
  const float inv = 1.f / Lsum;
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + (static_cast<int64_t>(row) * p.Hq + h) * D;
#pragma unroll
  for (int e = 0; e < E; ++e) out[lane + 32 * e] = __float2bfloat16_rn(acc[e] * inv);
}

template <int D, bool kPersist>
cudaError_t launch_tc_d(const TcParams& p, int grid, cudaStream_t stream) {
  static int attr_dev_mask = 0;  // devices on which the smem opt-in was set (first 31)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const int bit = 1 << (dev & 31);
  if (!(attr_dev_mask & bit)) {
    // the setmaxnreg split moves registers inside the pool the CTA is launched
    // with; refuse to launch a build whose pool would be too small (the
    // increasing warpgroups would otherwise wait forever)
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_tc_kernel<D, kPersist>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs * 12 < 4 * kRegsCtl + 8 * kRegsSoftmax) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(attn_tc_kernel<D, kPersist>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Plan<D, kPersist>::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_dev_mask |= bit;
  }
  attn_tc_kernel<D, kPersist><<<static_cast<unsigned>(grid), kThreads, Plan<D, kPersist>::kSmemBytes, stream>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

int tc_smem_bytes(int head_dim) {
  return head_dim == 64 ? Plan<64, true>::kSmemBytes : head_dim == 128 ? Plan<128, true>::kSmemBytes : -1;
}

cudaError_t launch_attn_tc(const TcParams& p, int head_dim, int grid, cudaStream_t stream) {
  if (grid <= 0) return cudaSuccess;
  const bool persist = (p.mode == TC_STREAM);
  if (head_dim == 64) return persist ? launch_tc_d<64, true>(p, grid, stream) : launch_tc_d<64, false>(p, grid, stream);
  if (head_dim == 128)
    return persist ? launch_tc_d<128, true>(p, grid, stream) : launch_tc_d<128, false>(p, grid, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_stream_combine(const TcParams& p, int head_dim, int grid, cudaStream_t stream) {
  const int warps = p.P * p.Hq;
  const int blocks = (warps + 7) / 8;
  if (blocks == 0) return cudaSuccess;
  if (head_dim == 64)
    combine_kernel<64><<<blocks, 256, 0, stream>>>(p, grid);
  else if (head_dim == 128)
    combine_kernel<128><<<blocks, 256, 0, stream>>>(p, grid);
  else
    return cudaErrorInvalidValue;
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swa
