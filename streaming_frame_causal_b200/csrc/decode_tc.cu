// decode_tc.cu -- GQA decode against the rolling KV cache on the tensor cores
// (sm_100a), bf16 in, f32 accumulate, head_dim 64 or 128.
//
// What it computes (sliding-window explainer, rolling-buffer decode): the new
// token's G query heads of a KV group attend, with softmax(q k^T / sqrt(D)), to
// the valid slots of the group's W-slot cache, the new token's own K/V already
// written into slot pos mod W (decode_append_kernel runs first).
//
// Layout of the work.  With one query token there are only G <= 16 query rows
// per (batch, KV head), so the products run with the keys as the M dimension:
//   S^T[128 keys x 16] = K_tile[128 x D] . Q^T        (A = K, K-major; B = Q, K-major)
//   O^T[128 x 16]     += V_tile^T[. x 128] . P^T      (A = V, MN-major; B = P^T, K-major)
// (the second product always has M = 128; at head_dim 64 its rows 64..127 are
// never read)
// S^T lands in tensor memory with one key per lane, so the softmax is spread
// over 128 threads (one key each, G scores per thread); the head-wise maximum
// of a tile is a warp shuffle reduction plus an exchange between four warps.
// P^T goes to shared memory in the 128-byte-swizzled K-major layout and feeds
// the second product; O^T (lane = output dimension) is rescaled in place when a
// head's running maximum grows by more than 2^8.  Columns G..15 of S^T and O^T
// come from neighbouring heads or stale P rows and are never read.
//
// Work: units of (batch, KV head, piece of the key range), pieces of whole
// 128-key tiles.  A persistent CTA per SM takes units c, c + grid, ... and runs
// them back to back: K/V tiles flow through a three-stage ring across unit
// boundaries, Q is double-buffered, and each unit's (O, max, sum) is a partial
// that decode_combine_kernel merges.
//
// CTA (192 threads): warp 0 TMA producer, warp 1 TMEM allocator and (lane 0)
// MMA issuer, warps 2-5 softmax (warp w handles the TMEM lane quarter w mod 4).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"
#include "tile_sched.h"

namespace swa {
namespace {

constexpr int kTcdThreads = 192;
constexpr int kTcdKeys = 128;       // keys per tile (M of the first product)
constexpr int kTcdN = 16;           // query-head columns (N of both products; G <= 16 used)
constexpr int kTcdSub = kTcdKeys * 128;           // one 64-column swizzled sub-tile of K or V: 16 KB
constexpr int kTcdSmallSub = kTcdN * 128;         // Q or P^T sub-tile: 16 rows x 128 bytes
constexpr int kTcdSmall = 2 * kTcdSmallSub;       // Q or P^T buffer: 4 KB
constexpr uint32_t kTcdTmemCols = 64;               // S^T 2 x 16 | O^T 16 (+ 16 unused)

// Shared-memory plan per head_dim: the K/V ring, 2 Q and 2 P^T buffers, the
// softmax exchange area, barriers.  At head_dim 64 a K or V tile is one
// 64-column sub-tile and the ring is deeper (five 32 KB stages).
template <int D>
struct TcdPlan {
  static_assert(D == 64 || D == 128, "head_dim");
  static constexpr int kSubs = D / 64;
  static constexpr int kStages = (D == 64) ? 5 : 3;
  static constexpr int kTile = kSubs * kTcdSub;       // K (or V) tile
  static constexpr int kStage = 2 * kTile;            // K + V
  static constexpr int kOffQ = kStages * kStage;      // 2 Q buffers
  static constexpr int kOffP = kOffQ + 2 * kTcdSmall; // 2 P^T buffers
  static constexpr int kOffRed = kOffP + 2 * kTcdSmall;  // [2][4][16] tile maxima, [4][16] row sums
  static constexpr int kOffBar = kOffRed + 3 * 4 * kTcdN * 4;
  static constexpr int kNumBars = 2 + 2 + 2 * kStages + 2 + 2 + 2 + 3 + 1;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffTmemSlot + 16 + 1024;  // + alignment slack
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

// kind::f16 instruction descriptor with A MN-major (transpose A, bit 15)
constexpr uint32_t kIdescS = idesc_bf16_f32(128, kTcdN, 0);
constexpr uint32_t kIdescO = idesc_bf16_f32(128, kTcdN, 0) | (1u << 15);

// 2-D tiled bulk tensor load; c0 is 0 or 64 (the 16-byte rule holds)
SWA_DEV void tma_load_2d(uint32_t dst, const void* tmap, uint32_t mbar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(mbar)
      : "memory");
}

SWA_DEV void st_shared_b16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

SWA_DEV void st_shared_zero16(uint32_t addr) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0u) : "memory");
}

struct TcdUnit {
  int b, kvh, piece, t_begin, t_end, T;
};

SWA_DEV TcdUnit tcd_unit(const DecodeParams& p, int unit) {
  TcdUnit u;
  const int item = unit / p.chunks;
  u.piece = unit - item * p.chunks;
  u.b = item / p.Hkv;
  u.kvh = item - u.b * p.Hkv;
  u.t_begin = u.piece * p.chunk_len;
  u.t_end = imin(u.t_begin + p.chunk_len, p.n_valid);
  u.T = u.t_end > u.t_begin ? cdiv(u.t_end - u.t_begin, kTcdKeys) : 0;
  return u;
}

template <int D, int G>
__global__ void __launch_bounds__(kTcdThreads, 1) decode_tc_kernel(const __grid_constant__ DecodeParams p) {
  static_assert(G >= 1 && G <= kTcdN, "query heads per KV head");
  using PL = TcdPlan<D>;
  constexpr int kTcdStages = PL::kStages;
  constexpr int kTcdStage = PL::kStage;
  constexpr int kTcdTile = PL::kTile;
  constexpr int kOffQ = PL::kOffQ;
  constexpr int kOffP = PL::kOffP;
  constexpr int kOffRed = PL::kOffRed;
  constexpr int kOffBar = PL::kOffBar;
  constexpr int kOffTmemSlot = PL::kOffTmemSlot;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_units = p.B * p.Hkv * p.chunks;
  griddep_launch_dependents();  // the combine launches now and waits for this grid

  const uint32_t bar0 = base + kOffBar;
  auto q_full = [&](int i) { return bar0 + 8u * i; };
  auto q_free = [&](int i) { return bar0 + 8u * (2 + i); };
  auto kv_full = [&](int s) { return bar0 + 8u * (4 + s); };
  auto kv_empty = [&](int s) { return bar0 + 8u * (4 + kTcdStages + s); };
  constexpr int kB = 4 + 2 * kTcdStages;
  auto s_full = [&](int i) { return bar0 + 8u * (kB + i); };
  auto p_full = [&](int i) { return bar0 + 8u * (kB + 2 + i); };
  auto p_free = [&](int i) { return bar0 + 8u * (kB + 4 + i); };
  const uint32_t o_done = bar0 + 8u * (kB + 6);  // every second product complete
  const uint32_t o_full = bar0 + 8u * (kB + 7);  // a unit's last second product complete
  const uint32_t drain = bar0 + 8u * (kB + 8);
  // barrier of the 128 softmax threads (an mbarrier, so the wait is bounded)
  const uint32_t xbar = bar0 + 8u * (kB + 9);

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full(i), 1);
      mbar_init(q_free(i), 1);
      mbar_init(s_full(i), 1);
      mbar_init(p_full(i), 128);
      mbar_init(p_free(i), 1);
    }
    for (int s = 0; s < kTcdStages; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    mbar_init(o_done, 1);
    mbar_init(o_full, 1);
    mbar_init(drain, 1);
    mbar_init(xbar, 128);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(base + kOffTmemSlot, kTcdTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + kOffTmemSlot);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      tma_prefetch_desc(&p.tm_q);
      int lu = 0, jj = 0;  // units loaded, key tiles loaded
      bool ok = true;
      for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
        const TcdUnit u = tcd_unit(p, unit);
        if (u.T == 0) continue;
        const int qb = lu & 1;
        if (lu >= 2 && !mbar_wait(q_free(qb), ((lu >> 1) - 1) & 1, p.err, ERR_WAIT_TMA)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(q_full(qb), PL::kSubs * kTcdSmallSub);
        for (int sub = 0; sub < PL::kSubs; ++sub)
          tma_load_2d(base + kOffQ + qb * kTcdSmall + sub * kTcdSmallSub, &p.tm_q, q_full(qb), sub * 64,
                      u.b * p.Hq + u.kvh * G);
        // the new token's append (the kernel ahead, programmatic launch) must have
        // landed before the first cache tile is read; Q is an input of its own
        if (lu == 0) griddep_wait();
        ++lu;
        for (int j = 0; j < u.T; ++j, ++jj) {
          const int st = jj % kTcdStages;
          if (jj >= kTcdStages && !mbar_wait(kv_empty(st), ((jj / kTcdStages) - 1) & 1, p.err, ERR_WAIT_TMA)) {
            ok = false;
            break;
          }
          const int row = u.t_begin + j * kTcdKeys;
          const uint32_t dst = base + st * kTcdStage;
          mbar_arrive_expect_tx(kv_full(st), kTcdStage);
          for (int sub = 0; sub < PL::kSubs; ++sub) {
            tma_load_4d(dst + sub * kTcdSub, &p.tm_k, kv_full(st), sub * 64, u.kvh, row, u.b);
            tma_load_4d(dst + kTcdTile + sub * kTcdSub, &p.tm_v, kv_full(st), sub * 64, u.kvh, row, u.b);
          }
        }
      }
      // never leave with a bulk copy still landing in shared memory
      for (int j = jj - kTcdStages; j < jj; ++j)
        if (j >= 0) mbar_wait(kv_full(j % kTcdStages), (j / kTcdStages) & 1, p.err, ERR_WAIT_TMA);
      for (int i = lu - 2; i < lu; ++i)
        if (i >= 0) mbar_wait(q_full(i & 1), (i >> 1) & 1, p.err, ERR_WAIT_TMA);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint64_t dk0 = sdesc_sw128(base, 16, 1024);                    // K of stage 0 (A, K-major)
      // V of stage 0 (A, MN-major): the second 64-row group of M is the second
      // sub-tile at head_dim 128; at 64 it is the next 16 KB of shared memory
      // (rows D..127 of O^T, never read)
      const uint64_t dv0 = sdesc_sw128(base + kTcdTile, kTcdSub, 1024);
      const uint64_t dq0 = sdesc_sw128(base + kOffQ, 16, 1024);            // Q buffer 0 (B, K-major)
      const uint64_t dp0 = sdesc_sw128(base + kOffP, 16, 1024);            // P^T buffer 0 (B, K-major)
      constexpr uint64_t kStageStep = kTcdStage >> 4;
      constexpr uint64_t kSmallStep = kTcdSmall >> 4;
      auto issue_s = [&](int jj, int qb) {
        const uint64_t dk = dk0 + (jj % kTcdStages) * kStageStep;
        const uint64_t dq = dq0 + qb * kSmallStep;
        const uint32_t tS = tmem + (jj & 1) * kTcdN;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tS, dk + (((kk >> 2) * kTcdSub + (kk & 3) * 32) >> 4),
                 dq + (((kk >> 2) * kTcdSmallSub + (kk & 3) * 32) >> 4), kIdescS, kk > 0 ? 1u : 0u);
      };
      auto issue_o = [&](int jj, bool acc) {
        const uint64_t dv = dv0 + (jj % kTcdStages) * kStageStep;
        const uint64_t dp = dp0 + (jj & 1) * kSmallStep;
#pragma unroll
        for (int kk = 0; kk < kTcdKeys / 16; ++kk)
          mma_ss(tmem + 2 * kTcdN, dv + ((kk * 16 * 128) >> 4),
                 dp + (((kk >> 2) * kTcdSmallSub + (kk & 3) * 32) >> 4), kIdescO, (acc || kk > 0) ? 1u : 0u);
      };
      // The first product of tile jj+1 is issued before the second product of
      // tile jj, so the softmax of jj+1 can start while P^T(jj) is multiplied.
      int lu = 0, jj = 0;
      int prev = -1;  // tile whose second product is pending
      bool prev_first = false, prev_last = false, ok = true;
      auto finish_prev = [&]() -> bool {
        if (!mbar_wait(p_full(prev & 1), (prev >> 1) & 1, p.err, ERR_WAIT_MMA)) return false;
        tc_fence_after();
        issue_o(prev, !prev_first);
        mma_commit(kv_empty(prev % kTcdStages));
        mma_commit(p_free(prev & 1));
        mma_commit(o_done);
        if (prev_last) mma_commit(o_full);
        return true;
      };
      for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
        const TcdUnit u = tcd_unit(p, unit);
        if (u.T == 0) continue;
        const int qb = lu & 1;
        if (!mbar_wait(q_full(qb), (lu >> 1) & 1, p.err, ERR_WAIT_MMA)) {
          ok = false;
          break;
        }
        ++lu;
        for (int j = 0; j < u.T; ++j, ++jj) {
          if (!mbar_wait(kv_full(jj % kTcdStages), (jj / kTcdStages) & 1, p.err, ERR_WAIT_MMA)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s(jj, qb);
          mma_commit(s_full(jj & 1));
          if (j == u.T - 1) mma_commit(q_free(qb));
          if (prev >= 0 && !finish_prev()) {
            ok = false;
            break;
          }
          prev = jj;
          prev_first = (j == 0);
          prev_last = (j == u.T - 1);
        }
      }
      if (ok && prev >= 0) finish_prev();
      if (jj > 0) {
        mma_commit(drain);
        mbar_wait(drain, 0, p.err, ERR_WAIT_MMA);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;          // TMEM lane quarter
    const int r = quarter * 32 + lane;     // key within a tile; output dimension in O^T
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_off + 2 * kTcdN;
    float* red = reinterpret_cast<float*>(gbase + kOffRed);  // [2][4][16] maxima, then [4][16] sums
    const float sl2 = p.scale_log2;
    int jj = 0, nu = 0, nx = 0;  // tiles, finished units, softmax-barrier phases so far
    bool ok = true;
    auto softmax_sync = [&]() -> bool {
      mbar_arrive(xbar);
      return __all_sync(0xffffffffu, mbar_wait(xbar, (nx++) & 1, p.err, ERR_WAIT_SOFTMAX));
    };
    for (int unit = blockIdx.x; unit < n_units && ok; unit += gridDim.x) {
      const TcdUnit u = tcd_unit(p, unit);
      const int64_t pbase = ((static_cast<int64_t>(u.b) * p.Hkv + u.kvh) * p.chunks + u.piece) * G;
      if (u.T == 0) {
        // an empty piece contributes nothing to the combine
        if (r < G) {
          p.part_ml[(pbase + r) * 2 + 0] = -INFINITY;
          p.part_ml[(pbase + r) * 2 + 1] = 0.f;
        }
        continue;
      }
      float m[G], l[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
      }
      for (int j = 0; j < u.T; ++j, ++jj) {
        const int sb = jj & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(s_full(sb), (jj >> 1) & 1, p.err, ERR_WAIT_SOFTMAX))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t sv[16];
        tmem_ld16(tmem + lane_off + sb * kTcdN, sv);
        tmem_wait_ld();
        const bool valid = u.t_begin + j * kTcdKeys + r < u.t_end;
        if (!valid) {
          // A key past the valid window still has a V row in the tile: cache
          // slots the caller never wrote.  Its P is 0, but 0 x NaN is NaN, so
          // the row is zeroed before the second product reads it (the
          // proxy fence before the p_full arrival orders these stores first).
          const uint32_t vrow = base + (jj % kTcdStages) * kTcdStage + kTcdTile + r * 128;
#pragma unroll
          for (int sub = 0; sub < PL::kSubs; ++sub)
#pragma unroll
            for (int c = 0; c < 128; c += 16) st_shared_zero16(vrow + sub * kTcdSub + c);
        }
        float x[G];
#pragma unroll
        for (int h = 0; h < G; ++h) x[h] = valid ? __uint_as_float(sv[h]) * sl2 : -INFINITY;
        // tile maximum per head: warp reduction, then the four warps through shared memory
        float* rb = red + sb * 4 * kTcdN;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float v = x[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
          if (lane == 0) rb[quarter * kTcdN + h] = v;
        }
        if (!softmax_sync()) {
          ok = false;
          break;
        }
        float tmax[G];
#pragma unroll
        for (int h = 0; h < G; ++h)
          tmax[h] = fmaxf(fmaxf(rb[h], rb[kTcdN + h]), fmaxf(rb[2 * kTcdN + h], rb[3 * kTcdN + h]));
        // P^T buffer sb is free once the second product of tile jj-2 has completed
        if (jj >= 2 && !__all_sync(0xffffffffu,
                                   mbar_wait(p_free(sb), ((jj >> 1) - 1) & 1, p.err, ERR_WAIT_SOFTMAX))) {
          ok = false;
          break;
        }
        if (j == 0) {
#pragma unroll
          for (int h = 0; h < G; ++h) m[h] = tmax[h];
        } else {
          bool grow = false;
#pragma unroll
          for (int h = 0; h < G; ++h) grow |= tmax[h] > m[h] + 8.f;
          if (grow) {
            // O^T holds tiles up to jj-1 of this unit: wait for the last of them,
            // then rescale the heads whose reference maximum moves
            if (!__all_sync(0xffffffffu, mbar_wait(o_done, (jj - 1) & 1, p.err, ERR_WAIT_SOFTMAX))) {
              ok = false;
              break;
            }
            tc_fence_after();
            uint32_t ov[16];
            tmem_ld16(tO, ov);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < G; ++h) {
              if (tmax[h] > m[h] + 8.f) {
                const float alpha = ex2_approx(m[h] - tmax[h]);
                ov[h] = __float_as_uint(__uint_as_float(ov[h]) * alpha);
                l[h] *= alpha;
                m[h] = tmax[h];
              }
            }
            tmem_st16(tO, ov);
            tmem_wait_st();
          }
        }
        // P^T[h][key] in the 128-byte-swizzled K-major layout (row h, 64-key sub-tiles)
        const uint32_t pb = base + kOffP + sb * kTcdSmall + (r >> 6) * kTcdSmallSub;
        const int col = r & 63;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float pe = ex2_approx(x[h] - m[h]);
          l[h] += pe;
          const __nv_bfloat16 bv = __float2bfloat16_rn(pe);
          st_shared_b16(pb + h * 128 + ((((col >> 3) ^ (h & 7))) << 4) + (col & 7) * 2,
                        *reinterpret_cast<const uint16_t*>(&bv));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full(sb));
      }
      if (!ok) break;
      // ---- unit epilogue: partial O (unnormalised), max in log2 units, sum
      if (!__all_sync(0xffffffffu, mbar_wait(o_full, nu & 1, p.err, ERR_WAIT_EPI))) {
        ok = false;
        break;
      }
      ++nu;
      tc_fence_after();
      uint32_t ov[16];
      tmem_ld16(tO, ov);
      tmem_wait_ld();
      if (r < D) {
#pragma unroll
        for (int h = 0; h < G; ++h) p.part_o[(pbase + h) * D + r] = __uint_as_float(ov[h]);
      }
      float* lsum = red + 2 * 4 * kTcdN;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float v = l[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) lsum[quarter * kTcdN + h] = v;
      }
      if (!softmax_sync()) {
        ok = false;
        break;
      }
      if (r < G) {
        float mh = m[0];
#pragma unroll
        for (int h = 1; h < G; ++h)
          if (h == r) mh = m[h];
        p.part_ml[(pbase + r) * 2 + 0] = mh;
        p.part_ml[(pbase + r) * 2 + 1] =
            (lsum[r] + lsum[kTcdN + r]) + (lsum[2 * kTcdN + r] + lsum[3 * kTcdN + r]);
      }
      // the sums buffer is rewritten only after the next unit's first tile
      // exchange, which every thread reaches after reading it here
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTcdTmemCols);
  }
}

// the new token's K/V into slot pos mod W of every (batch, KV head), 16 bytes a thread
__global__ void decode_append_kernel(const DecodeParams p) {
  griddep_launch_dependents();  // the decode sets up and loads Q meanwhile
  const int64_t per_b = static_cast<int64_t>(p.Hkv) * p.D / 8;  // 16-byte chunks of one token
  const int64_t n = static_cast<int64_t>(p.B) * per_b;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = i / per_b;
    const int64_t dst = (b * p.W + p.slot) * per_b + (i - b * per_b);
    reinterpret_cast<uint4*>(p.k_cache)[dst] = reinterpret_cast<const uint4*>(p.k_new)[i];
    reinterpret_cast<uint4*>(p.v_cache)[dst] = reinterpret_cast<const uint4*>(p.v_new)[i];
  }
}

template <int D, int G>
cudaError_t launch_tcd(const DecodeParams& p, int grid, cudaStream_t stream) {
  constexpr int kSmem = TcdPlan<D>::kSmem;
  static DeviceOnce attr_set;  // devices on which the smem opt-in was set
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (!attr_set.done(dev)) {
    const cudaError_t e =
        cudaFuncSetAttribute(decode_tc_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (e != cudaSuccess) return e;
    attr_set.mark(dev);
  }
  // after the append on the same stream: programmatic launch (see the producer)
  return launch_after(decode_tc_kernel<D, G>, dim3(grid), dim3(kTcdThreads), kSmem, stream, p);
}

}  // namespace

int decode_tc_pieces(int B, int Hkv, int n_valid, int max_pieces, int sms) {
  // Pieces per (batch, KV head): units are spread round-robin over one CTA per
  // SM, so the time is about (units per CTA) x (tiles per unit + one tile of
  // per-unit cost: Q, the first product's latency, the partial store).
  const int64_t items = static_cast<int64_t>(B) * Hkv;
  const int tiles = cdiv(imax(n_valid, 1), kTcdKeys);
  int best = 1;
  int64_t best_cost = -1;
  for (int c = 1; c <= imin(max_pieces, tiles); ++c) {
    const int64_t units = items * c;
    const int64_t grid = std::min<int64_t>(units, sms);
    const int64_t per_cta = (units + grid - 1) / grid;
    const int64_t cost = per_cta * (cdiv(tiles, c) + 1);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = c;
    }
  }
  return best;
}

DecodeTcPlan decode_tc_plan(int B, int Hkv, int n_valid, int max_pieces, int sms) {
  DecodeTcPlan pl;
  pl.pieces = decode_tc_pieces(B, Hkv, n_valid, max_pieces, sms);
  pl.piece_len = cdiv(cdiv(n_valid, pl.pieces), kTcdKeys) * kTcdKeys;
  pl.grid = static_cast<int>(std::min<int64_t>(static_cast<int64_t>(B) * Hkv * pl.pieces, sms));
  return pl;
}

bool decode_tc_supported(int D, int G) { return (D == 64 || D == 128) && G >= 1 && G <= 8; }

// p.chunks on entry: the partial slots the workspace holds per (batch, KV head)
cudaError_t launch_decode_tc(const DecodeParams& p_in, int sms, cudaStream_t stream) {
  const int G = p_in.Hq / p_in.Hkv;
  if (!decode_tc_supported(p_in.D, G)) return cudaErrorInvalidValue;
  DecodeParams p = p_in;
  if (!encode_4d_sw128(&p.tm_k, p.k_cache, p.D, p.Hkv, p.W, p.B) ||
      !encode_4d_sw128(&p.tm_v, p.v_cache, p.D, p.Hkv, p.W, p.B) ||
      !encode_2d_sw128(&p.tm_q, p.q, p.D, static_cast<int64_t>(p.B) * p.Hq, kTcdN))
    return cudaErrorInvalidValue;
  const DecodeTcPlan pl = decode_tc_plan(p.B, p.Hkv, p.n_valid, p_in.chunks, sms);
  p.chunks = pl.pieces;
  p.chunk_len = pl.piece_len;
  const int grid = pl.grid;
  const int64_t n16 = static_cast<int64_t>(p.B) * p.Hkv * p.D / 8;
  decode_append_kernel<<<static_cast<int>(std::min<int64_t>(1024, (n16 + 255) / 256)), 256, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (p.D == 128) {
    switch (G) {
      case 1: e = launch_tcd<128, 1>(p, grid, stream); break;
      case 2: e = launch_tcd<128, 2>(p, grid, stream); break;
      case 3: e = launch_tcd<128, 3>(p, grid, stream); break;
      case 4: e = launch_tcd<128, 4>(p, grid, stream); break;
      case 5: e = launch_tcd<128, 5>(p, grid, stream); break;
      case 6: e = launch_tcd<128, 6>(p, grid, stream); break;
      case 7: e = launch_tcd<128, 7>(p, grid, stream); break;
      default: e = launch_tcd<128, 8>(p, grid, stream); break;
    }
  } else {
    switch (G) {
      case 1: e = launch_tcd<64, 1>(p, grid, stream); break;
      case 2: e = launch_tcd<64, 2>(p, grid, stream); break;
      case 3: e = launch_tcd<64, 3>(p, grid, stream); break;
      case 4: e = launch_tcd<64, 4>(p, grid, stream); break;
      case 5: e = launch_tcd<64, 5>(p, grid, stream); break;
      case 6: e = launch_tcd<64, 6>(p, grid, stream); break;
      case 7: e = launch_tcd<64, 7>(p, grid, stream); break;
      default: e = launch_tcd<64, 8>(p, grid, stream); break;
    }
  }
  if (e != cudaSuccess) return e;
  e = launch_decode_combine(p, stream);
  count_launches(3);
  return e;
}

}  // namespace swa
