// decode.cu -- single-token grouped-query decode against a rolling KV buffer
// (sliding-window attention explainer: the key/value of position i is written to
// slot i mod W, overwriting position i - W, and the new token attends to the W
// cached positions; grouped-query attention shares each KV head among Hq/Hkv
// query heads).
//
// Memory-bound: every K/V byte of the buffer is read once.  Grid (chunk, kv
// head, batch); a CTA streams one chunk of slots of one (batch, kv head) and
// serves all G query heads of the group from the same loaded rows.  At head_dim
// 128, sixteen lanes cooperate on one cached row (one 16-byte chunk of q, K, V
// and O per lane and head), so a thread needs ~114 registers and four CTAs (16
// warps) fit an SM; at head_dim 64 eight lanes share a row.  Scores use the scale folded into q (log2 units) and an
// online softmax whose reference maximum only moves when a score exceeds it by
// more than 2^8, so the accumulators are rarely rescaled.  Per-chunk partials
// (max, sum, numerator) are merged by a second small kernel.
//
// The CTA whose chunk contains slot pos mod W uses the new token's K/V for that
// slot and writes it into the cache; no other CTA reads that row.
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cmath>
#include <cstdint>

#include <cuda.h>

#include "internal.h"
#include "ptx.cuh"
#include "tile_sched.h"

namespace swa {
namespace {

constexpr int kDecThreads = 128;  // 4 warps
constexpr int kDecRows = 32;      // cache rows per pipeline stage

SWA_DEV float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
SWA_DEV float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

SWA_DEV void unpack8(const uint4 u, float2* f) {
  f[0] = make_float2(bf_lo(u.x), bf_hi(u.x));
  f[1] = make_float2(bf_lo(u.y), bf_hi(u.y));
  f[2] = make_float2(bf_lo(u.z), bf_hi(u.z));
  f[3] = make_float2(bf_lo(u.w), bf_hi(u.w));
}

SWA_DEV void tma_load_3d(uint32_t dst, const void* tmap, uint32_t mbar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(mbar)
      : "memory");
}

// Sum each of the G per-lane partial scores x[g] over the LPR lanes of a row
// group, leaving every lane with all G sums.  Butterfly with halving: at the
// level with xor offset LPR/2^k the lanes whose offset bit is set keep the upper
// half of their remaining heads and send the lower half (and the other way
// round), so after log2(G) levels each lane holds one head's partial sum over
// 2^log2(G) lanes; the remaining offsets finish that sum, and G shuffles from
// the lanes owning each head broadcast the results.  log2(G) + G - 1 + log2(LPR/G)
// shuffles per group instead of G log2(LPR).
template <int G, int LPR>
SWA_DEV void reduce_heads(float (&x)[G], int lane) {
  static_assert(G <= LPR, "at most one head per lane of a row group");
  float v[G];
#pragma unroll
  for (int g = 0; g < G; ++g) v[g] = x[g];
#pragma unroll
  for (int n = G, off = LPR / 2; n > 1; n >>= 1, off >>= 1) {
    const bool up = (lane & off) != 0;
    const int half = n / 2;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = up ? v[i] : v[half + i];
      const float keep = up ? v[half + i] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
#pragma unroll
  for (int off = LPR / (2 * G); off >= 1; off >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
  // lane owns head h = sum over levels k of (lane bit LPR/2^k set ? G/2^k : 0)
  const int base = lane & ~(LPR - 1);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    int src = base;
#pragma unroll
    for (int k = 1, off = LPR / 2; (G >> k) > 0; ++k, off >>= 1)
      if (g & (G >> k)) src |= off;
    x[g] = __shfl_sync(0xffffffffu, v[0], src);
  }
}

// LPR lanes share a cached row; ST stages of kDecRows rows are in flight per CTA.
template <int D, int LPR, int ST>
struct DecPlan {
  static_assert(LPR == 8 || LPR == 16, "8 or 16 lanes per row");
  static_assert(D % (8 * LPR) == 0, "whole 16-byte chunks per lane");
  static constexpr int kNV = D / (8 * LPR);  // 16-byte chunks per lane per row
  static constexpr int kRPW = 32 / LPR;      // rows a warp covers per pass
  static constexpr int kPasses = kDecRows / (4 * kRPW);
  static constexpr int kRowBytes = D * 2;
  static constexpr int kTileBytes = kDecRows * kRowBytes;  // K (or V) rows of one stage
  static constexpr int kOffK = 0;
  static constexpr int kOffV = ST * kTileBytes;
  static constexpr int kOffBar = 2 * ST * kTileBytes;
  static constexpr int kSmemBytes = kOffBar + 2 * ST * 8 + 128;
  // CTAs per SM the launch bounds ask for (registers for 16 warps per SM when a
  // lane holds one chunk of q and O per head)
  static constexpr int kMinBlocks = (LPR == 16) ? 4 : 1;
};

// Lane (grp, sub) of a warp handles row grp of each pass and owns the head_dim
// elements of chunks sub + LPR v (v < kNV), i.e. [8 (sub + LPR v), +8): its
// 16-byte reads of a row hit distinct bank quads, so a warp's read of its rows
// takes the minimum number of shared-memory wavefronts.
template <int D, int G, int LPR, int ST>
__global__ void __launch_bounds__(kDecThreads, DecPlan<D, LPR, ST>::kMinBlocks)
    decode_kernel(const __grid_constant__ DecodeParams p) {
  using PL = DecPlan<D, LPR, ST>;
  constexpr int NV = PL::kNV;
  constexpr int kDecStages = ST;
  extern __shared__ __align__(128) uint8_t dsm[];
  const int c = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane / LPR, sub = lane % LPR;
  const int t_begin = c * p.chunk_len;
  const int t_end = imin(t_begin + p.chunk_len, p.n_valid);
  const int n_st = t_end > t_begin ? cdiv(t_end - t_begin, kDecRows) : 0;
  const uint32_t sbase = smem_u32(dsm);
  const uint32_t bar_full = sbase + PL::kOffBar;
  const uint32_t bar_empty = bar_full + 8 * kDecStages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(bar_full + 8 * s, 1);
      mbar_init(bar_empty + 8 * s, 4);
    }
    fence_barrier_init();
  }
  __syncthreads();
  auto issue = [&](int i) {
    const int s = i % kDecStages;
    const int row = b * p.W + t_begin + i * kDecRows;
    mbar_arrive_expect_tx(bar_full + 8 * s, 2 * PL::kTileBytes);
    tma_load_3d(sbase + PL::kOffK + s * PL::kTileBytes, &p.tm_k, bar_full + 8 * s, 0, kvh, row);
    tma_load_3d(sbase + PL::kOffV + s * PL::kTileBytes, &p.tm_v, bar_full + 8 * s, 0, kvh, row);
  };
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
    for (int i = 0; i < imin(kDecStages, n_st); ++i) issue(i);
  }

  const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(p.q);
  float2 q[G][4 * NV];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const __nv_bfloat16* qp = qb + (static_cast<int64_t>(b) * p.Hq + kvh * G + g) * D + sub * 8;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      unpack8(*reinterpret_cast<const uint4*>(qp + v * 8 * LPR), &q[g][4 * v]);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        q[g][4 * v + e] = make_float2(q[g][4 * v + e].x * p.scale_log2, q[g][4 * v + e].y * p.scale_log2);
    }
  }
  float2 o[G][4 * NV];
  float m[G], l[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 4 * NV; ++e) o[g][e] = make_float2(0.f, 0.f);
  }
  const int64_t row_elems = static_cast<int64_t>(p.Hkv) * D;
  const int64_t new_off = (static_cast<int64_t>(b) * p.Hkv + kvh) * D + sub * 8;
  bool ok = true;

  for (int i = 0; i < n_st && ok; ++i) {
    const int s = i % kDecStages;
    ok = __all_sync(0xffffffffu, mbar_wait(bar_full + 8 * s, (i / kDecStages) & 1, p.err, ERR_WAIT_TMA));
    if (!ok) break;
    const uint8_t* ks = dsm + PL::kOffK + s * PL::kTileBytes;
    const uint8_t* vs = dsm + PL::kOffV + s * PL::kTileBytes;
#pragma unroll
    for (int pass = 0; pass < PL::kPasses; ++pass) {
      const int row = (warp * PL::kPasses + pass) * PL::kRPW + grp;  // row within the stage
      const int t = t_begin + i * kDecRows + row;
      const bool valid = t < t_end;
      uint4 kr[NV], vr[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        kr[v] = *reinterpret_cast<const uint4*>(ks + row * PL::kRowBytes + v * 16 * LPR + sub * 16);
        vr[v] = *reinterpret_cast<const uint4*>(vs + row * PL::kRowBytes + v * 16 * LPR + sub * 16);
      }
      if (valid && t == p.slot) {
        // the new token: its K/V come from the inputs and go into the cache here
        const __nv_bfloat16* kn = reinterpret_cast<const __nv_bfloat16*>(p.k_new) + new_off;
        const __nv_bfloat16* vn = reinterpret_cast<const __nv_bfloat16*>(p.v_new) + new_off;
        __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(p.k_cache) +
                            (static_cast<int64_t>(b) * p.W + t) * row_elems + kvh * D + sub * 8;
        __nv_bfloat16* vc = reinterpret_cast<__nv_bfloat16*>(p.v_cache) +
                            (static_cast<int64_t>(b) * p.W + t) * row_elems + kvh * D + sub * 8;
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          kr[v] = *reinterpret_cast<const uint4*>(kn + v * 8 * LPR);
          vr[v] = *reinterpret_cast<const uint4*>(vn + v * 8 * LPR);
          *reinterpret_cast<uint4*>(kc + v * 8 * LPR) = kr[v];
          *reinterpret_cast<uint4*>(vc + v * 8 * LPR) = vr[v];
        }
      }
      float2 kf[4 * NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) unpack8(kr[v], &kf[4 * v]);
      float sc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 4 * NV; ++e) acc = __ffma2_rn(q[g][e], kf[e], acc);
        sc[g] = acc.x + acc.y;
      }
      reduce_heads<G, LPR>(sc, lane);
      if (valid) {
        float2 vf[4 * NV];
#pragma unroll
        for (int v = 0; v < NV; ++v) unpack8(vr[v], &vf[4 * v]);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          if (m[g] == -INFINITY || sc[g] > m[g] + 8.f) {
            // move the reference maximum (rare after the first rows)
            const float corr = (m[g] == -INFINITY) ? 0.f : ex2_approx(m[g] - sc[g]);
            l[g] *= corr;
#pragma unroll
            for (int e = 0; e < 4 * NV; ++e) o[g][e] = make_float2(o[g][e].x * corr, o[g][e].y * corr);
            m[g] = sc[g];
          }
          const float pe = ex2_approx(sc[g] - m[g]);
          l[g] += pe;
          const float2 p2 = make_float2(pe, pe);
#pragma unroll
          for (int e = 0; e < 4 * NV; ++e) o[g][e] = __ffma2_rn(p2, vf[e], o[g][e]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty + 8 * s);
    if (threadIdx.x == 0 && i + kDecStages < n_st) {
      // refill this stage once all four warps have read it
      if (!mbar_wait(bar_empty + 8 * s, (i / kDecStages) & 1, p.err, ERR_WAIT_TMA)) ok = false;
      else issue(i + kDecStages);
    }
  }
  // never leave with a bulk copy still landing in shared memory
  if (threadIdx.x == 0) {
    for (int i = imax(0, n_st - kDecStages); i < n_st; ++i)
      mbar_wait(bar_full + 8 * (i % kDecStages), (i / kDecStages) & 1, p.err, ERR_WAIT_TMA);
  }

  // ---- merge the row groups of each warp with shuffles, then the four warps
  // through shared memory (reusing the first stage's K tile)
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float M = m[g];
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float wgt = (m[g] == -INFINITY) ? 0.f : ex2_approx(m[g] - M);
    float lw = l[g] * wgt;
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) lw += __shfl_xor_sync(0xffffffffu, lw, off);
#pragma unroll
    for (int e = 0; e < 4 * NV; ++e) {
      float x = o[g][e].x * wgt, y = o[g][e].y * wgt;
#pragma unroll
      for (int off = LPR; off < 32; off <<= 1) {
        x += __shfl_xor_sync(0xffffffffu, x, off);
        y += __shfl_xor_sync(0xffffffffu, y, off);
      }
      o[g][e] = make_float2(x, y);
    }
    m[g] = M;
    l[g] = lw;
  }
  __syncthreads();
  float* sm_o = reinterpret_cast<float*>(dsm);              // [4][G][D]
  float* sm_ml = sm_o + 4 * G * D;                          // [4][G][2]
  if (grp == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (sub == 0) {
        sm_ml[(warp * G + g) * 2] = m[g];
        sm_ml[(warp * G + g) * 2 + 1] = l[g];
      }
#pragma unroll
      for (int v = 0; v < NV; ++v)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int d = 8 * (sub + LPR * v) + 2 * e;
          sm_o[(warp * G + g) * D + d] = o[g][4 * v + e].x;
          sm_o[(warp * G + g) * D + d + 1] = o[g][4 * v + e].y;
        }
    }
  }
  __syncthreads();
  const int64_t part = ((static_cast<int64_t>(b) * p.Hkv + kvh) * p.chunks + c) * G;
  for (int idx = threadIdx.x; idx < G * D; idx += kDecThreads) {
    const int g = idx / D, d = idx - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int r = 0; r < 4; ++r) M = fmaxf(M, sm_ml[(r * G + g) * 2]);
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float mr = sm_ml[(r * G + g) * 2];
      const float wgt = (mr == -INFINITY) ? 0.f : ex2_approx(mr - M);
      L += wgt * sm_ml[(r * G + g) * 2 + 1];
      acc += wgt * sm_o[(r * G + g) * D + d];
    }
    p.part_o[(part + g) * D + d] = acc;
    if (d == 0) {
      p.part_ml[(part + g) * 2] = M;
      p.part_ml[(part + g) * 2 + 1] = L;
    }
  }
}

// merge chunk partials: one warp per (batch, query head)
template <int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(const DecodeParams p) {
  const int gw = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= p.B * p.Hq) return;
  const int b = gw / p.Hq, h = gw - b * p.Hq;
  const int G = p.Hq / p.Hkv;
  const int kvh = h / G, g = h - kvh * G;
  float M = -INFINITY;
  for (int c = 0; c < p.chunks; ++c) {
    const int64_t part = (((static_cast<int64_t>(b) * p.Hkv + kvh) * p.chunks + c) * G + g);
    M = fmaxf(M, p.part_ml[part * 2]);
  }
  constexpr int E = D / 32;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  float L = 0.f;
  for (int c = 0; c < p.chunks; ++c) {
    const int64_t part = (((static_cast<int64_t>(b) * p.Hkv + kvh) * p.chunks + c) * G + g);
    const float mc = p.part_ml[part * 2];
    if (mc == -INFINITY) continue;
    const float wgt = exp2f(mc - M);
    L += wgt * p.part_ml[part * 2 + 1];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] += wgt * p.part_o[part * D + lane + 32 * e];
  }
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + static_cast<int64_t>(gw) * D;
  const float inv = 1.f / L;
#pragma unroll
  for (int e = 0; e < E; ++e) out[lane + 32 * e] = __float2bfloat16_rn(acc[e] * inv);
}

// f32 path: write the new token's K/V into its slot (attention then runs on the
// SIMT kernel in decode mode)
__global__ void decode_write_f32_kernel(const DecodeParams p) {
  const int64_t n = static_cast<int64_t>(p.B) * p.Hkv * p.D;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = i / (static_cast<int64_t>(p.Hkv) * p.D);
    const int64_t r = i - b * p.Hkv * p.D;
    const int64_t dst = (b * p.W + p.slot) * p.Hkv * p.D + r;
    reinterpret_cast<float*>(p.k_cache)[dst] = reinterpret_cast<const float*>(p.k_new)[i];
    reinterpret_cast<float*>(p.v_cache)[dst] = reinterpret_cast<const float*>(p.v_new)[i];
  }
}

}  // namespace

int decode_chunks(int B, int Hkv, int W) {
  // Key chunks per (batch, KV head).  A CTA's time is about its rows plus a
  // fixed cost (set-up, pipeline fill, partial write: ~2 stages of rows); the
  // kernel's time is that times the number of waves of CTAs over 148 SMs with 4
  // resident each.  Pick the count that minimises it, with chunks of at least
  // 2 pipeline stages (at most 32 chunks).
  const int64_t pairs = static_cast<int64_t>(B) * Hkv;
  const int64_t slots = 148LL * 4;
  const int cmax = imax(1, imin(32, cdiv(W, 2 * kDecRows)));
  int best = 1;
  double best_cost = 1e300;
  for (int c = 1; c <= cmax; ++c) {
    const int64_t waves = (pairs * c + slots - 1) / slots;
    const double cost = static_cast<double>(waves) * (static_cast<double>(W) / c + 2.0 * kDecRows);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = c;
    }
  }
  return best;
}

int decode_chunk_len(int n_valid, int chunks) {
  // whole pipeline stages per chunk
  return cdiv(cdiv(n_valid, chunks), kDecRows) * kDecRows;
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int D, int W) {
  const int chunks = decode_chunks(B, Hkv, W);
  const int G = Hq / Hkv;
  const size_t n = static_cast<size_t>(B) * Hkv * chunks * G;
  return n * D * sizeof(float) + n * 2 * sizeof(float);
}

namespace {
template <int D, int G, int LPR, int ST>
cudaError_t launch_dec(const DecodeParams& p, cudaStream_t stream) {
  using PL = DecPlan<D, LPR, ST>;
  static int attr_dev_mask = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const int bit = 1 << (dev & 31);
  if (!(attr_dev_mask & bit)) {
    const cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, G, LPR, ST>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, PL::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_dev_mask |= bit;
  }
  dim3 grid(p.chunks, p.Hkv, p.B);
  decode_kernel<D, G, LPR, ST><<<grid, kDecThreads, PL::kSmemBytes, stream>>>(p);
  decode_combine_kernel<D><<<(p.B * p.Hq + 7) / 8, 256, 0, stream>>>(p);
  count_launches(2);
  return cudaGetLastError();
}
template <int D, int G>
cudaError_t launch_dec_pick(const DecodeParams& p, cudaStream_t stream) {
  if constexpr (D == 128) return launch_dec<D, G, 16, 3>(p, stream);
  else return launch_dec<D, G, 8, 4>(p, stream);
}
}  // namespace

cudaError_t launch_decode_combine(const DecodeParams& p, cudaStream_t stream) {
  if (p.D == 128)
    decode_combine_kernel<128><<<(p.B * p.Hq + 7) / 8, 256, 0, stream>>>(p);
  else if (p.D == 64)
    decode_combine_kernel<64><<<(p.B * p.Hq + 7) / 8, 256, 0, stream>>>(p);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_decode_bf16(const DecodeParams& p_in, cudaStream_t stream) {
  const int G = p_in.Hq / p_in.Hkv;
  // head_dim 128: the tensor-core kernel (decode_tc.cu)
  if (decode_tc_supported(p_in.D, G)) return launch_decode_tc(p_in, device_sms(), stream);
  DecodeParams p = p_in;
  // K/V caches viewed as rows [B*W, Hkv, D]; one box = 32 rows of one KV head
  if (!encode_rows_map(&p.tm_k, p.k_cache, p.D, p.Hkv, static_cast<int64_t>(p.B) * p.W, kDecRows) ||
      !encode_rows_map(&p.tm_v, p.v_cache, p.D, p.Hkv, static_cast<int64_t>(p.B) * p.W, kDecRows))
    return cudaErrorInvalidValue;
  p.chunk_len = decode_chunk_len(p.n_valid, p.chunks);
  // head_dim 128: 16 lanes per row, 3 stages (one chunk of q and O per lane and
  // head, so four CTAs fit an SM by registers and shared memory; 8 lanes per row
  // and 4 stages measured 268 vs 253 us on B=64, W=4096).  head_dim 64: 8 lanes,
  // 4 stages.
#define SWA_DEC_CASE(DD, GG) \
  if (p.D == DD && G == GG) return launch_dec_pick<DD, GG>(p, stream);
  SWA_DEC_CASE(128, 1) SWA_DEC_CASE(128, 2) SWA_DEC_CASE(128, 4) SWA_DEC_CASE(128, 8)
  SWA_DEC_CASE(64, 1) SWA_DEC_CASE(64, 2) SWA_DEC_CASE(64, 4) SWA_DEC_CASE(64, 8)
#undef SWA_DEC_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_write_f32(const DecodeParams& p, cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(p.B) * p.Hkv * p.D;
  const int blocks = static_cast<int>(imin(1024, static_cast<int>((n + 255) / 256)));
  decode_write_f32_kernel<<<blocks, 256, 0, stream>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swa
