// decode.cu -- single-token grouped-query decode against a rolling KV buffer
// (sliding-window attention explainer: the key/value of position i is written to
// slot i mod W, overwriting position i - W, and the new token attends to the W
// cached positions; grouped-query attention shares each KV head among Hq/Hkv
// query heads).
//
// Memory-bound: every K/V byte of the buffer is read once.  Grid (chunk, kv
// head, batch); a CTA streams one chunk of slots of one (batch, kv head) and
// serves all G query heads of the group from the same loaded rows.  Eight lanes
// cooperate on one cached row (16-byte vector loads, each lane a contiguous
// slice of head_dim), so a warp covers four rows per step with fully used
// 256-byte segments.  Scores use the scale folded into q (log2 units) and an
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

#include "internal.h"
#include "ptx.cuh"
#include "tile_sched.h"

namespace swa {
namespace {

constexpr int kDecThreads = 128;   // 4 warps x 4 row-groups = 16 rows per step
constexpr int kRowsPerStep = 16;

SWA_DEV float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
SWA_DEV float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

SWA_DEV uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const DecodeParams p) {
  constexpr int EL = D / 8;   // head_dim elements per lane
  constexpr int NV = EL / 8;  // 16-byte vectors per lane per row
  const int c = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int grp = lane >> 3, sub = lane & 7;
  const int t_begin = c * p.chunk_len;
  const int t_end = imin(t_begin + p.chunk_len, p.n_valid);

  const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(p.q);
  float2 q[G][EL / 2];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const __nv_bfloat16* qp = qb + (static_cast<int64_t>(b) * p.Hq + kvh * G + g) * D + sub * EL;
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const uint4 u = *reinterpret_cast<const uint4*>(qp + v * 8);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        q[g][v * 4 + e] = make_float2(bf_lo(w[e]) * p.scale_log2, bf_hi(w[e]) * p.scale_log2);
    }
  }
  float2 o[G][EL / 2];
  float m[G], l[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < EL / 2; ++e) o[g][e] = make_float2(0.f, 0.f);
  }

  const int64_t row_elems = static_cast<int64_t>(p.Hkv) * D;
  const __nv_bfloat16* kc = reinterpret_cast<const __nv_bfloat16*>(p.k_cache) +
                            static_cast<int64_t>(b) * p.W * row_elems + kvh * D + sub * EL;
  const __nv_bfloat16* vc = reinterpret_cast<const __nv_bfloat16*>(p.v_cache) +
                            static_cast<int64_t>(b) * p.W * row_elems + kvh * D + sub * EL;
  const int64_t new_off = (static_cast<int64_t>(b) * p.Hkv + kvh) * D + sub * EL;

  // rows t_begin + 16k + tl; the loop bound is warp-uniform so the group
  // reductions below always see all 32 lanes
  for (int tb = t_begin + warp * 4; tb < t_end; tb += kRowsPerStep) {
    const int t = tb + grp;
    const bool valid = t < t_end;
    uint4 kr[NV], vr[NV];
    if (valid && t == p.slot) {
      const __nv_bfloat16* kn = reinterpret_cast<const __nv_bfloat16*>(p.k_new) + new_off;
      const __nv_bfloat16* vn = reinterpret_cast<const __nv_bfloat16*>(p.v_new) + new_off;
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        kr[v] = *reinterpret_cast<const uint4*>(kn + v * 8);
        vr[v] = *reinterpret_cast<const uint4*>(vn + v * 8);
        *reinterpret_cast<uint4*>(const_cast<__nv_bfloat16*>(kc) + t * row_elems + v * 8) = kr[v];
        *reinterpret_cast<uint4*>(const_cast<__nv_bfloat16*>(vc) + t * row_elems + v * 8) = vr[v];
      }
    } else if (valid) {
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        kr[v] = ld_stream(kc + t * row_elems + v * 8);
        vr[v] = ld_stream(vc + t * row_elems + v * 8);
      }
    } else {
#pragma unroll
      for (int v = 0; v < NV; ++v) kr[v] = vr[v] = make_uint4(0u, 0u, 0u, 0u);
    }
    float2 kf[EL / 2], vf[EL / 2];
#pragma unroll
    for (int v = 0; v < NV; ++v) {
      const uint32_t wk[4] = {kr[v].x, kr[v].y, kr[v].z, kr[v].w};
      const uint32_t wv[4] = {vr[v].x, vr[v].y, vr[v].z, vr[v].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        kf[v * 4 + e] = make_float2(bf_lo(wk[e]), bf_hi(wk[e]));
        vf[v * 4 + e] = make_float2(bf_lo(wv[e]), bf_hi(wv[e]));
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < EL / 2; ++e) acc = __ffma2_rn(q[g][e], kf[e], acc);
      float s = acc.x + acc.y;
      s += __shfl_xor_sync(0xffffffffu, s, 1);
      s += __shfl_xor_sync(0xffffffffu, s, 2);
      s += __shfl_xor_sync(0xffffffffu, s, 4);
      if (valid) {
        if (m[g] == -INFINITY || s > m[g] + 8.f) {
          // move the reference maximum (rare after the first rows)
          const float corr = (m[g] == -INFINITY) ? 0.f : ex2_approx(m[g] - s);
          l[g] *= corr;
#pragma unroll
          for (int e = 0; e < EL / 2; ++e) o[g][e] = make_float2(o[g][e].x * corr, o[g][e].y * corr);
          m[g] = s;
        }
        const float pe = ex2_approx(s - m[g]);
        l[g] += pe;
        const float2 p2 = make_float2(pe, pe);
#pragma unroll
        for (int e = 0; e < EL / 2; ++e) o[g][e] = __ffma2_rn(p2, vf[e], o[g][e]);
      }
    }
  }

  // ---- merge the four row groups of each warp with shuffles, then the four
  // warps through shared memory
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float M = fmaxf(m[g], __shfl_xor_sync(0xffffffffu, m[g], 8));
    M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 16));
    const float wgt = (m[g] == -INFINITY) ? 0.f : ex2_approx(m[g] - M);
    float lw = l[g] * wgt;
    lw += __shfl_xor_sync(0xffffffffu, lw, 8);
    lw += __shfl_xor_sync(0xffffffffu, lw, 16);
#pragma unroll
    for (int e = 0; e < EL / 2; ++e) {
      float x = o[g][e].x * wgt, y = o[g][e].y * wgt;
      x += __shfl_xor_sync(0xffffffffu, x, 8);
      x += __shfl_xor_sync(0xffffffffu, x, 16);
      y += __shfl_xor_sync(0xffffffffu, y, 8);
      y += __shfl_xor_sync(0xffffffffu, y, 16);
      o[g][e] = make_float2(x, y);
    }
    m[g] = M;
    l[g] = lw;
  }
  __shared__ float sm_m[4][G], sm_l[4][G];
  __shared__ float sm_o[4][G][D];
  if (grp == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (sub == 0) {
        sm_m[warp][g] = m[g];
        sm_l[warp][g] = l[g];
      }
#pragma unroll
      for (int e = 0; e < EL / 2; ++e) {
        sm_o[warp][g][sub * EL + 2 * e] = o[g][e].x;
        sm_o[warp][g][sub * EL + 2 * e + 1] = o[g][e].y;
      }
    }
  }
  __syncthreads();
  const int64_t part = ((static_cast<int64_t>(b) * p.Hkv + kvh) * p.chunks + c) * G;
  for (int idx = threadIdx.x; idx < G * D; idx += kDecThreads) {
    const int g = idx / D, d = idx - g * D;
    float M = -INFINITY;
#pragma unroll
    for (int r = 0; r < 4; ++r) M = fmaxf(M, sm_m[r][g]);
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float mr = sm_m[r][g];
      const float wgt = (mr == -INFINITY) ? 0.f : ex2_approx(mr - M);
      L += wgt * sm_l[r][g];
      acc += wgt * sm_o[r][g][d];
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
  // enough CTAs for ~28 per SM on 148 SMs, chunks of at least 64 slots
  const int64_t pairs = static_cast<int64_t>(B) * Hkv;
  int chunks = static_cast<int>((148LL * 28 + pairs - 1) / pairs);
  chunks = imax(1, imin(chunks, cdiv(W, 64)));
  return chunks;
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int D, int W) {
  const int chunks = decode_chunks(B, Hkv, W);
  const int G = Hq / Hkv;
  const size_t n = static_cast<size_t>(B) * Hkv * chunks * G;
  return n * D * sizeof(float) + n * 2 * sizeof(float);
}

cudaError_t launch_decode_bf16(const DecodeParams& p, cudaStream_t stream) {
  const int G = p.Hq / p.Hkv;
  dim3 grid(p.chunks, p.Hkv, p.B);
#define SWA_DEC_CASE(DD, GG)                                                   \
  if (p.D == DD && G == GG) {                                                  \
    decode_kernel<DD, GG><<<grid, kDecThreads, 0, stream>>>(p);                \
    decode_combine_kernel<DD><<<(p.B * p.Hq + 7) / 8, 256, 0, stream>>>(p);    \
    count_launches(2);                                                         \
    return cudaGetLastError();                                                 \
  }
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
