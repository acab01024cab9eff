// decode.cu -- the parts of the single-token grouped-query decode around its
// tensor-core kernel (decode_tc.cu): the merge of the per-piece partials, the
// f32 path's write of the new token, the workspace sizing, and the dispatch.
//
// Sliding-window attention explainer (rolling buffer, grouped-query
// attention): the key/value of position i is written to slot i mod W,
// overwriting position i - W, and the new token's Hq query heads attend to the
// W cached positions, each KV head shared by Hq/Hkv query heads.
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

// slots per step of the workspace sizing below
constexpr int kDecRows = 32;

// merge the per-piece partials: one warp per (batch, query head)
template <int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(const DecodeParams p) {
  griddep_wait();  // launched behind the decode (programmatic launch): its partials first
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
  // Partial slots per (batch, KV head) that the workspace provides (the decode
  // uses at most this many pieces of the window).  The count minimises waves x
  // (slots per piece + two 32-slot steps) over 148 SMs x 4, at most 32; it fixes
  // swa_decode_workspace_bytes, so it is kept as the sizing rule.
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

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int D, int W) {
  const int chunks = decode_chunks(B, Hkv, W);
  const int G = Hq / Hkv;
  const size_t n = static_cast<size_t>(B) * Hkv * chunks * G;
  return n * D * sizeof(float) + n * 2 * sizeof(float);
}

cudaError_t launch_decode_combine(const DecodeParams& p, cudaStream_t stream) {
  const dim3 grid((p.B * p.Hq + 7) / 8);
  if (p.D == 128) return launch_after(decode_combine_kernel<128>, grid, dim3(256), 0, stream, p);
  if (p.D == 64) return launch_after(decode_combine_kernel<64>, grid, dim3(256), 0, stream, p);
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_bf16(const DecodeParams& p, cudaStream_t stream) {
  // head_dim 64 and 128, 1 to 8 query heads per KV head: the tensor-core
  // kernel (decode_tc.cu); the entry points accept no other bf16 shape
  if (!decode_tc_supported(p.D, p.Hq / p.Hkv)) return cudaErrorInvalidValue;
  return launch_decode_tc(p, device_sms(), stream);
}

cudaError_t launch_decode_write_f32(const DecodeParams& p, cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(p.B) * p.Hkv * p.D;
  const int blocks = static_cast<int>(imin(1024, static_cast<int>((n + 255) / 256)));
  decode_write_f32_kernel<<<blocks, 256, 0, stream>>>(p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swa
