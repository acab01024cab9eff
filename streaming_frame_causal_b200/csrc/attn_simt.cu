// attn_simt.cu -- float32 attention on the CUDA cores, for the configurations
// whose contract is float32 end to end (the tiny 8-frame check case and any
// f32 call).  One warp per (batch, query row, head); lanes split head_dim; keys
// are walked one by one with an online softmax in float32.
//
// The key set per query row is the same schedule the tensor-core path uses:
// frame intervals ("Mask Generation in CausalAttention": window start
// max(0, i - W_f + 1) plus retained scale frames), the token band t-W+1..t
// (sliding-window explainer), the streaming cache's retained segments, or the
// valid slots of a rolling decode buffer.
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"
#include "tile_sched.h"

namespace swa {
namespace {

template <int D>
__global__ void __launch_bounds__(128) attn_simt_kernel(const SimtParams p) {
  constexpr int E = D / 32;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int64_t total = static_cast<int64_t>(p.B) * p.Nq * p.Hq;
  if (gw >= total) return;
  const int h = static_cast<int>(gw % p.Hq);
  const int row = static_cast<int>((gw / p.Hq) % p.Nq);
  const int b = static_cast<int>(gw / (static_cast<int64_t>(p.Hq) * p.Nq));
  const int kvh = h / (p.Hq / p.Hkv);

  const int64_t q_ld = p.q_ld ? p.q_ld : static_cast<int64_t>(p.Hq) * D;
  const int64_t kv_ld = p.kv_ld ? p.kv_ld : static_cast<int64_t>(p.Hkv) * D;
  float qv[E];
  const float* qp = p.q + (static_cast<int64_t>(b) * p.Nq + row) * q_ld + static_cast<int64_t>(p.q_h0 + h) * D;
#pragma unroll
  for (int e = 0; e < E; ++e) qv[e] = qp[lane + 32 * e] * p.scale;

  int nseg = 0;
  int lo[2], hi[2];
  const int* grow = nullptr;
  const int* glen = nullptr;
  if (p.mode == SIMT_FRAME) {
    int flo[2], fhi[2];
    nseg = frame_intervals(row / p.P, p.Wf, p.S, flo, fhi);
    for (int s = 0; s < nseg; ++s) {
      lo[s] = flo[s] * p.P;
      hi[s] = fhi[s] * p.P;
    }
  } else if (p.mode == SIMT_BAND) {
    nseg = 1;
    lo[0] = imax(0, row - p.W + 1);
    hi[0] = row + 1;
  } else if (p.mode == SIMT_STREAM) {
    grow = p.seg_row;
    glen = p.seg_len;
    nseg = p.meta_hdr[5];
    if (nseg < 0 || nseg > p.max_segs) {
      if (lane == 0) latch_error(p.err, ERR_BAD_META);
      return;
    }
  } else {  // SIMT_DECODE
    nseg = 1;
    lo[0] = 0;
    hi[0] = p.n_valid;
  }

  float m = -INFINITY, l = 0.f, o[E];
#pragma unroll
  for (int e = 0; e < E; ++e) o[e] = 0.f;
  for (int s = 0; s < nseg; ++s) {
    const int a = grow ? grow[s] : lo[s];
    const int z = grow ? grow[s] + glen[s] : hi[s];
    for (int key = a; key < z; ++key) {
      const int64_t koff = (static_cast<int64_t>(b) * p.Nk + key) * kv_ld + static_cast<int64_t>(p.kv_h0 + kvh) * D;
      float d = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) d = fmaf(qv[e], p.k[koff + lane + 32 * e], d);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
      const float m_new = fmaxf(m, d);
      const float c = expf(m - m_new);
      const float pe = expf(d - m_new);
      l = l * c + pe;
#pragma unroll
      for (int e = 0; e < E; ++e) o[e] = fmaf(pe, p.v[koff + lane + 32 * e], o[e] * c);
      m = m_new;
    }
  }
  float* op = p.out + (static_cast<int64_t>(b) * p.Nq + row) * q_ld + static_cast<int64_t>(p.q_h0 + h) * D;
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < E; ++e) op[lane + 32 * e] = o[e] * inv;
}

}  // namespace

cudaError_t launch_attn_simt(const SimtParams& p, cudaStream_t stream) {
  const int64_t warps = static_cast<int64_t>(p.B) * p.Nq * p.Hq;
  const int64_t blocks = (warps + 3) / 4;
  if (blocks == 0) return cudaSuccess;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  switch (p.D) {
    case 32: attn_simt_kernel<32><<<static_cast<unsigned>(blocks), 128, 0, stream>>>(p); break;
    case 64: attn_simt_kernel<64><<<static_cast<unsigned>(blocks), 128, 0, stream>>>(p); break;
    case 128: attn_simt_kernel<128><<<static_cast<unsigned>(blocks), 128, 0, stream>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace swa
