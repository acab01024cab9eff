// prologue.cu -- the attention prologue of a streaming frame ("Method forward",
// block forward listing: the compiled attn_pre step "norm1 + qkv linear +
// reshape + q_norm + k_norm + RoPE + format"), written as two kernels:
//
//   ln_rows_kernel   norm1: LayerNorm over C of each token, bf16 out
//   qkv_pre_kernel   qkv = norm1(x) @ w_qkv^T + b_qkv on the tensor cores
//                    (tcgen05, TMA-fed 4-stage ring, accumulator in TMEM), and
//                    in the epilogue, per 128-token x 128-feature tile: the bias,
//                    per-head LayerNorm of the q and k sections, RoPE on q and k
//                    (the (2i, 2i+1) pairs times the caller's complex table: the
//                    I/O page's complex-valued 3-D RoPE format), bf16 stores.
//                    K and V can go straight into a frame slot of the paged
//                    cache, so the streaming append needs no second copy.
//
// Readings where the listing names a step but not its form: LayerNorms with
// weight and bias and a caller-given epsilon, a qkv bias, RoPE as a complex
// product with a per-token table [P, D/2] of (cos, sin).
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cmath>
#include <cstdint>

#include "internal.h"
#include "ptx.cuh"
#include "tile_sched.h"

namespace swa {
namespace {

// 2-D tiled TMA load into shared memory (x = innermost coordinate, in elements;
// x times the element size must be a multiple of 16 bytes)
SWA_DEV void tma_load_2d(uint32_t dst, const void* tmap, uint32_t mbar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(mbar)
      : "memory");
}

// ---------------------------------------------------------------- norm1
// One warp per token row; each lane owns the 16-byte chunks lane, lane + 32, ...
__global__ void __launch_bounds__(256) ln_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                      const float* __restrict__ w, const float* __restrict__ b,
                                                      __nv_bfloat16* __restrict__ out, int P, int C, float eps) {
  griddep_launch_dependents();  // the qkv GEMM may set up and load weights meanwhile
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= P) return;
  constexpr int kMaxChunks = 8;  // C <= 2048
  const int nch = C / 256;       // 8-element chunks per lane
  const __nv_bfloat16* xr = x + static_cast<int64_t>(row) * C;
  // all of the row's loads, the LayerNorm weight and bias included, are issued
  // before any is used (no early exit in the loop, so the unrolled loads are
  // independent): one memory round trip per row
  uint4 raw[kMaxChunks];
  float4 wq[kMaxChunks][2], bq[kMaxChunks][2];
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c) {
    const int col = (c * 32 + lane) * 8;
    const bool in = c < nch;
    raw[c] = in ? *reinterpret_cast<const uint4*>(xr + col) : make_uint4(0, 0, 0, 0);
    wq[c][0] = in ? __ldg(reinterpret_cast<const float4*>(w + col)) : make_float4(0.f, 0.f, 0.f, 0.f);
    wq[c][1] = in ? __ldg(reinterpret_cast<const float4*>(w + col + 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
    bq[c][0] = in ? __ldg(reinterpret_cast<const float4*>(b + col)) : make_float4(0.f, 0.f, 0.f, 0.f);
    bq[c][1] = in ? __ldg(reinterpret_cast<const float4*>(b + col + 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float v[kMaxChunks * 8];
  float s = 0.f;
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c) {
    if (c >= nch) break;
    const uint4 u = raw[c];
    const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[c * 8 + 2 * e] = __uint_as_float(w4[e] << 16);
      v[c * 8 + 2 * e + 1] = __uint_as_float(w4[e] & 0xffff0000u);
      s += v[c * 8 + 2 * e] + v[c * 8 + 2 * e + 1];
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  const float mean = s / C;
  float q = 0.f;
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c) {
    if (c >= nch) break;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float d = v[c * 8 + e] - mean;
      q += d * d;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) q += __shfl_xor_sync(0xffffffffu, q, off);
  const float rs = rsqrtf(q / C + eps);
  __nv_bfloat16* orow = out + static_cast<int64_t>(row) * C;
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c) {
    if (c >= nch) break;
    const int col = (c * 32 + lane) * 8;
    const float4 w0 = wq[c][0], w1 = wq[c][1], b0 = bq[c][0], b1 = bq[c][1];
    const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a0 = (v[c * 8 + 2 * e] - mean) * rs * wv[2 * e] + bv[2 * e];
      const float a1 = (v[c * 8 + 2 * e + 1] - mean) * rs * wv[2 * e + 1] + bv[2 * e + 1];
      o[e] = pack_bf16x2(a0, a1);
    }
    *reinterpret_cast<uint4*>(orow + col) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ---------------------------------------------------------------- qkv GEMM
constexpr double kTwoPi = 6.283185307179586476925286766559;
constexpr double kInvTwoPi = 0.15915494309189533576888376337251;

constexpr int kPreThreads = 192;  // warp 0 TMA, warp 1 MMA + TMEM, warps 2-5 epilogue
constexpr int kPreM = 128;        // tokens per tile
constexpr int kPreN = 128;        // output features per tile (2 heads of 64 or 1 of 128)
constexpr int kPreStages = 3;     // 96 KB of ring: two CTAs per SM, one's epilogue overlaps
                                  // the other's main loop
constexpr int kPreABytes = kPreM * 64 * 2;  // 16 KB: 128 rows x 64 columns
constexpr int kPreBBytes = kPreN * 64 * 2;  // 16 KB
constexpr int kPreStageBytes = kPreABytes + kPreBBytes;
constexpr int kPreOffBar = kPreStages * kPreStageBytes;
// the tile's per-feature epilogue constants, staged once: bias, then the q/k
// norm weight and bias of each feature's head position (3 x 128 floats)
constexpr int kPreOffPar = kPreOffBar + 128;
constexpr int kPreSmem = kPreOffPar + 3 * kPreN * 4 + 1024;

template <int D>
__global__ void __launch_bounds__(kPreThreads, 2) qkv_pre_kernel(const __grid_constant__ PreParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw_base);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kPreM;
  const int n0 = blockIdx.y * kPreN;
  const int KC = p.C / 64;  // 64-column chunks of the reduction
  const uint32_t bar0 = base + kPreOffBar;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kPreStages + s); };
  const uint32_t acc_full = bar0 + 8u * (2 * kPreStages);
  const uint32_t tmem_slot = acc_full + 8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPreStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(acc_full, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kPreN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + (tmem_slot - base));

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&p.tm_a);
      tma_prefetch_desc(&p.tm_b);
      // the first stages' weight tiles do not depend on norm1, which may still
      // run (programmatic launch): load them, then wait for norm1's output
      const int first = KC < kPreStages ? KC : kPreStages;
      for (int kc = 0; kc < first; ++kc) {
        mbar_arrive_expect_tx(full(kc), kPreStageBytes);
        tma_load_2d(base + kc * kPreStageBytes + kPreABytes, &p.tm_b, full(kc), kc * 64, n0);
      }
      griddep_wait();
      for (int kc = 0; kc < first; ++kc) tma_load_2d(base + kc * kPreStageBytes, &p.tm_a, full(kc), kc * 64, m0);
      int issued = first;
      for (int kc = first; kc < KC; ++kc) {
        const int s = kc % kPreStages;
        if (!mbar_wait(empty(s), ((kc / kPreStages) - 1) & 1, p.err, ERR_WAIT_TMA)) break;
        const uint32_t dst = base + s * kPreStageBytes;
        mbar_arrive_expect_tx(full(s), kPreStageBytes);
        tma_load_2d(dst, &p.tm_a, full(s), kc * 64, m0);
        tma_load_2d(dst + kPreABytes, &p.tm_b, full(s), kc * 64, n0);
        ++issued;
      }
      for (int kc = issued - kPreStages; kc < issued; ++kc) {
        if (kc < 0) continue;
        mbar_wait(full(kc % kPreStages), (kc / kPreStages) & 1, p.err, ERR_WAIT_TMA);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kPreM, kPreN, 0);
      const uint64_t da0 = sdesc_sw128(base, 16, 1024);
      const uint64_t db0 = sdesc_sw128(base + kPreABytes, 16, 1024);
      bool ok = true;
      for (int kc = 0; kc < KC && ok; ++kc) {
        const int s = kc % kPreStages;
        if (!mbar_wait(full(s), (kc / kPreStages) & 1, p.err, ERR_WAIT_MMA)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t step = static_cast<uint64_t>(s * (kPreStageBytes >> 4));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem, da0 + step + 2 * kk, db0 + step + 2 * kk, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
        mma_commit(empty(s));
      }
      mma_commit(acc_full);
      mbar_wait(acc_full, 0, p.err, ERR_WAIT_MMA);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;  // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;
    const int row = m0 + r;
    const int sec = n0 / p.C;            // 0: q, 1: k, 2: v
    const int h0 = (n0 - sec * p.C) / D;  // first head of this tile
    // while the main loop runs, stage the tile's bias and norm constants in
    // shared memory (thread r takes feature r of the tile), so the epilogue's
    // loop reads no global memory except the RoPE table
    float* par = reinterpret_cast<float*>(gbase + kPreOffPar);
    {
      const float* nwg = sec == 0 ? p.qn_w : p.kn_w;
      const float* nbg = sec == 0 ? p.qn_b : p.kn_b;
      par[r] = __ldg(p.b_qkv + n0 + r);
      par[kPreN + r] = sec < 2 ? __ldg(nwg + (r % D)) : 0.f;
      par[2 * kPreN + r] = sec < 2 ? __ldg(nbg + (r % D)) : 0.f;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");  // the four epilogue warps
    // head_dim 64: this token's RoPE table row (32 pairs, the same for both
    // heads of the tile) is loaded into registers before the accumulator is ready
    float4 rotv[D == 64 ? 16 : 1];
    if constexpr (D == 64) {
      const float4* rt = reinterpret_cast<const float4*>(p.rot + static_cast<int64_t>(row < p.P ? row : 0) * D);
#pragma unroll
      for (int i = 0; i < 16; ++i) rotv[i] = (p.rot && row < p.P) ? __ldg(rt + i) : make_float4(1.f, 0.f, 1.f, 0.f);
    }
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0, p.err, ERR_WAIT_EPI));
    if (ok) {
      tc_fence_after();
      const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;

      // load 32 columns of this thread's row (+ bias) from TMEM
      auto load32 = [&](int hh, int c0, float* v) {
        __syncwarp();  // tcgen05.ld is warp-collective: all lanes converged
        uint32_t a[32];
        tmem_ld32(tmem + lane_off + hh * D + c0, a);
        tmem_wait_ld();
        const float4* bias = reinterpret_cast<const float4*>(par + hh * D + c0);
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const float4 bb = bias[j / 4];
          v[j] = __uint_as_float(a[j]) + bb.x;
          v[j + 1] = __uint_as_float(a[j + 1]) + bb.y;
          v[j + 2] = __uint_as_float(a[j + 2]) + bb.z;
          v[j + 3] = __uint_as_float(a[j + 3]) + bb.w;
        }
      };
      // this token's (h, w) grid position for the generated 3-D RoPE
      const int rope_k = row - p.rope_special;
      const int rope_h = (p.rot || rope_k < 0) ? 0 : rope_k / p.rope_grid_w;
      const int rope_w = (p.rot || rope_k < 0) ? 0 : rope_k - rope_h * p.rope_grid_w;
#pragma unroll 1
      for (int hh = 0; hh < kPreN / D; ++hh) {
        const bool valid = row < p.P;
        const int h = h0 + hh;
        uint8_t* dst;
        if (sec == 0)
          dst = reinterpret_cast<uint8_t*>(p.q_out) + (static_cast<int64_t>(valid ? row : 0) * p.H + h) * D * 2;
        else
          dst = (sec == 1 ? p.k_dst : p.v_dst) + static_cast<int64_t>(valid ? row : 0) * p.kv_row_bytes + h * D * 2;
        // q and k: LayerNorm statistics of the head first (sum and sum of squares)
        float mean = 0.f, rs = 1.f;
        if (sec < 2) {
          float s1 = 0.f, s2 = 0.f;
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            float v[32];
            load32(hh, c0, v);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              s1 += v[j];
              s2 += v[j] * v[j];
            }
          }
          mean = s1 / D;
          rs = rsqrtf(fmaxf(s2 / D - mean * mean, 0.f) + p.eps);
        }
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) {
          float v[32];
          load32(hh, c0, v);
          if (sec < 2) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              const float4 ww = *reinterpret_cast<const float4*>(par + kPreN + hh * D + c0 + j);
              const float4 bb = *reinterpret_cast<const float4*>(par + 2 * kPreN + hh * D + c0 + j);
              v[j] = (v[j] - mean) * rs * ww.x + bb.x;
              v[j + 1] = (v[j + 1] - mean) * rs * ww.y + bb.y;
              v[j + 2] = (v[j + 2] - mean) * rs * ww.z + bb.z;
              v[j + 3] = (v[j + 3] - mean) * rs * ww.w + bb.w;
            }
            if (valid && p.rot) {
              // RoPE: pairs (2i, 2i+1) times (cos, sin) of pair i; two pairs per 16-byte load
              const float4* rt = reinterpret_cast<const float4*>(p.rot + static_cast<int64_t>(row) * D + c0);
#pragma unroll
              for (int j = 0; j < 32; j += 4) {
                const float4 cs = (D == 64) ? rotv[((c0 + j) / 4) % (D == 64 ? 16 : 1)] : __ldg(rt + j / 4);
                const float x0 = v[j], x1 = v[j + 1], x2 = v[j + 2], x3 = v[j + 3];
                v[j] = x0 * cs.x - x1 * cs.y;
                v[j + 1] = x0 * cs.y + x1 * cs.x;
                v[j + 2] = x2 * cs.z - x3 * cs.w;
                v[j + 3] = x2 * cs.w + x3 * cs.z;
              }
            } else if (valid) {
              // 3-D RoPE generated here: the pair's angle pos * inv_freq in double,
              // reduced to [-pi, pi] in double, then sin and cos in float
#pragma unroll
              for (int j = 0; j < 32; j += 2) {
                const int pair = (c0 + j) >> 1;
                const int pos = pair < p.rope_nt ? p.rope_frame : (pair < p.rope_nt + p.rope_nh ? rope_h : rope_w);
                const double ang = static_cast<double>(pos) * p.rope_inv_freq[pair];
                const double red = fma(-rint(ang * kInvTwoPi), kTwoPi, ang);
                float sn, cs;
                __sincosf(static_cast<float>(red), &sn, &cs);
                const float x0 = v[j], x1 = v[j + 1];
                v[j] = x0 * cs - x1 * sn;
                v[j + 1] = x0 * sn + x1 * cs;
              }
            }
          }
          if (valid) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              uint4 u;
              u.x = pack_bf16x2(v[j], v[j + 1]);
              u.y = pack_bf16x2(v[j + 2], v[j + 3]);
              u.z = pack_bf16x2(v[j + 4], v[j + 5]);
              u.w = pack_bf16x2(v[j + 6], v[j + 7]);
              *reinterpret_cast<uint4*>(dst + (c0 + j) * 2) = u;
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kPreN);
  }
}

// ---------------------------------------------------------------- 3-D RoPE table
// One thread per (token, pair): token k of frame t sits at (t, h, w) = (t,
// (k - s) / grid_w, (k - s) % grid_w) for patch tokens, (t, 0, 0) for the s
// special tokens; pair j of an axis band of n pairs turns by pos * theta^(-j/n).
// The bands split the head_dim/2 pairs as t | h | w with h = w = head_dim / 6
// pairs (the I/O page's 3-D RoPE, WanRotaryPosEmbed).  Angles in double so the
// table does not lose accuracy at large frame indices.
__global__ void rope3d_table_kernel(float* __restrict__ rot, int frame, int P, int ns, int grid_w, int half,
                                    int n_t, int n_h, double log_theta) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(P) * half) return;
  const int k = static_cast<int>(idx / half);
  const int j = static_cast<int>(idx - static_cast<int64_t>(k) * half);
  const int h = k < ns ? 0 : (k - ns) / grid_w;
  const int w = k < ns ? 0 : (k - ns) % grid_w;
  int pos, jj, n;
  if (j < n_t) {
    pos = frame; jj = j; n = n_t;
  } else if (j < n_t + n_h) {
    pos = h; jj = j - n_t; n = n_h;
  } else {
    pos = w; jj = j - n_t - n_h; n = half - n_t - n_h;
  }
  const double ang = static_cast<double>(pos) * exp(-log_theta * jj / n);
  double sn, cs;
  sincos(ang, &sn, &cs);
  reinterpret_cast<float2*>(rot)[idx] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
}

template <int D>
cudaError_t launch_pre_d(const PreParams& p, cudaStream_t stream) {
  static DeviceOnce attr_set;  // devices on which the smem opt-in was set
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (!attr_set.done(dev)) {
    const cudaError_t e =
        cudaFuncSetAttribute(qkv_pre_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPreSmem);
    if (e != cudaSuccess) return e;
    attr_set.mark(dev);
  }
  dim3 grid(cdiv(p.P, kPreM), 3 * p.C / kPreN);
  // after norm1 on the same stream: programmatic launch (see the producer)
  const cudaError_t e = launch_after(qkv_pre_kernel<D>, grid, dim3(kPreThreads), kPreSmem, stream, p);
  count_launches(1);
  return e;
}

}  // namespace

cudaError_t launch_ln_rows(const void* x, const float* w, const float* b, void* out, int P, int C, float eps,
                           cudaStream_t stream) {
  if (P <= 0) return cudaSuccess;
  ln_rows_kernel<<<cdiv(P, 8), 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(x), w, b,
                                                  static_cast<__nv_bfloat16*>(out), P, C, eps);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_rope3d_table(float* rot, int frame, int P, int num_special, int grid_w, int head_dim,
                                double theta, cudaStream_t stream) {
  const int half = head_dim / 2;
  const int n_h = head_dim / 6;
  const int n_t = half - 2 * n_h;
  const int64_t n = static_cast<int64_t>(P) * half;
  if (n <= 0) return cudaSuccess;
  rope3d_table_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
      rot, frame, P, num_special, grid_w, half, n_t, n_h, std::log(theta));
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_qkv_pre(const PreParams& p, cudaStream_t stream) {
  if (p.P <= 0) return cudaSuccess;
  if (p.D == 64) return launch_pre_d<64>(p, stream);
  if (p.D == 128) return launch_pre_d<128>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace swa
