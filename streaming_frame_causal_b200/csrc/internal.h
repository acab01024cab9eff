// internal.h -- declarations shared by the host API (api.cu) and the kernel
// translation units.  Not part of the public C ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>

namespace swa {

// One bit per device (ids 0..63) recording that a per-device setting, such as a
// kernel's shared-memory opt-in, has been made; safe for concurrent host
// threads.  Devices beyond 63 are never marked, so the setting is simply
// repeated on every call there.
struct DeviceOnce {
  std::atomic<uint64_t> mask{0};
  bool done(int dev) const {
    return dev >= 0 && dev < 64 && ((mask.load(std::memory_order_acquire) >> dev) & 1u);
  }
  void mark(int dev) {
    if (dev >= 0 && dev < 64) mask.fetch_or(uint64_t{1} << dev, std::memory_order_acq_rel);
  }
};

enum TcMode : int { TC_FRAME = 0, TC_STREAM = 1, TC_BAND = 2 };

// Parameters of the tcgen05 attention kernel (passed by value as a
// __grid_constant__ so the TMA descriptors are addressable by the kernel).
struct TcParams {
  CUtensorMap tm_q;   // Q as 4-D {D, Hq, Nq, B}, box {64, 1, 128, 1}, 128-byte swizzle
  CUtensorMap tm_k;   // K as 4-D {D, Hkv, Nk, B}
  CUtensorMap tm_v;   // V, same shape as K
  void* out;          // bf16 [B, Nq, Hq, D] (final output)
  float* part_o;      // f32 [splits, Nq, Hq, D] (split-KV partial numerators)
  float* part_ml;     // f32 [splits, Nq, Hq, 2] (running max in log2 units, row sum)
  const int* seg_row; // stream mode: key segments (storage row, length) on the device
  const int* seg_len;
  const int* meta_hdr;
  int* err;           // device error flag
  int mode;
  int B, Nq, Hq, Hkv;
  int P, F, S, Wf, n_pairs;  // frame mode (P, n_pairs also stream mode)
  int W, n_qtiles;           // band mode
  int splits, max_segs;      // stream mode
  float scale_log2;          // log2(e) / sqrt(D)
  int64_t out_ld;            // elements between consecutive token rows of out (0: Hq * D)
  int out_h0;                // head of out that query head 0 writes (a head slice of wider rows)
};

cudaError_t launch_attn_tc(const TcParams& p, int head_dim, int64_t n_items, cudaStream_t stream);
// merge ``splits`` (<= 32) split-KV partials [splits, rows, H, D] into bf16 out rows
// out_ld elements apart (heads from out_h0); a programmatic launch that waits for
// the attend ahead of it on the stream
cudaError_t launch_combine(const float* part_o, const float* part_ml, void* out, int rows, int H, int splits,
                           int head_dim, int64_t out_ld, int out_h0, cudaStream_t stream);
int tc_smem_bytes(int head_dim);

// ---------------------------------------------------------------- SIMT f32 path
enum SimtMode : int { SIMT_FRAME = 0, SIMT_BAND = 1, SIMT_STREAM = 2, SIMT_DECODE = 3 };

struct SimtParams {
  const float* q;    // [B, Nq, Hq, D]
  const float* k;    // [B, Nk, Hkv, D] (stream: page storage rows; decode: [B, W, Hkv, D])
  const float* v;
  float* out;        // [B, Nq, Hq, D]
  const int* seg_row;
  const int* seg_len;
  const int* meta_hdr;
  int* err;
  int mode;
  int B, Nq, Nk, Hq, Hkv, D;
  int P, S, Wf;      // frame
  int W;             // band
  int n_valid;       // decode: valid slots
  int max_segs;
  float scale;
  int64_t q_ld;      // elements between token rows of q and out (0: Hq * D)
  int q_h0;          // head of q / out that query head 0 reads and writes
  int64_t kv_ld;     // elements between token rows of k and v (0: Hkv * D)
  int kv_h0;         // head of k / v that KV head 0 reads
};

cudaError_t launch_attn_simt(const SimtParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- stream cache
struct AppendParams {
  const uint8_t* k_src;  // [P, H, D] of the new frame
  const uint8_t* v_src;
  uint8_t* k_store;      // page storage [total_rows, H, D]
  uint8_t* v_store;
  int* meta;             // the layer's metadata block
  int* err;              // device error flag
  int frame;             // index of the frame being appended
  int P, S, Wc, ppf, page_tokens, n_slots, num_special, cross_special;
  int row_bytes;         // H * D * element size (multiple of 16)
  int off_slot_frame, off_page_table, off_seg_row, off_seg_len;
  int max_pages, max_segs;
  int copy;              // 0: move specials and rewrite metadata only (the frame's K/V
                         // are written into its slot by the attn_pre prologue)
  int64_t src_row_bytes; // bytes between consecutive tokens of k_src / v_src
  int64_t src_off;       // byte offset of the cached heads within a source token row
};

cudaError_t launch_append_evict(const AppendParams& p, cudaStream_t stream);

// Non-keyframe attend, preparation: the frame's K/V go to the scratch frame's
// pages, and the layer's non-keyframe area gets the persistent key runs plus the
// scratch run (the persistent metadata is only read).
struct TransientParams {
  const uint8_t* k_src;  // [P, H, D] of the non-keyframe
  const uint8_t* v_src;
  uint8_t* k_store;      // page storage [total_rows, H, D]
  uint8_t* v_store;
  int* meta;             // the layer's metadata block
  int* err;              // device error flag
  int P, row_bytes, page_tokens, scratch_page;
  int off_seg_row, off_seg_len, max_segs, t_off;
};

cudaError_t launch_transient_prepare(const TransientParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- decode
struct DecodeParams {
  CUtensorMap tm_k;   // K cache [B, W, Hkv, D] as 4-D, box 64 x 1 x 128 x 1, 128-byte swizzle
  CUtensorMap tm_v;   // V cache, the same
  CUtensorMap tm_q;   // q as [B*Hq, D], box 64 x 16, 128-byte swizzle
  const void* q;      // [B, Hq, D]
  const void* k_new;  // [B, Hkv, D]
  const void* v_new;
  void* k_cache;      // [B, W, Hkv, D]
  void* v_cache;
  void* out;          // [B, Hq, D]
  float* part_o;      // [B, Hkv, chunks, G, D]
  float* part_ml;     // [B, Hkv, chunks, G, 2]
  int* err;
  long long pos;
  int W, B, Hq, Hkv, D, chunks, chunk_len, n_valid, slot;
  float scale_log2;
};

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int D, int W);
// tensor-core decode (head_dim 64 or 128, G = 1..8): appends the new token,
// runs the persistent kernel and the combine; p.chunks = partial slots available
bool decode_tc_supported(int D, int G);
int decode_tc_pieces(int B, int Hkv, int n_valid, int max_pieces, int sms);
// the launch the tensor-core decode makes: pieces of the valid window per
// (batch, KV head), slots per piece (whole 128-key tiles), persistent CTAs
struct DecodeTcPlan {
  int pieces, piece_len, grid;
};
DecodeTcPlan decode_tc_plan(int B, int Hkv, int n_valid, int max_pieces, int sms);
cudaError_t launch_decode_tc(const DecodeParams& p, int sms, cudaStream_t stream);
cudaError_t launch_decode_combine(const DecodeParams& p, cudaStream_t stream);
// bf16 [B, N, H, D] as a 4-D map {D, H, N, B}, box 64 x 1 x 128 x 1, 128-byte swizzle
bool encode_4d_sw128(CUtensorMap* m, const void* base, int D, int H, int64_t N, int B);
int device_sms();
// bf16 matrix [rows, inner] (inner contiguous) as a 2-D map; box = 64 columns x
// box_rows rows, 128-byte swizzle
bool encode_2d_sw128(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int box_rows);

// ---------------------------------------------------------------- attn_pre prologue
struct PreParams {
  CUtensorMap tm_a;     // norm1 output [P, C] bf16, box 64 x 128
  CUtensorMap tm_b;     // w_qkv [3C, C] bf16, box 64 x 128
  const float* b_qkv;   // [3C]
  const float* qn_w;    // [D] q_norm weight / bias
  const float* qn_b;
  const float* kn_w;    // [D] k_norm weight / bias
  const float* kn_b;
  const float* rot;     // [P, D/2, 2]: (cos, sin) per token and pair
  void* q_out;          // [P, H, D] bf16
  uint8_t* k_dst;       // K rows: [P, H, D] at row stride k_row_bytes (a buffer or cache slot rows)
  uint8_t* v_dst;
  int64_t kv_row_bytes; // H * D * 2
  int* err;
  int P, C, H, D;
  float eps;
  // 3-D RoPE generated in the epilogue when rot is null: token k sits at
  // (t, h, w) = (rope_frame, (k - s) / rope_grid_w, (k - s) % rope_grid_w) for
  // k >= s = rope_special and at (rope_frame, 0, 0) below; pair j < rope_nt turns
  // by t, j < rope_nt + rope_nh by h, the rest by w, times rope_inv_freq[j]
  int rope_frame, rope_special, rope_grid_w, rope_nt, rope_nh;
  double rope_inv_freq[64];
};
cudaError_t launch_ln_rows(const void* x, const float* w, const float* b, void* out, int P, int C, float eps,
                           cudaStream_t stream);
cudaError_t launch_qkv_pre(const PreParams& p, cudaStream_t stream);
cudaError_t launch_rope3d_table(float* rot, int frame, int P, int num_special, int grid_w, int head_dim,
                                double theta, cudaStream_t stream);
int decode_chunks(int B, int Hkv, int W);
cudaError_t launch_decode_bf16(const DecodeParams& p, cudaStream_t stream);
cudaError_t launch_decode_write_f32(const DecodeParams& p, cudaStream_t stream);

// ---------------------------------------------------------------- misc
// device address of the library's error flag on the current device (nullptr on failure)
int* device_error_flag();
// 0 (SWA_OK) with *err = that flag; SWA_ERR_TIMEOUT while an error latched by an
// earlier launch on the device is uncleared; SWA_ERR_CUDA if the flag cannot be set up
int device_ready_status(int** err);
// counts kernel launches (every launch_* helper adds what it enqueued)
void count_launches(int n);

// Launch ``kernel`` so that it may start before the kernel ahead of it on
// ``stream`` has finished (programmatic dependent launch): the kernel's own set-up
// and its loads of inputs that kernel does not write overlap that kernel's tail;
// it calls griddep_wait() before touching anything the kernel ahead writes.
template <typename... Params, typename... Args>
cudaError_t launch_after(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                         Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}
cudaError_t launch_exp2_poly(const float* x, float* y, int n, cudaStream_t stream);
cudaError_t launch_debug_wait(int* err, long long timeout_ns, cudaStream_t stream);

}  // namespace swa
