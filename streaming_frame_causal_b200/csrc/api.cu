// api.cu -- the C ABI declared in include/swa.h: argument validation, tensor-map
// (TMA descriptor) encoding, the streaming cache's buffer layout and host-side
// frame counters, launch sizing and dispatch to the kernels.  No device memory is
// allocated here: every buffer belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <atomic>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/swa.h"
#include "internal.h"
#include "tile_sched.h"

using namespace swa;

namespace swa {
namespace {
std::atomic<uint64_t> g_launches{0};
}
void count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }
}  // namespace swa

extern "C" uint64_t swa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

// ------------------------------------------------------------------ device flag
// The device error flag of each GPU is the first int of a 16-byte slot; its
// second 8 bytes hold the device address of that GPU's word in a page of pinned,
// mapped host memory (a static page of this library, registered once per
// process: a registration, not an allocation).  Kernels that give up a bounded
// wait set both (latch_error), so every entry point can refuse to launch while
// an error is latched by reading host memory, with no device synchronization.
namespace {
struct __align__(16) ErrSlot {
  int flag;
  int pad;
  unsigned long long host;
};
__device__ ErrSlot g_swa_err = {0, 0, 0ull};

constexpr int kMaxDevices = 64;
constexpr int kHostWordStride = 16;  // ints: one 64-byte line per device
alignas(4096) int g_host_err[kMaxDevices * kHostWordStride] = {0};
bool g_host_err_mapped = false;
int* g_err_ptr[kMaxDevices] = {nullptr};
int g_num_sms[kMaxDevices] = {0};
std::mutex g_mu;

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return (d >= 0 && d < kMaxDevices) ? d : -1;
}

volatile int* host_err_word(int d) { return g_host_err + d * kHostWordStride; }

// Device flag of the current device, set up on first use: its address, and the
// host mirror word's device address written into the slot.  Without a mapped
// host page (registration refused) the slot's host pointer stays 0 and latched
// errors surface only through swa_device_error_check.
int* err_ptr() {
  const int d = current_device();
  if (d < 0) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[d]) {
    static bool tried = false;
    if (!tried) {
      tried = true;
      g_host_err_mapped = cudaHostRegister(g_host_err, sizeof(g_host_err),
                                           cudaHostRegisterMapped | cudaHostRegisterPortable) == cudaSuccess;
      if (!g_host_err_mapped) cudaGetLastError();  // clear the error a refused registration leaves
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_swa_err) != cudaSuccess) return nullptr;
    unsigned long long host_dev = 0;
    if (g_host_err_mapped) {
      void* hp = nullptr;
      if (cudaHostGetDevicePointer(&hp, const_cast<int*>(host_err_word(d)), 0) == cudaSuccess)
        host_dev = reinterpret_cast<unsigned long long>(hp);
      else
        cudaGetLastError();
    }
    if (cudaMemcpy(static_cast<uint8_t*>(p) + 8, &host_dev, sizeof(host_dev), cudaMemcpyHostToDevice) !=
        cudaSuccess)
      return nullptr;
    g_err_ptr[d] = static_cast<int*>(p);
  }
  return g_err_ptr[d];
}

// SWA_OK with *err = the current device's flag; SWA_ERR_TIMEOUT while an error
// latched by an earlier launch on this device is uncleared; SWA_ERR_CUDA if the
// flag cannot be set up.
swa_status device_ready(int** err) {
  int* e = err_ptr();
  if (!e) return SWA_ERR_CUDA;
  const int d = current_device();
  if (d >= 0 && *host_err_word(d) != 0) return SWA_ERR_TIMEOUT;
  *err = e;
  return SWA_OK;
}

int num_sms() {
  const int d = current_device();
  if (d < 0) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_num_sms[d]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0) n = 148;
    g_num_sms[d] = n;
  }
  return g_num_sms[d];
}

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// bf16 tensor [B, N, H, D] (D contiguous) as a 4-D map {D, H, N, B}; box = 64
// columns x 1 head x 128 rows, 128-byte swizzle (one box = one 16 KB operand
// sub-tile in the layout the tcgen05 descriptors expect).
// row_elems: elements between consecutive tokens (0: H * D, a contiguous tensor;
// larger when the map covers a head slice of wider token rows).
bool make_map(CUtensorMap* m, const void* base, int D, int H, int64_t N, int B, int64_t row_elems = 0) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  if (row_elems == 0) row_elems = static_cast<int64_t>(H) * D;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(row_elems) * 2,
                                 static_cast<cuuint64_t>(N) * row_elems * 2};
  const cuuint32_t box[4] = {64, 1, 128, 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }


}  // namespace

bool swa::encode_2d_sw128(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool swa::encode_4d_sw128(CUtensorMap* m, const void* base, int D, int H, int64_t N, int B) {
  return make_map(m, base, D, H, N, B);
}

int swa::device_sms() { return num_sms(); }

namespace {

swa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SWA_OK : SWA_ERR_CUDA; }

bool tc_head_dim(int d) { return d == 64 || d == 128; }
bool simt_head_dim(int d) { return d == 32 || d == 64 || d == 128; }

float scale_log2(int D) { return static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(D))); }

}  // namespace

namespace swa {
int* device_error_flag() { return err_ptr(); }
int device_ready_status(int** err) { return device_ready(err); }
}  // namespace swa

// ==================================================================== status
extern "C" const char* swa_status_str(int s) {
  switch (s) {
    case SWA_OK: return "ok";
    case SWA_ERR_ARG: return "invalid argument";
    case SWA_ERR_SHAPE: return "inconsistent shape";
    case SWA_ERR_ORDER: return "frame out of order";
    case SWA_ERR_CAPACITY: return "capacity exceeded";
    case SWA_ERR_CUDA: return "CUDA error";
    case SWA_ERR_TIMEOUT: return "device wait timed out";
    case SWA_ERR_UNSUPPORTED: return "unsupported dtype/head_dim";
    default: return "unknown status";
  }
}

extern "C" int swa_version(void) { return 100; }

// ================================================================= scheduler
extern "C" int swa_sched_frame_intervals(int i, int sliding_window_size, int num_frame_per_block,
                                         int num_frame_for_scale, int* lo, int* hi) {
  if (!lo || !hi || i < 0 || num_frame_per_block < 1) return SWA_ERR_ARG;
  const int Wf = window_frames(sliding_window_size, num_frame_per_block);
  return frame_intervals(i, Wf, imax(0, num_frame_for_scale), lo, hi);
}

extern "C" int64_t swa_sched_prefill(int B, int S, int P, int heads, int sliding_window_size,
                                     int num_frame_per_block, int num_frame_for_scale, int32_t* out,
                                     int64_t cap) {
  if (B < 0 || S < 0 || P < 1 || heads < 1 || num_frame_per_block < 1) return SWA_ERR_ARG;
  const int n_pairs = qpairs_per_frame(P);
  const int64_t n = static_cast<int64_t>(S) * B * heads * n_pairs;
  if (!out) return n;
  const int Wf = window_frames(sliding_window_size, num_frame_per_block);
  const int Sc = imax(0, num_frame_for_scale);
  for (int64_t w = 0; w < n && w < cap; ++w) {
    const PrefillItem it = prefill_item(w, B, heads, S, n_pairs);
    int lo[2], hi[2];
    const int ns = frame_intervals(it.f, Wf, Sc, lo, hi);
    int tiles = 0, toks = 0;
    for (int s = 0; s < ns; ++s) {
      tiles += cdiv((hi[s] - lo[s]) * P, kTileRows);
      toks += (hi[s] - lo[s]) * P;
    }
    int32_t* r = out + 8 * w;
    r[0] = it.b;
    r[1] = it.h;
    r[2] = it.f;
    r[3] = it.f * P + 2 * it.pair * kTileRows;
    r[4] = qtile_rows(P, 2 * it.pair);
    r[5] = qtile_rows(P, 2 * it.pair + 1);
    r[6] = tiles;
    r[7] = toks;
  }
  return n;
}

namespace {
int choose_splits(int T, int items_per_split, int max_splits, int sms);
}

extern "C" int swa_sched_stream(int key_tiles, int heads, int P, int max_splits, int sms, int32_t* out) {
  if (key_tiles < 1 || heads < 1 || P < 1 || max_splits < 1 || max_splits > 32 || sms < 1 || !out)
    return SWA_ERR_ARG;
  const int items = heads * qpairs_per_frame(P);
  const int splits = choose_splits(key_tiles, items, max_splits, sms);
  int lo = key_tiles, hi = 0;  // fewest and most key tiles of a split
  for (int s = 0; s < splits; ++s) {
    int t0, t1;
    split_range(key_tiles, splits, s, &t0, &t1);
    lo = imin(lo, t1 - t0);
    hi = imax(hi, t1 - t0);
  }
  out[0] = splits;
  out[1] = items * splits;
  out[2] = lo;
  out[3] = hi;
  return SWA_OK;
}

extern "C" int swa_sched_decode(int B, int Hkv, int W, long long pos, int sms, int32_t* out) {
  if (B < 1 || Hkv < 1 || W < 1 || pos < 0 || sms < 1 || !out) return SWA_ERR_ARG;
  const int n_valid = (pos >= W - 1) ? W : static_cast<int>(pos + 1);
  const int slots = decode_chunks(B, Hkv, W);
  const DecodeTcPlan pl = decode_tc_plan(B, Hkv, n_valid, slots, sms);
  out[0] = pl.pieces;
  out[1] = pl.piece_len;
  out[2] = pl.grid;
  out[3] = slots;
  out[4] = n_valid;
  return SWA_OK;
}

// ==================================================================== prefill
namespace {
// The prefill over heads [head0, head0 + heads) of token rows ``row_stride``
// elements apart (the whole tensor when head0 = 0 and row_stride = heads * D).
swa_status prefill_impl(const void* q, const void* k, const void* v, void* out, int B, int S, int P,
                        int64_t row_stride, int head0, int heads, int head_dim, int sliding_window_size,
                        int num_frame_per_block, int num_frame_for_scale, int dtype, void* stream) {
  if (B == 0 || S == 0) return SWA_OK;
  if (!q || !k || !v || !out) return SWA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SWA_ERR_ARG;
  const int esize = dtype == SWA_F32 ? 4 : 2;
  if ((row_stride * esize) % 16 != 0 || (static_cast<int64_t>(head0) * head_dim * esize) % 16 != 0)
    return SWA_ERR_ARG;
  int* err = nullptr;
  if (const swa_status ds = device_ready(&err)) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int N = S * P;
  const int Wf = window_frames(sliding_window_size, num_frame_per_block);
  const int Sc = imax(0, num_frame_for_scale);
  if (dtype == SWA_F32) {
    if (!simt_head_dim(head_dim)) return SWA_ERR_UNSUPPORTED;
    SimtParams p{};
    p.q = static_cast<const float*>(q);
    p.k = static_cast<const float*>(k);
    p.v = static_cast<const float*>(v);
    p.out = static_cast<float*>(out);
    p.err = err;
    p.mode = SIMT_FRAME;
    p.B = B;
    p.Nq = N;
    p.Nk = N;
    p.Hq = heads;
    p.Hkv = heads;
    p.D = head_dim;
    p.P = P;
    p.S = Sc;
    p.Wf = Wf;
    p.scale = 1.f / std::sqrt(static_cast<float>(head_dim));
    p.q_ld = p.kv_ld = row_stride;
    p.q_h0 = p.kv_h0 = head0;
    return cuda_status(launch_attn_simt(p, st));
  }
  if (!tc_head_dim(head_dim)) return SWA_ERR_UNSUPPORTED;
  const size_t off = static_cast<size_t>(head0) * head_dim * 2;
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  if (!make_map(&p.tm_q, static_cast<const uint8_t*>(q) + off, head_dim, heads, N, B, row_stride) ||
      !make_map(&p.tm_k, static_cast<const uint8_t*>(k) + off, head_dim, heads, N, B, row_stride) ||
      !make_map(&p.tm_v, static_cast<const uint8_t*>(v) + off, head_dim, heads, N, B, row_stride))
    return SWA_ERR_CUDA;
  p.out = out;
  p.out_ld = row_stride;
  p.out_h0 = head0;
  p.err = err;
  p.mode = TC_FRAME;
  p.B = B;
  p.Nq = N;
  p.Hq = heads;
  p.Hkv = heads;
  p.P = P;
  p.F = S;
  p.S = Sc;
  p.Wf = Wf;
  p.n_pairs = qpairs_per_frame(P);
  p.splits = 1;
  p.scale_log2 = scale_log2(head_dim);
  const int64_t items = static_cast<int64_t>(S) * B * heads * p.n_pairs;
  if (items > 0x7fffffffLL) return SWA_ERR_SHAPE;
  return cuda_status(launch_attn_tc(p, head_dim, items, st));
}
}  // namespace

extern "C" swa_status swa_prefill(const void* q, const void* k, const void* v, void* out, int B, int S, int P,
                                  int C, int heads, int head_dim, int sliding_window_size,
                                  int num_frame_per_block, int num_frame_for_scale, int dtype, void* stream) {
  if (B < 0 || S < 0 || P < 1 || heads < 1 || head_dim < 1 || num_frame_per_block < 1) return SWA_ERR_ARG;
  if (dtype != SWA_F32 && dtype != SWA_BF16) return SWA_ERR_ARG;
  if (C != heads * head_dim) return SWA_ERR_SHAPE;
  if (static_cast<int64_t>(S) * P > 0x7fffffffLL) return SWA_ERR_SHAPE;
  return prefill_impl(q, k, v, out, B, S, P, C, 0, heads, head_dim, sliding_window_size, num_frame_per_block,
                      num_frame_for_scale, dtype, stream);
}

extern "C" swa_status swa_prefill_heads(const void* q, const void* k, const void* v, void* out, int B, int S,
                                        int P, int row_stride, int head0, int heads, int head_dim,
                                        int sliding_window_size, int num_frame_per_block, int num_frame_for_scale,
                                        int dtype, void* stream) {
  if (B < 0 || S < 0 || P < 1 || heads < 1 || head_dim < 1 || num_frame_per_block < 1 || head0 < 0)
    return SWA_ERR_ARG;
  if (dtype != SWA_F32 && dtype != SWA_BF16) return SWA_ERR_ARG;
  if (static_cast<int64_t>(row_stride) < static_cast<int64_t>(head0 + heads) * head_dim) return SWA_ERR_SHAPE;
  if (static_cast<int64_t>(S) * P > 0x7fffffffLL) return SWA_ERR_SHAPE;
  return prefill_impl(q, k, v, out, B, S, P, row_stride, head0, heads, head_dim, sliding_window_size,
                      num_frame_per_block, num_frame_for_scale, dtype, stream);
}

// =================================================================== band GQA
extern "C" swa_status swa_band_prefill(const void* q, const void* k, const void* v, void* out, int B, int N,
                                       int Hq, int Hkv, int head_dim, int window, int dtype, void* stream) {
  if (B < 0 || N < 0 || Hq < 1 || Hkv < 1 || head_dim < 1 || window < 1) return SWA_ERR_ARG;
  if (dtype != SWA_F32 && dtype != SWA_BF16) return SWA_ERR_ARG;
  if (Hq % Hkv) return SWA_ERR_SHAPE;
  if (B == 0 || N == 0) return SWA_OK;
  if (!q || !k || !v || !out) return SWA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SWA_ERR_ARG;
  int* err = nullptr;
  if (const swa_status ds = device_ready(&err)) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == SWA_F32) {
    if (!simt_head_dim(head_dim)) return SWA_ERR_UNSUPPORTED;
    SimtParams p{};
    p.q = static_cast<const float*>(q);
    p.k = static_cast<const float*>(k);
    p.v = static_cast<const float*>(v);
    p.out = static_cast<float*>(out);
    p.err = err;
    p.mode = SIMT_BAND;
    p.B = B;
    p.Nq = N;
    p.Nk = N;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.D = head_dim;
    p.W = window;
    p.scale = 1.f / std::sqrt(static_cast<float>(head_dim));
    return cuda_status(launch_attn_simt(p, st));
  }
  if (!tc_head_dim(head_dim)) return SWA_ERR_UNSUPPORTED;
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  if (!make_map(&p.tm_q, q, head_dim, Hq, N, B) || !make_map(&p.tm_k, k, head_dim, Hkv, N, B) ||
      !make_map(&p.tm_v, v, head_dim, Hkv, N, B))
    return SWA_ERR_CUDA;
  p.out = out;
  p.err = err;
  p.mode = TC_BAND;
  p.B = B;
  p.Nq = N;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.W = window;
  p.n_qtiles = cdiv(N, kTileRows);
  p.splits = 1;
  p.scale_log2 = scale_log2(head_dim);
  const int G = Hq / Hkv;
  const int per_group = (G % 2 == 0) ? G / 2 : G;
  const int64_t items = static_cast<int64_t>(p.n_qtiles) * B * Hkv * per_group;
  if (items > 0x7fffffffLL) return SWA_ERR_SHAPE;
  return cuda_status(launch_attn_tc(p, head_dim, items, st));
}

// ==================================================================== decode
extern "C" size_t swa_decode_workspace_bytes(int B, int Hq, int Hkv, int head_dim, int W) {
  if (B < 1 || Hq < 1 || Hkv < 1 || head_dim < 1 || W < 1 || Hq % Hkv) return 0;
  return decode_workspace_bytes(B, Hq, Hkv, head_dim, W);
}

extern "C" swa_status swa_decode(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                 void* v_cache, long long pos, int W, int B, int Hq, int Hkv, int head_dim,
                                 void* out, void* workspace, size_t workspace_bytes, int dtype, void* stream) {
  if (pos < 0 || W < 1 || B < 0 || Hq < 1 || Hkv < 1 || head_dim < 1) return SWA_ERR_ARG;
  if (dtype != SWA_F32 && dtype != SWA_BF16) return SWA_ERR_ARG;
  if (Hq % Hkv) return SWA_ERR_SHAPE;
  if (B == 0) return SWA_OK;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !out) return SWA_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
      !aligned16(v_cache) || !aligned16(out))
    return SWA_ERR_ARG;
  int* err = nullptr;
  if (const swa_status ds = device_ready(&err)) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DecodeParams p{};
  p.q = q;
  p.k_new = k_new;
  p.v_new = v_new;
  p.k_cache = k_cache;
  p.v_cache = v_cache;
  p.out = out;
  p.err = err;
  p.pos = pos;
  p.W = W;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.D = head_dim;
  p.slot = static_cast<int>(pos % W);
  p.n_valid = (pos >= W - 1) ? W : static_cast<int>(pos + 1);
  p.scale_log2 = scale_log2(head_dim);
  if (dtype == SWA_F32) {
    if (!simt_head_dim(head_dim)) return SWA_ERR_UNSUPPORTED;
    cudaError_t e = launch_decode_write_f32(p, st);
    if (e != cudaSuccess) return SWA_ERR_CUDA;
    SimtParams s{};
    s.q = static_cast<const float*>(q);
    s.k = static_cast<const float*>(k_cache);
    s.v = static_cast<const float*>(v_cache);
    s.out = static_cast<float*>(out);
    s.err = err;
    s.mode = SIMT_DECODE;
    s.B = B;
    s.Nq = 1;
    s.Nk = W;
    s.Hq = Hq;
    s.Hkv = Hkv;
    s.D = head_dim;
    s.n_valid = p.n_valid;
    s.scale = 1.f / std::sqrt(static_cast<float>(head_dim));
    return cuda_status(launch_attn_simt(s, st));
  }
  if (head_dim != 64 && head_dim != 128) return SWA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G < 1 || G > 8) return SWA_ERR_UNSUPPORTED;
  const size_t need = decode_workspace_bytes(B, Hq, Hkv, head_dim, W);
  if (!workspace || workspace_bytes < need) return SWA_ERR_CAPACITY;
  if (!aligned16(workspace)) return SWA_ERR_ARG;
  p.chunks = decode_chunks(B, Hkv, W);
  const size_t n_part = static_cast<size_t>(B) * Hkv * p.chunks * G;
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = p.part_o + n_part * head_dim;
  return cuda_status(launch_decode_bf16(p, st));
}

// ================================================================= streaming
struct swa_stream {
  swa_stream_cfg cfg;
  int n_slots, ppf, special_pages, max_pages, max_segs;
  int scratch_page;  // first page of the non-keyframe scratch frame (after the special region)
  int t_off;         // offset (ints) of the non-keyframe header + key runs in a layer's metadata
  int64_t total_rows;
  int row_bytes;
  int meta_ints;
  size_t meta_stride, store_bytes, part_bytes;
  uint8_t* base;
  uint8_t* meta0;
  uint8_t* store0;
  float* part_o;
  float* part_ml;
  std::vector<int> n_frames;
  std::vector<CUtensorMap> tm_k, tm_v;
};

namespace {

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct StreamGeom {
  int n_slots, ppf, special_pages, max_pages, max_segs, meta_ints, row_bytes, scratch_page, t_off;
  int64_t total_rows;
  size_t meta_stride, store_bytes, part_bytes, total;
};

bool stream_geom(const swa_stream_cfg* c, StreamGeom* g) {
  if (!c) return false;
  if (c->num_layers < 1 || c->heads < 1 || c->head_dim < 1 || c->P < 1 || c->scale_frames < 0 ||
      c->page_tokens < 1 || c->num_special < 0 || c->num_special > c->P || c->max_frames < 1 ||
      c->max_splits < 1 || c->max_splits > 32 || (c->dtype != SWA_F32 && c->dtype != SWA_BF16))
    return false;
  const int esize = c->dtype == SWA_F32 ? 4 : 2;
  g->row_bytes = c->heads * c->head_dim * esize;
  if (g->row_bytes % 16) return false;
  g->ppf = cdiv(c->P, c->page_tokens);
  const int Wc = c->window_frames;
  g->n_slots = (Wc > 0) ? c->scale_frames + Wc : c->max_frames;
  const int max_evicted = (Wc > 0) ? imax(0, c->max_frames - c->scale_frames - Wc) : 0;
  const int64_t sp_tokens = c->cross_frame_special ? static_cast<int64_t>(max_evicted) * c->num_special : 0;
  g->special_pages = static_cast<int>(cdiv(static_cast<int>(sp_tokens), c->page_tokens));
  const int64_t pages = static_cast<int64_t>(g->n_slots) * g->ppf + g->special_pages;
  // one more frame of pages after the special region: the non-keyframe scratch frame
  if ((pages + g->ppf) * c->page_tokens > 0x7fffffffLL) return false;
  g->max_pages = static_cast<int>(pages);
  g->scratch_page = static_cast<int>(pages);
  g->max_segs = g->n_slots + 1;
  g->total_rows = (pages + g->ppf) * c->page_tokens;
  g->meta_ints = 8 + g->n_slots + g->max_pages + 2 * g->max_segs;
  // non-keyframe area after the published layout: header + key runs (one more run)
  g->t_off = g->meta_ints;
  g->meta_stride = round256(static_cast<size_t>(g->meta_ints + 8 + 2 * (g->max_segs + 1)) * 4);
  g->store_bytes = round256(static_cast<size_t>(g->total_rows) * g->row_bytes);
  const size_t rows_h = static_cast<size_t>(c->P) * c->heads;
  // split-KV partials of the attend: O, then max and sum
  g->part_bytes = round256(static_cast<size_t>(c->max_splits) * rows_h * c->head_dim * 4) +
                  round256(static_cast<size_t>(c->max_splits) * rows_h * 2 * 4);
  g->total = g->meta_stride * c->num_layers + 2 * g->store_bytes * c->num_layers + g->part_bytes;
  return true;
}

swa_status stream_check_layer(const swa_stream* h, int global_idx) {
  if (!h) return SWA_ERR_ARG;
  if (global_idx < 0 || global_idx >= h->cfg.num_layers) return SWA_ERR_CAPACITY;
  return SWA_OK;
}

int* layer_meta(const swa_stream* h, int l) { return reinterpret_cast<int*>(h->meta0 + h->meta_stride * l); }
uint8_t* layer_k(const swa_stream* h, int l) { return h->store0 + h->store_bytes * (2 * l); }
uint8_t* layer_v(const swa_stream* h, int l) { return h->store0 + h->store_bytes * (2 * l + 1); }

}  // namespace

extern "C" size_t swa_stream_cache_bytes(const swa_stream_cfg* cfg) {
  StreamGeom g;
  if (!stream_geom(cfg, &g)) return 0;
  return g.total;
}

extern "C" size_t swa_stream_bytes(const swa_stream_cfg* cfg) { return swa_stream_cache_bytes(cfg); }

extern "C" swa_status swa_stream_create(swa_stream** out, const swa_stream_cfg* cfg, void* dev_buf,
                                        size_t bytes, void* stream) {
  return swa_stream_init(out, cfg, dev_buf, bytes, stream);
}

extern "C" swa_status swa_stream_init(swa_stream** out, const swa_stream_cfg* cfg, void* dev_buf,
                                      size_t bytes, void* stream) {
  if (!out || !cfg || !dev_buf) return SWA_ERR_ARG;
  *out = nullptr;
  StreamGeom g;
  if (!stream_geom(cfg, &g)) return SWA_ERR_ARG;
  if (bytes < g.total) return SWA_ERR_CAPACITY;
  if (reinterpret_cast<uintptr_t>(dev_buf) & 255u) return SWA_ERR_ARG;
  if (cfg->dtype == SWA_BF16 && !tc_head_dim(cfg->head_dim)) return SWA_ERR_UNSUPPORTED;
  if (cfg->dtype == SWA_F32 && !simt_head_dim(cfg->head_dim)) return SWA_ERR_UNSUPPORTED;
  swa_stream* h = new (std::nothrow) swa_stream();
  if (!h) return SWA_ERR_CAPACITY;
  h->cfg = *cfg;
  h->n_slots = g.n_slots;
  h->ppf = g.ppf;
  h->special_pages = g.special_pages;
  h->max_pages = g.max_pages;
  h->max_segs = g.max_segs;
  h->total_rows = g.total_rows;
  h->scratch_page = g.scratch_page;
  h->t_off = g.t_off;
  h->row_bytes = g.row_bytes;
  h->meta_ints = g.meta_ints;
  h->meta_stride = g.meta_stride;
  h->store_bytes = g.store_bytes;
  h->part_bytes = g.part_bytes;
  h->base = static_cast<uint8_t*>(dev_buf);
  h->meta0 = h->base;
  h->store0 = h->base + g.meta_stride * cfg->num_layers;
  uint8_t* part = h->store0 + 2 * g.store_bytes * cfg->num_layers;
  const size_t rows_h = static_cast<size_t>(cfg->P) * cfg->heads;
  h->part_o = reinterpret_cast<float*>(part);
  h->part_ml = reinterpret_cast<float*>(part + round256(static_cast<size_t>(cfg->max_splits) * rows_h *
                                                        cfg->head_dim * 4));
  h->n_frames.assign(cfg->num_layers, 0);
  if (cfg->dtype == SWA_BF16) {
    h->tm_k.resize(cfg->num_layers);
    h->tm_v.resize(cfg->num_layers);
    for (int l = 0; l < cfg->num_layers; ++l) {
      if (!make_map(&h->tm_k[l], layer_k(h, l), cfg->head_dim, cfg->heads, h->total_rows, 1) ||
          !make_map(&h->tm_v[l], layer_v(h, l), cfg->head_dim, cfg->heads, h->total_rows, 1)) {
        delete h;
        return SWA_ERR_CUDA;
      }
    }
  }
  const swa_status s = swa_stream_reset(h, stream);
  if (s != SWA_OK) {
    delete h;
    return s;
  }
  *out = h;
  return SWA_OK;
}

extern "C" void swa_stream_destroy(swa_stream* h) { delete h; }

extern "C" swa_status swa_stream_reset(swa_stream* h, void* stream) {
  if (!h) return SWA_ERR_ARG;
  int* err = nullptr;
  if (const swa_status ds = device_ready(&err)) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // metadata: all -1 (empty slots, no eviction); counters rewritten per append
  cudaError_t e = cudaMemsetAsync(h->meta0, 0xff, h->meta_stride * h->cfg.num_layers, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(h->store0, 0, 2 * h->store_bytes * h->cfg.num_layers, st);
  if (e != cudaSuccess) return SWA_ERR_CUDA;
  for (int l = 0; l < h->cfg.num_layers; ++l) {
    // header counters start at zero (frames, evicted, specials) and -1 (last evicted)
    const int hdr[8] = {0, 0, 0, -1, 0, 0, 0, 0};
    e = cudaMemcpyAsync(layer_meta(h, l), hdr, sizeof(hdr), cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return SWA_ERR_CUDA;
  }
  // the header copies come from the stack: finish them before returning
  if (cudaStreamSynchronize(st) != cudaSuccess) return SWA_ERR_CUDA;
  std::fill(h->n_frames.begin(), h->n_frames.end(), 0);
  return SWA_OK;
}

namespace {
AppendParams append_params(swa_stream* h, int global_idx, int frame_idx, const void* k_frame,
                           const void* v_frame, int* err) {
  AppendParams p{};
  p.k_src = static_cast<const uint8_t*>(k_frame);
  p.v_src = static_cast<const uint8_t*>(v_frame);
  p.k_store = layer_k(h, global_idx);
  p.v_store = layer_v(h, global_idx);
  p.meta = layer_meta(h, global_idx);
  p.err = err;
  p.frame = frame_idx;
  p.P = h->cfg.P;
  p.S = h->cfg.scale_frames;
  p.Wc = h->cfg.window_frames;
  p.ppf = h->ppf;
  p.page_tokens = h->cfg.page_tokens;
  p.n_slots = h->n_slots;
  p.num_special = h->cfg.num_special;
  p.cross_special = h->cfg.cross_frame_special ? 1 : 0;
  p.row_bytes = h->row_bytes;
  p.off_slot_frame = 8;
  p.off_page_table = 8 + h->n_slots;
  p.off_seg_row = p.off_page_table + h->max_pages;
  p.off_seg_len = p.off_seg_row + h->max_segs;
  p.max_pages = h->max_pages;
  p.max_segs = h->max_segs;
  p.copy = 1;
  p.src_row_bytes = h->row_bytes;
  p.src_off = 0;
  return p;
}
}  // namespace

namespace {
// Append from k_frame / v_frame whose token rows are row_stride elements apart,
// the cached heads starting at head ``head0`` of each row.
swa_status stream_append_impl(swa_stream* h, int global_idx, int frame_idx, const void* k_frame, const void* v_frame,
                              int64_t row_stride, int head0, void* stream) {
  swa_status s = stream_check_layer(h, global_idx);
  if (s != SWA_OK) return s;
  if (!k_frame || !v_frame || !aligned16(k_frame) || !aligned16(v_frame)) return SWA_ERR_ARG;
  const int esize = h->cfg.dtype == SWA_F32 ? 4 : 2;
  if (head0 < 0 || row_stride < static_cast<int64_t>(head0 + h->cfg.heads) * h->cfg.head_dim) return SWA_ERR_SHAPE;
  if ((row_stride * esize) % 16 != 0 || (static_cast<int64_t>(head0) * h->cfg.head_dim * esize) % 16 != 0)
    return SWA_ERR_ARG;
  if (frame_idx != h->n_frames[global_idx]) return SWA_ERR_ORDER;
  if (frame_idx >= h->cfg.max_frames) return SWA_ERR_CAPACITY;
  int* err = nullptr;
  if (const swa_status ds = device_ready(&err)) return ds;
  AppendParams p = append_params(h, global_idx, frame_idx, k_frame, v_frame, err);
  p.src_row_bytes = row_stride * esize;
  p.src_off = static_cast<int64_t>(head0) * h->cfg.head_dim * esize;
  const cudaError_t e = launch_append_evict(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return SWA_ERR_CUDA;
  h->n_frames[global_idx] = frame_idx + 1;
  return SWA_OK;
}
}  // namespace

extern "C" swa_status swa_stream_append_evict(swa_stream* h, int global_idx, int frame_idx, const void* k_frame,
                                              const void* v_frame, void* stream) {
  if (!h) return SWA_ERR_ARG;
  return stream_append_impl(h, global_idx, frame_idx, k_frame, v_frame,
                            static_cast<int64_t>(h->cfg.heads) * h->cfg.head_dim, 0, stream);
}

extern "C" swa_status swa_stream_append_evict_heads(swa_stream* h, int global_idx, int frame_idx,
                                                    const void* k_frame, const void* v_frame, int row_stride,
                                                    int head0, void* stream) {
  if (!h) return SWA_ERR_ARG;
  return stream_append_impl(h, global_idx, frame_idx, k_frame, v_frame, row_stride, head0, stream);
}

// ================================================================ attn_pre prologue
namespace {
bool pre_shape_ok(int P, int C, int heads) {
  if (P < 0 || heads < 1 || C < 1 || C % heads) return false;
  const int D = C / heads;
  return (D == 64 || D == 128) && C % 256 == 0 && C <= 2048;  // C % 128: whole feature tiles
}

// The 3-D RoPE the prologue generates itself (null rot): frame index, special
// tokens at (t, 0, 0), patch-grid width and frequency base.
struct RopeGen {
  int frame, special, grid_w;
  double theta;
};

bool rope_gen_ok(const RopeGen& g, int P) {
  return g.frame >= 0 && g.special >= 0 && g.special <= P && g.grid_w >= 1 && g.theta > 1.0;
}

swa_status run_attn_pre(const void* x, const float* ln_w, const float* ln_b, const void* w_qkv,
                        const float* b_qkv, const float* qn_w, const float* qn_b, const float* kn_w,
                        const float* kn_b, const float* rot, int P, int C, int heads, float eps, void* xn_ws,
                        void* q_out, uint8_t* k_dst, uint8_t* v_dst, cudaStream_t st,
                        const RopeGen* gen = nullptr) {
  int* err = nullptr;
  if (const swa_status ds = device_ready(&err)) return ds;
  if (launch_ln_rows(x, ln_w, ln_b, xn_ws, P, C, eps, st) != cudaSuccess) return SWA_ERR_CUDA;
  PreParams p;
  std::memset(&p, 0, sizeof(p));
  if (!encode_2d_sw128(&p.tm_a, xn_ws, C, P, 128) || !encode_2d_sw128(&p.tm_b, w_qkv, C, 3LL * C, 128))
    return SWA_ERR_CUDA;
  p.b_qkv = b_qkv;
  p.qn_w = qn_w;
  p.qn_b = qn_b;
  p.kn_w = kn_w;
  p.kn_b = kn_b;
  p.rot = rot;
  p.q_out = q_out;
  p.k_dst = k_dst;
  p.v_dst = v_dst;
  p.kv_row_bytes = static_cast<int64_t>(C) * 2;
  p.err = err;
  p.P = P;
  p.C = C;
  p.H = heads;
  p.D = C / heads;
  p.eps = eps;
  if (!rot) {
    // bands t | h | w of (D/2 - 2*(D/6), D/6, D/6) pairs; pair j of a band of n
    // pairs turns by pos * theta^(-j/n) (the same rule as swa_rope3d_table)
    const int half = p.D / 2, n_h = p.D / 6, n_t = half - 2 * n_h;
    p.rope_frame = gen->frame;
    p.rope_special = gen->special;
    p.rope_grid_w = gen->grid_w;
    p.rope_nt = n_t;
    p.rope_nh = n_h;
    const double lt = std::log(gen->theta);
    for (int j = 0; j < half; ++j) {
      const int jj = j < n_t ? j : (j < n_t + n_h ? j - n_t : j - n_t - n_h);
      const int n = j < n_t ? n_t : (j < n_t + n_h ? n_h : half - n_t - n_h);
      p.rope_inv_freq[j] = std::exp(-lt * jj / n);
    }
  }
  return cuda_status(launch_qkv_pre(p, st));
}
}  // namespace

extern "C" swa_status swa_attn_pre(const void* x, const float* ln_w, const float* ln_b, const void* w_qkv,
                                   const float* b_qkv, const float* qn_w, const float* qn_b, const float* kn_w,
                                   const float* kn_b, const float* rot, int P, int C, int heads, float eps,
                                   void* xn_ws, void* q_out, void* k_out, void* v_out, void* stream) {
  if (!pre_shape_ok(P, C, heads)) return (P < 0 || heads < 1 || C < 1) ? SWA_ERR_ARG : SWA_ERR_UNSUPPORTED;
  if (!(eps > 0.f)) return SWA_ERR_ARG;
  if (P == 0) return SWA_OK;
  const void* ptrs[] = {x, ln_w, ln_b, w_qkv, b_qkv, qn_w, qn_b, kn_w, kn_b, rot, xn_ws, q_out, k_out, v_out};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return SWA_ERR_ARG;
  return run_attn_pre(x, ln_w, ln_b, w_qkv, b_qkv, qn_w, qn_b, kn_w, kn_b, rot, P, C, heads, eps, xn_ws, q_out,
                      static_cast<uint8_t*>(k_out), static_cast<uint8_t*>(v_out), static_cast<cudaStream_t>(stream));
}

extern "C" swa_status swa_attn_pre_rope3d(const void* x, const float* ln_w, const float* ln_b, const void* w_qkv,
                                          const float* b_qkv, const float* qn_w, const float* qn_b,
                                          const float* kn_w, const float* kn_b, int frame_idx, int num_special,
                                          int grid_w, double theta, int P, int C, int heads, float eps,
                                          void* xn_ws, void* q_out, void* k_out, void* v_out, void* stream) {
  if (!pre_shape_ok(P, C, heads)) return (P < 0 || heads < 1 || C < 1) ? SWA_ERR_ARG : SWA_ERR_UNSUPPORTED;
  if (!(eps > 0.f)) return SWA_ERR_ARG;
  const RopeGen gen{frame_idx, num_special, grid_w, theta};
  if (!rope_gen_ok(gen, P)) return SWA_ERR_ARG;
  if (P == 0) return SWA_OK;
  const void* ptrs[] = {x, ln_w, ln_b, w_qkv, b_qkv, qn_w, qn_b, kn_w, kn_b, xn_ws, q_out, k_out, v_out};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return SWA_ERR_ARG;
  return run_attn_pre(x, ln_w, ln_b, w_qkv, b_qkv, qn_w, qn_b, kn_w, kn_b, nullptr, P, C, heads, eps, xn_ws, q_out,
                      static_cast<uint8_t*>(k_out), static_cast<uint8_t*>(v_out), static_cast<cudaStream_t>(stream),
                      &gen);
}

extern "C" swa_status swa_rope3d_table(int frame_idx, int P, int num_special, int grid_w, int head_dim,
                                       double theta, float* rot_out, void* stream) {
  if (frame_idx < 0 || P < 0 || num_special < 0 || num_special > P || grid_w < 1 || head_dim < 6 ||
      head_dim % 2 || !(theta > 1.0))
    return SWA_ERR_ARG;
  if (P == 0) return SWA_OK;
  if (!rot_out || !aligned16(rot_out)) return SWA_ERR_ARG;
  int* err = nullptr;
  if (const swa_status ds = device_ready(&err)) return ds;
  return cuda_status(launch_rope3d_table(rot_out, frame_idx, P, num_special, grid_w, head_dim, theta,
                                         static_cast<cudaStream_t>(stream)));
}

namespace {
swa_status stream_append_pre_impl(swa_stream* h, int global_idx, int frame_idx, const void* x, const float* ln_w,
                                  const float* ln_b, const void* w_qkv, const float* b_qkv, const float* qn_w,
                                  const float* qn_b, const float* kn_w, const float* kn_b, const float* rot,
                                  float eps, void* xn_ws, void* q_out, void* stream, const RopeGen* gen) {
  swa_status s = stream_check_layer(h, global_idx);
  if (s != SWA_OK) return s;
  const swa_stream_cfg& c = h->cfg;
  if (c.dtype != SWA_BF16) return SWA_ERR_UNSUPPORTED;
  const int C = c.heads * c.head_dim;
  if (!pre_shape_ok(c.P, C, c.heads)) return SWA_ERR_UNSUPPORTED;
  if (!(eps > 0.f)) return SWA_ERR_ARG;
  if (gen && !rope_gen_ok(*gen, c.P)) return SWA_ERR_ARG;
  const void* ptrs[] = {x, ln_w, ln_b, w_qkv, b_qkv, qn_w, qn_b, kn_w, kn_b, xn_ws, q_out};
  for (const void* q : ptrs)
    if (!q || !aligned16(q)) return SWA_ERR_ARG;
  if (!gen && (!rot || !aligned16(rot))) return SWA_ERR_ARG;
  if (frame_idx != h->n_frames[global_idx]) return SWA_ERR_ORDER;
  if (frame_idx >= c.max_frames) return SWA_ERR_CAPACITY;
  int* err = nullptr;
  if (const swa_status ds = device_ready(&err)) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // eviction (the evicted frame's specials leave its slot first) and metadata,
  // then the prologue writes the frame's K/V into that slot
  AppendParams ap = append_params(h, global_idx, frame_idx, nullptr, nullptr, err);
  ap.copy = 0;
  if (launch_append_evict(ap, st) != cudaSuccess) return SWA_ERR_CUDA;
  h->n_frames[global_idx] = frame_idx + 1;
  const int64_t slot_row0 = static_cast<int64_t>(stream_slot(frame_idx, c.scale_frames, c.window_frames)) *
                            h->ppf * c.page_tokens;
  uint8_t* kd = layer_k(h, global_idx) + slot_row0 * h->row_bytes;
  uint8_t* vd = layer_v(h, global_idx) + slot_row0 * h->row_bytes;
  return run_attn_pre(x, ln_w, ln_b, w_qkv, b_qkv, qn_w, qn_b, kn_w, kn_b, gen ? nullptr : rot, c.P, C, c.heads,
                      eps, xn_ws, q_out, kd, vd, st, gen);
}
}  // namespace

extern "C" swa_status swa_stream_append_evict_pre(swa_stream* h, int global_idx, int frame_idx, const void* x,
                                                  const float* ln_w, const float* ln_b, const void* w_qkv,
                                                  const float* b_qkv, const float* qn_w, const float* qn_b,
                                                  const float* kn_w, const float* kn_b, const float* rot, float eps,
                                                  void* xn_ws, void* q_out, void* stream) {
  return stream_append_pre_impl(h, global_idx, frame_idx, x, ln_w, ln_b, w_qkv, b_qkv, qn_w, qn_b, kn_w, kn_b, rot,
                                eps, xn_ws, q_out, stream, nullptr);
}

extern "C" swa_status swa_stream_append_evict_pre_rope3d(swa_stream* h, int global_idx, int frame_idx,
                                                         const void* x, const float* ln_w, const float* ln_b,
                                                         const void* w_qkv, const float* b_qkv, const float* qn_w,
                                                         const float* qn_b, const float* kn_w, const float* kn_b,
                                                         int num_special, int grid_w, double theta, float eps,
                                                         void* xn_ws, void* q_out, void* stream) {
  const RopeGen gen{frame_idx, num_special, grid_w, theta};
  return stream_append_pre_impl(h, global_idx, frame_idx, x, ln_w, ln_b, w_qkv, b_qkv, qn_w, qn_b, kn_w, kn_b,
                                nullptr, eps, xn_ws, q_out, stream, &gen);
}

namespace {

// split count for the streaming attend, in units of one pair's key tile: each
// wave of CTAs costs its key tiles plus about 8 tiles of start-up and epilogue
// (measured on B200 at 8 scale + 64 window frames of 1004 tokens: 443, 420 and
// 460 us for 4, 9 and 16 splits fit 1.45 us per tile and 12.5 us per wave), and
// every split adds a little to the combine
int choose_splits(int T, int items_per_split, int max_splits, int sms) {
  int best = 1;
  double best_cost = 1e300;
  for (int k = 1; k <= max_splits && k <= T; ++k) {
    const int64_t ctas = static_cast<int64_t>(items_per_split) * k;
    const int64_t waves = (ctas + sms - 1) / sms;
    const double cost = static_cast<double>(waves) * (cdiv(T, k) + 8) + (k > 1 ? 0.25 * k : 0.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = k;
    }
  }
  return best;
}

}  // namespace

namespace {
// The attend of a frame's queries against key runs listed in device metadata:
// hdr (n_segs at hdr[5]), run rows and lengths, at most max_segs runs, which
// cover n_frames_keys full frames plus n_special special tokens.
// q_frame and out: token rows q_ld elements apart, the layer's heads starting at
// head q_h0 of each row (q_ld 0: the contiguous [P, heads, head_dim] frame).
swa_status stream_attend_impl(swa_stream* h, int global_idx, const void* q_frame, void* out, cudaStream_t st,
                              const int* hdr, const int* seg_row, const int* seg_len, int max_segs,
                              int n_frames_keys, int n_special, int64_t q_ld = 0, int q_h0 = 0) {
  int* err = nullptr;
  if (const swa_status ds = device_ready(&err)) return ds;
  const swa_stream_cfg& c = h->cfg;
  if (c.dtype == SWA_F32) {
    SimtParams p{};
    p.q = static_cast<const float*>(q_frame);
    p.k = reinterpret_cast<const float*>(layer_k(h, global_idx));
    p.v = reinterpret_cast<const float*>(layer_v(h, global_idx));
    p.out = static_cast<float*>(out);
    p.seg_row = seg_row;
    p.seg_len = seg_len;
    p.meta_hdr = hdr;
    p.err = err;
    p.mode = SIMT_STREAM;
    p.B = 1;
    p.Nq = c.P;
    p.Nk = static_cast<int>(h->total_rows);
    p.Hq = c.heads;
    p.Hkv = c.heads;
    p.D = c.head_dim;
    p.max_segs = max_segs;
    p.scale = 1.f / std::sqrt(static_cast<float>(c.head_dim));
    p.q_ld = q_ld;
    p.q_h0 = q_h0;
    return cuda_status(launch_attn_simt(p, st));
  }
  const int T = n_frames_keys * cdiv(c.P, kTileRows) + cdiv(n_special, kTileRows);
  const int n_pairs = qpairs_per_frame(c.P);
  const int items = c.heads * n_pairs;
  const int splits = choose_splits(T, items, c.max_splits, num_sms());
  TcParams p;
  std::memset(&p, 0, sizeof(p));
  if (!make_map(&p.tm_q, static_cast<const uint8_t*>(q_frame) + static_cast<size_t>(q_h0) * c.head_dim * 2,
                c.head_dim, c.heads, c.P, 1, q_ld))
    return SWA_ERR_CUDA;
  p.out_ld = q_ld;
  p.out_h0 = q_h0;
  p.tm_k = h->tm_k[global_idx];
  p.tm_v = h->tm_v[global_idx];
  p.out = out;
  p.part_o = h->part_o;
  p.part_ml = h->part_ml;
  p.seg_row = seg_row;
  p.seg_len = seg_len;
  p.meta_hdr = hdr;
  p.err = err;
  p.mode = TC_STREAM;
  p.B = 1;
  p.Nq = c.P;
  p.Hq = c.heads;
  p.Hkv = c.heads;
  p.P = c.P;
  p.n_pairs = n_pairs;
  p.splits = splits;
  p.max_segs = max_segs;
  p.scale_log2 = scale_log2(c.head_dim);
  cudaError_t e = launch_attn_tc(p, c.head_dim, static_cast<int64_t>(items) * splits, st);
  if (e != cudaSuccess) return SWA_ERR_CUDA;
  if (splits == 1) return SWA_OK;  // every item wrote its rows of out itself
  // the combine merges the splits, launched behind the attend so that its CTAs are
  // resident and waiting when the attend's last wave ends
  const int64_t out_ld = q_ld ? q_ld : static_cast<int64_t>(c.heads) * c.head_dim;
  return cuda_status(launch_combine(h->part_o, h->part_ml, out, c.P, c.heads, splits, c.head_dim, out_ld, q_h0, st));
}
}  // namespace

namespace {
swa_status stream_attend_heads_impl(swa_stream* h, int global_idx, int frame_idx, const void* q_frame, void* out,
                                    int64_t row_stride, int head0, void* stream) {
  swa_status s = stream_check_layer(h, global_idx);
  if (s != SWA_OK) return s;
  if (!q_frame || !out || !aligned16(q_frame) || !aligned16(out)) return SWA_ERR_ARG;
  const swa_stream_cfg& c = h->cfg;
  const int esize = c.dtype == SWA_F32 ? 4 : 2;
  if (head0 < 0 || row_stride < static_cast<int64_t>(head0 + c.heads) * c.head_dim) return SWA_ERR_SHAPE;
  if ((row_stride * esize) % 16 != 0 || (static_cast<int64_t>(head0) * c.head_dim * esize) % 16 != 0)
    return SWA_ERR_ARG;
  if (h->n_frames[global_idx] == 0 || frame_idx != h->n_frames[global_idx] - 1) return SWA_ERR_ORDER;
  int* meta = layer_meta(h, global_idx);
  const int off_seg_row = 8 + h->n_slots + h->max_pages;
  const int off_seg_len = off_seg_row + h->max_segs;
  const int i = frame_idx;
  const int n_ret = stream_retained(i, c.scale_frames, c.window_frames);
  const int n_special =
      c.cross_frame_special ? stream_n_evicted(i, c.scale_frames, c.window_frames) * c.num_special : 0;
  return stream_attend_impl(h, global_idx, q_frame, out, static_cast<cudaStream_t>(stream), meta,
                            meta + off_seg_row, meta + off_seg_len, h->max_segs, n_ret, n_special, row_stride, head0);
}
}  // namespace

extern "C" swa_status swa_stream_attend(swa_stream* h, int global_idx, int frame_idx, const void* q_frame,
                                        void* out, void* stream) {
  if (!h) return SWA_ERR_ARG;
  return stream_attend_heads_impl(h, global_idx, frame_idx, q_frame, out,
                                  static_cast<int64_t>(h->cfg.heads) * h->cfg.head_dim, 0, stream);
}

extern "C" swa_status swa_stream_attend_heads(swa_stream* h, int global_idx, int frame_idx, const void* q_frame,
                                              void* out, int row_stride, int head0, void* stream) {
  if (!h) return SWA_ERR_ARG;
  return stream_attend_heads_impl(h, global_idx, frame_idx, q_frame, out, row_stride, head0, stream);
}

extern "C" swa_status swa_stream_attend_transient(swa_stream* h, int global_idx, const void* q_frame,
                                                  const void* k_frame, const void* v_frame, void* out,
                                                  void* stream) {
  swa_status s = stream_check_layer(h, global_idx);
  if (s != SWA_OK) return s;
  if (!q_frame || !k_frame || !v_frame || !out || !aligned16(q_frame) || !aligned16(k_frame) ||
      !aligned16(v_frame) || !aligned16(out))
    return SWA_ERR_ARG;
  int* err = nullptr;
  if (const swa_status ds = device_ready(&err)) return ds;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const swa_stream_cfg& c = h->cfg;
  int* meta = layer_meta(h, global_idx);
  TransientParams tp{};
  tp.k_src = static_cast<const uint8_t*>(k_frame);
  tp.v_src = static_cast<const uint8_t*>(v_frame);
  tp.k_store = layer_k(h, global_idx);
  tp.v_store = layer_v(h, global_idx);
  tp.meta = meta;
  tp.err = err;
  tp.P = c.P;
  tp.row_bytes = c.heads * c.head_dim * (c.dtype == SWA_F32 ? 4 : 2);
  tp.page_tokens = c.page_tokens;
  tp.scratch_page = h->scratch_page;
  tp.off_seg_row = 8 + h->n_slots + h->max_pages;
  tp.off_seg_len = tp.off_seg_row + h->max_segs;
  tp.max_segs = h->max_segs;
  tp.t_off = h->t_off;
  if (launch_transient_prepare(tp, st) != cudaSuccess) return SWA_ERR_CUDA;
  // keys: the frames and specials the cache holds after its last keyframe, plus this frame
  const int nf = h->n_frames[global_idx];
  const int n_ret = nf > 0 ? stream_retained(nf - 1, c.scale_frames, c.window_frames) : 0;
  const int n_special = (nf > 0 && c.cross_frame_special)
                            ? stream_n_evicted(nf - 1, c.scale_frames, c.window_frames) * c.num_special
                            : 0;
  int* th = meta + h->t_off;
  return stream_attend_impl(h, global_idx, q_frame, out, st, th, th + 8, th + 8 + (h->max_segs + 1),
                            h->max_segs + 1, n_ret + 1, n_special);
}

extern "C" swa_status swa_stream_meta_layout(const swa_stream* h, swa_meta_layout* out) {
  if (!h || !out) return SWA_ERR_ARG;
  out->n_ints = h->meta_ints;
  out->n_slots = h->n_slots;
  out->pages_per_frame = h->ppf;
  out->max_pages = h->max_pages;
  out->max_segs = h->max_segs;
  out->off_slot_frame = 8;
  out->off_page_table = 8 + h->n_slots;
  out->off_seg_row = out->off_page_table + h->max_pages;
  out->off_seg_len = out->off_seg_row + h->max_segs;
  return SWA_OK;
}

extern "C" swa_status swa_stream_get_meta_raw(const swa_stream* h, int global_idx, int32_t* dst, size_t n_ints,
                                              void* stream) {
  swa_status s = stream_check_layer(h, global_idx);
  if (s != SWA_OK) return s;
  if (!dst) return SWA_ERR_ARG;
  if (n_ints < static_cast<size_t>(h->meta_ints)) return SWA_ERR_CAPACITY;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(dst, layer_meta(h, global_idx), static_cast<size_t>(h->meta_ints) * 4,
                                  cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  return cuda_status(e);
}

extern "C" swa_status swa_stream_get_meta(const swa_stream* h, int global_idx, swa_meta_host* m, void* stream) {
  swa_status s = stream_check_layer(h, global_idx);
  if (s != SWA_OK) return s;
  if (!m) return SWA_ERR_ARG;
  std::vector<int32_t> raw(static_cast<size_t>(h->meta_ints));
  s = swa_stream_get_meta_raw(h, global_idx, raw.data(), raw.size(), stream);
  if (s != SWA_OK) return s;
  const int off_slot = 8, off_page = 8 + h->n_slots, off_row = off_page + h->max_pages,
            off_len = off_row + h->max_segs;
  m->n_frames = raw[0];
  m->n_evicted = raw[1];
  m->n_special_tokens = raw[2];
  m->last_evicted = raw[3];
  m->n_last_evicted = raw[3] >= 0 ? 1 : 0;
  m->n_pages = raw[4];
  m->n_segs = raw[5];
  m->n_retained = raw[6];
  m->n_slots = h->n_slots;
  if (m->n_pages < 0 || m->n_pages > h->max_pages || m->n_segs < 0 || m->n_segs > h->max_segs)
    return SWA_ERR_CUDA;  // the device metadata is not a state the append kernel writes
  if ((m->slot_frame && m->slot_cap < m->n_slots) || (m->page_table && m->page_cap < m->n_pages) ||
      ((m->seg_row || m->seg_len) && m->seg_cap < m->n_segs))
    return SWA_ERR_CAPACITY;
  if (m->slot_frame) std::memcpy(m->slot_frame, raw.data() + off_slot, sizeof(int32_t) * m->n_slots);
  if (m->page_table) std::memcpy(m->page_table, raw.data() + off_page, sizeof(int32_t) * m->n_pages);
  if (m->seg_row) std::memcpy(m->seg_row, raw.data() + off_row, sizeof(int32_t) * m->n_segs);
  if (m->seg_len) std::memcpy(m->seg_len, raw.data() + off_len, sizeof(int32_t) * m->n_segs);
  return SWA_OK;
}

extern "C" void* swa_stream_k_storage(const swa_stream* h, int global_idx) {
  if (stream_check_layer(h, global_idx) != SWA_OK) return nullptr;
  return layer_k(h, global_idx);
}

extern "C" void* swa_stream_v_storage(const swa_stream* h, int global_idx) {
  if (stream_check_layer(h, global_idx) != SWA_OK) return nullptr;
  return layer_v(h, global_idx);
}

// ============================================================ device errors
extern "C" swa_status swa_device_error_check(void* stream) {
  int* err = err_ptr();
  if (!err) return SWA_ERR_CUDA;
  const int d = current_device();
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, err, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return SWA_ERR_CUDA;
  // the stream is idle: the host mirror holds everything its kernels latched
  if (d >= 0 && *host_err_word(d) != 0) v = 1;
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyAsync(err, &zero, sizeof(int), cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (d >= 0) *host_err_word(d) = 0;
    return SWA_ERR_TIMEOUT;
  }
  return SWA_OK;
}

extern "C" swa_status swa_debug_wait_timeout(int timeout_us, void* stream) {
  if (timeout_us < 1 || timeout_us > 10000000) return SWA_ERR_ARG;
  int* err = nullptr;
  if (const swa_status ds = device_ready(&err)) return ds;
  return cuda_status(launch_debug_wait(err, static_cast<long long>(timeout_us) * 1000, static_cast<cudaStream_t>(stream)));
}

extern "C" swa_status swa_debug_exp2_poly(const float* x, float* y, int n, void* stream) {
  if (n < 0) return SWA_ERR_ARG;
  if (n == 0) return SWA_OK;
  if (!x || !y) return SWA_ERR_ARG;
  int* err = nullptr;
  if (const swa_status ds = device_ready(&err)) return ds;
  return cuda_status(launch_exp2_poly(x, y, n, static_cast<cudaStream_t>(stream)));
}
