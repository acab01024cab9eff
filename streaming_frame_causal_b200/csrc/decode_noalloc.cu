// decode_noalloc.cu -- the rolling GQA decode for callers that cannot allocate
// device memory.
//
// swa_decode needs a scratch workspace for its split-K partials, which the caller
// allocates.  Some callers cannot make that allocation: a process whose device
// memory is entirely reserved up front by another allocator (so a raw cudaMalloc
// would fail or fragment the pool), a host program that forbids allocation calls
// once it is running (cudaMalloc may synchronize the device and take unbounded
// time), or a plugin interface that hands the code its inputs and outputs but no
// way to obtain memory.  swa_decode_noalloc serves them: it runs the same decode
// kernels, with the scratch taken from a fixed array compiled into this library.
//
// The array is a file-scope __device__ variable of SWA_DECODE_NOALLOC_SCRATCH_BYTES
// (16 MiB).  Every GPU that loads the library holds it until the process exits.
// Host code cannot use the array's name as a device address, so the first call on
// each device (with that device current) looks the address up with
// cudaGetSymbolAddress and caches it; make that first call before any stream
// capture.  All calls on a device share the one array: calls that overlap on the
// GPU (different streams, or different host threads) race on it and must be
// serialized by the caller.  The decode kernel writes every partial it later reads,
// so nothing left over from an earlier call needs clearing.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/swa.h"
#include "internal.h"
#include "tile_sched.h"

namespace {

constexpr size_t kScratchBytes = SWA_DECODE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDev = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDev] = {nullptr};

// Device address of the scratch array on the current device (looked up once per
// device); nullptr if the lookup fails.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&ptr), g_decode_scratch) != cudaSuccess || !ptr)
      return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" swa_status swa_decode_noalloc(const void* q, const void* k_new, const void* v_new, void* k_cache,
                                         void* v_cache, long long pos, int W, int B, int Hq, int Hkv,
                                         int head_dim, void* out, int dtype, void* stream) {
  if (pos < 0 || W < 1 || B < 0 || Hq < 1 || Hkv < 1 || head_dim < 1) return SWA_ERR_ARG;
  if (dtype != SWA_F32 && dtype != SWA_BF16) return SWA_ERR_ARG;
  if (Hq % Hkv) return SWA_ERR_SHAPE;
  // only the bf16 decode uses scratch memory; the f32 decode needs none (use swa_decode)
  if (dtype != SWA_BF16 || (head_dim != 64 && head_dim != 128)) return SWA_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (G < 1 || G > 8) return SWA_ERR_UNSUPPORTED;
  if (B == 0) return SWA_OK;
  // reject requests whose partials do not fit the fixed array
  const size_t need = swa::decode_workspace_bytes(B, Hq, Hkv, head_dim, W);
  if (need > kScratchBytes) return SWA_ERR_CAPACITY;
  if (!q || !k_new || !v_new || !k_cache || !v_cache || !out) return SWA_ERR_ARG;
  if (!al16(q) || !al16(k_new) || !al16(v_new) || !al16(k_cache) || !al16(v_cache) || !al16(out))
    return SWA_ERR_ARG;
  int* err = nullptr;
  if (const int ds = swa::device_ready_status(&err)) return static_cast<swa_status>(ds);
  void* scratch = scratch_on_current_device();
  if (!scratch) return SWA_ERR_CUDA;

  swa::DecodeParams p{};
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
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(head_dim)));
  p.chunks = swa::decode_chunks(B, Hkv, W);
  const size_t n_part = static_cast<size_t>(B) * Hkv * p.chunks * G;
  p.part_o = static_cast<float*>(scratch);
  p.part_ml = p.part_o + n_part * head_dim;
  return swa::launch_decode_bf16(p, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SWA_OK : SWA_ERR_CUDA;
}
