// Decode without a caller-provided workspace.
//
// hd_attn_decode needs device scratch for its split-KV partial results and
// takes it from the caller.  Some callers cannot hand over device memory:
// code that runs where a cudaMalloc is not allowed or not wanted (inside a
// framework's memory pool that owns every allocation, in a latency-critical
// serving loop that must never hit the allocator, or in a host integration
// that has no allocator of its own).  For them, hd_attn_decode_noalloc uses a
// fixed scratch area that lives in this library's own device memory instead.
//
// The scratch is one file-scope device array of HD_DECODE_NOALLOC_SCRATCH_BYTES
// (every GPU that loads the library keeps it until the process exits).  Its
// device address is looked up once per device with cudaGetSymbolAddress, with
// that device current, the first time the entry point runs on it; that first
// call should therefore be made before any stream capture begins.  The address
// is kept for the life of the process, which assumes the device keeps one
// primary context throughout (a cudaDeviceReset between calls would leave the
// kept address stale).  Every call
// shares the one array: two calls whose kernels overlap on the GPU (different
// streams, no ordering between them) race on it.  Nothing in it needs to start
// at zero: each call writes every partial it later reads.
#include <mutex>

#include "hd_common.cuh"
#include "hd_launch.h"

namespace hd {

static __device__ __align__(256) uint8_t g_decode_scratch[HD_DECODE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on first
// use per device).  Returns nullptr and sets *err when the lookup fails.
void* scratch_for_current_device(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    *err = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

int sm_count();  // capi.cu

}  // namespace hd

using namespace hd;

extern "C" hd_status hd_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                            const int32_t* ctx_len, void* o, float* lse, int B, int n, int Lmax,
                                            int Hq, int Hkv, int D, hd_mode mode, int window, float scale,
                                            hd_dtype in_dt, hd_dtype out_dt, int32_t* dev_status, void* stream) {
  // Same argument rules as hd_attn_decode.
  if (B < 0 || n < 1 || Lmax < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || window < 0) return HD_ERR_INVALID_ARG;
  if (mode != HD_INTRA && mode != HD_CROSS) return HD_ERR_INVALID_ARG;
  if ((in_dt != HD_F32 && in_dt != HD_BF16) || (out_dt != HD_F32 && out_dt != HD_BF16) || !(scale > 0.f) ||
      scale == INFINITY)
    return HD_ERR_INVALID_ARG;
  if (D != 128 || in_dt != HD_BF16) return HD_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(n) * Lmax > (1ll << 30)) return HD_ERR_INVALID_ARG;
  if (B == 0) return HD_OK;
  if (!q || !k_cache || !v_cache || !ctx_len || !o) return HD_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) || !aligned(ctx_len, 4))
    return HD_ERR_INVALID_ARG;
  if (lse && !aligned(lse, 4)) return HD_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return HD_ERR_CUDA;
  const DecPlan pl = decode_plan(B, n, Lmax, Hq, Hkv, mode == HD_CROSS, sms);
  if (pl.units > 65535) return HD_ERR_UNSUPPORTED;
  // Sizes whose partial results do not fit the fixed scratch are refused.
  if (decode_workspace_bytes(pl) > static_cast<size_t>(HD_DECODE_NOALLOC_SCRATCH_BYTES)) return HD_ERR_UNSUPPORTED;
  cudaError_t err = cudaSuccess;
  void* ws = scratch_for_current_device(&err);
  if (!ws) return HD_ERR_CUDA;
  err = launch_decode(q, k_cache, v_cache, ctx_len, o, lse, B, n, Lmax, Hq, Hkv, window, scale, mode == HD_CROSS,
                      out_dt == HD_BF16, ws, dev_status, sms, static_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? HD_OK : HD_ERR_CUDA;
}
