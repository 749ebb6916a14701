// Multi-stream expansion and final-stream gather: pure HBM streams.
//
// expand ("Hidden Decoding at Scale", "Multi-Stream Expansion and Training
// Objective", eq. S_t = E_k(x_i)):  out[b, i*n + s, :] = tables[s, ids[b,i], :]
// gather (same section; only the final stream feeds the LM head):
//                                   out[b, i, :] = h[b, i*n + n-1, :]
//
// stream interleave (stream parallelism, "Persistent KV and the KV-mirror
// Saving": the KV is sharded across ranks by stream; a cross-stream layer
// gathers every rank's shard and restores the expanded order):
//                                   out[b, i*n + r + R*l, :] = parts[r, b, i*(n/R) + l, :]
//
// All are row copies of R = d * elem_size bytes (a multiple of 16).  One
// warp moves one row with 16-byte vector loads and stores; each lane keeps
// kUnroll loads in flight before storing, and the grid is a multiple of the
// SM count with warps striding over rows.
#include "hd_common.cuh"
#include "hd_launch.h"

namespace hd {

constexpr int kCopyThreads = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ uint4 ld_nc_v4(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Copy one row of `nvec` 16-byte vectors with one warp.
__device__ __forceinline__ void warp_copy_row(const uint4* __restrict__ src,
                                              uint4* __restrict__ dst, int nvec, int lane) {
  int v = lane;
  for (; v + 32 * (kUnroll - 1) < nvec; v += 32 * kUnroll) {
    uint4 r[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) r[u] = ld_nc_v4(src + v + 32 * u);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) dst[v + 32 * u] = r[u];
  }
  for (; v < nvec; v += 32) dst[v] = ld_nc_v4(src + v);
}

__device__ __forceinline__ void warp_zero_row(uint4* __restrict__ dst, int nvec, int lane) {
  for (int v = lane; v < nvec; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
}

// rows = B * L * n output rows, row r = (b*L + i)*n + s.
__global__ void __launch_bounds__(kCopyThreads) expand_kernel(
    const uint4* __restrict__ tables, const int32_t* __restrict__ ids, uint4* __restrict__ out,
    int64_t rows, int n, int64_t V, int nvec, int32_t* status) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kCopyThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kCopyThreads) >> 5;
  for (int64_t r = warp; r < rows; r += nwarps) {
    const int64_t tok = r / n;  // b*L + i
    const int s = static_cast<int>(r - tok * n);
    const int32_t id = __ldg(ids + tok);
    uint4* dst = out + r * nvec;
    if (id < 0 || static_cast<int64_t>(id) >= V) {
      warp_zero_row(dst, nvec, lane);
      if (lane == 0) report(status, HD_ERR_BAD_TOKEN);
      continue;
    }
    const uint4* src = tables + (static_cast<int64_t>(s) * V + id) * nvec;
    warp_copy_row(src, dst, nvec, lane);
  }
}

// rows = B * L output rows; source row = r*n + n - 1.
__global__ void __launch_bounds__(kCopyThreads) gather_kernel(
    const uint4* __restrict__ h, uint4* __restrict__ out, int64_t rows, int n, int nvec) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kCopyThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kCopyThreads) >> 5;
  for (int64_t r = warp; r < rows; r += nwarps) {
    const uint4* src = h + (r * n + (n - 1)) * nvec;
    warp_copy_row(src, out + r * nvec, nvec, lane);
  }
}

// rows = B*L*n output rows, row (b*L + i)*n + s with s = r + R*l, from rank
// part r (part_rows rows each) row (b*L + i)*(n/R) + l.
__global__ void __launch_bounds__(kCopyThreads) stream_interleave_kernel(
    const uint4* __restrict__ parts, uint4* __restrict__ out, int64_t rows, int n, int R, int64_t part_rows,
    int nvec) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kCopyThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kCopyThreads) >> 5;
  const int nl = n / R;
  for (int64_t r = warp; r < rows; r += nwarps) {
    const int64_t tok = r / n;  // b*L + i
    const int s = static_cast<int>(r - tok * n);
    const int rk = s % R, l = s / R;
    const uint4* src = parts + (static_cast<int64_t>(rk) * part_rows + tok * nl + l) * nvec;
    warp_copy_row(src, out + r * nvec, nvec, lane);
  }
}

// ------------------------------------------------------------------- host

static int copy_grid(int64_t rows, int sms) {
  const int64_t warps_per_cta = kCopyThreads / 32;
  int64_t want = (rows + warps_per_cta - 1) / warps_per_cta;
  int64_t cap = static_cast<int64_t>(sms) * 8;  // 8 CTAs (64 warps) per SM
  if (want > cap) want = cap;
  if (want < 1) want = 1;
  return static_cast<int>(want);
}

cudaError_t launch_expand(const void* tables, const int32_t* ids, void* out, int64_t rows,
                          int n, int64_t V, int row_bytes, int sms, int32_t* status,
                          cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  expand_kernel<<<copy_grid(rows, sms), kCopyThreads, 0, st>>>(
      static_cast<const uint4*>(tables), ids, static_cast<uint4*>(out), rows, n, V,
      row_bytes / 16, status);
  return cudaGetLastError();
}

cudaError_t launch_stream_interleave(const void* parts, void* out, int64_t rows, int n, int R, int row_bytes,
                                     int sms, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  stream_interleave_kernel<<<copy_grid(rows, sms), kCopyThreads, 0, st>>>(
      static_cast<const uint4*>(parts), static_cast<uint4*>(out), rows, n, R, rows / R, row_bytes / 16);
  return cudaGetLastError();
}

cudaError_t launch_gather(const void* h, void* out, int64_t rows, int n, int row_bytes, int sms,
                          cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  gather_kernel<<<copy_grid(rows, sms), kCopyThreads, 0, st>>>(
      static_cast<const uint4*>(h), static_cast<uint4*>(out), rows, n, row_bytes / 16);
  return cudaGetLastError();
}

}  // namespace hd
