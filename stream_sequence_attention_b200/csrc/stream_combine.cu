// Stream-parallel cross-stream decode: the merge of the R ranks' partial
// results for one rank's own stream queries, reading every rank's partial
// where it lies (another GPU's memory through a peer mapping, or local).
//
// ("Hidden Decoding at Scale", "Persistent KV and the KV-mirror Saving": the
// intra-stream KV is sharded across ranks by stream.)  Rank rho's partial for
// query (b, s, h) is the softmax over the visible keys of rho's cache streams,
// normalised within them, with its log-sum-exp (-inf where it saw no key).
// Rank r owns the queries of streams s = r + R*l.  For each such row
//   O = sum_rho e^(lse_rho - M) O_rho / sum_rho e^(lse_rho - M),
//   lse = M + log sum_rho e^(lse_rho - M),  M = max_rho lse_rho,
// which is the softmax over the union of the ranks' keys.  Only these rows
// are read from each rank: the exchange and the merge are one pass.
#include "hd_common.cuh"
#include "hd_launch.h"

namespace hd {

struct CombinePtrs {
  const void* o[kPeerMaxRanks];
  const float* lse[kPeerMaxRanks];
};

// One warp per local row (b, l, h) of [B, n/R, Hq].
template <bool IN_BF16>
__global__ void attn_combine_streams_kernel(const __grid_constant__ CombinePtrs cp, void* __restrict__ o,
                                            float* __restrict__ lse, int R, int B, int n, int Hq, int D, int r,
                                            int out_bf16) {
  const int nl = n / R;
  const int64_t rows = static_cast<int64_t>(B) * nl * Hq;
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int h = static_cast<int>(row % Hq);
  const int64_t bl = row / Hq;
  const int l = static_cast<int>(bl % nl);
  const int64_t b = bl / nl;
  const int64_t src = (b * n + r + static_cast<int64_t>(R) * l) * Hq + h;  // row in [B, n, Hq]
  float M = -INFINITY;
  for (int rho = 0; rho < R; ++rho) M = fmaxf(M, cp.lse[rho][src]);
  float L = 0.f;
  if (M != -INFINITY)
    for (int rho = 0; rho < R; ++rho) L += expf(cp.lse[rho][src] - M);  // exp(-inf) = 0
  const float inv = L > 0.f ? 1.f / L : 0.f;
  for (int c = lane; c < D / 4; c += 32) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
      for (int rho = 0; rho < R; ++rho) {
        const float lr = cp.lse[rho][src];
        if (lr == -INFINITY) continue;
        const float w = expf(lr - M) * inv;
        const int64_t off = src * D + 4 * c;
        float4 v;
        if (IN_BF16) {
          const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(cp.o[rho]) + off);
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
          const float2 bb = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
          v = make_float4(a.x, a.y, bb.x, bb.y);
        } else {
          v = *reinterpret_cast<const float4*>(static_cast<const float*>(cp.o[rho]) + off);
        }
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
      }
    }
    const int64_t off = row * D + 4 * c;
    if (out_bf16) {
      uint2 w2;
      w2.x = pack_bf16x2(acc.x, acc.y);
      w2.y = pack_bf16x2(acc.z, acc.w);
      *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(o) + off) = w2;
    } else {
      *reinterpret_cast<float4*>(static_cast<float*>(o) + off) = acc;
    }
  }
  if (lse && lane == 0) lse[row] = (M == -INFINITY) ? -INFINITY : M + logf(L);
}

// ------------------------------------------------------------------- host

cudaError_t launch_attn_combine_streams(const void* const* o_parts, const float* const* lse_parts, void* o,
                                        float* lse, int R, int B, int n, int Hq, int D, int r, bool in_bf16,
                                        bool out_bf16, cudaStream_t st) {
  if (R < 1 || R > kPeerMaxRanks) return cudaErrorInvalidValue;
  CombinePtrs cp = {};
  for (int i = 0; i < R; ++i) {
    cp.o[i] = o_parts[i];
    cp.lse[i] = lse_parts[i];
  }
  const int64_t rows = static_cast<int64_t>(B) * (n / R) * Hq;
  if (rows == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (rows * 32 + threads - 1) / threads;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  if (in_bf16)
    attn_combine_streams_kernel<true><<<static_cast<unsigned>(blocks), threads, 0, st>>>(cp, o, lse, R, B, n, Hq, D,
                                                                                       r, out_bf16 ? 1 : 0);
  else
    attn_combine_streams_kernel<false><<<static_cast<unsigned>(blocks), threads, 0, st>>>(cp, o, lse, R, B, n, Hq, D,
                                                                                        r, out_bf16 ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace hd
