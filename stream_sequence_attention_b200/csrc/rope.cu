// Rotary position embedding over the expanded sequence, in place on q and k.
//
// ("Hidden Decoding at Scale", "Multi-Stream Expansion and Training
// Objective": the expanded sequence runs with contiguous RoPE positions.)
// Row r of sequence b is at position pos = pos_base + pos_mult*pos0[b] + r;
// the first rot_dim features rotate pairwise by pos * theta_j with
// theta_j = base^(-2j/rot_dim): pairs (j, j + rot_dim/2) or (2j, 2j + 1).
//
// HBM-bound (every element read and written once).  One CTA per position:
// its rot_dim/2 angles and their cos/sin are formed once in float64 (the
// angle reaches 2^31 rad, beyond what a float32 product and reduction keep
// to bf16 accuracy) and shared by all Hq + Hkv heads of q and k, which the
// CTA then rotates four pairs per thread with 8- or 16-byte accesses.
#include "hd_common.cuh"
#include "hd_launch.h"

namespace hd {

constexpr int kRopeThreads = 128;

__device__ __forceinline__ void load4(const void* p, bool bf16, float (&v)[4]) {
  if (bf16) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    v[0] = a.x;
    v[1] = a.y;
    v[2] = b.x;
    v[3] = b.y;
  } else {
    const float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x;
    v[1] = f.y;
    v[2] = f.z;
    v[3] = f.w;
  }
}

__device__ __forceinline__ void store4(void* p, bool bf16, const float (&v)[4]) {
  if (bf16) {
    uint2 u;
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) = u;
  } else {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

template <bool BF16>
__global__ void __launch_bounds__(kRopeThreads) rope_kernel(const RopeParams p) {
  __shared__ float2 cs[kRopeMaxPairs];
  constexpr int ES = BF16 ? 2 : 4;
  const int64_t row = blockIdx.x;  // b*P + r
  const int b = static_cast<int>(row / p.P);
  const int r = static_cast<int>(row - static_cast<int64_t>(b) * p.P);
  const int64_t pos = p.pos_base + p.pos_mult * (p.pos0 ? static_cast<int64_t>(p.pos0[b]) : 0) + r;
  const int half = p.rot / 2;
  for (int j = threadIdx.x; j < half; j += kRopeThreads) {
    double s, c;
    sincos(static_cast<double>(pos) * p.theta[j], &s, &c);
    cs[j] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
  __syncthreads();
  const int groups = p.rot / 8;  // four pairs per item
  const int items = (p.Hq + p.Hkv) * groups;
  for (int it = threadIdx.x; it < items; it += kRopeThreads) {
    const int h = it / groups;
    const int g = it - h * groups;
    uint8_t* x = h < p.Hq ? static_cast<uint8_t*>(p.q) + ((row * p.Hq + h) * p.D) * ES
                          : static_cast<uint8_t*>(p.k) + ((row * p.Hkv + (h - p.Hq)) * p.D) * ES;
    const int j0 = 4 * g;  // first pair of this item
    float a[4], bb[4];
    if (p.layout == HD_ROPE_HALF) {
      load4(x + j0 * ES, BF16, a);
      load4(x + (j0 + half) * ES, BF16, bb);
    } else {
      float e0[4], e1[4];
      load4(x + 2 * j0 * ES, BF16, e0);
      load4(x + (2 * j0 + 4) * ES, BF16, e1);
      a[0] = e0[0], bb[0] = e0[1], a[1] = e0[2], bb[1] = e0[3];
      a[2] = e1[0], bb[2] = e1[1], a[3] = e1[2], bb[3] = e1[3];
    }
    float ra[4], rb[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 t = cs[j0 + e];
      ra[e] = fmaf(a[e], t.x, -bb[e] * t.y);
      rb[e] = fmaf(a[e], t.y, bb[e] * t.x);
    }
    if (p.layout == HD_ROPE_HALF) {
      store4(x + j0 * ES, BF16, ra);
      store4(x + (j0 + half) * ES, BF16, rb);
    } else {
      const float e0[4] = {ra[0], rb[0], ra[1], rb[1]};
      const float e1[4] = {ra[2], rb[2], ra[3], rb[3]};
      store4(x + 2 * j0 * ES, BF16, e0);
      store4(x + (2 * j0 + 4) * ES, BF16, e1);
    }
  }
}

cudaError_t launch_rope(const RopeParams& p, bool bf16, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.P;
  if (rows <= 0) return cudaSuccess;
  if (rows > 0x7fffffff) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(rows));
  if (bf16)
    rope_kernel<true><<<grid, kRopeThreads, 0, st>>>(p);
  else
    rope_kernel<false><<<grid, kRopeThreads, 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace hd
