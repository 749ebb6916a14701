// Rotary position embedding over the expanded sequence, in place on q and k.
//
// ("Hidden Decoding at Scale", "Multi-Stream Expansion and Training
// Objective": the expanded sequence runs with contiguous RoPE positions.)
// Row r of sequence b is at position pos = pos_base + pos_mult*pos0[b] + r;
// the first rot_dim features rotate pairwise by pos * theta_j with
// theta_j = base^(-2j/rot_dim): pairs (j, j + rot_dim/2) or (2j, 2j + 1).
//
// HBM-bound (every element read and written once).  One CTA per position:
// its rot_dim/2 cos/sin pairs are formed once and shared by all Hq + Hkv
// heads of q and k.  The angle pos*theta_j reaches 2^31 rad, far beyond what
// a float32 product keeps to bf16 accuracy, so it is reduced exactly: the
// host passes theta_j/(2 pi) as a 64-bit fixed-point fraction of a turn F_j,
// and pos*F_j mod 2^64 (an integer product) is the angle's fraction of a
// turn; float32 sincospi of it is accurate to ~2e-7 rad.
#include "hd_common.cuh"
#include "hd_launch.h"

namespace hd {

// Launch shape (compile-time; the defaults are the measured best on B200):
// threads per CTA, head rows a thread loads before it stores any, and
// whether bf16 rows use 16-byte accesses (8 pairs per item).
#ifndef HD_ROPE_THREADS
#define HD_ROPE_THREADS 64
#endif
#ifndef HD_ROPE_CHUNK
#define HD_ROPE_CHUNK 1
#endif
#ifndef HD_ROPE_WIDE
#define HD_ROPE_WIDE 1
#endif
// 1: the CTA forms one cos/sin table in shared memory behind a barrier;
// 0: every thread forms its own NP pairs while its loads are in flight.
#ifndef HD_ROPE_SMEM_TABLE
#define HD_ROPE_SMEM_TABLE 1
#endif
constexpr int kRopeThreads = HD_ROPE_THREADS;
constexpr int kRopeChunk = HD_ROPE_CHUNK;

// NP consecutive elements <-> floats (16 bytes per access for NP*ES == 16).
template <int NP, bool BF16>
__device__ __forceinline__ void load_n(const uint8_t* p, float (&v)[NP]) {
  if constexpr (BF16) {
    static_assert(NP == 4 || NP == 8, "");
    if constexpr (NP == 8) {
      const uint4 u = *reinterpret_cast<const uint4*>(p);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
        v[2 * e] = f.x;
        v[2 * e + 1] = f.y;
      }
    } else {
      const uint2 u = *reinterpret_cast<const uint2*>(p);
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
      const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
      v[0] = a.x, v[1] = a.y, v[2] = b.x, v[3] = b.y;
    }
  } else {
    static_assert(NP == 4, "");
    const float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x, v[1] = f.y, v[2] = f.z, v[3] = f.w;
  }
}

template <int NP, bool BF16>
__device__ __forceinline__ void store_n(uint8_t* p, const float (&v)[NP]) {
  if constexpr (BF16) {
    if constexpr (NP == 8) {
      uint4 u;
      u.x = pack_bf16x2(v[0], v[1]);
      u.y = pack_bf16x2(v[2], v[3]);
      u.z = pack_bf16x2(v[4], v[5]);
      u.w = pack_bf16x2(v[6], v[7]);
      *reinterpret_cast<uint4*>(p) = u;
    } else {
      uint2 u;
      u.x = pack_bf16x2(v[0], v[1]);
      u.y = pack_bf16x2(v[2], v[3]);
      *reinterpret_cast<uint2*>(p) = u;
    }
  } else {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

// One CTA per position.  Thread t owns pair group g = t mod G (NP pairs:
// in the rotate-half form NP consecutive features from each half, in the
// interleaved form 2*NP consecutive features) of head slots t/G, t/G + T/G,
// ... over the Hq + Hkv heads of q then k.  It loads up to kRopeChunk head
// rows before it rotates and stores any of them (the stores go to the loaded
// addresses, so later loads cannot be moved above them), and its first loads
// are in flight while the CTA forms the cos/sin table.
template <int NP, bool BF16>
__global__ void __launch_bounds__(kRopeThreads) rope_kernel(const RopeParams p) {
  __shared__ float2 cs[kRopeMaxPairs];
  constexpr int ES = BF16 ? 2 : 4;
  const int64_t row = blockIdx.x;  // b*P + r
  const int half = p.rot / 2;
  const int G = half / NP;
  const int HS = kRopeThreads / G;  // head rows per pass
  const int hs = threadIdx.x / G;
  const int g = threadIdx.x - hs * G;
  const int j0 = NP * g;
  const int H = p.Hq + p.Hkv;
  const bool active = hs < HS;
  const bool is_half = p.layout == HD_ROPE_HALF;
  const int off_a = (is_half ? j0 : 2 * j0) * ES;
  const int off_b = (is_half ? j0 + half : 2 * j0 + NP) * ES;
  uint8_t* const qrow = static_cast<uint8_t*>(p.q) + row * p.Hq * p.D * ES;
  uint8_t* const krow = static_cast<uint8_t*>(p.k) + row * p.Hkv * p.D * ES;
  auto head_ptr = [&](int h) -> uint8_t* {
    return h < p.Hq ? qrow + h * p.D * ES : krow + (h - p.Hq) * p.D * ES;
  };

  float va[kRopeChunk][NP], vb[kRopeChunk][NP];
  int h0 = hs;
  auto load_chunk = [&]() {
#pragma unroll
    for (int u = 0; u < kRopeChunk; ++u) {
      const int h = h0 + u * HS;
      if (active && h < H) {
        uint8_t* x = head_ptr(h);
        load_n<NP, BF16>(x + off_a, va[u]);
        load_n<NP, BF16>(x + off_b, vb[u]);
      }
    }
  };
  load_chunk();

  const int b = static_cast<int>(row / p.P);
  const int r = static_cast<int>(row - static_cast<int64_t>(b) * p.P);
  const int64_t pos = p.pos_base + p.pos_mult * (p.pos0 ? static_cast<int64_t>(p.pos0[b]) : 0) + r;
  // cos/sin of pos * theta_j: pos * fturn[j] mod 2^64 is the angle's
  // fraction of a turn; as a signed value times 2^-63 it is t in [-1, 1)
  // with angle = pi * t.
  auto cos_sin = [&](int j) -> float2 {
    const uint64_t turns = static_cast<uint64_t>(pos) * p.fturn[j];
    const float tt = static_cast<float>(static_cast<int64_t>(turns)) * 0x1p-63f;
    float sn, cn;
    sincospif(tt, &sn, &cn);
    return make_float2(cn, sn);
  };
  // This thread's NP cos/sin pairs: rotate-half pairs j0 + e; interleaved
  // pairs j0 + e over va then vb.
  float2 t[NP];
  if (HD_ROPE_SMEM_TABLE) {
    for (int j = threadIdx.x; j < half; j += kRopeThreads) cs[j] = cos_sin(j);
    __syncthreads();
    if (!active) return;
#pragma unroll
    for (int e = 0; e < NP; ++e) t[e] = cs[j0 + e];
  } else {
    if (!active) return;
#pragma unroll
    for (int e = 0; e < NP; ++e) t[e] = cos_sin(j0 + e);
  }

  for (;;) {
#pragma unroll
    for (int u = 0; u < kRopeChunk; ++u) {
      const int h = h0 + u * HS;
      if (h < H) {
        float ra[NP], rb[NP];
        if (is_half) {
#pragma unroll
          for (int e = 0; e < NP; ++e) {
            ra[e] = fmaf(va[u][e], t[e].x, -vb[u][e] * t[e].y);
            rb[e] = fmaf(va[u][e], t[e].y, vb[u][e] * t[e].x);
          }
        } else {
#pragma unroll
          for (int e = 0; e < NP / 2; ++e) {
            const float2 t0 = t[e], t1 = t[NP / 2 + e];
            ra[2 * e] = fmaf(va[u][2 * e], t0.x, -va[u][2 * e + 1] * t0.y);
            ra[2 * e + 1] = fmaf(va[u][2 * e], t0.y, va[u][2 * e + 1] * t0.x);
            rb[2 * e] = fmaf(vb[u][2 * e], t1.x, -vb[u][2 * e + 1] * t1.y);
            rb[2 * e + 1] = fmaf(vb[u][2 * e], t1.y, vb[u][2 * e + 1] * t1.x);
          }
        }
        uint8_t* x = head_ptr(h);
        store_n<NP, BF16>(x + off_a, ra);
        store_n<NP, BF16>(x + off_b, rb);
      }
    }
    h0 += kRopeChunk * HS;
    if (h0 >= H) break;
    load_chunk();
  }
}

// ------------------------------------------------------------------- host

void rope_fill_turns(RopeParams& p, int rot_dim, double base) {
  // theta_j / (2 pi) in turns, as a 64-bit binary fraction (long double:
  // 64-bit mantissa); theta_j <= 1 so the fraction is below 1/(2 pi).
  const long double two_pi = 6.283185307179586476925286766559005768L;
  for (int j = 0; j < rot_dim / 2; ++j) {
    const long double turns = powl(static_cast<long double>(base), -2.0L * j / rot_dim) / two_pi;
    p.fturn[j] = static_cast<uint64_t>(ldexpl(turns, 64));
  }
}

cudaError_t launch_rope(const RopeParams& p, bool bf16, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.P;
  if (rows <= 0) return cudaSuccess;
  if (rows > 0x7fffffff) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(rows));
  if (bf16) {
    if (HD_ROPE_WIDE && p.rot % 16 == 0)
      rope_kernel<8, true><<<grid, kRopeThreads, 0, st>>>(p);
    else
      rope_kernel<4, true><<<grid, kRopeThreads, 0, st>>>(p);
  } else {
    rope_kernel<4, false><<<grid, kRopeThreads, 0, st>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace hd
