// Stream-Factorized Attention forward for float32 inputs on CUDA cores.
//
// ("Hidden Decoding at Scale", "Stream-Factorized Attention", Figure 2.)
// The call's geometry (AttnGeom, hd_launch.h) maps every query token to the
// key stream it reads and to its position there: intra mode is n streams of
// L tokens read in place over the interleaved layout (stride-n addressing, no
// de-interleave in memory); cross mode is one stream of n*L positions; the
// final-stream variants ("Persistent KV and the KV-mirror Saving") read
// queries of the last stream only.  Key j is visible to query token i iff
// j <= pos(i) and, with a window W > 0, pos(i) - j < W.
//
// This path exists for float32 inputs, where the 1e-4 parity bound rules
// out tensor-core rounding.  One CTA owns 64 query tokens of one
// (batch, head, stream); two threads share a query row, each holding half of
// the head dimension, and K/V tiles of 32 keys are staged in shared memory.
#include "hd_common.cuh"
#include "hd_launch.h"

namespace hd {

constexpr int kF32Rows = 64;
constexpr int kF32Keys = 32;
constexpr int kF32Threads = 128;

template <int D>
__global__ void __launch_bounds__(kF32Threads) attn_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    void* __restrict__ o, float* __restrict__ lse, const AttnGeom g, int Hq, int Hkv, int W, float scale_log2,
    int out_bf16) {
  constexpr int DH = D / 2;
  __shared__ __align__(16) float Ks[kF32Keys][D];
  __shared__ __align__(16) float Vs[kF32Keys][D];

  const int nqb = (g.Lq + kF32Rows - 1) / kF32Rows;
  const int qblk = nqb - 1 - static_cast<int>(blockIdx.x);  // longest first
  const int hs = blockIdx.y;                                 // h * ns + s
  const int h = hs / g.ns, s = hs - (hs / g.ns) * g.ns;
  const int b = blockIdx.z;
  const int G = Hq / Hkv;
  const int kvh = h / G;
  const int skv = g.kv_stream >= 0 ? g.kv_stream : s;

  const int tid = threadIdx.x;
  const int r = tid >> 1, half = tid & 1;
  const int q0 = qblk * kF32Rows;
  const int i = q0 + r;
  const bool row_ok = i < g.Lq;
  const int qb = g.qoff + s * g.qsstride;  // key index offset of this query stream
  const int pi = (row_ok ? i : g.Lq - 1) * g.qstride + qb;  // key index of this query

  float qr[DH], acc[DH];
  {
    const int ic = row_ok ? i : g.Lq - 1;
    const float* qp =
        q + ((static_cast<int64_t>(b) * g.q_ns * g.Lq + static_cast<int64_t>(ic) * g.q_ns + s) * Hq + h) * D +
        half * DH;
#pragma unroll
    for (int d = 0; d < DH; ++d) {
      qr[d] = qp[d] * scale_log2;
      acc[d] = 0.f;
    }
  }
  float m = -INFINITY, l = 0.f;

  const int last = min(q0 + kF32Rows - 1, g.Lq - 1);
  const int hi_tok = min(last * g.qstride + qb, g.Lk - 1);
  const int lo_tok = W > 0 ? max(0, q0 * g.qstride + qb - W + 1) : 0;
  const int64_t kv_row = static_cast<int64_t>(g.kv_ns) * Hkv * D;  // token stride in k/v
  const int64_t kv_base = (static_cast<int64_t>(b) * g.kv_ns * g.Lk * Hkv + static_cast<int64_t>(skv) * Hkv + kvh) * D;
  const float* kb = k + kv_base;
  const float* vb = v + kv_base;

  for (int k0 = lo_tok; k0 <= hi_tok; k0 += kF32Keys) {
    __syncthreads();
    for (int e = tid; e < kF32Keys * (D / 4); e += kF32Threads) {
      const int c = e / (D / 4), d4 = e - c * (D / 4);
      const int j = k0 + c;
      float4 kv4 = make_float4(0.f, 0.f, 0.f, 0.f), vv4 = kv4;
      if (j <= hi_tok) {
        kv4 = reinterpret_cast<const float4*>(kb + j * kv_row)[d4];
        vv4 = reinterpret_cast<const float4*>(vb + j * kv_row)[d4];
      }
      reinterpret_cast<float4*>(&Ks[c][0])[d4] = kv4;
      reinterpret_cast<float4*>(&Vs[c][0])[d4] = vv4;
    }
    __syncthreads();

    float sc[kF32Keys];
    float mt = -INFINITY;
#pragma unroll
    for (int c = 0; c < kF32Keys; ++c) {
      float part = 0.f;
#pragma unroll
      for (int d = 0; d < DH; ++d) part = fmaf(qr[d], Ks[c][half * DH + d], part);
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      const int j = k0 + c;
      const bool vis = (j <= hi_tok) && (j <= pi) && (W <= 0 || pi - j < W);
      sc[c] = vis ? part : -INFINITY;
      mt = fmaxf(mt, sc[c]);
    }
    const float mn = fmaxf(m, mt);
    if (mn == -INFINITY) continue;  // nothing visible yet for this row
    const float alpha = exp2f(m - mn);  // m = -inf -> 0
    l *= alpha;
#pragma unroll
    for (int d = 0; d < DH; ++d) acc[d] *= alpha;
    m = mn;
#pragma unroll
    for (int c = 0; c < kF32Keys; ++c) {
      const float p = exp2f(sc[c] - m);
      l += p;
#pragma unroll
      for (int d = 0; d < DH; ++d) acc[d] = fmaf(p, Vs[c][half * DH + d], acc[d]);
    }
  }

  if (!row_ok) return;
  const int64_t orow = (static_cast<int64_t>(b) * g.o_rows + static_cast<int64_t>(i) * g.o_ns + s) * Hq + h;
  const float inv = 1.f / l;
  if (out_bf16) {
    __nv_bfloat16* op = static_cast<__nv_bfloat16*>(o) + orow * D + half * DH;
#pragma unroll
    for (int d = 0; d < DH; ++d) op[d] = __float2bfloat16_rn(acc[d] * inv);
  } else {
    float* op = static_cast<float*>(o) + orow * D + half * DH;
#pragma unroll
    for (int d = 0; d < DH; ++d) op[d] = acc[d] * inv;
  }
  if (lse && half == 0) {
    lse[(static_cast<int64_t>(b) * Hq + h) * g.o_rows + static_cast<int64_t>(i) * g.o_ns + s] =
        (m + log2f(l)) * 0.69314718055994531f;
  }
}

cudaError_t launch_attn_f32(const float* q, const float* k, const float* v, void* o, float* lse,
                            const AttnGeom& g, int Hq, int Hkv, int D, int W, float scale, bool out_bf16,
                            cudaStream_t st) {
  const int nqb = (g.Lq + kF32Rows - 1) / kF32Rows;
  dim3 grid(nqb, Hq * g.ns, g.B);
  const float scale_log2 = scale * 1.4426950408889634f;
  if (D == 64) {
    attn_f32_kernel<64><<<grid, kF32Threads, 0, st>>>(q, k, v, o, lse, g, Hq, Hkv, W, scale_log2,
                                                      out_bf16 ? 1 : 0);
  } else {
    attn_f32_kernel<128><<<grid, kF32Threads, 0, st>>>(q, k, v, o, lse, g, Hq, Hkv, W, scale_log2,
                                                       out_bf16 ? 1 : 0);
  }
  return cudaGetLastError();
}

}  // namespace hd
