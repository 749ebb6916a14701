// Backward of Stream-Factorized Attention: the per-row preparation shared by
// both backward paths, and the float32 CUDA-core path.
//
// ("Hidden Decoding at Scale", "Stream-Factorized Attention", Figure 2; the
// layers are trained through, "Computational Cost".)  With P the softmax of
// the forward and delta_i = <dO_i, O_i> = sum_j P_ij <dO_i, v_j>:
//   dS_ij = P_ij (<dO_i, v_j> - delta_i),  dV = P^T dO,
//   dQ = scale dS K,  dK = scale dS^T Q  (dK, dV summed over a GQA group).
// P is recomputed from the forward's lse: P_ij = 2^(scale log2e <q_i,k_j> - lse_i log2e).
//
// float32 path: one CTA owns 64 query rows (dQ kernel) or 64 key rows (dK/dV
// kernel) of one (batch, head, stream); four threads share a row, each
// holding a quarter of the head dimension; the other side's rows are staged
// in shared memory 32 at a time.
#include "hd_common.cuh"
#include "hd_launch.h"

namespace hd {

// ------------------------------------------------------------ preparation

// Each row (b, p, h) is read by LPR lanes with 16-byte loads (a warp covers
// 32/LPR rows): delta = <dO, o> in float32 and lse in log2 units, stored
// stream-major.  Threads past the last row write the padding.
template <int D, bool BF16>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const void* __restrict__ o, const void* __restrict__ dO,
                                                       const float* __restrict__ lse, BwdWs ws,
                                                       const AttnGeom g, int Hq, int64_t rows, int64_t pad) {
  constexpr int ES = BF16 ? 2 : 4;
  constexpr int LPR = D * ES / 16;  // lanes per row
  constexpr int RPW = 32 / LPR;     // rows per warp
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t w = tid >> 5;
  const int lane = threadIdx.x & 31;
  const int Lpad = bwd_lpad(g.Lq);
  const int64_t row_warps = (rows + RPW - 1) / RPW;
  if (w < row_warps) {
    const int64_t row = w * RPW + lane / LPR;
    const int part = lane % LPR;
    float acc = 0.f;
    if (row < rows) {
      const uint4 a = reinterpret_cast<const uint4*>(o)[row * LPR + part];
      const uint4 b = reinterpret_cast<const uint4*>(dO)[row * LPR + part];
      if (BF16) {
        const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
        const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fa = __bfloat1622float2(pa[e]), fb = __bfloat1622float2(pb[e]);
          acc = fmaf(fa.x, fb.x, fmaf(fa.y, fb.y, acc));
        }
      } else {
        acc = __uint_as_float(a.x) * __uint_as_float(b.x) + __uint_as_float(a.y) * __uint_as_float(b.y) +
              __uint_as_float(a.z) * __uint_as_float(b.z) + __uint_as_float(a.w) * __uint_as_float(b.w);
      }
    }
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (part == 0 && row < rows) {
      // row = (b*P + p)*Hq + h, p = i*ns + s
      const int64_t P = static_cast<int64_t>(g.ns) * g.Lq;
      const int h = static_cast<int>(row % Hq);
      const int64_t bp = row / Hq;
      const int b = static_cast<int>(bp / P);
      const int64_t p = bp - b * P;
      const int i = static_cast<int>(p / g.ns), s = static_cast<int>(p - static_cast<int64_t>(i) * g.ns);
      const float l2 = lse[(static_cast<int64_t>(b) * Hq + h) * P + p] * 1.4426950408889634f;
      const int64_t at = ((static_cast<int64_t>(b) * Hq + h) * g.ns + s) * Lpad + i;
      ws.nl2[at] = -l2;
      ws.delta[at] = acc;
    }
  } else {
    const int per = Lpad - g.Lq;
    const int64_t e = (w - row_warps) * 32 + lane;
    if (per > 0 && e < pad) {
      const int64_t line = e / per;  // (b*Hq + h)*ns + s
      const int i = g.Lq + static_cast<int>(e - line * per);
      ws.nl2[line * Lpad + i] = -INFINITY;
      ws.delta[line * Lpad + i] = 0.f;
    }
  }
}

// ------------------------------------------------------------------- host

cudaError_t launch_bwd_prep(const void* o, const void* dO, const float* lse, BwdWs ws, const AttnGeom& g, int Hq,
                            int D, bool bf16, cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(g.B) * g.ns * g.Lq * Hq;
  const int64_t pad = static_cast<int64_t>(g.B) * Hq * g.ns * (bwd_lpad(g.Lq) - g.Lq);
  const int rpw = 32 / (D * (bf16 ? 2 : 4) / 16);
  const int64_t warps = (rows + rpw - 1) / rpw + (pad + 31) / 32;
  const int64_t blocks = (warps * 32 + 255) / 256;
  if (blocks <= 0) return cudaSuccess;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(blocks));
  if (D == 64) {
    if (bf16)
      bwd_prep_kernel<64, true><<<grid, 256, 0, st>>>(o, dO, lse, ws, g, Hq, rows, pad);
    else
      bwd_prep_kernel<64, false><<<grid, 256, 0, st>>>(o, dO, lse, ws, g, Hq, rows, pad);
  } else {
    if (bf16)
      bwd_prep_kernel<128, true><<<grid, 256, 0, st>>>(o, dO, lse, ws, g, Hq, rows, pad);
    else
      bwd_prep_kernel<128, false><<<grid, 256, 0, st>>>(o, dO, lse, ws, g, Hq, rows, pad);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------- float32 path

constexpr int kBwRows = 64;     // rows owned by one CTA
constexpr int kBwTile = 32;     // rows of the other side staged per step
constexpr int kBwThreads = 256; // four threads per owned row

__device__ __forceinline__ float quad_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x;
}

// dQ: CTA = 64 query tokens of one (b, query head, stream).
template <int D>
__global__ void __launch_bounds__(kBwThreads) attn_bwd_dq_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const float* __restrict__ dO, const BwdWs ws, float* __restrict__ dq, const AttnGeom g, int Hq,
    int Hkv, int W, float sl2, float scale) {
  constexpr int DQ = D / 4;
  __shared__ __align__(16) float Ks[kBwTile][D];
  __shared__ __align__(16) float Vs[kBwTile][D];
  const int nqb = (g.Lq + kBwRows - 1) / kBwRows;
  const int qblk = nqb - 1 - static_cast<int>(blockIdx.x);  // longest first
  const int hs = blockIdx.y;                                 // h * ns + s
  const int h = hs / g.ns, s = hs - h * g.ns;
  const int b = blockIdx.z;
  const int kvh = h / (Hq / Hkv);
  const int skv = g.kv_stream >= 0 ? g.kv_stream : s;
  const int tid = threadIdx.x, r = tid >> 2, part = tid & 3;
  const int q0 = qblk * kBwRows;
  const int i = q0 + r;
  const bool row_ok = i < g.Lq;
  const int ic = row_ok ? i : g.Lq - 1;
  const int pic = ic * g.qstride + g.qoff;  // key index of this query
  const int64_t qrow = ((static_cast<int64_t>(b) * g.q_ns * g.Lq + static_cast<int64_t>(ic) * g.q_ns + s) * Hq + h) * D;
  float qr[DQ], dor[DQ], acc[DQ];
#pragma unroll
  for (int d = 0; d < DQ; ++d) {
    qr[d] = q[qrow + part * DQ + d] * sl2;
    dor[d] = dO[qrow + part * DQ + d];
    acc[d] = 0.f;
  }
  const int64_t lat = ((static_cast<int64_t>(b) * Hq + h) * g.ns + s) * bwd_lpad(g.Lq) + ic;
  const float2 ld = make_float2(ws.nl2[lat], ws.delta[lat]);
  const int hi = min(min(q0 + kBwRows - 1, g.Lq - 1) * g.qstride + g.qoff, g.Lk - 1);
  const int lo = W > 0 ? max(0, q0 * g.qstride + g.qoff - W + 1) : 0;
  const int64_t kv_stride = static_cast<int64_t>(g.kv_ns) * Hkv * D;
  const int64_t kv_base = (static_cast<int64_t>(b) * g.kv_ns * g.Lk * Hkv + static_cast<int64_t>(skv) * Hkv + kvh) * D;
  for (int k0 = lo; k0 <= hi; k0 += kBwTile) {
    __syncthreads();
    for (int e = tid; e < kBwTile * (D / 4); e += kBwThreads) {
      const int c = e / (D / 4), d4 = e - c * (D / 4);
      const int j = k0 + c;
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f), bb = a;
      if (j <= hi) {
        a = reinterpret_cast<const float4*>(k + kv_base + j * kv_stride)[d4];
        bb = reinterpret_cast<const float4*>(v + kv_base + j * kv_stride)[d4];
      }
      reinterpret_cast<float4*>(&Ks[c][0])[d4] = a;
      reinterpret_cast<float4*>(&Vs[c][0])[d4] = bb;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < kBwTile; ++c) {
      float sd = 0.f, pd = 0.f;
#pragma unroll
      for (int d = 0; d < DQ; ++d) {
        sd = fmaf(qr[d], Ks[c][part * DQ + d], sd);
        pd = fmaf(dor[d], Vs[c][part * DQ + d], pd);
      }
      sd = quad_sum(sd);
      pd = quad_sum(pd);
      const int j = k0 + c;
      const bool vis = j <= hi && j <= pic && (W <= 0 || pic - j < W);
      const float p = vis ? exp2f(sd + ld.x) : 0.f;
      const float ds = p * (pd - ld.y);
#pragma unroll
      for (int d = 0; d < DQ; ++d) acc[d] = fmaf(ds, Ks[c][part * DQ + d], acc[d]);
    }
  }
  if (!row_ok) return;
#pragma unroll
  for (int d = 0; d < DQ; ++d) dq[qrow + part * DQ + d] = acc[d] * scale;
}

// dK, dV: CTA = 64 key tokens of one (b, KV head, stream), all query heads of
// its group.
template <int D>
__global__ void __launch_bounds__(kBwThreads) attn_bwd_dkv_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const float* __restrict__ dO, const BwdWs ws, float* __restrict__ dk, float* __restrict__ dv,
    const AttnGeom g, int Hq, int Hkv, int W, float sl2, float scale) {
  constexpr int DQ = D / 4;
  __shared__ __align__(16) float Qs[kBwTile][D];
  __shared__ __align__(16) float Os[kBwTile][D];
  __shared__ float2 Ls[kBwTile];
  const int kblk = blockIdx.x;  // causal: the first key blocks have the most queries
  const int kns = g.kv_stream >= 0 ? 1 : g.kv_ns;
  const int hs = blockIdx.y;    // kvh * kns + key stream
  const int kvh = hs / kns, ks = hs - kvh * kns;
  const int skv = g.kv_stream >= 0 ? g.kv_stream : ks;  // stream of the K/V view
  const int s = g.kv_stream >= 0 ? 0 : ks;              // query stream reading it
  const int b = blockIdx.z;
  const int G = Hq / Hkv;
  const int tid = threadIdx.x, r = tid >> 2, part = tid & 3;
  const int k0 = kblk * kBwRows;
  const int j = k0 + r;
  const bool row_ok = j < g.Lk;
  const int jc = row_ok ? j : g.Lk - 1;
  const int64_t krow =
      ((static_cast<int64_t>(b) * g.kv_ns * g.Lk + static_cast<int64_t>(jc) * g.kv_ns + skv) * Hkv + kvh) * D;
  float kr[DQ], vr[DQ], ak[DQ], av[DQ];
#pragma unroll
  for (int d = 0; d < DQ; ++d) {
    kr[d] = k[krow + part * DQ + d] * sl2;
    vr[d] = v[krow + part * DQ + d];
    ak[d] = 0.f;
    av[d] = 0.f;
  }
  // queries with k0 <= pos(i) (and pos(i) - (k0 + 63) < W), pos(i) = i*qstride + qoff
  const int lo = k0 <= g.qoff ? 0 : (k0 - g.qoff + g.qstride - 1) / g.qstride;
  const int hi = W > 0 ? min(g.Lq - 1, (k0 + kBwRows - 1 + W - 1 - g.qoff) / g.qstride) : g.Lq - 1;
  const int Lpad = bwd_lpad(g.Lq);
  const int64_t q_stride = static_cast<int64_t>(g.q_ns) * Hq * D;
  for (int hh = 0; hh < G; ++hh) {
    const int h = kvh * G + hh;
    const int64_t q_base = (static_cast<int64_t>(b) * g.q_ns * g.Lq * Hq + static_cast<int64_t>(s) * Hq + h) * D;
    const int64_t l_base = ((static_cast<int64_t>(b) * Hq + h) * g.ns + s) * Lpad;
    for (int i0 = lo; i0 <= hi; i0 += kBwTile) {
      __syncthreads();
      for (int e = tid; e < kBwTile * (D / 4); e += kBwThreads) {
        const int c = e / (D / 4), d4 = e - c * (D / 4);
        const int i = i0 + c;
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f), bb = a;
        if (i <= hi) {
          a = reinterpret_cast<const float4*>(q + q_base + i * q_stride)[d4];
          bb = reinterpret_cast<const float4*>(dO + q_base + i * q_stride)[d4];
        }
        reinterpret_cast<float4*>(&Qs[c][0])[d4] = a;
        reinterpret_cast<float4*>(&Os[c][0])[d4] = bb;
      }
      if (tid < kBwTile)
        Ls[tid] = (i0 + tid <= hi) ? make_float2(ws.nl2[l_base + i0 + tid], ws.delta[l_base + i0 + tid])
                                   : make_float2(INFINITY, 0.f);
      __syncthreads();
#pragma unroll 4
      for (int c = 0; c < kBwTile; ++c) {
        float sd = 0.f, pd = 0.f;
#pragma unroll
        for (int d = 0; d < DQ; ++d) {
          sd = fmaf(kr[d], Qs[c][part * DQ + d], sd);
          pd = fmaf(vr[d], Os[c][part * DQ + d], pd);
        }
        sd = quad_sum(sd);
        pd = quad_sum(pd);
        const int i = i0 + c;
        const int pi = i * g.qstride + g.qoff;
        const bool vis = i <= hi && pi >= jc && (W <= 0 || pi - jc < W);
        const float2 l = Ls[c];
        const float p = vis ? exp2f(sd + l.x) : 0.f;
        const float ds = p * (pd - l.y);
#pragma unroll
        for (int d = 0; d < DQ; ++d) {
          av[d] = fmaf(p, Os[c][part * DQ + d], av[d]);
          ak[d] = fmaf(ds, Qs[c][part * DQ + d], ak[d]);
        }
      }
    }
  }
  if (!row_ok) return;
#pragma unroll
  for (int d = 0; d < DQ; ++d) {
    dk[krow + part * DQ + d] = ak[d] * scale;
    dv[krow + part * DQ + d] = av[d];
  }
}

cudaError_t launch_attn_bwd_f32(const float* q, const float* k, const float* v, const float* dO, BwdWs ws,
                                float* dq, float* dk, float* dv, const AttnGeom& g, int Hq, int Hkv, int D, int W,
                                float scale, cudaStream_t st) {
  const int nb = (g.Lq + kBwRows - 1) / kBwRows;
  const int nkb = (g.Lk + kBwRows - 1) / kBwRows;
  const int kns = g.kv_stream >= 0 ? 1 : g.kv_ns;
  const float sl2 = scale * 1.4426950408889634f;
  const dim3 gq(nb, Hq * g.ns, g.B), gk(nkb, Hkv * kns, g.B);
  if (g.kv_stream >= 0 && g.kv_ns > 1) {  // key streams no query reads: zero gradients
    const size_t bytes = static_cast<size_t>(g.B) * g.kv_ns * g.Lk * Hkv * D * sizeof(float);
    cudaError_t e = cudaMemsetAsync(dk, 0, bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, bytes, st);
    if (e != cudaSuccess) return e;
  }
  if (D == 64) {
    attn_bwd_dq_f32_kernel<64><<<gq, kBwThreads, 0, st>>>(q, k, v, dO, ws, dq, g, Hq, Hkv, W, sl2, scale);
    attn_bwd_dkv_f32_kernel<64><<<gk, kBwThreads, 0, st>>>(q, k, v, dO, ws, dk, dv, g, Hq, Hkv, W, sl2, scale);
  } else {
    attn_bwd_dq_f32_kernel<128><<<gq, kBwThreads, 0, st>>>(q, k, v, dO, ws, dq, g, Hq, Hkv, W, sl2, scale);
    attn_bwd_dkv_f32_kernel<128><<<gk, kBwThreads, 0, st>>>(q, k, v, dO, ws, dk, dv, g, Hq, Hkv, W, sl2, scale);
  }
  return cudaGetLastError();
}

}  // namespace hd
