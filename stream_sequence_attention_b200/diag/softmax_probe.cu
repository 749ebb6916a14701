// Diagnostic probe (not part of the library): clock64 timing of the phases of
// the attention kernel's softmax on one 128-score row per thread, the same
// arithmetic as a tile of the tcgen05 attention kernel, with 4 or 8 warps per
// CTA (one or two warps per SM sub-partition) and one CTA per SM:
//   0 tensor-memory load of the row (four 32-column loads, wait)
//   1 row max (3-input max, 4 chains)
//   2 exponents (packed f32x2 FMA; on the FMA-pipe pairs the saturating shift)
//   3 exponentials, bf16 pack and row sum
//   4 tensor-memory store of P (four 16-column stores, wait)
// SEL picks the pairs evaluated on the FMA pipe (exp2_sat2): 0 none, 1 one in
// three, 2 one in two, 3 two in five, 4 three in eight, 5 one in four.
// Built and run by stream_sequence_attention_b200/diag_softmax.py.
#include "hd_common.cuh"

using namespace hd;

namespace {
constexpr int kHi = 8;  // exponents reach the rescale threshold

template <int SEL>
__device__ __forceinline__ bool fma_pair(int c) {
  return SEL == 1   ? (c % 3) == 2
         : SEL == 2 ? (c & 1) == 1
         : SEL == 3 ? ((c % 5) == 1 || (c % 5) == 3)
         : SEL == 4 ? ((c & 7) == 2 || (c & 7) == 5 || (c & 7) == 7)
         : SEL == 5 ? (c & 3) == 3
                    : false;
}

template <int SEL>
__global__ void __launch_bounds__(256, 1) softmax_phases(const float* in, float* out, unsigned long long* clk,
                                                         int iters) {
  __shared__ uint32_t slot;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    tmem_alloc(smem_u32(&slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = slot;
  // warp w: lanes 32 (w % 4) .. of the 128-column buffer w / 4
  const uint32_t sS = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + (warp >> 2) * 128;
  uint32_t sv[128];
  for (int c = 0; c < 128; ++c) sv[c] = __float_as_uint(in[(threadIdx.x * 131 + c) & 4095]);
#pragma unroll
  for (int j = 0; j < 4; ++j) tmem_st32(sS + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * j]));
  tmem_wait_st();
  unsigned long long t[5] = {0, 0, 0, 0, 0};
  float acc = 0.f;
  const float sl2 = 0.127f;
  for (int it = 0; it < iters; ++it) {
    long long a = clock64(), b;
#pragma unroll
    for (int j = 0; j < 4; ++j) tmem_ld32(sS + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * j]));
    tmem_wait_ld();
    b = clock64();
    t[0] += b - a;
    a = b;
    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int c = 0; c < 128; c += 2)
      mx[(c >> 1) & 3] = fmax3(mx[(c >> 1) & 3], __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]));
    const float nmu = -(fmax3(fmax3(mx[0], mx[1], mx[2]), mx[3], mx[3]) * sl2 + acc * 1e-30f);
    b = clock64();
    t[1] += b - a;
    a = b;
    const uint64_t s2 = pack_f32x2(sl2, sl2), n2 = pack_f32x2(nmu, nmu);
    const float k1 = sl2 / (126.f + kHi), k2 = (nmu + 126.f) / (126.f + kHi);
#pragma unroll
    for (int c = 0; c < 64; ++c) {
      if (fma_pair<SEL>(c)) {
        sv[2 * c] = __float_as_uint(fma_sat(__uint_as_float(sv[2 * c]), k1, k2));
        sv[2 * c + 1] = __float_as_uint(fma_sat(__uint_as_float(sv[2 * c + 1]), k1, k2));
      } else {
        float a0, a1;
        unpack_f32x2(fma_f32x2(pack_f32x2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), s2, n2), a0,
                     a1);
        sv[2 * c] = __float_as_uint(a0);
        sv[2 * c + 1] = __float_as_uint(a1);
      }
    }
    b = clock64();
    t[2] += b - a;
    a = b;
    float ls[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    uint32_t pk[64];
#pragma unroll
    for (int c = 0; c < 64; ++c) {
      float p0, p1;
      if (fma_pair<SEL>(c)) {
        unpack_f32x2(exp2_sat2<kHi>(pack_f32x2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1]))), p0, p1);
      } else {
        p0 = ex2(__uint_as_float(sv[2 * c]));
        p1 = ex2(__uint_as_float(sv[2 * c + 1]));
      }
      ls[c & 7] += p0 + p1;
      pk[c] = pack_bf16x2(p0, p1);
    }
    b = clock64();
    t[3] += b - a;
    a = b;
    // P into the upper 64 columns, so that the scores below stay for the
    // next iteration
#pragma unroll
    for (int j = 0; j < 4; ++j) tmem_st16(sS + 64 + 16 * j, &pk[16 * j]);
    tmem_wait_st();
    b = clock64();
    t[4] += b - a;
    acc += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
#pragma unroll
    for (int j = 2; j < 4; ++j) tmem_st32(sS + 32 * j, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * j]));
    tmem_wait_st();
  }
  out[blockIdx.x * blockDim.x + threadIdx.x] = acc;
  if (lane == 0)
    for (int i = 0; i < 5; ++i) clk[(blockIdx.x * 8 + warp) * 8 + i] = t[i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 256);
}

template <int SEL>
cudaError_t launch(const float* in, float* out, unsigned long long* clk, int ctas, int threads, int iters) {
  softmax_phases<SEL><<<ctas, threads>>>(in, out, clk, iters);
  return cudaGetLastError();
}
}  // namespace

// clk: ctas x 8 warps x 8 counters (5 used), cycles summed over iters.
extern "C" int softmax_probe(int sel, int ctas, int threads, int iters, unsigned long long* clk_host) {
  if (ctas < 1 || ctas > 1024 || (threads != 128 && threads != 256) || iters < 1) return -1;
  float *in = nullptr, *out = nullptr;
  unsigned long long* clk = nullptr;
  const size_t nclk = static_cast<size_t>(ctas) * 64;
  if (cudaMalloc(&in, 4096 * sizeof(float)) != cudaSuccess) return -2;
  cudaMalloc(&out, static_cast<size_t>(ctas) * 256 * sizeof(float));
  cudaMalloc(&clk, nclk * sizeof(unsigned long long));
  cudaMemset(clk, 0, nclk * sizeof(unsigned long long));
  float h[4096];
  for (int i = 0; i < 4096; ++i) h[i] = static_cast<float>((i * 2654435761u) % 1000u) / 50.f - 10.f;
  cudaMemcpy(in, h, sizeof(h), cudaMemcpyHostToDevice);
  cudaError_t e;
  switch (sel) {
    case 0: e = launch<0>(in, out, clk, ctas, threads, iters); break;
    case 1: e = launch<1>(in, out, clk, ctas, threads, iters); break;
    case 2: e = launch<2>(in, out, clk, ctas, threads, iters); break;
    case 3: e = launch<3>(in, out, clk, ctas, threads, iters); break;
    case 4: e = launch<4>(in, out, clk, ctas, threads, iters); break;
    default: e = launch<5>(in, out, clk, ctas, threads, iters); break;
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  cudaMemcpy(clk_host, clk, nclk * sizeof(unsigned long long), cudaMemcpyDeviceToHost);
  cudaFree(in);
  cudaFree(out);
  cudaFree(clk);
  return static_cast<int>(e);
}
