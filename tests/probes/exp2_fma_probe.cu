// Test probe: evaluates the FMA-pipe exponentials (exp2_fma, the packed
// exp2_fma2, and exp2_sat2 behind its saturating shift) and the MUFU form
// (ex2) of the attention kernels' shared header on given inputs, so a GPU
// test can compare them.  Built by tests/test_gpu_exp2_fma.py.
#include "hd_common.cuh"

__global__ void exp2_probe_kernel(const float* x, float* fma_out, float* mufu_out, float* pair_out, float* sat_out,
                                  int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    fma_out[i] = hd::exp2_fma(x[i]);
    mufu_out[i] = hd::ex2(x[i]);
    // the packed form on the pair (x[i], x[i ^ 1])
    float a, b;
    const int j = ((i ^ 1) < n) ? (i ^ 1) : i;
    hd::unpack_f32x2(hd::exp2_fma2(x[i], x[j]), a, b);
    pair_out[i] = a;
    // the saturating form: y = sat((x + 126) / 134), as the attention
    // kernel shifts an exponent x <= 8 (its rescale threshold)
    const float k1 = 1.f / 134.f, k2 = 126.f / 134.f;
    hd::unpack_f32x2(hd::exp2_sat2<8>(hd::pack_f32x2(hd::fma_sat(x[i], k1, k2), hd::fma_sat(x[j], k1, k2))), a,
                     b);
    sat_out[i] = a;
  }
}

extern "C" int exp2_probe(const float* x, float* fma_out, float* mufu_out, float* pair_out, float* sat_out, int n) {
  if (n <= 0) return 0;
  exp2_probe_kernel<<<(n + 255) / 256, 256>>>(x, fma_out, mufu_out, pair_out, sat_out, n);
  return static_cast<int>(cudaDeviceSynchronize());
}
