// Test probe: evaluates the FMA-pipe exponential (exp2_fma) and the MUFU
// form (ex2) of the attention kernels' shared header on given inputs, so a
// GPU test can compare them.  Built by tests/test_gpu_exp2_fma.py.
#include "hd_common.cuh"

__global__ void exp2_probe_kernel(const float* x, float* fma_out, float* mufu_out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    fma_out[i] = hd::exp2_fma(x[i]);
    mufu_out[i] = hd::ex2(x[i]);
  }
}

extern "C" int exp2_probe(const float* x, float* fma_out, float* mufu_out, int n) {
  if (n <= 0) return 0;
  exp2_probe_kernel<<<(n + 255) / 256, 256>>>(x, fma_out, mufu_out, n);
  return static_cast<int>(cudaDeviceSynchronize());
}
