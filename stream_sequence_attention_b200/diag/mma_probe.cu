// Diagnostic probe (not part of the library): cycles per tcgen05.mma step for
// the issue patterns of the attention kernels.  One CTA per SM; warp 0 issues
// M = N = 128, K = 16 bf16 MMAs (shared-memory operands are left
// uninitialised: only the timing is used), one elected lane per MMA, as the
// kernels do.  Patterns:
//  0: 128 SS MMAs (M=N=128, K=16) into one accumulator, one commit at the end
//  1: 16 bursts of [8 SS MMAs; commit]                      (commit after every burst)
//  2: 16 bursts of [8 TS MMAs (A from TMEM); commit]
//  3: 8 x [8 TS (acc0); 8 SS (acc1); commit; 8 TS (acc2); 8 SS (acc3); commit]  (forward's order, 2 heads)
//  4: pattern 3 with a wait on each commit's mbarrier before the next group (fully serialized)
// Built and run by stream_sequence_attention_b200/diag_mma.py.
#include "hd_common.cuh"

using namespace hd;

__global__ void __launch_bounds__(128, 1) mma_probe(int pattern, unsigned long long* out) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint32_t slot;
  __shared__ __align__(8) uint64_t mbar[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) { mbar_init(smem_u32(&mbar[0]), 1); mbar_init(smem_u32(&mbar[1]), 1); fence_barrier_init(); }
  if (warp == 0) { tmem_alloc(smem_u32(&slot), 512); tmem_relinquish(); }
  tc_fence_before(); __syncthreads(); tc_fence_after();
  const uint32_t tmem = slot;
  const uint32_t sb = smem_u32(smem);
  constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);
  constexpr uint32_t idO = idesc_bf16_f32(128, 128, false, true);
  const uint64_t ad = smem_desc_sw128(sb, 16, 1024), bd = smem_desc_sw128(sb + 32768, 16, 1024);
  const uint64_t vd = smem_desc_sw128(sb + 65536, 16384, 1024);
  volatile int noab = 0;
  if (warp == 0) {
    auto burst_ss = [&](uint32_t acc) {
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off16 = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
        mma_ss_elect(tmem + acc, ad + off16, bd + off16, idS, kk > 0);
      }
    };
    auto burst_ts = [&](uint32_t acc, uint32_t a) {
      for (int kk = 0; kk < 8; ++kk) mma_ts_elect(tmem + acc, tmem + a + kk * 8, vd + ((kk * 2048) >> 4), idO, kk > 0);
    };
    // warm up
    burst_ss(0);
    tc_commit_elect(smem_u32(&mbar[0]));
    mbar_wait(smem_u32(&mbar[0]), 0, &noab);
    const long long t0 = clock64();
    int n = 0;
    if (pattern == 0) {
      for (int i = 0; i < 16; ++i) { burst_ss(0); n += 8; }
      tc_commit_elect(smem_u32(&mbar[1]));
      mbar_wait(smem_u32(&mbar[1]), 0, &noab);
    } else if (pattern == 1 || pattern == 2) {
      for (int i = 0; i < 16; ++i) {
        if (pattern == 1) burst_ss(0); else burst_ts(256, 0);
        n += 8;
        tc_commit_elect(smem_u32(&mbar[1]));
      }
      tc_commit_elect(smem_u32(&mbar[0]));
      mbar_wait(smem_u32(&mbar[0]), 1, &noab);
    } else {
      int c = 0;
      for (int i = 0; i < 8; ++i) {
        burst_ts(256, 0); burst_ss(0); n += 16;
        tc_commit_elect(smem_u32(&mbar[1]));
        if (pattern == 4) { mbar_wait(smem_u32(&mbar[1]), c & 1, &noab); }
        ++c;
        burst_ts(384, 128); burst_ss(128); n += 16;
        tc_commit_elect(smem_u32(&mbar[1]));
        if (pattern == 4) { mbar_wait(smem_u32(&mbar[1]), c & 1, &noab); }
        ++c;
      }
      if (pattern == 3) {
        tc_commit_elect(smem_u32(&mbar[0]));
        mbar_wait(smem_u32(&mbar[0]), 1, &noab);
      }
    }
    const long long t1 = clock64();
    if (lane == 0) { out[blockIdx.x * 2] = t1 - t0; out[blockIdx.x * 2 + 1] = n; }
  }
  tc_fence_before(); __syncthreads(); tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// host: ctas x {cycles, MMAs}.
extern "C" int run_mma(int pattern, int ctas, unsigned long long* host) {
  if (pattern < 0 || pattern > 4 || ctas < 1 || ctas > 1024) return -1;
  unsigned long long* d = nullptr;
  if (cudaMalloc(&d, static_cast<size_t>(ctas) * 2 * 8) != cudaSuccess) return -2;
  cudaMemset(d, 0, static_cast<size_t>(ctas) * 2 * 8);
  const int smem = 96 * 1024 + 1024;
  cudaFuncSetAttribute(mma_probe, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  mma_probe<<<ctas, 128, smem>>>(pattern, d);
  int e = static_cast<int>(cudaDeviceSynchronize());
  cudaMemcpy(host, d, static_cast<size_t>(ctas) * 2 * 8, cudaMemcpyDeviceToHost);
  cudaFree(d);
  return e;
}
