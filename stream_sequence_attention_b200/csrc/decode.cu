// Decode against the per-stream KV cache.
//
// ("Hidden Decoding at Scale", "Persistent KV and the KV-mirror Saving": a
// separate KV cache is kept for every stream; "Inference Throughput": the n
// streams of a token are processed together in one pass.)
//
// For sequence b with T = ctx_len[b] tokens per stream, the stream-s query of
// the new token T-1 sees
//   intra: (j, s)  for j <= T-1               (and T-1-j < W, tokens)
//   cross: (j, s') with p' = j*n + s' <= p = (T-1)*n + s  (and p-p' < W)
// i.e. exactly the prefill row of position p.
//
// Under stream parallelism a rank's cache holds only nc of the n streams,
// local stream l being global stream soff + sstride*l; in cross mode the
// kernel then returns each query's softmax over the visible keys of those
// streams (O = 0 and lse = -inf where there are none), to be merged across
// ranks.  The whole cache is the case nc = n, soff = 0, sstride = 1.
//
// The step is HBM-bound (each cached K/V byte is read once per step), so the
// design is about streaming: a work unit is one KV head of one sequence
// (cross: all n*G query rows that share it -- the cache is read once and
// reused by every stream's queries; intra: the G query rows of one stream),
// its token range is split across CTAs, and each CTA streams 64-token K/V
// tiles through a 3-stage TMA pipeline (one producer warp) into the compute
// warps: four per 16 query rows, each taking 16 keys of every tile, running
// QK^T and PV on the warp-level tensor-core MMA (m16n8k16 bf16 -> f32) with
// an online softmax that only rescales O when the row max rises by more than
// 2^8.  The four warps' partial (max, sum, O) are merged in shared memory and
// written to the workspace, and a small combine kernel merges the splits.
#include <cstdlib>
#include <cstring>

#include "hd_common.cuh"
#include "hd_launch.h"

namespace hd {

namespace dec {
constexpr int kTok = 64;        // tokens per K/V tile
constexpr int kStages = 3;
constexpr int kRowsMax = 32;    // query rows per unit
constexpr int kBox = kTok * 128;        // one 64-token x 128-byte TMA box
constexpr int kD = 128;
constexpr int kHalf = kD / 64;          // boxes per row
constexpr int kStageBytes = 2 * kHalf * kBox;  // K + V
constexpr int kQPitch = kD + 8;         // bf16 elements per padded Q row
constexpr int kQBytes = kRowsMax * kQPitch * 2;
constexpr int kStageOff = 0;
constexpr int kQOff = kStages * kStageBytes;
constexpr int kBarOff = kQOff + kQBytes;
constexpr int kBytes = kBarOff + 2 * kStages * 8 + 16;
constexpr int kAlloc = kBytes + 1024;
static_assert(4 * kRowsMax * kD * 4 + 2 * 4 * kRowsMax * 4 <= kStages * kStageBytes,
              "combine scratch must fit in the stage buffers");
}  // namespace dec

struct DecParams {
  const __nv_bfloat16* q;
  const int32_t* ctx;
  float* ws_o;    // [nsplit][rows_total][D]
  float* ws_lse;  // [nsplit][rows_total], log2 units
  int32_t* status;
  int B, n, Lmax, Hq, Hkv, W, cross, nsplit, rg_count;
  int nc, soff, sstride;  // cache streams and their global stream ids
  // Test hook (environment HD_TEST_STALL_DECODE=1): the producer of CTA
  // (0, 0) issues no loads, so its compute warps' waits run out and the
  // kernel must take its timeout path.  0 in normal use.
  int stall_first;
  float scale_log2;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Address of the 16-byte chunk `chunk` of row `row` inside a 128B-swizzled
// TMA box (rows of 128 bytes, chunk index XOR row mod 8).
__device__ __forceinline__ uint32_t sw128(uint32_t box, int row, int chunk) {
  return box + row * 128 + ((chunk ^ (row & 7)) << 4);
}

struct DecUnit {
  int b, s, kvh, r0, R;  // rows [r0, r0+R) of the unit's row space
};

__device__ __forceinline__ DecUnit dec_unit(int u, const DecParams& p) {
  DecUnit x;
  const int G = p.Hq / p.Hkv;
  const int rg = u % p.rg_count;
  u /= p.rg_count;
  x.kvh = u % p.Hkv;
  u /= p.Hkv;
  if (p.cross) {
    x.s = 0;
    x.b = u;
  } else {
    x.s = u % p.n;
    x.b = u / p.n;
  }
  const int rows = p.cross ? p.n * G : G;
  x.r0 = rg * dec::kRowsMax;
  x.R = min(dec::kRowsMax, rows - x.r0);
  return x;
}

// Unit row r (0-based within the unit's row space) -> (stream, head).
__device__ __forceinline__ void dec_row(const DecUnit& x, const DecParams& p, int r, int& s, int& h) {
  const int G = p.Hq / p.Hkv;
  if (p.cross) {
    s = r / G;
    h = x.kvh * G + (r - s * G);
  } else {
    s = x.s;
    h = x.kvh * G + r;
  }
}

// Compute warps per CTA: one 16-row m-tile per group of four warps; the four
// warps of a group split every 64-key tile into 16-key quarters.
template <int MT>
struct DecShape {
  static constexpr int kCompute = 4 * MT;
  static constexpr int kThreads = 32 * (kCompute + 1);
};

#ifndef HD_DEC_MT2_CTAS
#define HD_DEC_MT2_CTAS 2
#endif
template <int MT>
__global__ void __launch_bounds__(DecShape<MT>::kThreads, MT == 2 ? HD_DEC_MT2_CTAS : 2)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DecParams p) {
  using namespace dec;
  constexpr int kCompute = DecShape<MT>::kCompute;
  constexpr int kThr = DecShape<MT>::kThreads;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t full0 = sbase + kBarOff, empty0 = full0 + kStages * 8;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kBarOff + 2 * kStages * 8);
  volatile int* no_abort = abort_flag + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const DecUnit x = dec_unit(blockIdx.y, p);
  const int split = blockIdx.x;
  const int rows_total = p.B * p.n * p.Hq;

  // Token range of this split.
  const int T = __ldg(p.ctx + x.b);
  const bool bad_T = T < 1 || T > p.Lmax;
  int jlo = 0;
  if (!bad_T && p.W > 0) {
    jlo = p.cross ? ((T - 1) * p.n - p.W + 1) / p.n : T - p.W;  // conservative for cross
    if (jlo < 0) jlo = 0;
  }
  const int base = jlo & ~(kTok - 1);
  const int span = bad_T ? 0 : T - base;
  const int chunk = ((span + p.nsplit - 1) / p.nsplit + kTok - 1) & ~(kTok - 1);
  const int c_lo = base + split * chunk;
  const int c_hi = bad_T ? c_lo : min(T, c_lo + chunk);
  const int ntok_tiles = c_hi > c_lo ? (c_hi - c_lo + kTok - 1) / kTok : 0;
  const int nstreams = p.cross ? p.nc : 1;
  const int ntiles = ntok_tiles * nstreams;

  if (threadIdx.x == 0) {
    if (bad_T && split == 0) report(p.status, HD_ERR_INVALID_ARG);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, kCompute);
    }
    *abort_flag = 0;
    *no_abort = 0;
    fence_barrier_init();
  }
  // Q rows -> padded shared tile (rows >= R are zero).
  {
    __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(smem + kQOff);
    for (int e = threadIdx.x; e < MT * 16 * (kD / 8); e += kThr) {
      const int r = e / (kD / 8), c8 = e - r * (kD / 8);
      uint4 val = make_uint4(0, 0, 0, 0);
      if (r < x.R) {
        int s, h;
        dec_row(x, p, x.r0 + r, s, h);
        val = reinterpret_cast<const uint4*>(p.q + ((static_cast<int64_t>(x.b) * p.n + s) * p.Hq + h) * kD)[c8];
      }
      *reinterpret_cast<uint4*>(qs + r * kQPitch + c8 * 8) = val;
    }
  }
  __syncthreads();

  if (warp == kCompute) {
    if (lane == 0 && ntiles > 0 && !(p.stall_first && blockIdx.x == 0 && blockIdx.y == 0)) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int issued[kStages] = {};
      bool ok = true;
      for (int t = 0; t < ntiles; ++t) {
        const int st = t % kStages;
        if (!mbar_wait(empty0 + 8 * st, ((t / kStages) & 1) ^ 1, abort_flag)) { ok = false; break; }
        const int sp = p.cross ? t / ntok_tiles : x.s;
        const int j0 = c_lo + (p.cross ? t % ntok_tiles : t) * kTok;
        const uint32_t sb = sbase + kStageOff + st * kStageBytes;
        mbar_arrive_expect_tx(full0 + 8 * st, kStageBytes);
#pragma unroll
        for (int hh = 0; hh < kHalf; ++hh) {
          tma_load_5d(sb + hh * kBox, &tmK, full0 + 8 * st, hh * 64, x.kvh, j0, sp, x.b);
          tma_load_5d(sb + (kHalf + hh) * kBox, &tmV, full0 + 8 * st, hh * 64, x.kvh, j0, sp, x.b);
        }
        ++issued[st];
      }
      if (!ok) {
        *abort_flag = 1;
        report(p.status, HD_ERR_TIMEOUT);
        for (int i = 0; i < kStages; ++i)
          if (issued[i]) mbar_wait(full0 + 8 * i, (issued[i] - 1) & 1, no_abort);
      }
    }
    __syncthreads();  // matches the compute warps' final barrier
    return;
  }

  // ------------------------------------------------------ compute warps
  const int mt = warp >> 2;        // this warp's 16-row m-tile
  const int kq = warp & 3;         // this warp's key quarter of every tile
  const int kw = kq * 16;
  const int g = lane >> 2, tq = lane & 3;
  const uint32_t qs = sbase + kQOff;
  float o[kD / 8][4];
#pragma unroll
  for (int nt = 0; nt < kD / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
  // Running max (log2 units) and sum of the two rows this thread holds.  The
  // max is only raised when a tile exceeds it by more than 2^8, so O is
  // rarely rescaled; any reference max gives the same final O / l.
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  int srow[2];
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int r = mt * 16 + g + hh * 8;
    int s, h;
    dec_row(x, p, x.r0 + min(r, x.R - 1), s, h);
    srow[hh] = s;
  }

  bool ok = true;
  for (int t = 0; t < ntiles; ++t) {
    const int st = t % kStages;
    const bool got = mbar_wait(full0 + 8 * st, (t / kStages) & 1, abort_flag);
    if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
    const int sp = p.cross ? t / ntok_tiles : x.s;
    const int j0 = c_lo + (p.cross ? t % ntok_tiles : t) * kTok;
    const uint32_t kbox = sbase + kStageOff + st * kStageBytes;
    const uint32_t vbox = kbox + kHalf * kBox;

    // S = Q K^T for this warp's 16 rows x 16 keys.
    float sc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < kD / 16; ++kk) {
      const int mi = lane >> 3, rr = lane & 7;
      uint32_t b0, b1, b2, b3, a0, a1, a2, a3;
      {
        const int key = kw + rr + ((mi >> 1) << 3);
        const int ch = (kk & 3) * 2 + (mi & 1);
        ldsm_x4(sw128(kbox + (kk >> 2) * kBox, key, ch), b0, b1, b2, b3);
      }
      {
        const int row = mt * 16 + rr + ((mi & 1) << 3);
        const int col = kk * 16 + ((mi >> 1) << 3);
        ldsm_x4(qs + (row * kQPitch + col) * 2, a0, a1, a2, a3);
      }
      mma_bf16_16816(sc[0], a0, a1, a2, a3, b0, b1);
      mma_bf16_16816(sc[1], a0, a1, a2, a3, b2, b3);
    }

    // Scale, mask, online softmax with lazy rescaling.
    const bool edge = (j0 + kTok > T - 1) || (p.W > 0);
    uint32_t pa[4];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      float mx = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float y = sc[nt][hh * 2 + e] * p.scale_log2;
          if (edge) {
            const int j = j0 + kw + nt * 8 + tq * 2 + e;
            bool vis;
            if (p.cross) {
              const int64_t pq = static_cast<int64_t>(T - 1) * p.n + srow[hh];
              const int64_t pk = static_cast<int64_t>(j) * p.n + (p.soff + p.sstride * sp);
              vis = pk <= pq && (p.W <= 0 || pq - pk < p.W);
            } else {
              vis = j <= T - 1 && (p.W <= 0 || T - 1 - j < p.W);
            }
            if (!vis) y = -INFINITY;
          }
          sc[nt][hh * 2 + e] = y;
          mx = fmaxf(mx, y);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      if (mx > mrow[hh] + 8.0f) {  // uniform across the quad holding the row
        const float alpha = ex2(mrow[hh] - mx);  // mrow = -inf -> 0
        lrow[hh] *= alpha;
#pragma unroll
        for (int nt = 0; nt < kD / 8; ++nt) {
          o[nt][hh * 2 + 0] *= alpha;
          o[nt][hh * 2 + 1] *= alpha;
        }
        mrow[hh] = mx;
      }
      const float mu = (mrow[hh] == -INFINITY) ? 0.f : mrow[hh];
      float ls = 0.f;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float pv = ex2(sc[nt][hh * 2 + e] - mu);
          sc[nt][hh * 2 + e] = pv;
          ls += pv;
        }
      lrow[hh] += ls;
    }
    pa[0] = pack_bf16x2(sc[0][0], sc[0][1]);
    pa[1] = pack_bf16x2(sc[0][2], sc[0][3]);
    pa[2] = pack_bf16x2(sc[1][0], sc[1][1]);
    pa[3] = pack_bf16x2(sc[1][2], sc[1][3]);

    // O += P V.
#pragma unroll
    for (int c = 0; c < kD / 16; ++c) {
      uint32_t b0, b1, b2, b3;
      const int mi = lane >> 3, rr = lane & 7;
      const int key = kw + rr + ((mi & 1) << 3);
      const int ch = ((2 * c) & 7) + (mi >> 1);
      ldsm_x4_t(sw128(vbox + (c >> 2) * kBox, key, ch), b0, b1, b2, b3);
      mma_bf16_16816(o[2 * c], pa[0], pa[1], pa[2], pa[3], b0, b1);
      mma_bf16_16816(o[2 * c + 1], pa[0], pa[1], pa[2], pa[3], b2, b3);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * st);
  }
  if (!ok) {
    *abort_flag = 1;
    report(p.status, HD_ERR_TIMEOUT);
  }

  // Quad-reduce the row sums.
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    float l = lrow[hh];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    lrow[hh] = l;
  }

  // Merge the four key quarters of each m-tile through shared memory (the
  // stage buffers are idle now).
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kCompute) : "memory");
  float* so = reinterpret_cast<float*>(smem + kStageOff);  // [4 quarters][32 rows][D]
  float* sm = so + 4 * kRowsMax * kD;                      // [4][32]
  float* sl = sm + 4 * kRowsMax;                           // [4][32]
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int r = mt * 16 + g + hh * 8;
    if (tq == 0) {
      sm[kq * kRowsMax + r] = mrow[hh];
      sl[kq * kRowsMax + r] = lrow[hh];
    }
#pragma unroll
    for (int nt = 0; nt < kD / 8; ++nt) {
      float2 v2 = make_float2(o[nt][hh * 2], o[nt][hh * 2 + 1]);
      *reinterpret_cast<float2*>(so + (kq * kRowsMax + r) * kD + nt * 8 + tq * 2) = v2;
    }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kCompute) : "memory");
  {
    const int tid = threadIdx.x;   // 0 .. 32*kCompute-1
    const int r = tid >> 3;        // 16*MT rows, 8 threads per row
    const int d0 = (tid & 7) * (kD / 8);
    if (r < x.R) {
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < 4; ++w) M = fmaxf(M, sm[w * kRowsMax + r]);
      float wgt[4], L = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = sm[w * kRowsMax + r];
        wgt[w] = (mw == -INFINITY) ? 0.f : ex2(mw - M);
        L += wgt[w] * sl[w * kRowsMax + r];
      }
      int s, h;
      dec_row(x, p, x.r0 + r, s, h);
      const int64_t row = (static_cast<int64_t>(x.b) * p.n + s) * p.Hq + h;
      float* dst = p.ws_o + (static_cast<int64_t>(split) * rows_total + row) * kD + d0;
      const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
      for (int d = 0; d < kD / 8; d += 4) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float4 v4 = *reinterpret_cast<const float4*>(so + (w * kRowsMax + r) * kD + d0 + d);
          acc.x += wgt[w] * v4.x;
          acc.y += wgt[w] * v4.y;
          acc.z += wgt[w] * v4.z;
          acc.w += wgt[w] * v4.w;
        }
        acc.x *= inv;
        acc.y *= inv;
        acc.z *= inv;
        acc.w *= inv;
        *reinterpret_cast<float4*>(dst + d) = acc;
      }
      if ((tid & 7) == 0)
        p.ws_lse[static_cast<int64_t>(split) * rows_total + row] = L > 0.f ? M + __log2f(L) : -INFINITY;
    }
  }
  __syncthreads();
}

// One warp per output row: merge the split partials.
__global__ void decode_combine_kernel(const float* __restrict__ ws_o, const float* __restrict__ ws_lse,
                                      void* __restrict__ o, float* __restrict__ lse, int rows, int nsplit,
                                      int out_bf16) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, ws_lse[static_cast<int64_t>(s) * rows + warp]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < nsplit; ++s) {
      const float ls = ws_lse[static_cast<int64_t>(s) * rows + warp];
      if (ls == -INFINITY) continue;
      const float w = ex2(ls - M);
      L += w;
      const float4 v = reinterpret_cast<const float4*>(ws_o + (static_cast<int64_t>(s) * rows + warp) * dec::kD)[lane];
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
    const float inv = 1.f / L;
    acc.x *= inv;
    acc.y *= inv;
    acc.z *= inv;
    acc.w *= inv;
  }
  if (out_bf16) {
    uint2 w2;
    w2.x = pack_bf16x2(acc.x, acc.y);
    w2.y = pack_bf16x2(acc.z, acc.w);
    reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(o) + static_cast<int64_t>(warp) * dec::kD)[lane] = w2;
  } else {
    reinterpret_cast<float4*>(static_cast<float*>(o) + static_cast<int64_t>(warp) * dec::kD)[lane] = acc;
  }
  if (lse && lane == 0)
    lse[warp] = (M == -INFINITY) ? -INFINITY : (M + log2f(L)) * 0.69314718055994531f;
}

// One warp per row: merge R partial results over disjoint key sets (stream
// parallelism: each rank's softmax over its own streams' keys).  o_parts
// [R][rows][D] normalised within their part, lse_parts [R][rows] natural
// log, -inf for a part with no visible key:
//   O = sum_r e^(lse_r - M) O_r / sum_r e^(lse_r - M),  LSE = M + log sum_r e^(lse_r - M).
template <bool IN_BF16>
__global__ void attn_combine_kernel(const void* __restrict__ o_parts, const float* __restrict__ lse_parts,
                                    void* __restrict__ o, float* __restrict__ lse, int R, int64_t rows, int D,
                                    int out_bf16) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  float M = -INFINITY;
  for (int r = 0; r < R; ++r) M = fmaxf(M, lse_parts[r * rows + row]);
  float L = 0.f;
  if (M != -INFINITY)
    for (int r = 0; r < R; ++r) L += expf(lse_parts[r * rows + row] - M);  // exp(-inf) = 0
  const float inv = L > 0.f ? 1.f / L : 0.f;
  for (int c = lane; c < D / 4; c += 32) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (M != -INFINITY) {
      for (int r = 0; r < R; ++r) {
        const float lr = lse_parts[r * rows + row];
        if (lr == -INFINITY) continue;
        const float w = expf(lr - M) * inv;
        const int64_t off = (r * rows + row) * D + 4 * c;
        float4 v;
        if (IN_BF16) {
          const uint2 u = *reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(o_parts) + off);
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
          const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
          v = make_float4(a.x, a.y, b.x, b.y);
        } else {
          v = *reinterpret_cast<const float4*>(static_cast<const float*>(o_parts) + off);
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

cudaError_t launch_attn_combine(const void* o_parts, const float* lse_parts, void* o, float* lse, int R,
                                int64_t rows, int D, bool in_bf16, bool out_bf16, cudaStream_t st) {
  if (rows == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (rows * 32 + threads - 1) / threads;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  if (in_bf16)
    attn_combine_kernel<true><<<static_cast<unsigned>(blocks), threads, 0, st>>>(o_parts, lse_parts, o, lse, R, rows,
                                                                                 D, out_bf16 ? 1 : 0);
  else
    attn_combine_kernel<false><<<static_cast<unsigned>(blocks), threads, 0, st>>>(o_parts, lse_parts, o, lse, R,
                                                                                  rows, D, out_bf16 ? 1 : 0);
  return cudaGetLastError();
}

// ------------------------------------------------------------------- host


// (D, Hkv, Lmax, n, B) view of the [B, n, Lmax, Hkv, D] cache; box 64 x 1 x 64 x 1 x 1.
static bool make_cache_view(const TmapKey& k, CUtensorMap* m) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  const cuuint64_t B = k.dims[0], n = k.dims[1], Lmax = k.dims[2], Hkv = k.dims[3];
  const cuuint64_t D = dec::kD, e = 2;
  const cuuint64_t dims[5] = {D, Hkv, Lmax, n, B};
  const cuuint64_t strides[4] = {D * e, Hkv * D * e, Lmax * Hkv * D * e, n * Lmax * Hkv * D * e};
  const cuuint32_t box[5] = {64, 1, (cuuint32_t)dec::kTok, 1, 1};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(k.ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool encode_cache_view(CUtensorMap* m, const void* ptr, int B, int n, int Lmax, int Hkv) {
  TmapKey k;
  std::memset(&k, 0, sizeof(k));
  k.ptr = ptr;
  k.dims[0] = B;
  k.dims[1] = n;
  k.dims[2] = Lmax;
  k.dims[3] = Hkv;
  k.kind = 2;
  return tmap_cached(k, m, make_cache_view);
}

DecPlan decode_plan(int B, int n, int Lmax, int Hq, int Hkv, bool cross, int sms) {
  DecPlan pl;
  const int G = Hq / Hkv;
  const int rows = cross ? n * G : G;
  pl.rg_count = (rows + dec::kRowsMax - 1) / dec::kRowsMax;
  pl.units = (cross ? B * Hkv : B * n * Hkv) * pl.rg_count;
  const int per_unit_rows = rows < dec::kRowsMax ? rows : dec::kRowsMax;
  pl.mt = per_unit_rows > 16 ? 2 : 1;
  // Enough CTAs for ~8 waves of 2 CTAs per SM, at least one 64-token tile each.
  const int64_t target = static_cast<int64_t>(sms) * 2 * 8;
  int64_t ns = (target + pl.units - 1) / pl.units;
  const int64_t max_ns = (Lmax + dec::kTok - 1) / dec::kTok;
  if (ns > max_ns) ns = max_ns;
  if (ns < 1) ns = 1;
  pl.nsplit = static_cast<int>(ns);
  pl.rows_total = static_cast<int64_t>(B) * n * Hq;
  return pl;
}

size_t decode_workspace_bytes(const DecPlan& pl) {
  const size_t o = static_cast<size_t>(pl.nsplit) * pl.rows_total * dec::kD * sizeof(float);
  const size_t l = static_cast<size_t>(pl.nsplit) * pl.rows_total * sizeof(float);
  return ((o + 255) & ~static_cast<size_t>(255)) + ((l + 255) & ~static_cast<size_t>(255));
}

cudaError_t launch_decode(const void* q, const void* kc, const void* vc, const int32_t* ctx, void* o,
                          float* lse, int B, int n, int Lmax, int Hq, int Hkv, int W, float scale,
                          bool cross, bool out_bf16, void* ws, int32_t* status, int sms, cudaStream_t st,
                          int nc, int soff, int sstride) {
  const DecPlan pl = decode_plan(B, n, Lmax, Hq, Hkv, cross, sms);
  if (nc <= 0) nc = n;
#ifndef HD_DECODE_CROSS_TC
#define HD_DECODE_CROSS_TC 1
#endif
  if (HD_DECODE_CROSS_TC && decode_tc_supported(n, Hq, Hkv, dec::kD, cross)) {
    // Cross mode on the tensor-core kernel; its split count stays within the
    // plan the workspace was sized for.
    const size_t o_bytes = static_cast<size_t>(pl.nsplit) * pl.rows_total * dec::kD * sizeof(float);
    float* ws_o = static_cast<float*>(ws);
    float* ws_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ((o_bytes + 255) & ~static_cast<size_t>(255)));
    const int ns = decode_tc_nsplit(pl.units, Lmax, pl.nsplit, sms);
    cudaError_t err = launch_decode_tc(q, kc, vc, ctx, ws_o, ws_lse, B, n, Lmax, Hq, Hkv, W, scale, ns, status, st,
                                       nc, soff, sstride);
    if (err != cudaSuccess) return err;
    const int rows = static_cast<int>(pl.rows_total);
    const int threads = 256;
    const int blocks = (rows * 32 + threads - 1) / threads;
    decode_combine_kernel<<<blocks, threads, 0, st>>>(ws_o, ws_lse, o, lse, rows, ns, out_bf16 ? 1 : 0);
    return cudaGetLastError();
  }
  CUtensorMap mk, mv;
  if (!encode_cache_view(&mk, kc, B, nc, Lmax, Hkv) || !encode_cache_view(&mv, vc, B, nc, Lmax, Hkv))
    return cudaErrorInvalidValue;
  DecParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.ctx = ctx;
  const size_t o_bytes = static_cast<size_t>(pl.nsplit) * pl.rows_total * dec::kD * sizeof(float);
  p.ws_o = static_cast<float*>(ws);
  p.ws_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + ((o_bytes + 255) & ~static_cast<size_t>(255)));
  p.status = status;
  p.B = B;
  p.n = n;
  p.nc = nc;
  p.soff = soff;
  p.sstride = sstride;
  p.Lmax = Lmax;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.W = W;
  p.cross = cross ? 1 : 0;
  p.nsplit = pl.nsplit;
  p.rg_count = pl.rg_count;
  p.scale_log2 = scale * 1.4426950408889634f;
  static const int stall = [] {
    const char* e = getenv("HD_TEST_STALL_DECODE");
    return (e && e[0] == '1') ? 1 : 0;
  }();
  p.stall_first = stall;
  if (pl.units > 65535) return cudaErrorInvalidValue;
  dim3 grid(pl.nsplit, pl.units);
  cudaError_t err;
  if (pl.mt == 2) {
    err = cudaFuncSetAttribute(decode_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kAlloc);
    if (err != cudaSuccess) return err;
    decode_kernel<2><<<grid, DecShape<2>::kThreads, dec::kAlloc, st>>>(mk, mv, p);
  } else {
    err = cudaFuncSetAttribute(decode_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kAlloc);
    if (err != cudaSuccess) return err;
    decode_kernel<1><<<grid, DecShape<1>::kThreads, dec::kAlloc, st>>>(mk, mv, p);
  }
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int rows = static_cast<int>(pl.rows_total);
  const int threads = 256;
  const int blocks = (rows * 32 + threads - 1) / threads;
  decode_combine_kernel<<<blocks, threads, 0, st>>>(p.ws_o, p.ws_lse, o, lse, rows, pl.nsplit, out_bf16 ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace hd
