// Cross-stream decode on the 5th-generation tensor cores (tcgen05 + tensor
// memory) of sm_100a.
//
// ("Hidden Decoding at Scale", "Persistent KV and the KV-mirror Saving" and
// "Inference Throughput": the n stream queries of a new token read every
// stream's cache.)  In cross mode the n*G query rows of one KV head (n
// streams x G heads of the group) share every cached key, so a unit is one
// (sequence, KV head) with its rows -- up to 32 per unit, more rows making
// more row groups -- and its token range is split across CTAs as in the
// warp-MMA kernel; the partial results go to the same workspace and the same
// split-merge kernel.
//
// Each cached K/V byte is read once per step, so the kernel is meant to run
// at the HBM rate.  The warp-level MMA form reads every K, V and Q fragment
// through shared memory once per 16-row m-tile (three times the tile's
// bytes per tile); here the tensor core reads its operands from shared
// memory itself, with the keys as the MMA's M dimension:
//   S^T [128 keys x 32 rows] = K [128 x D] . Q^T        (tensor memory)
//   O^T [D x 32 rows]       += V^T [D x 128] . P^T      (tensor memory)
// V^T is the V tile as TMA wrote it, read as an MN-major operand; P^T is
// written by the softmax warps as a K-major [32 rows x 128 keys] tile.
//
// CTA = 10 warps, one CTA per SM:
//   warps 0-3  softmax warpgroup 0: the even tiles; then the epilogue
//   warps 4-7  softmax warpgroup 1: the odd tiles
//   warp 8     TMA producer: 128-token K and V tiles, 3 stages
//   warp 9     MMA issuer: S(t+1) is issued before P V(t), so the tensor core
//              computes the next scores while a warpgroup works
// A softmax thread owns one key lane of S^T (warp w reads tensor-memory lanes
// 32*(w mod 4)...).  Each warpgroup keeps its own running max m, row sums l
// and accumulator O_g^T, so the two never wait for one another; the
// epilogue merges the two (m, l, O) like two splits.
// Tensor memory: S_g^T in columns [32g, 32g + 32), O_g^T in [64 + 32g, ...).
//
// Softmax of a tile: the row maxima of each warp's 32 keys by a warp
// reduction, exchanged between the four warps of the warpgroup through
// shared memory and an mbarrier.  The running max of a row only moves when
// the tile exceeds it by more than 2^8 -- rare after the first tile, and
// detected with one vote -- and then O_g^T's columns and the row sums are
// rescaled; the final O / l does not depend on which max was used.  Row sums
// are kept per thread (its key lanes) and reduced once at the end.
#include <cstdlib>
#include <cstring>

#include "hd_common.cuh"
#include "hd_launch.h"

namespace hd {

namespace dtc {
constexpr int kTok = 128;                // keys per tile (MMA M)
constexpr int kN = 32;                   // query rows per unit, padded (MMA N)
constexpr int kD = 128;
constexpr int kStages = 3;
constexpr int kThreads = 320;
constexpr int kWarpTMA = 8;
constexpr int kWarpMMA = 9;
constexpr uint32_t kTmemCols = 128;
constexpr int kBlk = kTok * 128;         // one 64-feature column block of a K/V tile
constexpr int kTile = 2 * kBlk;          // a K or V tile (D = 128)
constexpr int kRBlk = kN * 128;          // one 64-wide column block of Q or P (32 rows)
constexpr int K_OFF = 0;
constexpr int V_OFF = K_OFF + kStages * kTile;
constexpr int Q_OFF = V_OFF + kStages * kTile;
constexpr int P_OFF = Q_OFF + 2 * kRBlk;            // one P^T tile per warpgroup
constexpr int MX_OFF = P_OFF + 2 * 2 * kRBlk;       // [2 groups][4 warps][32 rows] float
constexpr int LS_OFF = MX_OFF + 2 * 4 * kN * 4;     // [2 groups][4 warps][32 rows] float
constexpr int ML_OFF = LS_OFF + 2 * 4 * kN * 4;     // [2 groups][32 rows] float (running max)
constexpr int BAR_OFF = ML_OFF + 2 * kN * 4;
// B_EMPTY: a stage's K half is free (S of its tile done); B_VEMPTY: its V
// half is free (P V done).  With HD_DTC_SPLIT_EMPTY=0 both halves wait for P V.
#ifndef HD_DTC_SPLIT_EMPTY
#define HD_DTC_SPLIT_EMPTY 1
#endif
constexpr int B_KFULL = 0, B_VFULL = B_KFULL + kStages, B_EMPTY = B_VFULL + kStages, B_VEMPTY = B_EMPTY + kStages,
              B_QFULL = B_VEMPTY + kStages,
              B_SFULL = B_QFULL + 1, B_PFULL = B_SFULL + 2, B_PVDONE = B_PFULL + 2, B_MX = B_PVDONE + 2,
              B_LS = B_MX + 2, B_DRAIN = B_LS + 1, NBAR = B_DRAIN + 1;
constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
constexpr int kBytes = MISC_OFF + 16;
constexpr int kAlloc = kBytes + 1024;
static_assert(kAlloc <= 227 * 1024, "shared memory");
}  // namespace dtc

struct DtcParams {
  const __nv_bfloat16* q;
  const int32_t* ctx;
  float* ws_o;    // [nsplit][rows_total][D]
  float* ws_lse;  // [nsplit][rows_total], log2 units
  int32_t* status;
  int B, n, Lmax, Hq, Hkv, W, nsplit;
  int nc, soff, sstride;  // cache streams and their global stream ids
  // Test hook (environment HD_TEST_STALL_DECODE=1): the producer of CTA
  // (0, 0) issues no loads, so the other roles' waits run out and the kernel
  // must take its timeout path.  0 in normal use.
  int stall_first;
  float scale_log2;
};

__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

// 32 lanes x 16 consecutive 32-bit columns of tensor memory.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void st_shared_b16(uint32_t addr, __nv_bfloat16 v) {
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(*reinterpret_cast<uint16_t*>(&v)) : "memory");
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__global__ void __launch_bounds__(dtc::kThreads, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const DtcParams p) {
  using namespace dtc;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + BAR_OFF + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + MISC_OFF + 4);
  volatile int* no_abort = reinterpret_cast<volatile int*>(smem + MISC_OFF + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.Hq / p.Hkv;
  // Unit = (sequence, KV head, row group): rows [r0, r0 + R) of the n*G
  // query rows that share the KV head, at most kN per group (each group
  // streams the cache once).
  const int rg_count = (p.n * G + kN - 1) / kN;
  const int rg = blockIdx.y % rg_count;
  const int kvh = (blockIdx.y / rg_count) % p.Hkv;
  const int b = blockIdx.y / rg_count / p.Hkv;
  const int r0 = rg * kN;
  const int R = min(kN, p.n * G - r0);
  const int split = blockIdx.x;
  const int rows_total = p.B * p.n * p.Hq;

  // Token range of this split (tiles of kTok tokens of every cache stream).
  const int T = __ldg(p.ctx + b);
  const bool bad_T = T < 1 || T > p.Lmax;
  int jlo = 0;
  if (!bad_T && p.W > 0) {
    jlo = ((T - 1) * p.n - p.W + 1) / p.n;  // conservative: the mask decides
    if (jlo < 0) jlo = 0;
  }
  const int base = jlo & ~(kTok - 1);
  const int span = bad_T ? 0 : T - base;
  const int chunk = ((span + p.nsplit - 1) / p.nsplit + kTok - 1) & ~(kTok - 1);
  const int c_lo = base + split * chunk;
  const int c_hi = bad_T ? c_lo : min(T, c_lo + chunk);
  const int ntok = c_hi > c_lo ? (c_hi - c_lo + kTok - 1) / kTok : 0;
  const int ntiles = ntok * p.nc;

  if (threadIdx.x == 0) {
    if (bad_T && split == 0) report(p.status, HD_ERR_INVALID_ARG);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar(B_KFULL + i), 1);
      mbar_init(bar(B_VFULL + i), 1);
      mbar_init(bar(B_EMPTY + i), 1);
      mbar_init(bar(B_VEMPTY + i), 1);
    }
    mbar_init(bar(B_QFULL), 256);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_SFULL + i), 1);
      mbar_init(bar(B_PFULL + i), 4);
      mbar_init(bar(B_PVDONE + i), 1);
      mbar_init(bar(B_MX + i), 4);
    }
    mbar_init(bar(B_LS), 8);
    mbar_init(bar(B_DRAIN), 1);
    *abort_flag = 0;
    *no_abort = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMMA) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&]() {
    *abort_flag = 1;
    report(p.status, HD_ERR_TIMEOUT);
  };

  if (warp == kWarpTMA) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && ntiles > 0 && !(p.stall_first && blockIdx.x == 0 && blockIdx.y == 0)) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      int k_issued[kStages] = {}, v_issued[kStages] = {};
      bool ok = true;
      for (int t = 0; t < ntiles; ++t) {
        const int st = t % kStages;
        if (!mbar_wait(bar(B_EMPTY + st), ((t / kStages) & 1) ^ 1, abort_flag)) { ok = false; break; }
        const int sp = t / ntok;
        const int j0 = c_lo + (t - sp * ntok) * kTok;
        mbar_arrive_expect_tx(bar(B_KFULL + st), kTile);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          tma_load_5d(sbase + K_OFF + st * kTile + hh * kBlk, &tmK, bar(B_KFULL + st), hh * 64, kvh, j0, sp, b);
        ++k_issued[st];
        if (HD_DTC_SPLIT_EMPTY &&
            !mbar_wait(bar(B_VEMPTY + st), ((t / kStages) & 1) ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(bar(B_VFULL + st), kTile);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          tma_load_5d(sbase + V_OFF + st * kTile + hh * kBlk, &tmV, bar(B_VFULL + st), hh * 64, kvh, j0, sp, b);
        ++v_issued[st];
      }
      if (!ok) {
        fail();
        for (int i = 0; i < kStages; ++i) {
          if (k_issued[i]) mbar_wait(bar(B_KFULL + i), (k_issued[i] - 1) & 1, no_abort);
          if (v_issued[i]) mbar_wait(bar(B_VFULL + i), (v_issued[i] - 1) & 1, no_abort);
        }
      }
    }
  } else if (warp == kWarpMMA) {
    // ---------------------------------------------------------------- MMA
    // Tile t belongs to warpgroup g = t & 1 (its S^T, P^T and O^T buffers).
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(kTok, kN, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(kD, kN, true, false);
      const uint32_t qbase = sbase + Q_OFF;
      auto issue_S = [&](int t) {
        const uint32_t kbase = sbase + K_OFF + (t % kStages) * kTile;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t ka = kbase + (kk >> 2) * kBlk + (kk & 3) * 32;
          const uint32_t qa = qbase + (kk >> 2) * kRBlk + (kk & 3) * 32;
          mma_ss(tmem + (t & 1) * kN, smem_desc_sw128(ka, 16, 1024), smem_desc_sw128(qa, 16, 1024), idS,
                 kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(B_SFULL + (t & 1)));
        if (HD_DTC_SPLIT_EMPTY) tc_commit(bar(B_EMPTY + t % kStages));
      };
      bool ok = mbar_wait(bar(B_QFULL), 0, abort_flag);
      if (ok && ntiles > 0) {
        if (!mbar_wait(bar(B_KFULL + 0), 0, abort_flag)) {
          ok = false;
        } else {
          tc_fence_after();
          issue_S(0);
        }
      }
      for (int t = 0; ok && t < ntiles; ++t) {
        // S(t+1) overwrites the S^T buffer that softmax(t-1) read; P V(t-1),
        // issued only after P(t-1) was complete, precedes it in issue order.
        if (t + 1 < ntiles) {
          const int s1 = (t + 1) % kStages;
          if (!mbar_wait(bar(B_KFULL + s1), ((t + 1) / kStages) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_S(t + 1);
        }
        const int st = t % kStages;
        const int g = t & 1;
        if (!mbar_wait(bar(B_PFULL + g), (t >> 1) & 1, abort_flag) ||
            !mbar_wait(bar(B_VFULL + st), (t / kStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t vbase = sbase + V_OFF + st * kTile;
        const uint32_t pbase = sbase + P_OFF + g * 2 * kRBlk;
#pragma unroll
        for (int kk = 0; kk < kTok / 16; ++kk) {
          // V^T is MN-major (features contiguous): 16 keys = 16 rows of 128 B.
          const uint64_t adesc = smem_desc_sw128(vbase + kk * 2048, kBlk, 1024);
          const uint64_t bdesc = smem_desc_sw128(pbase + (kk >> 2) * kRBlk + (kk & 3) * 32, 16, 1024);
          mma_ss(tmem + (2 + g) * kN, adesc, bdesc, idO, (t > 1 || kk > 0) ? 1u : 0u);
        }
        tc_commit(bar(B_PVDONE + g));
        tc_commit(bar(HD_DTC_SPLIT_EMPTY ? B_VEMPTY + st : B_EMPTY + st));
      }
      if (!ok) fail();
      tc_commit(bar(B_DRAIN));
      mbar_wait(bar(B_DRAIN), 0, no_abort);
    }
  } else {
    // ---------------------------------------------- softmax + epilogue
    const int g = warp >> 2;          // warpgroup
    const int wq = warp & 3;          // tensor-memory lane quarter
    const int tid = threadIdx.x & 127;
    const uint32_t lane_addr = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t sS = tmem + lane_addr + g * kN;
    const uint32_t sO = tmem + lane_addr + (2 + g) * kN;
    // Q rows -> K-major 128-byte-swizzled [32 rows x 128 features] tile.
    {
      for (int e = threadIdx.x; e < kN * (kD / 8); e += 256) {
        const int r = e >> 4, c = e & 15;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (r < R) {
          const int s = (r0 + r) / G, h = kvh * G + (r0 + r - s * G);
          val = reinterpret_cast<const uint4*>(p.q + ((static_cast<int64_t>(b) * p.n + s) * p.Hq + h) * kD)[c];
        }
        *reinterpret_cast<uint4*>(smem + Q_OFF + (c >> 3) * kRBlk + r * 128 + (((c & 7) ^ (r & 7)) << 4)) = val;
      }
      fence_async_smem();
      mbar_arrive(bar(B_QFULL));
    }
    const int64_t pq_base = static_cast<int64_t>(T - 1) * p.n;
    // Running max m (log2 units) per row, uniform over the warpgroup, kept
    // as nmu = -max(m, -1e30): exp2(s + nmu) stays finite for rows that have
    // seen no key yet (m = -inf), and exp2(-nmu - x) is 0 for them as the
    // rescale factor exp2(m - x) must be.
    float nmu[kN], l[kN];
#pragma unroll
    for (int r = 0; r < kN; ++r) {
      nmu[r] = 1e30f;
      l[r] = 0.f;
    }
    float m_own = -1e30f;  // max(m[lane], -1e30)
    const float sl2 = p.scale_log2;
    const int key = wq * 32 + lane;  // this thread's key lane of every tile
    float* mx_s = reinterpret_cast<float*>(smem + MX_OFF) + g * 4 * kN;
    // Shared address of P^T element (row r, this key): row r at r*128 bytes,
    // 16-byte chunk (key mod 64)/8 XOR (r mod 8) -- eight bases, one per r mod 8.
    uint32_t pa[8];
    {
      const uint32_t pb = sbase + P_OFF + g * 2 * kRBlk + (key >> 6) * kRBlk + (key & 7) * 2;
      const int kc = (key & 63) >> 3;
#pragma unroll
      for (int i = 0; i < 8; ++i) pa[i] = pb + ((kc ^ i) << 4);
    }
    bool ok = true;
    int u = 0;  // this warpgroup's tile count
    for (int t = g; t < ntiles; t += 2, ++u) {
      const int sp = t / ntok;
      const int j0 = c_lo + (t - sp * ntok) * kTok;
      bool got = mbar_wait(bar(B_SFULL + g), u & 1, abort_flag);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[kN];
      tmem_ld32(sS, sv);
      tmem_wait_ld();
      if ((j0 + kTok > T - 1) || (p.W > 0)) {
        // Key p' = j*n + (its global stream) is visible to row r (stream
        // r div G, position (T-1)*n + r div G) iff, with dk = p' - (T-1)*n,
        // dk <= r div G and (W = 0 or r div G - dk < W), i.e. r >= dk*G and
        // (W = 0 or r < (W + dk)*G) for the unit's row r; keys of the next
        // split (j >= c_hi) are not this CTA's.  Rows >= R are padding.
        const int j = j0 + key;
        const int64_t dk = static_cast<int64_t>(j) * p.n + (p.soff + p.sstride * sp) - pq_base;
        // In this group's row numbering r = r' - r0 (all in 64 bits, clamped).
        const int64_t big = static_cast<int64_t>(1) << 40;
        const int64_t lo_g = j >= c_hi ? big : dk <= 0 ? 0 : dk * G;
        const int64_t x = static_cast<int64_t>(p.W) + dk;
        const int64_t hi_g = p.W <= 0 ? big : x <= 0 ? 0 : x * G;
        const int rlo = static_cast<int>(min(max(lo_g - r0, static_cast<int64_t>(0)), static_cast<int64_t>(kN)));
        const int rhi = static_cast<int>(min(max(hi_g - r0, static_cast<int64_t>(0)), static_cast<int64_t>(kN)));
#pragma unroll
        for (int r = 0; r < kN; ++r)
          if (r < rlo || r >= rhi) sv[r] = __float_as_uint(-INFINITY);
      }
      // Row maxima of this warp's keys (raw scores; scale > 0 commutes).
#pragma unroll
      for (int r = 0; r < kN; r += 4) {
        const float4 w4 = make_float4(warp_max_f32(__uint_as_float(sv[r])), warp_max_f32(__uint_as_float(sv[r + 1])),
                                      warp_max_f32(__uint_as_float(sv[r + 2])),
                                      warp_max_f32(__uint_as_float(sv[r + 3])));
        if (lane == 0) reinterpret_cast<float4*>(mx_s + wq * kN)[r >> 2] = w4;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_MX + g));
      got = mbar_wait(bar(B_MX + g), u & 1, abort_flag);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      // Tile max of row `lane` (log2 units); the same in every warp.
      const float tm = fmaxf(fmaxf(mx_s[lane], mx_s[kN + lane]), fmaxf(mx_s[2 * kN + lane], mx_s[3 * kN + lane])) * sl2;
      const bool rise = __any_sync(0xffffffffu, tm > m_own + 8.0f);
      // P^T buffer g and O_g^T are in use by P V of this group's last tile.
      if (u > 0) {
        got = mbar_wait(bar(B_PVDONE + g), (u - 1) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      }
      if (rise) {  // uniform over the warpgroup: same inputs, same decision
        // O_g^T holds P V of this group's earlier tiles (complete: waited above).
        uint32_t ov[kN];
        if (u > 0) {
          tc_fence_after();
          tmem_ld32(sO, ov);
          tmem_wait_ld();
        }
#pragma unroll
        for (int r = 0; r < kN; ++r) {
          const float tmr = __shfl_sync(0xffffffffu, tm, r);
          if (tmr > 8.0f - nmu[r]) {
            const float alpha = ex2(-nmu[r] - tmr);  // 0 for a row that had no key
            l[r] *= alpha;
            nmu[r] = -tmr;
            if (u > 0) ov[r] = __float_as_uint(__uint_as_float(ov[r]) * alpha);
          }
        }
        if (tm > m_own + 8.0f) m_own = tm;
        if (u > 0) {
          tmem_st32(sO, ov);
          tmem_wait_st();
        }
      }
      // P^T: row r, key `key` of a K-major swizzled [32 x 128] tile.
#pragma unroll
      for (int r = 0; r < kN; ++r) {
        const float pv = ex2(fmaf(__uint_as_float(sv[r]), sl2, nmu[r]));
        l[r] += pv;
        st_shared_b16(pa[r & 7] + r * 128, __float2bfloat16_rn(pv));
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_PFULL + g));
    }
    if (!ok) fail();
    // Row sums over the warp's lanes (lane r keeps row r), then the merge.
    float* ls = reinterpret_cast<float*>(smem + LS_OFF);
    float* ml = reinterpret_cast<float*>(smem + ML_OFF);
    float lrow = 0.f;
#pragma unroll
    for (int r = 0; r < kN; ++r) {
      float v = l[r];
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      if (lane == r) lrow = v;
    }
    ls[(g * 4 + wq) * kN + lane] = lrow;
    if (wq == 0) ml[g * kN + lane] = m_own <= -1e30f ? -INFINITY : m_own;
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(B_LS));
    if (g == 0) {
      bool got = ok && mbar_wait(bar(B_LS), 0, abort_flag);
      // Tiles of each group: t = g, g + 2, ...
      const int n0 = (ntiles + 1) / 2, n1 = ntiles / 2;
      if (__all_sync(0xffffffffu, got) && n0 > 0) {
        got = mbar_wait(bar(B_PVDONE + 0), (n0 - 1) & 1, abort_flag);
        if (got && n1 > 0) got = mbar_wait(bar(B_PVDONE + 1), (n1 - 1) & 1, abort_flag);
      }
      if (__all_sync(0xffffffffu, got)) {
        tc_fence_after();
        const int d = tid;  // O^T lane = feature
#pragma unroll
        for (int half = 0; half < 2; ++half) {
        uint32_t o0[16], o1[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          o0[e] = 0u;
          o1[e] = 0u;
        }
        if (n0 > 0) tmem_ld16(tmem + lane_addr + 2 * kN + 16 * half, o0);
        if (n1 > 0) tmem_ld16(tmem + lane_addr + 3 * kN + 16 * half, o1);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int r = 16 * half + e;
          if (r >= R) break;
          const float m0 = ml[r], m1 = ml[kN + r];
          const float M = fmaxf(m0, m1);
          const float w0 = m0 == -INFINITY ? 0.f : ex2(m0 - M);
          const float w1 = m1 == -INFINITY ? 0.f : ex2(m1 - M);
          const float L0 = ls[r] + ls[kN + r] + ls[2 * kN + r] + ls[3 * kN + r];
          const float L1 = ls[4 * kN + r] + ls[5 * kN + r] + ls[6 * kN + r] + ls[7 * kN + r];
          const float L = w0 * L0 + w1 * L1;
          const float inv = L > 0.f ? 1.f / L : 0.f;
          const float ov = (w0 * __uint_as_float(o0[e]) + w1 * __uint_as_float(o1[e])) * inv;
          const int s = (r0 + r) / G, h = kvh * G + (r0 + r - s * G);
          const int64_t row = (static_cast<int64_t>(b) * p.n + s) * p.Hq + h;
          p.ws_o[(static_cast<int64_t>(split) * rows_total + row) * kD + d] = ov;
          if (d == r) p.ws_lse[static_cast<int64_t>(split) * rows_total + row] = L > 0.f ? M + __log2f(L) : -INFINITY;
        }
        }
      } else {
        fail();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ------------------------------------------------------------------- host

// (D, Hkv, Lmax, nc, B) view of a [B, nc, Lmax, Hkv, 128] cache; box 64 x 1 x 128 x 1 x 1.
static bool make_cache_view128(const TmapKey& k, CUtensorMap* m) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  const cuuint64_t B = k.dims[0], n = k.dims[1], Lmax = k.dims[2], Hkv = k.dims[3];
  const cuuint64_t D = dtc::kD, e = 2;
  const cuuint64_t dims[5] = {D, Hkv, Lmax, n, B};
  const cuuint64_t strides[4] = {D * e, Hkv * D * e, Lmax * Hkv * D * e, n * Lmax * Hkv * D * e};
  const cuuint32_t box[5] = {64, 1, (cuuint32_t)dtc::kTok, 1, 1};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(k.ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool encode_cache_view128(CUtensorMap* m, const void* ptr, int B, int n, int Lmax, int Hkv) {
  TmapKey k;
  std::memset(&k, 0, sizeof(k));
  k.ptr = ptr;
  k.dims[0] = B;
  k.dims[1] = n;
  k.dims[2] = Lmax;
  k.dims[3] = Hkv;
  k.kind = 4;
  return tmap_cached(k, m, make_cache_view128);
}

bool decode_tc_supported(int n, int Hq, int Hkv, int D, bool cross) {
  (void)n;
  (void)Hq;
  (void)Hkv;
  return cross && D == dtc::kD;
}

// Splits per unit: at least ~2 waves of one CTA per SM, the count whose
// last wave is fullest, never more than the workspace was sized for.
int decode_tc_nsplit(int units, int Lmax, int cap, int sms) {
  int max_ns = (Lmax + dtc::kTok - 1) / dtc::kTok;
  if (max_ns > cap) max_ns = cap;
  if (max_ns < 1) max_ns = 1;
#ifndef HD_DTC_MIN_WAVES
#define HD_DTC_MIN_WAVES 2
#endif
  int lo = (HD_DTC_MIN_WAVES * sms + units - 1) / units;
  if (lo < 1) lo = 1;
  if (lo > max_ns) lo = max_ns;
  int best = lo;
  double best_eff = -1.0;
  for (int ns = lo; ns <= max_ns && ns <= lo + 8; ++ns) {
    const int64_t x = static_cast<int64_t>(units) * ns;
    const int64_t waves = (x + sms - 1) / sms;
    const double eff = static_cast<double>(x) / static_cast<double>(waves * sms);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = ns;
    }
  }
  return best;
}

cudaError_t launch_decode_tc(const void* q, const void* kc, const void* vc, const int32_t* ctx, float* ws_o,
                             float* ws_lse, int B, int n, int Lmax, int Hq, int Hkv, int W, float scale, int nsplit,
                             int32_t* status, cudaStream_t st, int nc, int soff, int sstride) {
  CUtensorMap mk, mv;
  if (!encode_cache_view128(&mk, kc, B, nc, Lmax, Hkv) || !encode_cache_view128(&mv, vc, B, nc, Lmax, Hkv))
    return cudaErrorInvalidValue;
  DtcParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.ctx = ctx;
  p.ws_o = ws_o;
  p.ws_lse = ws_lse;
  p.status = status;
  p.B = B;
  p.n = n;
  p.Lmax = Lmax;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.W = W;
  p.nsplit = nsplit;
  p.nc = nc;
  p.soff = soff;
  p.sstride = sstride;
  p.scale_log2 = scale * 1.4426950408889634f;
  static const int stall = [] {
    const char* e = getenv("HD_TEST_STALL_DECODE");
    return (e && e[0] == '1') ? 1 : 0;
  }();
  p.stall_first = stall;
  const int64_t units = static_cast<int64_t>(B) * Hkv * ((n * (Hq / Hkv) + dtc::kN - 1) / dtc::kN);
  if (units > 65535 || units < 1) return cudaErrorInvalidValue;
  cudaError_t err = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dtc::kAlloc);
  if (err != cudaSuccess) return err;
  decode_tc_kernel<<<dim3(nsplit, static_cast<unsigned>(units)), dtc::kThreads, dtc::kAlloc, st>>>(mk, mv, p);
  return cudaGetLastError();
}

}  // namespace hd
