// Backward of Stream-Factorized Attention, bf16 in / f32 accumulate, on the
// tcgen05 tensor cores and tensor memory of sm_100a.
//
// ("Hidden Decoding at Scale", "Stream-Factorized Attention", Figure 2; the
// layers are trained through, "Computational Cost".)  Same stream views as
// the forward: q/k/v/dO [B, ns*Ls, H, D] are read through 5-D TMA maps
// (D, H, ns, Ls, B), so intra mode (ns = n) and cross mode (ns = 1, Ls = nL)
// are the same kernels and keys of other streams are never loaded.  P is
// recomputed from the forward's lse; per-row (-lse*log2e, delta = <dO, O>)
// come from the preparation kernel, stream-major and padded to 128 tokens
// with (-inf, 0) so padded queries contribute nothing.
//
// Two kernels, each owning its output (no atomics):
//
// attn_bwd_dkv_kernel -- unit = 128 keys of one (batch, stream, KV head);
//   walks every query tile of every query head of the GQA group that sees
//   the key block.  Tensor memory: S^T [0,128) dP^T [128,256) dV [256,256+D)
//   dK [256+D,256+2D).  Per query tile:  S^T = K Q^T,  dP^T = V dO^T,
//   P^T = 2^(S^T scale log2e - lse2) (masked to 0),  dS^T = P^T (dP^T - delta),
//   dV += P^T dO,  dK += dS^T Q, with P^T and dS^T written back as bf16 over
//   their own f32 columns and fed to the tensor core from tensor memory.
//   MMA issue order  dV(t) S(t+1) | dK(t) dP(t+1): while the softmax warps
//   compute P(t+1) the tensor core runs dK(t) and dP(t+1); while they compute
//   dS(t+1) it runs dV(t+1) and S(t+2).  Overwrites are safe because one
//   thread's tcgen05.mma operations execute in issue order.
//
// attn_bwd_dq_kernel -- unit = 128 queries of one (batch, stream, query head);
//   walks the visible key tiles.  Tensor memory: S double-buffered [0,256),
//   dP [256,384), dQ [384,384+D).  Per key tile:  S = Q K^T,  dP = dO V^T,
//   dS = P (dP - delta) written as bf16 over S,  dQ += dS K.  MMA order
//   dQ(t) dP(t+1) S(t+2): the next S is ready when the softmax warps finish
//   the current tile.
//
// CTA = 10 warps: 0-7 elementwise (warp w owns tensor-memory lanes
// 32*(w&3).. and the column half w>>2 of each 128-column tile), 8 TMA
// producer, 9 MMA issuer.  Persistent, longest units first.  Every wait is
// bounded (1 s), after which the kernel records HD_ERR_TIMEOUT, lets its
// copies land, drains its MMAs and frees tensor memory.
#include <cstdlib>

#include "hd_common.cuh"
#include "hd_launch.h"

namespace hd {

namespace bw {
constexpr int BT = 128;  // tile rows (queries or keys)
constexpr int kThreads = 320;
constexpr int kWarpTMA = 8;
constexpr int kWarpMMA = 9;
constexpr uint32_t kTmemCols = 512;
constexpr int kLdBytes = BT * 8;  // -lse2[128] then delta[128] of one query tile
// One exponential pair in kPolyEvery of the P tiles (both kernels) on the
// FMA pipe, to offload the MUFU unit (0: all on MUFU): the exponent x
// (<= 0 up to rounding for a visible pair; masked pairs are zeroed after)
// is shifted and clamped to y = sat((x + 126) / (126 + kPolyHi)) by one
// saturating FMA per element, then exp2_sat2 (relative error < 1e-4, below
// the bf16 rounding of P).
#ifndef HD_BW_POLY_EVERY
#define HD_BW_POLY_EVERY 3
#endif
constexpr int kPolyEvery = HD_BW_POLY_EVERY;
constexpr int kPolyHi = 1;
constexpr float kPolyInv = 1.f / (126.f + kPolyHi);
__host__ __device__ constexpr bool poly_pair(int c) {
  return kPolyEvery > 0 && (c % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1;
}
// 2^x of the pairs of a 64-column row piece, x in pv (in place).
__device__ __forceinline__ void exp2_row64(float (&pv)[64]) {
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    if (poly_pair(c)) {
      const float y0 = fma_sat(pv[2 * c], kPolyInv, 126.f * kPolyInv);
      const float y1 = fma_sat(pv[2 * c + 1], kPolyInv, 126.f * kPolyInv);
      unpack_f32x2(exp2_sat2<kPolyHi>(pack_f32x2(y0, y1)), pv[2 * c], pv[2 * c + 1]);
    } else {
      pv[2 * c] = ex2(pv[2 * c]);
      pv[2 * c + 1] = ex2(pv[2 * c + 1]);
    }
  }
}
// Elementwise arithmetic as packed f32x2 operations (exponents of P for a
// whole tile first, then the exponentials; dS = P (dP - delta) in pairs)
// when nonzero.
#ifndef HD_BW_PACKED
#define HD_BW_PACKED 1
#endif
constexpr bool kPacked = HD_BW_PACKED != 0;


template <int D>
struct Tile {
  static constexpr int KB = D / 64;     // 128-byte column blocks per row
  static constexpr int BLK = BT * 128;  // one 128-row x 128-byte block
  static constexpr int TILE = BLK * KB;
};

// dK/dV kernel: K, V resident per unit; Q (+ its lse/delta) and dO in 2 stages.
template <int D>
struct LayKV {
  using T = Tile<D>;
  static constexpr int QST = 2;
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + T::TILE;
  static constexpr int Q_OFF = V_OFF + T::TILE;
  static constexpr int O_OFF = Q_OFF + QST * T::TILE;
  static constexpr int LD_OFF = O_OFF + QST * T::TILE;
  static constexpr int BAR_OFF = LD_OFF + QST * kLdBytes;
  static constexpr int B_KVFULL = 0, B_KVEMPTY = 1, B_QFULL = 2, B_QEMPTY = B_QFULL + QST,
                       B_OFULL = B_QEMPTY + QST, B_OEMPTY = B_OFULL + QST, B_SFULL = B_OEMPTY + QST,
                       B_DPFULL = B_SFULL + 1, B_PFULL = B_DPFULL + 1, B_DSFULL = B_PFULL + 1,
                       B_ACCFULL = B_DSFULL + 1, B_ACCEMPTY = B_ACCFULL + 1, B_DRAIN = B_ACCEMPTY + 1,
                       NBAR = B_DRAIN + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int ALLOC = MISC_OFF + 16 + 1024;
};

// dQ kernel: Q, dO resident per unit; K in 3 stages, V in 2.
template <int D>
struct LayQ {
  using T = Tile<D>;
  static constexpr int KST = 3, VST = 2;
  static constexpr int Q_OFF = 0;
  static constexpr int O_OFF = Q_OFF + T::TILE;
  static constexpr int K_OFF = O_OFF + T::TILE;
  static constexpr int V_OFF = K_OFF + KST * T::TILE;
  static constexpr int BAR_OFF = V_OFF + VST * T::TILE;
  static constexpr int B_QFULL = 0, B_QEMPTY = 1, B_KFULL = 2, B_KEMPTY = B_KFULL + KST,
                       B_VFULL = B_KEMPTY + KST, B_VEMPTY = B_VFULL + VST, B_SFULL = B_VEMPTY + VST,
                       B_DPFULL = B_SFULL + 2, B_DSFULL = B_DPFULL + 1, B_ACCFULL = B_DSFULL + 1,
                       B_ACCEMPTY = B_ACCFULL + 1, B_DRAIN = B_ACCEMPTY + 1, NBAR = B_DRAIN + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int ALLOC = MISC_OFF + 16 + 1024;
};
// Diagnostic build only (HD_BW_TRACE): per-role clock counters of the dK/dV
// kernel, kBwTraceSlots per CTA (see hd_bw_trace_fetch).
#ifndef HD_BW_TRACE
#define HD_BW_TRACE 0
#endif
constexpr bool kTrace = HD_BW_TRACE != 0;
}  // namespace bw

#if HD_BW_TRACE
constexpr int kBwTraceCtas = 1024;
constexpr int kBwTraceSlots = 16;
__device__ unsigned long long g_bw_trace[kBwTraceCtas * kBwTraceSlots];
#endif

struct BwParams {
  BwdWs ws;  // -lse2 and delta planes, stream-major, padded
  void* dq;
  void* dk;
  void* dv;
  int32_t* status;
  AttnGeom g;  // query token i of stream s sits at key index i*qstride + qoff
  int Lpad, Hq, Hkv, W;
  int nqb;  // 128-token query blocks per query stream
  int nkb;  // 128-token key blocks per key stream
  int kns;  // key streams the dK/dV kernel walks
  float scale_log2, scale;
  int total_units;
  // Test hook (environment HD_TEST_STALL_BWD=1): the MMA warp of CTA 0 of
  // the dK/dV kernel never signals its S tiles, so the elementwise wait runs
  // out and the kernel must take its timeout path.  0 in normal use.
  int stall_first_s;
};

// Key index of query token i (of any query stream; the backward takes no
// per-stream offset).
__device__ __forceinline__ int bw_pos(const BwParams& p, int i) { return i * p.g.qstride + p.g.qoff; }

// dK/dV unit: key block ascending (causal: the first blocks see the most
// query tiles), then (b, key stream, kvh).  Its tiles j = 0 .. G*nqt-1 walk
// the query tiles that see the block from the last one down, the G heads of
// the group inside: the CTAs that run the other key blocks of the same
// (b, stream, kvh) at the same time then read the same Q and dO tiles, which
// stay in L2.  nqt = 0 when no query sees the block (its dK, dV are zero).
struct KvUnit {
  int b, skv, sq, kvh, kblk, qt_lo, qt_hi, nqt;
};
// Unit schedule of a CTA: rounds of gridDim.x units in the longest-first
// order, walked forwards in even rounds and backwards in odd ones, so that
// every CTA gets a similar total.  The k-th unit of this CTA, -1 when the
// rounds are exhausted, -2 when round k has none for it.
#ifndef HD_TC_SNAKE
#define HD_TC_SNAKE 1
#endif
__device__ __forceinline__ int bw_unit_of(int k, int total) {
  const int base = k * static_cast<int>(gridDim.x);
  if (base >= total) return -1;
  const int c = (HD_TC_SNAKE && (k & 1)) ? static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x)
                                         : static_cast<int>(blockIdx.x);
  return base + c < total ? base + c : -2;
}

__device__ __forceinline__ KvUnit kv_unit(int u, const BwParams& p) {
  const int per = p.g.B * p.kns * p.Hkv;
  KvUnit x;
  x.kblk = u / per;
  int rem = u - x.kblk * per;
  x.kvh = rem % p.Hkv;
  rem /= p.Hkv;
  const int ks = rem % p.kns;
  x.b = rem / p.kns;
  x.skv = p.g.kv_stream >= 0 ? p.g.kv_stream : ks;  // stream of the K/V view
  x.sq = p.g.kv_stream >= 0 ? 0 : ks;               // query stream reading it
  const int k0 = x.kblk * bw::BT;
  // queries with k0 <= pos(i) (and pos(i) - (k0 + 127) < W)
  const int i_lo = k0 <= p.g.qoff ? 0 : (k0 - p.g.qoff + p.g.qstride - 1) / p.g.qstride;
  const int i_hi = p.W > 0 ? min(p.g.Lq - 1, (k0 + bw::BT - 1 + p.W - 1 - p.g.qoff) / p.g.qstride) : p.g.Lq - 1;
  x.qt_lo = i_lo / bw::BT;
  x.qt_hi = i_hi / bw::BT;
  x.nqt = i_lo <= i_hi ? x.qt_hi - x.qt_lo + 1 : 0;
  return x;
}
__device__ __forceinline__ int kv_tile_qt(const KvUnit& x, int j, int G) { return x.qt_hi - j / G; }
__device__ __forceinline__ int kv_tile_head(const KvUnit& x, int j, int G) { return x.kvh * G + j % G; }

// dQ unit: query block descending (causal: the last blocks see the most key
// tiles), then (b, query stream, h).
struct QUnit {
  int b, s, skv, h, qblk, kt_lo, nkt;
};
__device__ __forceinline__ QUnit q_unit(int u, const BwParams& p) {
  const int per = p.g.B * p.g.ns * p.Hq;
  QUnit x;
  const int qi = u / per;
  int rem = u - qi * per;
  x.qblk = p.nqb - 1 - qi;
  x.h = rem % p.Hq;
  rem /= p.Hq;
  x.s = rem % p.g.ns;
  x.b = rem / p.g.ns;
  x.skv = p.g.kv_stream >= 0 ? p.g.kv_stream : x.s;
  const int q0 = x.qblk * bw::BT;
  const int qlast = min(q0 + bw::BT - 1, p.g.Lq - 1);
  const int kt_hi = bw_pos(p, qlast) / bw::BT;
  x.kt_lo = p.W > 0 ? max(0, bw_pos(p, q0) - p.W + 1) / bw::BT : 0;
  x.nkt = kt_hi - x.kt_lo + 1;
  return x;
}

// acc(tmem d) (+)= A(smem, K-major, 128 rows) * B(smem, K-major, 128 rows)^T
// over the D-long reduction: the S-type products (S, dP, S^T, dP^T).
template <int D>
__device__ __forceinline__ void mma_rows_rows(uint32_t d, uint32_t a_smem, uint32_t b_smem) {
  using T = bw::Tile<D>;
  constexpr uint32_t id = idesc_bf16_f32(bw::BT, bw::BT, false, false);
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk >> 2) * T::BLK + (kk & 3) * 32;
    mma_ss(d, smem_desc_sw128(a_smem + off, 16, 1024), smem_desc_sw128(b_smem + off, 16, 1024), id,
           kk > 0 ? 1u : 0u);
  }
}

// acc(tmem d, 128 x D) (+)= A(tmem, 128 x 128 bf16, packed by column halves:
// elements [64h, 64h+64) in columns [a + 64h, a + 64h + 32)) * B(smem tile
// [128 rows][D], MN-major): the dV, dK and dQ products.
template <int D>
__device__ __forceinline__ void mma_tmem_rows(uint32_t d, uint32_t a_tmem, uint32_t b_smem, bool acc) {
  using T = bw::Tile<D>;
  constexpr uint32_t id = idesc_bf16_f32(bw::BT, D, false, true);
#pragma unroll
  for (int kk = 0; kk < bw::BT / 16; ++kk) {
    const uint64_t bdesc = smem_desc_sw128(b_smem + kk * 2048, T::BLK, 1024);
    mma_ts(d, a_tmem + 64 * (kk >> 2) + 8 * (kk & 3), bdesc, id, (acc || kk > 0) ? 1u : 0u);
  }
}

// Store 64 f32 values of one row as bf16 (scaled) to 16-byte-aligned global memory.
__device__ __forceinline__ void store_row64_bf16(__nv_bfloat16* dst, const uint32_t (&a)[32], const uint32_t (&b)[32],
                                                 float mul) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint4 w;
    w.x = pack_bf16x2(__uint_as_float(a[8 * e + 0]) * mul, __uint_as_float(a[8 * e + 1]) * mul);
    w.y = pack_bf16x2(__uint_as_float(a[8 * e + 2]) * mul, __uint_as_float(a[8 * e + 3]) * mul);
    w.z = pack_bf16x2(__uint_as_float(a[8 * e + 4]) * mul, __uint_as_float(a[8 * e + 5]) * mul);
    w.w = pack_bf16x2(__uint_as_float(a[8 * e + 6]) * mul, __uint_as_float(a[8 * e + 7]) * mul);
    d4[e] = w;
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    uint4 w;
    w.x = pack_bf16x2(__uint_as_float(b[8 * e + 0]) * mul, __uint_as_float(b[8 * e + 1]) * mul);
    w.y = pack_bf16x2(__uint_as_float(b[8 * e + 2]) * mul, __uint_as_float(b[8 * e + 3]) * mul);
    w.z = pack_bf16x2(__uint_as_float(b[8 * e + 4]) * mul, __uint_as_float(b[8 * e + 5]) * mul);
    w.w = pack_bf16x2(__uint_as_float(b[8 * e + 6]) * mul, __uint_as_float(b[8 * e + 7]) * mul);
    d4[4 + e] = w;
  }
}

// Write columns [c0, c0 + D/2) of a 128 x D f32 accumulator row (this
// thread's lane) to dst as bf16 times mul.
template <int D>
__device__ __forceinline__ void acc_half_to_global(uint32_t taddr, __nv_bfloat16* dst, float mul, bool ok) {
  if constexpr (D == 128) {
    uint32_t a[32], b[32];
    tmem_ld32(taddr, a);
    tmem_ld32(taddr + 32, b);
    tmem_wait_ld();
    if (ok) store_row64_bf16(dst, a, b, mul);
  } else {
    uint32_t a[32];
    tmem_ld32(taddr, a);
    tmem_wait_ld();
    if (ok) {
      uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(a[8 * e + 0]) * mul, __uint_as_float(a[8 * e + 1]) * mul);
        w.y = pack_bf16x2(__uint_as_float(a[8 * e + 2]) * mul, __uint_as_float(a[8 * e + 3]) * mul);
        w.z = pack_bf16x2(__uint_as_float(a[8 * e + 4]) * mul, __uint_as_float(a[8 * e + 5]) * mul);
        w.w = pack_bf16x2(__uint_as_float(a[8 * e + 6]) * mul, __uint_as_float(a[8 * e + 7]) * mul);
        d4[e] = w;
      }
    }
  }
}

// ======================================================= dK / dV kernel

template <int D>
__global__ void __launch_bounds__(bw::kThreads, 1)
    attn_bwd_dkv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                        const BwParams p) {
  using Lay = bw::LayKV<D>;
  using T = bw::Tile<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + Lay::BAR_OFF + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::MISC_OFF + 4);
  volatile int* no_abort = reinterpret_cast<volatile int*>(smem + Lay::MISC_OFF + 8);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.Hq / p.Hkv;

  if (threadIdx.x == 0) {
    mbar_init(bar(Lay::B_KVFULL), 1);
    mbar_init(bar(Lay::B_KVEMPTY), 1);
    for (int i = 0; i < Lay::QST; ++i) {
      mbar_init(bar(Lay::B_QFULL + i), 1);
      mbar_init(bar(Lay::B_QEMPTY + i), 1);
      mbar_init(bar(Lay::B_OFULL + i), 1);
      mbar_init(bar(Lay::B_OEMPTY + i), 1);
    }
    mbar_init(bar(Lay::B_SFULL), 1);
    mbar_init(bar(Lay::B_DPFULL), 1);
    mbar_init(bar(Lay::B_PFULL), 256);
    mbar_init(bar(Lay::B_DSFULL), 256);
    mbar_init(bar(Lay::B_ACCFULL), 1);
    mbar_init(bar(Lay::B_ACCEMPTY), 256);
    mbar_init(bar(Lay::B_DRAIN), 1);
    *abort_flag = 0;
    *no_abort = 0;
    fence_barrier_init();
  }
  if (warp == bw::kWarpTMA && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  if (warp == bw::kWarpMMA) {
    tmem_alloc(smem_u32(tmem_slot), bw::kTmemCols);
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

  if (warp == bw::kWarpTMA) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int t = 0, ul = 0, kv_issued = 0;
      int q_issued[Lay::QST] = {}, o_issued[Lay::QST] = {};
      bool ok = true;
      for (int k = 0, u = bw_unit_of(0, p.total_units); ok && u != -1;
           ul += (u >= 0), u = bw_unit_of(++k, p.total_units)) {
        if (u < 0) continue;  // round k has no unit for this CTA
        const KvUnit x = kv_unit(u, p);
        if (!mbar_wait(bar(Lay::B_KVEMPTY), (ul & 1) ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(bar(Lay::B_KVFULL), 2 * T::TILE);
#pragma unroll
        for (int kb = 0; kb < T::KB; ++kb) {
          tma_load_5d(sbase + Lay::K_OFF + kb * T::BLK, &tmK, bar(Lay::B_KVFULL), kb * 64, x.kvh, x.skv,
                      x.kblk * bw::BT, x.b);
          tma_load_5d(sbase + Lay::V_OFF + kb * T::BLK, &tmV, bar(Lay::B_KVFULL), kb * 64, x.kvh, x.skv,
                      x.kblk * bw::BT, x.b);
        }
        ++kv_issued;
        const int nt = G * x.nqt;
        for (int j = 0; j < nt; ++j, ++t) {
          const int h = kv_tile_head(x, j, G);
          const int qt = kv_tile_qt(x, j, G);
          const int st = t % Lay::QST;
          const uint32_t ph = ((t / Lay::QST) & 1) ^ 1;
          if (!mbar_wait(bar(Lay::B_QEMPTY + st), ph, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(Lay::B_QFULL + st), T::TILE + bw::kLdBytes);
#pragma unroll
          for (int kb = 0; kb < T::KB; ++kb)
            tma_load_5d(sbase + Lay::Q_OFF + st * T::TILE + kb * T::BLK, &tmQ, bar(Lay::B_QFULL + st), kb * 64, h,
                        x.sq, qt * bw::BT, x.b);
          {
            const int64_t at = ((static_cast<int64_t>(x.b) * p.Hq + h) * p.g.ns + x.sq) * p.Lpad + qt * bw::BT;
            bulk_load(sbase + Lay::LD_OFF + st * bw::kLdBytes, p.ws.nl2 + at, bw::kLdBytes / 2,
                      bar(Lay::B_QFULL + st));
            bulk_load(sbase + Lay::LD_OFF + st * bw::kLdBytes + bw::kLdBytes / 2, p.ws.delta + at,
                      bw::kLdBytes / 2, bar(Lay::B_QFULL + st));
          }
          ++q_issued[st];
          if (!mbar_wait(bar(Lay::B_OEMPTY + st), ph, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(Lay::B_OFULL + st), T::TILE);
#pragma unroll
          for (int kb = 0; kb < T::KB; ++kb)
            tma_load_5d(sbase + Lay::O_OFF + st * T::TILE + kb * T::BLK, &tmO, bar(Lay::B_OFULL + st), kb * 64, h,
                        x.sq, qt * bw::BT, x.b);
          ++o_issued[st];
        }
      }
      if (!ok) {
        fail();
        if (kv_issued) mbar_wait(bar(Lay::B_KVFULL), (kv_issued - 1) & 1, no_abort);
        for (int i = 0; i < Lay::QST; ++i) {
          if (q_issued[i]) mbar_wait(bar(Lay::B_QFULL + i), (q_issued[i] - 1) & 1, no_abort);
          if (o_issued[i]) mbar_wait(bar(Lay::B_OFULL + i), (o_issued[i] - 1) & 1, no_abort);
        }
      }
    }
  } else if (warp == bw::kWarpMMA) {
    // ---------------------------------------------------------------- MMA
    // Per tile t:  [P(t) ready] dV(t) S(t+1)  [dS(t) ready] dK(t) dP(t+1).
    if (lane == 0) {
      const uint32_t tS = tmem, tDP = tmem + 128, tDV = tmem + 256, tDK = tmem + 256 + D;
      int t = 0, ul = 0;
      bool ok = true;
      // Diagnostic counters (HD_BW_TRACE): waiting for P, for dS, for the
      // Q/dO/K/V stages and the accumulators; total.
      unsigned long long mw[4] = {0, 0, 0, 0};
      const long long mt0 = bw::kTrace ? clock64() : 0;
      auto tw = [&](int which, uint32_t b, uint32_t par) {
        if constexpr (bw::kTrace) {
          const long long t0 = clock64();
          const bool r = mbar_wait(b, par, abort_flag);
          mw[which] += static_cast<unsigned long long>(clock64() - t0);
          return r;
        } else {
          return mbar_wait(b, par, abort_flag);
        }
      };
      auto issue_S = [&](int tt) {
        const int st = tt % Lay::QST;
        mma_rows_rows<D>(tS, sbase + Lay::K_OFF, sbase + Lay::Q_OFF + st * T::TILE);
        if (!(p.stall_first_s && blockIdx.x == 0)) tc_commit(bar(Lay::B_SFULL));
      };
      auto issue_dP = [&](int tt) {
        const int st = tt % Lay::QST;
        mma_rows_rows<D>(tDP, sbase + Lay::V_OFF, sbase + Lay::O_OFF + st * T::TILE);
        tc_commit(bar(Lay::B_DPFULL));
      };
      for (int k = 0, u = bw_unit_of(0, p.total_units); ok && u != -1;
           ul += (u >= 0), u = bw_unit_of(++k, p.total_units)) {
        if (u < 0) continue;  // round k has no unit for this CTA
        const KvUnit x = kv_unit(u, p);
        const int nt = G * x.nqt;
        if (!tw(2, bar(Lay::B_KVFULL), ul & 1)) { ok = false; break; }
        if (nt == 0) {  // no query sees this key block: nothing to accumulate
          tc_commit(bar(Lay::B_ACCFULL));
          tc_commit(bar(Lay::B_KVEMPTY));
          continue;
        }
        if (!tw(2, bar(Lay::B_QFULL + t % Lay::QST), (t / Lay::QST) & 1)) { ok = false; break; }
        tc_fence_after();
        issue_S(t);
        if (!tw(2, bar(Lay::B_OFULL + t % Lay::QST), (t / Lay::QST) & 1)) { ok = false; break; }
        tc_fence_after();
        issue_dP(t);
        for (int j = 0; j < nt; ++j, ++t) {
          const int st = t % Lay::QST;
          const int stn = (t + 1) % Lay::QST;
          const uint32_t phn = ((t + 1) / Lay::QST) & 1;
          if (!tw(0, bar(Lay::B_PFULL), t & 1)) { ok = false; break; }
          if (j == 0 && ul > 0 && !tw(2, bar(Lay::B_ACCEMPTY), (ul - 1) & 1)) { ok = false; break; }
          tc_fence_after();
          mma_tmem_rows<D>(tDV, tS, sbase + Lay::O_OFF + st * T::TILE, j > 0);
          tc_commit(bar(Lay::B_OEMPTY + st));
          if (j + 1 < nt) {
            if (!tw(2, bar(Lay::B_QFULL + stn), phn)) { ok = false; break; }
            tc_fence_after();
            issue_S(t + 1);
          }
          if (!tw(1, bar(Lay::B_DSFULL), t & 1)) { ok = false; break; }
          tc_fence_after();
          mma_tmem_rows<D>(tDK, tDP, sbase + Lay::Q_OFF + st * T::TILE, j > 0);
          tc_commit(bar(Lay::B_QEMPTY + st));
          if (j + 1 < nt) {
            if (!tw(2, bar(Lay::B_OFULL + stn), phn)) { ok = false; break; }
            tc_fence_after();
            issue_dP(t + 1);
          }
        }
        if (!ok) break;
        tc_commit(bar(Lay::B_ACCFULL));
        tc_commit(bar(Lay::B_KVEMPTY));
      }
      if (!ok) fail();
      tc_commit(bar(Lay::B_DRAIN));
      mbar_wait(bar(Lay::B_DRAIN), 0, no_abort);
#if HD_BW_TRACE
      mw[3] = static_cast<unsigned long long>(clock64() - mt0);
      if (blockIdx.x < kBwTraceCtas)
        for (int c = 0; c < 4; ++c) g_bw_trace[blockIdx.x * kBwTraceSlots + 8 + c] = mw[c];
#endif
    }
  } else {
    // ------------------------------------------- elementwise + epilogue
    const int ch = warp >> 2;  // column half
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_addr + 64 * ch;
    const uint32_t tDP = tmem + lane_addr + 128 + 64 * ch;
    const float sl2 = p.scale_log2;
    int t = 0, ul = 0;
    bool ok = true;
    // Diagnostic counters (HD_BW_TRACE): waiting for S, forming P, waiting
    // for dP, forming dS, tiles, epilogue.
    unsigned long long tr[6] = {0, 0, 0, 0, 0, 0};
    long long tmark = bw::kTrace ? clock64() : 0;
    auto tick = [&](int i) {
      if constexpr (bw::kTrace) {
        const long long tt = clock64();
        tr[i] += static_cast<unsigned long long>(tt - tmark);
        tmark = tt;
      }
    };
    for (int k = 0, u = bw_unit_of(0, p.total_units); ok && u != -1;
         ul += (u >= 0), u = bw_unit_of(++k, p.total_units)) {
      if (u < 0) continue;  // round k has no unit for this CTA
      const KvUnit x = kv_unit(u, p);
      const int nt = G * x.nqt;
      const int k0 = x.kblk * bw::BT;
      const int jkey = k0 + r;  // this thread's key token
      for (int j = 0; j < nt; ++j, ++t) {
        const int st = t % Lay::QST;
        const int q0 = kv_tile_qt(x, j, G) * bw::BT + 64 * ch;  // first query of this half
        if (bw::kTrace) tmark = clock64();
        bool got = mbar_wait(bar(Lay::B_SFULL), t & 1, abort_flag);
        got = got && mbar_wait(bar(Lay::B_QFULL + st), (t / Lay::QST) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tick(0);
        tc_fence_after();
        uint32_t sv[64];
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        // lse2 / delta of this half's 64 queries: 16-byte broadcast loads
        // (every lane reads the same address), four columns per load.
        const float4* l4 = reinterpret_cast<const float4*>(smem + Lay::LD_OFF + st * bw::kLdBytes) + 16 * ch;
        const float4* d4 = reinterpret_cast<const float4*>(smem + Lay::LD_OFF + st * bw::kLdBytes + 512) + 16 * ch;
        tmem_wait_ld();
        const bool need_mask = (bw_pos(p, q0) < k0 + bw::BT - 1) || (p.W > 0 && bw_pos(p, q0 + 63) - k0 >= p.W);
        float pv[64];
        if constexpr (bw::kPacked) {
          const uint64_t s2 = pack_f32x2(sl2, sl2);
#pragma unroll
          for (int c4 = 0; c4 < 16; ++c4) {
            const float4 l = l4[c4];
            unpack_f32x2(fma_f32x2(pack_f32x2(__uint_as_float(sv[4 * c4]), __uint_as_float(sv[4 * c4 + 1])), s2,
                                   pack_f32x2(l.x, l.y)),
                         pv[4 * c4], pv[4 * c4 + 1]);
            unpack_f32x2(fma_f32x2(pack_f32x2(__uint_as_float(sv[4 * c4 + 2]), __uint_as_float(sv[4 * c4 + 3])), s2,
                                   pack_f32x2(l.z, l.w)),
                         pv[4 * c4 + 2], pv[4 * c4 + 3]);
          }
          bw::exp2_row64(pv);
        } else {
#pragma unroll
          for (int c4 = 0; c4 < 16; ++c4) {
            const float4 l = l4[c4];
            pv[4 * c4 + 0] = ex2(fmaf(__uint_as_float(sv[4 * c4 + 0]), sl2, l.x));
            pv[4 * c4 + 1] = ex2(fmaf(__uint_as_float(sv[4 * c4 + 1]), sl2, l.y));
            pv[4 * c4 + 2] = ex2(fmaf(__uint_as_float(sv[4 * c4 + 2]), sl2, l.z));
            pv[4 * c4 + 3] = ex2(fmaf(__uint_as_float(sv[4 * c4 + 3]), sl2, l.w));
          }
        }
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int pi = bw_pos(p, q0 + c);
            if (pi < jkey || (p.W > 0 && pi - jkey >= p.W)) pv[c] = 0.f;
          }
        }
        {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(pv[2 * e], pv[2 * e + 1]);
          tmem_st16(tS, pk);
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(pv[32 + 2 * e], pv[32 + 2 * e + 1]);
          tmem_st16(tS + 16, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(Lay::B_PFULL));
        tick(1);
        got = mbar_wait(bar(Lay::B_DPFULL), t & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tick(2);
        tc_fence_after();
        tmem_ld32(tDP, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(tDP + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_ld();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[16];
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const int c = 32 * half + 4 * e4;
            const float4 d = d4[8 * half + e4];
            if constexpr (bw::kPacked) {
              pk[2 * e4] = pack_bf16x2_of(
                  mul_f32x2(pack_f32x2(pv[c], pv[c + 1]),
                            sub_f32x2(pack_f32x2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])),
                                      pack_f32x2(d.x, d.y))));
              pk[2 * e4 + 1] = pack_bf16x2_of(
                  mul_f32x2(pack_f32x2(pv[c + 2], pv[c + 3]),
                            sub_f32x2(pack_f32x2(__uint_as_float(sv[c + 2]), __uint_as_float(sv[c + 3])),
                                      pack_f32x2(d.z, d.w))));
            } else {
              pk[2 * e4] =
                  pack_bf16x2(pv[c] * (__uint_as_float(sv[c]) - d.x), pv[c + 1] * (__uint_as_float(sv[c + 1]) - d.y));
              pk[2 * e4 + 1] = pack_bf16x2(pv[c + 2] * (__uint_as_float(sv[c + 2]) - d.z),
                                           pv[c + 3] * (__uint_as_float(sv[c + 3]) - d.w));
            }
          }
          tmem_st16(tDP + 16 * half, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(Lay::B_DSFULL));
        tick(3);
        if (bw::kTrace) ++tr[4];
      }
      if (!ok) break;
      if (bw::kTrace) tmark = clock64();
      // Epilogue: dV and scale*dK rows of this unit's keys.
      const bool got = mbar_wait(bar(Lay::B_ACCFULL), ul & 1, abort_flag);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      const bool row_ok = jkey < p.g.Lk;
      const int64_t orow = ((static_cast<int64_t>(x.b) * p.g.kv_ns * p.g.Lk +
                             static_cast<int64_t>(row_ok ? jkey : 0) * p.g.kv_ns + x.skv) * p.Hkv + x.kvh) * D +
                           ch * (D / 2);
      if (nt == 0) {  // no query sees these keys
        if (row_ok) {
          uint4* a = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dv) + orow);
          uint4* c = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.dk) + orow);
#pragma unroll
          for (int e = 0; e < D / 16; ++e) a[e] = c[e] = make_uint4(0, 0, 0, 0);
        }
      } else {
        acc_half_to_global<D>(tmem + lane_addr + 256 + ch * (D / 2), static_cast<__nv_bfloat16*>(p.dv) + orow, 1.f,
                              row_ok);
        acc_half_to_global<D>(tmem + lane_addr + 256 + D + ch * (D / 2), static_cast<__nv_bfloat16*>(p.dk) + orow,
                              p.scale, row_ok);
      }
      tc_fence_before();
      mbar_arrive(bar(Lay::B_ACCEMPTY));
      tick(5);
    }
    if (!ok) fail();
#if HD_BW_TRACE
    if (threadIdx.x == 0 && blockIdx.x < kBwTraceCtas)
      for (int c = 0; c < 6; ++c) g_bw_trace[blockIdx.x * kBwTraceSlots + c] = tr[c];
#endif
  }

  __syncthreads();
  if (warp == bw::kWarpMMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, bw::kTmemCols);
  }
}

// ============================================================ dQ kernel

template <int D>
__global__ void __launch_bounds__(bw::kThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                       const BwParams p) {
  using Lay = bw::LayQ<D>;
  using T = bw::Tile<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sbase = smem_u32(smem);
  auto bar = [&](int i) -> uint32_t { return sbase + Lay::BAR_OFF + 8 * i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::MISC_OFF + 4);
  volatile int* no_abort = reinterpret_cast<volatile int*>(smem + Lay::MISC_OFF + 8);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = p.Hq / p.Hkv;

  if (threadIdx.x == 0) {
    mbar_init(bar(Lay::B_QFULL), 1);
    mbar_init(bar(Lay::B_QEMPTY), 1);
    for (int i = 0; i < Lay::KST; ++i) {
      mbar_init(bar(Lay::B_KFULL + i), 1);
      mbar_init(bar(Lay::B_KEMPTY + i), 1);
    }
    for (int i = 0; i < Lay::VST; ++i) {
      mbar_init(bar(Lay::B_VFULL + i), 1);
      mbar_init(bar(Lay::B_VEMPTY + i), 1);
    }
    mbar_init(bar(Lay::B_SFULL + 0), 1);
    mbar_init(bar(Lay::B_SFULL + 1), 1);
    mbar_init(bar(Lay::B_DPFULL), 1);
    mbar_init(bar(Lay::B_DSFULL), 256);
    mbar_init(bar(Lay::B_ACCFULL), 1);
    mbar_init(bar(Lay::B_ACCEMPTY), 256);
    mbar_init(bar(Lay::B_DRAIN), 1);
    *abort_flag = 0;
    *no_abort = 0;
    fence_barrier_init();
  }
  if (warp == bw::kWarpTMA && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  if (warp == bw::kWarpMMA) {
    tmem_alloc(smem_u32(tmem_slot), bw::kTmemCols);
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

  if (warp == bw::kWarpTMA) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int t = 0, ul = 0, q_issued = 0;
      int k_issued[Lay::KST] = {}, v_issued[Lay::VST] = {};
      bool ok = true;
      for (int k = 0, u = bw_unit_of(0, p.total_units); ok && u != -1;
           ul += (u >= 0), u = bw_unit_of(++k, p.total_units)) {
        if (u < 0) continue;  // round k has no unit for this CTA
        const QUnit x = q_unit(u, p);
        const int kvh = x.h / G;
        if (!mbar_wait(bar(Lay::B_QEMPTY), (ul & 1) ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(bar(Lay::B_QFULL), 2 * T::TILE);
#pragma unroll
        for (int kb = 0; kb < T::KB; ++kb) {
          tma_load_5d(sbase + Lay::Q_OFF + kb * T::BLK, &tmQ, bar(Lay::B_QFULL), kb * 64, x.h, x.s, x.qblk * bw::BT,
                      x.b);
          tma_load_5d(sbase + Lay::O_OFF + kb * T::BLK, &tmO, bar(Lay::B_QFULL), kb * 64, x.h, x.s, x.qblk * bw::BT,
                      x.b);
        }
        ++q_issued;
        for (int j = 0; j < x.nkt; ++j, ++t) {
          const int kt = x.kt_lo + j;
          const int ks = t % Lay::KST;
          if (!mbar_wait(bar(Lay::B_KEMPTY + ks), ((t / Lay::KST) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(Lay::B_KFULL + ks), T::TILE);
#pragma unroll
          for (int kb = 0; kb < T::KB; ++kb)
            tma_load_5d(sbase + Lay::K_OFF + ks * T::TILE + kb * T::BLK, &tmK, bar(Lay::B_KFULL + ks), kb * 64, kvh,
                        x.skv, kt * bw::BT, x.b);
          ++k_issued[ks];
          const int vs = t % Lay::VST;
          if (!mbar_wait(bar(Lay::B_VEMPTY + vs), ((t / Lay::VST) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(Lay::B_VFULL + vs), T::TILE);
#pragma unroll
          for (int kb = 0; kb < T::KB; ++kb)
            tma_load_5d(sbase + Lay::V_OFF + vs * T::TILE + kb * T::BLK, &tmV, bar(Lay::B_VFULL + vs), kb * 64, kvh,
                        x.skv, kt * bw::BT, x.b);
          ++v_issued[vs];
        }
      }
      if (!ok) {
        fail();
        if (q_issued) mbar_wait(bar(Lay::B_QFULL), (q_issued - 1) & 1, no_abort);
        for (int i = 0; i < Lay::KST; ++i)
          if (k_issued[i]) mbar_wait(bar(Lay::B_KFULL + i), (k_issued[i] - 1) & 1, no_abort);
        for (int i = 0; i < Lay::VST; ++i)
          if (v_issued[i]) mbar_wait(bar(Lay::B_VFULL + i), (v_issued[i] - 1) & 1, no_abort);
      }
    }
  } else if (warp == bw::kWarpMMA) {
    // ---------------------------------------------------------------- MMA
    // Unit start: S(t0) dP(t0) S(t0+1); per tile t: [dS(t) ready] dQ(t)
    // dP(t+1) S(t+2).  S(t) lives in buffer t&1.
    if (lane == 0) {
      const uint32_t tDP = tmem + 256, tDQ = tmem + 384;
      int t = 0, ul = 0;
      bool ok = true;
      auto issue_S = [&](int tt) -> bool {
        const int ks = tt % Lay::KST;
        if (!mbar_wait(bar(Lay::B_KFULL + ks), (tt / Lay::KST) & 1, abort_flag)) return false;
        tc_fence_after();
        mma_rows_rows<D>(tmem + (tt & 1) * 128, sbase + Lay::Q_OFF, sbase + Lay::K_OFF + ks * T::TILE);
        tc_commit(bar(Lay::B_SFULL + (tt & 1)));
        return true;
      };
      auto issue_dP = [&](int tt) -> bool {
        const int vs = tt % Lay::VST;
        if (!mbar_wait(bar(Lay::B_VFULL + vs), (tt / Lay::VST) & 1, abort_flag)) return false;
        tc_fence_after();
        mma_rows_rows<D>(tDP, sbase + Lay::O_OFF, sbase + Lay::V_OFF + vs * T::TILE);
        tc_commit(bar(Lay::B_DPFULL));
        tc_commit(bar(Lay::B_VEMPTY + vs));
        return true;
      };
      for (int k = 0, u = bw_unit_of(0, p.total_units); ok && u != -1;
           ul += (u >= 0), u = bw_unit_of(++k, p.total_units)) {
        if (u < 0) continue;  // round k has no unit for this CTA
        const QUnit x = q_unit(u, p);
        const int nt = x.nkt;
        if (!mbar_wait(bar(Lay::B_QFULL), ul & 1, abort_flag)) { ok = false; break; }
        const int t0 = t;
        if (!issue_S(t0) || !issue_dP(t0) || (nt > 1 && !issue_S(t0 + 1))) { ok = false; break; }
        for (int j = 0; j < nt; ++j, ++t) {
          if (!mbar_wait(bar(Lay::B_DSFULL), t & 1, abort_flag)) { ok = false; break; }
          if (j == 0 && ul > 0 && !mbar_wait(bar(Lay::B_ACCEMPTY), (ul - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          mma_tmem_rows<D>(tDQ, tmem + (t & 1) * 128, sbase + Lay::K_OFF + (t % Lay::KST) * T::TILE, j > 0);
          tc_commit(bar(Lay::B_KEMPTY + t % Lay::KST));
          if (j + 1 < nt && !issue_dP(t + 1)) { ok = false; break; }
          if (j + 2 < nt && !issue_S(t + 2)) { ok = false; break; }
        }
        if (!ok) break;
        tc_commit(bar(Lay::B_ACCFULL));
        tc_commit(bar(Lay::B_QEMPTY));
      }
      if (!ok) fail();
      tc_commit(bar(Lay::B_DRAIN));
      mbar_wait(bar(Lay::B_DRAIN), 0, no_abort);
    }
  } else {
    // ------------------------------------------- elementwise + epilogue
    const int ch = warp >> 2;  // column half (keys [64ch, 64ch+64) of a tile)
    const int r = (warp & 3) * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tDP = tmem + lane_addr + 256 + 64 * ch;
    const float sl2 = p.scale_log2;
    int t = 0, ul = 0;
    bool ok = true;
    for (int k = 0, u = bw_unit_of(0, p.total_units); ok && u != -1;
         ul += (u >= 0), u = bw_unit_of(++k, p.total_units)) {
      if (u < 0) continue;  // round k has no unit for this CTA
      const QUnit x = q_unit(u, p);
      const int iq = x.qblk * bw::BT + r;  // this thread's query token
      const int64_t lat = ((static_cast<int64_t>(x.b) * p.Hq + x.h) * p.g.ns + x.s) * p.Lpad + iq;
      const int piq = bw_pos(p, iq);  // key index of this thread's query
      const float2 ld = make_float2(p.ws.nl2[lat], p.ws.delta[lat]);
      for (int j = 0; j < x.nkt; ++j, ++t) {
        const int k0 = (x.kt_lo + j) * bw::BT + 64 * ch;  // first key of this half
        const uint32_t tS = tmem + lane_addr + (t & 1) * 128 + 64 * ch;
        bool got = mbar_wait(bar(Lay::B_SFULL + (t & 1)), (t >> 1) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tc_fence_after();
        uint32_t sv[64];
        tmem_ld32(tS, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_ld();
        const int qfirst = x.qblk * bw::BT;
        const bool need_mask =
            (k0 + 63 > bw_pos(p, qfirst)) || (p.W > 0 && k0 < bw_pos(p, qfirst + bw::BT - 1) - p.W + 1);
        float pv[64];
        if constexpr (bw::kPacked) {
          const uint64_t s2 = pack_f32x2(sl2, sl2), l2 = pack_f32x2(ld.x, ld.x);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            unpack_f32x2(fma_f32x2(pack_f32x2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), s2, l2),
                         pv[2 * c], pv[2 * c + 1]);
          bw::exp2_row64(pv);
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) pv[c] = ex2(fmaf(__uint_as_float(sv[c]), sl2, ld.x));
        }
        if (need_mask) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            const int jk = k0 + c;
            if (jk > piq || (p.W > 0 && piq - jk >= p.W)) pv[c] = 0.f;
          }
        }
        got = mbar_wait(bar(Lay::B_DPFULL), t & 1, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tc_fence_after();
        tmem_ld32(tDP, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(tDP + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_ld();
        {
          uint32_t pk[16];
          const uint64_t d2 = pack_f32x2(ld.y, ld.y);
          auto ds_pair = [&](int c) -> uint32_t {
            if constexpr (bw::kPacked)
              return pack_bf16x2_of(mul_f32x2(
                  pack_f32x2(pv[c], pv[c + 1]),
                  sub_f32x2(pack_f32x2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), d2)));
            else
              return pack_bf16x2(pv[c] * (__uint_as_float(sv[c]) - ld.y),
                                 pv[c + 1] * (__uint_as_float(sv[c + 1]) - ld.y));
          };
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = ds_pair(2 * e);
          tmem_st16(tS, pk);
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = ds_pair(32 + 2 * e);
          tmem_st16(tS + 16, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(Lay::B_DSFULL));
      }
      if (!ok) break;
      const bool got = mbar_wait(bar(Lay::B_ACCFULL), ul & 1, abort_flag);
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tc_fence_after();
      const bool row_ok = iq < p.g.Lq;
      const int64_t orow = ((static_cast<int64_t>(x.b) * p.g.q_ns * p.g.Lq +
                             static_cast<int64_t>(row_ok ? iq : 0) * p.g.q_ns + x.s) * p.Hq + x.h) * D +
                           ch * (D / 2);
      acc_half_to_global<D>(tmem + lane_addr + 384 + ch * (D / 2), static_cast<__nv_bfloat16*>(p.dq) + orow, p.scale,
                            row_ok);
      tc_fence_before();
      mbar_arrive(bar(Lay::B_ACCEMPTY));
    }
    if (!ok) fail();
  }

  __syncthreads();
  if (warp == bw::kWarpMMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, bw::kTmemCols);
  }
}

// ------------------------------------------------------------------- host

template <int D>
static cudaError_t launch_bwd_tc_d(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                   const CUtensorMap& mo, BwParams p, int kv_units, int q_units, int sms,
                                   cudaStream_t st) {
  cudaError_t err;
  const int skv = bw::LayKV<D>::ALLOC, sq = bw::LayQ<D>::ALLOC;
  err = cudaFuncSetAttribute(attn_bwd_dkv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, skv);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(attn_bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, sq);
  if (err != cudaSuccess) return err;
  p.total_units = kv_units;
  attn_bwd_dkv_kernel<D><<<kv_units < sms ? kv_units : sms, bw::kThreads, skv, st>>>(mq, mk, mv, mo, p);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  p.total_units = q_units;
  attn_bwd_dq_kernel<D><<<q_units < sms ? q_units : sms, bw::kThreads, sq, st>>>(mq, mk, mv, mo, p);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_tc(const void* q, const void* k, const void* v, const void* dO, BwdWs ws,
                               void* dq, void* dk, void* dv, const AttnGeom& g, int Hq, int Hkv, int D, int W,
                               float scale, int32_t* status, int sms, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mo;
  if (!encode_stream_view(&mq, q, g.B, g.Lq, g.q_ns, Hq, D) || !encode_stream_view(&mk, k, g.B, g.Lk, g.kv_ns, Hkv, D) ||
      !encode_stream_view(&mv, v, g.B, g.Lk, g.kv_ns, Hkv, D) || !encode_stream_view(&mo, dO, g.B, g.Lq, g.q_ns, Hq, D))
    return cudaErrorInvalidValue;
  BwParams p;
  p.ws = ws;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.status = status;
  p.g = g;
  p.Lpad = bwd_lpad(g.Lq);
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.W = W;
  p.nqb = p.Lpad / bw::BT;
  p.nkb = (g.Lk + bw::BT - 1) / bw::BT;
  p.kns = g.kv_stream >= 0 ? 1 : g.kv_ns;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.scale = scale;
  static const int stall = [] {
    const char* e = getenv("HD_TEST_STALL_BWD");
    return (e && e[0] == '1') ? 1 : 0;
  }();
  p.stall_first_s = stall;
  // Key streams no query reads (a single read stream of several) get zero
  // gradients; the kernel writes the read stream's.
  if (g.kv_stream >= 0 && g.kv_ns > 1) {
    const size_t bytes = static_cast<size_t>(g.B) * g.kv_ns * g.Lk * Hkv * D * 2;
    cudaError_t e = cudaMemsetAsync(dk, 0, bytes, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, bytes, st);
    if (e != cudaSuccess) return e;
  }
  const int64_t kv_units = static_cast<int64_t>(p.nkb) * g.B * p.kns * Hkv;
  const int64_t q_units = static_cast<int64_t>(p.nqb) * g.B * g.ns * Hq;
  if (q_units <= 0) return cudaSuccess;
  if (q_units > 0x7fffffff || kv_units > 0x7fffffff) return cudaErrorInvalidValue;
  if (D == 64) return launch_bwd_tc_d<64>(mq, mk, mv, mo, p, (int)kv_units, (int)q_units, sms, st);
  return launch_bwd_tc_d<128>(mq, mk, mv, mo, p, (int)kv_units, (int)q_units, sms, st);
}

#if HD_BW_TRACE
// Diagnostic build only: copy out / reset the dK/dV kernel's per-role clock
// counters (kBwTraceSlots per CTA).
extern "C" int hd_bw_trace_fetch(unsigned long long* dst, int count) {
  if (count > kBwTraceCtas * kBwTraceSlots) count = kBwTraceCtas * kBwTraceSlots;
  return static_cast<int>(cudaMemcpyFromSymbol(dst, g_bw_trace, sizeof(unsigned long long) * count));
}
extern "C" int hd_bw_trace_clear() {
  static unsigned long long zero[kBwTraceCtas * kBwTraceSlots];
  return static_cast<int>(cudaMemcpyToSymbol(g_bw_trace, zero, sizeof(zero)));
}
#endif

}  // namespace hd
