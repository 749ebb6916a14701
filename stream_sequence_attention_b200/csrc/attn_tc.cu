// Stream-Factorized Attention forward, bf16 in / f32 accumulate, on the
// 5th-generation tensor cores (tcgen05 + tensor memory) of sm_100a.
//
// ("Hidden Decoding at Scale", "Stream-Factorized Attention", Figure 2.)
// Both modes run as "ns independent causal streams of Ls tokens": intra mode
// is (ns = n, Ls = L), cross mode is (ns = 1, Ls = n*L).  The stream
// structure lives entirely in the TMA tensor maps: q/k/v [B, ns*Ls, H, D] are
// described as the 5-D tensor (D, H, ns, Ls, B), so a box of 128 tokens of
// one stream is 128 rows at stride ns*H*D -- stride-n addressing in
// hardware, no de-interleave pass, and keys of other streams are never
// loaded.  A key at token j is visible to the query at token i iff j <= i
// and (W == 0 or i - j < W); tiles entirely outside that band are never
// visited and only the diagonal / band-edge tiles are masked.
//
// Work unit: 128 query tokens of one (batch, stream) for TWO query heads of
// the same KV head (GQA), which need exactly the same K/V tiles: every K/V
// tile brought into shared memory feeds both heads.  Units are ordered
// longest-first (query block descending); the kernel is persistent, one CTA
// per SM walking units with a static stride.
//
// CTA = 10 warps:
//   warps 0-3  softmax / O-rescale / epilogue of head slot 0 (thread r owns
//              query row r = tensor-memory lane r)
//   warps 4-7  the same for head slot 1
//   warp 8     TMA producer: Q (both heads), K (3 stages), V (2 stages)
//   warp 9     MMA issuer
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O0 [256,384)
// O1 [384,512).  P (bf16, two per column) overwrites the first 64 columns of
// its S buffer.  The MMA warp issues, per tile, PV_0(t) S_0(t+1) PV_1(t)
// S_1(t+1): S_h(t+1) lands in the columns PV_h(t) reads, which is safe
// because tcgen05.mma operations issued by one thread execute in order.
// While one softmax warpgroup works, the tensor core runs the other head's
// PV and next S -- the two warpgroups ping-pong against the tensor core.
//
// Softmax: running max m per row in log2 units; O is rescaled only when a
// tile raises the max by more than 2^8 (the final 1/l makes the result
// independent of which max was used).  The row max uses 3-input max.
// On tiles without masking one exponential pair in three (tc::kPolyEvery)
// runs on the FMA pipe instead of the MUFU unit, whose 16 results per clock
// per SM would otherwise bound the softmax at the tensor core's own rate:
// the exponent is shifted and clamped by one saturating FMA per element
// (masked -inf and anything below -126 land on -126; the top of the range
// is the rescale threshold), then rounded to the nearest integer by the
// 1.5 * 2^23 constant, a cubic gives 2^f on [-1/2, 1/2] and an integer
// multiply-add puts n in the exponent field (relative error < 1e-4, below
// the bf16 rounding of P).  Masked tiles stay on the MUFU unit, which
// returns an exact 0 for -inf.
#include <climits>
#include <cstdlib>
#include <cstring>
#include <type_traits>

#include "hd_common.cuh"
#include "hd_launch.h"

namespace hd {

namespace tc {
constexpr int BM = 128;
constexpr int BN = 128;
// MMA issuers: one warp issuing for both head slots (1), or one warp per head
// slot (2), so that a head's P V and next S never wait behind the other
// head's issue order.
#ifndef HD_TC_ISSUERS
#define HD_TC_ISSUERS 1
#endif
constexpr int kIssuers = HD_TC_ISSUERS;
static_assert(kIssuers == 1 || kIssuers == 2, "one or two MMA issuers");
// Register split (1): 12 warps, the third warpgroup (producer, MMA
// issuer(s), gather, idle) gives registers to the two softmax warpgroups with
// setmaxnreg: launched at 168 per thread (65536 / 384), it drops to kRegsAux
// and the softmax warps rise to kRegsSoftmax.  (0): 10 or 11 warps, 168
// registers for every thread.
#ifndef HD_TC_REGSPLIT
#define HD_TC_REGSPLIT 0
#endif
constexpr bool kRegSplit = HD_TC_REGSPLIT != 0;
constexpr uint32_t kRegsAux = 104;
constexpr uint32_t kRegsSoftmax = 200;
static_assert(256 * kRegsSoftmax + 128 * kRegsAux <= 384 * 168, "register split exceeds the launch");
// Warps: two softmax warpgroups (0-7), the TMA producer (8), the MMA
// issuer(s) (9, and 10 with two), and in the rank-shard form with gather the
// gather warp after them.
constexpr int kThreads = kRegSplit ? 384 : 32 * (9 + kIssuers);
// Threads of a launch of the form with NM key/value sources.
__host__ __device__ constexpr int threads_of(int NM) { return kRegSplit ? 384 : (NM > 1 ? kThreads + 32 : kThreads); }
constexpr int kWarpTMA = 8;
constexpr int kWarpMMA = 9;
constexpr int kWarpGather = 9 + kIssuers;  // rank-shard form with gather only
// The MMA issuer's loop runs on all 32 lanes of its warp, one elected lane
// issuing each MMA and commit (1), or on lane 0 alone (0).
#ifndef HD_TC_MMA_WARP
#define HD_TC_MMA_WARP 1
#endif
constexpr bool kMmaWarp = HD_TC_MMA_WARP != 0;
// L2 policies on the TMA copies (1): K/V tiles, read again by every later
// query block of their group, kept (evict_last); Q tiles and the O stores,
// touched once, streamed (evict_first).  0: no policy.
#ifndef HD_TC_L2HINT
#define HD_TC_L2HINT 0
#endif
constexpr bool kL2Hint = HD_TC_L2HINT != 0;
constexpr int VST = 2;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// On tiles without masking, one exp2 pair in kPolyEvery is evaluated on the
// FMA pipe in packed f32x2 arithmetic (0 = all on the MUFU unit): with
// kPolySat its exponent is shifted and clamped by one saturating FMA per
// element and exp2_sat2 takes it from there, else exp2_fma2 (ALU clamp and
// exponent add; exponents above 0, up to the rescale threshold, included).
#ifndef HD_TC_POLY_EVERY
#define HD_TC_POLY_EVERY 3
#endif
constexpr int kPolyEvery = HD_TC_POLY_EVERY;
#ifndef HD_TC_POLY_SAT
#define HD_TC_POLY_SAT 1
#endif
constexpr bool kPolySat = HD_TC_POLY_SAT != 0;
// Optional explicit choice of the FMA-pipe pairs: bit (c mod 16) of the mask
// selects pair c of a tile row (kPolySat form; 0 = one in kPolyEvery).
#ifndef HD_TC_POLY_PAT
#define HD_TC_POLY_PAT 0
#endif
constexpr uint32_t kPolyPat = HD_TC_POLY_PAT;
// The FMA-pipe pairs also in the fused-RoPE form (1), or MUFU only there (0).
#ifndef HD_TC_ROPE_POLY
#define HD_TC_ROPE_POLY 1
#endif
constexpr bool kRopePoly = HD_TC_ROPE_POLY != 0;
// Row sums of P in packed f32x2 adds (1) or scalar adds (0).
#ifndef HD_TC_PSUM
#define HD_TC_PSUM 0
#endif
constexpr bool kPackedSum = HD_TC_PSUM != 0;
__host__ __device__ constexpr bool poly_pair(int c) {
  return kPolyPat != 0 ? ((kPolyPat >> (c & 15)) & 1u) != 0
                       : (kPolyEvery > 0 && (c % (kPolyEvery > 0 ? kPolyEvery : 1)) == kPolyEvery - 1);
}
// The two softmax warpgroups take turns (ping-pong) when nonzero.
#ifndef HD_TC_PINGPONG
#define HD_TC_PINGPONG 0
#endif
constexpr bool kPingPong = HD_TC_PINGPONG != 0;
// Epilogue: O / l leaves through shared memory, one TMA store per warp and
// 128-byte column chunk (1), or as per-thread global stores (0).
#ifndef HD_TC_TMA_STORE
#define HD_TC_TMA_STORE 1
#endif
constexpr bool kTmaStore = HD_TC_TMA_STORE != 0;
// Softmax arithmetic per tile: the exponents of the whole row first, as
// packed f32x2 FMAs, then the exponentials (1); or exponent and exponential
// column pair by column pair (0).
#ifndef HD_TC_MASK2
#define HD_TC_MASK2 1
#endif
// Masked tiles: the visible columns of a row are one interval [lo, hi] of
// the tile, so each score takes two compares against constants.
constexpr bool kMask2 = HD_TC_MASK2 != 0;
#ifndef HD_TC_EPI_ALL
#define HD_TC_EPI_ALL 1
#endif
// bf16 TMA-store epilogue: read all of O from tensor memory at once and
// release it before the stores.
constexpr bool kEpiAll = HD_TC_EPI_ALL != 0;
#ifndef HD_TC_SPLIT
#define HD_TC_SPLIT 1
#endif
constexpr bool kSplit = HD_TC_SPLIT != 0;
// Diagnostic build only: per-role clock counters (see hd_tc_trace_fetch).
#ifndef HD_TC_TRACE
#define HD_TC_TRACE 0
#endif
constexpr bool kTrace = HD_TC_TRACE != 0;

template <int D>
struct Layout {
  static constexpr int KB = D / 64;     // 128-byte column blocks per row
  static constexpr int BLK = BM * 128;  // bytes of one 128-row x 128-byte block
  static constexpr int TILE = BLK * KB; // bytes of a 128-row tile
  // K stages: 3, or 2 at D = 128 when the epilogue's staging (32 KB) takes
  // the third stage's shared memory.
  static constexpr int KST = (kTmaStore && D == 128) ? 2 : 3;
  static constexpr int Q_OFF = 0;       // head slots 0 and 1
  static constexpr int K_OFF = Q_OFF + 2 * TILE;
  static constexpr int V_OFF = K_OFF + KST * TILE;
  // Epilogue staging: one 128-row x 128-byte block per head slot (each warp
  // owns its 32 rows, 4 KB).
  static constexpr int O_OFF = V_OFF + VST * TILE;
  static constexpr int BAR_OFF = O_OFF + (kTmaStore ? 2 * BLK : 0);
  static constexpr int B_QFULL = 0, B_QEMPTY = 1, B_KFULL = 2, B_KEMPTY = B_KFULL + KST,
                       B_VFULL = B_KEMPTY + KST, B_VEMPTY = B_VFULL + VST, B_SFULL = B_VEMPTY + VST,
                       B_PFULL = B_SFULL + 2, B_ODONE = B_PFULL + 2, B_OEMPTY = B_ODONE + 2,
                       B_ORD = B_OEMPTY + 2, B_DRAIN = B_ORD + 2, B_QROT = B_DRAIN + 1, NBAR = B_QROT + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int ALLOC = BYTES + 1024;
};
}  // namespace tc

#if HD_TC_TRACE
// Per-CTA clock counters of the diagnostic build: kTraceSlots per CTA.
constexpr int kTraceCtas = 1024;
constexpr int kTraceSlots = 32;
__device__ unsigned long long g_tc_trace[kTraceCtas * kTraceSlots];
#endif

struct TcParams {
  void* o;
  float* lse;
  int32_t* status;
  AttnGeom g;
  int Hq, Hkv, W;
  float scale_log2;
  int out_bf16;
  int nqb, npairs;
  int total_units;
  // Rotary embedding of the query rows inside the kernel (the ROPE
  // instantiation): rope_half pairs in layout rope_layout (hd_rope_layout),
  // rope_fturn[j] = theta_j / (2 pi) as a 64-bit fixed-point fraction of a
  // turn; query (i, s) sits at position i * q_ns + s of the expanded
  // sequence.
  int rope_half, rope_layout;
  uint64_t rope_fturn[kRopeMaxPairs / 2];
  // Test hook (environment HD_TEST_STALL_FIRST_S=1): the MMA warp of CTA 0
  // never signals its first S tile, so the softmax wait runs out and the
  // kernel must take its timeout path.  0 in normal use.
  int stall_first_s;
};

struct TcUnit {
  int b, s, kvh, qblk, h0, h1, t_lo, t_hi;  // h1 < 0: only one head in this unit
};

// Unit schedule of a CTA: rounds of gridDim.x units in the longest-first
// order, walked forwards in even rounds and backwards in odd ones, so that
// every CTA gets a similar total (with a plain stride the first CTAs would
// always take the longest unit of each round).  Returns the k-th unit of
// this CTA, -1 when the rounds are exhausted, -2 when round k has none for
// it.  Every role walks the same sequence.
#ifndef HD_TC_SNAKE
#define HD_TC_SNAKE 1
#endif
__device__ __forceinline__ int tc_unit_of(int k, int total) {
  const int base = k * static_cast<int>(gridDim.x);
  if (base >= total) return -1;
  const int c = (HD_TC_SNAKE && (k & 1)) ? static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x)
                                         : static_cast<int>(blockIdx.x);
  return base + c < total ? base + c : -2;
}

__device__ __forceinline__ TcUnit tc_unit(int u, const TcParams& p) {
  const int G = p.Hq / p.Hkv;
  const int per = p.g.B * p.g.ns * p.Hkv * p.npairs;
  const int qi = u / per;
  int rem = u - qi * per;
  TcUnit x;
  x.qblk = p.nqb - 1 - qi;
  const int pair = rem % p.npairs;
  rem /= p.npairs;
  x.kvh = rem % p.Hkv;
  rem /= p.Hkv;
  x.s = rem % p.g.ns;
  x.b = rem / p.g.ns;
  x.h0 = x.kvh * G + 2 * pair;
  x.h1 = (2 * pair + 1 < G) ? x.h0 + 1 : -1;
  // Key range of the block: up to the key index of its last query, from the
  // window start of its first query.
  const int q0 = x.qblk * tc::BM;
  const int qlast = min(q0 + tc::BM - 1, p.g.Lq - 1);
  const int qb = p.g.qoff + x.s * p.g.qsstride;  // key index offset of this query stream
  x.t_hi = (qlast * p.g.qstride + qb) / tc::BN;
  x.t_lo = p.W > 0 ? max(0, q0 * p.g.qstride + qb - p.W + 1) / tc::BN : 0;
  return x;
}

// ------------------------------------------------- flags between CTAs

// Publish data written with ordinary stores (by the calling warp, whose
// lanes fenced and synchronised before) to readers in other CTAs that read
// it through the tensor-memory-access (async) proxy: flag += 1, release.
__device__ __forceinline__ void flag_publish(unsigned long long* f) {
  asm volatile("fence.proxy.async.global;" ::: "memory");
  asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(f) : "memory");
}

// Wait until *f >= target (acquire), then order later TMA reads after it.
// Bounded like mbar_wait.
__device__ __forceinline__ bool flag_wait_ge(const unsigned long long* f, unsigned long long target,
                                             volatile int* abort) {
  auto ready = [&]() {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(f) : "memory");
    return v >= target;
  };
  bool ok = ready();
  if (!ok) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1;; ++it) {
      if (ready()) { ok = true; break; }
      if ((it & 15) == 0) {
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
      }
    }
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return ok;
}

// Key/value sources.  NM == 1: one sequence in the expanded order (every
// regular call).  NM == kPeerMaxRanks: the R rank shards of a stream-parallel
// cross-stream layer.  Key tile [k0, k0 + 128) holds tokens k0/n .. k0/n +
// 128/n - 1 of all n streams; in rank rho's shard (local stream l = global
// stream rho + R*l at local row token*(n/R) + l) they are the contiguous rows
// [k0/R, k0/R + 128/R).  So a tile is R boxes of 128/R rows, one per shard,
// and shared-memory row c = rho*(128/R) + t holds key k0 + perm[c] with
// perm[c] = (t / (n/R))*n + rho + R*(t mod (n/R)).  The MMAs do not depend on
// the key order inside a tile (the same order feeds S and P V); only the
// mask needs perm.
struct PartsInfo {
  int R, rows, self;
  // The R shards lie at one stride in memory (kv.k[0]/kv.v[0] then view them
  // as one 5-D tensor (D, H, rows, B, R): a tile is one box per 64 features).
  int stacked;
  uint8_t perm[tc::BN];
  // In-kernel gather (flags != nullptr): the shards of ngath ranks (the
  // others, and this rank's own when gself) are copied from src to dst in
  // items of up to kPeerSub16 16-byte units, ordered key tile first;
  // flags[b*nkt + kt] counts the finished items of key tile kt of sequence
  // b, complete at per_flag.
  int ngath, gself;
  const uint4* src_k[kPeerMaxRanks];
  const uint4* src_v[kPeerMaxRanks];
  uint4* dst_k[kPeerMaxRanks];
  uint4* dst_v[kPeerMaxRanks];
  unsigned long long* flags;
  unsigned long long per_flag;
  int64_t shard_rows;
  int nkt, nsub, nitems, row16;
  // Test hook (environment HD_TEST_STALL_GATHER=1): CTA 0 never publishes
  // its first item, so a tile never becomes ready and the producer's wait
  // must run out.  0 in normal use.
  int stall_gather;
};
struct NoParts {};
template <int NM>
struct KvSrc {
  CUtensorMap k[NM];
  CUtensorMap v[NM];
  std::conditional_t<(NM > 1), PartsInfo, NoParts> x;
};

// The gather warp: copies its share of the items (item w goes to CTA
// w mod grid) with 16-byte loads, U in flight per lane, then publishes each.
// It never waits on another CTA, so with every CTA resident (cooperative
// launch) every flag is eventually published.
template <int U>
__device__ __forceinline__ void gather_items(const PartsInfo& x, int B, int lane, volatile int* abort) {
  for (int w = blockIdx.x; w < x.nitems; w += gridDim.x) {
    if (*abort) return;
    int rem = w;
    const int sub = rem % x.nsub;
    rem /= x.nsub;
    const int kind = rem & 1;
    rem >>= 1;
    const int rr = rem % x.ngath;
    rem /= x.ngath;
    const int b = rem % B;
    const int kt = rem / B;
    const int rho = x.gself ? rr : (rr < x.self ? rr : rr + 1);
    const int64_t r0 = static_cast<int64_t>(kt) * x.rows;
    const int64_t r1 = min(r0 + x.rows, x.shard_rows);
    const int64_t n16 = (r1 - r0) * x.row16;
    const int64_t s0 = static_cast<int64_t>(sub) * kPeerSub16;
    const int64_t s1 = min(s0 + kPeerSub16, n16);
    const int64_t base = (static_cast<int64_t>(b) * x.shard_rows + r0) * x.row16;
    const uint4* src = (kind ? x.src_v[rho] : x.src_k[rho]) + base;
    uint4* dst = (kind ? x.dst_v[rho] : x.dst_k[rho]) + base;
    for (int64_t i0 = s0 + lane; i0 < s1; i0 += 32 * U) {
      uint4 t[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + 32 * u < s1) t[u] = __ldcs(src + i0 + 32 * u);
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i0 + 32 * u < s1) dst[i0 + 32 * u] = t[u];
    }
    __threadfence();
    __syncwarp();
    if (lane == 0 && !(x.stall_gather && blockIdx.x == 0 && w == 0))
      flag_publish(x.flags + static_cast<int64_t>(b) * x.nkt + kt);
  }
}

// cos and sin of the angle pos * theta_j, fturn = theta_j / (2 pi) as a
// 64-bit fraction of a turn: bits 32..63 of pos * fturn (exact, mod 2^64)
// are the fraction of a turn, from two 32-bit multiplies.  Its top bit
// flipped and the next 22 bits under the exponent of 1.0f give 1.5 + the
// signed fraction in [-1/2, 1/2); one FMA turns that into the angle in
// [-pi, pi), where sin.approx / cos.approx are accurate to ~1e-6.
__device__ __forceinline__ float2 rope_cos_sin(uint32_t pos, uint64_t fturn) {
  const uint32_t t = pos * static_cast<uint32_t>(fturn >> 32) + __umulhi(pos, static_cast<uint32_t>(fturn));
  const float f = __uint_as_float((t >> 9) ^ 0x3FC00000u);
  const float a = fmaf(f, 6.28318530717958647692f, -9.42477796076937971538f);  // (f - 1.5) * 2 pi
  float sn, cn;
  asm("sin.approx.f32 %0, %1;" : "=f"(sn) : "f"(a));
  asm("cos.approx.f32 %0, %1;" : "=f"(cn) : "f"(a));
  return make_float2(cn, sn);
}

// bf16 pair (low, high half of w) as a packed f32 pair.
__device__ __forceinline__ uint64_t bf16x2_to_f32x2(uint32_t w) {
  return pack_f32x2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// Rotary embedding of one query row in place in a 128-byte-swizzled Q tile
// (row r at qrow; 64-feature blocks blk bytes apart), row position pos:
// pairs (j, j + half) or (2j, 2j + 1), j < half, (a, b) -> (a cos - b sin,
// a sin + b cos) at the angle pos * theta_j.
template <int NP>
__device__ __forceinline__ void rope_rotate_row(uint8_t* qrow, int blk, int r, uint32_t pos, int half, int layout,
                                                const uint64_t (&fturn)[NP]) {
  // 16-byte unit holding features f .. f+7 (f a multiple of 8) of the row:
  // 128-byte swizzle within each 64-feature block.
  auto unit = [&](int f) -> uint4* {
    return reinterpret_cast<uint4*>(qrow + (f >> 6) * blk + ((((f & 63) >> 3) ^ (r & 7)) << 4));
  };
  if (layout == HD_ROPE_HALF) {
    // pairs (j, j + half): the units at features j = 8v and j + half
#pragma unroll
    for (int v = 0; v < NP / 8; ++v) {
      if (8 * v < half) {
        uint4* pa = unit(8 * v);
        uint4* pb = unit(8 * v + half);
        const uint4 ua = *pa, ub = *pb;
        uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w}, wb[4] = {ub.x, ub.y, ub.z, ub.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          // features (j, j + 1) of both halves as packed pairs: a' = a c - b s,
          // b' = a s + b c
          const uint64_t a2 = bf16x2_to_f32x2(wa[e]), b2 = bf16x2_to_f32x2(wb[e]);
          const float2 t0 = rope_cos_sin(pos, fturn[8 * v + 2 * e]);
          const float2 t1 = rope_cos_sin(pos, fturn[8 * v + 2 * e + 1]);
          const uint64_t c2 = pack_f32x2(t0.x, t1.x), s2 = pack_f32x2(t0.y, t1.y);
          wa[e] = pack_bf16x2_of(sub_f32x2(mul_f32x2(a2, c2), mul_f32x2(b2, s2)));
          wb[e] = pack_bf16x2_of(fma_f32x2(a2, s2, mul_f32x2(b2, c2)));
        }
        *pa = make_uint4(wa[0], wa[1], wa[2], wa[3]);
        *pb = make_uint4(wb[0], wb[1], wb[2], wb[3]);
      }
    }
  } else {
    // pairs (2j, 2j + 1): the unit at feature 8v holds pairs 4v .. 4v + 3
#pragma unroll
    for (int v = 0; v < NP / 4; ++v) {
      if (4 * v < half) {
        uint4* pa = unit(8 * v);
        const uint4 ua = *pa;
        uint32_t wa[4] = {ua.x, ua.y, ua.z, ua.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fa = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&wa[e]));
          const float2 t = rope_cos_sin(pos, fturn[4 * v + e]);
          wa[e] = pack_bf16x2(fmaf(fa.x, t.x, -fa.y * t.y), fmaf(fa.x, t.y, fa.y * t.x));
        }
        *pa = make_uint4(wa[0], wa[1], wa[2], wa[3]);
      }
    }
  }
}

// ROPE: the query rows are rotated in the Q tile at the start of each unit
// (a separate instantiation, so the other forms carry none of its code).
template <int D, int NM, bool ROPE = false>
__global__ void __launch_bounds__(tc::threads_of(NM), 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ KvSrc<NM> kv,
                   const __grid_constant__ CUtensorMap tmO, const TcParams p) {
  using Lay = tc::Layout<D>;
  constexpr bool kParts = NM > 1;
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

  if (threadIdx.x == 0) {
    mbar_init(bar(Lay::B_QFULL), 1);
    // Stages are released by every MMA issuer.
    mbar_init(bar(Lay::B_QEMPTY), tc::kIssuers);
    for (int i = 0; i < Lay::KST; ++i) {
      mbar_init(bar(Lay::B_KFULL + i), 1);
      mbar_init(bar(Lay::B_KEMPTY + i), tc::kIssuers);
    }
    for (int i = 0; i < tc::VST; ++i) {
      mbar_init(bar(Lay::B_VFULL + i), 1);
      mbar_init(bar(Lay::B_VEMPTY + i), tc::kIssuers);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(Lay::B_SFULL + i), 1);
      mbar_init(bar(Lay::B_PFULL + i), 128);
      mbar_init(bar(Lay::B_ODONE + i), 1);
      mbar_init(bar(Lay::B_OEMPTY + i), 128);
    }
    mbar_init(bar(Lay::B_ORD + 0), 128);
    mbar_init(bar(Lay::B_ORD + 1), 128);
    mbar_init(bar(Lay::B_QROT + 0), 128);
    mbar_init(bar(Lay::B_QROT + 1), 128);
    mbar_init(bar(Lay::B_DRAIN), tc::kIssuers);
    *abort_flag = 0;
    *no_abort = 0;
    fence_barrier_init();
  }
  if (warp == tc::kWarpTMA && lane == 0) {
    tma_prefetch_desc(&tmQ);
    if (tc::kTmaStore) tma_prefetch_desc(&tmO);
#pragma unroll
    for (int i = 0; i < NM; ++i) {
      if constexpr (kParts) {
        if (i >= (kv.x.stacked ? 1 : kv.x.R)) break;
      }
      tma_prefetch_desc(&kv.k[i]);
      tma_prefetch_desc(&kv.v[i]);
    }
  }
  if (warp == tc::kWarpMMA) {
    tmem_alloc(smem_u32(tmem_slot), tc::kTmemCols);
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
  // One 128-key tile of K or V into the stage at `dst`.
  auto load_kv_tile = [&](const CUtensorMap* maps, uint32_t dst, uint32_t full, const TcUnit& x, int skv, int kt,
                          uint64_t pol) {
    if constexpr (kParts) {
      if (kv.x.stacked) {
        // One box covers the tile's rows of every rank, rank-major.
#pragma unroll
        for (int kb = 0; kb < Lay::KB; ++kb)
          tma_load_5d(dst + kb * Lay::BLK, &maps[0], full, kb * 64, x.kvh, kt * kv.x.rows, x.b, 0);
      } else {
#pragma unroll
        for (int rho = 0; rho < NM; ++rho) {
          if (rho >= kv.x.R) break;
#pragma unroll
          for (int kb = 0; kb < Lay::KB; ++kb)
            tma_load_5d(dst + kb * Lay::BLK + rho * kv.x.rows * 128, &maps[rho], full, kb * 64, x.kvh, 0,
                        kt * kv.x.rows, x.b);
        }
      }
    } else {
#pragma unroll
      for (int kb = 0; kb < Lay::KB; ++kb) {
        if constexpr (tc::kL2Hint)
          tma_load_5d_hint(dst + kb * Lay::BLK, &maps[0], full, kb * 64, x.kvh, skv, kt * tc::BN, x.b, pol);
        else
          tma_load_5d(dst + kb * Lay::BLK, &maps[0], full, kb * 64, x.kvh, skv, kt * tc::BN, x.b);
      }
    }
  };

  if (warp >= 8) {
  // Producer, MMA issuer, gather (each warp its own role).
  if constexpr (tc::kRegSplit) regs_decrease<tc::kRegsAux>();
  if (warp == tc::kWarpTMA) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const uint64_t pol_keep = tc::kL2Hint ? l2_policy_evict_last() : 0;
      const uint64_t pol_once = tc::kL2Hint ? l2_policy_evict_first() : 0;
      auto load = [&](uint32_t dst, const CUtensorMap* m, uint32_t b, int c0, int c1, int c2, int c3, int c4,
                      uint64_t pol) {
        if constexpr (tc::kL2Hint)
          tma_load_5d_hint(dst, m, b, c0, c1, c2, c3, c4, pol);
        else
          tma_load_5d(dst, m, b, c0, c1, c2, c3, c4);
      };
      int t = 0, ul = 0, q_issued = 0;
      int k_issued[Lay::KST] = {}, v_issued[tc::VST] = {};
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int u = tc_unit_of(k, p.total_units);
        if (u == -1) break;
        if (u < 0) continue;
        const TcUnit x = tc_unit(u, p);
        if (!mbar_wait(bar(Lay::B_QEMPTY), (ul & 1) ^ 1, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(bar(Lay::B_QFULL), Lay::TILE * (x.h1 >= 0 ? 2 : 1));
#pragma unroll
        for (int kb = 0; kb < Lay::KB; ++kb) {
          load(sbase + Lay::Q_OFF + kb * Lay::BLK, &tmQ, bar(Lay::B_QFULL), kb * 64, x.h0, x.s, x.qblk * tc::BM,
               x.b, pol_once);
          if (x.h1 >= 0)
            load(sbase + Lay::Q_OFF + Lay::TILE + kb * Lay::BLK, &tmQ, bar(Lay::B_QFULL), kb * 64, x.h1, x.s,
                 x.qblk * tc::BM, x.b, pol_once);
        }
        ++q_issued;
        const int skv = p.g.kv_stream >= 0 ? p.g.kv_stream : x.s;
        for (int kt = x.t_lo; kt <= x.t_hi; ++kt, ++t) {
          if constexpr (kParts) {
            // Gathered shards: wait until every item of this key tile landed.
            if (kv.x.flags &&
                !flag_wait_ge(kv.x.flags + static_cast<int64_t>(x.b) * kv.x.nkt + kt, kv.x.per_flag, abort_flag)) {
              ok = false;
              break;
            }
          }
          const int ks = t % Lay::KST;
          if (!mbar_wait(bar(Lay::B_KEMPTY + ks), ((t / Lay::KST) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(Lay::B_KFULL + ks), Lay::TILE);
          load_kv_tile(kv.k, sbase + Lay::K_OFF + ks * Lay::TILE, bar(Lay::B_KFULL + ks), x, skv, kt, pol_keep);
          ++k_issued[ks];
          const int vs = t % tc::VST;
          if (!mbar_wait(bar(Lay::B_VEMPTY + vs), ((t / tc::VST) & 1) ^ 1, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(bar(Lay::B_VFULL + vs), Lay::TILE);
          load_kv_tile(kv.v, sbase + Lay::V_OFF + vs * Lay::TILE, bar(Lay::B_VFULL + vs), x, skv, kt, pol_keep);
          ++v_issued[vs];
        }
        ++ul;
      }
      if (!ok) {
        fail();
        // Let every copy already issued land before the CTA can exit.
        if (q_issued) mbar_wait(bar(Lay::B_QFULL), (q_issued - 1) & 1, no_abort);
        for (int i = 0; i < Lay::KST; ++i)
          if (k_issued[i]) mbar_wait(bar(Lay::B_KFULL + i), (k_issued[i] - 1) & 1, no_abort);
        for (int i = 0; i < tc::VST; ++i)
          if (v_issued[i]) mbar_wait(bar(Lay::B_VFULL + i), (v_issued[i] - 1) & 1, no_abort);
      }
    }
  } else if (warp >= tc::kWarpMMA && warp < tc::kWarpMMA + tc::kIssuers) {
    // ---------------------------------------------------------------- MMA
    // With one issuer the order per tile t is PV_0(t) S_0(t+1) PV_1(t)
    // S_1(t+1); with two, each issues PV_h(t) S_h(t+1) for its own head
    // slot h.  S_h(t+1) overwrites the columns P_h(t) occupies; tcgen05.mma
    // from one thread executes in issue order, so PV_h(t) has read P_h(t) by
    // then.  Each issuer releases every Q/K/V stage once (its commit, or a
    // plain arrive when it has no head in the unit).
    if (tc::kMmaWarp || lane == 0) {
      // One lane issues (the loop on lane 0, or the whole warp's loop with an
      // elected lane per MMA and commit).
      auto mma_s = [&](uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc) {
        if constexpr (tc::kMmaWarp)
          mma_ss_elect(d, a, b, id, acc);
        else
          mma_ss(d, a, b, id, acc);
      };
      auto mma_t = [&](uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc) {
        if constexpr (tc::kMmaWarp)
          mma_ts_elect(d, a, b, id, acc);
        else
          mma_ts(d, a, b, id, acc);
      };
      auto commit = [&](uint32_t b) {
        if constexpr (tc::kMmaWarp)
          tc_commit_elect(b);
        else
          tc_commit(b);
      };
      constexpr uint32_t idS = idesc_bf16_f32(tc::BM, tc::BN, false, false);
      constexpr uint32_t idO = idesc_bf16_f32(tc::BM, D, false, true);
      const int me = warp - tc::kWarpMMA;  // issuer index
      auto issue_S = [&](int h, int kst) {
        // Descriptors once per tile; the K-steps add their byte offset / 16.
        const uint64_t qd = smem_desc_sw128(sbase + Lay::Q_OFF + h * Lay::TILE, 16, 1024);
        const uint64_t kd = smem_desc_sw128(sbase + Lay::K_OFF + kst * Lay::TILE, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off16 = ((kk >> 2) * Lay::BLK + (kk & 3) * 32) >> 4;
          mma_s(tmem + h * 128, qd + off16, kd + off16, idS, kk > 0 ? 1u : 0u);
        }
        if (!(p.stall_first_s && blockIdx.x == 0)) commit(bar(Lay::B_SFULL + h));
      };
      auto issue_PV = [&](int h, int vst, bool acc) {
        // V tile is MN-major (D contiguous): 16 keys = 16 rows of 128 B.
        const uint64_t vd = smem_desc_sw128(sbase + Lay::V_OFF + vst * Lay::TILE, Lay::BLK, 1024);
#pragma unroll
        for (int kk = 0; kk < tc::BN / 16; ++kk)
          mma_t(tmem + 256 + h * 128, tmem + h * 128 + kk * 8, vd + ((kk * 2048) >> 4), idO,
                 (acc || kk > 0) ? 1u : 0u);
      };
      int t = 0, ul = 0;
      int ts[2] = {0, 0};  // P_h V MMAs issued per head slot
      int us[2] = {0, 0};  // units per head slot
      bool ok = true;
      // Diagnostic counters (HD_TC_TRACE): waiting for P, for Q/K/V/O, total.
      unsigned long long mw[3] = {0, 0, 0};
      const long long mt0 = tc::kTrace ? clock64() : 0;
      auto timed_wait = [&](int which, uint32_t b, uint32_t par) {
        if constexpr (tc::kTrace) {
          const long long t0 = clock64();
          const bool r = mbar_wait(b, par, abort_flag);
          mw[which] += static_cast<unsigned long long>(clock64() - t0);
          return r;
        } else {
          return mbar_wait(b, par, abort_flag);
        }
      };
      for (int k = 0; ok; ++k) {
        const int u = tc_unit_of(k, p.total_units);
        if (u == -1) break;
        if (u < 0) continue;
        const TcUnit x = tc_unit(u, p);
        // Head slots this issuer serves in this unit: [h_lo, h_hi).
        const int h_lo = tc::kIssuers == 2 ? me : 0;
        const int h_hi = tc::kIssuers == 2 ? (me == 0 || x.h1 >= 0 ? me + 1 : me) : (x.h1 >= 0 ? 2 : 1);
        const bool mine = h_hi > h_lo;
        auto release = [&](uint32_t b) {
          if (mine)
            commit(b);
          else if (lane == 0)
            mbar_arrive(b);
        };
        const int nt = x.t_hi - x.t_lo + 1;
        if (!timed_wait(1, bar(Lay::B_QFULL), ul & 1)) { ok = false; break; }
        if constexpr (ROPE) {
          // The softmax warps rotate their query rows in place first.
          for (int h = h_lo; h < h_hi; ++h)
            if (!timed_wait(1, bar(Lay::B_QROT + h), us[h] & 1)) { ok = false; break; }
          if (!ok) break;
        }
        {
          const int ks = t % Lay::KST;
          if (!timed_wait(1, bar(Lay::B_KFULL + ks), (t / Lay::KST) & 1)) { ok = false; break; }
          tc_fence_after();
          for (int h = h_lo; h < h_hi; ++h) issue_S(h, ks);
          release(bar(Lay::B_KEMPTY + ks));
          if (nt == 1) release(bar(Lay::B_QEMPTY));
        }
        for (int jj = 0; ok && jj < nt; ++jj, ++t) {
          const int vs = t % tc::VST;
          if (!timed_wait(1, bar(Lay::B_VFULL + vs), (t / tc::VST) & 1)) { ok = false; break; }
          const bool nxt = jj + 1 < nt;
          const int ksn = (t + 1) % Lay::KST;
          // An issuer with no head in the unit still sees each stage full
          // before it releases it.
          if (!mine && nxt && !timed_wait(1, bar(Lay::B_KFULL + ksn), ((t + 1) / Lay::KST) & 1)) {
            ok = false;
            break;
          }
          for (int h = h_lo; h < h_hi; ++h) {
            if (!timed_wait(0, bar(Lay::B_PFULL + h), ts[h] & 1)) { ok = false; break; }
            if (jj == 0 && us[h] > 0 && !timed_wait(1, bar(Lay::B_OEMPTY + h), (us[h] - 1) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_PV(h, vs, jj > 0);
            ++ts[h];
            if (nxt) {
              if (h == h_lo && !timed_wait(1, bar(Lay::B_KFULL + ksn), ((t + 1) / Lay::KST) & 1)) {
                ok = false;
                break;
              }
              issue_S(h, ksn);
            } else {
              commit(bar(Lay::B_ODONE + h));
            }
          }
          if (!ok) break;
          release(bar(Lay::B_VEMPTY + vs));
          if (nxt) {
            release(bar(Lay::B_KEMPTY + ksn));
            if (jj + 1 == nt - 1) release(bar(Lay::B_QEMPTY));
          }
        }
        for (int h = h_lo; h < h_hi; ++h) us[h]++;
        ++ul;
      }
      if (!ok) fail();
      // Drain: every MMA issued above has completed before TMEM is freed.
      commit(bar(Lay::B_DRAIN));
      mbar_wait(bar(Lay::B_DRAIN), 0, no_abort);
#if HD_TC_TRACE
      mw[2] = static_cast<unsigned long long>(clock64() - mt0);
      if (blockIdx.x < kTraceCtas && lane == 0)
        for (int c = 0; c < 3; ++c) g_tc_trace[blockIdx.x * kTraceSlots + 24 + 3 * me + c] = mw[c];
#endif
    }
  } else if (warp == tc::kWarpGather) {
    // ------------------------------------------------------------- gather
    if constexpr (kParts) {
      if (kv.x.flags) gather_items<16>(kv.x, p.g.B, lane, abort_flag);
    }
  }
  } else {
    // ------------------------------------------------- softmax + epilogue
    if constexpr (tc::kRegSplit) regs_increase<tc::kRegsSoftmax>();
    const int slot = warp >> 2;
    const int r = threadIdx.x & 127;  // tensor-memory lane
    const uint32_t lane_addr = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t sS = tmem + lane_addr + slot * 128;        // S_h, then P_h
    const uint32_t sO = tmem + lane_addr + 256 + slot * 128;  // O_h
    const float sl2 = p.scale_log2;
    int sc = 0, uc = 0, oc = 0;
    bool ok = true;
    bool stored = false;  // this warp has TMA stores in flight (lane 0)
    // Diagnostic counters (HD_TC_TRACE): wait for S, score load, max and
    // mask, exponents to P published, row sum, epilogue wait for the last
    // P V, rest of the epilogue, tiles; then the score load to P published
    // on masked tiles and their count, and on a unit's first tile.
    unsigned long long tr[12] = {0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0, 0};
    long long tfrom = 0;
    long long tmark = tc::kTrace ? clock64() : 0;
    auto tick = [&](int i) {
      if constexpr (tc::kTrace) {
        const long long t = clock64();
        tr[i] += static_cast<unsigned long long>(t - tmark);
        tmark = t;
      }
    };
    int uall = 0;  // units of this CTA so far (phases of B_QFULL)
    int rot_done = -1;  // unit slot k whose query rows this warpgroup rotated ahead
    // ROPE: rotate this thread's query row of unit xr (the uq-th unit of the
    // CTA, B_QFULL phase uq & 1) in the Q tile, then publish the tile to the
    // MMA issuer ("Multi-Stream Expansion and Training Objective": contiguous
    // positions over the expanded sequence).
    auto rotate_q = [&](const TcUnit& xr, int uq) -> bool {
      const bool got = mbar_wait(bar(Lay::B_QFULL), uq & 1, abort_flag);
      if (!__all_sync(0xffffffffu, got)) return false;
      const int ir = xr.qblk * tc::BM + r;
      if (ir < p.g.Lq)
        rope_rotate_row(smem + Lay::Q_OFF + slot * Lay::TILE + r * 128, Lay::BLK, r,
                        static_cast<uint32_t>(ir * p.g.q_ns + xr.s), p.rope_half, p.rope_layout, p.rope_fturn);
      // The tensor core reads the tile through the async proxy.
      fence_proxy_async_smem();
      mbar_arrive(bar(Lay::B_QROT + slot));
      return true;
    };
    for (int k = 0; ok; ++k) {
      const int u = tc_unit_of(k, p.total_units);
      if (u == -1) break;
      if (u < 0) continue;
      const int ucur = uall++;
      const TcUnit x = tc_unit(u, p);
      const int h = slot ? x.h1 : x.h0;
      if (h < 0) continue;  // uniform across the warpgroup
      const bool paired = x.h1 >= 0;
      const int q0 = x.qblk * tc::BM;
      const int i = q0 + r;
      const int qb = p.g.qoff + x.s * p.g.qsstride;  // key index offset of this query stream
      const int pi = i * p.g.qstride + qb;             // key index of this row's query
      const int pfirst = q0 * p.g.qstride + qb;         // ... of the block's first query
      const int plast = (q0 + tc::BM - 1) * p.g.qstride + qb;
      float m = -INFINITY, l = 0.f;
      const int nt = x.t_hi - x.t_lo + 1;
      if constexpr (ROPE) {
        // Rotated ahead at the end of the previous unit, or now.
        if (rot_done != k && !rotate_q(x, ucur)) {
          ok = false;
          break;
        }
      }
      for (int jj = 0; jj < nt; ++jj, ++sc) {
        const int k0 = (x.t_lo + jj) * tc::BN;
        if (tc::kTrace) tmark = clock64();
        bool got = mbar_wait(bar(Lay::B_SFULL + slot), sc & 1, abort_flag);
        // Ping-pong: the two warpgroups take turns for the softmax arithmetic
        // (slot 0 first), so each runs alone on the SM sub-partitions while
        // the tensor core works on the other head.
        if (tc::kPingPong && got && paired) {
          if (slot == 1)
            got = mbar_wait(bar(Lay::B_ORD + 1), oc & 1, abort_flag);
          else if (oc > 0)
            got = mbar_wait(bar(Lay::B_ORD + 0), (oc - 1) & 1, abort_flag);
        }
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        tick(0);
        tc_fence_after();
        uint32_t sv[128];
        tmem_ld32(sS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(sS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_ld32(sS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
        tmem_ld32(sS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
        tmem_wait_ld();
        tick(1);
        if (tc::kTrace) tfrom = tmark;
        const bool need_mask = (k0 + tc::BN - 1 > pfirst) || (p.W > 0 && k0 < plast - p.W + 1);
        if (need_mask) {
          if constexpr (tc::kMask2 && !kParts) {
            // Column c holds key k0 + c: visible for k0 + c <= pi and, with
            // a window, pi - (k0 + c) < W.
            const int hi = pi - k0;
            const int lo = p.W > 0 ? pi - p.W + 1 - k0 : INT_MIN;
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c > hi || c < lo) sv[c] = __float_as_uint(-INFINITY);
          } else {
#pragma unroll
            for (int c = 0; c < 128; ++c) {
              int j = k0 + c;
              if constexpr (kParts) j = k0 + kv.x.perm[c];
              if (j > pi || (p.W > 0 && pi - j >= p.W)) sv[c] = __float_as_uint(-INFINITY);
            }
          }
        }
        // Row max of the raw scores (scale > 0 commutes with max): 3-input
        // max, 4 independent chains.
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 128; c += 2)
          mx[(c >> 1) & 3] = fmax3(mx[(c >> 1) & 3], __uint_as_float(sv[c]), __uint_as_float(sv[c + 1]));
        const float mraw = fmax3(fmax3(mx[0], mx[1], mx[2]), mx[3], mx[3]);
        const float mt = mraw * sl2;  // -inf stays -inf
        bool resc = false;
        float alpha = 1.f;
        if (jj == 0) {
          m = mt;
        } else if (mt > m + tc::kRescaleThreshold) {
          alpha = ex2(m - mt);
          l *= alpha;
          m = mt;
          resc = true;
        }
        const float nmu = (m == -INFINITY) ? 0.f : -m;
        tick(2);
        // P = 2^(s*scale - m) as bf16 pairs, written over the S columns 16 at
        // a time (column 16j of P holds S columns 32j.. already consumed).
        float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        uint64_t ls2[4] = {0, 0, 0, 0};  // packed pairs of 0.f
        if ((tc::kPolyEvery > 0 || tc::kPolyPat != 0) && tc::kPolySat && tc::kSplit && (!ROPE || tc::kRopePoly) &&
            !need_mask) {
          // The exponent x = s * scale * log2 e - m lies in [-inf, T] (T =
          // kRescaleThreshold: the max is raised only past it): the FMA-pipe
          // pairs take y = sat((x + 126) / (126 + T)), the rest x itself.
          constexpr int kHi = static_cast<int>(tc::kRescaleThreshold);
          static_assert(kHi == tc::kRescaleThreshold, "integral threshold");
          constexpr float kInvSpan = 1.f / (126.f + kHi);
          const uint64_t s2 = pack_f32x2(sl2, sl2), n2 = pack_f32x2(nmu, nmu);
          const float k1 = sl2 * kInvSpan, k2 = (nmu + 126.f) * kInvSpan;
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            if (tc::poly_pair(c)) {
              sv[2 * c] = __float_as_uint(fma_sat(__uint_as_float(sv[2 * c]), k1, k2));
              sv[2 * c + 1] = __float_as_uint(fma_sat(__uint_as_float(sv[2 * c + 1]), k1, k2));
            } else {
              float a0, a1;
              unpack_f32x2(fma_f32x2(pack_f32x2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), s2, n2),
                           a0, a1);
              sv[2 * c] = __float_as_uint(a0);
              sv[2 * c + 1] = __float_as_uint(a1);
            }
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int c = 16 * j + e;
              float p0, p1;
              if (tc::poly_pair(c)) {
                unpack_f32x2(exp2_sat2<kHi>(pack_f32x2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1]))), p0,
                             p1);
              } else {
                p0 = ex2(__uint_as_float(sv[2 * c]));
                p1 = ex2(__uint_as_float(sv[2 * c + 1]));
              }
              if constexpr (tc::kPackedSum) {
                ls2[e & 3] = add_f32x2(ls2[e & 3], pack_f32x2(p0, p1));
              } else {
                ls[e & 7] += p0 + p1;
              }
              pk[e] = pack_bf16x2(p0, p1);
            }
            tmem_st16(sS + 16 * j, pk);
          }
          if constexpr (tc::kPackedSum) {
#pragma unroll
            for (int e = 0; e < 4; ++e) unpack_f32x2(ls2[e], ls[2 * e], ls[2 * e + 1]);
          }
        } else {
        if constexpr (tc::kSplit) {
          const uint64_t s2 = pack_f32x2(sl2, sl2), n2 = pack_f32x2(nmu, nmu);
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            float a0, a1;
            unpack_f32x2(fma_f32x2(pack_f32x2(__uint_as_float(sv[2 * c]), __uint_as_float(sv[2 * c + 1])), s2, n2),
                         a0, a1);
            sv[2 * c] = __float_as_uint(a0);
            sv[2 * c + 1] = __float_as_uint(a1);
          }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = 16 * j + e;
            float a0, a1;
            if constexpr (tc::kSplit) {
              a0 = __uint_as_float(sv[2 * c]);
              a1 = __uint_as_float(sv[2 * c + 1]);
            } else {
              a0 = fmaf(__uint_as_float(sv[2 * c]), sl2, nmu);
              a1 = fmaf(__uint_as_float(sv[2 * c + 1]), sl2, nmu);
            }
            float p0, p1;
            if (tc::kPolyEvery > 0 && !tc::kPolySat && !need_mask &&
                (e % (tc::kPolyEvery > 0 ? tc::kPolyEvery : 1)) == tc::kPolyEvery - 1) {
              // this pair on the FMA pipe (unmasked tiles: no -inf exponent)
              unpack_f32x2(exp2_fma2(a0, a1), p0, p1);
            } else {
              p0 = ex2(a0);
              p1 = ex2(a1);
            }
            ls[e & 7] += p0 + p1;
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(sS + 16 * j, pk);
        }
        }
        if (tc::kPingPong && paired) {
          mbar_arrive(bar(Lay::B_ORD + (slot ^ 1)));
          ++oc;
        }
        if (__any_sync(0xffffffffu, resc)) {
          // O_h is stable: the commit that signalled S_h of this tile also
          // covers the P_h V MMA issued before it.
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t ov[32];
            tmem_ld32(sO + c * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st32(sO + c * 32, ov);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(Lay::B_PFULL + slot));
        tick(3);
        if constexpr (tc::kTrace) {
          const unsigned long long d = static_cast<unsigned long long>(tmark - tfrom);
          if (need_mask) {
            tr[8] += d;
            ++tr[9];
          }
          if (jj == 0) tr[10] += d;
        }
        l += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
        if constexpr (ROPE) {
          // After the unit's last P: rotate the next unit's query rows while
          // the tensor core runs this unit's last P V, so that the next S can
          // start right behind it.  Q(next) is on its way: the last S of this
          // unit has released the tile.
          if (jj == nt - 1) {
            int k2 = k + 1, u2;
            while ((u2 = tc_unit_of(k2, p.total_units)) == -2) ++k2;
            if (u2 >= 0) {
              const TcUnit x2 = tc_unit(u2, p);
              if ((slot ? x2.h1 : x2.h0) >= 0) {
                if (!rotate_q(x2, uall)) {
                  ok = false;
                  break;
                }
                rot_done = k2;
              }
            }
          }
        }
        tick(4);
        if (tc::kTrace) ++tr[7];
      }
      if (!ok) break;
      // Epilogue: O / l -> global once the last P V MMA of this head is done.
      const bool got = mbar_wait(bar(Lay::B_ODONE + slot), uc & 1, abort_flag);
      ++uc;
      if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
      tick(5);
      tc_fence_after();
      const float inv = 1.f / l;
      const bool row_ok = i < p.g.Lq;
      if constexpr (tc::kTmaStore) {
        // O / l by 128-byte column chunks: this warp's 32 rows of a chunk go
        // through its own 4 KB of staging (128-byte swizzle, the layout of
        // the tensor map) and out with one TMA store; rows past Lq are
        // clipped by it.  The tensor memory is released after the last
        // chunk's load.
        const int wq = warp & 3;
        uint8_t* stg = smem + Lay::O_OFF + slot * Lay::BLK + wq * 32 * 128;
        const uint32_t stg_s = smem_u32(stg);
        const int row0 = q0 + 32 * wq;
        const int rl = r & 31;
        auto put = [&](int chunk, const uint4* w) {
          if (lane == 0 && stored) bulk_wait_group_read<0>();
          __syncwarp();
#pragma unroll
          for (int uu = 0; uu < 8; ++uu)
            *reinterpret_cast<uint4*>(stg + rl * 128 + ((uu ^ (rl & 7)) << 4)) = w[uu];
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < p.g.Lq) {
            if constexpr (tc::kL2Hint)
              tma_store_5d_hint(&tmO, stg_s, chunk * (p.out_bf16 ? 64 : 32), h, x.s, row0, x.b,
                                l2_policy_evict_first());
            else
              tma_store_5d(&tmO, stg_s, chunk * (p.out_bf16 ? 64 : 32), h, x.s, row0, x.b);
            bulk_commit_group();
            stored = true;
          }
        };
        if (tc::kEpiAll && p.out_bf16) {
          uint32_t ov[D];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) tmem_ld32(sO + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[c * 32]));
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar(Lay::B_OEMPTY + slot));
#pragma unroll
          for (int ch = 0; ch < D / 64; ++ch) {
            uint4 w[8];
#pragma unroll
            for (int uu = 0; uu < 8; ++uu) {
              const int c0 = ch * 64 + uu * 8;
              w[uu].x = pack_bf16x2(__uint_as_float(ov[c0 + 0]) * inv, __uint_as_float(ov[c0 + 1]) * inv);
              w[uu].y = pack_bf16x2(__uint_as_float(ov[c0 + 2]) * inv, __uint_as_float(ov[c0 + 3]) * inv);
              w[uu].z = pack_bf16x2(__uint_as_float(ov[c0 + 4]) * inv, __uint_as_float(ov[c0 + 5]) * inv);
              w[uu].w = pack_bf16x2(__uint_as_float(ov[c0 + 6]) * inv, __uint_as_float(ov[c0 + 7]) * inv);
            }
            put(ch, w);
          }
        } else if (p.out_bf16) {
#pragma unroll
          for (int ch = 0; ch < D / 64; ++ch) {
            uint32_t ov[64];
            tmem_ld32(sO + ch * 64, *reinterpret_cast<uint32_t(*)[32]>(&ov[0]));
            tmem_ld32(sO + ch * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[32]));
            tmem_wait_ld();
            if (ch == D / 64 - 1) {
              tc_fence_before();
              mbar_arrive(bar(Lay::B_OEMPTY + slot));
            }
            uint4 w[8];
#pragma unroll
            for (int uu = 0; uu < 8; ++uu) {
              const int c0 = uu * 8;
              w[uu].x = pack_bf16x2(__uint_as_float(ov[c0 + 0]) * inv, __uint_as_float(ov[c0 + 1]) * inv);
              w[uu].y = pack_bf16x2(__uint_as_float(ov[c0 + 2]) * inv, __uint_as_float(ov[c0 + 3]) * inv);
              w[uu].z = pack_bf16x2(__uint_as_float(ov[c0 + 4]) * inv, __uint_as_float(ov[c0 + 5]) * inv);
              w[uu].w = pack_bf16x2(__uint_as_float(ov[c0 + 6]) * inv, __uint_as_float(ov[c0 + 7]) * inv);
            }
            put(ch, w);
          }
        } else {
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t ov[32];
            tmem_ld32(sO + ch * 32, ov);
            tmem_wait_ld();
            if (ch == D / 32 - 1) {
              tc_fence_before();
              mbar_arrive(bar(Lay::B_OEMPTY + slot));
            }
            uint4 w[8];
#pragma unroll
            for (int uu = 0; uu < 8; ++uu)
              w[uu] = make_uint4(__float_as_uint(__uint_as_float(ov[4 * uu + 0]) * inv),
                                 __float_as_uint(__uint_as_float(ov[4 * uu + 1]) * inv),
                                 __float_as_uint(__uint_as_float(ov[4 * uu + 2]) * inv),
                                 __float_as_uint(__uint_as_float(ov[4 * uu + 3]) * inv));
            put(ch, w);
          }
        }
      } else {
        const int64_t orow =
            (static_cast<int64_t>(x.b) * p.g.o_rows + static_cast<int64_t>(i) * p.g.o_ns + x.s) * p.Hq + h;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(sO + c * 32, ov);
          tmem_wait_ld();
          if (row_ok) {
            if (p.out_bf16) {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + orow * D + c * 32);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(ov[8 * e + 0]) * inv, __uint_as_float(ov[8 * e + 1]) * inv);
                w.y = pack_bf16x2(__uint_as_float(ov[8 * e + 2]) * inv, __uint_as_float(ov[8 * e + 3]) * inv);
                w.z = pack_bf16x2(__uint_as_float(ov[8 * e + 4]) * inv, __uint_as_float(ov[8 * e + 5]) * inv);
                w.w = pack_bf16x2(__uint_as_float(ov[8 * e + 6]) * inv, __uint_as_float(ov[8 * e + 7]) * inv);
                dst[e] = w;
              }
            } else {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow * D + c * 32);
#pragma unroll
              for (int e = 0; e < 8; ++e)
                dst[e] = make_float4(__uint_as_float(ov[4 * e + 0]) * inv, __uint_as_float(ov[4 * e + 1]) * inv,
                                     __uint_as_float(ov[4 * e + 2]) * inv, __uint_as_float(ov[4 * e + 3]) * inv);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(bar(Lay::B_OEMPTY + slot));
      }
      if (row_ok && p.lse)
        p.lse[(static_cast<int64_t>(x.b) * p.Hq + h) * p.g.o_rows + static_cast<int64_t>(i) * p.g.o_ns + x.s] =
            (m + log2f(l)) * 0.69314718055994531f;
      tick(6);
    }
    // Every TMA store has finished reading its staging before the CTA's
    // shared memory can go away.
    if (tc::kTmaStore && lane == 0 && stored) bulk_wait_group<0>();
    if (!ok) fail();
#if HD_TC_TRACE
    if (r == 0 && blockIdx.x < kTraceCtas)
      for (int c = 0; c < 12; ++c) g_tc_trace[blockIdx.x * kTraceSlots + slot * 12 + c] = tr[c];
#endif
  }

  __syncthreads();
  if (warp == tc::kWarpMMA) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, tc::kTmemCols);
  }
}

// ------------------------------------------------------------------- host

// (D, H, ns, Ls, B) view of a [B, ns*Ls, H, D] bf16 tensor; box = 64 x 1 x 1 x rows x 1
// with rows = 128 (kind 1) or the key's `pad` (kind 3: one rank's part of a key tile).
static bool make_stream_view(const TmapKey& k, CUtensorMap* m) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  const cuuint64_t B = k.dims[0], Ls = k.dims[1], ns = k.dims[2], H = k.dims[3], D = k.dims[4];
  const cuuint64_t dims[5] = {D, H, ns, Ls, B};
  const cuuint64_t e = 2;
  const cuuint64_t strides[4] = {D * e, H * D * e, ns * H * D * e, Ls * ns * H * D * e};
  const cuuint32_t rows = k.kind == 3 ? static_cast<cuuint32_t>(k.pad) : static_cast<cuuint32_t>(tc::BM);
  const cuuint32_t box[5] = {64, 1, 1, rows, 1};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(k.ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// (D, H, ns, Ls, B) view of the output [B, ns*Ls, H, D], bf16 or f32 (element
// bytes in the key's `pad`), with a box of one 128-byte column chunk x 32
// rows: one warp's share of the epilogue's TMA stores.
static bool make_out_view(const TmapKey& k, CUtensorMap* m) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  const cuuint64_t B = k.dims[0], Ls = k.dims[1], ns = k.dims[2], H = k.dims[3], D = k.dims[4];
  const cuuint64_t e = static_cast<cuuint64_t>(k.pad);
  const cuuint64_t dims[5] = {D, H, ns, Ls, B};
  const cuuint64_t strides[4] = {D * e, H * D * e, ns * H * D * e, Ls * ns * H * D * e};
  const cuuint32_t box[5] = {static_cast<cuuint32_t>(128 / e), 1, 1, 32, 1};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, e == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 5, const_cast<void*>(k.ptr),
             dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The output view of a call's geometry (o [B, o_rows, Hq, D] with query (i, s)
// at row i*o_ns + s, o_rows = o_ns*Lq); all zero when the epilogue stores
// per thread.
static bool encode_out_view(CUtensorMap* m, void* o, const AttnGeom& g, int Hq, int D, bool out_bf16) {
  std::memset(m, 0, sizeof(*m));
  if (!tc::kTmaStore) return true;
  if (static_cast<int64_t>(g.o_ns) * g.Lq != g.o_rows) return false;
  TmapKey k;
  std::memset(&k, 0, sizeof(k));
  k.ptr = o;
  k.dims[0] = g.B;
  k.dims[1] = g.Lq;
  k.dims[2] = g.o_ns;
  k.dims[3] = Hq;
  k.dims[4] = D;
  k.kind = 6;
  k.pad = out_bf16 ? 2 : 4;
  return tmap_cached(k, m, make_out_view);
}

bool encode_stream_view(CUtensorMap* m, const void* ptr, int B, int Ls, int ns, int H, int D) {
  TmapKey k;
  std::memset(&k, 0, sizeof(k));
  k.ptr = ptr;
  k.dims[0] = B;
  k.dims[1] = Ls;
  k.dims[2] = ns;
  k.dims[3] = H;
  k.dims[4] = D;
  k.kind = 1;
  return tmap_cached(k, m, make_stream_view);
}

// R rank shards [B, rows, H, D] at a stride of `step` bytes, viewed as the 5-D
// tensor (D, H, rows, B, R) with a box of 64 x 1 x box_rows x 1 x R.
static bool make_stacked_view(const TmapKey& k, CUtensorMap* m) {
  EncodeTiledFn enc = get_encode_tiled();
  if (!enc) return false;
  const cuuint64_t B = k.dims[0], rows = k.dims[1], R = k.dims[2], H = k.dims[3], D = k.dims[4];
  const cuuint64_t e = 2;
  const cuuint64_t dims[5] = {D, H, rows, B, R};
  const cuuint64_t strides[4] = {D * e, H * D * e, rows * H * D * e, static_cast<cuuint64_t>(k.extra)};
  const cuuint32_t box[5] = {64, 1, static_cast<cuuint32_t>(k.pad), 1, static_cast<cuuint32_t>(R)};
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(k.ptr), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool encode_stacked_view(CUtensorMap* m, const void* ptr, int B, int64_t rows, int R, int H, int D,
                                int box_rows, int64_t step) {
  TmapKey k;
  std::memset(&k, 0, sizeof(k));
  k.ptr = ptr;
  k.dims[0] = B;
  k.dims[1] = rows;
  k.dims[2] = R;
  k.dims[3] = H;
  k.dims[4] = D;
  k.kind = 5;
  k.pad = box_rows;
  k.extra = step;
  return tmap_cached(k, m, make_stacked_view);
}

// Stride of R addresses in arithmetic progression (a positive multiple of 16
// bytes, at least `min_step`), or 0.
static int64_t stack_step(const void* const* a, int R, int64_t min_step) {
  if (R < 2) return 0;
  const int64_t d = reinterpret_cast<intptr_t>(a[1]) - reinterpret_cast<intptr_t>(a[0]);
  if (d < min_step || d % 16 || d >= (static_cast<int64_t>(1) << 40)) return 0;
  for (int i = 2; i < R; ++i)
    if (reinterpret_cast<intptr_t>(a[i]) - reinterpret_cast<intptr_t>(a[i - 1]) != d) return 0;
  return d;
}

// One rank shard [B, rows, H, D] with a box of `box_rows` rows.
static bool encode_shard_view(CUtensorMap* m, const void* ptr, int B, int64_t rows, int H, int D, int box_rows) {
  TmapKey k;
  std::memset(&k, 0, sizeof(k));
  k.ptr = ptr;
  k.dims[0] = B;
  k.dims[1] = rows;
  k.dims[2] = 1;
  k.dims[3] = H;
  k.dims[4] = D;
  k.kind = 3;
  k.pad = box_rows;
  return tmap_cached(k, m, make_stream_view);
}

int attn_tc_smem_bytes(int D) { return D == 64 ? tc::Layout<64>::ALLOC : tc::Layout<128>::ALLOC; }

// Parameters common to both forms; false if the unit count overflows.
static bool fill_params(TcParams& p, void* o, float* lse, const AttnGeom& g, int Hq, int Hkv, int W, float scale,
                        bool out_bf16, int32_t* status) {
  p.o = o;
  p.lse = lse;
  p.status = status;
  p.g = g;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.W = W;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.out_bf16 = out_bf16 ? 1 : 0;
  p.nqb = (g.Lq + tc::BM - 1) / tc::BM;
  const int G = Hq / Hkv;
  p.npairs = (G + 1) / 2;
  const int64_t units = static_cast<int64_t>(p.nqb) * g.B * g.ns * Hkv * p.npairs;
  if (units < 0 || units > 0x7fffffff) return false;
  p.total_units = static_cast<int>(units);
  static const int stall = [] {
    const char* e = getenv("HD_TEST_STALL_FIRST_S");
    return (e && e[0] == '1') ? 1 : 0;
  }();
  p.stall_first_s = stall;
  p.rope_half = 0;
  p.rope_layout = 0;
  return true;
}

cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, void* o, float* lse, const AttnGeom& g,
                           int Hq, int Hkv, int D, int W, float scale, bool out_bf16, int32_t* status, int sms,
                           cudaStream_t st, const RopeParams* rope) {
  CUtensorMap mq, mo;
  KvSrc<1> kv;
  if (!encode_stream_view(&mq, q, g.B, g.Lq, g.q_ns, Hq, D) ||
      !encode_stream_view(&kv.k[0], k, g.B, g.Lk, g.kv_ns, Hkv, D) ||
      !encode_stream_view(&kv.v[0], v, g.B, g.Lk, g.kv_ns, Hkv, D) || !encode_out_view(&mo, o, g, Hq, D, out_bf16))
    return cudaErrorInvalidValue;
  TcParams p;
  if (!fill_params(p, o, lse, g, Hq, Hkv, W, scale, out_bf16, status)) return cudaErrorInvalidValue;
  if (p.total_units == 0) return cudaSuccess;
  if (rope) {
    const int half = rope->rot / 2;
    if (half < 4 || half > kRopeMaxPairs / 2 || half % 4 || 2 * half > D ||
        (rope->layout == HD_ROPE_HALF && half % 8))
      return cudaErrorInvalidValue;
    p.rope_half = half;
    p.rope_layout = rope->layout;
    for (int j = 0; j < half; ++j) p.rope_fturn[j] = rope->fturn[j];
  }
  const int grid = p.total_units < sms ? p.total_units : sms;
  const int smem = attn_tc_smem_bytes(D);
  auto go = [&](auto kernel) {
    cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return err;
    kernel<<<grid, tc::threads_of(1), smem, st>>>(mq, kv, mo, p);
    return cudaGetLastError();
  };
  if (rope) return D == 64 ? go(attn_tc_kernel<64, 1, true>) : go(attn_tc_kernel<128, 1, true>);
  return D == 64 ? go(attn_tc_kernel<64, 1>) : go(attn_tc_kernel<128, 1>);
}

int64_t parts_flag_count(int B, int n, int L) {
  return static_cast<int64_t>(B) * ((static_cast<int64_t>(n) * L + tc::BN - 1) / tc::BN);
}

template <int D>
static cudaError_t launch_parts_kernel(const CUtensorMap& mq, const KvSrc<kPeerMaxRanks>& kv, const CUtensorMap& mo,
                                       const TcParams& p, int grid, bool cooperative, cudaStream_t st) {
  const int smem = attn_tc_smem_bytes(D);
  cudaError_t err =
      cudaFuncSetAttribute(attn_tc_kernel<D, kPeerMaxRanks>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(tc::threads_of(kPeerMaxRanks));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = cooperative ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, attn_tc_kernel<D, kPeerMaxRanks>, mq, kv, mo, p);
}

cudaError_t launch_attn_tc_parts(const void* q, const PartsArgs& a, void* o, float* lse, const AttnGeom& g, int n,
                                 int Hq, int Hkv, int D, int W, float scale, bool out_bf16, int32_t* status, int sms,
                                 cudaStream_t st) {
  const int R = a.R;
  if (R < 1 || R > kPeerMaxRanks || n % R || tc::BN % n || a.self < 0 || a.self >= R) return cudaErrorInvalidValue;
  const int nl = n / R;
  const int L = g.Lq;
  const int rows = tc::BN / R;
  const int64_t shard_rows = static_cast<int64_t>(nl) * L;
  const bool gather = R > 1 && a.k_dst[0 == a.self ? 1 : 0] != nullptr;
  const bool gself = gather && a.k_dst[a.self] != nullptr && a.v_dst[a.self] != nullptr;
  CUtensorMap mq, mo;
  if (!encode_stream_view(&mq, q, g.B, g.Lq, g.q_ns, Hq, D) || !encode_out_view(&mo, o, g, Hq, D, out_bf16))
    return cudaErrorInvalidValue;
  KvSrc<kPeerMaxRanks> kv;
  std::memset(&kv, 0, sizeof(kv));
  PartsInfo& x = kv.x;
  // The shards the attention reads: the copies where the kernel gathers them.
  const void* rk[kPeerMaxRanks];
  const void* rv[kPeerMaxRanks];
  for (int rho = 0; rho < R; ++rho) {
    const bool copied = gather && (rho != a.self || gself);
    rk[rho] = copied ? a.k_dst[rho] : a.k_src[rho];
    rv[rho] = copied ? a.v_dst[rho] : a.v_src[rho];
    x.src_k[rho] = static_cast<const uint4*>(a.k_src[rho]);
    x.src_v[rho] = static_cast<const uint4*>(a.v_src[rho]);
    x.dst_k[rho] = static_cast<uint4*>(a.k_dst[rho]);
    x.dst_v[rho] = static_cast<uint4*>(a.v_dst[rho]);
  }
  const int64_t shard_bytes = static_cast<int64_t>(g.B) * shard_rows * Hkv * D * 2;
  const int64_t sk = stack_step(rk, R, shard_bytes), sv = stack_step(rv, R, shard_bytes);
  x.stacked = sk > 0 && sv > 0;
  if (x.stacked) {
    if (!encode_stacked_view(&kv.k[0], rk[0], g.B, shard_rows, R, Hkv, D, rows, sk) ||
        !encode_stacked_view(&kv.v[0], rv[0], g.B, shard_rows, R, Hkv, D, rows, sv))
      return cudaErrorInvalidValue;
  } else {
    for (int rho = 0; rho < R; ++rho)
      if (!encode_shard_view(&kv.k[rho], rk[rho], g.B, shard_rows, Hkv, D, rows) ||
          !encode_shard_view(&kv.v[rho], rv[rho], g.B, shard_rows, Hkv, D, rows))
        return cudaErrorInvalidValue;
  }
  x.R = R;
  x.rows = rows;
  x.self = a.self;
  x.ngath = gather ? (gself ? R : R - 1) : 0;
  x.gself = gself ? 1 : 0;
  for (int c = 0; c < tc::BN; ++c) {
    const int rho = c / rows, t = c % rows;
    x.perm[c] = static_cast<uint8_t>((t / nl) * n + rho + R * (t % nl));
  }
  x.shard_rows = shard_rows;
  x.nkt = static_cast<int>((static_cast<int64_t>(n) * L + tc::BN - 1) / tc::BN);
  x.row16 = Hkv * D * 2 / 16;
  const int64_t tile16 = static_cast<int64_t>(rows) * x.row16;
  x.nsub = static_cast<int>((tile16 + kPeerSub16 - 1) / kPeerSub16);
  x.flags = gather ? a.flags : nullptr;
  x.per_flag = static_cast<unsigned long long>(2 * x.ngath) * x.nsub;
  const int64_t items = gather ? static_cast<int64_t>(x.nkt) * g.B * x.ngath * 2 * x.nsub : 0;
  if (items > 0x7fffffff) return cudaErrorInvalidValue;
  x.nitems = static_cast<int>(items);
  static const int stall = [] {
    const char* e = getenv("HD_TEST_STALL_GATHER");
    return (e && e[0] == '1') ? 1 : 0;
  }();
  x.stall_gather = stall;
  TcParams p;
  if (!fill_params(p, o, lse, g, Hq, Hkv, W, scale, out_bf16, status)) return cudaErrorInvalidValue;
  if (p.total_units == 0) return cudaSuccess;
  if (gather) {
    if (!a.flags) return cudaErrorInvalidValue;
    cudaError_t err = cudaMemsetAsync(a.flags, 0, parts_flag_count(g.B, n, L) * sizeof(unsigned long long), st);
    if (err != cudaSuccess) return err;
  }
  const int grid = p.total_units < sms ? p.total_units : sms;
  // A producer may wait for an item of any CTA: all CTAs must be resident.
  return D == 64 ? launch_parts_kernel<64>(mq, kv, mo, p, grid, gather, st)
                 : launch_parts_kernel<128>(mq, kv, mo, p, grid, gather, st);
}

#if HD_TC_TRACE
// Diagnostic build only: copy (or clear) the per-CTA clock counters.
extern "C" int hd_tc_trace_fetch(unsigned long long* dst, int count) {
  if (count > kTraceCtas * kTraceSlots) count = kTraceCtas * kTraceSlots;
  return static_cast<int>(cudaMemcpyFromSymbol(dst, g_tc_trace, sizeof(unsigned long long) * count));
}
extern "C" int hd_tc_trace_clear() {
  static unsigned long long zeros[kTraceCtas * kTraceSlots];
  return static_cast<int>(cudaMemcpyToSymbol(g_tc_trace, zeros, sizeof(zeros)));
}
#endif

}  // namespace hd
