// Host-side launchers shared between the C-ABI shim and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace hd {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's tensor-map encoder (fetched once through the runtime).
EncodeTiledFn get_encode_tiled();

cudaError_t launch_expand(const void* tables, const int32_t* ids, void* out, int64_t rows, int n,
                          int64_t V, int row_bytes, int sms, int32_t* status, cudaStream_t st);
cudaError_t launch_gather(const void* h, void* out, int64_t rows, int n, int row_bytes, int sms,
                          cudaStream_t st);
// Geometry of one attention call, common to both attention kernels.  The
// kernels walk query tokens i in [0, Lq) of ns query streams s.  Query token
// i of stream s reads the key stream kv_stream (or s when kv_stream < 0),
// where it sits at key index pos(i, s) = i*qstride + qoff + s*qsstride; key j
// is visible iff j <= pos(i, s) and, with a window W > 0, pos(i, s) - j < W.
//   q   [B, q_ns*Lq, Hq, D]    query (i, s) is row i*q_ns + s
//   k,v [B, kv_ns*Lk, Hkv, D]  key (j, t) is row j*kv_ns + t
//   o   [B, o_rows, Hq, D]     query (i, s) writes row i*o_ns + s
//   lse [B, Hq, o_rows]
struct AttnGeom {
  int B;
  int ns, Lq, q_ns;
  int kv_ns, Lk, kv_stream;
  int qstride, qoff;
  int qsstride = 0;
  int o_rows, o_ns;
};

// Cache of encoded TMA maps (tmap_cache.cu).  The key is zero-initialised
// and compared bytewise: base pointer, the view's dimensions, and a kind tag
// naming the view (box and layout).
struct TmapKey {
  const void* ptr;
  int64_t dims[5];
  int32_t kind;
  int32_t pad;
  int64_t extra;  // kind-specific (the rank stride of a stacked shard view)
};
bool tmap_cached(const TmapKey& key, CUtensorMap* out, bool (*make)(const TmapKey&, CUtensorMap*));

// TMA view (D, H, ns, Ls, B) of a [B, ns*Ls, H, D] bf16 tensor with a
// 64 x 1 x 1 x 128 x 1 box and 128-byte swizzle: one box is 128 tokens of one
// stream and head, 64 features wide.
bool encode_stream_view(CUtensorMap* m, const void* ptr, int B, int Ls, int ns, int H, int D);

cudaError_t launch_attn_f32(const float* q, const float* k, const float* v, void* o, float* lse,
                            const AttnGeom& g, int Hq, int Hkv, int D, int W, float scale, bool out_bf16,
                            cudaStream_t st);
struct RopeParams;
// rope (nullable): the query rows are rotated inside the kernel, row (i, s)
// at position i*q_ns + s (regular geometry only), with rope->rot, ->layout
// and ->fturn as for launch_rope.
cudaError_t launch_attn_tc(const void* q, const void* k, const void* v, void* o, float* lse, const AttnGeom& g,
                           int Hq, int Hkv, int D, int W, float scale, bool out_bf16, int32_t* status, int sms,
                           cudaStream_t st, const RopeParams* rope = nullptr);

// Cross-stream prefill of one rank's queries (geometry as for the shard
// call) with the keys/values held as R rank shards [B, (n/R)*L, Hkv, D]
// instead of one interleaved sequence.  n must divide 128 (a 128-key tile is
// 128/R rows of every shard).  Without gather (k_dst == nullptr) every shard
// is read where it lies.  With gather, shard rho != self is copied once from
// k_src[rho] to k_dst[rho] inside the kernel (overlapped with the attention,
// published per (batch, key tile) through `flags`) and read from k_dst.
constexpr int kPeerMaxRanks = 8;
constexpr int kPeerSub16 = 1024;  // 16-byte units per gather item (16 KiB)
struct PartsArgs {
  int R, self;
  const void* k_src[kPeerMaxRanks];
  const void* v_src[kPeerMaxRanks];
  void* k_dst[kPeerMaxRanks];  // all nullptr: no gather; [self] optional (then
  void* v_dst[kPeerMaxRanks];  // the own shard is copied there as well)
  unsigned long long* flags;   // [B * key tiles], zeroed by the launcher
};
int64_t parts_flag_count(int B, int n, int L);
cudaError_t launch_attn_tc_parts(const void* q, const PartsArgs& a, void* o, float* lse, const AttnGeom& g, int n,
                                 int Hq, int Hkv, int D, int W, float scale, bool out_bf16, int32_t* status, int sms,
                                 cudaStream_t st);

// Backward.  Regular geometry only (qstride 1, qoff 0, kv_stream -1, the
// key streams equal the query streams).  The workspace holds two float
// planes, -lse * log2 e (so P = 2^(s scale log2 e + nl2) is one FMA and an
// exponential) and delta = <dO, o>, each indexed ((b*Hq + h)*ns + s)*Lpad + i
// with Lpad = Lq rounded up to 128; the padding rows are (-inf, 0) so they
// contribute nothing.  Separate planes let a kernel fetch four consecutive
// tokens' values in one 16-byte load.
constexpr int kBwdPad = 128;
__host__ __device__ inline int bwd_lpad(int Lq) { return (Lq + kBwdPad - 1) / kBwdPad * kBwdPad; }
struct BwdWs {
  float* nl2;
  float* delta;
};
inline int64_t bwd_plane(const AttnGeom& g, int Hq) { return static_cast<int64_t>(g.B) * Hq * g.ns * bwd_lpad(g.Lq); }
inline BwdWs bwd_ws(void* base, const AttnGeom& g, int Hq) {
  float* p = static_cast<float*>(base);
  return BwdWs{p, p + bwd_plane(g, Hq)};
}
cudaError_t launch_bwd_prep(const void* o, const void* dO, const float* lse, BwdWs ws, const AttnGeom& g, int Hq,
                            int D, bool bf16, cudaStream_t st);
cudaError_t launch_attn_bwd_f32(const float* q, const float* k, const float* v, const float* dO, BwdWs ws,
                                float* dq, float* dk, float* dv, const AttnGeom& g, int Hq, int Hkv, int D, int W,
                                float scale, cudaStream_t st);
cudaError_t launch_attn_bwd_tc(const void* q, const void* k, const void* v, const void* dO, BwdWs ws,
                               void* dq, void* dk, void* dv, const AttnGeom& g, int Hq, int Hkv, int D, int W,
                               float scale, int32_t* status, int sms, cudaStream_t st);

// Rotary embedding (rope.cu).  fturn[j] = theta_j / (2 pi) as a 64-bit
// fixed-point fraction of a turn, theta_j = base^(-2j/rot), j < rot/2.
constexpr int kRopeMaxPairs = 128;
struct RopeParams {
  void* q;
  void* k;
  const int32_t* pos0;
  int B, P, Hq, Hkv, D, rot, layout;
  int64_t pos_base, pos_mult;
  uint64_t fturn[kRopeMaxPairs];
};
cudaError_t launch_rope(const RopeParams& p, bool bf16, cudaStream_t st);
// theta_j / (2 pi) as 64-bit fixed-point turns into p.fturn (j < rot/2).
void rope_fill_turns(RopeParams& p, int rot_dim, double base);

// Stream parallelism: re-interleave rank shards (copy rows of row_bytes),
// and merge partial softmax results over disjoint key sets.
cudaError_t launch_stream_interleave(const void* parts, void* out, int64_t rows, int n, int R, int row_bytes,
                                     int sms, cudaStream_t st);
cudaError_t launch_attn_combine(const void* o_parts, const float* lse_parts, void* o, float* lse, int R,
                                int64_t rows, int D, bool in_bf16, bool out_bf16, cudaStream_t st);
// The same merge for rank r's own stream rows only, each part given by its
// own pointer ([B, n, Hq, D] and [B, n, Hq]; peer memory allowed).
cudaError_t launch_attn_combine_streams(const void* const* o_parts, const float* const* lse_parts, void* o,
                                        float* lse, int R, int B, int n, int Hq, int D, int r, bool in_bf16,
                                        bool out_bf16, cudaStream_t st);

// Decode work decomposition: units (one KV head of one sequence, and for
// intra mode one stream), row groups of at most 32 query rows, token splits.
struct DecPlan {
  int units, rg_count, nsplit, mt;
  int64_t rows_total;
};
DecPlan decode_plan(int B, int n, int Lmax, int Hq, int Hkv, bool cross, int sms);
size_t decode_workspace_bytes(const DecPlan& pl);
// Cross-stream decode on tcgen05 (decode_tc.cu), D = 128: the n*G query rows
// of a KV head in groups of at most 32.  Writes nsplit partials to the split
// workspace (the same format as the warp-MMA decode kernel).
bool decode_tc_supported(int n, int Hq, int Hkv, int D, bool cross);
int decode_tc_nsplit(int units, int Lmax, int cap, int sms);
cudaError_t launch_decode_tc(const void* q, const void* kc, const void* vc, const int32_t* ctx, float* ws_o,
                             float* ws_lse, int B, int n, int Lmax, int Hq, int Hkv, int W, float scale, int nsplit,
                             int32_t* status, cudaStream_t st, int nc, int soff, int sstride);
// nc, soff, sstride: the cache holds nc streams, local stream l being global
// stream soff + sstride*l (stream parallelism, cross mode); nc = 0 means the
// whole cache (nc = n, soff = 0, sstride = 1).
cudaError_t launch_decode(const void* q, const void* kc, const void* vc, const int32_t* ctx, void* o,
                          float* lse, int B, int n, int Lmax, int Hq, int Hkv, int W, float scale,
                          bool cross, bool out_bf16, void* ws, int32_t* status, int sms, cudaStream_t st,
                          int nc = 0, int soff = 0, int sstride = 1);

}  // namespace hd
