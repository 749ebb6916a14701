// C ABI of the library (include/hd.h): argument checks, the mode -> stream
// view mapping, and dispatch to the kernels.  Nothing here allocates device
// memory or synchronises (the IPC calls only map and unmap other processes'
// allocations).
#include <cmath>
#include <cstring>
#include <mutex>

#include "hd_common.cuh"
#include "hd_launch.h"

namespace hd {

// The driver's tensor-map encoder, fetched through the runtime so the
// library does not link libcuda directly.
EncodeTiledFn get_encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// SM count of the current device, cached per device.
int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 0;
  if (dev < 64 && cache[dev] > 0) return cache[dev];
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < 64) cache[dev] = v;
  return v;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static int esize(hd_dtype dt) { return dt == HD_BF16 ? 2 : 4; }

static bool valid_dtype(hd_dtype dt) { return dt == HD_F32 || dt == HD_BF16; }

static hd_status cuda_status(cudaError_t e) { return e == cudaSuccess ? HD_OK : HD_ERR_CUDA; }

}  // namespace hd

using namespace hd;

extern "C" {

hd_status hd_expand_embed(const void* tables, const int32_t* ids, void* out, int B, int L, int n, int64_t V,
                          int d, hd_dtype dt, int32_t* dev_status, void* stream) {
  if (B < 0 || L < 0 || n < 1 || V < 1 || d < 1 || !valid_dtype(dt)) return HD_ERR_INVALID_ARG;
  const int64_t row_bytes = static_cast<int64_t>(d) * esize(dt);
  if (row_bytes % 16 || row_bytes > (1 << 30)) return HD_ERR_INVALID_ARG;
  const int64_t rows = static_cast<int64_t>(B) * L * n;
  if (rows == 0) return HD_OK;
  // The kernel reads ids one int32 at a time: 4-byte alignment suffices
  // (a view such as ids[:, 1:] is accepted).
  if (!tables || !ids || !out || !aligned16(tables) || !aligned16(out) || (reinterpret_cast<uintptr_t>(ids) & 3u))
    return HD_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return HD_ERR_CUDA;
  return cuda_status(launch_expand(tables, ids, out, rows, n, V, static_cast<int>(row_bytes), sms, dev_status,
                                   static_cast<cudaStream_t>(stream)));
}

hd_status hd_final_stream_gather(const void* h, void* out, int B, int L, int n, int d, hd_dtype dt,
                                 void* stream) {
  if (B < 0 || L < 0 || n < 1 || d < 1 || !valid_dtype(dt)) return HD_ERR_INVALID_ARG;
  const int64_t row_bytes = static_cast<int64_t>(d) * esize(dt);
  if (row_bytes % 16 || row_bytes > (1 << 30)) return HD_ERR_INVALID_ARG;
  const int64_t rows = static_cast<int64_t>(B) * L;
  if (rows == 0) return HD_OK;
  if (!h || !out || !aligned16(h) || !aligned16(out)) return HD_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return HD_ERR_CUDA;
  return cuda_status(
      launch_gather(h, out, rows, n, static_cast<int>(row_bytes), sms, static_cast<cudaStream_t>(stream)));
}

// Argument checks shared by both attention entry points.
static hd_status check_attn_args(const void* q, const void* k, const void* v, void* o, float* lse, int B, int L,
                                 int n, int Hq, int Hkv, int D, hd_mode mode, int window, float scale,
                                 hd_dtype in_dt, hd_dtype out_dt) {
  if (B < 0 || L < 1 || n < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || window < 0) return HD_ERR_INVALID_ARG;
  if (mode != HD_INTRA && mode != HD_CROSS) return HD_ERR_INVALID_ARG;
  if (!valid_dtype(in_dt) || !valid_dtype(out_dt) || !std::isfinite(scale) || !(scale > 0.f))
    return HD_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return HD_ERR_UNSUPPORTED;
  const int64_t P = static_cast<int64_t>(n) * L;
  if (P > (1ll << 30) || static_cast<int64_t>(B) * P * Hq > (1ll << 40)) return HD_ERR_INVALID_ARG;
  if (B == 0) return HD_OK;
  if (!q || !k || !v || !o || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return HD_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return HD_ERR_INVALID_ARG;
  return HD_OK;
}

// Regular (all-query) geometry of hd_attn_fwd for the given mode.
static AttnGeom regular_geom(int B, int L, int n, hd_mode mode) {
  const int P = n * L;
  AttnGeom g;
  g.B = B;
  g.ns = mode == HD_INTRA ? n : 1;
  g.Lq = mode == HD_INTRA ? L : P;
  g.q_ns = g.ns;
  g.kv_ns = g.ns;
  g.Lk = g.Lq;
  g.kv_stream = -1;
  g.qstride = 1;
  g.qoff = 0;
  g.o_rows = P;
  g.o_ns = g.ns;
  return g;
}

// Queries: the L final-stream rows.  Intra: they read stream n-1 of the
// interleaved K/V in place.  Cross: query i sits at position i*n + n-1 of the
// single nL-position stream.
static AttnGeom final_stream_geom(int B, int L, int n, hd_mode mode) {
  AttnGeom g;
  g.B = B;
  g.ns = 1;
  g.Lq = L;
  g.q_ns = 1;
  g.o_rows = L;
  g.o_ns = 1;
  if (mode == HD_INTRA) {
    g.kv_ns = n;
    g.Lk = L;
    g.kv_stream = n - 1;
    g.qstride = 1;
    g.qoff = 0;
  } else {
    g.kv_ns = 1;
    g.Lk = n * L;
    g.kv_stream = -1;
    g.qstride = n;
    g.qoff = n - 1;
  }
  return g;
}

static hd_status run_attn(const void* q, const void* k, const void* v, void* o, float* lse, const AttnGeom& g,
                          int Hq, int Hkv, int D, int window, float scale, hd_dtype in_dt, hd_dtype out_dt,
                          int32_t* dev_status, void* stream) {
  const bool out_bf16 = out_dt == HD_BF16;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (in_dt == HD_F32) {
    if (static_cast<int64_t>(Hq) * g.ns > 65535 || g.B > 65535) return HD_ERR_UNSUPPORTED;
    return cuda_status(launch_attn_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                                       static_cast<const float*>(v), o, lse, g, Hq, Hkv, D, window, scale, out_bf16,
                                       st));
  }
  const int sms = sm_count();
  if (sms <= 0) return HD_ERR_CUDA;
  return cuda_status(launch_attn_tc(q, k, v, o, lse, g, Hq, Hkv, D, window, scale, out_bf16, dev_status, sms, st));
}

hd_status hd_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int L, int n,
                      int Hq, int Hkv, int D, hd_mode mode, int window, float scale, hd_dtype in_dt,
                      hd_dtype out_dt, int32_t* dev_status, void* stream) {
  hd_status stt = check_attn_args(q, k, v, o, lse, B, L, n, Hq, Hkv, D, mode, window, scale, in_dt, out_dt);
  if (stt != HD_OK || B == 0) return stt;
  // Intra: n streams of L tokens, read in place.  Cross: one stream of n*L positions.
  const AttnGeom g = regular_geom(B, L, n, mode);
  return run_attn(q, k, v, o, lse, g, Hq, Hkv, D, window, scale, in_dt, out_dt, dev_status, stream);
}

hd_status hd_attn_fwd_final_stream(const void* q_final, const void* k, const void* v, void* o, float* lse, int B,
                                   int L, int n, int Hq, int Hkv, int D, hd_mode mode, int window, float scale,
                                   hd_dtype in_dt, hd_dtype out_dt, int32_t* dev_status, void* stream) {
  hd_status stt = check_attn_args(q_final, k, v, o, lse, B, L, n, Hq, Hkv, D, mode, window, scale, in_dt, out_dt);
  if (stt != HD_OK || B == 0) return stt;
  const AttnGeom g = final_stream_geom(B, L, n, mode);
  return run_attn(q_final, k, v, o, lse, g, Hq, Hkv, D, window, scale, in_dt, out_dt, dev_status, stream);
}

size_t hd_attn_bwd_workspace(int B, int L, int n, int Hq, hd_mode mode) {
  if (B < 1 || L < 1 || n < 1 || Hq < 1 || (mode != HD_INTRA && mode != HD_CROSS)) return 0;
  if (static_cast<int64_t>(n) * L > (1ll << 30)) return 0;
  const AttnGeom g = regular_geom(B, L, n, mode);
  return static_cast<size_t>(2 * bwd_plane(g, Hq)) * sizeof(float);
}

hd_status hd_attn_fwd_rope(const void* q, void* k, const void* v, void* o, float* lse, int B, int L, int n, int Hq,
                           int Hkv, int D, hd_mode mode, int window, float scale, int rot_dim, double base,
                           hd_rope_layout layout, hd_dtype in_dt, hd_dtype out_dt, int32_t* dev_status,
                           void* stream) {
  hd_status stt = check_attn_args(q, k, v, o, lse, B, L, n, Hq, Hkv, D, mode, window, scale, in_dt, out_dt);
  if (stt != HD_OK) return stt;
  if (layout != HD_ROPE_HALF && layout != HD_ROPE_INTERLEAVED) return HD_ERR_INVALID_ARG;
  if (rot_dim < 8 || rot_dim > D || rot_dim % (layout == HD_ROPE_HALF ? 16 : 8)) return HD_ERR_INVALID_ARG;
  if (!std::isfinite(base) || !(base > 0.0)) return HD_ERR_INVALID_ARG;
  if (in_dt != HD_BF16) return HD_ERR_UNSUPPORTED;
  if (B == 0) return HD_OK;
  const int sms = sm_count();
  if (sms <= 0) return HD_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RopeParams rp;
  std::memset(&rp, 0, sizeof(rp));
  rp.q = nullptr;
  rp.k = k;
  rp.pos0 = nullptr;
  rp.B = B;
  rp.P = n * L;
  rp.Hq = 0;
  rp.Hkv = Hkv;
  rp.D = D;
  rp.rot = rot_dim;
  rp.layout = layout;
  rp.pos_base = 0;
  rp.pos_mult = 0;
  rope_fill_turns(rp, rot_dim, base);
  // k rotated in place (what a cache of this layer keeps); the query rows
  // rotated inside the attention kernel.
  if (launch_rope(rp, true, st) != cudaSuccess) return HD_ERR_CUDA;
  const AttnGeom g = regular_geom(B, L, n, mode);
  return cuda_status(launch_attn_tc(q, k, v, o, lse, g, Hq, Hkv, D, window, scale, out_dt == HD_BF16, dev_status,
                                    sms, st, &rp));
}

static hd_status run_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO,
                              const float* lse, void* dq, void* dk, void* dv, const AttnGeom& g, int Hq, int Hkv,
                              int D, int window, float scale, hd_dtype dt, void* workspace, size_t ws_bytes,
                              int32_t* dev_status, void* stream) {
  if (!o || !dO || !lse || !dk || !dv || !workspace || !aligned16(o) || !aligned16(dO) || !aligned16(dk) ||
      !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return HD_ERR_INVALID_ARG;
  if (ws_bytes < static_cast<size_t>(2 * bwd_plane(g, Hq)) * sizeof(float)) return HD_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const BwdWs ws = bwd_ws(workspace, g, Hq);
  const bool bf16 = dt == HD_BF16;
  cudaError_t e = launch_bwd_prep(o, dO, lse, ws, g, Hq, D, bf16, st);
  if (e != cudaSuccess) return HD_ERR_CUDA;
  if (!bf16) {
    if (static_cast<int64_t>(Hq) * g.ns > 65535 || static_cast<int64_t>(Hkv) * g.kv_ns > 65535 || g.B > 65535)
      return HD_ERR_UNSUPPORTED;
    return cuda_status(launch_attn_bwd_f32(static_cast<const float*>(q), static_cast<const float*>(k),
                                           static_cast<const float*>(v), static_cast<const float*>(dO), ws,
                                           static_cast<float*>(dq), static_cast<float*>(dk), static_cast<float*>(dv),
                                           g, Hq, Hkv, D, window, scale, st));
  }
  const int sms = sm_count();
  if (sms <= 0) return HD_ERR_CUDA;
  return cuda_status(
      launch_attn_bwd_tc(q, k, v, dO, ws, dq, dk, dv, g, Hq, Hkv, D, window, scale, dev_status, sms, st));
}

hd_status hd_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                      void* dq, void* dk, void* dv, int B, int L, int n, int Hq, int Hkv, int D, hd_mode mode,
                      int window, float scale, hd_dtype dt, void* workspace, size_t ws_bytes, int32_t* dev_status,
                      void* stream) {
  hd_status stt = check_attn_args(q, k, v, dq, nullptr, B, L, n, Hq, Hkv, D, mode, window, scale, dt, dt);
  if (stt != HD_OK || B == 0) return stt;
  return run_attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, regular_geom(B, L, n, mode), Hq, Hkv, D, window, scale, dt,
                      workspace, ws_bytes, dev_status, stream);
}

hd_status hd_attn_bwd_final_stream(const void* q_final, const void* k, const void* v, const void* o_final,
                                   const void* dO_final, const float* lse_final, void* dq_final, void* dk, void* dv,
                                   int B, int L, int n, int Hq, int Hkv, int D, hd_mode mode, int window, float scale,
                                   hd_dtype dt, void* workspace, size_t ws_bytes, int32_t* dev_status,
                                   void* stream) {
  hd_status stt = check_attn_args(q_final, k, v, dq_final, nullptr, B, L, n, Hq, Hkv, D, mode, window, scale, dt, dt);
  if (stt != HD_OK || B == 0) return stt;
  return run_attn_bwd(q_final, k, v, o_final, dO_final, lse_final, dq_final, dk, dv, final_stream_geom(B, L, n, mode),
                      Hq, Hkv, D, window, scale, dt, workspace, ws_bytes, dev_status, stream);
}

size_t hd_attn_decode_workspace(int B, int n, int Lmax, int Hq, int Hkv, int D, hd_mode mode) {
  if (B < 1 || n < 1 || Lmax < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || D != 128) return 0;
  if (mode != HD_INTRA && mode != HD_CROSS) return 0;
  const int sms = sm_count();
  if (sms <= 0) return 0;
  return decode_workspace_bytes(decode_plan(B, n, Lmax, Hq, Hkv, mode == HD_CROSS, sms));
}

// Argument checks shared by the decode entry points; nc = cache streams.
static hd_status check_decode_args(const void* q, const void* k_cache, const void* v_cache, const int32_t* ctx_len,
                                   void* o, float* lse, int B, int n, int nc, int Lmax, int Hq, int Hkv, int D,
                                   hd_mode mode, int window, float scale, hd_dtype in_dt, hd_dtype out_dt,
                                   void* workspace) {
  if (B < 0 || n < 1 || nc < 1 || Lmax < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || window < 0) return HD_ERR_INVALID_ARG;
  if (mode != HD_INTRA && mode != HD_CROSS) return HD_ERR_INVALID_ARG;
  if (!valid_dtype(in_dt) || !valid_dtype(out_dt) || !std::isfinite(scale) || !(scale > 0.f))
    return HD_ERR_INVALID_ARG;
  if (D != 128 || in_dt != HD_BF16) return HD_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(n) * Lmax > (1ll << 30)) return HD_ERR_INVALID_ARG;
  if (B == 0) return HD_OK;
  if (!q || !k_cache || !v_cache || !ctx_len || !o || !workspace) return HD_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) || (reinterpret_cast<uintptr_t>(ctx_len) & 3u))
    return HD_ERR_INVALID_ARG;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return HD_ERR_INVALID_ARG;
  return HD_OK;
}

hd_status hd_attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* ctx_len,
                         void* o, float* lse, int B, int n, int Lmax, int Hq, int Hkv, int D, hd_mode mode,
                         int window, float scale, hd_dtype in_dt, hd_dtype out_dt, void* workspace,
                         size_t ws_bytes, int32_t* dev_status, void* stream) {
  hd_status stt = check_decode_args(q, k_cache, v_cache, ctx_len, o, lse, B, n, n, Lmax, Hq, Hkv, D, mode, window,
                                    scale, in_dt, out_dt, workspace);
  if (stt != HD_OK || B == 0) return stt;
  const int sms = sm_count();
  if (sms <= 0) return HD_ERR_CUDA;
  const DecPlan pl = decode_plan(B, n, Lmax, Hq, Hkv, mode == HD_CROSS, sms);
  if (pl.units > 65535) return HD_ERR_UNSUPPORTED;
  if (ws_bytes < decode_workspace_bytes(pl)) return HD_ERR_INVALID_ARG;
  return cuda_status(launch_decode(q, k_cache, v_cache, ctx_len, o, lse, B, n, Lmax, Hq, Hkv, window, scale,
                                   mode == HD_CROSS, out_dt == HD_BF16, workspace, dev_status, sms,
                                   static_cast<cudaStream_t>(stream)));
}

// Geometry of rank r's queries in a stream-parallel cross-stream layer.
static AttnGeom shard_geom(int B, int L, int n, int R, int r) {
  const int nl = n / R;
  AttnGeom g;
  g.B = B;
  g.ns = nl;
  g.Lq = L;
  g.q_ns = nl;
  g.kv_ns = 1;
  g.Lk = n * L;
  g.kv_stream = 0;
  g.qstride = n;
  g.qoff = r;
  g.qsstride = R;
  g.o_rows = nl * L;
  g.o_ns = nl;
  return g;
}

static bool valid_shard(int n, int R, int r) { return R >= 1 && n >= 1 && n % R == 0 && r >= 0 && r < R; }

hd_status hd_attn_decode_shard(const void* q, const void* k_cache_loc, const void* v_cache_loc,
                               const int32_t* ctx_len, void* o, float* lse, int B, int n, int R, int r, int Lmax,
                               int Hq, int Hkv, int D, int window, float scale, hd_dtype in_dt, hd_dtype out_dt,
                               void* workspace, size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (!valid_shard(n, R, r)) return HD_ERR_INVALID_ARG;
  hd_status stt = check_decode_args(q, k_cache_loc, v_cache_loc, ctx_len, o, lse, B, n, n / R, Lmax, Hq, Hkv, D,
                                    HD_CROSS, window, scale, in_dt, out_dt, workspace);
  if (stt != HD_OK || B == 0) return stt;
  if (!lse) return HD_ERR_INVALID_ARG;  // the partial is useless without its lse
  const int sms = sm_count();
  if (sms <= 0) return HD_ERR_CUDA;
  const DecPlan pl = decode_plan(B, n, Lmax, Hq, Hkv, true, sms);
  if (pl.units > 65535) return HD_ERR_UNSUPPORTED;
  if (ws_bytes < decode_workspace_bytes(pl)) return HD_ERR_INVALID_ARG;
  return cuda_status(launch_decode(q, k_cache_loc, v_cache_loc, ctx_len, o, lse, B, n, Lmax, Hq, Hkv, window, scale,
                                   true, out_dt == HD_BF16, workspace, dev_status, sms,
                                   static_cast<cudaStream_t>(stream), n / R, r, R));
}

hd_status hd_attn_fwd_shard(const void* q_loc, const void* k, const void* v, void* o_loc, float* lse, int B, int L,
                            int n, int R, int r, int Hq, int Hkv, int D, int window, float scale, hd_dtype in_dt,
                            hd_dtype out_dt, int32_t* dev_status, void* stream) {
  if (!valid_shard(n, R, r)) return HD_ERR_INVALID_ARG;
  hd_status stt = check_attn_args(q_loc, k, v, o_loc, lse, B, L, n, Hq, Hkv, D, HD_CROSS, window, scale, in_dt, out_dt);
  if (stt != HD_OK || B == 0) return stt;
  return run_attn(q_loc, k, v, o_loc, lse, shard_geom(B, L, n, R, r), Hq, Hkv, D, window, scale, in_dt, out_dt,
                  dev_status, stream);
}

// Shared checks of the rank-shard calls; *pa gets the shard pointers.
static hd_status parts_args(const void* q_loc, const void* const* k_src, const void* const* v_src, void* o_loc,
                            float* lse, int B, int L, int n, int R, int r, int Hq, int Hkv, int D, int window,
                            float scale, hd_dtype in_dt, hd_dtype out_dt, PartsArgs* pa) {
  if (!valid_shard(n, R, r) || R > kPeerMaxRanks || 128 % n) return HD_ERR_INVALID_ARG;
  if (!k_src || !v_src) return HD_ERR_INVALID_ARG;
  // q_loc doubles as the k/v placeholder of the common checks; the shards are checked below.
  hd_status stt = check_attn_args(q_loc, q_loc, q_loc, o_loc, lse, B, L, n, Hq, Hkv, D, HD_CROSS, window, scale,
                                  in_dt, out_dt);
  if (stt != HD_OK) return stt;
  if (in_dt != HD_BF16) return HD_ERR_UNSUPPORTED;
  std::memset(pa, 0, sizeof(*pa));
  pa->R = R;
  pa->self = r;
  for (int rho = 0; rho < R; ++rho) {
    if (B > 0 && (!k_src[rho] || !v_src[rho] || !aligned16(k_src[rho]) || !aligned16(v_src[rho])))
      return HD_ERR_INVALID_ARG;
    pa->k_src[rho] = k_src[rho];
    pa->v_src[rho] = v_src[rho];
  }
  return HD_OK;
}

hd_status hd_attn_fwd_parts(const void* q_loc, const void* const* k_parts, const void* const* v_parts, void* o_loc,
                            float* lse, int B, int L, int n, int R, int r, int Hq, int Hkv, int D, int window,
                            float scale, hd_dtype in_dt, hd_dtype out_dt, int32_t* dev_status, void* stream) {
  PartsArgs pa;
  hd_status stt = parts_args(q_loc, k_parts, v_parts, o_loc, lse, B, L, n, R, r, Hq, Hkv, D, window, scale, in_dt,
                             out_dt, &pa);
  if (stt != HD_OK || B == 0) return stt;
  const int sms = sm_count();
  if (sms <= 0) return HD_ERR_CUDA;
  return cuda_status(launch_attn_tc_parts(q_loc, pa, o_loc, lse, shard_geom(B, L, n, R, r), n, Hq, Hkv, D, window,
                                          scale, out_dt == HD_BF16, dev_status, sms,
                                          static_cast<cudaStream_t>(stream)));
}

size_t hd_attn_peer_flags_bytes(int B, int L, int n) {
  if (B < 0 || L < 0 || n < 1) return 0;
  return static_cast<size_t>(parts_flag_count(B, n, L)) * sizeof(unsigned long long);
}

hd_status hd_attn_fwd_peer_gather(const void* q_loc, const void* const* k_src, const void* const* v_src,
                                  void* const* k_dst, void* const* v_dst, void* flags, size_t flags_bytes,
                                  void* o_loc, float* lse, int B, int L, int n, int R, int r, int Hq, int Hkv, int D,
                                  int window, float scale, hd_dtype in_dt, hd_dtype out_dt, int32_t* dev_status,
                                  void* stream) {
  PartsArgs pa;
  hd_status stt = parts_args(q_loc, k_src, v_src, o_loc, lse, B, L, n, R, r, Hq, Hkv, D, window, scale, in_dt,
                             out_dt, &pa);
  if (stt != HD_OK || B == 0) return stt;
  if (R > 1) {
    if (!k_dst || !v_dst || !flags || (reinterpret_cast<uintptr_t>(flags) & 7u) ||
        flags_bytes < hd_attn_peer_flags_bytes(B, L, n))
      return HD_ERR_INVALID_ARG;
    for (int rho = 0; rho < R; ++rho) {
      if (rho == r) {
        // Optional: given both, the own shard is copied there too.
        if (k_dst[rho] && v_dst[rho]) {
          if (!aligned16(k_dst[rho]) || !aligned16(v_dst[rho])) return HD_ERR_INVALID_ARG;
          pa.k_dst[rho] = k_dst[rho];
          pa.v_dst[rho] = v_dst[rho];
        }
        continue;
      }
      if (!k_dst[rho] || !v_dst[rho] || !aligned16(k_dst[rho]) || !aligned16(v_dst[rho])) return HD_ERR_INVALID_ARG;
      pa.k_dst[rho] = k_dst[rho];
      pa.v_dst[rho] = v_dst[rho];
    }
    pa.flags = static_cast<unsigned long long*>(flags);
  }
  const int sms = sm_count();
  if (sms <= 0) return HD_ERR_CUDA;
  return cuda_status(launch_attn_tc_parts(q_loc, pa, o_loc, lse, shard_geom(B, L, n, R, r), n, Hq, Hkv, D, window,
                                          scale, out_dt == HD_BF16, dev_status, sms,
                                          static_cast<cudaStream_t>(stream)));
}

hd_status hd_attn_combine_streams(const void* const* o_parts, const float* const* lse_parts, void* o_loc,
                                  float* lse_loc, int B, int n, int Hq, int D, int R, int r, hd_dtype in_dt,
                                  hd_dtype out_dt, void* stream) {
  if (B < 0 || Hq < 1 || D < 4 || D % 4 || !valid_shard(n, R, r) || R > kPeerMaxRanks || !valid_dtype(in_dt) ||
      !valid_dtype(out_dt))
    return HD_ERR_INVALID_ARG;
  if (B == 0) return HD_OK;
  if (!o_parts || !lse_parts || !o_loc || !aligned16(o_loc) || (lse_loc && (reinterpret_cast<uintptr_t>(lse_loc) & 3u)))
    return HD_ERR_INVALID_ARG;
  for (int rho = 0; rho < R; ++rho)
    if (!o_parts[rho] || !lse_parts[rho] || !aligned16(o_parts[rho]) ||
        (reinterpret_cast<uintptr_t>(lse_parts[rho]) & 3u))
      return HD_ERR_INVALID_ARG;
  return cuda_status(launch_attn_combine_streams(o_parts, lse_parts, o_loc, lse_loc, R, B, n, Hq, D, r,
                                                 in_dt == HD_BF16, out_dt == HD_BF16,
                                                 static_cast<cudaStream_t>(stream)));
}

static_assert(sizeof(cudaIpcMemHandle_t) == HD_IPC_HANDLE_BYTES, "IPC handle size");

hd_status hd_ipc_export(const void* ptr, void* handle, size_t* offset) {
  if (!ptr || !handle || !offset) return HD_ERR_INVALID_ARG;
  using RangeFn = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);
  static RangeFn range = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<RangeFn>(p);
    return static_cast<RangeFn>(nullptr);
  }();
  if (!range) return HD_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) return HD_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>(base)) != cudaSuccess) return HD_ERR_CUDA;
  std::memcpy(handle, &h, sizeof(h));
  *offset = static_cast<size_t>(reinterpret_cast<CUdeviceptr>(ptr) - base);
  return HD_OK;
}

hd_status hd_ipc_open(const void* handle, void** base) {
  if (!handle || !base) return HD_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  return cuda_status(cudaIpcOpenMemHandle(base, h, cudaIpcMemLazyEnablePeerAccess));
}

hd_status hd_ipc_close(void* base) {
  if (!base) return HD_ERR_INVALID_ARG;
  return cuda_status(cudaIpcCloseMemHandle(base));
}

hd_status hd_stream_interleave(const void* parts, void* out, int R, int B, int L, int n, int64_t row_elems,
                               hd_dtype dt, void* stream) {
  if (B < 0 || L < 0 || !valid_shard(n, R, 0) || row_elems < 1 || !valid_dtype(dt)) return HD_ERR_INVALID_ARG;
  const int64_t row_bytes = row_elems * esize(dt);
  if (row_bytes % 16 || row_bytes > (1 << 30)) return HD_ERR_INVALID_ARG;
  const int64_t rows = static_cast<int64_t>(B) * L * n;
  if (rows == 0) return HD_OK;
  if (!parts || !out || !aligned16(parts) || !aligned16(out)) return HD_ERR_INVALID_ARG;
  const int sms = sm_count();
  if (sms <= 0) return HD_ERR_CUDA;
  return cuda_status(launch_stream_interleave(parts, out, rows, n, R, static_cast<int>(row_bytes), sms,
                                              static_cast<cudaStream_t>(stream)));
}

hd_status hd_attn_combine(const void* o_parts, const float* lse_parts, void* o, float* lse, int R, int64_t rows,
                          int D, hd_dtype in_dt, hd_dtype out_dt, void* stream) {
  if (R < 1 || rows < 0 || D < 4 || D % 4 || !valid_dtype(in_dt) || !valid_dtype(out_dt)) return HD_ERR_INVALID_ARG;
  if (rows == 0) return HD_OK;
  if (!o_parts || !lse_parts || !o || (reinterpret_cast<uintptr_t>(o_parts) & 15u) ||
      (reinterpret_cast<uintptr_t>(o) & 15u) || (reinterpret_cast<uintptr_t>(lse_parts) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return HD_ERR_INVALID_ARG;
  return cuda_status(launch_attn_combine(o_parts, lse_parts, o, lse, R, rows, D, in_dt == HD_BF16,
                                         out_dt == HD_BF16, static_cast<cudaStream_t>(stream)));
}

hd_status hd_rope(void* q, void* k, const int32_t* pos0, int B, int P, int Hq, int Hkv, int D, int rot_dim,
                  double base, int64_t pos_base, int64_t pos_mult, hd_rope_layout layout, hd_dtype dt, void* stream) {
  if (B < 0 || P < 0 || Hq < 0 || Hkv < 0 || !valid_dtype(dt)) return HD_ERR_INVALID_ARG;
  if (layout != HD_ROPE_HALF && layout != HD_ROPE_INTERLEAVED) return HD_ERR_INVALID_ARG;
  if (D % 8 || D < 8 || D > 2 * kRopeMaxPairs || rot_dim % 8 || rot_dim < 8 || rot_dim > D)
    return HD_ERR_INVALID_ARG;
  if (!std::isfinite(base) || !(base > 0.0)) return HD_ERR_INVALID_ARG;
  const int heads = (q ? Hq : 0) + (k ? Hkv : 0);
  if (B == 0 || P == 0 || heads == 0) return HD_OK;
  if ((q && !aligned16(q)) || (k && !aligned16(k)) || (pos0 && (reinterpret_cast<uintptr_t>(pos0) & 3u)))
    return HD_ERR_INVALID_ARG;
  // Positions must stay within +-2^31: pos_base + pos_mult*pos0 + r for
  // pos0 in int32 range is checked against the host-known parts only.
  const int64_t lim = 1ll << 31;
  if (pos_base <= -lim || pos_base + P >= lim || pos_mult < -lim || pos_mult > lim) return HD_ERR_INVALID_ARG;
  RopeParams p;
  p.q = q;
  p.k = k;
  p.pos0 = pos0;
  p.B = B;
  p.P = P;
  p.Hq = q ? Hq : 0;
  p.Hkv = k ? Hkv : 0;
  p.D = D;
  p.rot = rot_dim;
  p.layout = layout;
  p.pos_base = pos_base;
  p.pos_mult = pos_mult;
  rope_fill_turns(p, rot_dim, base);
  return cuda_status(launch_rope(p, dt == HD_BF16, static_cast<cudaStream_t>(stream)));
}

const char* hd_status_string(hd_status st) {
  switch (st) {
    case HD_OK: return "HD_OK";
    case HD_ERR_INVALID_ARG: return "HD_ERR_INVALID_ARG";
    case HD_ERR_UNSUPPORTED: return "HD_ERR_UNSUPPORTED";
    case HD_ERR_CUDA: return "HD_ERR_CUDA";
    case HD_ERR_TIMEOUT: return "HD_ERR_TIMEOUT";
    case HD_ERR_BAD_TOKEN: return "HD_ERR_BAD_TOKEN";
  }
  return "HD_ERR_UNKNOWN";
}

int hd_version(void) { return 100; }

}  // extern "C"
