/*
 * hd.h — C ABI of the B200 (sm_100a) Hidden Decoding hot path.
 *
 * Method source: the WeLM blog page "Hidden Decoding at Scale" (sections
 * "Multi-Stream Expansion and Training Objective", "Stream-Factorized
 * Attention" with Figure 2, "Persistent KV and the KV-mirror Saving",
 * "Inference Throughput").
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Indexing is 0-based: token i in [0, L), stream s in [0, n), physical
 *    position p = i*n + s of the expanded sequence (the page's t = (i-1)n + k).
 *    The final stream is s = n-1.
 *  - All tensors are dense, row-major (last index fastest), on the current
 *    CUDA device, owned by the caller.  Base pointers must be 16-byte aligned
 *    (int32 token ids: 4-byte aligned).
 *  - The library allocates no device memory and never synchronises: every
 *    call is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and returns at once.  Scratch memory is passed in by the caller
 *    (the decode and backward workspaces), except for
 *    hd_attn_decode_noalloc, which uses a fixed scratch array that is part
 *    of the library's own device image (see that call).
 *  - Host-side argument errors return a status synchronously and launch
 *    nothing.  Problems found on the device (a token id out of range, a
 *    pipeline wait that ran out of time) are written to `*dev_status` (a
 *    device int32, nullable, first error wins, never reset by the library);
 *    no kernel traps.
 *  - Element types: HD_F32 = float32, HD_BF16 = bfloat16.
 */
#ifndef HD_H_
#define HD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HD_OK = 0,
  HD_ERR_INVALID_ARG = 1, /* null pointer, bad size, misalignment           */
  HD_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. head_dim 96)    */
  HD_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed            */
  HD_ERR_TIMEOUT = 4,     /* device: a bounded pipeline wait gave up         */
  HD_ERR_BAD_TOKEN = 5    /* device: token id outside [0, V)                 */
} hd_status;

typedef enum { HD_F32 = 0, HD_BF16 = 1 } hd_dtype;

typedef enum {
  HD_INTRA = 0, /* Figure 2(c): causal inside each stream                    */
  HD_CROSS = 1  /* Figure 2(a)/(b): causal over the interleaved nL order     */
} hd_mode;

/*
 * Multi-stream expansion ("Multi-Stream Expansion and Training Objective",
 * eq. S_t = E_k(x_i)):   out[b, i*n + s, :] = tables[s, ids[b, i], :]
 *
 *   tables  [n, V, d]   element type `dt`
 *   ids     [B, L]      int32, each in [0, V); 4-byte aligned
 *   out     [B, n*L, d] element type `dt`
 * d*sizeof(dt) must be a multiple of 16 bytes.  A row whose id is out of
 * range is written as zeros and HD_ERR_BAD_TOKEN is recorded in *dev_status.
 * The copy is bit-exact.
 */
hd_status hd_expand_embed(const void* tables, const int32_t* ids, void* out,
                          int B, int L, int n, int64_t V, int d, hd_dtype dt,
                          int32_t* dev_status, void* stream);

/*
 * Stream-Factorized Attention forward ("Stream-Factorized Attention",
 * Figure 2).  For every batch b, query head h and position p = i*n + s:
 *   O[b,p,h,:] = sum_{p' in vis(p)} softmax_{p'}(scale * <q[b,p,h], k[b,p',g]>) v[b,p',g]
 * with g = h / (Hq/Hkv) (GQA, consecutive grouping) and
 *   HD_INTRA: vis(p) = {(j, s) : j <= i, and i - j < window if window > 0}
 *   HD_CROSS: vis(p) = {p' : p' <= p,   and p - p' < window if window > 0}
 * (window counts tokens of the stream in intra mode, physical positions in
 * cross mode; 0 = no window).
 *
 *   q   [B, n*L, Hq,  D]  element type `in_dt`
 *   k,v [B, n*L, Hkv, D]  element type `in_dt`
 *   o   [B, n*L, Hq,  D]  element type `out_dt`
 *   lse [B, Hq, n*L]      float32 natural-log log-sum-exp, nullable
 * D must be 64 or 128; Hq % Hkv == 0; L >= 1; n >= 1; scale finite and > 0.
 * in_dt = HD_BF16 runs the tcgen05/TMEM tensor-core kernel (fp32 accumulate);
 * in_dt = HD_F32 runs the fp32 CUDA-core kernel.
 */
hd_status hd_attn_fwd(const void* q, const void* k, const void* v, void* o,
                      float* lse, int B, int L, int n, int Hq, int Hkv, int D,
                      hd_mode mode, int window, float scale, hd_dtype in_dt,
                      hd_dtype out_dt, int32_t* dev_status, void* stream);

/*
 * Final-stream queries only ("Persistent KV and the KV-mirror Saving": in the
 * mirrored layers only the final stream is run, against keys and values that
 * an earlier layer produced for every stream).  The rows of hd_attn_fwd at the
 * final-stream positions p = i*n + n-1, computed without the other queries:
 *   O[b,i,h,:] = sum_{p' in vis(i*n + n-1)} softmax(scale <qf[b,i,h], k[b,p',g]>) v[b,p',g]
 * with vis as in hd_attn_fwd (intra: keys (j, n-1), j <= i; cross: all
 * p' <= i*n + n-1; optional window in the same units).
 *
 *   q_final [B, L, Hq, D]     element type `in_dt` (the final-stream queries)
 *   k, v    [B, n*L, Hkv, D]  element type `in_dt` (all streams)
 *   o       [B, L, Hq, D]     element type `out_dt`
 *   lse     [B, Hq, L]        float32, nullable
 * Same argument rules and kernels as hd_attn_fwd.
 */
hd_status hd_attn_fwd_final_stream(const void* q_final, const void* k, const void* v,
                                   void* o, float* lse, int B, int L, int n, int Hq,
                                   int Hkv, int D, hd_mode mode, int window, float scale,
                                   hd_dtype in_dt, hd_dtype out_dt, int32_t* dev_status,
                                   void* stream);

/*
 * Backward of hd_attn_fwd ("Computational Cost", "Near-Linear Training Cost":
 * the layers are trained through; the pages print no backward, so this is
 * the gradient of the forward's definition).  Given the forward's inputs, its
 * output o and lse, and dO = dLoss/dO, per (b, query head h) with
 * P = softmax(scale q k^T) over vis(p) and delta_p = <dO[p], o[p]>:
 *   dv[p'] = sum_{h in group} sum_p P[p,p'] dO[p]
 *   dS[p,p'] = P[p,p'] (<dO[p], v[p']> - delta_p)
 *   dq[p]  = scale sum_{p'} dS[p,p'] k[p']
 *   dk[p'] = scale sum_{h in group} sum_p dS[p,p'] q[p]
 * (group = the Hq/Hkv query heads that read KV head p''s head).
 *
 *   q, o, dO [B, n*L, Hq,  D]  element type `dt`
 *   k, v     [B, n*L, Hkv, D]  element type `dt`
 *   lse      [B, Hq, n*L]      float32, as written by hd_attn_fwd (required)
 *   dq       [B, n*L, Hq,  D]  element type `dt`, overwritten
 *   dk, dv   [B, n*L, Hkv, D]  element type `dt`, overwritten
 *   workspace: device scratch of at least hd_attn_bwd_workspace(...) bytes,
 *              256-byte aligned, owned by the caller, no initialisation
 *              needed, dead after the call completes.
 * Same shape, mode, window and scale rules as hd_attn_fwd.  dt = HD_BF16
 * runs tcgen05/TMEM tensor-core kernels (fp32 accumulate, one bf16 rounding
 * of P and dS); dt = HD_F32 runs fp32 CUDA-core kernels.  Output buffers must
 * not overlap the inputs.
 */
hd_status hd_attn_bwd(const void* q, const void* k, const void* v, const void* o,
                      const void* dO, const float* lse, void* dq, void* dk, void* dv,
                      int B, int L, int n, int Hq, int Hkv, int D, hd_mode mode,
                      int window, float scale, hd_dtype dt, void* workspace,
                      size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * Backward of hd_attn_fwd_final_stream (the KV-mirror layers are trained
 * through too): the gradient of the final-stream queries' attention with
 * respect to q_final and to every stream's k and v.  Same definition as
 * hd_attn_bwd with the query rows at positions i*n + n-1.
 *
 *   q_final, o_final, dO_final, dq_final [B, L, Hq, D]  element type `dt`
 *   k, v, dk, dv                         [B, n*L, Hkv, D] element type `dt`
 *   lse_final [B, Hq, L] float32 from hd_attn_fwd_final_stream (required)
 *   workspace: >= hd_attn_bwd_workspace(B, L, 1, Hq, HD_INTRA) bytes (L query
 *              rows in one stream), 256-byte aligned.
 * Keys no final-stream query sees (intra mode: the streams 0 .. n-2) get
 * dk = dv = 0.  Same argument rules and kernels as hd_attn_bwd.
 */
hd_status hd_attn_bwd_final_stream(const void* q_final, const void* k, const void* v,
                                   const void* o_final, const void* dO_final,
                                   const float* lse_final, void* dq_final, void* dk,
                                   void* dv, int B, int L, int n, int Hq, int Hkv, int D,
                                   hd_mode mode, int window, float scale, hd_dtype dt,
                                   void* workspace, size_t ws_bytes, int32_t* dev_status,
                                   void* stream);

/* Workspace bytes hd_attn_bwd needs for these sizes (0 on invalid sizes).
 * It holds two floats per (b, query head, position), padded per stream to a
 * multiple of 128 tokens. */
size_t hd_attn_bwd_workspace(int B, int L, int n, int Hq, hd_mode mode);

/*
 * Decode against the per-stream KV cache ("Persistent KV and the KV-mirror
 * Saving": a separate cache per stream; "Inference Throughput": the n streams
 * of a token are processed together in one pass).  For every b, the new
 * token is T-1 with T = ctx_len[b] (tokens per stream, new token included;
 * its K/V are already in the cache).  The stream-s query of that token sees
 *   HD_INTRA: (j, s)  for j <= T-1            (and T-1-j < window)
 *   HD_CROSS: (j, s') for j <  T-1, any s',   and (T-1, s') for s' <= s
 *             (and p - p' < window, physical positions p = j*n + s)
 * which is exactly the prefill row of position (T-1)*n + s.
 *
 *   q        [B, n, Hq, D]            element type `in_dt` (HD_BF16 only)
 *   k_cache  [B, n, Lmax, Hkv, D]     stream-major, element type `in_dt`
 *   v_cache  [B, n, Lmax, Hkv, D]
 *   ctx_len  [B] int32 on the device, 1 <= T <= Lmax
 *   o        [B, n, Hq, D]            element type `out_dt`
 *   lse      [B, n, Hq] float32, nullable
 *   workspace: device scratch of at least hd_attn_decode_workspace(...) bytes,
 *              256-byte aligned, owned by the caller; its contents need no
 *              initialisation and are dead after the call completes.
 * Values of ctx_len outside [1, Lmax] record HD_ERR_INVALID_ARG in
 * *dev_status and leave the rows of that sequence as zeros.
 */
hd_status hd_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                         const int32_t* ctx_len, void* o, float* lse, int B,
                         int n, int Lmax, int Hq, int Hkv, int D, hd_mode mode,
                         int window, float scale, hd_dtype in_dt, hd_dtype out_dt,
                         void* workspace, size_t ws_bytes, int32_t* dev_status,
                         void* stream);

/* Workspace bytes hd_attn_decode needs for these sizes on the current device
 * (0 on invalid sizes). */
size_t hd_attn_decode_workspace(int B, int n, int Lmax, int Hq, int Hkv, int D,
                                hd_mode mode);

/* Size of the fixed device scratch used by hd_attn_decode_noalloc (64 MiB). */
#define HD_DECODE_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * hd_attn_decode without a workspace argument: the same computation, inputs,
 * outputs and argument rules as hd_attn_decode, for callers that cannot
 * allocate device memory or hand it to the library (an allocator-free
 * serving loop, a host that owns no CUDA allocator, code running where a
 * cudaMalloc is not permitted).  The pages have no counterpart of this call;
 * it exists only for such callers.
 *
 * The split-KV partial results go to a fixed HD_DECODE_NOALLOC_SCRATCH_BYTES
 * array in the library's own device memory (present on every GPU that loads
 * the library, until the process exits).  Nothing is allocated: no cudaMalloc,
 * cudaFree or allocating library routine is called.
 *  - Sizes whose scratch need (hd_attn_decode_workspace for the same sizes)
 *    exceeds HD_DECODE_NOALLOC_SCRATCH_BYTES return HD_ERR_UNSUPPORTED and
 *    launch nothing; use hd_attn_decode with a workspace for those.
 *  - The first call on a device looks up the scratch's device address for
 *    that device; make that first call before any stream capture.  The
 *    address is kept for the life of the process: the call assumes each
 *    device keeps one primary context throughout (no cudaDeviceReset
 *    between calls, which would leave the kept address stale).
 *  - All calls share the one scratch array.  Calls whose kernels can overlap
 *    on the GPU (different streams with no ordering between them) race on it
 *    and give wrong results; order them on one stream or with events.
 *  - The scratch needs no clearing: every call writes each partial it reads.
 */
hd_status hd_attn_decode_noalloc(const void* q, const void* k_cache,
                                 const void* v_cache, const int32_t* ctx_len,
                                 void* o, float* lse, int B, int n, int Lmax,
                                 int Hq, int Hkv, int D, hd_mode mode, int window,
                                 float scale, hd_dtype in_dt, hd_dtype out_dt,
                                 int32_t* dev_status, void* stream);

/*
 * Stream parallelism ("Persistent KV and the KV-mirror Saving": the
 * intra-stream KV is sharded across ranks by stream).  With R ranks (R
 * divides n), rank r holds the streams s = r + R*l, l < n/R, stored in the
 * expanded order of its own streams: local row i*(n/R) + l is token i of
 * global stream r + R*l.  Intra-stream layers need nothing new (call
 * hd_attn_fwd / hd_attn_decode on the local tensors with n/R streams).  A
 * cross-stream prefill layer either gathers every rank's K/V shard (a
 * collective the caller runs, e.g. an NCCL all-gather into [R, ...]) and runs
 * hd_attn_fwd_parts on the gathered shards as they lie (or, for shapes that
 * call does not take, hd_stream_interleave + hd_attn_fwd_shard), or runs
 * hd_attn_fwd_peer_gather, whose kernel pulls the peers' shards itself while
 * it computes.  Cross-stream decode runs hd_attn_decode_shard on every rank
 * for all n stream queries against the local cache streams, then either
 * gathers the partials and merges them with hd_attn_combine, or merges its own
 * stream rows straight from the ranks' partials with hd_attn_combine_streams.
 */

/*
 *   out[b, i*n + r + R*l, :] = parts[r, b, i*(n/R) + l, :]
 *   parts [R, B, (n/R)*L, row_elems], out [B, n*L, row_elems], type `dt`.
 * row_elems*sizeof(dt) must be a multiple of 16 bytes.  Bit-exact copy.
 */
hd_status hd_stream_interleave(const void* parts, void* out, int R, int B, int L,
                               int n, int64_t row_elems, hd_dtype dt, void* stream);

/*
 * Merge R partial attention results over disjoint key sets:
 *   O[row] = sum_r w_r o_parts[r, row] / sum_r w_r,  w_r = exp(lse_parts[r, row] - M),
 *   lse[row] = M + log sum_r w_r,  M = max_r lse_parts[r, row];
 * a part with lse = -inf (no visible key) has weight 0; a row whose parts
 * are all empty gets O = 0 and lse = -inf.
 *   o_parts [R, rows, D] type `in_dt`;  lse_parts [R, rows] float32 (natural log);
 *   o [rows, D] type `out_dt`;  lse [rows] float32 (nullable).  D % 4 == 0.
 */
hd_status hd_attn_combine(const void* o_parts, const float* lse_parts, void* o,
                          float* lse, int R, int64_t rows, int D, hd_dtype in_dt,
                          hd_dtype out_dt, void* stream);

/*
 * Cross-stream prefill attention of rank r's queries against every stream's
 * keys: for local row i*(n/R) + l (global position p = i*n + r + R*l)
 *   O = sum_{p' in vis(p)} softmax(scale <q, k[p']>) v[p']   (HD_CROSS rules)
 *
 *   q_loc [B, (n/R)*L, Hq, D]  element type `in_dt`
 *   k, v  [B, n*L, Hkv, D]     all streams, expanded order (hd_stream_interleave)
 *   o_loc [B, (n/R)*L, Hq, D]  element type `out_dt`
 *   lse   [B, Hq, (n/R)*L]     float32, nullable
 * Same kernels and argument rules as hd_attn_fwd (cross mode).
 */
hd_status hd_attn_fwd_shard(const void* q_loc, const void* k, const void* v, void* o_loc,
                            float* lse, int B, int L, int n, int R, int r, int Hq,
                            int Hkv, int D, int window, float scale, hd_dtype in_dt,
                            hd_dtype out_dt, int32_t* dev_status, void* stream);

/*
 * Cross-stream decode restricted to rank r's cache streams: for every
 * stream query s of the new token, the softmax over the visible keys (the
 * HD_CROSS rules of hd_attn_decode) that lie in streams r + R*l only.
 *
 *   q            [B, n, Hq, D]           all n stream queries, `in_dt` (HD_BF16)
 *   k/v_cache_loc [B, n/R, Lmax, Hkv, D] the local streams, `in_dt`
 *   ctx_len      [B] int32 on the device
 *   o            [B, n, Hq, D]           `out_dt`: the partial O (normalised over
 *                                        this rank's keys; 0 where it has none)
 *   lse          [B, n, Hq] float32 (required): log-sum-exp over this rank's
 *                keys, -inf where it has none
 *   workspace    >= hd_attn_decode_workspace(B, n, Lmax, Hq, Hkv, D, HD_CROSS)
 * Merge the R ranks' (o, lse) with hd_attn_combine.
 */
hd_status hd_attn_decode_shard(const void* q, const void* k_cache_loc,
                               const void* v_cache_loc, const int32_t* ctx_len, void* o,
                               float* lse, int B, int n, int R, int r, int Lmax, int Hq,
                               int Hkv, int D, int window, float scale, hd_dtype in_dt,
                               hd_dtype out_dt, void* workspace, size_t ws_bytes,
                               int32_t* dev_status, void* stream);

/*
 * The merge of hd_attn_combine for rank r's own stream queries, with the
 * exchange fused in: each rank's partial is read where it lies (another
 * GPU's memory through hd_ipc_open, or local), and only rank r's rows:
 *   o_loc[b, l, h] = merge over rho of (o_parts[rho], lse_parts[rho]) at row
 *                    (b, r + R*l, h)     (the hd_attn_combine formula)
 *   o_parts[rho]   [B, n, Hq, D] `in_dt`: rank rho's hd_attn_decode_shard o
 *   lse_parts[rho] [B, n, Hq] float32: its lse
 *   o_loc          [B, n/R, Hq, D] `out_dt`;  lse_loc [B, n/R, Hq] float32, nullable
 * (host arrays of R device pointers).  1 <= R <= HD_MAX_RANKS, R divides n,
 * D % 4 == 0.  The caller orders the peers' writes of their partials before
 * the call (e.g. a barrier collective on `stream`).
 */
hd_status hd_attn_combine_streams(const void* const* o_parts, const float* const* lse_parts,
                                  void* o_loc, float* lse_loc, int B, int n, int Hq, int D,
                                  int R, int r, hd_dtype in_dt, hd_dtype out_dt, void* stream);

/*
 * Cross-stream prefill without the re-interleaved copy.  The operation is
 * that of hd_attn_fwd_shard (rank r's queries, HD_CROSS rules over all n*L
 * keys), with the keys and values given as the R ranks' shards:
 *
 *   k_parts[rho], v_parts[rho]  host arrays of R device pointers; rank rho's
 *       shard [B, (n/R)*L, Hkv, D], whose row i*(n/R) + l holds token i of
 *       global stream rho + R*l (e.g. the R slots of an all-gather).
 *
 * A 128-key tile of the expanded order is 128/R consecutive rows of every
 * shard, so the kernel reads the shards where they lie (fastest when they
 * lie at one stride, e.g. one [R, ...] tensor: then a key tile is one TMA box
 * per 64 features instead of one per rank).  bf16 input only;
 * 1 <= R <= HD_MAX_RANKS, R divides n, n divides 128.  Other arguments and
 * errors as hd_attn_fwd_shard.  The shards are read many times: they belong
 * in this GPU's memory (for peers' memory use hd_attn_fwd_peer_gather).
 */
#define HD_MAX_RANKS 8
hd_status hd_attn_fwd_parts(const void* q_loc, const void* const* k_parts,
                            const void* const* v_parts, void* o_loc, float* lse, int B,
                            int L, int n, int R, int r, int Hq, int Hkv, int D, int window,
                            float scale, hd_dtype in_dt, hd_dtype out_dt,
                            int32_t* dev_status, void* stream);

/*
 * hd_attn_fwd_parts with the exchange fused in.  k_src[rho], v_src[rho]
 * (rho != r) are the other ranks' shards, normally peer memory (hd_ipc_open):
 * a warp in every CTA copies each of them once into k_dst[rho], v_dst[rho]
 * (this GPU, same shape), in key-tile order, while the attention runs; each
 * key tile is read only after its own pieces have landed.  k_src[r],
 * v_src[r] are this rank's shard: read in place when k_dst[r] or v_dst[r]
 * is NULL, else copied there as well.  When the R slots the attention reads
 * lie at one stride in memory (e.g. k_dst/v_dst are the R slots of one
 * [R, B, (n/R)*L, Hkv, D] tensor, own slot included), each key tile is one
 * TMA box per 64 features instead of one per rank.
 *   flags  device workspace of hd_attn_peer_flags_bytes(B, L, n) bytes,
 *          zeroed by the call on `stream`; calls that may run at the same
 *          time need separate flags (and separate k_dst/v_dst).
 * The launch is cooperative (all CTAs resident at once); where the GPU cannot
 * host them together (e.g. shared with other work) the call returns
 * HD_ERR_CUDA without running the attention (only the flags were zeroed).
 * Ordering across
 * ranks is the caller's: every shard must be complete before the call runs,
 * and no rank may overwrite its shard before the other ranks' calls that
 * read it have finished (e.g. one barrier collective per layer on `stream`
 * with two shard buffers used in turn).  Results equal hd_attn_fwd_parts;
 * k_dst/v_dst end up bit-identical to k_src/v_src.  A piece that never
 * lands ends the waits after about one second with HD_ERR_TIMEOUT in
 * *dev_status.
 */
size_t hd_attn_peer_flags_bytes(int B, int L, int n);
hd_status hd_attn_fwd_peer_gather(const void* q_loc, const void* const* k_src,
                                  const void* const* v_src, void* const* k_dst,
                                  void* const* v_dst, void* flags, size_t flags_bytes,
                                  void* o_loc, float* lse, int B, int L, int n, int R, int r,
                                  int Hq, int Hkv, int D, int window, float scale,
                                  hd_dtype in_dt, hd_dtype out_dt, int32_t* dev_status,
                                  void* stream);

/*
 * CUDA IPC for the shards of hd_attn_fwd_peer_gather.
 * hd_ipc_export: handle (HD_IPC_HANDLE_BYTES bytes, host) of the device
 *   allocation that contains `ptr`, and ptr's byte offset in it.  Fails
 *   (HD_ERR_CUDA) for memory that CUDA IPC cannot share.
 * hd_ipc_open: in another process, map that allocation; *base is its start
 *   (add the offset); peer access is enabled as needed.
 * hd_ipc_close: unmap a base returned by hd_ipc_open.
 */
#define HD_IPC_HANDLE_BYTES 64
hd_status hd_ipc_export(const void* ptr, void* handle, size_t* offset);
hd_status hd_ipc_open(const void* handle, void** base);
hd_status hd_ipc_close(void* base);

typedef enum {
  HD_ROPE_HALF = 0,      /* pairs (j, j + rot_dim/2): the rotate-half form   */
  HD_ROPE_INTERLEAVED = 1 /* pairs (2j, 2j + 1): the RoFormer paper's form    */
} hd_rope_layout;

/*
 * Rotary position embedding over the expanded sequence ("Multi-Stream
 * Expansion and Training Objective": the expanded sequence runs with
 * contiguous RoPE positions), applied in place to q and k in one launch.
 * The pages fix only the positions; the rotation is the standard rotary
 * embedding.  Row r of sequence b sits at position
 *   pos(b, r) = pos_base + pos_mult * pos0[b] + r      (pos0 NULL: 0)
 * so a prefill of the expanded sequence (P = n*L, pos_base = 0) gives
 * pos = i*n + s, and the decode rows of the new token ([B, n, H, D] with
 * pos0 = ctx_len, pos_mult = n, pos_base = -n) give pos = (T-1)*n + s.
 * The first rot_dim features rotate pairwise by pos * theta_j,
 * theta_j = base^(-2j/rot_dim), j < rot_dim/2:
 *   (x_a, x_b) -> (x_a cos - x_b sin, x_a sin + x_b cos);
 * features past rot_dim are unchanged.
 *
 *   q    [B, P, Hq,  D]  element type `dt`, rotated in place (nullable)
 *   k    [B, P, Hkv, D]  element type `dt`, rotated in place (nullable)
 *   pos0 [B] int32 on the device (nullable)
 * rot_dim % 8 == 0, 8 <= rot_dim <= D <= 256, D % 8 == 0, base finite and
 * > 0, |pos| < 2^31 for every row.  The angle is reduced exactly (64-bit
 * fixed-point turns), cos/sin and the rotation run in float32 (angle error
 * < 2e-7 rad), and the result rounds once to `dt`.
 */
hd_status hd_rope(void* q, void* k, const int32_t* pos0, int B, int P, int Hq,
                  int Hkv, int D, int rot_dim, double base, int64_t pos_base,
                  int64_t pos_mult, hd_rope_layout layout, hd_dtype dt,
                  void* stream);

/*
 * hd_attn_fwd with the rotary embedding of hd_rope fused in ("Multi-Stream
 * Expansion and Training Objective": the expanded sequence runs with
 * contiguous RoPE positions; "Stream-Factorized Attention", Figure 2):
 *   O = hd_attn_fwd(rope(q), rope(k), v)
 * with rope as hd_rope at the contiguous positions of the expanded sequence
 * (row p of a sequence at position p = i*n + s; pos_base = 0, pos_mult = 0).
 *   q     [B, n*L, Hq, D]  bf16, read only: its rows are rotated inside the
 *                          attention kernel, in the tile, and never written
 *                          back
 *   k     [B, n*L, Hkv, D] bf16, rotated IN PLACE (on return k holds rope(k),
 *                          the keys a cache of this layer keeps)
 *   v, o, lse, mode, window, scale: as hd_attn_fwd (out_dt bf16 or f32)
 *   rot_dim, base, layout: as hd_rope; rot_dim <= D, and a multiple of 16
 *                          (HD_ROPE_HALF) or of 8 (HD_ROPE_INTERLEAVED)
 * in_dt must be HD_BF16 (HD_ERR_UNSUPPORTED otherwise).  Two launches on
 * `stream`: the rotation of k, then the attention.  The angles are reduced
 * exactly as in hd_rope (position times the 64-bit fixed-point fraction of a
 * turn, mod one turn); for the query rows the top 23 bits of that fraction
 * give the angle in float32, whose cos/sin come from the special-function
 * unit (absolute error about 1e-6), so q's rotation can differ from
 * hd_rope's in the last bit of a bf16 value.  Measured at parity with
 * hd_rope + hd_attn_fwd on the same inputs (the rotation of q costs the
 * attention kernel about what hd_rope's pass over q costs).
 */
hd_status hd_attn_fwd_rope(const void* q, void* k, const void* v, void* o,
                           float* lse, int B, int L, int n, int Hq, int Hkv, int D,
                           hd_mode mode, int window, float scale, int rot_dim,
                           double base, hd_rope_layout layout, hd_dtype in_dt,
                           hd_dtype out_dt, int32_t* dev_status, void* stream);

/*
 * Final-stream gather ("Multi-Stream Expansion and Training Objective": only
 * the final stream E_n of each token feeds the shared LM head; Figure 1):
 *   out[b, i, :] = h[b, i*n + n-1, :]
 *   h   [B, n*L, d] element type `dt`;  out [B, L, d].
 * d*sizeof(dt) must be a multiple of 16 bytes.  Bit-exact copy.
 */
hd_status hd_final_stream_gather(const void* h, void* out, int B, int L, int n,
                                 int d, hd_dtype dt, void* stream);

/* Human-readable name of a status code (static storage). */
const char* hd_status_string(hd_status st);

/* Library version, major*10000 + minor*100 + patch. */
int hd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HD_H_ */
