/*
 * dz.h -- C ABI of libdz: chunk-causal multi-head attention with 3D (t,h,w)
 * rotary position embedding and a KV cache of clean chunks, for the Causal WAN
 * DiT of DreamZero, on NVIDIA B200 (sm_100a).
 *
 * The operation (sources are the pages' titles and sections):
 *   - 40 heads of head_dim 128 over a hidden size of 5120; causal
 *     self-attention inside every DiT block, followed by cross-attention to
 *     the visual + language conditioning ("DreamZero (WAM) 模型架构", §2.3
 *     block diagram, §5 hyper-parameter table).
 *   - RoPE on the video latent sequence (same page, §2.3 input construction).
 *   - The model runs autoregressively over chunks of a fixed number of latent
 *     frames; the current noisy chunk attends to the clean context of earlier
 *     chunks and never to future tokens; in training this is teacher forcing
 *     ("World Action Models are Zero-shot Policies", hyper.ai summary, section
 *     "方法", paragraph 3; paper walkthrough, training objective, Fig. 14).
 *   - A KV cache of clean chunks is kept between requests; after a chunk's
 *     actions execute, its predicted frames in the cache are replaced by the
 *     real observation (hyper.ai summary, "方法" paragraph 4; "DreamZero
 *     单卡推理", "架构" and "连续请求").
 *
 * Conventions for every call:
 *   - Tensors q, k, v, out and the cache are bfloat16 in BSHD order: element
 *     (b, s, h, d) at ((b*S + s)*H + h)*D + d, i.e. the [B, S, 5120] hidden
 *     state viewed per head.  D (head_dim) is 128.
 *   - All pointers to tensors are DEVICE pointers, 16-byte aligned, owned by
 *     the caller; the library never frees them.  The library owns only the
 *     handle and what dz_attn_create allocates for it (rotary tables, the
 *     split-KV workspace and a device status word).
 *   - Calls are stream-ordered and asynchronous: they enqueue work on
 *     `stream` (a cudaStream_t, may be 0) and return without synchronising.
 *     A call on one handle must not overlap another call on the same handle
 *     on a different stream (they share the workspace).
 *   - Errors are returned as dz_status; nothing is enqueued when a call
 *     returns an error.  Argument checks happen on the host before launch.
 *     Device-side failures (a bounded wait that ran out) are recorded in the
 *     handle's status word and read back by dz_attn_sync_status.
 */
#ifndef DZ_H_
#define DZ_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DZ_OK = 0,
  DZ_ERR_INVALID_ARG = 1, /* null pointer, bad enum, negative or zero size     */
  DZ_ERR_ALIGNMENT = 2,   /* a tensor pointer is not 16-byte aligned           */
  DZ_ERR_SHAPE = 3,       /* unsupported shape: head_dim, heads, positions ... */
  DZ_ERR_CAPACITY = 4,    /* cache or handle capacity would be exceeded        */
  DZ_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed                 */
  DZ_ERR_UNSUPPORTED = 6, /* valid request this build does not implement       */
  DZ_ERR_TIMEOUT = 7,     /* a device-side bounded wait ran out                */
  DZ_ERR_BOUNDS = 8       /* a device index check failed (bounds-checked build) */
} dz_status;

typedef struct dz_attn* dz_attn_t; /* opaque handle */

/* Handle parameters (dz_attn_create).
 *   num_heads          H, 1..256 (the model uses 40).
 *   head_dim           must be 128.
 *   rope_base          frequency base of the rotary ladder (10000).
 *   rope_pairs_t/h/w   rotary pairs per axis; must sum to head_dim/2 (22/21/21).
 *                      Pair j of axis a turns by pos_a * rope_base^(-2j/(2*pairs_a)).
 *   max_batch          largest batch of any call on this handle.
 *   max_q_tokens       largest number of query tokens per batch item (sizes the
 *                      split-KV counters).
 *   max_pos_t/h/w      exclusive bounds of the (t, h, w) token positions the
 *                      rotary tables cover; a call whose tokens reach beyond
 *                      them returns DZ_ERR_SHAPE.
 *   prerotate_tokens   0, or the largest query length (per batch item) of
 *                      DECODE / TEACHER_FORCING / PREFILL calls for which q and
 *                      the call's own k are rotated once per call into a
 *                      handle-owned workspace (2 * max_batch * prerotate_tokens
 *                      * H * 256 bytes, allocated by dz_attn_create) before the
 *                      attention kernel runs; a key tile is read by many query
 *                      groups, so rotating it once is cheaper than rotating it
 *                      on each load.  With 0 (or longer calls) the attention
 *                      kernel rotates the tiles as it loads them.
 */
typedef struct {
  int32_t num_heads;
  int32_t head_dim;
  double rope_base;
  int32_t rope_pairs_t, rope_pairs_h, rope_pairs_w;
  int32_t max_batch;
  int32_t max_q_tokens;
  int32_t max_pos_t, max_pos_h, max_pos_w;
  int32_t prerotate_tokens;
} dz_attn_desc;

typedef enum {
  /* Current noisy chunk (q, k, v hold L tokens) over cache[0:len] and itself.
   * Every key is visible.  q and the chunk's own k are rotated in-kernel at
   * the positions of chunk `num_chunks`; cache keys are used as stored (the
   * cache holds keys that were rotated before they were appended). */
  DZ_MODE_DECODE = 0,
  /* q, k, v hold 2N chunks: clean chunks 0..N-1 then noisy chunks 0..N-1
   * (N = num_chunks).  Clean i sees clean <= i; noisy i sees clean < i and
   * noisy i.  Noisy chunk i is rotated at the positions of clean chunk i. */
  DZ_MODE_TEACHER_FORCING = 1,
  /* q, k, v hold N clean chunks; chunk c sees chunks <= c (block causal). */
  DZ_MODE_PREFILL = 2,
  /* Cross-attention: q holds N chunks, k and v hold kv_len condition tokens
   * (text then image); every key visible; no rotary. */
  DZ_MODE_CROSS = 3
} dz_mode;

/* Flag OR-ed into dz_chunk_layout.mode: q and the call's own k are already
 * rotated (for example by dz_qkv_rope), so the call does not rotate them.
 * Cache keys are always used as stored.  An interface choice of this library;
 * the pages have no counterpart. */
#define DZ_MODE_ROTATED 0x100

/* Token layout of one call.  A chunk is frames_per_chunk latent frames of
 * grid_h x grid_w tokens, frame-major then row then column, followed by
 * n_action action tokens: chunk_len L = F*grid_h*grid_w + n_action.
 * Token positions: video token (frame f, row r, column c) of chunk n sits at
 * (t_offset + n*F + f, r, c); an action token of chunk n at (t_offset + n*F, 0, 0).
 *   mode        dz_mode.
 *   batch       B (1..max_batch).
 *   num_chunks  DECODE: index of the current chunk (its rotary position);
 *               TEACHER_FORCING: clean chunks N; PREFILL / CROSS: chunks in q.
 *   t_offset    absolute latent-frame index of chunk 0 (0 after a reset).
 *   kv_len      CROSS: condition tokens per batch item; ignored otherwise.
 */
typedef struct {
  int32_t mode;
  int32_t batch;
  int32_t frames_per_chunk;
  int32_t grid_h, grid_w;
  int32_t n_action;
  int32_t num_chunks;
  int32_t t_offset;
  int32_t kv_len;
} dz_chunk_layout;

/* Caller-held KV-cache descriptor.  k and v are DEVICE buffers of bfloat16
 * [batch][capacity_tokens][H][128] (BSHD).  len_tokens is host-side state:
 * dz_kvcache_append advances it; a reset is `len_tokens = 0`.  chunk_len is
 * the token count of one chunk (L), used by dz_kvcache_replace. */
typedef struct {
  void* k;
  void* v;
  int32_t batch;
  int32_t capacity_tokens;
  int32_t len_tokens;
  int32_t chunk_len;
} dz_kvcache;

/* Create a handle for the current CUDA device.  Allocates the rotary tables,
 * the split-KV workspace and the status word (cudaMalloc; synchronous).
 * Errors: DZ_ERR_INVALID_ARG (null), DZ_ERR_SHAPE (head_dim != 128, pairs do
 * not sum to 64, non-positive sizes), DZ_ERR_CUDA. */
dz_status dz_attn_create(dz_attn_t* out, const dz_attn_desc* desc);

/* Release the handle and its device memory (synchronises the device first). */
dz_status dz_attn_destroy(dz_attn_t handle);

/* 3D rotary embedding ("DreamZero (WAM) 模型架构", §2.3, RoPE on the latent
 * sequence): y[b, s, h, :] = R(pos(s)) x[b, s, h, :] for x, y bf16 [B][S][H][128].
 * Token s is token s % L of chunk first_chunk + s / L of `layout` (mode,
 * batch, num_chunks and kv_len are ignored).  Pairs (x[2j], x[2j+1]) turn by
 * the angle p*omega_j: x' = x0 cos - x1 sin, y' = x0 sin + x1 cos, computed in
 * fp32 from fp64-built tables and rounded to bf16 (nearest even).  y may equal
 * x (in place); other overlap is not allowed.
 * Errors: DZ_ERR_INVALID_ARG, DZ_ERR_ALIGNMENT, DZ_ERR_SHAPE (positions
 * beyond the handle's tables), DZ_ERR_CUDA. */
dz_status dz_rope3d(dz_attn_t handle, const void* x, void* y, int32_t B, int32_t S,
                    const dz_chunk_layout* layout, int32_t first_chunk, void* stream);

/* Chunk-causal attention: out = softmax(R q (R k)^T / sqrt(128), chunk mask) v
 * per batch item and head, for the mode in `layout` (see dz_mode; with
 * DZ_MODE_ROTATED or-ed in, q and k are taken as already rotated).
 *   q    bf16 [B][Sq][H][128]; Sq = L (DECODE), 2*N*L (TEACHER_FORCING),
 *        N*L (PREFILL, CROSS).
 *   k, v bf16 [B][Sk][H][128]; Sk = Sq, or kv_len for CROSS.
 *   cache  DECODE only (may be NULL: no cached keys); its batch must equal
 *        layout->batch; keys cache[0:len_tokens] come first.  NULL otherwise.
 *   out  bf16 [B][Sq][H][128]; must not alias q, k, v or the cache.
 * Scores are accumulated in fp32 from bf16 operands (rotated q/k rounded to
 * bf16), softmax in fp32, probabilities rounded to bf16 for the PV product,
 * fp32 accumulation, output rounded to bf16.
 * Errors: DZ_ERR_INVALID_ARG, DZ_ERR_ALIGNMENT, DZ_ERR_SHAPE,
 * DZ_ERR_CAPACITY (batch or tokens beyond the handle), DZ_ERR_UNSUPPORTED
 * (more than 2^31 / (SM count + 1) key tiles of 128 keys in one call),
 * DZ_ERR_CUDA. */
dz_status dz_chunk_attn_forward(dz_attn_t handle, const void* q, const void* k, const void* v,
                                const dz_kvcache* cache, const dz_chunk_layout* layout,
                                void* out, void* stream);

/* FP8 variant of dz_chunk_attn_forward (the walkthrough of "World Action Models
 * are Zero-shot Policies", system optimisations: on Blackwell the DiT runs in
 * FP8 / NVFP4 with the rotary embedding kept in higher precision).  q8, k8 and,
 * in DECODE, cache->k hold ROTATED q and k as E4M3 codes (one byte per element,
 * same [B][S][H][128] layout; code = E4M3(x * multiplier), see dz_quantize_e4m3)
 * with multipliers q_scale and k_scale; v, cache->v and out are bf16 as in
 * dz_chunk_attn_forward.  Scores = (q8 . k8) / (q_scale * k_scale) / sqrt(128):
 * QK^T runs on E4M3 operands with fp32 accumulation; softmax, P (bf16), PV and
 * the output are as in the bf16 path.  No rotation is applied (DZ_MODE_ROTATED
 * is implied); modes as in dz_chunk_attn_forward.
 * Errors: as dz_chunk_attn_forward, and DZ_ERR_INVALID_ARG for a multiplier that
 * is not finite and positive. */
dz_status dz_chunk_attn_forward_e4m3(dz_attn_t handle, const void* q8, const void* k8,
                                     const void* v, const dz_kvcache* cache,
                                     const dz_chunk_layout* layout, float q_scale, float k_scale,
                                     void* out, void* stream);

/* dz_rope3d followed by dz_quantize_e4m3 in one pass: y8 receives the E4M3 codes of
 * the rotated bf16 values times `scale`, the same bytes the two calls give.  x bf16
 * [B][S][H][128], y8 uint8 [B][S][H][128], both 16-byte aligned, no overlap.
 * Errors: as dz_rope3d, and DZ_ERR_INVALID_ARG for a scale that is not finite and
 * positive or y8 == x. */
dz_status dz_rope3d_e4m3(dz_attn_t handle, const void* x, void* y8, int32_t B, int32_t S,
                         const dz_chunk_layout* layout, int32_t first_chunk, float scale,
                         void* stream);

/* E4M3 quantisation of n bf16 values: y[i] = E4M3(float(x[i]) * scale), the
 * product formed in fp32 and rounded to the nearest E4M3 value (ties to even),
 * magnitudes past 448 saturating to 448, sign kept (-0 for negatives that round
 * to zero), NaN to a NaN code.  x bf16 [n], y uint8 [n], both 16-byte aligned.
 * Errors: DZ_ERR_INVALID_ARG (n < 0, scale not finite and positive),
 * DZ_ERR_ALIGNMENT, DZ_ERR_CUDA. */
dz_status dz_quantize_e4m3(dz_attn_t handle, const void* x, void* y, int64_t n, float scale,
                           void* stream);

/* Append one chunk (KV cache of clean chunks: "DreamZero 单卡推理", "架构"
 * table -- the DiT runner keeps the attention KV; "连续请求" -- KV carried
 * across requests).  Copies k, v bf16 [cache->batch][L][H][128]
 * (L = cache->chunk_len) into cache rows [len_tokens, len_tokens + L) of every
 * batch item and advances cache->len_tokens by L on success.  k must already
 * be rotated (dz_rope3d at the chunk's positions).  Bit-exact copy.
 * Errors: DZ_ERR_CAPACITY (would exceed capacity_tokens; nothing written),
 * DZ_ERR_INVALID_ARG, DZ_ERR_ALIGNMENT, DZ_ERR_CUDA. */
dz_status dz_kvcache_append(dz_attn_t handle, dz_kvcache* cache, const void* k, const void* v,
                            void* stream);

/* Replace chunk `chunk_index` of the cache by the real observation's keys and
 * values (hyper.ai summary of the paper, "方法" paragraph 4: after the action
 * chunk executes, the predicted frames in the KV cache are replaced by the
 * real observation).  Overwrites rows [c*L, (c+1)*L) (L = cache->chunk_len)
 * of every batch item with k, v bf16 [batch][L][H][128]; len_tokens is
 * unchanged.  Bit-exact copy.
 * Errors: DZ_ERR_INVALID_ARG (chunk not fully inside [0, len_tokens)),
 * DZ_ERR_ALIGNMENT, DZ_ERR_CUDA. */
dz_status dz_kvcache_replace(dz_attn_t handle, dz_kvcache* cache, int32_t chunk_index,
                             const void* k, const void* v, void* stream);

/* Training form of the attention: dz_chunk_attn_forward for DZ_MODE_PREFILL or
 * DZ_MODE_TEACHER_FORCING (no cache), which also writes, for every query row,
 * the log2-domain normaliser of its softmax,
 *   lse[b][h][s] = log2( sum over visible keys j of 2^(S_sj * log2(e)) ),
 *   S = (R q)(R k)^T / sqrt(128) in fp32,
 * as fp32 [B][H][Sq] (16-byte aligned).  dz_chunk_attn_backward consumes it.
 * Errors: as dz_chunk_attn_forward, and DZ_ERR_UNSUPPORTED for other modes. */
dz_status dz_chunk_attn_forward_lse(dz_attn_t handle, const void* q, const void* k, const void* v,
                                    const dz_chunk_layout* layout, void* out, void* lse,
                                    void* stream);

/* Backward of the prefill / teacher-forcing attention (the training form of the
 * chunk mask: hyper.ai summary of the paper, "方法" (teacher forcing); the
 * walkthrough's training objective, Fig. 14).  Given the forward's inputs
 * q, k, v (unrotated), its output `out`, its `lse` (dz_chunk_attn_forward_lse)
 * and the output gradient `dout` (all bf16 [B][S][H][128] but lse), writes the
 * gradients of sum(dout * out) with respect to q, k and v:
 *   dv = P^T dout,  dP = dout v^T,  dS = P * (dP - rowsum(dout * out)),
 *   dq = R^T (dS (R k)) / sqrt(128),  dk = R^T (dS^T (R q)) / sqrt(128),
 * accumulated in fp32 and rounded once to bf16 (dq, dk, dv [B][S][H][128]).
 * Uses the handle's rotation workspace (prerotate_tokens >= S) and its split
 * workspace (B * H * S floats); calls on one handle must not overlap.
 * Errors: DZ_ERR_INVALID_ARG, DZ_ERR_ALIGNMENT, DZ_ERR_SHAPE, DZ_ERR_UNSUPPORTED
 * (DECODE or CROSS), DZ_ERR_CAPACITY (batch, tokens or workspaces beyond the
 * handle), DZ_ERR_CUDA. */
dz_status dz_chunk_attn_backward(dz_attn_t handle, const void* q, const void* k, const void* v,
                                 const void* out, const void* dout, const void* lse,
                                 const dz_chunk_layout* layout, void* dq, void* dk, void* dv,
                                 void* stream);

/* QKV projection with the rotary embedding and the KV-cache append fused into
 * one GEMM ("DreamZero (WAM) 模型架构", §2.3 block diagram: the causal
 * self-attention of each DiT block takes the normalised, modulated hidden
 * state [B, T, 5120]; RoPE acts on the latent sequence).  For the S tokens of
 * each batch item:
 *   [q | k | v] = x W^T  (fp32 accumulation of bf16 products),
 *   q, k turned by R(pos(s)) in fp32 (the rule of dz_rope3d: token s is token
 *   s % L of chunk first_chunk + s / L of `layout`), then q, k, v rounded once
 *   to bf16.
 *   x    bf16 [B][S][d_model], row-major; d_model a positive multiple of 64.
 *   w    bf16 [3 * H * 128][d_model]: row n is output feature n; rows
 *        [0, H*128) give q (head-major, 128 per head), then k, then v.
 *   q_out, k_out, v_out  bf16 [B][S][H][128] (H = the handle's num_heads).
 *   cache  NULL, or a cache to append to: k and v are also written to rows
 *        [len_tokens, len_tokens + S) of every batch item and len_tokens
 *        advances by S (S must equal cache->chunk_len; batch must match).
 * No bias term (the pages give none).  All pointers 16-byte aligned.
 * Errors: DZ_ERR_INVALID_ARG, DZ_ERR_ALIGNMENT, DZ_ERR_SHAPE (d_model, or
 * positions beyond the handle's tables), DZ_ERR_CAPACITY (batch beyond the
 * handle, cache full), DZ_ERR_CUDA; nothing is written on error. */
dz_status dz_qkv_rope(dz_attn_t handle, const void* x, const void* w, int32_t B, int32_t S,
                      int32_t d_model, const dz_chunk_layout* layout, int32_t first_chunk,
                      void* q_out, void* k_out, void* v_out, dz_kvcache* cache, void* stream);

/* The same attention as dz_chunk_attn_forward, for callers that cannot call
 * cudaMalloc: code that runs while a stream is being captured in global mode,
 * runtimes that hand out device memory only from a pool they reserved up
 * front, or plug-ins held to a fixed memory budget.  The paper has no
 * counterpart; this is an interface choice of this library.
 *
 * It needs no handle and allocates nothing.  Its scratch memory (split
 * results, split counters, a status word: 16.25 MiB) and its rotary tables
 * (up to 294912 (cos, sin) entries, 2.25 MiB) are static device arrays of the
 * library, which every GPU that loads the library holds until the process
 * exits.  Limits (DZ_ERR_CAPACITY beyond them):
 *   desc->max_batch * num_heads * ceil(desc->max_q_tokens / 256) * 2 <= 65536,
 *   max_pos_t*pairs_t + max_pos_h*pairs_h + max_pos_w*pairs_w <= 294912;
 * the split uses at most 63 CTAs, so large calls run slower than through a
 * handle.  The first call on a device looks up the arrays' device addresses,
 * and the first call with a given rotary configuration (base, pairs, max_pos)
 * waits until the device is idle (earlier calls may still read the old tables)
 * and then fills the tables with a synchronous copy: make those calls before
 * any stream capture.  Every call clears the split counters on `stream` and
 * then uses the same arrays, which keep the last call's contents: calls that
 * overlap on the GPU (other streams, other threads) race and give wrong
 * results.  A device-side timeout (a bounded wait that ran out, leaving `out`
 * incomplete) is kept in the static status word until dz_attn_sync_status(NULL,
 * stream) reads and clears it.  Arguments as dz_chunk_attn_forward, with desc
 * in place of the handle. */
dz_status dz_chunk_attn_forward_noalloc(const dz_attn_desc* desc, const void* q, const void* k,
                                        const void* v, const dz_kvcache* cache,
                                        const dz_chunk_layout* layout, void* out, void* stream);

/* Synchronise `stream`, read and clear the handle's device status word.
 * Returns DZ_ERR_TIMEOUT if a kernel's bounded wait ran out since the last
 * read (that call's output is incomplete), DZ_ERR_BOUNDS if a kernel of the
 * bounds-checked test build found an index outside its buffer (the access was
 * skipped; never returned by the product build), DZ_ERR_CUDA on a CUDA error,
 * else DZ_OK.  With a NULL handle it reads and clears the status word of the
 * allocation-free calls (dz_chunk_attn_forward_noalloc) on the current device
 * instead (DZ_OK if none was made there). */
dz_status dz_attn_sync_status(dz_attn_t handle, void* stream);

/* Static English name of a status code. */
const char* dz_status_string(dz_status status);

#ifdef __cplusplus
}
#endif

#endif /* DZ_H_ */
