/*
 * olmo3.h - C ABI of the OLMo 3 hybrid sliding-window attention library (libolmo3.so).
 *
 * The library computes, on one B200 (sm_100a), the attention hot path of OLMo 3
 * inference as the pages define it, and the attention block's two projections with
 * their norms fused in:
 *
 *   [PATTERN] "OLMo 3's Sliding-Window Attention Pattern" (scratchllm.com problem page):
 *             "Which layers are full", "The sliding-window mask", "Hint".
 *   [CASE]    "Case Study: OLMo 3" (scratchllm.com learn page), "The architecture":
 *             ingredient 1 (bias-free projections, GQA), 2 (QK-norm), 3 (RoPE,
 *             theta = 500,000, rotate half), 4 (sliding-window attention),
 *             6 (reordered norm), 7 (YaRN on the full layers of the long-context model).
 *   [COUNT]   "Count OLMo 3's Parameters" (scratchllm.com), "What to count":
 *             QK-norm gains of sizes H*d and G*d.
 *   [README]  "Olmo-3 End-to-End Implementation" (GitHub README): "Inference Pipeline",
 *             "KV Cache Implementation", "Technical Details".
 *   [SERVING] "Olmo 3 7B" (inference-research record): a windowed decode kernel plus
 *             per-layer-type cache management; one kernel serves sliding and full layers.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers unless the name ends in _host.  The
 *     caller owns every buffer (inputs, outputs, caches, workspace); the library
 *     allocates nothing and keeps no per-call state.
 *   - Layouts are row-major, innermost dimension last:
 *       q [B, T, H, d], k and v [B, T, G, d], attention output [B, T, H, d];
 *       decode query/output [B, H, d]; cache K and V [total_slots, G, d].
 *     bf16 means IEEE bfloat16 (2 bytes), f32 means IEEE binary32.
 *   - d (head size) must be 64 or 128; H must be a multiple of G.
 *   - `stream` is a cudaStream_t cast to void* (NULL = legacy default stream).
 *     Calls are asynchronous and stream-ordered.
 *   - Return value: OLMO3_OK or a negative status.  Arguments are validated on
 *     the host before anything is launched; a failed validation launches nothing.
 *   - Errors found on the device (a position beyond a cache's capacity, a kv_len
 *     out of range, a bounded wait that gave up) are OR-ed as OLMO3_DEVERR_* bits
 *     into *err_dev when err_dev is not NULL; the kernel then skips the offending
 *     access instead of trapping.  The caller zeroes *err_dev and reads it back.
 */
#ifndef OLMO3_H
#define OLMO3_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define OLMO3_OK               0
#define OLMO3_ERR_INVALID_ARG (-1)  /* null pointer, negative size, bad enum, misalignment */
#define OLMO3_ERR_UNSUPPORTED (-2)  /* d not in {64,128}, H % G != 0, H/G > 16, too-wide rows */
#define OLMO3_ERR_WORKSPACE   (-3)  /* workspace missing or smaller than required */
#define OLMO3_ERR_CUDA        (-4)  /* a CUDA runtime call or launch failed */

/* ---- device error bits (OR-ed into *err_dev) -------------------------- */
#define OLMO3_DEVERR_CAPACITY  1    /* a position maps beyond the cache's capacity/slots */
#define OLMO3_DEVERR_KV_LEN    2    /* kv_len < 1, beyond capacity, or above max_kv_len */
#define OLMO3_DEVERR_TIMEOUT   4    /* a bounded pipeline wait gave up; outputs invalid */

/* ---- enums -------------------------------------------------------------- */
#define OLMO3_SLIDING 0             /* query t sees key s iff s <= t and t - s < window */
#define OLMO3_FULL    1             /* query t sees key s iff s <= t */
#define OLMO3_F32     0
#define OLMO3_BF16    1

/*
 * olmo3_layer_types - the hybrid layer pattern.  [PATTERN] "Which layers are
 * full"; [CASE] ingredient 4: layer l (from 0) is full when l mod 4 == 3 or l is
 * the last layer, sliding otherwise.
 *   n_layers  >= 0.
 *   out_host  HOST array of n_layers bytes; receives OLMO3_SLIDING / OLMO3_FULL.
 * Host-only; never touches the GPU.  INVALID_ARG on n_layers < 0 or NULL out_host
 * (with n_layers > 0).
 */
int olmo3_layer_types(int n_layers, uint8_t *out_host);

/*
 * olmo3_attn_mask - writes the T x T mask of one layer type, the same predicate
 * every attention kernel applies.  [PATTERN] "The sliding-window mask" (a full
 * layer gets the plain causal mask).
 *   out_dev   device uint8 [T, T]: out[t*T + s] = 1 if query t may attend key s.
 *   window    >= 1 (ignored for OLMO3_FULL).
 * For tests and debugging; T*T bytes must fit the caller's buffer.
 */
int olmo3_attn_mask(int T, int window, int layer_type, uint8_t *out_dev, void *stream);

/*
 * olmo3_qknorm_rope - fused QK-norm + RoPE (+ optional bf16 cast of v).
 *   [CASE] ingredient 2: RMSNorm of the projected queries and keys before
 *   attention, one gain per feature ([COUNT]: H*d for queries, G*d for keys),
 *   computed over the whole H*d (G*d) vector of a token:
 *       y = x / sqrt(mean(x^2) + eps) * gain.
 *   [CASE] ingredient 3 and [README] "Inference Pipeline": rotate-half RoPE at
 *   absolute position p = pos_offset[b] + t, pair (i, i + d/2) of every head:
 *       a = p * theta^(-2i/d),
 *       y'_i = y_i cos a - y_{i+d/2} sin a,  y'_{i+d/2} = y_{i+d/2} cos a + y_i sin a.
 *   Angles are formed and reduced in fp64; the norm and rotation run in fp32.
 *
 *   q, k        [B,T,H,d] / [B,T,G,d], element type in_dtype (OLMO3_F32 or OLMO3_BF16).
 *   v, v_out    optional: when v_out != NULL, v [B,T,G,d] (in_dtype) is copied to
 *               v_out as bf16 (a cast; no norm, no rotation: RoPE is on q and k only).
 *   gain_q      f32 [H*d];  gain_k  f32 [G*d].
 *   q_out,k_out bf16, same shapes as q, k.  May alias q, k when in_dtype == BF16.
 *   pos_offset  int32 [B], position of token t = 0 of sequence b.
 *   eps >= 0, theta > 0.  Requires H*d <= 8192 and G*d <= 8192.
 */
int olmo3_qknorm_rope(const void *q, const void *k, const void *v, int in_dtype,
                      const float *gain_q, const float *gain_k,
                      void *q_out, void *k_out, void *v_out,
                      const int32_t *pos_offset, int B, int T, int H, int G, int d,
                      float eps, double theta, void *stream);

/*
 * olmo3_qknorm_rope_yarn - olmo3_qknorm_rope with YaRN-rescaled RoPE, for the
 * full-attention layers of the long-context model ([CASE] ingredient 7: RoPE on the
 * full layers is rescaled with YaRN from the 8,192 training positions to 65,536;
 * [SERVING]: factor 8 from an 8192 base).  The pages give only the factor and the
 * base; the rest is the YaRN method's "NTK-by-parts" rule: pair i turns
 * r = original_context * f_i / (2 pi) times over the original context, keeps its
 * frequency f_i = theta^(-2i/d) when r >= beta_fast, uses f_i / factor when
 * r <= beta_slow, and blends linearly in between; the rotated q and k are both
 * multiplied by 0.1 ln(factor) + 1 (the attention temperature).  factor == 1 is
 * exactly olmo3_qknorm_rope.  Typical: factor 8, original_context 8192,
 * beta_fast 32, beta_slow 1.  Other arguments as olmo3_qknorm_rope.
 */
int olmo3_qknorm_rope_yarn(const void *q, const void *k, const void *v, int in_dtype,
                           const float *gain_q, const float *gain_k,
                           void *q_out, void *k_out, void *v_out,
                           const int32_t *pos_offset, int B, int T, int H, int G, int d,
                           float eps, double theta, double factor, int original_context,
                           double beta_fast, double beta_slow, void *stream);

/*
 * olmo3_kv_cache - a preallocated per-layer-type cache ([SERVING]: per-layer-type
 * cache management; replaces the concatenation-grown cache of [README] "KV Cache
 * Implementation").
 *   k, v         bf16 [total_slots, G, d]; row (slot, g) holds a key (value) after
 *                QK-norm and RoPE, at its absolute position.
 *   seq_base     device int64 [B]: first slot of sequence b.  Sequence b owns slots
 *                seq_base[b] .. seq_base[b] + capacity - 1.
 *   total_slots  rows in k and v (bounds every access).
 *   capacity     slots per sequence.  Sliding layers: a ring, capacity == window,
 *                position p lives in slot p mod window.  Full layers: linear,
 *                position p lives in slot p (p < capacity).
 */
typedef struct olmo3_kv_cache {
    void *k;
    void *v;
    const int64_t *seq_base;
    int64_t total_slots;
    int capacity;
    int layer_type;
    int window;
    int B;
    int G;
    int d;
} olmo3_kv_cache;

/*
 * olmo3_kv_append - writes T new rows per sequence (positions pos_offset[b] + t)
 * into the cache: ring slot p mod window (sliding) or slot p (full).  When T >
 * window on a sliding layer only the last `window` rows are written (the others
 * would be overwritten by the same call).  [README] "Inference Pipeline" step 3
 * (update cache with new key/value pairs).
 *   c           cache descriptor (HOST pointer to the struct; its pointers are device).
 *   k_new,v_new bf16 [B, T, G, d] (k_new after QK-norm and RoPE).
 *   pos_offset  int32 [B].
 *   slot_out    optional int32 [B, T]: slot written, or -1 for a row not written.
 *   err_dev     optional: OLMO3_DEVERR_CAPACITY when a row maps beyond capacity or
 *               total_slots (that row is skipped).
 */
int olmo3_kv_append(const olmo3_kv_cache *c, const void *k_new, const void *v_new,
                    const int32_t *pos_offset, int T, int32_t *slot_out, int *err_dev,
                    void *stream);

/*
 * olmo3_attn_prefill - causal self-attention of a fresh sequence over itself,
 * band-limited for sliding layers.  [PATTERN] mask; [CASE] ingredients 1 and 4.
 *   O[b,t,h] = sum_{s allowed} softmax_s(scale * q_t . k_s) v_s, allowed =
 *   s <= t and (layer_type == FULL or t - s < window); query head h reads
 *   key/value head h / (H/G).
 *   q           bf16 [B,T,H,d] (after QK-norm + RoPE);  k, v  bf16 [B,T,G,d].
 *   out         bf16 [B,T,H,d].
 *   lse_out     optional f32 [B,H,T]: natural-log softmax denominator of the
 *               scaled logits.
 *   scale       logit scale (1/sqrt(d) in the binding by default).
 *   Positions are 0..T-1.  Tensor-core kernel (tcgen05, TMEM accumulators, TMA).
 *   Base pointers must be 16-byte aligned.
 *   err_dev     optional: OLMO3_DEVERR_TIMEOUT if a pipeline wait gave up.
 */
int olmo3_attn_prefill(const void *q, const void *k, const void *v, void *out,
                       int B, int T, int H, int G, int d, int layer_type, int window,
                       float scale, float *lse_out, int *err_dev, void *stream);

/*
 * olmo3_attn_prefill_chunk - a chunk of T prompt tokens per sequence at positions
 * pos_offset[b] + t attends over the cache of its sequence (the positions before
 * the chunk) plus the chunk itself, and the chunk is appended to the cache.  This
 * is prefill with a position offset into a live cache ([README] "Inference
 * Pipeline": RoPE with position offsets for cache compatibility), so a long prompt
 * can be fed in pieces; the result equals the rows of a one-shot prefill.
 *   q           bf16 [B, T, H, d] after QK-norm + RoPE at positions pos_offset[b] + t.
 *   k_new,v_new bf16 [B, T, G, d] (k_new after QK-norm + RoPE).
 *   c           the layer's cache (HOST pointer to the struct), holding positions
 *               0 .. pos_offset[b] - 1 of each sequence (the ring: its last window).
 *   pos_offset  int32 [B].  out bf16 [B, T, H, d];  lse_out optional f32 [B, H, T].
 *   Full layers: the chunk is appended first (it overwrites nothing), then the
 *   chunk attends over cache rows 0 .. pos_offset + T - 1; no workspace is used.
 *   Sliding layers: appending first would overwrite keys the chunk's early rows
 *   still need, so the chunk attends first and is appended after.  When window is
 *   a multiple of 128 the keys are read in place, 128-position tiles from the ring
 *   before pos_offset and from k_new / v_new after it, and only the one tile that
 *   straddles pos_offset is copied into `workspace`; for any other window the
 *   window [pos_offset - window + 1, pos_offset) is gathered from the ring together
 *   with the chunk into `workspace`.  Size: olmo3_attn_prefill_chunk_workspace_size
 *   (2 * B * 128 * G * d * 2 bytes, or 2 * B * (window - 1 + T) * G * d * 2).
 *   Cache slots never written must hold finite values (allocate caches zeroed).
 *   err_dev as for olmo3_kv_append and olmo3_attn_prefill.
 */
size_t olmo3_attn_prefill_chunk_workspace_size(int B, int T, int G, int d, int layer_type, int window);
int olmo3_attn_prefill_chunk(const void *q, const void *k_new, const void *v_new,
                             const olmo3_kv_cache *c, const int32_t *pos_offset, int T, int H,
                             void *out, float scale, float *lse_out, void *workspace,
                             size_t ws_bytes, int *err_dev, void *stream);

/*
 * olmo3_attn_decode_workspace_size - bytes of f32 workspace olmo3_attn_decode
 * needs for these sizes (the split-KV partials).  max_kv_len is the largest
 * kv_len of the call; num_splits as for olmo3_attn_decode (0 = automatic).
 * Returns 0 on invalid arguments.
 */
size_t olmo3_attn_decode_workspace_size(int B, int H, int G, int d, int max_kv_len,
                                        int layer_type, int window, int num_splits);

/*
 * olmo3_attn_decode - one new query token per sequence over its cache
 * ([README] "Inference Pipeline" step 3; [SERVING]: a sliding layer reads
 * exactly min(kv_len, window) entries, a full layer kv_len).
 *   q           bf16 [B, H, d] after QK-norm + RoPE at position kv_len[b] - 1, whose
 *               key/value row is already appended.
 *   c           cache of this layer (HOST pointer to the struct).
 *   kv_len      int32 [B]: tokens of sequence b so far (new token included), >= 1.
 *   max_kv_len  host upper bound of kv_len (sizes the split plan).
 *   out         bf16 [B, H, d];  lse_out optional f32 [B, H].
 *   num_splits  split-KV pieces per (sequence, head); 0 = automatic.
 *   workspace   f32 scratch of olmo3_attn_decode_workspace_size() bytes (ws_bytes).
 *   err_dev     optional: OLMO3_DEVERR_KV_LEN (that sequence's output is zeroed),
 *               OLMO3_DEVERR_TIMEOUT.
 * The valid entries of sequence b are slots 0 .. n-1 of its range, n = kv_len for
 * full layers and min(kv_len, window) for sliding layers: every key held by the
 * ring is inside the window of the newest token, so no further mask is needed.
 */
int olmo3_attn_decode(const void *q, int H, const olmo3_kv_cache *c,
                      const int32_t *kv_len, int max_kv_len, void *out, float *lse_out,
                      float scale, int num_splits, void *workspace, size_t ws_bytes,
                      int *err_dev, void *stream);

/*
 * olmo3_attn_decode_noalloc - olmo3_attn_decode for callers that cannot allocate
 * device memory.  The pages have no counterpart: this is a library convenience.
 *   Some callers only ever receive input and output buffers from a host framework
 *   (a plugin or custom-operator interface with no workspace argument), or run
 *   without an allocator of their own, where a cudaMalloc would synchronise the
 *   device or break a fixed memory budget.  This entry point takes the same
 *   arguments as olmo3_attn_decode minus the workspace, and keeps the split-KV
 *   partials in a buffer of OLMO3_NOALLOC_SCRATCH_BYTES that the library holds as
 *   a file-scope device array (present on every GPU that loads the library, until
 *   the process exits).  It calls no cudaMalloc, cudaFree or allocating routine.
 *   Limit: a call whose olmo3_attn_decode_workspace_size() exceeds
 *   OLMO3_NOALLOC_SCRATCH_BYTES returns OLMO3_ERR_WORKSPACE and launches nothing
 *   (a smaller num_splits lowers the need).
 *   Set-up: the first call on each device looks up the buffer's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call before
 *   any stream capture.
 *   Sharing: every call uses the same buffer and it keeps the last call's
 *   contents (harmless: each value read is written earlier in the same call).
 *   Calls that overlap on the GPU (other streams, other threads) race on it:
 *   order them on one stream or serialise them.
 */
#define OLMO3_NOALLOC_SCRATCH_BYTES (16u << 20)
int olmo3_attn_decode_noalloc(const void *q, int H, const olmo3_kv_cache *c,
                              const int32_t *kv_len, int max_kv_len, void *out,
                              float *lse_out, float scale, int num_splits, int *err_dev,
                              void *stream);

/*
 * olmo3_out_proj_postnorm_residual - the attention block's output side: the
 * bias-free output projection, then the reordered norm and the residual add
 * ([CASE] ingredients 1 and 6, "Reordered norm": h = x + RMSNorm(Attention(x)),
 * the norm acting on the projected attention output before the addition):
 *     Y = attn W_o^T,   h = x + Y / sqrt(mean_j(Y_j^2) + eps) * gain.
 *   attn    bf16 [M, K]: the attention output, heads side by side (K = H*d).
 *   w_o     bf16 [D, K]: row j maps the attention features to model feature j.
 *   gain    f32 [D];  x  bf16 [M, D] residual stream;  h_out bf16 [M, D] (may alias x).
 *   workspace  olmo3_out_proj_workspace_size(M, D) bytes (per-row sums of squares and
 *              per-row-block counters; zeroed by the call itself).
 *   err_dev    optional device int; OLMO3_DEVERR_TIMEOUT is or-ed in when a wait gave up.
 *   Requires K % 64 == 0, D % 8 == 0 and D <= 256 * (SM count).  One persistent
 *   kernel on tcgen05 tensor cores (128 x 256 tiles, f32 accumulation in tensor
 *   memory): the norm of a row needs all of its D features, which span several
 *   tiles, so each tile publishes its share of the row sums, waits (bounded) for
 *   the other tiles of its 128 rows, then writes h; Y never goes to HBM.
 */
size_t olmo3_out_proj_workspace_size(int M, int D);
int olmo3_out_proj_postnorm_residual(const void *attn, const void *w_o, const float *gain,
                                     const void *x, void *h_out, int M, int D, int K, float eps,
                                     void *workspace, size_t ws_bytes, int *err_dev, void *stream);

/*
 * olmo3_qkv_proj_qknorm_rope - the attention block's input side in one kernel:
 * the bias-free Q, K and V projections of the block input ([CASE] ingredient 1;
 * ingredient 6 leaves that input un-normed), then QK-norm and RoPE on q and k
 * exactly as olmo3_qknorm_rope_yarn (plain RoPE when rope_factor == 1):
 *     [q | k | v] = x W_qkv^T,  q <- RoPE(RMSNorm_{H*d}(q) gain_q),  k likewise over G*d.
 *   x       bf16 [B, T, D] (D = model width; rows b*T + t).
 *   w_qkv   bf16 [(H + 2G) d, D]: rows of W_q (H*d), then W_k (G*d), then W_v (G*d).
 *   gain_q  f32 [H*d];  gain_k  f32 [G*d];  pos_offset int32 [B] as olmo3_qknorm_rope.
 *   q_out   bf16 [B, T, H, d];  k_out, v_out  bf16 [B, T, G, d]; none may alias x.
 *   theta, rope_factor, original_context, beta_fast, beta_slow: as olmo3_qknorm_rope_yarn.
 *   workspace  olmo3_qkv_proj_workspace_size(B*T) bytes, 16-byte aligned (per-row
 *              sums of squares of q and k, per-row-block counters; zeroed by the call).
 *   err_dev    optional device int; OLMO3_DEVERR_TIMEOUT is or-ed in when a wait gave up.
 *   Requires d in {64, 128}, D % 64 == 0, H*d and G*d multiples of 256, and
 *   H*d, G*d <= 256 * (SM count); OLMO3_ERR_UNSUPPORTED otherwise.
 *   One persistent tcgen05 kernel (128 x 256 tiles): the epilogue applies the gains
 *   and the rotation to the f32 accumulator, and the per-row RMSNorm factor (which
 *   needs the sums over all q or all k tiles of the row) once every tile of the
 *   row's 128-row block has published its share.
 */
size_t olmo3_qkv_proj_workspace_size(int M);
int olmo3_qkv_proj_qknorm_rope(const void *x, const void *w_qkv, const float *gain_q,
                               const float *gain_k, void *q_out, void *k_out, void *v_out,
                               const int32_t *pos_offset, int B, int T, int H, int G, int d,
                               int D, float eps, double theta, double rope_factor,
                               int original_context, double beta_fast, double beta_slow,
                               void *workspace, size_t ws_bytes, int *err_dev, void *stream);

/* olmo3_status_string - a static English description of a status code. */
const char *olmo3_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* OLMO3_H */
