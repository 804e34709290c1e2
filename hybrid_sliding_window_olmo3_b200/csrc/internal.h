// Host-side launchers of the kernels, called by the C ABI in olmo3_abi.cu after
// argument validation.  Each returns a cudaError_t from the launch.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "olmo3.h"

namespace olmo3 {

struct RopeTable {
  double inv_freq[64];  // angle per position of pair i < d/2 (theta^(-2i/d) for plain RoPE)
  float out_scale;      // applied to the rotated q and k (1; YaRN's attention temperature)
};

cudaError_t launch_qknorm_rope(const void *q, const void *k, const void *v, int in_dtype, const float *gain_q,
                               const float *gain_k, void *q_out, void *k_out, void *v_out,
                               const int32_t *pos_offset, int B, int T, int H, int G, int d, float eps,
                               const RopeTable &tab, cudaStream_t stream);

cudaError_t launch_kv_append(const olmo3_kv_cache &c, const void *k_new, const void *v_new,
                             const int32_t *pos_offset, int T, int32_t *slot_out, int *err, cudaStream_t stream);

cudaError_t launch_attn_mask(int T, int window, int layer_type, uint8_t *out, cudaStream_t stream);

// Split plan of the decode kernel (keys per split and splits per (sequence, head)).
struct DecodePlan {
  int chunk;
  int n_splits;
};
DecodePlan plan_decode(int B, int G, int n_max, int num_splits, bool mma);
constexpr int kDecodeTile = 32;     // keys per pipeline stage, one query head per key/value head
constexpr int kDecodeGqaTile = 64;  // keys per pipeline stage, several query heads per key/value head
constexpr int kDecodeGrain = 64;    // split chunks are multiples of this many keys
constexpr int kDecodeMaxGroup = 16; // query heads per key/value head the decode kernels accept
// The grouped-query decode (H/G > 1) reads 128-byte-swizzled 64x64 tiles; the
// one-head decode reads unswizzled d x 32 tiles.
inline bool decode_uses_mma(int H, int G) { return H / G > 1; }

cudaError_t launch_attn_decode(const CUtensorMap &tmK, const CUtensorMap &tmV, const void *q, int H,
                               const olmo3_kv_cache &c, const int32_t *kv_len, const DecodePlan &plan, void *out,
                               float *lse_out, float scale, float *ws, int *err, cudaStream_t stream);

constexpr int kPrefillBM = 128;  // query rows per CTA
constexpr int kPrefillBN = 128;  // keys per tile

// Where the keys of a prefill come from (see attn_prefill_kernel).
constexpr int kPrefillFresh = 0;   // the sequence itself, positions 0 .. T-1
constexpr int kPrefillCache = 1;   // a linear cache already holding the chunk
constexpr int kPrefillWindow = 2;  // a gathered window of a ring plus the chunk
constexpr int kPrefillRing = 3;    // a ring read in place, the chunk, and one bridge tile

// Extra key sources of kPrefillRing (3-d maps like tmK / tmV): the chunk's own
// keys and values [B*T, G, d], and the bridge tile [B*128, G, d] that holds the
// 128 positions around the chunk's start (ring rows before it, chunk rows after).
struct PrefillExtraMaps {
  CUtensorMap k_new, v_new, k_br, v_br;
};

// tmK / tmV are 3-d maps over [rows, G, d] with 64 x 1 x 128 boxes (128-byte swizzle).
// For kPrefillRing, tmK / tmV map the cache [total_slots, G, d] and `extra` the other
// sources; the window must be a multiple of kPrefillBN.  `extra` is ignored otherwise.
cudaError_t launch_attn_prefill(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV, void *out,
                                float *lse_out, int B, int Tq, int Tk, int H, int G, int d, int layer_type,
                                int window, float scale, int mode, const int32_t *pos_offset,
                                const int64_t *seq_base, int *err, cudaStream_t stream,
                                const PrefillExtraMaps *extra = nullptr);

// The bridge tile of kPrefillRing: rows j < 128 of [B, 128, G, d] hold position
// 128 * floor(p0 / 128) + j: from the ring below p0, from the chunk from p0 on, zeros
// past the chunk.
cudaError_t launch_bridge_tile(const olmo3_kv_cache &c, const void *k_new, const void *v_new,
                               const int32_t *pos_offset, int T, void *k_out, void *v_out, cudaStream_t stream);

// Copies, for each sequence, the window of keys a chunk at pos_offset[b] needs:
// rows j < Tk of [B, Tk, G, d] hold position max(0, p0 - window + 1) + j, from the
// ring for positions < p0 and from the chunk after; rows past the chunk are zeroed.
cudaError_t launch_gather_window(const olmo3_kv_cache &c, const void *k_new, const void *v_new,
                                 const int32_t *pos_offset, int T, int Tk, void *k_out, void *v_out,
                                 cudaStream_t stream);

// Persistent tcgen05 GEMMs with the row norm fused into the epilogue (proj_gemm.cu).
// A norm group (the q or the k columns of a row, or a whole Wo row) may span at
// most proj_gemm_max_tiles_per_row() 256-column tiles.  The workspace starts with proj_gemm_flags_bytes(M, groups) bytes that the
// launcher zeroes (per-row sums of squares and per-row-block counters; groups = 2
// for q and k, 1 for Wo).
int proj_gemm_max_tiles_per_row();
size_t proj_gemm_flags_bytes(int M, int groups);
constexpr int kProjTileN = 256;

// q, k, v = split(X W^T); q, k <- RoPE(RMSNorm(.)) as in launch_qknorm_rope.
// tmX: 2-d map over X [B*T, Dm] with 64 x 128 boxes; tmW over W [(H+2G) d, Dm] with
// 64 x 256 boxes (both 128-byte swizzle).  Requires H*d and G*d multiples of 256.
cudaError_t launch_qkv_proj(const CUtensorMap &tmX, const CUtensorMap &tmW, void *q, void *k, void *v,
                            const float *gain_q, const float *gain_k, const int32_t *pos_offset, int B, int T, int H,
                            int G, int d, int Dm, float eps, const RopeTable &tab, void *ws, int *err,
                            cudaStream_t stream);

// h = x + (A B^T) rsqrt(rowmean((A B^T)^2) + eps) gain.  tmA: 2-d map over A [M, K]
// with 64 x 128 boxes; tmB: over B [N, K] with 64 x 256 boxes.
cudaError_t launch_out_proj(const CUtensorMap &tmA, const CUtensorMap &tmB, const float *gain, const void *x, void *h,
                            int M, int N, int K, float eps, void *ws, int *err, cudaStream_t stream);

}  // namespace olmo3
