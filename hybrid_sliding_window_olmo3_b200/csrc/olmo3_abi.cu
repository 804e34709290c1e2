// The C ABI of libolmo3 (declared in include/olmo3.h): host-side argument
// validation, TMA tensor-map encoding and kernel launches.  Nothing here
// allocates device memory; every buffer belongs to the caller.
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "internal.h"
#include "olmo3.h"

using namespace olmo3;

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool encoder_ready() {
  std::call_once(g_encode_once, [] {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode != nullptr;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_d(int d) { return d == 64 || d == 128; }
bool valid_type(int t) { return t == OLMO3_SLIDING || t == OLMO3_FULL; }
cudaStream_t as_stream(void *s) { return static_cast<cudaStream_t>(s); }
int cuda_status(cudaError_t e) { return e == cudaSuccess ? OLMO3_OK : OLMO3_ERR_CUDA; }

// bf16 tensor of rank `rank` (dims innermost first, byte strides of dims 1..rank-1).
bool encode_bf16(CUtensorMap *tm, const void *base, int rank, const cuuint64_t *dims, const cuuint64_t *strides,
                 const cuuint32_t *box, CUtensorMapSwizzle swz) {
  if (!encoder_ready()) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = g_encode(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void *>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// q / out [B, T, H, d] as a 4-d map (query tiles of 128 rows of one head).
bool encode_q(CUtensorMap *tm, const void *q, int B, int T, int H, int d) {
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(kPrefillBM), 1};
  const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
  return encode_bf16(tm, q, 4, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// K or V rows [rows, G, d] as a 3-d map (key tiles of 128 rows of one key/value head).
bool encode_kv(CUtensorMap *tm, const void *base, int64_t rows, int G, int d) {
  const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kPrefillBN)};
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)G, (cuuint64_t)rows};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)G * d * 2};
  return encode_bf16(tm, base, 3, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

int validate_cache(const olmo3_kv_cache *c) {
  if (c == nullptr || c->k == nullptr || c->v == nullptr || c->seq_base == nullptr) return OLMO3_ERR_INVALID_ARG;
  if (!valid_type(c->layer_type) || c->B < 0 || c->G < 1 || c->capacity < 1 || c->total_slots < 1 ||
      c->window < 1)
    return OLMO3_ERR_INVALID_ARG;
  if (!valid_d(c->d)) return OLMO3_ERR_UNSUPPORTED;
  if (c->layer_type == OLMO3_SLIDING && c->capacity != c->window) return OLMO3_ERR_INVALID_ARG;
  if (c->total_slots >= (int64_t(1) << 31)) return OLMO3_ERR_UNSUPPORTED;
  if (!aligned16(c->k) || !aligned16(c->v)) return OLMO3_ERR_INVALID_ARG;
  return OLMO3_OK;
}

}  // namespace

extern "C" {

const char *olmo3_status_string(int status) {
  switch (status) {
    case OLMO3_OK: return "ok";
    case OLMO3_ERR_INVALID_ARG: return "invalid argument";
    case OLMO3_ERR_UNSUPPORTED: return "unsupported shape";
    case OLMO3_ERR_WORKSPACE: return "workspace missing or too small";
    case OLMO3_ERR_CUDA: return "CUDA error";
    default: return "unknown status";
  }
}

int olmo3_layer_types(int n_layers, uint8_t *out_host) {
  if (n_layers < 0 || (n_layers > 0 && out_host == nullptr)) return OLMO3_ERR_INVALID_ARG;
  for (int l = 0; l < n_layers; ++l)
    out_host[l] = (l % 4 == 3 || l == n_layers - 1) ? OLMO3_FULL : OLMO3_SLIDING;
  return OLMO3_OK;
}

int olmo3_attn_mask(int T, int window, int layer_type, uint8_t *out_dev, void *stream) {
  if (T < 0 || !valid_type(layer_type) || (layer_type == OLMO3_SLIDING && window < 1)) return OLMO3_ERR_INVALID_ARG;
  if (T == 0) return OLMO3_OK;
  if (out_dev == nullptr) return OLMO3_ERR_INVALID_ARG;
  return cuda_status(launch_attn_mask(T, window, layer_type, out_dev, as_stream(stream)));
}

namespace {
// NTK-by-parts: pair i turns r = original_context * f_i / (2 pi) times over the
// original context; it keeps f_i when r >= beta_fast, becomes f_i / factor when
// r <= beta_slow, and blends linearly in between.  factor 1 is plain RoPE.
bool yarn_table(int d, double theta, double factor, int original_context, double beta_fast, double beta_slow,
                RopeTable *tab) {
  if (!(theta > 0.0) || !(factor >= 1.0) || original_context < 1 || !(beta_fast > beta_slow)) return false;
  const double two_pi = 6.283185307179586476925286766559;
  for (int i = 0; i < 64; ++i) {
    if (i >= d / 2) {
      tab->inv_freq[i] = 0.0;
      continue;
    }
    const double f = pow(theta, -2.0 * i / d);
    if (factor == 1.0) {
      tab->inv_freq[i] = f;
      continue;
    }
    const double r = original_context * f / two_pi;
    double keep = (r - beta_slow) / (beta_fast - beta_slow);
    keep = keep < 0.0 ? 0.0 : (keep > 1.0 ? 1.0 : keep);
    tab->inv_freq[i] = f * keep + (f / factor) * (1.0 - keep);
  }
  tab->out_scale = factor > 1.0 ? static_cast<float>(0.1 * log(factor) + 1.0) : 1.0f;
  return true;
}

// The persistent projection GEMMs need every tile of a 128-row block resident at
// once: at most one SM's worth of tiles per row.
int tiles_per_row_status(int tiles) {
  const int max_tiles = proj_gemm_max_tiles_per_row();
  if (max_tiles <= 0) return OLMO3_ERR_CUDA;
  return tiles > max_tiles ? OLMO3_ERR_UNSUPPORTED : OLMO3_OK;
}

int qknorm_rope_common(const void *q, const void *k, const void *v, int in_dtype, const float *gain_q,
                       const float *gain_k, void *q_out, void *k_out, void *v_out, const int32_t *pos_offset, int B,
                       int T, int H, int G, int d, float eps, const RopeTable &tab, void *stream) {
  if (B < 0 || T < 0 || H < 1 || G < 1 || !(eps >= 0.f) || (in_dtype != OLMO3_F32 && in_dtype != OLMO3_BF16))
    return OLMO3_ERR_INVALID_ARG;
  if (!valid_d(d)) return OLMO3_ERR_UNSUPPORTED;
  if (H * d > 8192 || G * d > 8192) return OLMO3_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * T == 0) return OLMO3_OK;
  if (static_cast<int64_t>(B) * T > 0x7fffffffLL) return OLMO3_ERR_UNSUPPORTED;
  if (!q || !k || !gain_q || !gain_k || !q_out || !k_out || !pos_offset || (v_out && !v))
    return OLMO3_ERR_INVALID_ARG;
  const void *ptrs[] = {q, k, gain_q, gain_k, q_out, k_out};
  for (const void *p : ptrs)
    if (!aligned16(p)) return OLMO3_ERR_INVALID_ARG;
  if (v_out && (!aligned16(v) || !aligned16(v_out))) return OLMO3_ERR_INVALID_ARG;
  return cuda_status(launch_qknorm_rope(q, k, v, in_dtype, gain_q, gain_k, q_out, k_out, v_out, pos_offset, B, T,
                                        H, G, d, eps, tab, as_stream(stream)));
}
}  // namespace

int olmo3_qknorm_rope(const void *q, const void *k, const void *v, int in_dtype, const float *gain_q,
                      const float *gain_k, void *q_out, void *k_out, void *v_out, const int32_t *pos_offset, int B,
                      int T, int H, int G, int d, float eps, double theta, void *stream) {
  if (!(theta > 0.0)) return OLMO3_ERR_INVALID_ARG;
  RopeTable tab;
  for (int i = 0; i < 64; ++i) tab.inv_freq[i] = i < d / 2 ? pow(theta, -2.0 * i / d) : 0.0;
  tab.out_scale = 1.0f;
  return qknorm_rope_common(q, k, v, in_dtype, gain_q, gain_k, q_out, k_out, v_out, pos_offset, B, T, H, G, d, eps,
                            tab, stream);
}

int olmo3_qknorm_rope_yarn(const void *q, const void *k, const void *v, int in_dtype, const float *gain_q,
                           const float *gain_k, void *q_out, void *k_out, void *v_out, const int32_t *pos_offset,
                           int B, int T, int H, int G, int d, float eps, double theta, double factor,
                           int original_context, double beta_fast, double beta_slow, void *stream) {
  RopeTable tab;
  if (!yarn_table(d, theta, factor, original_context, beta_fast, beta_slow, &tab)) return OLMO3_ERR_INVALID_ARG;
  return qknorm_rope_common(q, k, v, in_dtype, gain_q, gain_k, q_out, k_out, v_out, pos_offset, B, T, H, G, d, eps,
                            tab, stream);
}

int olmo3_kv_append(const olmo3_kv_cache *c, const void *k_new, const void *v_new, const int32_t *pos_offset,
                    int T, int32_t *slot_out, int *err_dev, void *stream) {
  int st = validate_cache(c);
  if (st != OLMO3_OK) return st;
  if (T < 0 || c->B > 65535) return OLMO3_ERR_INVALID_ARG;
  if (T == 0 || c->B == 0) return OLMO3_OK;
  if (!k_new || !v_new || !pos_offset || !aligned16(k_new) || !aligned16(v_new)) return OLMO3_ERR_INVALID_ARG;
  return cuda_status(launch_kv_append(*c, k_new, v_new, pos_offset, T, slot_out, err_dev, as_stream(stream)));
}

int olmo3_attn_prefill(const void *q, const void *k, const void *v, void *out, int B, int T, int H, int G, int d,
                       int layer_type, int window, float scale, float *lse_out, int *err_dev, void *stream) {
  if (B < 0 || T < 0 || H < 1 || G < 1 || !valid_type(layer_type) || window < 1 || !isfinite(scale))
    return OLMO3_ERR_INVALID_ARG;
  if (!valid_d(d) || H % G != 0) return OLMO3_ERR_UNSUPPORTED;
  if (B > 65535 || (T + kPrefillBM - 1) / kPrefillBM > 65535) return OLMO3_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * T >= (int64_t(1) << 31)) return OLMO3_ERR_UNSUPPORTED;
  if (B == 0 || T == 0) return OLMO3_OK;
  if (!q || !k || !v || !out) return OLMO3_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return OLMO3_ERR_INVALID_ARG;
  CUtensorMap tmQ, tmK, tmV;
  if (!encode_q(&tmQ, q, B, T, H, d) || !encode_kv(&tmK, k, static_cast<int64_t>(B) * T, G, d) ||
      !encode_kv(&tmV, v, static_cast<int64_t>(B) * T, G, d))
    return OLMO3_ERR_CUDA;
  return cuda_status(launch_attn_prefill(tmQ, tmK, tmV, out, lse_out, B, T, T, H, G, d, layer_type, window, scale,
                                         kPrefillFresh, nullptr, nullptr, err_dev, as_stream(stream)));
}

size_t olmo3_attn_prefill_chunk_workspace_size(int B, int T, int G, int d, int layer_type, int window) {
  if (B < 0 || T < 0 || G < 1 || !valid_d(d) || !valid_type(layer_type) || window < 1) return 0;
  if (layer_type == OLMO3_FULL) return 0;
  if (window % kPrefillBN == 0)  // the ring is read in place; only the bridge tile is copied
    return 2 * static_cast<size_t>(B) * kPrefillBN * G * d * 2;
  return 2 * static_cast<size_t>(B) * (static_cast<size_t>(window) - 1 + T) * G * d * 2;
}

int olmo3_attn_prefill_chunk(const void *q, const void *k_new, const void *v_new, const olmo3_kv_cache *c,
                             const int32_t *pos_offset, int T, int H, void *out, float scale, float *lse_out,
                             void *workspace, size_t ws_bytes, int *err_dev, void *stream) {
  int st = validate_cache(c);
  if (st != OLMO3_OK) return st;
  if (T < 0 || H < 1 || !isfinite(scale)) return OLMO3_ERR_INVALID_ARG;
  if (H % c->G != 0) return OLMO3_ERR_UNSUPPORTED;
  if (c->B > 65535 || (T + kPrefillBM - 1) / kPrefillBM > 65535) return OLMO3_ERR_UNSUPPORTED;
  if (c->B == 0 || T == 0) return OLMO3_OK;
  if (!q || !k_new || !v_new || !out || !pos_offset) return OLMO3_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(out)) return OLMO3_ERR_INVALID_ARG;
  const int B = c->B, G = c->G, d = c->d;
  const size_t need = olmo3_attn_prefill_chunk_workspace_size(B, T, G, d, c->layer_type, c->window);
  const int Tk = c->window - 1 + T;
  if (c->layer_type == OLMO3_SLIDING) {
    if (workspace == nullptr || ws_bytes < need || !aligned16(workspace)) return OLMO3_ERR_WORKSPACE;
    if (static_cast<int64_t>(B) * Tk >= (int64_t(1) << 31)) return OLMO3_ERR_UNSUPPORTED;
  }
  cudaStream_t s = as_stream(stream);
  CUtensorMap tmQ, tmK, tmV;
  if (!encode_q(&tmQ, q, B, T, H, d)) return OLMO3_ERR_CUDA;
  if (c->layer_type == OLMO3_FULL) {
    // the chunk goes into the linear cache first (it overwrites nothing), then the
    // chunk's rows attend over the cache rows 0 .. pos_offset + T - 1
    if (!encode_kv(&tmK, c->k, c->total_slots, G, d) || !encode_kv(&tmV, c->v, c->total_slots, G, d))
      return OLMO3_ERR_CUDA;
    cudaError_t e = launch_kv_append(*c, k_new, v_new, pos_offset, T, nullptr, err_dev, s);
    if (e != cudaSuccess) return OLMO3_ERR_CUDA;
    return cuda_status(launch_attn_prefill(tmQ, tmK, tmV, out, lse_out, B, T, 0, H, G, d, OLMO3_FULL, c->window,
                                           scale, kPrefillCache, pos_offset, c->seq_base, err_dev, s));
  }
  if (c->window % kPrefillBN == 0) {
    // sliding, window a multiple of the key tile: the chunk's rows read their keys in
    // place, ring tiles from the cache and chunk tiles from k_new / v_new; only the
    // tile that straddles the chunk's start is copied (the bridge); then the chunk is
    // appended.
    void *bk = workspace;
    void *bv = static_cast<uint8_t *>(workspace) + need / 2;
    PrefillExtraMaps xm;
    if (!encode_kv(&tmK, c->k, c->total_slots, G, d) || !encode_kv(&tmV, c->v, c->total_slots, G, d) ||
        !encode_kv(&xm.k_new, k_new, static_cast<int64_t>(B) * T, G, d) ||
        !encode_kv(&xm.v_new, v_new, static_cast<int64_t>(B) * T, G, d) ||
        !encode_kv(&xm.k_br, bk, static_cast<int64_t>(B) * kPrefillBN, G, d) ||
        !encode_kv(&xm.v_br, bv, static_cast<int64_t>(B) * kPrefillBN, G, d))
      return OLMO3_ERR_CUDA;
    cudaError_t e = launch_bridge_tile(*c, k_new, v_new, pos_offset, T, bk, bv, s);
    if (e != cudaSuccess) return OLMO3_ERR_CUDA;
    e = launch_attn_prefill(tmQ, tmK, tmV, out, lse_out, B, T, 0, H, G, d, OLMO3_SLIDING, c->window, scale,
                            kPrefillRing, pos_offset, c->seq_base, err_dev, s, &xm);
    if (e != cudaSuccess) return OLMO3_ERR_CUDA;
    return cuda_status(launch_kv_append(*c, k_new, v_new, pos_offset, T, nullptr, err_dev, s));
  }
  // sliding, any other window: the ring's window and the chunk are gathered side by
  // side, attended, then the chunk is appended
  void *wk = workspace;
  void *wv = static_cast<uint8_t *>(workspace) + need / 2;
  if (!encode_kv(&tmK, wk, static_cast<int64_t>(B) * Tk, G, d) || !encode_kv(&tmV, wv, static_cast<int64_t>(B) * Tk, G, d))
    return OLMO3_ERR_CUDA;
  cudaError_t e = launch_gather_window(*c, k_new, v_new, pos_offset, T, Tk, wk, wv, s);
  if (e != cudaSuccess) return OLMO3_ERR_CUDA;
  e = launch_attn_prefill(tmQ, tmK, tmV, out, lse_out, B, T, Tk, H, G, d, OLMO3_SLIDING, c->window, scale,
                          kPrefillWindow, pos_offset, c->seq_base, err_dev, s);
  if (e != cudaSuccess) return OLMO3_ERR_CUDA;
  return cuda_status(launch_kv_append(*c, k_new, v_new, pos_offset, T, nullptr, err_dev, s));
}

size_t olmo3_out_proj_workspace_size(int M, int D) {
  if (M < 0 || D < 1) return 0;
  return (proj_gemm_flags_bytes(M, 1) + 255) & ~static_cast<size_t>(255);
}

int olmo3_out_proj_postnorm_residual(const void *attn, const void *w_o, const float *gain, const void *x, void *h_out,
                                     int M, int D, int K, float eps, void *workspace, size_t ws_bytes, int *err_dev,
                                     void *stream) {
  int st = OLMO3_OK;
  if (M < 0 || D < 1 || K < 1 || !(eps >= 0.f)) return OLMO3_ERR_INVALID_ARG;
  if (K % 64 != 0 || D % 8 != 0 || static_cast<int64_t>(M) * D >= (int64_t(1) << 31)) return OLMO3_ERR_UNSUPPORTED;
  if (M == 0) return OLMO3_OK;
  if (!attn || !w_o || !gain || !x || !h_out) return OLMO3_ERR_INVALID_ARG;
  const void *ptrs[] = {attn, w_o, gain, x, h_out};
  for (const void *p : ptrs)
    if (!aligned16(p)) return OLMO3_ERR_INVALID_ARG;
  const size_t need = olmo3_out_proj_workspace_size(M, D);
  if (workspace == nullptr || ws_bytes < need || !aligned16(workspace)) return OLMO3_ERR_WORKSPACE;
  st = tiles_per_row_status((D + kProjTileN - 1) / kProjTileN);
  if (st != OLMO3_OK) return st;
  CUtensorMap tmA, tmB;
  const cuuint32_t box_a[2] = {64, 128}, box_b[2] = {64, 256};
  const cuuint64_t dims_a[2] = {(cuuint64_t)K, (cuuint64_t)M}, dims_b[2] = {(cuuint64_t)K, (cuuint64_t)D};
  const cuuint64_t stride[1] = {(cuuint64_t)K * 2};
  if (!encode_bf16(&tmA, attn, 2, dims_a, stride, box_a, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_bf16(&tmB, w_o, 2, dims_b, stride, box_b, CU_TENSOR_MAP_SWIZZLE_128B))
    return OLMO3_ERR_CUDA;
  return cuda_status(launch_out_proj(tmA, tmB, gain, x, h_out, M, D, K, eps, workspace, err_dev, as_stream(stream)));
}

size_t olmo3_qkv_proj_workspace_size(int M) {
  if (M < 0) return 0;
  return (proj_gemm_flags_bytes(M, 2) + 255) & ~static_cast<size_t>(255);
}

int olmo3_qkv_proj_qknorm_rope(const void *x, const void *w_qkv, const float *gain_q, const float *gain_k,
                               void *q_out, void *k_out, void *v_out, const int32_t *pos_offset, int B, int T, int H,
                               int G, int d, int D, float eps, double theta, double rope_factor, int original_context,
                               double beta_fast, double beta_slow, void *workspace, size_t ws_bytes, int *err_dev,
                               void *stream) {
  if (B < 0 || T < 0 || H < 1 || G < 1 || D < 1 || !(eps >= 0.f)) return OLMO3_ERR_INVALID_ARG;
  RopeTable tab;
  if (!yarn_table(d, theta, rope_factor, original_context, beta_fast, beta_slow, &tab)) return OLMO3_ERR_INVALID_ARG;
  if (!valid_d(d) || D % 64 != 0 || (H * d) % kProjTileN != 0 || (G * d) % kProjTileN != 0)
    return OLMO3_ERR_UNSUPPORTED;
  const int64_t M = static_cast<int64_t>(B) * T;
  const int64_t N = static_cast<int64_t>(H + 2 * G) * d;
  if (M * (D > N ? D : N) >= (int64_t(1) << 31)) return OLMO3_ERR_UNSUPPORTED;
  if (M == 0) return OLMO3_OK;
  if (!x || !w_qkv || !gain_q || !gain_k || !q_out || !k_out || !v_out || !pos_offset) return OLMO3_ERR_INVALID_ARG;
  const void *ptrs[] = {x, w_qkv, gain_q, gain_k, q_out, k_out, v_out};
  for (const void *p : ptrs)
    if (!aligned16(p)) return OLMO3_ERR_INVALID_ARG;
  const size_t need = olmo3_qkv_proj_workspace_size(static_cast<int>(M));
  if (workspace == nullptr || ws_bytes < need || !aligned16(workspace)) return OLMO3_ERR_WORKSPACE;
  const int st = tiles_per_row_status((H > G ? H : G) * d / kProjTileN);
  if (st != OLMO3_OK) return st;
  CUtensorMap tmX, tmW;
  const cuuint32_t box_x[2] = {64, 128}, box_w[2] = {64, 256};
  const cuuint64_t dims_x[2] = {(cuuint64_t)D, (cuuint64_t)M}, dims_w[2] = {(cuuint64_t)D, (cuuint64_t)N};
  const cuuint64_t stride[1] = {(cuuint64_t)D * 2};
  if (!encode_bf16(&tmX, x, 2, dims_x, stride, box_x, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_bf16(&tmW, w_qkv, 2, dims_w, stride, box_w, CU_TENSOR_MAP_SWIZZLE_128B))
    return OLMO3_ERR_CUDA;
  return cuda_status(launch_qkv_proj(tmX, tmW, q_out, k_out, v_out, gain_q, gain_k, pos_offset, B, T, H, G, d, D, eps,
                                     tab, workspace, err_dev, as_stream(stream)));
}

size_t olmo3_attn_decode_workspace_size(int B, int H, int G, int d, int max_kv_len, int layer_type, int window,
                                        int num_splits) {
  if (B < 0 || H < 1 || G < 1 || !valid_d(d) || H % G != 0 || max_kv_len < 1 || !valid_type(layer_type) ||
      window < 1 || num_splits < 0)
    return 0;
  const int n_max = layer_type == OLMO3_SLIDING ? (max_kv_len < window ? max_kv_len : window) : max_kv_len;
  const DecodePlan pl = plan_decode(B, G, n_max, num_splits, decode_uses_mma(H, G));
  return static_cast<size_t>(B) * H * pl.n_splits * (d + 2) * sizeof(float);
}

int olmo3_attn_decode(const void *q, int H, const olmo3_kv_cache *c, const int32_t *kv_len, int max_kv_len,
                      void *out, float *lse_out, float scale, int num_splits, void *workspace, size_t ws_bytes,
                      int *err_dev, void *stream) {
  int st = validate_cache(c);
  if (st != OLMO3_OK) return st;
  if (H < 1 || max_kv_len < 1 || num_splits < 0 || !isfinite(scale)) return OLMO3_ERR_INVALID_ARG;
  if (H % c->G != 0 || H / c->G > kDecodeMaxGroup) return OLMO3_ERR_UNSUPPORTED;
  if (c->B > 65535) return OLMO3_ERR_UNSUPPORTED;
  if (c->B == 0) return OLMO3_OK;
  if (!q || !kv_len || !out || !aligned16(q) || !aligned16(out)) return OLMO3_ERR_INVALID_ARG;
  const size_t need =
      olmo3_attn_decode_workspace_size(c->B, H, c->G, c->d, max_kv_len, c->layer_type, c->window, num_splits);
  if (workspace == nullptr || ws_bytes < need || !aligned16(workspace)) return OLMO3_ERR_WORKSPACE;
  const int n_max = c->layer_type == OLMO3_SLIDING ? (max_kv_len < c->window ? max_kv_len : c->window) : max_kv_len;
  const DecodePlan pl = plan_decode(c->B, c->G, n_max, num_splits, decode_uses_mma(H, c->G));
  if (pl.n_splits > 65535) return OLMO3_ERR_UNSUPPORTED;
  CUtensorMap tmK, tmV;
  const cuuint64_t dims[3] = {(cuuint64_t)c->d, (cuuint64_t)c->G, (cuuint64_t)c->total_slots};
  const cuuint64_t strides[2] = {(cuuint64_t)c->d * 2, (cuuint64_t)c->G * c->d * 2};
  const bool mma = decode_uses_mma(H, c->G);
  const cuuint32_t box_one[3] = {(cuuint32_t)c->d, 1, (cuuint32_t)kDecodeTile};
  const cuuint32_t box_mma[3] = {64, 1, (cuuint32_t)kDecodeGqaTile};
  const CUtensorMapSwizzle swz = mma ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  if (!encode_bf16(&tmK, c->k, 3, dims, strides, mma ? box_mma : box_one, swz) ||
      !encode_bf16(&tmV, c->v, 3, dims, strides, mma ? box_mma : box_one, swz))
    return OLMO3_ERR_CUDA;
  return cuda_status(launch_attn_decode(tmK, tmV, q, H, *c, kv_len, pl, out, lse_out, scale,
                                        static_cast<float *>(workspace), err_dev, as_stream(stream)));
}

}  // extern "C"
