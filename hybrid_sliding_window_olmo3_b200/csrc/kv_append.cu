// KV-cache append into a preallocated per-layer-type cache, and the mask export.
//
// "Olmo 3 7B" (inference-research record), serviceability join: a windowed
// decode kernel needs per-layer-type cache management; a sliding layer holds at
// most `window` tokens.  "Olmo-3 End-to-End Implementation", "KV Cache
// Implementation" grows the cache by concatenation; here it is a ring of exactly
// `window` slots (sliding layers, position p in slot p mod window) or a linear
// buffer (full layers, position p in slot p), written in place.
//
// One CTA per new row: 16-byte vector copies of the G*d keys and values.  Rows a
// later token of the same call would overwrite are skipped, so no two CTAs of a
// call write the same slot.
#include "common.cuh"
#include "internal.h"

namespace olmo3 {

constexpr int kAppendThreads = 128;

__global__ void __launch_bounds__(kAppendThreads) kv_append_kernel(
    uint4 *__restrict__ ck, uint4 *__restrict__ cv, const int64_t *__restrict__ seq_base, int64_t total_slots,
    int capacity, int layer_type, int window, int row_vec, const uint4 *__restrict__ k_new,
    const uint4 *__restrict__ v_new, const int32_t *__restrict__ pos_offset, int T, int32_t *__restrict__ slot_out,
    int *err) {
  const int t = blockIdx.x, b = blockIdx.y;
  const int64_t p = static_cast<int64_t>(pos_offset[b]) + t;
  bool write = true;
  int64_t slot = -1;
  if (p < 0) {
    write = false;
    if (threadIdx.x == 0) set_dev_error(err, OLMO3_DEVERR_CAPACITY);
  } else if (layer_type == OLMO3_SLIDING) {
    slot = p % window;
    write = t >= T - window;  // a later row of this call lands on the same slot otherwise
  } else {
    slot = p;
  }
  int64_t row = -1;
  if (write) {
    row = seq_base[b] + slot;
    if (slot >= capacity || row < 0 || row >= total_slots) {
      write = false;
      if (threadIdx.x == 0) set_dev_error(err, OLMO3_DEVERR_CAPACITY);
    }
  }
  if (slot_out != nullptr && threadIdx.x == 0)
    slot_out[static_cast<int64_t>(b) * T + t] = write ? static_cast<int32_t>(slot) : -1;
  if (!write) return;
  const int64_t src = (static_cast<int64_t>(b) * T + t) * row_vec;
  const int64_t dst = row * row_vec;
  for (int i = threadIdx.x; i < row_vec; i += kAppendThreads) {
    ck[dst + i] = k_new[src + i];
    cv[dst + i] = v_new[src + i];
  }
}

cudaError_t launch_kv_append(const olmo3_kv_cache &c, const void *k_new, const void *v_new,
                             const int32_t *pos_offset, int T, int32_t *slot_out, int *err, cudaStream_t stream) {
  const int row_vec = c.G * c.d * 2 / 16;  // 16-byte vectors per row
  dim3 grid(T, c.B);
  kv_append_kernel<<<grid, kAppendThreads, 0, stream>>>(
      static_cast<uint4 *>(c.k), static_cast<uint4 *>(c.v), c.seq_base, c.total_slots, c.capacity, c.layer_type,
      c.window, row_vec, static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), pos_offset, T,
      slot_out, err);
  return cudaGetLastError();
}

// Window gather for a prompt chunk at an offset on a sliding layer ("Olmo-3
// End-to-End Implementation", "Inference Pipeline": RoPE with position offsets for
// cache compatibility).  Before the chunk is appended, the ring still holds the
// window of positions [p0 - window + 1, p0); the chunk's rows need those keys and
// the chunk itself, in position order, so they are copied side by side into one
// [Tk, G, d] block per sequence.  Rows past the chunk are zeroed so that a partly
// used key tile never multiplies uninitialised values.
__global__ void __launch_bounds__(kAppendThreads) gather_window_kernel(
    const uint4 *__restrict__ ck, const uint4 *__restrict__ cv, const int64_t *__restrict__ seq_base,
    int64_t total_slots, int window, int row_vec, const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
    const int32_t *__restrict__ pos_offset, int T, int Tk, uint4 *__restrict__ k_out, uint4 *__restrict__ v_out) {
  const int j = blockIdx.x, b = blockIdx.y;
  const int p0 = pos_offset[b];
  const int kp0 = max(0, p0 - window + 1);
  const int p = kp0 + j;  // absolute position of this row
  const uint4 *sk = nullptr, *sv = nullptr;
  if (p < p0) {
    const int64_t row = seq_base[b] + (p % window);
    if (row >= 0 && row < total_slots) {
      sk = ck + row * row_vec;
      sv = cv + row * row_vec;
    }
  } else if (p < p0 + T) {
    const int64_t row = static_cast<int64_t>(b) * T + (p - p0);
    sk = k_new + row * row_vec;
    sv = v_new + row * row_vec;
  }
  uint4 *dk = k_out + (static_cast<int64_t>(b) * Tk + j) * row_vec;
  uint4 *dv = v_out + (static_cast<int64_t>(b) * Tk + j) * row_vec;
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (int i = threadIdx.x; i < row_vec; i += kAppendThreads) {
    dk[i] = sk ? sk[i] : z;
    dv[i] = sv ? sv[i] : z;
  }
}

cudaError_t launch_gather_window(const olmo3_kv_cache &c, const void *k_new, const void *v_new,
                                 const int32_t *pos_offset, int T, int Tk, void *k_out, void *v_out,
                                 cudaStream_t stream) {
  const int row_vec = c.G * c.d * 2 / 16;
  gather_window_kernel<<<dim3(Tk, c.B), kAppendThreads, 0, stream>>>(
      static_cast<const uint4 *>(c.k), static_cast<const uint4 *>(c.v), c.seq_base, c.total_slots, c.window,
      row_vec, static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), pos_offset, T, Tk,
      static_cast<uint4 *>(k_out), static_cast<uint4 *>(v_out));
  return cudaGetLastError();
}

// The one key tile of a sliding-layer chunk that straddles the chunk's start: the
// 128 positions from 128 * floor(p0 / 128), taken from the ring below p0 and from
// the chunk from p0 on (zeros past the chunk).  Every other key tile is read in
// place, from the ring or from the chunk (attn_prefill.cu, kPrefillRing).
__global__ void __launch_bounds__(kAppendThreads) bridge_tile_kernel(
    const uint4 *__restrict__ ck, const uint4 *__restrict__ cv, const int64_t *__restrict__ seq_base,
    int64_t total_slots, int window, int row_vec, const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
    const int32_t *__restrict__ pos_offset, int T, uint4 *__restrict__ k_out, uint4 *__restrict__ v_out) {
  const int j = blockIdx.x, b = blockIdx.y;
  const int p0 = pos_offset[b];
  const int p = (p0 >= 0 ? p0 / kPrefillBN : 0) * kPrefillBN + j;  // absolute position of this row
  const uint4 *sk = nullptr, *sv = nullptr;
  if (p < p0) {
    const int64_t row = seq_base[b] + (p % window);
    if (row >= 0 && row < total_slots) {
      sk = ck + row * row_vec;
      sv = cv + row * row_vec;
    }
  } else if (p0 >= 0 && p < p0 + T) {
    const int64_t row = static_cast<int64_t>(b) * T + (p - p0);
    sk = k_new + row * row_vec;
    sv = v_new + row * row_vec;
  }
  uint4 *dk = k_out + (static_cast<int64_t>(b) * kPrefillBN + j) * row_vec;
  uint4 *dv = v_out + (static_cast<int64_t>(b) * kPrefillBN + j) * row_vec;
  const uint4 z = make_uint4(0, 0, 0, 0);
  for (int i = threadIdx.x; i < row_vec; i += kAppendThreads) {
    dk[i] = sk ? sk[i] : z;
    dv[i] = sv ? sv[i] : z;
  }
}

cudaError_t launch_bridge_tile(const olmo3_kv_cache &c, const void *k_new, const void *v_new,
                               const int32_t *pos_offset, int T, void *k_out, void *v_out, cudaStream_t stream) {
  const int row_vec = c.G * c.d * 2 / 16;
  bridge_tile_kernel<<<dim3(kPrefillBN, c.B), kAppendThreads, 0, stream>>>(
      static_cast<const uint4 *>(c.k), static_cast<const uint4 *>(c.v), c.seq_base, c.total_slots, c.window,
      row_vec, static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), pos_offset, T,
      static_cast<uint4 *>(k_out), static_cast<uint4 *>(v_out));
  return cudaGetLastError();
}

// "OLMo 3's Sliding-Window Attention Pattern", "The sliding-window mask": the
// same predicate the attention kernels apply, written out as bytes.
__global__ void attn_mask_kernel(int T, int window, int layer_type, uint8_t *__restrict__ out) {
  const int64_t n = static_cast<int64_t>(T) * T;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / T, s = i - t * T;
    const bool ok = s <= t && (layer_type == OLMO3_FULL || t - s < window);
    out[i] = ok ? 1 : 0;
  }
}

cudaError_t launch_attn_mask(int T, int window, int layer_type, uint8_t *out, cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(T) * T;
  const int threads = 256;
  const int64_t blocks = (n + threads - 1) / threads;
  attn_mask_kernel<<<static_cast<unsigned>(blocks < 148 * 16 ? blocks : 148 * 16), threads, 0, stream>>>(
      T, window, layer_type, out);
  return cudaGetLastError();
}

}  // namespace olmo3
