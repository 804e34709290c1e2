// QK-norm + RoPE, one CTA per token.
//
// "Case Study: OLMo 3", "The architecture", ingredient 2 (QK-norm: RMSNorm of the
// projected queries and keys, one gain per feature of the whole H*d / G*d vector,
// see also "Count OLMo 3's Parameters", "What to count") and ingredient 3 (RoPE,
// theta = 500,000, pair i with i + d/2); "Olmo-3 End-to-End Implementation",
// "Inference Pipeline" (RoPE at position offset + t) and "Technical Details"
// (eps 1e-6; RoPE on queries and keys only).
//
// Memory-bound: q and k are read from HBM once and written once.  Each thread
// owns "pair chunks" (8 features i..i+7 of a head and their rotation partners
// i+d/2..i+d/2+7) and makes two passes over them with 16-byte vector loads: the
// first sums their squares for the block-wide RMS, the second re-reads them (from
// L2) to normalise, rotate and store.  Holding nothing across the reduction keeps
// the kernel at 40 registers, 6 CTAs (tokens) per SM in flight.  64 threads form
// cos/sin once per token: the angle is reduced to [-pi, pi] in fp64, then
// evaluated in fp32.
#include "common.cuh"
#include "internal.h"

namespace olmo3 {

constexpr int kNormThreads = 256;
constexpr int kMaxChunks = 2;  // pair chunks per thread: H*d/16 <= 512

__device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
  const float4 a = *reinterpret_cast<const float4 *>(p);
  const float4 b = *reinterpret_cast<const float4 *>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4 *>(p);
  float2 f;
  f = bf2_to_f2(u.x); x[0] = f.x; x[1] = f.y;
  f = bf2_to_f2(u.y); x[2] = f.x; x[3] = f.y;
  f = bf2_to_f2(u.z); x[4] = f.x; x[5] = f.y;
  f = bf2_to_f2(u.w); x[6] = f.x; x[7] = f.y;
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&x)[8]) {
  uint4 u;
  u.x = f2_to_bf2(x[0], x[1]);
  u.y = f2_to_bf2(x[2], x[3]);
  u.z = f2_to_bf2(x[4], x[5]);
  u.w = f2_to_bf2(x[6], x[7]);
  *reinterpret_cast<uint4 *>(p) = u;
}

__device__ __forceinline__ float block_sum(float v, float *red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int w = threadIdx.x / 32;
  if ((threadIdx.x & 31) == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kNormThreads / 32; ++i) s += red[i];
  return s;
}


// 16-byte load that bypasses L1 and that the compiler may not merge with an
// earlier load of the same address (the second pass re-reads from L2).
__device__ __forceinline__ uint4 ld_cg_u4(const void *p) {
  uint4 u;
  asm volatile("ld.global.cg.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w) : "l"(p));
  return u;
}

// Register copy of one pair chunk: packed bf16 (uint4) or 8 floats.
template <typename Tin> struct Chunk;
template <> struct Chunk<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16 *p) { u = *reinterpret_cast<const uint4 *>(p); }
  __device__ __forceinline__ void reload(const __nv_bfloat16 *p) { u = ld_cg_u4(p); }
  __device__ __forceinline__ void get(float (&x)[8]) const {
    float2 f;
    f = bf2_to_f2(u.x); x[0] = f.x; x[1] = f.y;
    f = bf2_to_f2(u.y); x[2] = f.x; x[3] = f.y;
    f = bf2_to_f2(u.z); x[4] = f.x; x[5] = f.y;
    f = bf2_to_f2(u.w); x[6] = f.x; x[7] = f.y;
  }
};
template <> struct Chunk<float> {
  float4 a, b;
  __device__ __forceinline__ void reload(const float *p) { load(p); }
  __device__ __forceinline__ void load(const float *p) {
    a = reinterpret_cast<const float4 *>(p)[0];
    b = reinterpret_cast<const float4 *>(p)[1];
  }
  __device__ __forceinline__ void get(float (&x)[8]) const {
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

// Sum of squares of this thread's pair chunks of one row, keeping nothing.
template <typename Tin, int D>
__device__ __forceinline__ float row_sumsq(const Tin *row, int n_heads) {
  constexpr int CPH = D / 16;
  float ssq = 0.f;
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c) {
    const int ci = threadIdx.x + c * kNormThreads;
    if (ci < n_heads * CPH) {
      const int h = ci / CPH, i0 = (ci % CPH) * 8;
      Chunk<Tin> lo, hi;
      lo.load(row + h * D + i0);
      hi.load(row + h * D + D / 2 + i0);
      float a[8], b[8];
      lo.get(a);
      hi.get(b);
#pragma unroll
      for (int j = 0; j < 8; ++j) ssq += a[j] * a[j] + b[j] * b[j];
    }
  }
  return ssq;
}

// Second pass: re-read each chunk (from L2), normalise, rotate and store it.
template <typename Tin, int D>
__device__ __forceinline__ void reload_norm_rotate_store(const Tin *in_row, __nv_bfloat16 *row, const float *gain,
                                                         int n_heads, float rinv, const float *s_cos,
                                                         const float *s_sin) {
  constexpr int CPH = D / 16;
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c) {
    const int ci = threadIdx.x + c * kNormThreads;
    if (ci < n_heads * CPH) {
      const int h = ci / CPH, i0 = (ci % CPH) * 8;
      Chunk<Tin> lo, hi;
      lo.reload(in_row + h * D + i0);
      hi.reload(in_row + h * D + D / 2 + i0);
      float glo[8], ghi[8], xlo[8], xhi[8], ylo[8], yhi[8];
      load8(gain + h * D + i0, glo);
      load8(gain + h * D + D / 2 + i0, ghi);
      lo.get(xlo);
      hi.get(xhi);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float a = xlo[j] * rinv * glo[j];
        const float bb = xhi[j] * rinv * ghi[j];
        const float cs = s_cos[i0 + j], sn = s_sin[i0 + j];
        ylo[j] = a * cs - bb * sn;
        yhi[j] = bb * cs + a * sn;
      }
      store8(row + h * D + i0, ylo);
      store8(row + h * D + D / 2 + i0, yhi);
    }
  }
}

// q_out / k_out may alias q / k: each element is read (in both passes) and then
// written by the same thread, and no other thread touches it.
template <typename Tin, int D>
__global__ void __launch_bounds__(kNormThreads, sizeof(Tin) == 2 ? 6 : 1) qknorm_rope_kernel(
    const Tin *q, const Tin *k, const Tin *__restrict__ v, const float *__restrict__ gain_q,
    const float *__restrict__ gain_k, __nv_bfloat16 *q_out, __nv_bfloat16 *k_out, __nv_bfloat16 *__restrict__ v_out,
    const int32_t *__restrict__ pos_offset, int T, int H, int G, float eps, RopeTable tab) {
  __shared__ float s_cos[D / 2], s_sin[D / 2];
  __shared__ float s_red[2][kNormThreads / 32];

  const int64_t tok = blockIdx.x;  // b * T + t
  const int b = static_cast<int>(tok / T);
  const int t = static_cast<int>(tok - static_cast<int64_t>(b) * T);

  const float ssq_q = row_sumsq<Tin, D>(q + tok * H * D, H);
  const float ssq_k = row_sumsq<Tin, D>(k + tok * G * D, G);

  if (threadIdx.x < D / 2) {
    constexpr double kTwoPi = 6.283185307179586476925286766559;
    const double p = static_cast<double>(pos_offset[b]) + static_cast<double>(t);
    const double a = p * tab.inv_freq[threadIdx.x];
    float sn, cs;
    sincosf(static_cast<float>(fma(-rint(a * (1.0 / kTwoPi)), kTwoPi, a)), &sn, &cs);
    s_cos[threadIdx.x] = cs * tab.out_scale;
    s_sin[threadIdx.x] = sn * tab.out_scale;
  }
  const float tq = block_sum(ssq_q, s_red[0]);
  const float tk = block_sum(ssq_k, s_red[1]);  // its __syncthreads also publishes s_cos / s_sin
  const float rq = 1.0f / sqrtf(tq / static_cast<float>(H * D) + eps);
  const float rk = 1.0f / sqrtf(tk / static_cast<float>(G * D) + eps);

  reload_norm_rotate_store<Tin, D>(q + tok * H * D, q_out + tok * H * D, gain_q, H, rq, s_cos, s_sin);
  reload_norm_rotate_store<Tin, D>(k + tok * G * D, k_out + tok * G * D, gain_k, G, rk, s_cos, s_sin);

  if (v_out != nullptr) {
    const Tin *vr = v + tok * G * D;
    __nv_bfloat16 *vo = v_out + tok * G * D;
    for (int e = threadIdx.x * 8; e < G * D; e += kNormThreads * 8) {
      float x[8];
      load8(vr + e, x);
      store8(vo + e, x);
    }
  }
}

template <typename Tin, int D>
static cudaError_t launch_typed(const void *q, const void *k, const void *v, const float *gq, const float *gk,
                                void *qo, void *ko, void *vo, const int32_t *pos, int B, int T, int H, int G,
                                float eps, const RopeTable &tab, cudaStream_t st) {
  const int64_t ntok = static_cast<int64_t>(B) * T;
  qknorm_rope_kernel<Tin, D><<<static_cast<unsigned>(ntok), kNormThreads, 0, st>>>(
      static_cast<const Tin *>(q), static_cast<const Tin *>(k), static_cast<const Tin *>(v), gq, gk,
      static_cast<__nv_bfloat16 *>(qo), static_cast<__nv_bfloat16 *>(ko), static_cast<__nv_bfloat16 *>(vo), pos, T,
      H, G, eps, tab);
  return cudaGetLastError();
}

cudaError_t launch_qknorm_rope(const void *q, const void *k, const void *v, int in_dtype, const float *gain_q,
                               const float *gain_k, void *q_out, void *k_out, void *v_out,
                               const int32_t *pos_offset, int B, int T, int H, int G, int d, float eps,
                               const RopeTable &tab, cudaStream_t stream) {
  if (in_dtype == OLMO3_F32) {
    if (d == 64)
      return launch_typed<float, 64>(q, k, v, gain_q, gain_k, q_out, k_out, v_out, pos_offset, B, T, H, G, eps, tab,
                                     stream);
    return launch_typed<float, 128>(q, k, v, gain_q, gain_k, q_out, k_out, v_out, pos_offset, B, T, H, G, eps, tab,
                                    stream);
  }
  if (d == 64)
    return launch_typed<__nv_bfloat16, 64>(q, k, v, gain_q, gain_k, q_out, k_out, v_out, pos_offset, B, T, H, G, eps,
                                           tab, stream);
  return launch_typed<__nv_bfloat16, 128>(q, k, v, gain_q, gain_k, q_out, k_out, v_out, pos_offset, B, T, H, G, eps,
                                          tab, stream);
}

}  // namespace olmo3
