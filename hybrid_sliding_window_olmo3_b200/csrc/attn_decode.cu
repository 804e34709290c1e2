// Split-KV decode attention over the per-layer-type cache, plus the combine.
//
// "Olmo 3 7B" (inference-research record), serviceability join: a local layer's
// decode reads exactly `window` cache entries (about 1 flop per byte, constant in
// context) while a full layer's reads grow with the context; one kernel serves
// both.  "Olmo-3 End-to-End Implementation", "Inference Pipeline": one new token
// per step attends over the cache.  GQA ("Case Study: OLMo 3", ingredient 1):
// query head h reads key/value head h / (H/G), so one CTA serves the R = H/G
// query heads of a key/value head and reads each cache row once for all of them.
//
// HBM-bound design: grid = (kv head g, split, sequence b) with g fastest, so
// neighbouring CTAs stream neighbouring rows of the [slots, G, d] cache.  A
// producer warp feeds 32-key tiles of K and V through a 4-stage TMA/mbarrier
// ring; 4 compute warps run the dot products with 16-byte shared loads, reduce
// them with warp shuffles (d/8 lanes per key) and keep an online softmax per lane
// group in fp32.  Each CTA writes one (max, sum, unnormalised output) partial
// per query head; the combine kernel merges the partials with log-sum-exp
// weights.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace olmo3 {

constexpr int kDecStages = 4;
constexpr int kDecWarps = 4;  // compute warps; one more warp produces
constexpr int kDecThreads = (kDecWarps + 1) * 32;

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D, int R>
struct DecodeSmem {
  static constexpr int kTileBytes = kDecodeTile * D * 2;          // one K (or V) tile
  static constexpr int kPipeBytes = kDecStages * 2 * kTileBytes;  // K and V rings
  static constexpr int kGroups = kDecWarps * (32 / (D / 8));      // lane groups per CTA
  static constexpr int kMergeBytes = kGroups * R * (D + 2) * 4;
  static constexpr int kBytes = kPipeBytes > kMergeBytes ? kPipeBytes : kMergeBytes;
};

__device__ __forceinline__ int valid_keys(int L, int layer_type, int window) {
  return layer_type == OLMO3_SLIDING ? min(L, window) : L;
}

template <int D, int R>
__global__ void __launch_bounds__(kDecThreads) attn_decode_split_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __nv_bfloat16 *__restrict__ q, const int64_t *__restrict__ seq_base, const int32_t *__restrict__ kv_len,
    int capacity, int layer_type, int window, int H, int chunk, int n_splits, float scale_log2,
    float *__restrict__ ws_o, float *__restrict__ ws_ml, int *err) {
  using S = DecodeSmem<D, R>;
  constexpr int LPK = D / 8;                        // lanes per key (8 features each)
  constexpr int KPW = 32 / LPK;                     // keys per warp pass
  constexpr int KEYS_PER_WARP = kDecodeTile / kDecWarps;
  constexpr int NIT = KEYS_PER_WARP / KPW;

  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t full_bar[kDecStages], empty_bar[kDecStages];
  __shared__ int s_abort;

  const int g = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int L = kv_len[b];
  const int n = valid_keys(L, layer_type, window);
  if (L < 1 || n > capacity || n > n_splits * chunk) {
    if (split == 0 && g == 0 && threadIdx.x == 0) set_dev_error(err, OLMO3_DEVERR_KV_LEN);
    return;  // the combine writes zeros for this sequence
  }
  const int k_begin = split * chunk;
  if (k_begin >= n) return;
  const int k_end = min(n, k_begin + chunk);
  const int ntiles = (k_end - k_begin + kDecodeTile - 1) / kDecodeTile;
  const int64_t base = seq_base[b];

  __nv_bfloat16 *sK = reinterpret_cast<__nv_bfloat16 *>(smem);
  __nv_bfloat16 *sV = sK + kDecStages * kDecodeTile * D;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kDecStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kDecWarps);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int lg = lane / LPK;  // lane group (key) inside the warp
  const int li = lane % LPK;  // features li*8 .. li*8+7
  float m[R], l[R], o[R][8];
  bool ok = true;

  if (warp == kDecWarps) {
    // ---------------- producer: one elected lane issues TMA ----------------
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % kDecStages;
        if (i >= kDecStages && !mbar_wait(&empty_bar[st], ((i / kDecStages) & 1) ^ 1, &s_abort)) {
          ok = false;
          break;
        }
        const int row = static_cast<int>(base + k_begin + i * kDecodeTile);
        mbar_arrive_expect_tx(&full_bar[st], 2 * S::kTileBytes);
        tma_load_3d(sK + st * kDecodeTile * D, &tmK, &full_bar[st], 0, g, row);
        tma_load_3d(sV + st * kDecodeTile * D, &tmV, &full_bar[st], 0, g, row);
        ++issued;
      }
      if (!ok) {
        s_abort = 1;
        set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
        // let the copies still in flight land before the CTA's shared memory goes away
        for (int j = max(0, issued - kDecStages); j < issued; ++j)
          mbar_wait(&full_bar[j % kDecStages], (j / kDecStages) & 1, nullptr);
      }
    }
  } else {
    // ---------------- compute warps ----------------
    float qf[R][8];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const uint4 u = *reinterpret_cast<const uint4 *>(q + (static_cast<int64_t>(b) * H + g * R + r) * D + li * 8);
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = bf2_to_f2(w4[j]);
        qf[r][2 * j] = f.x * scale_log2;
        qf[r][2 * j + 1] = f.y * scale_log2;
      }
      m[r] = -INFINITY;
      l[r] = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) o[r][j] = 0.f;
    }

    for (int i = 0; i < ntiles; ++i) {
      const int st = i % kDecStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[st], (i / kDecStages) & 1, &s_abort))) {
        ok = false;
        break;
      }
      const __nv_bfloat16 *kt = sK + st * kDecodeTile * D;
      const __nv_bfloat16 *vt = sV + st * kDecodeTile * D;
      const int key_base = k_begin + i * kDecodeTile;

      float s[R][NIT];
#pragma unroll
      for (int it = 0; it < NIT; ++it) {
        const int kk = warp * KEYS_PER_WARP + it * KPW + lg;
        const uint4 u = *reinterpret_cast<const uint4 *>(kt + kk * D + li * 8);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
        float kf[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = bf2_to_f2(w4[j]);
          kf[2 * j] = f.x;
          kf[2 * j + 1] = f.y;
        }
#pragma unroll
        for (int r = 0; r < R; ++r) {
          float a = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) a = fmaf(qf[r][j], kf[j], a);
          s[r][it] = a;
        }
      }
#pragma unroll
      for (int off = LPK / 2; off > 0; off >>= 1) {
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int it = 0; it < NIT; ++it) s[r][it] += __shfl_xor_sync(0xffffffffu, s[r][it], off);
      }
      float p[R][NIT];
#pragma unroll
      for (int r = 0; r < R; ++r) {
        float mt = -INFINITY;
#pragma unroll
        for (int it = 0; it < NIT; ++it) {
          const int key = key_base + warp * KEYS_PER_WARP + it * KPW + lg;
          if (key >= k_end) s[r][it] = -INFINITY;
          mt = fmaxf(mt, s[r][it]);
        }
        const float mn = fmaxf(m[r], mt);
        if (mn == -INFINITY) {  // nothing valid seen yet by this lane group
#pragma unroll
          for (int it = 0; it < NIT; ++it) p[r][it] = 0.f;
          continue;
        }
        const float alpha = fast_exp2(m[r] - mn);
        float rs = 0.f;
#pragma unroll
        for (int it = 0; it < NIT; ++it) {
          p[r][it] = fast_exp2(s[r][it] - mn);
          rs += p[r][it];
        }
        l[r] = l[r] * alpha + rs;
        m[r] = mn;
#pragma unroll
        for (int j = 0; j < 8; ++j) o[r][j] *= alpha;
      }
#pragma unroll
      for (int it = 0; it < NIT; ++it) {
        const int kk = warp * KEYS_PER_WARP + it * KPW + lg;
        const bool valid = key_base + kk < k_end;  // a partly used tile may hold uninitialised rows
        const uint4 u = *reinterpret_cast<const uint4 *>(vt + kk * D + li * 8);
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
        float vf[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = bf2_to_f2(w4[j]);
          vf[2 * j] = valid ? f.x : 0.f;
          vf[2 * j + 1] = valid ? f.y : 0.f;
        }
#pragma unroll
        for (int r = 0; r < R; ++r)
#pragma unroll
          for (int j = 0; j < 8; ++j) o[r][j] = fmaf(p[r][it], vf[j], o[r][j]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
    }
    if (!ok && lane == 0) {
      s_abort = 1;
      set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
    }
  }
  __syncthreads();  // every tile consumed (or drained): the rings can be reused
  if (s_abort) return;

  // ---------------- merge the lane groups' partials ----------------
  float *sm_m = reinterpret_cast<float *>(smem);
  float *sm_l = sm_m + S::kGroups * R;
  float *sm_o = sm_l + S::kGroups * R;
  if (warp < kDecWarps) {
    const int grp = warp * KPW + lg;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (li == 0) {
        sm_m[grp * R + r] = m[r];
        sm_l[grp * R + r] = l[r];
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) sm_o[(grp * R + r) * D + li * 8 + j] = o[r][j];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < R * D; idx += kDecThreads) {
    const int r = idx / D, dim = idx % D;
    float M = -INFINITY;
    for (int gi = 0; gi < S::kGroups; ++gi) M = fmaxf(M, sm_m[gi * R + r]);
    float acc = 0.f, den = 0.f;
    for (int gi = 0; gi < S::kGroups; ++gi) {
      const float mg = sm_m[gi * R + r];
      const float w = (mg == -INFINITY) ? 0.f : fast_exp2(mg - M);
      acc += w * sm_o[(gi * R + r) * D + dim];
      den += w * sm_l[gi * R + r];
    }
    const int64_t slot = (static_cast<int64_t>(b) * H + g * R + r) * n_splits + split;
    ws_o[slot * D + dim] = acc;
    if (dim == 0) {
      ws_ml[slot * 2] = M;
      ws_ml[slot * 2 + 1] = den;
    }
  }
}

// Merges the split partials of one (sequence, query head): out = sum_s w_s o_s /
// sum_s w_s l_s with w_s = 2^(m_s - max m).  Writes zeros for a sequence whose
// kv_len was rejected.
template <int D>
__global__ void __launch_bounds__(D) attn_decode_combine_kernel(const int32_t *__restrict__ kv_len, int capacity,
                                                                 int layer_type, int window, int H, int chunk,
                                                                 int n_splits, const float *__restrict__ ws_o,
                                                                 const float *__restrict__ ws_ml,
                                                                 __nv_bfloat16 *__restrict__ out,
                                                                 float *__restrict__ lse_out) {
  const int h = blockIdx.x, b = blockIdx.y, dim = threadIdx.x;
  const int L = kv_len[b];
  const int n = valid_keys(L, layer_type, window);
  const int64_t bh = static_cast<int64_t>(b) * H + h;
  if (L < 1 || n > capacity || n > n_splits * chunk) {
    out[bh * D + dim] = __float2bfloat16_rn(0.f);
    if (lse_out != nullptr && dim == 0) lse_out[bh] = -INFINITY;
    return;
  }
  const int ns = (n + chunk - 1) / chunk;
  const float *ml = ws_ml + bh * n_splits * 2;
  const float *po = ws_o + bh * n_splits * D;
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, ml[2 * s]);
  float acc = 0.f, den = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float w = fast_exp2(ml[2 * s] - M);
    acc += w * po[static_cast<int64_t>(s) * D + dim];
    den += w * ml[2 * s + 1];
  }
  out[bh * D + dim] = __float2bfloat16_rn(den > 0.f ? acc / den : 0.f);
  if (lse_out != nullptr && dim == 0) lse_out[bh] = (M + log2f(den)) * 0.69314718055994531f;
}

// ---------------------------------------------------------------------------
// Grouped-query decode (H/G = R > 1, e.g. the 32B's 5 query heads per key/value
// head): the R query rows of a key/value head form the M dimension of warp-level
// tensor-core products (mma.sync m16n8k16, bf16 in, fp32 accumulate; rows R..15
// are zero padding), so each cache row is read once for all R heads and the dot
// products cost 2 MMA instructions per key instead of R reductions on CUDA cores.
// A producer warp streams 64-key K and V tiles (128-byte swizzle, two 64-feature
// column blocks each) through a 3-stage TMA ring; each of 4 compute warps owns 16
// keys of a tile: S = Q K^T (ldmatrix of K), online softmax on the S fragments in
// fp32, and O += P V with P taken straight from the S fragments and V read with
// ldmatrix.trans.  The partials use the same workspace layout and combine as the
// one-head kernel.
// ---------------------------------------------------------------------------
#ifndef OLMO3_GQA_STAGES
#define OLMO3_GQA_STAGES 3
#endif
constexpr int kGqaStages = OLMO3_GQA_STAGES;
constexpr int kGqaWarps = 4;  // compute warps; one more warp produces
constexpr int kGqaThreads = (kGqaWarps + 1) * 32;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// c (16x8 f32) += a (16x16 bf16, row-major) * b (16x8 bf16, column-major)
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
struct GqaSmem {
  static constexpr int kTileBytes = kDecodeGqaTile * D * 2;  // one K or V tile
  static constexpr int kPipeBytes = kGqaStages * 2 * kTileBytes;
  static constexpr int kMergeBytes = kGqaWarps * 16 * (D + 2) * 4;
  static constexpr int kBytes = (kPipeBytes > kMergeBytes ? kPipeBytes : kMergeBytes) + 1024;
};

// byte offset of feature `dim` of key row `key` inside a 128-byte-swizzled tile
// stored as D/64 column blocks of 64 keys x 128 bytes
__device__ __forceinline__ uint32_t sw_off(int key, int dim) {
  const int chunk = (dim & 63) >> 3;
  return static_cast<uint32_t>((dim >> 6) * (kDecodeGqaTile * 128) + key * 128 + ((chunk ^ (key & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kGqaThreads) attn_decode_gqa_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const __nv_bfloat16 *__restrict__ q, const int64_t *__restrict__ seq_base, const int32_t *__restrict__ kv_len,
    int capacity, int layer_type, int window, int H, int R, int chunk, int n_splits, float scale_log2,
    float *__restrict__ ws_o, float *__restrict__ ws_ml, int *err) {
  using S = GqaSmem<D>;
  constexpr int NDB = D / 64;
  constexpr int KB = D / 16;  // k-blocks of Q K^T
  constexpr int NB = D / 8;   // n-blocks of P V

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[kGqaStages], empty_bar[kGqaStages];
  __shared__ int s_abort;
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sK = smem;
  uint8_t *sV = smem + kGqaStages * S::kTileBytes;

  const int g = blockIdx.x, split = blockIdx.y, b = blockIdx.z;
  const int L = kv_len[b];
  const int n = valid_keys(L, layer_type, window);
  if (L < 1 || n > capacity || n > n_splits * chunk) {
    if (split == 0 && g == 0 && threadIdx.x == 0) set_dev_error(err, OLMO3_DEVERR_KV_LEN);
    return;
  }
  const int k_begin = split * chunk;
  if (k_begin >= n) return;
  const int k_end = min(n, k_begin + chunk);
  const int ntiles = (k_end - k_begin + kDecodeGqaTile - 1) / kDecodeGqaTile;
  const int64_t base = seq_base[b];

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kGqaStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], kGqaWarps);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const int gr = lane >> 2;        // fragment row (query head) gr and gr + 8
  const int tq = (lane & 3) * 2;   // fragment column pair
  float o[NB][4];
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
  bool ok = true;

  if (warp == kGqaWarps) {
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      int issued = 0;
      for (int i = 0; i < ntiles; ++i) {
        const int st = i % kGqaStages;
        if (i >= kGqaStages && !mbar_wait(&empty_bar[st], ((i / kGqaStages) & 1) ^ 1, &s_abort)) {
          ok = false;
          break;
        }
        const int row = static_cast<int>(base + k_begin + i * kDecodeGqaTile);
        mbar_arrive_expect_tx(&full_bar[st], 2 * S::kTileBytes);
#pragma unroll
        for (int db = 0; db < NDB; ++db) {
          tma_load_3d(sK + st * S::kTileBytes + db * (kDecodeGqaTile * 128), &tmK, &full_bar[st], db * 64, g, row);
          tma_load_3d(sV + st * S::kTileBytes + db * (kDecodeGqaTile * 128), &tmV, &full_bar[st], db * 64, g, row);
        }
        ++issued;
      }
      if (!ok) {
        s_abort = 1;
        set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
        for (int j = max(0, issued - kGqaStages); j < issued; ++j)
          mbar_wait(&full_bar[j % kGqaStages], (j / kGqaStages) & 1, nullptr);
      }
    }
  } else {
    // Q fragments of the R query heads of this key/value head (rows >= R are zero)
    uint32_t qa[KB][4];
    {
      const __nv_bfloat16 *q_lo = q + (static_cast<int64_t>(b) * H + g * R + gr) * D;
      const __nv_bfloat16 *q_hi = q_lo + 8 * D;
      const bool v_lo = gr < R, v_hi = gr + 8 < R;
#pragma unroll
      for (int kb = 0; kb < KB; ++kb) {
        qa[kb][0] = v_lo ? *reinterpret_cast<const uint32_t *>(q_lo + kb * 16 + tq) : 0u;
        qa[kb][1] = v_hi ? *reinterpret_cast<const uint32_t *>(q_hi + kb * 16 + tq) : 0u;
        qa[kb][2] = v_lo ? *reinterpret_cast<const uint32_t *>(q_lo + kb * 16 + 8 + tq) : 0u;
        qa[kb][3] = v_hi ? *reinterpret_cast<const uint32_t *>(q_hi + kb * 16 + 8 + tq) : 0u;
      }
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) o[nb][0] = o[nb][1] = o[nb][2] = o[nb][3] = 0.f;

    for (int i = 0; i < ntiles; ++i) {
      const int st = i % kGqaStages;
      if (!__all_sync(0xffffffffu, mbar_wait(&full_bar[st], (i / kGqaStages) & 1, &s_abort))) {
        ok = false;
        break;
      }
      const uint32_t kbase = smem_u32(sK + st * S::kTileBytes);
      const uint32_t vbase = smem_u32(sV + st * S::kTileBytes);
      // S = Q K^T for this warp's 16 keys (two 8-key n-blocks)
      float sc[2][4];
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        sc[nb][0] = sc[nb][1] = sc[nb][2] = sc[nb][3] = 0.f;
        const int key = warp * 16 + nb * 8 + (lane & 7);
#pragma unroll
        for (int kb2 = 0; kb2 < KB / 2; ++kb2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kbase + sw_off(key, kb2 * 32 + (lane >> 3) * 8), b0, b1, b2, b3);
          mma_16816(sc[nb], qa[2 * kb2], b0, b1);
          mma_16816(sc[nb], qa[2 * kb2 + 1], b2, b3);
        }
      }
      // scores in log2 units, keys past the end masked
      const int key0 = k_begin + i * kDecodeGqaTile + warp * 16 + tq;
#pragma unroll
      for (int nb = 0; nb < 2; ++nb)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = key0 + nb * 8 + (e & 1);
          sc[nb][e] = key < k_end ? sc[nb][e] * scale_log2 : -INFINITY;
        }
      float mx_lo = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
      float mx_hi = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
      mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
      mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
      const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
      // rows that have seen no valid key keep weight 0 (and alpha 1)
      const float ref_lo = mn_lo == -INFINITY ? 0.f : mn_lo, ref_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
      const float a_lo = fast_exp2(m_lo - ref_lo), a_hi = fast_exp2(m_hi - ref_hi);
      m_lo = mn_lo;
      m_hi = mn_hi;
      float p[2][4];
#pragma unroll
      for (int nb = 0; nb < 2; ++nb) {
        p[nb][0] = fast_exp2(sc[nb][0] - ref_lo);
        p[nb][1] = fast_exp2(sc[nb][1] - ref_lo);
        p[nb][2] = fast_exp2(sc[nb][2] - ref_hi);
        p[nb][3] = fast_exp2(sc[nb][3] - ref_hi);
      }
      l_lo = l_lo * a_lo + ((p[0][0] + p[0][1]) + (p[1][0] + p[1][1]));
      l_hi = l_hi * a_hi + ((p[0][2] + p[0][3]) + (p[1][2] + p[1][3]));
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        o[nb][0] *= a_lo;
        o[nb][1] *= a_lo;
        o[nb][2] *= a_hi;
        o[nb][3] *= a_hi;
      }
      // V rows past the last key of a partly used tile may be uninitialised cache
      // slots: zero this warp's share of them (P is 0 there, but 0 x NaN is not 0)
      const int tile_key0 = k_begin + i * kDecodeGqaTile;
      if (tile_key0 + kDecodeGqaTile > k_end) {
        uint8_t *vt = sV + st * S::kTileBytes;
        for (int e = lane; e < 16 * NDB * 8; e += 32) {
          const int r = e / (NDB * 8), db = (e / 8) % NDB, c = e % 8;
          const int key = warp * 16 + r;
          if (tile_key0 + key >= k_end)
            *reinterpret_cast<uint4 *>(vt + db * (kDecodeGqaTile * 128) + key * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        }
        __syncwarp();
      }
      // P (16 rows x 16 keys) as the A operand, straight from the S fragments
      const uint32_t pa[4] = {f2_to_bf2(p[0][0], p[0][1]), f2_to_bf2(p[0][2], p[0][3]), f2_to_bf2(p[1][0], p[1][1]),
                              f2_to_bf2(p[1][2], p[1][3])};
      // O += P V: V rows are keys (warp*16 .. +15), read transposed
      const int mi = lane >> 3;
      const int vkey = warp * 16 + (lane & 7) + ((mi & 1) << 3);
#pragma unroll
      for (int nb2 = 0; nb2 < NB / 2; ++nb2) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbase + sw_off(vkey, nb2 * 16 + ((mi >> 1) << 3)), b0, b1, b2, b3);
        mma_16816(o[2 * nb2], pa, b0, b1);
        mma_16816(o[2 * nb2 + 1], pa, b2, b3);
      }
      if (tile_key0 + kDecodeGqaTile > k_end) fence_proxy_async_smem();  // before TMA refills what we zeroed
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty_bar[st]);
    }
    if (!ok && lane == 0) {
      s_abort = 1;
      set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
    }
    // complete the row sums over the quad
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
  }
  __syncthreads();
  if (s_abort) return;

  // merge the 4 warps' partials (rows < R) and write this split's (max, sum, output)
  float *sm_m = reinterpret_cast<float *>(smem);
  float *sm_l = sm_m + kGqaWarps * 16;
  float *sm_o = sm_l + kGqaWarps * 16;
  if (warp < kGqaWarps) {
    if ((lane & 3) == 0) {
      sm_m[warp * 16 + gr] = m_lo;
      sm_m[warp * 16 + gr + 8] = m_hi;
      sm_l[warp * 16 + gr] = l_lo;
      sm_l[warp * 16 + gr + 8] = l_hi;
    }
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      sm_o[(warp * 16 + gr) * D + nb * 8 + tq] = o[nb][0];
      sm_o[(warp * 16 + gr) * D + nb * 8 + tq + 1] = o[nb][1];
      sm_o[(warp * 16 + gr + 8) * D + nb * 8 + tq] = o[nb][2];
      sm_o[(warp * 16 + gr + 8) * D + nb * 8 + tq + 1] = o[nb][3];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < R * D; idx += kGqaThreads) {
    const int r = idx / D, dim = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kGqaWarps; ++w) M = fmaxf(M, sm_m[w * 16 + r]);
    float acc = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < kGqaWarps; ++w) {
      const float mw = sm_m[w * 16 + r];
      const float wt = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
      acc += wt * sm_o[(w * 16 + r) * D + dim];
      den += wt * sm_l[w * 16 + r];
    }
    const int64_t slot = (static_cast<int64_t>(b) * H + g * R + r) * n_splits + split;
    ws_o[slot * D + dim] = acc;
    if (dim == 0) {
      ws_ml[slot * 2] = M;
      ws_ml[slot * 2 + 1] = den;
    }
  }
}

DecodePlan plan_decode(int B, int G, int n_max, int num_splits, bool mma) {
  DecodePlan pl;
  const int64_t grains = (static_cast<int64_t>(n_max) + kDecodeGrain - 1) / kDecodeGrain;
  int64_t splits;
  if (num_splits > 0) {
    splits = num_splits;
  } else {
    // Enough CTAs for several waves of the resident CTAs (3 per SM for the one-head
    // kernel, 2 for the grouped-query kernel, whose stages are larger), but at
    // least 1024 keys per split: short splits spend their time filling the pipeline
    // (measured on the 32B sliding layer: 4 splits of 1024 keys take 27 us, 32 splits
    // of 128 keys 47 us).
    const int64_t target = mma ? 148 * 2 * 4 : 148 * 3 * 8;
    const int64_t pairs = static_cast<int64_t>(B) * G;
    splits = (target + pairs - 1) / pairs;
    const int64_t max_splits = (grains + 15) / 16;
    if (splits > max_splits) splits = max_splits;
  }
  if (splits < 1) splits = 1;
  if (splits > grains) splits = grains;
  const int64_t grains_per_split = (grains + splits - 1) / splits;
  pl.chunk = static_cast<int>(grains_per_split * kDecodeGrain);
  pl.n_splits = static_cast<int>((n_max + static_cast<int64_t>(pl.chunk) - 1) / pl.chunk);
  return pl;
}

template <int D, int R>
static cudaError_t launch_rd(const CUtensorMap &tmK, const CUtensorMap &tmV, const void *q, int H,
                             const olmo3_kv_cache &c, const int32_t *kv_len, const DecodePlan &pl, void *out,
                             float *lse_out, float scale, float *ws, int *err, cudaStream_t stream) {
  using S = DecodeSmem<D, R>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_decode_split_kernel<D, R>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, S::kBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int B = c.B;
  float *ws_o = ws;
  float *ws_ml = ws + static_cast<int64_t>(B) * H * pl.n_splits * D;
  const float scale_log2 = scale * 1.4426950408889634f;
  dim3 grid(c.G, pl.n_splits, B);
  attn_decode_split_kernel<D, R><<<grid, kDecThreads, S::kBytes, stream>>>(
      tmK, tmV, static_cast<const __nv_bfloat16 *>(q), c.seq_base, kv_len, c.capacity, c.layer_type, c.window, H,
      pl.chunk, pl.n_splits, scale_log2, ws_o, ws_ml, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_decode_combine_kernel<D><<<dim3(H, B), D, 0, stream>>>(kv_len, c.capacity, c.layer_type, c.window, H,
                                                              pl.chunk, pl.n_splits, ws_o, ws_ml,
                                                              static_cast<__nv_bfloat16 *>(out), lse_out);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_gqa(int R, const CUtensorMap &tmK, const CUtensorMap &tmV, const void *q, int H,
                              const olmo3_kv_cache &c, const int32_t *kv_len, const DecodePlan &pl, void *out,
                              float *lse_out, float scale, float *ws, int *err, cudaStream_t stream) {
  using S = GqaSmem<D>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(attn_decode_gqa_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int B = c.B;
  float *ws_o = ws;
  float *ws_ml = ws + static_cast<int64_t>(B) * H * pl.n_splits * D;
  dim3 grid(c.G, pl.n_splits, B);
  attn_decode_gqa_kernel<D><<<grid, kGqaThreads, S::kBytes, stream>>>(
      tmK, tmV, static_cast<const __nv_bfloat16 *>(q), c.seq_base, kv_len, c.capacity, c.layer_type, c.window, H, R,
      pl.chunk, pl.n_splits, scale * 1.4426950408889634f, ws_o, ws_ml, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_decode_combine_kernel<D><<<dim3(H, B), D, 0, stream>>>(kv_len, c.capacity, c.layer_type, c.window, H,
                                                              pl.chunk, pl.n_splits, ws_o, ws_ml,
                                                              static_cast<__nv_bfloat16 *>(out), lse_out);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_d(int R, const CUtensorMap &tmK, const CUtensorMap &tmV, const void *q, int H,
                            const olmo3_kv_cache &c, const int32_t *kv_len, const DecodePlan &pl, void *out,
                            float *lse_out, float scale, float *ws, int *err, cudaStream_t stream) {
  if (R != 1) return cudaErrorInvalidValue;
  return launch_rd<D, 1>(tmK, tmV, q, H, c, kv_len, pl, out, lse_out, scale, ws, err, stream);
}

cudaError_t launch_attn_decode(const CUtensorMap &tmK, const CUtensorMap &tmV, const void *q, int H,
                               const olmo3_kv_cache &c, const int32_t *kv_len, const DecodePlan &plan, void *out,
                               float *lse_out, float scale, float *ws, int *err, cudaStream_t stream) {
  const int R = H / c.G;
  if (decode_uses_mma(H, c.G)) {
    if (c.d == 64) return launch_gqa<64>(R, tmK, tmV, q, H, c, kv_len, plan, out, lse_out, scale, ws, err, stream);
    return launch_gqa<128>(R, tmK, tmV, q, H, c, kv_len, plan, out, lse_out, scale, ws, err, stream);
  }
  if (c.d == 64) return launch_d<64>(R, tmK, tmV, q, H, c, kv_len, plan, out, lse_out, scale, ws, err, stream);
  return launch_d<128>(R, tmK, tmV, q, H, c, kv_len, plan, out, lse_out, scale, ws, err, stream);
}

}  // namespace olmo3
