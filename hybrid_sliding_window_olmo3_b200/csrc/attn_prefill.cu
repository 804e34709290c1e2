// Band-limited prefill attention on the 5th-generation tensor cores (tcgen05).
//
// "OLMo 3's Sliding-Window Attention Pattern", "The sliding-window mask": query t
// sees key s iff s <= t and t - s < window (a full layer: s <= t).  "Case Study:
// OLMo 3", "The architecture", ingredient 4: three layers in four are sliding;
// ingredient 1: grouped-query attention (head h reads key/value head h/(H/G)).
//
// One CTA computes a 128-row query tile of one head.  Only the key tiles that
// intersect the band [t - window + 1, t] of its rows are visited, so a sliding
// layer costs O(T * window) instead of O(T^2); only the two edge tiles of the
// band apply the mask predicate.
//
// Warp roles (192 threads):
//   warps 0-3  softmax + epilogue: thread i owns query row i = TMEM lane i.
//   warp  4    TMA producer: Q once, then K and V tiles into a 2-stage ring.
//   warp  5    TMEM allocator and MMA issuer (one thread).
// Tensor memory (512 columns): S double buffer at columns [0,128) and [128,256)
// (fp32 128x128 score tiles), O accumulator at [256, 256 + d).
// Per key tile j: S_j = Q K_j^T on the tensor core while the softmax warps turn
// S_{j-1} into P_{j-1} (bf16, written to shared memory in the 128-byte-swizzled
// K-major layout the MMA reads); then O += P_j V_j with V read MN-major.  The
// running max is only raised (and O rescaled in TMEM) when a row's max grows by
// more than 2^8, so P stays <= 256 and most tiles skip the rescale.
// Every wait is bounded: on a timeout the CTA records OLMO3_DEVERR_TIMEOUT,
// drains its copies in flight, frees its tensor memory and exits.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace olmo3 {

constexpr int kBM = kPrefillBM;
constexpr int kBN = kPrefillBN;
constexpr int kPfStages = 2;
constexpr int kPfThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
struct PfLayout {
  static constexpr int kQBytes = kBM * D * 2;  // D/64 swizzled blocks of 128 rows x 128 B
  static constexpr int kKBytes = kBN * D * 2;
  static constexpr int kVBytes = kBN * D * 2;
  static constexpr int kPBytes = kBM * kBN * 2;  // 2 swizzled blocks of 128 rows x 128 B
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffV = kOffK + kPfStages * kKBytes;
  static constexpr int kOffP = kOffV + kPfStages * kVBytes;
  static constexpr int kUsed = kOffP + kPBytes;
  // at least 120 KB so that one CTA (and one 512-column TMEM allocation) fits an SM
  static constexpr int kDynBytes = (kUsed + 1024) > 120 * 1024 ? (kUsed + 1024) : 120 * 1024;
};

template <int D>
__global__ void __launch_bounds__(kPfThreads, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, __nv_bfloat16 *__restrict__ out,
                        float *__restrict__ lse_out, int T, int H, int G, int layer_type, int window,
                        float scale_log2, int n_qtiles, int *err) {
  using LY = PfLayout<D>;
  constexpr int NDB = D / 64;  // 64-feature (128-byte) blocks per row
  constexpr uint32_t IDESC_S = idesc_bf16_f32(kBM, kBN, 0);
  constexpr uint32_t IDESC_O = idesc_bf16_f32(kBM, D, 1);

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full, k_full[kPfStages], v_full[kPfStages], kv_empty[kPfStages];
  __shared__ uint64_t s_full[2], s_free[2], p_full, o_done, mma_drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem + LY::kOffQ;
  uint8_t *sK = smem + LY::kOffK;
  uint8_t *sV = smem + LY::kOffV;
  uint8_t *sP = smem + LY::kOffP;

  const int h = blockIdx.x;
  const int qt = n_qtiles - 1 - static_cast<int>(blockIdx.y);  // longest rows first
  const int b = blockIdx.z;
  const int g = h / (H / G);
  const int q0 = qt * kBM;
  const int q_last = min(q0 + kBM, T) - 1;
  const bool is_full = layer_type == OLMO3_FULL;
  const int64_t lo_key = static_cast<int64_t>(q0) - window + 1;
  const int64_t first_key = (is_full || lo_key < 0) ? 0 : lo_key;
  const int kt_first = static_cast<int>(first_key / kBN);
  const int n_kt = q_last / kBN - kt_first + 1;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int i = 0; i < kPfStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], kBM);
    }
    mbar_init(&p_full, kBM);
    mbar_init(&o_done, 1);
    mbar_init(&mma_drain, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 4) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(&q_full, LY::kQBytes);
#pragma unroll
      for (int db = 0; db < NDB; ++db) tma_load_4d(sQ + db * kBM * 128, &tmQ, &q_full, db * 64, h, q0, b);
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n_kt; ++j) {
        const int st = j % kPfStages;
        if (j >= kPfStages && !mbar_wait(&kv_empty[st], ((j / kPfStages) & 1) ^ 1, &s_abort)) {
          ok = false;
          break;
        }
        const int k0 = (kt_first + j) * kBN;
        mbar_arrive_expect_tx(&k_full[st], LY::kKBytes);
#pragma unroll
        for (int db = 0; db < NDB; ++db)
          tma_load_4d(sK + st * LY::kKBytes + db * kBN * 128, &tmK, &k_full[st], db * 64, g, k0, b);
        mbar_arrive_expect_tx(&v_full[st], LY::kVBytes);
#pragma unroll
        for (int db = 0; db < NDB; ++db)
          tma_load_4d(sV + st * LY::kVBytes + db * kBN * 128, &tmV, &v_full[st], db * 64, g, k0, b);
        ++issued;
      }
      if (!ok) {
        s_abort = 1;
        set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
        mbar_wait(&q_full, 0, nullptr);
        for (int j = max(0, issued - kPfStages); j < issued; ++j) {
          mbar_wait(&k_full[j % kPfStages], (j / kPfStages) & 1, nullptr);
          mbar_wait(&v_full[j % kPfStages], (j / kPfStages) & 1, nullptr);
        }
      }
    }
  } else if (warp == 5) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV), aP = smem_u32(sP);
      const uint32_t tO = tmem + 256;
      bool ok = mbar_wait(&q_full, 0, &s_abort);
      auto issue_s = [&](int j) -> bool {
        const int st = j % kPfStages, sb = j & 1;
        if (!mbar_wait(&k_full[st], (j / kPfStages) & 1, &s_abort)) return false;
        if (j >= 2 && !mbar_wait(&s_free[sb], ((j >> 1) - 1) & 1, &s_abort)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t qa = aQ + (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
          const uint32_t ka = aK + st * LY::kKBytes + (kk >> 2) * (kBN * 128) + (kk & 3) * 32;
          umma_bf16(tmem + sb * kBN, sw128_desc(qa, 16, 1024), sw128_desc(ka, 16, 1024), IDESC_S, kk > 0);
        }
        umma_commit(&s_full[sb]);
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int st = j % kPfStages;
        if (!mbar_wait(&p_full, j & 1, &s_abort)) return false;
        if (!mbar_wait(&v_full[st], (j / kPfStages) & 1, &s_abort)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint32_t pa = aP + (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
          const uint32_t va = aV + st * LY::kVBytes + kk * (16 * 128);
          umma_bf16(tO, sw128_desc(pa, 16, 1024), sw128_desc(va, kBN * 128, 1024), IDESC_O, (j > 0 || kk > 0));
        }
        umma_commit(&kv_empty[st]);
        umma_commit(&o_done);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 0; ok && j < n_kt; ++j) {
        if (j + 1 < n_kt) ok = issue_s(j + 1);
        if (ok) ok = issue_pv(j);
      }
      if (!ok) {
        s_abort = 1;
        set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
      }
      // every MMA this thread issued has completed before tensor memory is freed
      umma_commit(&mma_drain);
      mbar_wait(&mma_drain, 0, nullptr);
    }
  } else {
    // -------------------------- softmax + epilogue --------------------------
    const int row = threadIdx.x;  // TMEM lane and query row inside the tile
    const int t = q0 + row;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    float m_used = -INFINITY, lsum = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kt; ++j) {
      const int sb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[sb], (j >> 1) & 1, &s_abort))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[kBN / 32][32];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) tmem_ld32(tmem + lane_off + sb * kBN + c * 32, sr[c]);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&s_free[sb]);

      const int k0 = (kt_first + j) * kBN;
      const bool need_mask = !(k0 + kBN - 1 <= q0 && (is_full || (q0 + kBM - 1) - k0 < window));
      float mt = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float x = __uint_as_float(sr[c][i]) * scale_log2;
          if (need_mask) {
            const int key = k0 + c * 32 + i;
            const bool allowed = key <= t && (is_full || t - key < window);
            x = allowed ? x : -INFINITY;
          }
          sr[c][i] = __float_as_uint(x);
          mt = fmaxf(mt, x);
        }
      }
      const float mn = fmaxf(m_used, mt);
      const bool resc = mn > m_used + kRescaleLog2;  // false while the row has seen nothing
      float alpha = 1.f;
      if (resc) {
        alpha = ex2(m_used - mn);  // 0 when m_used == -inf
        m_used = mn;
      }
      const float m_eff = (m_used == -INFINITY) ? 0.f : m_used;
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p = ex2(__uint_as_float(sr[c][i]) - m_eff);
          rs += p;
          sr[c][i] = __float_as_uint(p);
        }
      }
      lsum = lsum * alpha + rs;

      // P_j overwrites P_{j-1} and O is rescaled: both wait for PV_{j-1}
      if (j > 0) {
        if (!__all_sync(0xffffffffu, mbar_wait(&o_done, (j - 1) & 1, &s_abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t orr[32];
            tmem_ld32(tmem + lane_off + 256 + c * 32, orr);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
            tmem_st32(tmem + lane_off + 256 + c * 32, orr);
          }
          tmem_wait_st();
        }
      }
      // P row -> shared memory, 128-byte swizzle: 16-byte chunk c of row r at c ^ (r % 8)
#pragma unroll
      for (int kb = 0; kb < kBN / 64; ++kb) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int e = kb * 64 + c * 8;
          uint4 u;
          u.x = f2_to_bf2(__uint_as_float(sr[e / 32][e % 32 + 0]), __uint_as_float(sr[e / 32][e % 32 + 1]));
          u.y = f2_to_bf2(__uint_as_float(sr[e / 32][e % 32 + 2]), __uint_as_float(sr[e / 32][e % 32 + 3]));
          u.z = f2_to_bf2(__uint_as_float(sr[e / 32][e % 32 + 4]), __uint_as_float(sr[e / 32][e % 32 + 5]));
          u.w = f2_to_bf2(__uint_as_float(sr[e / 32][e % 32 + 6]), __uint_as_float(sr[e / 32][e % 32 + 7]));
          *reinterpret_cast<uint4 *>(sP + kb * (kBM * 128) + row * 128 + ((c ^ (row & 7)) * 16)) = u;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full);
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&o_done, (n_kt - 1) & 1, &s_abort));
    if (!ok) {
      if (lane == 0) {
        s_abort = 1;
        set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
      }
    } else {
      tc_fence_after();
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      __nv_bfloat16 *orow = out + ((static_cast<int64_t>(b) * T + t) * H + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orr[32];
        tmem_ld32(tmem + lane_off + 256 + c * 32, orr);
        tmem_wait_ld();
        if (t < T) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 u;
            u.x = f2_to_bf2(__uint_as_float(orr[v * 8 + 0]) * inv, __uint_as_float(orr[v * 8 + 1]) * inv);
            u.y = f2_to_bf2(__uint_as_float(orr[v * 8 + 2]) * inv, __uint_as_float(orr[v * 8 + 3]) * inv);
            u.z = f2_to_bf2(__uint_as_float(orr[v * 8 + 4]) * inv, __uint_as_float(orr[v * 8 + 5]) * inv);
            u.w = f2_to_bf2(__uint_as_float(orr[v * 8 + 6]) * inv, __uint_as_float(orr[v * 8 + 7]) * inv);
            *reinterpret_cast<uint4 *>(orow + c * 32 + v * 8) = u;
          }
        }
      }
      if (lse_out != nullptr && t < T) {
        const float m_eff = (m_used == -INFINITY) ? 0.f : m_used;
        lse_out[(static_cast<int64_t>(b) * H + h) * T + t] = (m_eff + log2f(lsum)) * 0.69314718055994531f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
static cudaError_t launch_pf(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV, void *out,
                             float *lse_out, int B, int T, int H, int G, int layer_type, int window, float scale,
                             int *err, cudaStream_t stream) {
  using LY = PfLayout<D>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(attn_prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, LY::kDynBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int n_qtiles = (T + kBM - 1) / kBM;
  dim3 grid(H, n_qtiles, B);
  attn_prefill_kernel<D><<<grid, kPfThreads, LY::kDynBytes, stream>>>(
      tmQ, tmK, tmV, static_cast<__nv_bfloat16 *>(out), lse_out, T, H, G, layer_type, window,
      scale * 1.4426950408889634f, n_qtiles, err);
  return cudaGetLastError();
}

cudaError_t launch_attn_prefill(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV, void *out,
                                float *lse_out, int B, int T, int H, int G, int d, int layer_type, int window,
                                float scale, int *err, cudaStream_t stream) {
  if (d == 64) return launch_pf<64>(tmQ, tmK, tmV, out, lse_out, B, T, H, G, layer_type, window, scale, err, stream);
  return launch_pf<128>(tmQ, tmK, tmV, out, lse_out, B, T, H, G, layer_type, window, scale, err, stream);
}

}  // namespace olmo3
