// Output projection + reordered post-norm + residual on the tensor cores.
//
// "Case Study: OLMo 3", "The architecture", ingredient 1 (bias-free projections)
// and ingredient 6 ("Reordered norm"): h = x + RMSNorm(Attention(x)), where the
// attention output passes through W_o first and the norm (one gain per model
// feature) acts on the projected output, before the residual addition.
//
// Two kernels:
//   gemm_rowss_kernel  Y[M, N] = A[M, K] * B[N, K]^T with tcgen05.mma (bf16 in,
//                      f32 accumulate in TMEM).  One CTA per 128 x 256 tile: a
//                      producer warp streams 64-wide K slices of A and B through a
//                      4-stage TMA ring (128-byte swizzle), one thread issues the
//                      MMAs, 4 epilogue warps read the accumulator rows, store Y in
//                      bf16 and add each row's sum of squares (from the f32 values)
//                      to ss[M] — the norm needs the whole row, which spans N/256
//                      CTAs.
//   postnorm_residual_kernel  h = x + Y * rsqrt(ss / N + eps) * gain (one CTA per row).
// Every wait is bounded, as in the attention kernels.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace olmo3 {

constexpr int kGBM = 128, kGBN = 256, kGBK = 64, kGStages = 4;
constexpr int kGThreads = 192;  // warps 0-3 epilogue, warp 4 TMA, warp 5 MMA + TMEM
constexpr int kGABytes = kGBM * kGBK * 2;
constexpr int kGBBytes = kGBN * kGBK * 2;
constexpr int kGStageBytes = kGABytes + kGBBytes;
constexpr int kGSmemBytes = kGStages * kGStageBytes + 1024;

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *tm, uint64_t *bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__global__ void __launch_bounds__(kGThreads, 1)
    gemm_rowss_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                      __nv_bfloat16 *__restrict__ Y, float *__restrict__ ss, int M, int N, int K, int *err) {
  constexpr uint32_t IDESC = idesc_bf16_f32(kGBM, kGBN, 0);
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[kGStages], empty_bar[kGStages], acc_bar;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int n0 = blockIdx.x * kGBN, m0 = blockIdx.y * kGBM;
  const int nk = K / kGBK;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    mbar_init(&acc_bar, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&s_tmem, kGBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 4) {
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      int issued = 0;
      bool ok = true;
      for (int kc = 0; kc < nk; ++kc) {
        const int st = kc % kGStages;
        if (kc >= kGStages && !mbar_wait(&empty_bar[st], ((kc / kGStages) & 1) ^ 1, &s_abort)) {
          ok = false;
          break;
        }
        uint8_t *sa = smem + st * kGStageBytes;
        mbar_arrive_expect_tx(&full_bar[st], kGStageBytes);
        tma_load_2d(sa, &tmA, &full_bar[st], kc * kGBK, m0);
        tma_load_2d(sa + kGABytes, &tmB, &full_bar[st], kc * kGBK, n0);
        ++issued;
      }
      if (!ok) {
        s_abort = 1;
        set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
        for (int i = max(0, issued - kGStages); i < issued; ++i)
          mbar_wait(&full_bar[i % kGStages], (i / kGStages) & 1, nullptr);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      bool ok = true;
      for (int kc = 0; kc < nk; ++kc) {
        const int st = kc % kGStages;
        if (!mbar_wait(&full_bar[st], (kc / kGStages) & 1, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + st * kGStageBytes), sb = sa + kGABytes;
#pragma unroll
        for (int kk = 0; kk < kGBK / 16; ++kk)
          umma_bf16(tmem, sw128_desc(sa + kk * 32, 16, 1024), sw128_desc(sb + kk * 32, 16, 1024), IDESC,
                    (kc > 0 || kk > 0));
        umma_commit(&empty_bar[st]);
      }
      if (!ok) {
        s_abort = 1;
        set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
      }
      umma_commit(&acc_bar);  // also drains every MMA before the teardown
      mbar_wait(&acc_bar, 0, nullptr);
    }
  } else {
    // ------------------------------ epilogue ------------------------------
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&acc_bar, 0, &s_abort));
    if (ok && !s_abort) {
      tc_fence_after();
      const int row = m0 + threadIdx.x;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
      float sq = 0.f;
#pragma unroll 1
      for (int c = 0; c < kGBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        tmem_wait_ld();
        const int col = n0 + c * 32;
        if (row < M) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            if (col + v * 8 + 8 <= N) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                f[e] = __uint_as_float(r[v * 8 + e]);
                sq = fmaf(f[e], f[e], sq);
              }
              uint4 u;
              u.x = f2_to_bf2(f[0], f[1]);
              u.y = f2_to_bf2(f[2], f[3]);
              u.z = f2_to_bf2(f[4], f[5]);
              u.w = f2_to_bf2(f[6], f[7]);
              *reinterpret_cast<uint4 *>(Y + static_cast<int64_t>(row) * N + col + v * 8) = u;
            }
          }
        }
      }
      if (row < M) atomicAdd(ss + row, sq);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kGBN);
  }
}

// h[r] = x[r] + Y[r] * rsqrt(ss[r] / N + eps) * gain  (bf16 in and out, f32 math)
__global__ void __launch_bounds__(256) postnorm_residual_kernel(const __nv_bfloat16 *__restrict__ Y,
                                                                const float *__restrict__ ss,
                                                                const float *__restrict__ gain,
                                                                const __nv_bfloat16 *x, __nv_bfloat16 *h, int N,
                                                                float eps) {
  const int64_t r = blockIdx.x;
  const float rinv = 1.0f / sqrtf(ss[r] / static_cast<float>(N) + eps);
  for (int c = threadIdx.x * 8; c < N; c += 256 * 8) {
    const uint4 yu = *reinterpret_cast<const uint4 *>(Y + r * N + c);
    const uint4 xu = *reinterpret_cast<const uint4 *>(x + r * N + c);
    const float4 g0 = *reinterpret_cast<const float4 *>(gain + c);
    const float4 g1 = *reinterpret_cast<const float4 *>(gain + c + 4);
    const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
    const uint32_t yw[4] = {yu.x, yu.y, yu.z, yu.w}, xw[4] = {xu.x, xu.y, xu.z, xu.w};
    uint32_t ow[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 yf = bf2_to_f2(yw[j]), xf = bf2_to_f2(xw[j]);
      ow[j] = f2_to_bf2(fmaf(yf.x * rinv, gg[2 * j], xf.x), fmaf(yf.y * rinv, gg[2 * j + 1], xf.y));
    }
    *reinterpret_cast<uint4 *>(h + r * N + c) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  }
}

cudaError_t launch_out_proj(const CUtensorMap &tmA, const CUtensorMap &tmB, void *Y, float *ss, const float *gain,
                            const void *x, void *h, int M, int N, int K, float eps, int *err, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_rowss_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaError_t e = cudaMemsetAsync(ss, 0, sizeof(float) * static_cast<size_t>(M), stream);
  if (e != cudaSuccess) return e;
  dim3 grid((N + kGBN - 1) / kGBN, (M + kGBM - 1) / kGBM);
  gemm_rowss_kernel<<<grid, kGThreads, kGSmemBytes, stream>>>(tmA, tmB, static_cast<__nv_bfloat16 *>(Y), ss, M, N, K,
                                                                err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  postnorm_residual_kernel<<<M, 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(Y), ss, gain,
                                                  static_cast<const __nv_bfloat16 *>(x),
                                                  static_cast<__nv_bfloat16 *>(h), N, eps);
  return cudaGetLastError();
}

}  // namespace olmo3
