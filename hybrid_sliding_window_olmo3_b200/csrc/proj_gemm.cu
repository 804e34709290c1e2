// The attention block's two projections on the tensor cores, each with the
// normalisation that follows it fused into the GEMM epilogue.
//
//   QKV:  "Case Study: OLMo 3", "The architecture", ingredient 1 (bias-free
//         projections of the block input, which ingredient 6 leaves un-normed),
//         then ingredient 2 (QK-norm: RMSNorm over all H*d query and all G*d key
//         features) and ingredient 3 (RoPE, pair i with i + d/2) on q and k;
//         YaRN frequencies and temperature on full layers ("Olmo 3 7B", long-context
//         extension).  "Olmo-3 End-to-End Implementation", "Inference Pipeline":
//         token t of sequence b sits at position pos_offset[b] + t.
//   Wo:   ingredient 6 ("Reordered norm"): h = x + RMSNorm(attn W_o^T), one gain
//         per model feature.
//
// Both are Y = A B^T (bf16 operands, f32 accumulation in tensor memory, 128 x 256
// output tiles, K in 64-wide slices through a 4-stage TMA ring).  Their epilogues
// need a statistic of the whole output row (the sum of squares over H*d, G*d or D
// features), and a row spans several tiles.  So the kernel is persistent: one CTA
// per SM, launched cooperatively so that every CTA is resident; CTA c takes tiles
// c, c + grid, c + 2 grid, ... in row-block-major order, and its epilogue warps
//   1. read the accumulator and add the tile's share of each row's sum of squares
//      to a global array, then count the tile as published for its row block;
//   2. wait (bounded) until every tile of the row block that the norm spans has
//      published;
//   3. read the accumulator again and write the normalised result in bf16
//      (rotated, for q and k; plus the residual, for Wo).
// The accumulator is double-buffered in TMEM (2 x 256 columns), so the MMAs of the
// CTA's next tile run while its epilogue waits.
//
// Tile order.  Output columns are split into phases (QKV: the q columns, then the k
// and v columns, as one phase or, when their weights exceed 48 MB, as two; Wo: one
// phase), and each phase runs its row blocks in order, all of the phase's column
// tiles of a row block back to back.  A phase's weights (10-52 MB for the 7B and 32B
// models) then stay in L2 while every row block streams past them, instead of the
// whole W_qkv cycling through L2 once per wave.
// Deadlock freedom: position p of this order runs on CTA p mod grid after the tile at
// p - grid.  A tile waits only for the tiles of its norm group (its row block's q
// tiles, or k tiles, or all Wo tiles), which sit within fewer than `grid` consecutive
// positions; so every tile it waits for sits at a position below p + grid and is
// queued behind positions below p, and by induction over positions each tile
// publishes.
//
// RMSNorm commutes with the rotation up to the per-row factor, so nothing is
// written before the factor is known: no intermediate Y in HBM.
#include <math.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace olmo3 {

constexpr int kPBM = 128, kPBN = 256, kPBK = 64, kPStages = 4;
constexpr int kPThreads = 192;  // warps 0-3 epilogue (one accumulator row each), 4 TMA, 5 MMA + TMEM
constexpr int kPABytes = kPBM * kPBK * 2;
constexpr int kPBBytes = kPBN * kPBK * 2;
constexpr int kPStageBytes = kPABytes + kPBBytes;
constexpr int kPSmemBytes = kPStages * kPStageBytes + 1024;
// Weights of one QKV column phase above this size get a phase each for k and v.
constexpr size_t kQkvPhaseBytes = static_cast<size_t>(48) << 20;

// QKV epilogue: columns [0, Hd) of Y are q, [Hd, Hd + Gd) k, the rest v.
template <int D>
struct QkvEpilogue {
  __nv_bfloat16 *q, *k, *v;
  const float *gain_q, *gain_k;
  const int32_t *pos_offset;
  float *ss_q, *ss_k;  // [M] sums of squares of the raw projections
  int *count;          // [2 * row blocks]: q tiles and k tiles published
  int *abort_flag;     // set by the first CTA whose wait gives up
  int T, Hd, Gd;
  float eps;
  RopeTable tab;
};

// Wo epilogue: h = x + Y rsqrt(ss / N + eps) gain.
struct PostNormEpilogue {
  const __nv_bfloat16 *x;
  __nv_bfloat16 *h;
  const float *gain;
  float *ss;   // [M]
  int *count;  // [row blocks]
  int *abort_flag;
  float eps;
};

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *tm, uint64_t *bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Named barrier 1 over the 128 epilogue threads (warps 0-3).
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// Same barrier, returning whether any epilogue thread passed `p` true.
__device__ __forceinline__ bool epi_any(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\tsetp.ne.u32 a, %1, 0;\n\tbar.red.or.pred b, 1, 128, a;\n\tselp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(p))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ int ld_acquire_gpu(const int *p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Step 1 and 2 of the epilogue for one tile.  Every epilogue thread calls it; the
// result is the same in all of them.
__device__ __forceinline__ bool publish_and_wait(float *ss_row, float sq, int *count, int expected, int *abort_flag,
                                                 int *err, volatile int *s_abort, int *s_flag) {
  if (ss_row != nullptr) atomicAdd(ss_row, sq);
  __threadfence();
  epi_sync();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(count, 1);
    bool ok = true;
    if (ld_acquire_gpu(count) < expected) {
      const uint64_t t0 = globaltimer_ns();
      for (uint32_t it = 1;; ++it) {
        __nanosleep(32);
        if (ld_acquire_gpu(count) >= expected) break;
        if ((it & 15u) == 0 &&
            (ld_acquire_gpu(abort_flag) != 0 || globaltimer_ns() - t0 > kWaitLimitNs)) {
          ok = false;
          break;
        }
      }
    }
    if (!ok) {
      atomicExch(abort_flag, 1);
      set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
      *s_abort = 1;
    }
    __threadfence();
    *s_flag = ok ? 1 : 0;
  }
  epi_sync();
  return *reinterpret_cast<volatile int *>(s_flag) != 0;
}

__device__ __forceinline__ float row_sumsq(uint32_t taddr) {
  float sq = 0.f;
#pragma unroll 1
  for (int c = 0; c < kPBN / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + c * 32, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 32; ++e) sq = fmaf(__uint_as_float(r[e]), __uint_as_float(r[e]), sq);
  }
  return sq;
}

__device__ __forceinline__ void store32_bf16(__nv_bfloat16 *dst, const float (&f)[32]) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    uint4 u;
    u.x = f2_to_bf2(f[8 * v + 0], f[8 * v + 1]);
    u.y = f2_to_bf2(f[8 * v + 2], f[8 * v + 3]);
    u.z = f2_to_bf2(f[8 * v + 4], f[8 * v + 5]);
    u.w = f2_to_bf2(f[8 * v + 6], f[8 * v + 7]);
    reinterpret_cast<uint4 *>(dst)[v] = u;
  }
}

__device__ __forceinline__ void load32_f32(const float *p, float (&f)[32]) {
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    const float4 a = reinterpret_cast<const float4 *>(p)[v];
    f[4 * v + 0] = a.x;
    f[4 * v + 1] = a.y;
    f[4 * v + 2] = a.z;
    f[4 * v + 3] = a.w;
  }
}

template <int D>
__device__ __forceinline__ void epilogue_tile(const QkvEpilogue<D> &ep, uint32_t taddr, int rb, int nt, int M, int N,
                                              int *err, volatile int *s_abort, int *s_flag) {
  const int n0 = nt * kPBN;
  const int row = rb * kPBM + static_cast<int>(threadIdx.x);
  const bool in = row < M;
  if (n0 >= ep.Hd + ep.Gd) {  // v: plain bf16 store
    __nv_bfloat16 *dst = ep.v + static_cast<int64_t>(row) * ep.Gd + (n0 - ep.Hd - ep.Gd);
#pragma unroll 1
    for (int c = 0; c < kPBN / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + c * 32, r);
      tmem_wait_ld();
      float f[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(r[e]);
      if (in) store32_bf16(dst + c * 32, f);
    }
    return;
  }
  const bool is_q = n0 < ep.Hd;
  const int width = is_q ? ep.Hd : ep.Gd;
  const int col0 = is_q ? n0 : n0 - ep.Hd;
  float *ss = is_q ? ep.ss_q : ep.ss_k;
  const float sq = row_sumsq(taddr);
  if (!publish_and_wait(in ? ss + row : nullptr, sq, ep.count + 2 * rb + (is_q ? 0 : 1), width / kPBN,
                        ep.abort_flag, err, s_abort, s_flag))
    return;

  const float rinv = in ? 1.0f / sqrtf(__ldcg(ss + row) / static_cast<float>(width) + ep.eps) : 0.f;
  double pos = 0.0;
  if (in) {
    const int b = row / ep.T;
    pos = static_cast<double>(ep.pos_offset[b]) + static_cast<double>(row - b * ep.T);
  }
  __nv_bfloat16 *dst = (is_q ? ep.q : ep.k) + static_cast<int64_t>(row) * width + col0;
  const float *gain = (is_q ? ep.gain_q : ep.gain_k) + col0;
  constexpr double kTwoPi = 6.283185307179586476925286766559;
#pragma unroll
  for (int ic = 0; ic < D / 2; ic += 32) {
    // cos / sin of pos * f_i for 32 pairs: the angle is reduced to [-pi, pi] in
    // fp64 (it reaches ~1e6 rad at long positions), then evaluated in fp32.
    float cs[32], sn[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const double a = pos * ep.tab.inv_freq[ic + j];
      const double turns = rint(a * (1.0 / kTwoPi));
      float s, c;
      sincosf(static_cast<float>(fma(-turns, kTwoPi, a)), &s, &c);
      cs[j] = c * ep.tab.out_scale;
      sn[j] = s * ep.tab.out_scale;
    }
#pragma unroll 1
    for (int hh = 0; hh < kPBN / D; ++hh) {
      const int lo_col = hh * D + ic, hi_col = lo_col + D / 2;
      uint32_t rl[32], rh[32];
      tmem_ld32(taddr + lo_col, rl);
      tmem_ld32(taddr + hi_col, rh);
      tmem_wait_ld();
      float glo[32], ghi[32];
      load32_f32(gain + lo_col, glo);
      load32_f32(gain + hi_col, ghi);
      float zl[32], zh[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float a = __uint_as_float(rl[j]) * rinv * glo[j];
        const float b = __uint_as_float(rh[j]) * rinv * ghi[j];
        zl[j] = a * cs[j] - b * sn[j];
        zh[j] = b * cs[j] + a * sn[j];
      }
      if (in) {
        store32_bf16(dst + lo_col, zl);
        store32_bf16(dst + hi_col, zh);
      }
    }
  }
}

__device__ __forceinline__ void epilogue_tile(const PostNormEpilogue &ep, uint32_t taddr, int rb, int nt, int M, int N,
                                              int *err, volatile int *s_abort, int *s_flag) {
  const int n0 = nt * kPBN;
  const int row = rb * kPBM + static_cast<int>(threadIdx.x);
  const bool in = row < M;
  // Columns past N hold zeros (the weight tile is zero-filled there).
  const float sq = row_sumsq(taddr);
  const int n_tiles_n = (N + kPBN - 1) / kPBN;
  if (!publish_and_wait(in ? ep.ss + row : nullptr, sq, ep.count + rb, n_tiles_n, ep.abort_flag, err, s_abort,
                        s_flag))
    return;
  const float rinv = in ? 1.0f / sqrtf(__ldcg(ep.ss + row) / static_cast<float>(N) + ep.eps) : 0.f;
  const int64_t base = static_cast<int64_t>(row) * N;
#pragma unroll 1
  for (int c = 0; c < kPBN / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(taddr + c * 32, r);
    tmem_wait_ld();
    const int col = n0 + c * 32;
    if (in) {
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int cv = col + v * 8;
        if (cv + 8 <= N) {
          const uint4 xu = *reinterpret_cast<const uint4 *>(ep.x + base + cv);
          const float4 g0 = *reinterpret_cast<const float4 *>(ep.gain + cv);
          const float4 g1 = *reinterpret_cast<const float4 *>(ep.gain + cv + 4);
          const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
          const uint32_t xw[4] = {xu.x, xu.y, xu.z, xu.w};
          uint32_t ow[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 xf = bf2_to_f2(xw[j]);
            const float y0 = __uint_as_float(r[v * 8 + 2 * j]), y1 = __uint_as_float(r[v * 8 + 2 * j + 1]);
            ow[j] = f2_to_bf2(fmaf(y0 * rinv, gg[2 * j], xf.x), fmaf(y1 * rinv, gg[2 * j + 1], xf.y));
          }
          *reinterpret_cast<uint4 *>(ep.h + base + cv) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        }
      }
    }
  }
}

// Column phases of the tile order: phase i covers column tiles [col0[i], col0[i] +
// cols[i]) for every row block, at positions [start[i], start[i + 1]).
struct TileOrder {
  int n_phases;
  int col0[3], cols[3], start[4];
};

__device__ __forceinline__ void tile_at(const TileOrder &o, int pos, int &rb, int &nt) {
  int ph = 0;
#pragma unroll
  for (int i = 1; i < 3; ++i)
    if (i < o.n_phases && pos >= o.start[i]) ph = i;
  const int local = pos - o.start[ph];
  rb = local / o.cols[ph];
  nt = o.col0[ph] + (local - rb * o.cols[ph]);
}

template <class Epi>
__global__ void __launch_bounds__(kPThreads, 1)
    proj_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ Epi ep, const __grid_constant__ TileOrder order, int M, int N, int K,
                     int n_tiles, int *err) {
  constexpr uint32_t IDESC = idesc_bf16_f32(kPBM, kPBN, 0);
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full_bar[kPStages], empty_bar[kPStages], acc_full[2], acc_empty[2], drain_bar;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort, s_flag;
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int nk = K / kPBK;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kPStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 128);
    }
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    s_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&s_tmem, 2 * kPBN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 4) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        int rb, nt;
        tile_at(order, tile, rb, nt);
        for (int kc = 0; kc < nk; ++kc, ++it) {
          const int st = it % kPStages;
          if (it >= kPStages && !mbar_wait(&empty_bar[st], ((it / kPStages) & 1) ^ 1, &s_abort)) {
            ok = false;
            break;
          }
          uint8_t *sa = smem + st * kPStageBytes;
          mbar_arrive_expect_tx(&full_bar[st], kPStageBytes);
          tma_load_2d(sa, &tmA, &full_bar[st], kc * kPBK, rb * kPBM);
          tma_load_2d(sa + kPABytes, &tmB, &full_bar[st], kc * kPBK, nt * kPBN);
        }
      }
      if (!ok) {
        if (!s_abort) set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
        s_abort = 1;
        // Loads already issued still land in shared memory: wait for them.
        for (int i = max(0, it - kPStages); i < it; ++i)
          mbar_wait(&full_bar[i % kPStages], (i / kPStages) & 1, nullptr);
      }
    }
  } else if (warp == 5) {
    // ------------------------------ MMA issuer --------------------------------
    // The whole warp runs the loop with the same values (descriptors stay in
    // uniform registers); one elected lane issues each MMA and commit.
    int it = 0, lt = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++lt) {
      const int buf = lt & 1;
      if (lt >= 2 && !mbar_wait_warp(&acc_empty[buf], ((lt >> 1) & 1) ^ 1, &s_abort)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t acc = tmem + buf * kPBN;
      for (int kc = 0; kc < nk; ++kc, ++it) {
        const int st = it % kPStages;
        if (!mbar_wait_warp(&full_bar[st], (it / kPStages) & 1, &s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + st * kPStageBytes);
        const uint64_t da = sw128_desc(sa, 16, 1024), db = sw128_desc(sa + kPABytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < kPBK / 16; ++kk)
          umma_bf16_elect(acc, da + kk * 2, db + kk * 2, IDESC, (kc > 0 || kk > 0));  // +32 bytes per K step
        umma_commit_elect(&empty_bar[st]);
      }
      if (ok) umma_commit_elect(&acc_full[buf]);
    }
    if (!ok && lane == 0) {
      if (!s_abort) set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
      s_abort = 1;
    }
    umma_commit_elect(&drain_bar);  // completes once every MMA issued above has
    mbar_wait_warp(&drain_bar, 0, nullptr);
  } else {
    // ------------------------------ epilogue ----------------------------------
    int lt = 0;
    for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++lt) {
      const int buf = lt & 1;
      const bool got = mbar_wait(&acc_full[buf], (lt >> 1) & 1, &s_abort);
      if (epi_any(!got || s_abort)) {  // the same decision in all 128 threads
        if (threadIdx.x == 0) {
          if (!s_abort) set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
          s_abort = 1;
        }
        break;
      }
      tc_fence_after();
      int rb, nt;
      tile_at(order, tile, rb, nt);
      const uint32_t taddr = tmem + buf * kPBN + (static_cast<uint32_t>(warp * 32) << 16);
      epilogue_tile(ep, taddr, rb, nt, M, N, err, &s_abort, &s_flag);
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kPBN);
  }
}

namespace {

// SM count of the current device (the persistent grid), cached per device.
int device_sms() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

// phase_cols: column tiles of each phase, in column order.
TileOrder make_order(int M, const int *phase_cols, int n_phases) {
  TileOrder o = {};
  const int rbs = (M + kPBM - 1) / kPBM;
  o.n_phases = n_phases;
  int col = 0, pos = 0;
  for (int i = 0; i < n_phases; ++i) {
    o.col0[i] = col;
    o.cols[i] = phase_cols[i];
    o.start[i] = pos;
    col += phase_cols[i];
    pos += rbs * phase_cols[i];
  }
  o.start[n_phases] = pos;
  return o;
}

template <class Epi>
cudaError_t launch_persistent(const CUtensorMap &tmA, const CUtensorMap &tmB, const Epi &ep, const TileOrder &order,
                              int M, int N, int K, int max_group_tiles, void *zero_region, size_t zero_bytes,
                              int *err, cudaStream_t stream) {
  static std::mutex mu;
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!attr_set[dev]) {
      e = cudaFuncSetAttribute(proj_gemm_kernel<Epi>, cudaFuncAttributeMaxDynamicSharedMemorySize, kPSmemBytes);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  const int n_tiles = order.start[order.n_phases];
  const int sms = device_sms();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int grid = n_tiles < sms ? n_tiles : sms;
  if (max_group_tiles > grid) return cudaErrorNotSupported;  // the ABI rejects this first
  e = cudaMemsetAsync(zero_region, 0, zero_bytes, stream);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = kPSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, proj_gemm_kernel<Epi>, tmA, tmB, ep, order, M, N, K, n_tiles, err);
}

}  // namespace

int proj_gemm_max_tiles_per_row() { return device_sms(); }

size_t proj_gemm_flags_bytes(int M, int rows_per_norm_group) {
  const size_t rb = (static_cast<size_t>(M) + kPBM - 1) / kPBM;
  return static_cast<size_t>(M) * rows_per_norm_group * sizeof(float) +
         (rb * rows_per_norm_group + 1) * sizeof(int);
}

cudaError_t launch_qkv_proj(const CUtensorMap &tmX, const CUtensorMap &tmW, void *q, void *k, void *v,
                            const float *gain_q, const float *gain_k, const int32_t *pos_offset, int B, int T, int H,
                            int G, int d, int Dm, float eps, const RopeTable &tab, void *ws, int *err,
                            cudaStream_t stream) {
  const int M = B * T;
  const int rb = (M + kPBM - 1) / kPBM;
  float *ss_q = static_cast<float *>(ws);
  float *ss_k = ss_q + M;
  int *count = reinterpret_cast<int *>(ss_k + M);
  int *abort_flag = count + 2 * rb;
  const size_t zero_bytes = proj_gemm_flags_bytes(M, 2);
  const int N = (H + 2 * G) * d;
  // phases: the q columns, then the k and v columns, as one phase when their
  // weights are small enough to stay in L2 next to the streamed rows, else two
  const size_t kv_weight_bytes = static_cast<size_t>(2 * G * d) * Dm * 2;
  const bool split_kv = kv_weight_bytes > kQkvPhaseBytes;
  const int phase_cols[3] = {H * d / kPBN, (split_kv ? 1 : 2) * G * d / kPBN, G * d / kPBN};
  const TileOrder order = make_order(M, phase_cols, split_kv ? 3 : 2);
  const int group = (H * d > G * d ? H * d : G * d) / kPBN;
  if (d == 64) {
    QkvEpilogue<64> ep{static_cast<__nv_bfloat16 *>(q), static_cast<__nv_bfloat16 *>(k),
                       static_cast<__nv_bfloat16 *>(v), gain_q, gain_k, pos_offset, ss_q, ss_k, count, abort_flag,
                       T, H * d, G * d, eps, tab};
    return launch_persistent(tmX, tmW, ep, order, M, N, Dm, group, ws, zero_bytes, err, stream);
  }
  QkvEpilogue<128> ep{static_cast<__nv_bfloat16 *>(q), static_cast<__nv_bfloat16 *>(k),
                      static_cast<__nv_bfloat16 *>(v), gain_q, gain_k, pos_offset, ss_q, ss_k, count, abort_flag,
                      T, H * d, G * d, eps, tab};
  return launch_persistent(tmX, tmW, ep, order, M, N, Dm, group, ws, zero_bytes, err, stream);
}

cudaError_t launch_out_proj(const CUtensorMap &tmA, const CUtensorMap &tmB, const float *gain, const void *x, void *h,
                            int M, int N, int K, float eps, void *ws, int *err, cudaStream_t stream) {
  const int rb = (M + kPBM - 1) / kPBM;
  float *ss = static_cast<float *>(ws);
  int *count = reinterpret_cast<int *>(ss + M);
  PostNormEpilogue ep{static_cast<const __nv_bfloat16 *>(x), static_cast<__nv_bfloat16 *>(h), gain, ss, count,
                      count + rb, eps};
  const int cols = (N + kPBN - 1) / kPBN;
  return launch_persistent(tmA, tmB, ep, make_order(M, &cols, 1), M, N, K, cols, ws, proj_gemm_flags_bytes(M, 1),
                           err, stream);
}

}  // namespace olmo3
