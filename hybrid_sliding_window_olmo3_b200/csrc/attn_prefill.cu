// Band-limited prefill attention on the 5th-generation tensor cores (tcgen05).
//
// "OLMo 3's Sliding-Window Attention Pattern", "The sliding-window mask": query t
// sees key s iff s <= t and t - s < window (a full layer: s <= t).  "Case Study:
// OLMo 3", "The architecture", ingredient 4: three layers in four are sliding;
// ingredient 1: grouped-query attention (head h reads key/value head h/(H/G)).
//
// One CTA computes 256 query rows (two 128-row tiles, A and B) of one head.  Only
// the key tiles that intersect the band [t - window + 1, t] of its rows are
// visited, so a sliding layer costs O(T * window) instead of O(T^2); only the
// edge tiles of each band apply the mask predicate.
//
// Warp roles (384 threads, three warpgroups):
//   WG0 (warps 0-3)  softmax + epilogue of tile A: thread i owns row i = TMEM lane i.
//   WG1 (warps 4-7)  the same for tile B.
//   WG2 warp 8       TMA producer: both Q tiles once, then K_j, V_j, K_j+1, ... into
//                    a 4-slot ring (each slot holds one 128-key K or V tile).
//       warp 9       TMEM allocator and MMA issuer (the whole warp runs the issue
//                    loop on warp-uniform values; one elected lane issues).
// WG2 gives registers to the softmax warpgroups (setmaxnreg).
// Tensor memory (512 columns): S_A [0,128), S_B [128,256) fp32 score tiles,
// O_A [256, 256+d), O_B [256+d, 256+2d) fp32 accumulators.  P (bf16, two per
// 32-bit column) overwrites the first 64 columns of its S tile once S is read,
// and the PV product takes its A operand straight from tensor memory, so shared
// memory only carries Q, K and V (the S and PV products both read two operands
// at 128 rows x 128 columns, which is what the shared-memory bandwidth allows).
// Tensor-core order per key tile j:  PV_A(j), S_A(j+1), PV_B(j), S_B(j+1): while
// one softmax warpgroup turns its S into P the tensor core works for the other
// tile, so the two warpgroups alternate against a busy tensor core.  P is handed
// over in two halves of 64 keys (two barriers), so the first half of PV starts
// while the softmax computes the second.  A row's running max is only
// raised (and O rescaled in TMEM) when it grows by more than 2^8, so P <= 256 and
// most tiles skip the rescale.  P is rounded to nearest bf16 for the PV product;
// the row sum adds the f32 weights.
// Every wait is bounded: on a timeout the CTA records OLMO3_DEVERR_TIMEOUT,
// drains its copies and MMAs in flight, frees its tensor memory and exits.
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace olmo3 {

constexpr int kBM = kPrefillBM;  // rows per query tile
constexpr int kBN = kPrefillBN;  // keys per key tile
constexpr int kRing = 4;
constexpr int kPfThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;

#ifndef OLMO3_PF_CONTROL_REGS
#define OLMO3_PF_CONTROL_REGS 72
#endif
// Register split between the control warpgroup and the two softmax warpgroups:
// 128 x control + 256 x softmax must not exceed 384 x 168 (the launch budget).
constexpr uint32_t kControlRegs = OLMO3_PF_CONTROL_REGS;
constexpr uint32_t kSoftmaxRegs = ((384u * 168u - 128u * kControlRegs) / 256u) & ~7u;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

template <int D>
struct PfLayout {
  static constexpr int kQBytes = kBM * D * 2;   // one query tile: D/64 swizzled blocks of 128 rows x 128 B
  static constexpr int kKVBytes = kBN * D * 2;  // one K or V tile
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = kOffQ + 2 * kQBytes;
  static constexpr int kUsed = kOffRing + kRing * kKVBytes;
  static constexpr int kDynBytes = kUsed + 1024;  // + alignment slack for the 1024-byte swizzle atoms
};

// Key tiles (in units of kBN keys of the key rows) that query rows at absolute
// positions [t0, t1] need, when key row j holds absolute position kp0 + j and
// rows 0 .. klen-1 exist: [first, last], empty when last < first.
__device__ __forceinline__ void band_tiles(int t0, int t1, int kp0, int klen, bool is_full, int window,
                                           int &first, int &last) {
  const int64_t w_lo = static_cast<int64_t>(t0) - window + 1;
  const int64_t lo_abs = (is_full || w_lo < kp0) ? static_cast<int64_t>(kp0) : w_lo;
  const int64_t k_hi = static_cast<int64_t>(kp0) + klen - 1;
  const int64_t hi_abs = t1 < k_hi ? static_cast<int64_t>(t1) : k_hi;
  if (hi_abs < lo_abs) {
    first = 1;
    last = 0;
    return;
  }
  first = static_cast<int>((lo_abs - kp0) / kBN);
  last = static_cast<int>((hi_abs - kp0) / kBN);
}

template <int D, int MODE>
__global__ void __launch_bounds__(kPfThreads, 1)
    attn_prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, __nv_bfloat16 *__restrict__ out,
                        float *__restrict__ lse_out, int Tq, int Tk, int H, int G, int layer_type, int window,
                        float scale_log2, int n_blocks, const int32_t *__restrict__ pos_offset,
                        const int64_t *__restrict__ seq_base, int *err,
                        const __grid_constant__ PrefillExtraMaps xm) {
  using LY = PfLayout<D>;
  constexpr int NDB = D / 64;  // 64-feature (128-byte) blocks per row
  constexpr uint32_t IDESC_S = idesc_bf16_f32(kBM, kBN, 0);
  constexpr uint32_t IDESC_O = idesc_bf16_f32(kBM, D, 1);

  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t q_full, ring_full[kRing], ring_empty[kRing];
  __shared__ uint64_t s_full[2], p_full[2][2], o_done[2], mma_drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = smem + LY::kOffQ;
  uint8_t *sRing = smem + LY::kOffRing;

  const int h = blockIdx.x;
  const int qb = n_blocks - 1 - static_cast<int>(blockIdx.y);  // longest rows first
  const int b = blockIdx.z;
  const int g = h / (H / G);
  const int q0 = qb * 2 * kBM;
  const bool is_full = layer_type == OLMO3_FULL;

  // Positions.  Query row t (0 <= t < Tq) sits at absolute position qp0 + t; key
  // row j (0 <= j < klen) is row krow0 + j of the K/V tensor maps and sits at
  // absolute position kp0 + j.
  //   kPrefillFresh   a fresh sequence: qp0 = kp0 = 0, keys are the sequence itself.
  //   kPrefillCache   a chunk at pos_offset[b] over a linear cache that already holds
  //                   it: keys are cache rows seq_base[b] + j, positions 0 .. qp0+Tq-1.
  //   kPrefillWindow  a chunk at pos_offset[b] over a gathered window: rows b*Tk + j
  //                   hold positions max(0, qp0 - window + 1) .. qp0 + Tq - 1.
  //   kPrefillRing    the same keys read in place: a key tile of positions [P, P + 128)
  //                   (P a multiple of 128, window a multiple of 128) comes from ring
  //                   rows seq_base[b] + P mod window when P + 128 <= qp0, from chunk
  //                   rows b*Tq + P - qp0 when P >= qp0, else from the bridge tile.
  // MODE is a template parameter so that the fresh-sequence kernel carries none
  // of the offset arithmetic (it costs registers in the softmax loop).
  int qp0 = 0, kp0 = 0, klen = Tk;
  int64_t krow0 = static_cast<int64_t>(b) * Tk;
  if (MODE != kPrefillFresh) qp0 = pos_offset[b];
  if (MODE == kPrefillCache) {
    krow0 = seq_base[b];
    klen = qp0 + Tq;
  } else if (MODE == kPrefillWindow) {
    kp0 = max(0, qp0 - window + 1);
    klen = qp0 + Tq - kp0;
  } else if (MODE == kPrefillRing) {
    kp0 = (max(0, qp0 - window + 1) / kBN) * kBN;  // key tiles start on 128-position boundaries
    klen = qp0 + Tq - kp0;
    krow0 = seq_base[b];
  }

  // key-tile ranges: the union [kt_lo, kt_lo + n_kt) and, per query tile w, [lo_w, hi_w] inside it
  int lo[2], hi[2];
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    const int r0 = q0 + w * kBM;
    if (r0 < Tq) {
      band_tiles(qp0 + r0, qp0 + min(r0 + kBM, Tq) - 1, kp0, klen, is_full, window, lo[w], hi[w]);
    } else {
      lo[w] = 1;
      hi[w] = 0;  // empty: every row of this tile is past the sequence
    }
  }
  const int kt_lo = hi[0] >= lo[0] ? lo[0] : lo[1];
  const int kt_hi = hi[1] >= lo[1] ? hi[1] : hi[0];
  const int n_kt = kt_hi - kt_lo + 1;
#pragma unroll
  for (int w = 0; w < 2; ++w) {
    lo[w] -= kt_lo;
    hi[w] -= kt_lo;
  }

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&ring_full[i], 1);
      mbar_init(&ring_empty[i], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&p_full[w][0], kBM);
      mbar_init(&p_full[w][1], kBM);
      mbar_init(&o_done[w], 1);
    }
    mbar_init(&mma_drain, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp >= 8) {
    regs_dec<kControlRegs>();
    if (warp == 8 && lane == 0) {
      // ------------------------------ TMA producer ------------------------------
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if (MODE == kPrefillRing) {
        prefetch_tmap(&xm.k_new);
        prefetch_tmap(&xm.v_new);
        prefetch_tmap(&xm.k_br);
        prefetch_tmap(&xm.v_br);
      }
      mbar_arrive_expect_tx(&q_full, 2 * LY::kQBytes);
#pragma unroll
      for (int w = 0; w < 2; ++w)
#pragma unroll
        for (int db = 0; db < NDB; ++db)
          tma_load_4d(sQ + w * LY::kQBytes + db * kBM * 128, &tmQ, &q_full, db * 64, h, q0 + w * kBM, b);
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < 2 * n_kt; ++i) {
        const int slot = i % kRing;
        if (i >= kRing && !mbar_wait(&ring_empty[slot], ((i / kRing) & 1) ^ 1, &s_abort)) {
          ok = false;
          break;
        }
        int krow = static_cast<int>(krow0 + static_cast<int64_t>(kt_lo + (i >> 1)) * kBN);
        const CUtensorMap *tm = (i & 1) ? &tmV : &tmK;
        if (MODE == kPrefillRing) {
          const int ts = kp0 + (kt_lo + (i >> 1)) * kBN;  // absolute position of the tile's first key
          if (ts + kBN <= qp0) {
            krow = static_cast<int>(krow0 + ts % window);
          } else if (ts >= qp0) {
            tm = (i & 1) ? &xm.v_new : &xm.k_new;
            krow = b * Tq + (ts - qp0);
          } else {
            tm = (i & 1) ? &xm.v_br : &xm.k_br;
            krow = b * kBN;
          }
        }
        mbar_arrive_expect_tx(&ring_full[slot], LY::kKVBytes);
#pragma unroll
        for (int db = 0; db < NDB; ++db)
          tma_load_3d(sRing + slot * LY::kKVBytes + db * kBN * 128, tm, &ring_full[slot], db * 64, g, krow);
        ++issued;
      }
      if (!ok) {
        s_abort = 1;
        set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
        mbar_wait(&q_full, 0, nullptr);
        for (int i = max(0, issued - kRing); i < issued; ++i)
          mbar_wait(&ring_full[i % kRing], (i / kRing) & 1, nullptr);
      }
    } else if (warp == 9) {
      // ------------------------------ MMA issuer ------------------------------
      // The whole warp runs this loop with the same values (descriptors stay in
      // uniform registers); one elected lane issues each MMA and commit.
      const uint32_t aQ = smem_u32(sQ), aR = smem_u32(sRing);
      int cnt_pv[2] = {0, 0};
      bool ok = mbar_wait_warp(&q_full, 0, &s_abort);
      auto item_ready = [&](int i) -> bool {
        return mbar_wait_warp(&ring_full[i % kRing], (i / kRing) & 1, &s_abort);
      };
      auto issue_s = [&](int w, int j) {  // S_w = Q_w K_j^T (K_j is item 2j)
        const uint64_t dq = sw128_desc(aQ + w * LY::kQBytes, 16, 1024);
        const uint64_t dk = sw128_desc(aR + ((2 * j) % kRing) * LY::kKVBytes, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off16 = ((kk >> 2) * (kBN * 128) + (kk & 3) * 32) >> 4;  // address field, 16-byte units
          umma_bf16_elect(tmem + w * kBN, dq + off16, dk + off16, IDESC_S, kk > 0);
        }
        umma_commit_elect(&s_full[w]);
      };
      auto issue_pv = [&](int w, int j) -> bool {  // O_w += P_w V_j (V_j is item 2j+1, P_w in TMEM)
        const uint64_t dv = sw128_desc(aR + ((2 * j + 1) % kRing) * LY::kKVBytes, kBN * 128, 1024);
#pragma unroll
        for (int half = 0; half < 2; ++half) {  // keys [64 half, 64 half + 64): P columns [32 half, +32)
          if (!mbar_wait_warp(&p_full[w][half], cnt_pv[w] & 1, &s_abort)) return false;
          tc_fence_after();
#pragma unroll
          for (int k4 = 0; k4 < kBN / 32; ++k4) {
            const int kk = half * (kBN / 32) + k4;
            umma_bf16_ts_elect(tmem + 256 + w * D, tmem + w * kBN + kk * 8, dv + kk * ((16 * 128) >> 4), IDESC_O,
                               (cnt_pv[w] > 0 || kk > 0));
          }
        }
        umma_commit_elect(&o_done[w]);
        ++cnt_pv[w];
        return true;
      };
      auto active = [&](int w, int j) { return lo[w] <= j && j <= hi[w]; };

      if (n_kt <= 0) ok = false;  // cannot happen for a valid call: every row sees at least its own key
      if (ok) ok = item_ready(0);
      if (ok) {
        tc_fence_after();
        if (active(0, 0)) issue_s(0, 0);
        if (active(1, 0)) issue_s(1, 0);
        umma_commit_elect(&ring_empty[0]);
      }
      for (int j = 0; ok && j < n_kt; ++j) {
        if (!(ok = item_ready(2 * j + 1))) break;  // V_j
        tc_fence_after();
        if (active(0, j) && !(ok = issue_pv(0, j))) break;
        const bool more = j + 1 < n_kt;
        if (more) {
          if (!(ok = item_ready(2 * j + 2))) break;  // K_{j+1}
          tc_fence_after();
          if (active(0, j + 1)) issue_s(0, j + 1);
        }
        if (active(1, j) && !(ok = issue_pv(1, j))) break;
        umma_commit_elect(&ring_empty[(2 * j + 1) % kRing]);  // V_j consumed by both PVs
        if (more) {
          if (active(1, j + 1)) issue_s(1, j + 1);
          umma_commit_elect(&ring_empty[(2 * j + 2) % kRing]);  // K_{j+1} consumed by both S
        }
      }
      if (!ok && lane == 0) {
        s_abort = 1;
        set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
      }
      umma_commit_elect(&mma_drain);  // every MMA issued has completed before tensor memory is freed
      mbar_wait_warp(&mma_drain, 0, nullptr);
    }
  } else {
    regs_inc<kSoftmaxRegs>();
    // -------------------------- softmax + epilogue --------------------------
    const int w = warp >> 2;            // query tile of this warpgroup
    const int row = threadIdx.x & 127;  // TMEM lane and row inside the tile
    const int r0 = q0 + w * kBM;
    const int t = r0 + row;            // query row
    const int ta0 = qp0 + r0;          // absolute position of the tile's first row
    const int ta = qp0 + t;            // absolute position of this row
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + w * kBN;
    const uint32_t tO = tmem + lane_off + 256 + w * D;
    const uint64_t scale2 = f2pack(scale_log2, scale_log2);
    float m_used = -INFINITY, lsum = 0.f;
    int cnt = 0;
    bool ok = true;
    for (int j = lo[w]; j <= hi[w]; ++j, ++cnt) {
      // S_w(j) complete also means PV_w(j-1) complete (a commit tracks every earlier
      // MMA), so O_w may be rescaled and P_w overwritten below.
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[w], cnt & 1, &s_abort))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[kBN / 32][32];
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) tmem_ld32(tS + c * 32, sr[c]);
      tmem_wait_ld();

      const int k0 = (kt_lo + j) * kBN;  // key row of the tile's first column
      const int ka0 = kp0 + k0;           // its absolute position
      const bool need_mask = !(ka0 + kBN - 1 <= ta0 && (is_full || (ta0 + kBM - 1) - ka0 < window) &&
                               (MODE == kPrefillFresh || k0 + kBN <= klen));
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c)
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int ka = ka0 + c * 32 + i;
            const bool allowed = ka <= ta && (is_full || ta - ka < window) &&
                                 (MODE == kPrefillFresh || k0 + c * 32 + i < klen);
            if (!allowed) sr[c][i] = __float_as_uint(-INFINITY);
          }
      }
      // row max of the raw scores: 8 chains of 3-input max, then a tree
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = -INFINITY;
#pragma unroll
      for (int q = 0; q < kBN / 2; ++q)
        mx[q & 7] = fmax3(mx[q & 7], __uint_as_float(sr[q >> 4][(2 * q) & 31]),
                          __uint_as_float(sr[q >> 4][(2 * q + 1) & 31]));
      const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) *
                       scale_log2;
      const bool resc = mt > m_used + kRescaleLog2;  // false while the row has seen nothing
      float alpha = 1.f;
      if (resc) {
        alpha = ex2(m_used - mt);  // 0 when m_used == -inf
        m_used = mt;
      }
      const float neg_m = (m_used == -INFINITY) ? 0.f : -m_used;
      const uint64_t negm2 = f2pack(neg_m, neg_m);
      // O_w holds PV_w(j-1) (complete: see above); rescale it before PV_w(j) adds to it.
      if (cnt > 0 && __any_sync(0xffffffffu, resc)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(tO + c * 32, orr);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
          tmem_st32(tO + c * 32, orr);
        }
      }
      // P = 2^(s*scale - m), rounded to nearest bf16 (packed two per column) for the
      // tensor core; the row sum adds the f32 values.  P goes to the first 64
      // columns of S_w in two halves of 64 keys, each announced on its own barrier,
      // so the tensor core starts on the first half while the second is computed.
      uint64_t sm2[4] = {0, 0, 0, 0};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t pk[kBN / 4];
#pragma unroll
        for (int qq = 0; qq < kBN / 4; ++qq) {
          const int q = half * (kBN / 4) + qq;
          float x0, x1;
          f2unpack(ffma2(f2pack(__uint_as_float(sr[q >> 4][(2 * q) & 31]), __uint_as_float(sr[q >> 4][(2 * q + 1) & 31])),
                         scale2, negm2),
                   x0, x1);
          const float e0 = ex2(x0), e1 = ex2(x1);
          pk[qq] = f2_to_bf2(e0, e1);
          sm2[q & 3] = fadd2(sm2[q & 3], f2pack(e0, e1));
        }
        tmem_st32(tS + half * 32, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[w][half]);
      }
      float s0, s1, s2, s3, s4, s5, s6, s7;
      f2unpack(sm2[0], s0, s1);
      f2unpack(sm2[1], s2, s3);
      f2unpack(sm2[2], s4, s5);
      f2unpack(sm2[3], s6, s7);
      lsum = lsum * alpha + (((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7)));
    }
    if (ok && cnt > 0) ok = __all_sync(0xffffffffu, mbar_wait(&o_done[w], (cnt - 1) & 1, &s_abort));
    if (!ok) {
      if (lane == 0) {
        s_abort = 1;
        set_dev_error(err, OLMO3_DEVERR_TIMEOUT);
      }
    } else if (cnt > 0) {
      tc_fence_after();
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      __nv_bfloat16 *orow = out + ((static_cast<int64_t>(b) * Tq + t) * H + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orr[32];
        tmem_ld32(tO + c * 32, orr);
        tmem_wait_ld();
        if (t < Tq) {
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
      if (lse_out != nullptr && t < Tq) {
        const float m_eff = (m_used == -INFINITY) ? 0.f : m_used;
        lse_out[(static_cast<int64_t>(b) * H + h) * Tq + t] = (m_eff + log2f(lsum)) * 0.69314718055994531f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D, int MODE>
static cudaError_t launch_pf(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV, void *out,
                             float *lse_out, int B, int Tq, int Tk, int H, int G, int layer_type, int window,
                             float scale, const int32_t *pos_offset, const int64_t *seq_base, int *err,
                             cudaStream_t stream, const PrefillExtraMaps &xm) {
  using LY = PfLayout<D>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_prefill_kernel<D, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         LY::kDynBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int n_blocks = (Tq + 2 * kBM - 1) / (2 * kBM);
  dim3 grid(H, n_blocks, B);
  attn_prefill_kernel<D, MODE><<<grid, kPfThreads, LY::kDynBytes, stream>>>(
      tmQ, tmK, tmV, static_cast<__nv_bfloat16 *>(out), lse_out, Tq, Tk, H, G, layer_type, window,
      scale * 1.4426950408889634f, n_blocks, pos_offset, seq_base, err, xm);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_pf_mode(int mode, const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV,
                                  void *out, float *lse_out, int B, int Tq, int Tk, int H, int G, int layer_type,
                                  int window, float scale, const int32_t *pos_offset, const int64_t *seq_base,
                                  int *err, cudaStream_t stream, const PrefillExtraMaps &xm) {
  switch (mode) {
    case kPrefillFresh:
      return launch_pf<D, kPrefillFresh>(tmQ, tmK, tmV, out, lse_out, B, Tq, Tk, H, G, layer_type, window, scale,
                                         pos_offset, seq_base, err, stream, xm);
    case kPrefillCache:
      return launch_pf<D, kPrefillCache>(tmQ, tmK, tmV, out, lse_out, B, Tq, Tk, H, G, layer_type, window, scale,
                                         pos_offset, seq_base, err, stream, xm);
    case kPrefillRing:
      return launch_pf<D, kPrefillRing>(tmQ, tmK, tmV, out, lse_out, B, Tq, Tk, H, G, layer_type, window, scale,
                                        pos_offset, seq_base, err, stream, xm);
    default:
      return launch_pf<D, kPrefillWindow>(tmQ, tmK, tmV, out, lse_out, B, Tq, Tk, H, G, layer_type, window, scale,
                                          pos_offset, seq_base, err, stream, xm);
  }
}

cudaError_t launch_attn_prefill(const CUtensorMap &tmQ, const CUtensorMap &tmK, const CUtensorMap &tmV, void *out,
                                float *lse_out, int B, int Tq, int Tk, int H, int G, int d, int layer_type,
                                int window, float scale, int mode, const int32_t *pos_offset,
                                const int64_t *seq_base, int *err, cudaStream_t stream,
                                const PrefillExtraMaps *extra) {
  PrefillExtraMaps xm;
  if (extra != nullptr)
    xm = *extra;
  else
    memset(&xm, 0, sizeof(xm));
  if (d == 64)
    return launch_pf_mode<64>(mode, tmQ, tmK, tmV, out, lse_out, B, Tq, Tk, H, G, layer_type, window, scale,
                              pos_offset, seq_base, err, stream, xm);
  return launch_pf_mode<128>(mode, tmQ, tmK, tmV, out, lse_out, B, Tq, Tk, H, G, layer_type, window, scale,
                             pos_offset, seq_base, err, stream, xm);
}

}  // namespace olmo3
