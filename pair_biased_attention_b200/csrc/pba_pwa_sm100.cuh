// pba_pwa_sm100.cuh -- pair weighted averaging on sm_100a.
//
// For S sequences of N tokens and H heads ("Fold-CP: A Context Parallelism
// Framework for Biomolecular Modeling", Table 1 row "Pair Weighted Avg.",
// serial time B*H*S*N^2*D, distributed as a "2D ring + tiled softmax", and
// Figure 2, which groups it with the ring attention as a softmax whose
// partials are merged):
//     w[h][i][:]    = softmax_j( b[h][i][j] + mask_j )      (bias [H][N][N])
//     o[s][i][h][:] = sum_j w[h][i][j] v[s][j][h][:]        (v [S][N][H][D])
//     out = o * sigmoid(g) (gate [S][N][H][D], optional); lse[h][i]
// The pages name the operation but print no formula; this is the plain
// reading of a softmax over the pair-bias logits alone, shared by the
// sequences.
//
// The logits do not depend on the sequences, so the softmax is taken in two
// passes, as a tiled softmax may be:
//   pba_pwa_lse_kernel    the natural log-sum-exp of every weight row over its
//                         valid keys (one warp per row, HBM-bound);
//   pba_pwa_sm100_kernel  the weights exp(b - lse), already normalised, times
//                         the values.  No running maximum, no rescale of the
//                         accumulator and no row sum are left in the tile loop.
// A work unit is (head, 128 query rows, feature tile of kPwaDF = 256 features
// = 256/D sequences), feature tile fastest so that the CTAs running at the
// same time share each bias tile through L2.  Per 128-key tile, four softmax
// warpgroups each turn 32 of the keys, for all 128 rows, into bf16 weights in
// Tensor Memory; the MMA warp then multiplies the tile into the 256 features:
// 8 x M128 N256 K16 with A = the weights from Tensor Memory and B = the value
// tile, staged as 256/D MN-major slabs of [128 keys][D] (slabs LBO apart).
//
// Warp roles:
//   warps 0-15  softmax warpgroups g = 0..3 (keys 32g .. 32g+31 of each tile;
//               the row is the Tensor Memory lane of the thread)
//   warp 16     TMA producer of the value tiles
//   warp 17     allocates Tensor Memory, issues the MMAs
//   warp 18     key-mask warp (one keep word per key pair)
//   warp 19     TMA producer of the bias tiles
// Tensor Memory: O [0,256) fp32, P0 [256,320) and P1 [320,384) (bf16 pairs,
// double-buffered by tile parity).
#pragma once

#include <cuda.h>
#include <cstdint>

#include "pba_attn_sm100.cuh"
#include "pba_ptx.cuh"

namespace pba {

constexpr int kPwaBM = 128;                          // query rows per unit
constexpr int kPwaBN = 128;                          // keys per tile
constexpr int kPwaGroups = 4;                        // softmax warpgroups
constexpr int kPwaGroupKeys = kPwaBN / kPwaGroups;   // keys of a tile per warpgroup
constexpr int kPwaDF = 256;                          // features per unit
#ifndef PBA_PWA_BIAS_STAGES
#define PBA_PWA_BIAS_STAGES 2
#endif
constexpr int kPwaBiasStages = PBA_PWA_BIAS_STAGES;  // bias tiles in flight
constexpr int kPwaSoftmaxWarps = 4 * kPwaGroups;
constexpr int kPwaThreads = 32 * (kPwaSoftmaxWarps + 4);
constexpr int kPwaWarpProducer = kPwaSoftmaxWarps;
constexpr int kPwaWarpMma = kPwaSoftmaxWarps + 1;
constexpr int kPwaWarpMask = kPwaSoftmaxWarps + 2;
constexpr int kPwaWarpBiasProducer = kPwaSoftmaxWarps + 3;
constexpr uint32_t kPwaTmemCols = 512;
constexpr uint32_t kPwaColO = 0;
constexpr uint32_t kPwaColP = kPwaDF;  // P0; P1 follows after kPwaBN / 2 columns
static_assert(kPwaColP + 2 * (kPwaBN / 2) <= kPwaTmemCols, "Tensor Memory budget");
static_assert(kPwaGroupKeys == 32, "one 16-column Tensor Memory store per warpgroup and tile");
// One key pair in PBA_PWA_EXP_EMU_EVERY takes the software exp2 on the FMA
// pipe (0: none).  With sixteen softmax warps the exp2 unit is not the limit
// here (measured at S=64, N=4096, H=8, D=32: every third pair 0.72 ms, none
// 0.70 ms), so all pairs use the unit.
#ifndef PBA_PWA_EXP_EMU_EVERY
#define PBA_PWA_EXP_EMU_EVERY 0
#endif

struct PwaParams {
  CUtensorMap tm_v;     // v [S][N][H][D] as (D, N, H, S), box {D, 128, 1, kSlabs}
  CUtensorMap tm_bias;  // bias [H][N][N] as (N keys, N rows, H, 1), box {64, 128, 1, 1}
  int32_t S, N, H;
  int32_t n_qblocks;  // ceil(N / 128)
  int32_t n_ftiles;   // ceil(S / kSlabs)
  int32_t n_units;    // H * n_qblocks * n_ftiles
  int32_t masked;     // key mask given or N not a multiple of the key tile
  int32_t mask_vec4;  // mask readable as aligned 4-byte words
  const uint8_t *mask;
  uint16_t *out;
  const uint16_t *gate;
  const float *lse;  // [H][N], written by pba_pwa_lse_kernel before this kernel runs
  int *err;
  uint64_t timeout_ns;
};

template <int D>
struct PwaLayout {
  static_assert(D == 32 || D == 64, "head dimension");
  static constexpr int kSlabs = kPwaDF / D;                // sequences per feature tile
  static constexpr int kRowBytes = D * 2;
  static constexpr int kSwizzleMode = (D == 64) ? 2 : 4;   // 128-byte / 64-byte swizzle
  static constexpr int kAtomBytes = 8 * kRowBytes;         // 8 key rows
  static constexpr int kSlabBytes = kPwaBN * kRowBytes;    // one sequence's [128 keys][D]
  static constexpr int kVBytes = kSlabs * kSlabBytes;      // 64 KB
  static constexpr int kVStages = 2;
  static constexpr int kBiasBytes = kPwaBM * kPwaBN * 2;   // 32 KB
  static constexpr int kOffV = 0;
  static constexpr int kOffBias = kOffV + kVStages * kVBytes;
  static constexpr int kOffMaskWords = kOffBias + kPwaBiasStages * kBiasBytes;
  static constexpr int kOffBar = kOffMaskWords + kPwaBiasStages * (kPwaBN / 2) * 4;
  static constexpr int kBarVFull = 0;
  static constexpr int kBarVEmpty = kBarVFull + kVStages;
  static constexpr int kBarBiasFull = kBarVEmpty + kVStages;
  static constexpr int kBarBiasReady = kBarBiasFull + kPwaBiasStages;
  static constexpr int kBarBiasEmpty = kBarBiasReady + kPwaBiasStages;
  static constexpr int kBarPFull = kBarBiasEmpty + kPwaBiasStages;  // [weight buffer]
  static constexpr int kBarPFree = kBarPFull + 2;                   // [weight buffer]
  static constexpr int kBarODone = kBarPFree + 2;
  static constexpr int kBarOFree = kBarODone + 1;
  static constexpr int kBarDrain = kBarOFree + 1;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemSlot + 4;
  static constexpr int kBytes = kOffAbort + 4;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(kOffBias % 1024 == 0 && kBiasBytes % 1024 == 0 && kVBytes % 1024 == 0, "swizzle alignment");
};

struct PwaUnit {
  int h, q0, f;
};
__device__ __forceinline__ PwaUnit decode_pwa_unit(const PwaParams &p, int u) {
  const int f = u % p.n_ftiles;
  const int r = u / p.n_ftiles;
  return PwaUnit{r / p.n_qblocks, (r % p.n_qblocks) * kPwaBM, f};
}

// lse[row] = natural log of the sum over valid keys j of exp(bias[row][j]);
// -inf for a row with no valid key.  One warp per row of N (a multiple of 8)
// bf16 logits.  Each lane keeps an online maximum and a sum over 16-key
// steps (two 8-key chunks 32 chunks apart, so the warp's loads stay
// coalesced): masked keys become bf16 -inf through keep words, the step's
// maximum is taken once, and the exponents and sums run two keys per packed
// operation.  The lanes are merged at the end.
__global__ void __launch_bounds__(256) pba_pwa_lse_kernel(const uint16_t *bias, const uint8_t *mask, int mask_vec8,
                                                          float *lse, int N, int64_t rows) {
  const int64_t row = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;  // the same for every lane of the warp
  const uint4 *src = reinterpret_cast<const uint4 *>(bias + row * int64_t(N));
  const int nch = N / 8;  // 8-key chunks
  const float2 l2e2 = make_float2(kLog2e, kLog2e);
  float m = -INFINITY;
  float2 s2 = make_float2(0.f, 0.f);
  // keep words of the 8 keys from 8 mask bytes: 0xFFFF per key that takes part
  auto keep8 = [&](int c, uint32_t (&k)[4]) {
    uint32_t mb0, mb1;
    if (mask_vec8) {
      const uint2 m2 = __ldg(reinterpret_cast<const uint2 *>(mask + 8 * c));
      mb0 = m2.x;
      mb1 = m2.y;
    } else {
      mb0 = mb1 = 0u;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        mb0 |= uint32_t(__ldg(mask + 8 * c + q)) << (8 * q);
        mb1 |= uint32_t(__ldg(mask + 8 * c + 4 + q)) << (8 * q);
      }
    }
    const uint32_t v0 = __vcmpne4(mb0, 0u), v1 = __vcmpne4(mb1, 0u);  // 0xFF per byte that is nonzero
    k[0] = __byte_perm(v0, 0u, 0x1100);
    k[1] = __byte_perm(v0, 0u, 0x3322);
    k[2] = __byte_perm(v1, 0u, 0x1100);
    k[3] = __byte_perm(v1, 0u, 0x3322);
  };
  for (int c = lane; c < nch; c += 64) {
    uint32_t w[8];
    const bool second = c + 32 < nch;
    {
      const uint4 a = __ldg(src + c);
      const uint4 b = second ? __ldg(src + c + 32) : make_uint4(0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u, 0xFF80FF80u);
      w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
      w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
    if (mask != nullptr) {
      uint32_t k[8];
      keep8(c, *reinterpret_cast<uint32_t(*)[4]>(&k[0]));
      if (second) {
        keep8(c + 32, *reinterpret_cast<uint32_t(*)[4]>(&k[4]));
      } else {
#pragma unroll
        for (int e = 4; e < 8; ++e) k[e] = 0xFFFFFFFFu;  // already -inf
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) w[e] = (w[e] & k[e]) | (~k[e] & 0xFF80FF80u);
    }
    float2 x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = make_float2(bf16lo_to_f32(w[e]), bf16hi_to_f32(w[e]));
    float cm = fmaxf(x[0].x, x[0].y);
#pragma unroll
    for (int e = 1; e < 8; ++e) cm = max3f(cm, x[e].x, x[e].y);
    if (cm > m) {
      if (m != -INFINITY) {
        const float a = ex2_approx((m - cm) * kLog2e);
        s2 = fmul2(s2, make_float2(a, a));
      }
      m = cm;
    }
    if (m != -INFINITY) {
      const float neg = -m * kLog2e;
      const float2 neg2 = make_float2(neg, neg);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float2 a = ffma2(x[e], l2e2, neg2);
        s2 = fadd2(s2, make_float2(ex2_approx(a.x), ex2_approx(a.y)));
      }
    }
  }
  float s = s2.x + s2.y;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float t2 = __shfl_xor_sync(0xffffffffu, s, o);
    const float mm = fmaxf(m, m2);
    s = ((m == -INFINITY) ? 0.f : s * ex2_approx((m - mm) * kLog2e)) +
        ((m2 == -INFINITY) ? 0.f : t2 * ex2_approx((m2 - mm) * kLog2e));
    m = mm;
  }
  if (lane == 0) lse[row] = (m == -INFINITY) ? -INFINITY : m + logf(s);
}

template <int D, bool kGate, bool kMasked>
__global__ void __launch_bounds__(kPwaThreads, 1) pba_pwa_sm100_kernel(const __grid_constant__ PwaParams p) {
  using L = PwaLayout<D>;
  constexpr int kExpEmuEvery = PBA_PWA_EXP_EMU_EVERY;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffTmemSlot);
  int *abort_flag = reinterpret_cast<int *>(smem + L::kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nt = (p.N + kPwaBN - 1) / kPwaBN;  // key tiles per unit
  const int u_begin = blockIdx.x, u_step = gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::kVStages; ++s) {
      mbar_init(&bars[L::kBarVFull + s], 1);
      mbar_init(&bars[L::kBarVEmpty + s], 1);
    }
    for (int t = 0; t < kPwaBiasStages; ++t) {
      mbar_init(&bars[L::kBarBiasFull + t], 1);
      mbar_init(&bars[L::kBarBiasReady + t], 32);
      mbar_init(&bars[L::kBarBiasEmpty + t], kPwaGroups * kPwaBM);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[L::kBarPFull + b], kPwaGroups * kPwaBM);
      mbar_init(&bars[L::kBarPFree + b], 1);
    }
    mbar_init(&bars[L::kBarODone], 1);
    mbar_init(&bars[L::kBarOFree], kPwaGroups * kPwaBM);
    mbar_init(&bars[L::kBarDrain], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kPwaWarpMma) {
    tmem_alloc(tmem_slot, kPwaTmemCols);
    tmem_relinquish();
  }
  if (warp == kPwaWarpProducer && lane == 0) tma_prefetch_desc(&p.tm_v);
  if (warp == kPwaWarpBiasProducer && lane == 0) tma_prefetch_desc(&p.tm_bias);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.err, p.timeout_ns};
  WaitCtl wc_drain = wc;  // clean-up waits: ignore the abort word, keep the time limit
  int drain_abort = 0;
  wc_drain.abort_flag = &drain_abort;

  if (warp == kPwaWarpProducer) {
    // ================================================================ value tiles
    if (lane == 0) {
      const uint64_t pol_keep = l2_policy_evict_last();  // re-read by the other query blocks
      bool ok = true;
      int vc = 0;
      for (int u = u_begin; u < p.n_units && ok; u += u_step) {
        const PwaUnit un = decode_pwa_unit(p, u);
        for (int j = 0; j < nt && ok; ++j) {
          const int s = vc % L::kVStages;
          if (vc >= L::kVStages) ok = mbar_wait(&bars[L::kBarVEmpty + s], ((vc / L::kVStages) - 1) & 1, wc);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars[L::kBarVFull + s], L::kVBytes);
          // [kSlabs sequences][128 keys][D]; sequences past S read as zero
          tma_load_4d(smem + L::kOffV + s * L::kVBytes, &p.tm_v, &bars[L::kBarVFull + s], 0, j * kPwaBN, un.h,
                      un.f * L::kSlabs, pol_keep);
          ++vc;
        }
      }
      if (!ok)
        for (int s = 0; s < L::kVStages; ++s) {
          const int a = (vc - s + L::kVStages - 1) / L::kVStages;
          if (a > 0) mbar_wait(&bars[L::kBarVFull + s], (a - 1) & 1, wc_drain);
        }
    }
  } else if (warp == kPwaWarpBiasProducer) {
    // ================================================================ bias tiles
    if (lane == 0) {
      const uint64_t pol = l2_policy_evict_last();  // shared by the feature tiles of a row block
      bool ok = true;
      int gt = 0;  // bias tiles issued (all units)
      for (int u = u_begin; u < p.n_units && ok; u += u_step) {
        const PwaUnit un = decode_pwa_unit(p, u);
        for (int j = 0; j < nt && ok; ++j) {
          const int t = gt % kPwaBiasStages;
          if (gt >= kPwaBiasStages)
            ok = mbar_wait(&bars[L::kBarBiasEmpty + t], ((gt / kPwaBiasStages) - 1) & 1, wc);
          if (!ok) break;
          uint8_t *dst = smem + L::kOffBias + t * L::kBiasBytes;
          // [128 rows][128 keys] as two 64-key boxes, 128-byte swizzle
          mbar_arrive_expect_tx(&bars[L::kBarBiasFull + t], L::kBiasBytes);
          tma_load_4d(dst, &p.tm_bias, &bars[L::kBarBiasFull + t], j * kPwaBN, un.q0, un.h, 0, pol);
          tma_load_4d(dst + L::kBiasBytes / 2, &p.tm_bias, &bars[L::kBarBiasFull + t], j * kPwaBN + 64, un.q0, un.h,
                      0, pol);
          ++gt;
        }
      }
      if (!ok)
        for (int t = 0; t < kPwaBiasStages; ++t) {
          const int a = (gt - t + kPwaBiasStages - 1) / kPwaBiasStages;
          if (a > 0) mbar_wait(&bars[L::kBarBiasFull + t], (a - 1) & 1, wc_drain);
        }
    }
  } else if (warp == kPwaWarpMma) {
    // ================================================================ MMAs
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kPwaBM, kPwaDF, true);  // V is MN-major
      const uint32_t sV = smem_u32(smem + L::kOffV);
      constexpr uint32_t kDescHi = smem_desc_hi(L::kAtomBytes, L::kSwizzleMode);
      bool ok = true;
      int gt = 0, uc = 0;  // key tiles (all units), units
      for (int u = u_begin; u < p.n_units && ok; u += u_step, ++uc) {
        for (int j = 0; j < nt && ok; ++j, ++gt) {
          const int s = gt % L::kVStages;
          const int b = gt & 1;  // weight buffer
          ok = mbar_wait(&bars[L::kBarVFull + s], (gt / L::kVStages) & 1, wc);
          if (ok) ok = mbar_wait(&bars[L::kBarPFull + b], (gt >> 1) & 1, wc);
          // the first product of a unit overwrites O: the epilogue must have read it
          if (ok && j == 0 && uc > 0) ok = mbar_wait(&bars[L::kBarOFree], (uc - 1) & 1, wc);
          if (!ok) break;
          tc_fence_after_sync();
          // B: keys 16 kk .. 16 kk + 15 of every slab (slabs LBO apart)
          const uint32_t v_lo = smem_desc_lo(sV + s * L::kVBytes, L::kSlabBytes);
          const uint32_t a_tmem = tmem + kPwaColP + b * (kPwaBN / 2);
#pragma unroll 4
          for (int kk = 0; kk < kPwaBN / 16; ++kk)
            mma_bf16_ts(tmem + kPwaColO, a_tmem + kk * 8, desc_join(v_lo + kk * (16 * L::kRowBytes / 16), kDescHi),
                        idesc, (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&bars[L::kBarPFree + b]);
          tc_commit(&bars[L::kBarVEmpty + s]);
          if (j + 1 == nt) tc_commit(&bars[L::kBarODone]);
        }
      }
      tc_commit(&bars[L::kBarDrain]);
      mbar_wait(&bars[L::kBarDrain], 0, wc_drain);
    }
  } else if (warp == kPwaWarpMask) {
    // ================================================================ key-mask warp
    // One keep word per key pair beside each bias slot (0xFFFF per kept
    // half); lane l owns keys 4l..4l+3.  Keys past N are masked.
    bool ok = kMasked;
    int gt = 0;
    for (int u = u_begin; u < p.n_units && ok; u += u_step) {
      auto load_word = [&](int j) -> uint32_t {  // byte e nonzero = key 4*lane+e takes part
        const int key0 = j * kPwaBN + 4 * lane;
        if (p.mask == nullptr) return 0x01010101u;
        if (p.mask_vec4 && key0 + 3 < p.N) return __ldg(reinterpret_cast<const uint32_t *>(p.mask + key0));
        uint32_t wv = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (key0 + e < p.N) wv |= uint32_t(__ldg(p.mask + key0 + e) != 0) << (8 * e);
        return wv;
      };
      uint32_t next_word = load_word(0);
      for (int j = 0; j < nt && ok; ++j, ++gt) {
        const uint32_t word = next_word;
        if (j + 1 < nt) next_word = load_word(j + 1);
        const int key0 = j * kPwaBN + 4 * lane;
        uint32_t inv = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (key0 + e >= p.N || ((word >> (8 * e)) & 0xFFu) == 0) inv |= 1u << e;
        const uint2 keep = make_uint2(((inv & 1u) ? 0u : 0x0000FFFFu) | ((inv & 2u) ? 0u : 0xFFFF0000u),
                                      ((inv & 4u) ? 0u : 0x0000FFFFu) | ((inv & 8u) ? 0u : 0xFFFF0000u));
        const int t = gt % kPwaBiasStages;
        ok = mbar_wait<false>(&bars[L::kBarBiasFull + t], (gt / kPwaBiasStages) & 1, wc);
        if (!ok) break;
        reinterpret_cast<uint2 *>(smem + L::kOffMaskWords + t * (kPwaBN / 2) * 4)[lane] = keep;
        __syncwarp();
        mbar_arrive(&bars[L::kBarBiasReady + t]);
      }
    }
  } else {
    // ================================================================ softmax warpgroups
    const int g = warp >> 2;            // keys kPwaGroupKeys*g .. +kPwaGroupKeys-1 of each tile
    const int t = threadIdx.x & 127;    // row inside the unit
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tP = tmem + lane_base + kPwaColP + g * (kPwaGroupKeys / 2);
    const uint32_t tO = tmem + lane_base + kPwaColO + g * (kPwaDF / kPwaGroups);
    const float2 l2e2 = make_float2(kLog2e, kLog2e);
    // this warpgroup's keys: 64 bytes of the row's 128-byte swizzled box row
    const int box = (g * kPwaGroupKeys) / 64, chunk0 = ((g * kPwaGroupKeys) % 64) / 8;
    bool ok = true;
    int gt = 0, uc = 0;
    // the row's lse, loaded one unit ahead
    auto load_lse = [&](int uu) -> float {
      if (uu >= p.n_units) return -INFINITY;
      const PwaUnit nu = decode_pwa_unit(p, uu);
      return nu.q0 + t < p.N ? p.lse[int64_t(nu.h) * p.N + nu.q0 + t] : -INFINITY;
    };
    float next_lse = load_lse(u_begin);
    for (int u = u_begin; u < p.n_units && ok; u += u_step, ++uc) {
      const PwaUnit un = decode_pwa_unit(p, u);
      const int row = un.q0 + t;
      const bool live = row < p.N;
      // -lse*log2(e) of the row; a row with no valid key has lse = -inf and
      // -inf logits only, which the finite stand-in 0 keeps at weight 0
      const float lse_r = next_lse;
      next_lse = load_lse(u + u_step);
      const float neg = (lse_r == -INFINITY) ? 0.f : -lse_r * kLog2e;
      const float2 neg2 = make_float2(neg, neg);
      for (int j = 0; j < nt; ++j, ++gt) {
        const int slot = gt % kPwaBiasStages;
        ok = mbar_wait<false>(&bars[(kMasked ? L::kBarBiasReady : L::kBarBiasFull) + slot],
                              (gt / kPwaBiasStages) & 1, wc);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        const uint8_t *tile = smem + L::kOffBias + slot * L::kBiasBytes + box * (L::kBiasBytes / 2) + t * 128;
        const uint4 *kw = reinterpret_cast<const uint4 *>(smem + L::kOffMaskWords + slot * (kPwaBN / 2) * 4) +
                          g * (kPwaGroupKeys / 8);
        uint32_t pk[kPwaGroupKeys / 2];
#pragma unroll
        for (int c = 0; c < kPwaGroupKeys / 8; ++c) {
          const uint4 bv = *reinterpret_cast<const uint4 *>(tile + (((chunk0 + c) ^ (t & 7)) << 4));
          uint32_t wv[4] = {bv.x, bv.y, bv.z, bv.w};
          if (kMasked) {
            // masked halves become bf16 -inf: (w & keep) | (~keep & -inf)
            const uint4 kv = kw[c];
            const uint32_t keep[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) wv[e] = (wv[e] & keep[e]) | (~keep[e] & 0xFF80FF80u);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = c * 4 + e;  // key pair of this warpgroup
            const float2 a = ffma2(make_float2(bf16lo_to_f32(wv[e]), bf16hi_to_f32(wv[e])), l2e2, neg2);
            // every kExpEmuEvery-th key pair takes the software exp2 on the FMA pipe
            const float2 pv = (kExpEmuEvery > 0 && i % kExpEmuEvery == kExpEmuEvery - 1)
                                  ? exp2_poly2(a)
                                  : make_float2(ex2_approx(a.x), ex2_approx(a.y));
            pk[i] = pack_bf16x2(pv.x, pv.y);
          }
        }
        // the weight buffer of this tile was last read by the products of tile gt - 2
        const int b = gt & 1;
        if (gt >= 2) {
          ok = mbar_wait<false>(&bars[L::kBarPFree + b], ((gt >> 1) - 1) & 1, wc);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after_sync();
        }
        tmem_st16(tP + b * (kPwaBN / 2), pk);
        // The bias slot is released only after the store above, which takes
        // every weight of the tile and so cannot issue before all of the
        // slot's shared-memory loads have returned; released any earlier, the
        // next TMA write into the slot could overtake a load still in flight.
        mbar_arrive(&bars[L::kBarBiasEmpty + slot]);
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(&bars[L::kBarPFull + b]);
      }
      if (!ok) break;

      // -------------------------------------------------------------- epilogue
      // this warpgroup's 64 columns of O, as two 32-column chunks
      constexpr int kChunks = kPwaDF / kPwaGroups / 32;
      uint4 gpre[kGate ? kChunks * 4 : 1];
      if (kGate) {
        // the gate of both chunks is loaded before the wait for the products
#pragma unroll
        for (int cc = 0; cc < kChunks; ++cc) {
          const int c = g * (kPwaDF / kPwaGroups) + cc * 32;
          const int seq = un.f * L::kSlabs + c / D;
          if (live && seq < p.S) {
            const uint4 *gp = reinterpret_cast<const uint4 *>(p.gate + ((int64_t(seq) * p.N + row) * p.H + un.h) * D +
                                                              (c % D));
#pragma unroll
            for (int q = 0; q < 4; ++q) gpre[cc * 4 + q] = gp[q];
          }
        }
      }
      ok = mbar_wait<false>(&bars[L::kBarODone], uc & 1, wc);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after_sync();
#pragma unroll
      for (int cc = 0; cc < kChunks; ++cc) {
        uint32_t r[32];
        tmem_ld32(tO + cc * 32, r);
        tmem_wait_ld();
        reg_fence(r);
        if (cc + 1 == kChunks) {
          tc_fence_before_sync();
          mbar_arrive(&bars[L::kBarOFree]);  // O is in registers
        }
        const int c = g * (kPwaDF / kPwaGroups) + cc * 32;
        const int seq = un.f * L::kSlabs + c / D;
        if (live && seq < p.S) {
          const int64_t at = ((int64_t(seq) * p.N + row) * p.H + un.h) * D + (c % D);
          uint32_t ow[16];
          if (kGate) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 gv = gpre[cc * 4 + q];
              const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float o0 = __uint_as_float(r[8 * q + 2 * e]), o1 = __uint_as_float(r[8 * q + 2 * e + 1]);
                ow[4 * q + e] = pack_bf16x2(o0 * sigmoid_fast(bf16lo_to_f32(gw[e])),
                                            o1 * sigmoid_fast(bf16hi_to_f32(gw[e])));
              }
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) ow[e] = pack_bf16x2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
          }
          uint4 *op = reinterpret_cast<uint4 *>(p.out + at);
#pragma unroll
          for (int q = 0; q < 4; ++q) op[q] = make_uint4(ow[4 * q], ow[4 * q + 1], ow[4 * q + 2], ow[4 * q + 3]);
        }
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == kPwaWarpMma) tmem_dealloc(tmem, kPwaTmemCols);
}

}  // namespace pba
