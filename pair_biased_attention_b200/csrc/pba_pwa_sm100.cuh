// pba_pwa_sm100.cuh -- pair weighted averaging on sm_100a.
//
// For S sequences of N tokens and H heads ("Fold-CP: A Context Parallelism
// Framework for Biomolecular Modeling", Table 1 row "Pair Weighted Avg.",
// serial time B*H*S*N^2*D, distributed as a "2D ring + tiled softmax", and
// Figure 2, which groups it with the ring attention as a softmax whose
// partials are merged):
//     w[h][i][:]    = softmax_j( b[h][i][j] + mask_j )      (bias [H][N][N])
//     o[s][i][h][:] = sum_j w[h][i][j] v[s][j][h][:]        (v [S][N][H][D])
//     out = o * sigmoid(g) (gate [S][N][H][D], optional); lse[h][i] (optional)
// The pages name the operation but print no formula; this is the plain
// reading of a softmax over the pair-bias logits alone, shared by the
// sequences.
//
// The weights do not depend on s, so a CTA computes them once per key tile
// and multiplies them into a feature tile of kSlabs sequences at once: one
// M128 N(kSlabs*D = 192) K16 MMA per 16 keys, with the value tile staged as
// kSlabs MN-major slabs of [128 keys][D] (slabs LBO apart).  A work unit is
// (head, 256 query rows, feature tile), feature tile fastest so that the CTAs
// running at the same time share each bias tile through L2.
//
// Warp roles and rings follow the attention kernel (pba_attn_sm100.cuh):
//   warps 0-3 / 4-7  softmax warpgroups of query tiles 0 / 1 (row = thread)
//   warp 8           TMA producer of the value tiles
//   warp 9           allocates Tensor Memory, issues the P V MMAs
//   warp 10          key-mask warp (one keep word per key pair)
//   warp 11          TMA producer of the bias tiles
// Tensor Memory: P0 [0,64) P1 [64,128) (bf16 pairs), O0 [128,320) O1 [320,512).
#pragma once

#include <cuda.h>
#include <cstdint>

#include "pba_attn_sm100.cuh"
#include "pba_ptx.cuh"

namespace pba {

// Tile shape, warp roles and register split of this kernel (the same
// arrangement as the attention kernel's two-warpgroup form).
constexpr int kPwaBM = 128;           // query rows per tile
constexpr int kPwaBN = 128;           // keys per tile
constexpr int kPwaQTiles = 2;         // query tiles per unit
constexpr int kPwaBiasStages = 2;
constexpr int kPwaThreads = 384;      // 12 warps
constexpr int kPwaWarpProducer = 8;
constexpr int kPwaWarpMma = 9;
constexpr int kPwaWarpBiasProducer = 11;
constexpr uint32_t kPwaTmemCols = 512;
constexpr int kPwaRegsSoftmax = 224;
constexpr int kPwaRegsOther = 56;
constexpr int kPwaRegSplitTotal = 256 * kPwaRegsSoftmax + 128 * kPwaRegsOther;

struct PwaParams {
  CUtensorMap tm_v;     // v [S][N][H][D] as (D, N, H, S), box {D, 128, 1, kSlabs}
  CUtensorMap tm_bias;  // bias [H][N][N] as (N keys, N rows, H, 1), box {64, 128, 1, 1}
  int32_t S, N, H;
  int32_t n_qblocks;  // ceil(N / 256)
  int32_t n_ftiles;   // ceil(S / kSlabs)
  int32_t n_units;    // H * n_qblocks * n_ftiles
  int32_t masked;     // key mask given or N not a multiple of the key tile
  int32_t mask_vec4;  // mask readable as aligned 4-byte words
  const uint8_t *mask;
  uint16_t *out;
  const uint16_t *gate;
  float *lse;
  int *err;
  uint64_t timeout_ns;
};

template <int D>
struct PwaLayout {
  static_assert(D == 32 || D == 64, "head dimension");
  static constexpr int kSlabs = 192 / D;       // sequences per feature tile
  static constexpr int kDF = kSlabs * D;       // 192 features
  static constexpr int kRowBytes = D * 2;
  static constexpr int kSwizzleMode = (D == 64) ? 2 : 4;  // 128-byte / 64-byte swizzle
  static constexpr int kAtomBytes = 8 * kRowBytes;        // 8 key rows
  static constexpr int kSlabBytes = kPwaBN * kRowBytes;      // one sequence's [128 keys][D]
  static constexpr int kVBytes = kSlabs * kSlabBytes;
  static constexpr int kVStages = 2;
  static constexpr int kBiasBytes = kPwaBM * kPwaBN * 2;
  static constexpr int kBiasSlots = kPwaQTiles * kPwaBiasStages;
  static constexpr int kOffV = 0;
  static constexpr int kOffBias = kOffV + kVStages * kVBytes;
  static constexpr int kOffMaskWords = kOffBias + kBiasSlots * kBiasBytes;
  static constexpr int kOffBar = kOffMaskWords + kBiasSlots * (kPwaBN / 2) * 4;
  static constexpr int kBarVFull = 0;
  static constexpr int kBarVEmpty = kBarVFull + kVStages;
  static constexpr int kBarBiasFull = kBarVEmpty + kVStages;
  static constexpr int kBarBiasReady = kBarBiasFull + kBiasSlots;
  static constexpr int kBarBiasEmpty = kBarBiasReady + kBiasSlots;
  static constexpr int kBarPFull = kBarBiasEmpty + kBiasSlots;  // [w]
  static constexpr int kBarODone = kBarPFull + kPwaQTiles;
  static constexpr int kBarOFree = kBarODone + kPwaQTiles;
  static constexpr int kBarDrain = kBarOFree + kPwaQTiles;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemSlot + 4;
  static constexpr int kBytes = kOffAbort + 4;
  static constexpr int kSmemAlloc = kBytes + 1024;
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
  static_assert(2 * 64 + kPwaQTiles * kDF <= 512, "Tensor Memory budget");
};

struct PwaUnit {
  int h, q0, f;
};
__device__ __forceinline__ PwaUnit decode_pwa_unit(const PwaParams &p, int u) {
  const int f = u % p.n_ftiles;
  const int r = u / p.n_ftiles;
  return PwaUnit{r / p.n_qblocks, (r % p.n_qblocks) * (kPwaQTiles * kPwaBM), f};
}

template <int D, bool kGate, bool kMasked>
__global__ void __launch_bounds__(kPwaThreads, 1) pba_pwa_sm100_kernel(const __grid_constant__ PwaParams p) {
  using L = PwaLayout<D>;
  constexpr int kExpEmuEvery = (D == 32) ? PBA_EXP_EMU_EVERY_D32 : PBA_EXP_EMU_EVERY_D64;
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
    for (int i = 0; i < L::kBiasSlots; ++i) {
      mbar_init(&bars[L::kBarBiasFull + i], 1);
      mbar_init(&bars[L::kBarBiasReady + i], 32);
      mbar_init(&bars[L::kBarBiasEmpty + i], kPwaBM);
    }
    for (int w = 0; w < kPwaQTiles; ++w) {
      mbar_init(&bars[L::kBarPFull + w], kPwaBM);
      mbar_init(&bars[L::kBarODone + w], 1);
      mbar_init(&bars[L::kBarOFree + w], kPwaBM);
    }
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

  if (warp >= 8) {
    setmaxnreg_dec<kPwaRegsOther>();
    if (warp == kPwaWarpProducer) {
      // ============================================================== value tiles
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
      // ============================================================== bias tiles
      if (lane == 0) {
        const uint64_t pol = l2_policy_evict_last();  // shared by the feature tiles of a row block
        bool ok = true;
        int gt = 0, issued = 0;
        for (int u = u_begin; u < p.n_units && ok; u += u_step) {
          const PwaUnit un = decode_pwa_unit(p, u);
          for (int j = 0; j < nt && ok; ++j, ++gt) {
            const int t = gt % kPwaBiasStages;
            for (int w = 0; w < kPwaQTiles && ok; ++w) {
              const int slot = w * kPwaBiasStages + t;
              if (gt >= kPwaBiasStages)
                ok = mbar_wait(&bars[L::kBarBiasEmpty + slot], ((gt / kPwaBiasStages) - 1) & 1, wc);
              if (!ok) break;
              uint8_t *dst = smem + L::kOffBias + slot * L::kBiasBytes;
              mbar_arrive_expect_tx(&bars[L::kBarBiasFull + slot], L::kBiasBytes);
              tma_load_4d(dst, &p.tm_bias, &bars[L::kBarBiasFull + slot], j * kPwaBN, un.q0 + w * kPwaBM, un.h, 0, pol);
              tma_load_4d(dst + L::kBiasBytes / 2, &p.tm_bias, &bars[L::kBarBiasFull + slot], j * kPwaBN + 64,
                          un.q0 + w * kPwaBM, un.h, 0, pol);
              ++issued;
            }
          }
        }
        if (!ok)
          for (int w = 0; w < kPwaQTiles; ++w)
            for (int t = 0; t < kPwaBiasStages; ++t) {
              const int n_w = issued / kPwaQTiles + (w < issued % kPwaQTiles ? 1 : 0);
              const int a = (n_w - t + kPwaBiasStages - 1) / kPwaBiasStages;
              if (a > 0) mbar_wait(&bars[L::kBarBiasFull + w * kPwaBiasStages + t], (a - 1) & 1, wc_drain);
            }
      }
    } else if (warp == kPwaWarpMma) {
      // ============================================================== P V MMAs
      if (lane == 0) {
        const uint32_t idesc = idesc_bf16_f32(kPwaBM, L::kDF, true);  // V is MN-major
        const uint32_t sV = smem_u32(smem + L::kOffV);
        constexpr uint32_t kDescHi = smem_desc_hi(L::kAtomBytes, L::kSwizzleMode);
        bool ok = true;
        int vc = 0, gp = 0, uc = 0;
        for (int u = u_begin; u < p.n_units && ok; u += u_step, ++uc) {
          for (int j = 0; j < nt && ok; ++j) {
            const int s = vc % L::kVStages;
            ok = mbar_wait(&bars[L::kBarVFull + s], (vc / L::kVStages) & 1, wc);
            for (int w = 0; w < kPwaQTiles && ok; ++w) {
              if (!(ok = mbar_wait(&bars[L::kBarPFull + w], gp & 1, wc))) break;
              // the first P V of a unit overwrites O: the epilogue must have read it
              if (j == 0 && uc > 0 && !(ok = mbar_wait(&bars[L::kBarOFree + w], (uc - 1) & 1, wc))) break;
              tc_fence_after_sync();
              const uint32_t d_tmem = tmem + 128 + w * L::kDF;
              const uint32_t a_tmem = tmem + w * 64;
              // B: keys 16 kk .. 16 kk + 15 of every slab (slabs LBO apart)
              const uint32_t v_lo = smem_desc_lo(sV + s * L::kVBytes, L::kSlabBytes);
#pragma unroll 4
              for (int kk = 0; kk < kPwaBN / 16; ++kk)
                mma_bf16_ts(d_tmem, a_tmem + kk * 8, desc_join(v_lo + kk * (16 * L::kRowBytes / 16), kDescHi), idesc,
                            (j > 0 || kk > 0) ? 1u : 0u);
              tc_commit(&bars[L::kBarODone + w]);
            }
            if (!ok) break;
            tc_commit(&bars[L::kBarVEmpty + s]);
            ++vc;
            ++gp;
          }
        }
        tc_commit(&bars[L::kBarDrain]);
        mbar_wait(&bars[L::kBarDrain], 0, wc_drain);
      }
    } else {
      // ============================================================== key-mask warp
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
          for (int w = 0; w < kPwaQTiles && ok; ++w) {
            const int slot = w * kPwaBiasStages + t;
            ok = mbar_wait<false>(&bars[L::kBarBiasFull + slot], (gt / kPwaBiasStages) & 1, wc);
            if (!ok) break;
            reinterpret_cast<uint2 *>(smem + L::kOffMaskWords + slot * (kPwaBN / 2) * 4)[lane] = keep;
            __syncwarp();
            mbar_arrive(&bars[L::kBarBiasReady + slot]);
          }
        }
      }
    }
  } else {
    // ================================================================ softmax warpgroups
    setmaxnreg_inc<kPwaRegsSoftmax>();
    const int w = warp >> 2;
    const int t = threadIdx.x & 127;
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tP = tmem + lane_base + w * 64;
    const uint32_t tO = tmem + lane_base + 128 + w * L::kDF;
    bool ok = true;
    int gt = 0;
    for (int u = u_begin; u < p.n_units && ok; u += u_step) {
      float m_cur = -INFINITY;  // maximum used for P and l
      float l = 0.f;
      for (int j = 0; j < nt && ok; ++j, ++gt) {
        const int slot = w * kPwaBiasStages + (gt % kPwaBiasStages);
        ok = mbar_wait<false>(&bars[(kMasked ? L::kBarBiasReady : L::kBarBiasFull) + slot], (gt / kPwaBiasStages) & 1,
                              wc);
        if (!ok) break;
        const uint8_t *tile = smem + L::kOffBias + slot * L::kBiasBytes;
        // the logits of this row's 128 keys (masked ones -inf)
        float2 x[kPwaBN / 2];
#pragma unroll
        for (int c8 = 0; c8 < kPwaBN / 8; ++c8) {
          const int box = c8 >> 3, chunk = c8 & 7;
          const uint4 bv =
              *reinterpret_cast<const uint4 *>(tile + box * (L::kBiasBytes / 2) + t * 128 + ((chunk ^ (t & 7)) << 4));
          uint32_t wv[4] = {bv.x, bv.y, bv.z, bv.w};
          if (kMasked) {
            const uint4 kv = reinterpret_cast<const uint4 *>(smem + L::kOffMaskWords + slot * (kPwaBN / 2) * 4)[c8];
            const uint32_t keep[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) wv[e] = (wv[e] & keep[e]) | (~keep[e] & 0xFF80FF80u);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) x[c8 * 4 + e] = make_float2(bf16lo_to_f32(wv[e]), bf16hi_to_f32(wv[e]));
        }
        mbar_arrive(&bars[L::kBarBiasEmpty + slot]);

        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmaxf(x[i].x, x[i].y);
#pragma unroll
        for (int i = 8; i < kPwaBN / 2; ++i) m8[i & 7] = max3f(m8[i & 7], x[i].x, x[i].y);
        const float mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        const bool need = mx > m_cur + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = (m_cur == -INFINITY) ? 0.f : ex2_approx((m_cur - mx) * kLog2e);
          l *= alpha;
          m_cur = mx;
        }
        const float neg_m = (m_cur == -INFINITY) ? 0.f : -m_cur * kLog2e;
        const float2 l2e2 = make_float2(kLog2e, kLog2e), negm2 = make_float2(neg_m, neg_m);
        uint32_t pk[kPwaBN / 2];
        float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int i = 0; i < kPwaBN / 2; ++i) {
          const float2 a = ffma2(x[i], l2e2, negm2);
          const float2 pv = (kExpEmuEvery > 0 && i % kExpEmuEvery == kExpEmuEvery - 1)
                                ? exp2_poly2(a)
                                : make_float2(ex2_approx(a.x), ex2_approx(a.y));
          ls[i & 3] = fadd2(ls[i & 3], pv);
          pk[i] = pack_bf16x2(pv.x, pv.y);
        }
        const float2 lsum2 = fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3]));
        l += lsum2.x + lsum2.y;

        // P(j) overwrites the P buffer that P V(j-1) read
        if (gt > 0) {
          ok = mbar_wait<false>(&bars[L::kBarODone + w], (gt - 1) & 1, wc);
          if (!ok) break;
          tc_fence_after_sync();
          if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
            for (int c = 0; c < L::kDF; c += 32) {
              uint32_t o[32];
              tmem_ld32(tO + c, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tO + c, o);
            }
          }
        }
#pragma unroll
        for (int c = 0; c < kPwaBN / 2; c += 32) tmem_st32(tP + c, *reinterpret_cast<uint32_t(*)[32]>(&pk[c]));
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(&bars[L::kBarPFull + w]);
      }

      // -------------------------------------------------------------- epilogue
      if (ok) ok = mbar_wait<false>(&bars[L::kBarODone + w], (gt - 1) & 1, wc);
      if (!ok) break;
      tc_fence_after_sync();
      const PwaUnit un = decode_pwa_unit(p, u);
      const int row = un.q0 + w * kPwaBM + t;
      const bool live = row < p.N;
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < L::kDF; c += 32) {
        uint32_t r[32];
        tmem_ld32(tO + c, r);
        tmem_wait_ld();
        if (c + 32 == L::kDF) {
          tc_fence_before_sync();
          mbar_arrive(&bars[L::kBarOFree + w]);  // O is in registers
        }
        const int seq = un.f * L::kSlabs + c / D;
        if (live && seq < p.S) {
          const int64_t at = ((int64_t(seq) * p.N + row) * p.H + un.h) * D + (c % D);
          uint32_t pk[16];
          if (kGate) {
            const uint4 *gp = reinterpret_cast<const uint4 *>(p.gate + at);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 gv = gp[q];
              const uint32_t gw[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float o0 = __uint_as_float(r[8 * q + 2 * e]) * inv_l, o1 = __uint_as_float(r[8 * q + 2 * e + 1]) * inv_l;
                pk[4 * q + e] = pack_bf16x2(o0 / (1.f + __expf(-bf16lo_to_f32(gw[e]))),
                                            o1 / (1.f + __expf(-bf16hi_to_f32(gw[e]))));
              }
            }
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
          }
          uint4 *op = reinterpret_cast<uint4 *>(p.out + at);
#pragma unroll
          for (int q = 0; q < 4; ++q) op[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
        }
      }
      if (live && un.f == 0 && p.lse != nullptr)
        p.lse[int64_t(un.h) * p.N + row] = (l > 0.f) ? m_cur + logf(l) : -INFINITY;
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == kPwaWarpMma) tmem_dealloc(tmem, kPwaTmemCols);
}

}  // namespace pba
