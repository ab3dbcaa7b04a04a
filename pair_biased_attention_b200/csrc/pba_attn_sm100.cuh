// pba_attn_sm100.cuh -- pair-biased attention on the sm_100a tensor cores.
//
// Computes, per (batch b, head h) and query row i,
//     O_i = sum_j softmax_j( tau q_i.k_j + b_ij ) v_j
// over the keys of one call, as in "Fold-CP: A Context Parallelism Framework
// for Biomolecular Modeling" (Table 1 "Attn Pair Bias", Figure 2(c):
// attention of the local queries against a key/value/pair-bias block).  The
// softmax is accumulated online, tile by tile (the method of "Online
// normalizer calculation for softmax", listed under "Builds on" on the
// "Design-CP" page), so the same main loop serves a full pass (epilogue:
// bf16 O and the log-sum-exp) and one ring step (epilogue: the fp32 partial
// O_p, m_p, l_p that the tiled-softmax merge combines).  Triangle attention
// runs the same loop with the pair-tensor strides in the tile descriptors.
//
// Persistent: one CTA per SM walks the work units u = blockIdx.x,
// blockIdx.x + gridDim.x, ...; a unit is two 128-row query tiles of one
// (b, h).  Every ring and barrier phase runs on across units, so the next
// unit's Q, K, V and bias loads overlap the current unit's last tiles and
// epilogue.
//   warps 0-3   softmax warpgroup for query tile 0 (thread t owns row t)
//   warps 4-7   softmax warpgroup for query tile 1
//   warp 8      TMA producer of Q (per unit) and of K, V per 128-key tile
//   warp 9      allocates Tensor Memory and issues every tcgen05.mma
//   warp 10     key-mask warp (mask words, or -inf rows of a transposed tile)
//   warp 11     TMA producer of the two bias tiles per 128-key tile
// Tensor Memory (512 columns x 128 lanes of fp32):
//   [0,128) S0   [128,256) S1   [256,320) P0   [320,384) P1
//   [384,384+D) O0   [448,448+D) O1
// S_w = Q_w K^T (fp32), P_w = bf16 probabilities (two per column), O_w the
// running output.  MMA issue order per key tile j: S0(j+1), P0 V(j), S1(j+1),
// P1 V(j), so the next score tile is computed while the softmax warps work
// on this one.
#pragma once

#include <cuda.h>

#include "pba_ptx.cuh"

namespace pba {

constexpr int kBM = 128;          // query rows per tile (one TMEM lane each)
constexpr int kBN = 128;          // keys per tile
constexpr int kQTiles = 2;        // query tiles per unit
constexpr int kBiasStages = 2;    // bias ring depth per softmax warpgroup
constexpr int kAttnThreads = 384; // 12 warps
constexpr int kWarpProducer = 8;  // Q, K, V
constexpr int kWarpMma = 9;
constexpr int kWarpMask = 10;
constexpr int kWarpBiasProducer = 11;
constexpr uint32_t kTmemCols = 512;
// Per-thread register limits after the warpgroup reallocation.
constexpr int kRegsSoftmax = 224;
constexpr int kRegsOther = 56;
constexpr int kRegSplitTotal = 256 * kRegsSoftmax + 128 * kRegsOther;

enum Epilogue : int { kEpiForward = 0, kEpiPartial = 1 };

struct AttnParams {
  CUtensorMap tm_q, tm_k, tm_v, tm_bias;
  // D = 32, forward: the bf16 output (D, Nq, H, B), box {32, 32} with the
  // 64-byte swizzle, one warp's 32 rows per tensor store
  CUtensorMap tm_out;
  int32_t B, H, Nq, Nk;
  int32_t n_qblocks;     // ceil(Nq / 256)
  int32_t n_units;       // B * H * n_qblocks
  int32_t bias_h_bcast;  // bias head stride 0
  int32_t bias_b_bcast;  // bias batch stride 0
  int32_t needs_mask;    // key mask given or Nk not a multiple of the key tile
  int32_t mask_vec4;     // key mask rows readable as aligned 4-byte words
  float tau;
  const uint8_t *mask;
  int64_t mask_sb, mask_sk;
  void *out;  // bf16 O (forward) or fp32 O_p (partial)
  int64_t out_sb, out_sh, out_sn;
  float *lse;  // forward: log-sum-exp; partial: m_p
  int64_t lse_sb, lse_sh, lse_sn;
  float *l_part;  // partial: l_p (strides of lse)
  const uint16_t *gate;
  int64_t gate_sb, gate_sh, gate_sn;
  int *err;
  uint64_t timeout_ns;
};

template <int D>
struct AttnLayout {
  static_assert(D == 32 || D == 64, "head dimension");
  static constexpr int kRowBytes = D * 2;                   // one bf16 row of Q/K/V
  static constexpr int kSwizzleMode = (D == 64) ? 2 : 4;    // 128-byte / 64-byte swizzle
  static constexpr int kAtomBytes = 8 * kRowBytes;          // 8-row swizzle atom
  static constexpr int kKVStages = (D == 64) ? 2 : 4;
  static constexpr int kQBytes = kBM * kRowBytes;
  static constexpr int kKVBytes = kBN * kRowBytes;
  static constexpr int kBiasBytes = kBM * kBN * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQTiles * kQBytes;
  static constexpr int kOffV = kOffK + kKVStages * kKVBytes;
  static constexpr int kOffBias = kOffV + kKVStages * kKVBytes;
  // key-mask words: one u32 per key pair of a bias slot (0xFFFF per valid half)
  static constexpr int kOffMaskWords = kOffBias + kQTiles * kBiasStages * kBiasBytes;
  // D = 32: the forward epilogue's output rows, staged for tensor stores
  // ([128 rows][64 bytes] per query tile, 64-byte swizzle); at D = 64 there is
  // no room and the rows go straight to global memory
  static constexpr bool kOutStaged = (D == 32);
  static constexpr int kOffOut = kOffMaskWords + kQTiles * kBiasStages * (kBN / 2) * 4;
  static constexpr int kOffBar = kOffOut + (kOutStaged ? kQTiles * kBM * kRowBytes : 0);
  // barriers
  static constexpr int kBarQFull = 0;
  static constexpr int kBarQEmpty = 1;
  static constexpr int kBarKFull = 2;
  static constexpr int kBarVFull = kBarKFull + kKVStages;
  static constexpr int kBarKEmpty = kBarVFull + kKVStages;
  static constexpr int kBarVEmpty = kBarKEmpty + kKVStages;
  static constexpr int kBarBiasFull = kBarVEmpty + kKVStages;             // [w][t]
  static constexpr int kBarBiasReady = kBarBiasFull + kQTiles * kBiasStages;
  static constexpr int kBarBiasEmpty = kBarBiasReady + kQTiles * kBiasStages;
  static constexpr int kBarSFull = kBarBiasEmpty + kQTiles * kBiasStages;  // [w]
  static constexpr int kBarSFree = kBarSFull + kQTiles;
  static constexpr int kBarPFull = kBarSFree + kQTiles;
  static constexpr int kBarODone = kBarPFull + kQTiles;
  static constexpr int kBarOFree = kBarODone + kQTiles;  // [w]: epilogue has read O
  static constexpr int kBarDrain = kBarOFree + kQTiles;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemSlot + 4;
  static constexpr int kBytes = kOffAbort + 4;
  static constexpr int kSmemAlloc = kBytes + 1024;  // room to align the base to 1024
  static_assert(kSmemAlloc <= 232448, "shared memory budget");
};

// Natural-log constants of the base-2 softmax.
constexpr float kLog2e = 1.4426950408889634f;
// A row keeps its running maximum until a tile's maximum exceeds it by more
// than 8 (in log2 units), so most tiles skip the rescale of O; the stale
// maximum is used consistently for P and l, so the result is unchanged and the
// probabilities stay below 2^8.
constexpr float kRescaleThreshold = 8.0f / kLog2e;
// One key pair in kExpEmuEvery takes the software exp2 on the FMA pipe (0:
// none).  Neither head dimension gains from it: at D = 64 the softmax is
// issue-bound, and at D = 32 (triangle attention, tri1024) every share
// measured was slower than none: one pair in four +2 to +4 %, one in three
// +4 to +7 %, one in two +13 to +30 %.
#ifndef PBA_EXP_EMU_EVERY_D32
#define PBA_EXP_EMU_EVERY_D32 0
#endif
#ifndef PBA_EXP_EMU_EVERY_D64
#define PBA_EXP_EMU_EVERY_D64 0
#endif

// Work unit u -> (b, h, first query row); units are ordered query block
// fastest, then head, then batch, so concurrent CTAs share one head's K/V.
struct Unit {
  int b, h, q0;
};
__device__ __forceinline__ Unit decode_unit(const AttnParams &p, int u) {
  const int qblk = u % p.n_qblocks;
  const int bh = u / p.n_qblocks;
  return Unit{bh / p.H, bh % p.H, qblk * (kQTiles * kBM)};
}

template <int D, bool kBiasT, int kEpi, bool kGate, bool kMasked>
__global__ void __launch_bounds__(kAttnThreads, 1) pba_attn_sm100_kernel(const __grid_constant__ AttnParams p) {
  using L = AttnLayout<D>;
  constexpr int kExpEmuEvery = (D == 32) ? PBA_EXP_EMU_EVERY_D32 : PBA_EXP_EMU_EVERY_D64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffTmemSlot);
  int *abort_flag = reinterpret_cast<int *>(smem + L::kOffAbort);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int nt = (p.Nk + kBN - 1) / kBN;  // key tiles per unit
  const int u_begin = blockIdx.x, u_step = gridDim.x;

  if (threadIdx.x == 0) {
    mbar_init(&bars[L::kBarQFull], 1);
    mbar_init(&bars[L::kBarQEmpty], 1);
    for (int s = 0; s < L::kKVStages; ++s) {
      mbar_init(&bars[L::kBarKFull + s], 1);
      mbar_init(&bars[L::kBarVFull + s], 1);
      mbar_init(&bars[L::kBarKEmpty + s], 1);
      mbar_init(&bars[L::kBarVEmpty + s], 1);
    }
    for (int i = 0; i < kQTiles * kBiasStages; ++i) {
      mbar_init(&bars[L::kBarBiasFull + i], 1);
      mbar_init(&bars[L::kBarBiasReady + i], 32);
      mbar_init(&bars[L::kBarBiasEmpty + i], kBM);
    }
    for (int w = 0; w < kQTiles; ++w) {
      mbar_init(&bars[L::kBarSFull + w], 1);
      mbar_init(&bars[L::kBarSFree + w], kBM);
      mbar_init(&bars[L::kBarPFull + w], kBM);
      mbar_init(&bars[L::kBarODone + w], 1);
      mbar_init(&bars[L::kBarOFree + w], kBM);
    }
    mbar_init(&bars[L::kBarDrain], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kWarpProducer && lane == 0) {
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  if (warp == kWarpBiasProducer && lane == 0) tma_prefetch_desc(&p.tm_bias);
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{abort_flag, p.err, p.timeout_ns};
  WaitCtl wc_drain = wc;  // clean-up waits: ignore the abort word, keep the time limit
  int drain_abort = 0;
  wc_drain.abort_flag = &drain_abort;

  // Registers: the launch gives 168 per thread (384 x 168 = 64512).  The
  // producer/MMA/mask warpgroup (warps 8-11) gives most of its share to the
  // two softmax warpgroups: 128 x 56 + 256 x 224 = 64512.  Each
  // warpgroup changes its limit once, at the top of its own branch.
  if (warp >= 8) {
    setmaxnreg_dec<kRegsOther>();
    if (warp == kWarpProducer) {
      // ============================================================== Q/K/V TMA producer
      if (lane == 0) {
        const uint64_t pol_stream = l2_policy_evict_first();
        const uint64_t pol_keep = l2_policy_evict_last();
        bool ok = true;
        int kc = 0, vc = 0, uc = 0, qc = 0;  // K tiles, V tiles, units, Q loads issued
        // K runs one tile ahead of V: a K slot frees when both score MMAs of its
        // tile are done, a V slot only after both P V MMAs.
        auto load_k = [&](const Unit &un, int j) -> bool {
          const int s = kc % L::kKVStages;
          if (kc >= L::kKVStages && !mbar_wait(&bars[L::kBarKEmpty + s], ((kc / L::kKVStages) - 1) & 1, wc))
            return false;
          mbar_arrive_expect_tx(&bars[L::kBarKFull + s], L::kKVBytes);
          tma_load_4d(smem + L::kOffK + s * L::kKVBytes, &p.tm_k, &bars[L::kBarKFull + s], 0, j * kBN, un.h, un.b,
                      pol_keep);
          ++kc;
          return true;
        };
        auto load_v = [&](const Unit &un, int j) -> bool {
          const int s = vc % L::kKVStages;
          if (vc >= L::kKVStages && !mbar_wait(&bars[L::kBarVEmpty + s], ((vc / L::kKVStages) - 1) & 1, wc))
            return false;
          mbar_arrive_expect_tx(&bars[L::kBarVFull + s], L::kKVBytes);
          tma_load_4d(smem + L::kOffV + s * L::kKVBytes, &p.tm_v, &bars[L::kBarVFull + s], 0, j * kBN, un.h, un.b,
                      pol_keep);
          ++vc;
          return true;
        };
        for (int u = u_begin; u < p.n_units && ok; u += u_step, ++uc) {
          const Unit un = decode_unit(p, u);
          // Q slot: free once the last score MMAs of the previous unit are done
          if (uc > 0) ok = mbar_wait(&bars[L::kBarQEmpty], (uc - 1) & 1, wc);
          if (!ok) break;
          mbar_arrive_expect_tx(&bars[L::kBarQFull], kQTiles * L::kQBytes);
          for (int w = 0; w < kQTiles; ++w)
            tma_load_4d(smem + L::kOffQ + w * L::kQBytes, &p.tm_q, &bars[L::kBarQFull], 0, un.q0 + w * kBM, un.h,
                        un.b, pol_stream);
          ++qc;
          ok = load_k(un, 0);
          for (int j = 0; j < nt && ok; ++j) {
            if (j + 1 < nt) ok = load_k(un, j + 1);
            if (ok) ok = load_v(un, j);
          }
        }
        if (!ok) {
          // Let every copy already issued land before the CTA exits: each full
          // barrier has at most one armed phase that no consumer has waited for.
          // slot s was armed (n - s + stages - 1) / stages times after n issues
          if (qc) mbar_wait(&bars[L::kBarQFull], (qc - 1) & 1, wc_drain);
          for (int s = 0; s < L::kKVStages; ++s) {
            const int ak = (kc - s + L::kKVStages - 1) / L::kKVStages, av = (vc - s + L::kKVStages - 1) / L::kKVStages;
            if (ak > 0) mbar_wait(&bars[L::kBarKFull + s], (ak - 1) & 1, wc_drain);
            if (av > 0) mbar_wait(&bars[L::kBarVFull + s], (av - 1) & 1, wc_drain);
          }
        }
      }
    } else if (warp == kWarpBiasProducer) {
      // ============================================================== bias TMA producer
      if (lane == 0) {
        const uint64_t pol_stream = l2_policy_evict_first();
        bool ok = true;
        int gt = 0;      // key tiles started (all units)
        int issued = 0;  // bias tiles issued, warpgroup-major within a key tile
        for (int u = u_begin; u < p.n_units && ok; u += u_step) {
          const Unit un = decode_unit(p, u);
          const int hb = p.bias_h_bcast ? 0 : un.h;
          const int bb = p.bias_b_bcast ? 0 : un.b;
          for (int j = 0; j < nt && ok; ++j, ++gt) {
            const int t = gt % kBiasStages;
            for (int w = 0; w < kQTiles && ok; ++w) {
              const int slot = w * kBiasStages + t;
              if (gt >= kBiasStages)
                ok = mbar_wait(&bars[L::kBarBiasEmpty + slot], ((gt / kBiasStages) - 1) & 1, wc);
              if (!ok) break;
              uint8_t *dst = smem + L::kOffBias + slot * L::kBiasBytes;
              mbar_arrive_expect_tx(&bars[L::kBarBiasFull + slot], L::kBiasBytes);
              if (kBiasT) {
                // transposed bias tile: [128 keys][128 queries], no swizzle
                tma_load_4d(dst, &p.tm_bias, &bars[L::kBarBiasFull + slot], un.q0 + w * kBM, j * kBN, hb, bb,
                            pol_stream);
              } else {
                // [128 queries][128 keys] as two 64-key boxes, 128-byte swizzle
                tma_load_4d(dst, &p.tm_bias, &bars[L::kBarBiasFull + slot], j * kBN, un.q0 + w * kBM, hb, bb,
                            pol_stream);
                tma_load_4d(dst + L::kBiasBytes / 2, &p.tm_bias, &bars[L::kBarBiasFull + slot], j * kBN + 64,
                            un.q0 + w * kBM, hb, bb, pol_stream);
              }
              ++issued;
            }
          }
        }
        if (!ok)
          for (int w = 0; w < kQTiles; ++w)
            for (int t = 0; t < kBiasStages; ++t) {
              // tiles of warpgroup w issued: key tiles 0..n_w-1, slot t armed for those with tile % stages == t
              const int n_w = issued / kQTiles + (w < issued % kQTiles ? 1 : 0);
              const int a = (n_w - t + kBiasStages - 1) / kBiasStages;
              if (a > 0) mbar_wait(&bars[L::kBarBiasFull + w * kBiasStages + t], (a - 1) & 1, wc_drain);
            }
      }
    } else if (warp == kWarpMma) {
      // ============================================================== MMA issuer
      if (lane == 0) {
        const uint32_t idesc_s = idesc_bf16_f32(kBM, kBN, false);
        const uint32_t idesc_o = idesc_bf16_f32(kBM, D, true);
        const uint32_t sQ = smem_u32(smem + L::kOffQ);
        const uint32_t sK = smem_u32(smem + L::kOffK);
        const uint32_t sV = smem_u32(smem + L::kOffV);
        bool ok = true;
        int kc = 0, vc = 0;  // K and V tiles consumed
        int gs = 0;          // score tiles issued (all units), per warpgroup
        int gp = 0;          // P V tiles issued (all units), per warpgroup
        int uc = 0;
        // Descriptor high halves are fixed; the loops advance the address field
        // of the low half (16 bytes per unit): 32 bytes per K step inside a
        // swizzle row of Q and K, 16 key rows per K step down V.
        constexpr uint32_t kDescHi = smem_desc_hi(L::kAtomBytes, L::kSwizzleMode);
        auto issue_s = [&](int w, int s) {
          const uint32_t d_tmem = tmem + w * kBN;
          const uint32_t a_lo = smem_desc_lo(sQ + w * L::kQBytes, 16);
          const uint32_t b_lo = smem_desc_lo(sK + s * L::kKVBytes, 16);
#pragma unroll 4
          for (int kk = 0; kk < D / 16; ++kk)
            mma_bf16_ss(d_tmem, desc_join(a_lo + kk * 2, kDescHi), desc_join(b_lo + kk * 2, kDescHi), idesc_s,
                        kk > 0 ? 1u : 0u);
          tc_commit(&bars[L::kBarSFull + w]);
        };
        auto issue_pv = [&](int w, int s, bool first) {
          const uint32_t d_tmem = tmem + 384 + w * 64;
          const uint32_t a_tmem = tmem + 256 + w * 64;
          const uint32_t v_lo = smem_desc_lo(sV + s * L::kKVBytes, L::kKVBytes);
#pragma unroll 4
          for (int kk = 0; kk < kBN / 16; ++kk)
            mma_bf16_ts(d_tmem, a_tmem + kk * 8, desc_join(v_lo + kk * (16 * L::kRowBytes / 16), kDescHi), idesc_o,
                        (!first || kk > 0) ? 1u : 0u);
          tc_commit(&bars[L::kBarODone + w]);
        };
        // Per key tile j the order is S0(j+1), P0 V(j), S1(j+1), P1 V(j): each
        // warpgroup's next score tile and its P V follow its own progress, so
        // neither warpgroup's MMAs queue behind the other's softmax.
        for (int u = u_begin; u < p.n_units && ok; u += u_step, ++uc) {
          // first score tiles of the unit
          ok = mbar_wait(&bars[L::kBarQFull], uc & 1, wc);
          if (ok) ok = mbar_wait(&bars[L::kBarKFull + kc % L::kKVStages], (kc / L::kKVStages) & 1, wc);
          for (int w = 0; w < kQTiles && ok; ++w) {
            if (gs > 0 && !(ok = mbar_wait(&bars[L::kBarSFree + w], (gs - 1) & 1, wc))) break;
            tc_fence_after_sync();
            issue_s(w, kc % L::kKVStages);
          }
          if (!ok) break;
          tc_commit(&bars[L::kBarKEmpty + kc % L::kKVStages]);
          if (nt == 1) tc_commit(&bars[L::kBarQEmpty]);
          ++kc;
          ++gs;
          for (int j = 0; j < nt && ok; ++j) {
            const bool has_next = j + 1 < nt;
            const int sk = kc % L::kKVStages;
            const int sv = vc % L::kKVStages;
            if (has_next) ok = mbar_wait(&bars[L::kBarKFull + sk], (kc / L::kKVStages) & 1, wc);
            if (ok) ok = mbar_wait(&bars[L::kBarVFull + sv], (vc / L::kKVStages) & 1, wc);
            for (int w = 0; w < kQTiles && ok; ++w) {
              if (has_next) {
                if (!(ok = mbar_wait(&bars[L::kBarSFree + w], (gs - 1) & 1, wc))) break;
                tc_fence_after_sync();
                issue_s(w, sk);
              }
              if (!(ok = mbar_wait(&bars[L::kBarPFull + w], gp & 1, wc))) break;
              // the first P V of a unit overwrites O: the epilogue of the
              // previous unit must have read it
              if (j == 0 && uc > 0 && !(ok = mbar_wait(&bars[L::kBarOFree + w], (uc - 1) & 1, wc))) break;
              tc_fence_after_sync();
              issue_pv(w, sv, j == 0);
            }
            if (!ok) break;
            if (has_next) {
              tc_commit(&bars[L::kBarKEmpty + sk]);
              // after the unit's last score MMAs the Q slot can be refilled
              if (j + 2 == nt) tc_commit(&bars[L::kBarQEmpty]);
              ++kc;
              ++gs;
            }
            tc_commit(&bars[L::kBarVEmpty + sv]);
            ++vc;
            ++gp;
          }
        }
        // Every MMA issued above completes before Tensor Memory is released.
        tc_commit(&bars[L::kBarDrain]);
        mbar_wait(&bars[L::kBarDrain], 0, wc_drain);
      }
    } else {
      // ============================================================== key-mask warp
      // Lane l owns keys 4l..4l+3 of each tile; the mask bytes of tile j+1 are
      // loaded while tile j is processed.  For the untransposed bias tile the
      // warp writes one mask word per key pair beside the bias slot and the
      // softmax warps apply it while unpacking the bias; for the transposed
      // tile (one key per 256-byte row) it writes -inf over the masked rows.
      // Without a key mask and with whole key tiles the softmax warps wait on
      // the TMA barrier directly and this warp has nothing to do.
      bool ok = kBiasT ? (p.needs_mask != 0) : kMasked;
      int gt = 0;  // key tiles processed (all units)
      for (int u = u_begin; u < p.n_units && ok; u += u_step) {
        const Unit un = decode_unit(p, u);
        const uint8_t *mrow = p.mask ? p.mask + (int64_t)un.b * p.mask_sb : nullptr;
        auto load_word = [&](int j) -> uint32_t {  // byte e nonzero = key 4*lane+e takes part
          const int key0 = j * kBN + 4 * lane;
          if (mrow == nullptr) return 0x01010101u;
          if (p.mask_vec4 && key0 + 3 < p.Nk) return __ldg(reinterpret_cast<const uint32_t *>(mrow + key0));
          uint32_t wv = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (key0 + e < p.Nk) wv |= uint32_t(__ldg(mrow + (int64_t)(key0 + e) * p.mask_sk) != 0) << (8 * e);
          return wv;
        };
        uint32_t next_word = load_word(0);
        for (int j = 0; j < nt && ok; ++j, ++gt) {
          const uint32_t word = next_word;
          if (j + 1 < nt) next_word = load_word(j + 1);
          const int key0 = j * kBN + 4 * lane;
          uint32_t inv = 0;  // bit e: key 4*lane + e of the tile is masked or past the end
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (key0 + e >= p.Nk || ((word >> (8 * e)) & 0xFFu) == 0) inv |= 1u << e;
          // keep-masks of the key pairs (4l, 4l+1) and (4l+2, 4l+3)
          const uint2 keep = make_uint2(((inv & 1u) ? 0u : 0x0000FFFFu) | ((inv & 2u) ? 0u : 0xFFFF0000u),
                                        ((inv & 4u) ? 0u : 0x0000FFFFu) | ((inv & 8u) ? 0u : 0xFFFF0000u));
          const uint32_t any = kBiasT ? __ballot_sync(0xffffffffu, inv != 0) : 0u;
          const int t = gt % kBiasStages;
          for (int w = 0; w < kQTiles && ok; ++w) {
            const int slot = w * kBiasStages + t;
            ok = mbar_wait<false>(&bars[L::kBarBiasFull + slot], (gt / kBiasStages) & 1, wc);
            if (!ok) break;
            if (!kBiasT) {
              reinterpret_cast<uint2 *>(smem + L::kOffMaskWords + slot * (kBN / 2) * 4)[lane] = keep;
            } else if (any) {
              uint8_t *tile = smem + L::kOffBias + slot * L::kBiasBytes;
              uint32_t rem = any;
              while (rem) {
                const int src = __ffs(rem) - 1;
                rem &= rem - 1;
                uint32_t bits = __shfl_sync(0xffffffffu, inv, src);
                while (bits) {
                  const int e = __ffs(bits) - 1;
                  bits &= bits - 1;
                  // row 4*src+e of the [key][query] tile: 128 bf16 = 256 bytes
                  reinterpret_cast<uint2 *>(tile + (4 * src + e) * 256)[lane] =
                      make_uint2(0xFF80FF80u, 0xFF80FF80u);
                }
              }
              fence_proxy_async_smem();
            }
            __syncwarp();
            mbar_arrive(&bars[L::kBarBiasReady + slot]);
          }
        }
      }
    }
  } else {
    // ================================================================ softmax warpgroups
    setmaxnreg_inc<kRegsSoftmax>();
    const int w = warp >> 2;            // query tile
    const int t = threadIdx.x & 127;    // row inside the tile
    const uint32_t lane_base = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_base + w * kBN;
    const uint32_t tP = tmem + lane_base + 256 + w * 64;
    const uint32_t tO = tmem + lane_base + 384 + w * 64;
    const float tau = p.tau;
    const bool relay = kBiasT ? (p.needs_mask != 0) : kMasked;
    bool ok = true;
    int gt = 0;  // key tiles processed (all units)
    for (int u = u_begin; u < p.n_units && ok; u += u_step) {
      float m_cur = -INFINITY;   // maximum used for P and l
      float m_true = -INFINITY;  // true running maximum
      float l = 0.f;
      if (kGate && L::kOutStaged) {
        // The gate row goes into this thread's output staging row while the
        // unit's key tiles are processed; the epilogue reads it there and
        // then overwrites it with the output.  The previous unit's tensor
        // store must have read the rows first.
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
        const Unit gu = decode_unit(p, u);
        const int grow = gu.q0 + w * kBM + t;
        uint8_t *srow = smem + L::kOffOut + (w * kBM + t) * L::kRowBytes;
        if (grow < p.Nq) {
          const uint8_t *src = reinterpret_cast<const uint8_t *>(p.gate + gu.b * p.gate_sb + gu.h * p.gate_sh +
                                                                 (int64_t)grow * p.gate_sn);
#pragma unroll
          for (int c = 0; c < L::kRowBytes / 16; ++c) cp_async16(srow + ((c ^ ((t >> 1) & 3)) << 4), src + c * 16);
        }
        cp_async_commit();
      }
      for (int j = 0; j < nt && ok; ++j, ++gt) {
        // The bias tile lands long before it is used: wait for it first and
        // start loading its first part from shared memory, so that those loads
        // overlap the wait for the score tile and its Tensor Memory load.
        const int slot = w * kBiasStages + (gt % kBiasStages);
        ok = mbar_wait<false>(&bars[(relay ? L::kBarBiasReady : L::kBarBiasFull) + slot], (gt / kBiasStages) & 1, wc);
        if (!ok) break;
        const uint8_t *tile = smem + L::kOffBias + slot * L::kBiasBytes;
        // 8-key groups of the untransposed tile loaded ahead: half the tile
        // at D = 64, ten of sixteen at D = 32, where the registers allow it
        // (triangle attention, starting node, 1.838 -> 1.802 ms at N = 1024;
        // twelve groups 1.804 ms, and large16k gains nothing from ten)
        constexpr int kPre = (D == 32) ? 10 : kBN / 16;
        constexpr int kPreT = 32;        // keys of the transposed tile loaded ahead
        uint4 bpre[kPre];                // untransposed tile: 8 bf16 per group
        uint32_t tpre[kBiasT ? kPreT : 1];  // transposed tile: 1 bf16 per key
        if (kBiasT) {
          const uint16_t *col = reinterpret_cast<const uint16_t *>(tile) + t;
#pragma unroll
          for (int c = 0; c < kPreT; ++c) tpre[c] = col[c * kBM];
        } else {
#pragma unroll
          for (int c8 = 0; c8 < kPre; ++c8)
            bpre[c8] = *reinterpret_cast<const uint4 *>(tile + (c8 >> 3) * (L::kBiasBytes / 2) + t * 128 +
                                                        (((c8 & 7) ^ (t & 7)) << 4));
        }
        uint4 kpre[kMasked && !kBiasT ? kPre : 1];  // and their mask words
        if (kMasked && !kBiasT) {
#pragma unroll
          for (int c8 = 0; c8 < kPre; ++c8)
            kpre[c8] = reinterpret_cast<const uint4 *>(smem + L::kOffMaskWords + slot * (kBN / 2) * 4)[c8];
        }

        ok = mbar_wait<false>(&bars[L::kBarSFull + w], gt & 1, wc);
        if (!ok) break;
        tc_fence_after_sync();
        uint32_t sreg[kBN];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c)
          tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sreg[c * 32]));
        tmem_wait_ld();
        reg_fence(sreg);
        tc_fence_before_sync();
        // The score tile is free once it is in registers.  The ending node
        // (transposed bias tile, 128 column loads per thread) and D = 64
        // (half the bias tile and its mask words still to load) free it only
        // after their bias loads have returned (with the bias slot, below),
        // so that the next score MMAs, which stream their operands from
        // shared memory, do not starve those loads: tri1024 ending node
        // 1.900 -> 1.879 ms, large16k 2.062 -> 2.053 ms.  The starting node
        // at D = 32, with most of its tile loaded ahead, measured slower that
        // way (1.804 -> 1.823 ms).
        constexpr bool kLateSFree = kBiasT || D == 64;
        if (!kLateSFree) mbar_arrive(&bars[L::kBarSFree + w]);

        // x = tau * s + bias, two keys per packed fma
        float2 x[kBN / 2];
        const float2 tau2 = make_float2(tau, tau);
        if (kBiasT) {
          const uint16_t *col = reinterpret_cast<const uint16_t *>(tile) + t;
#pragma unroll
          for (int c = 0; c < kBN; c += 2) {
            const uint32_t b0 = c < kPreT ? tpre[c] : uint32_t(col[c * kBM]);
            const uint32_t b1 = c + 1 < kPreT ? tpre[c + 1] : uint32_t(col[(c + 1) * kBM]);
            const float2 bv = make_float2(__uint_as_float(b0 << 16), __uint_as_float(b1 << 16));
            x[c / 2] = ffma2(make_float2(__uint_as_float(sreg[c]), __uint_as_float(sreg[c + 1])), tau2, bv);
          }
        } else {
#pragma unroll
          for (int c8 = 0; c8 < kBN / 8; ++c8) {
            const int box = c8 >> 3, chunk = c8 & 7;
            const uint4 bv = c8 < kPre ? bpre[c8]
                                       : *reinterpret_cast<const uint4 *>(tile + box * (L::kBiasBytes / 2) + t * 128 +
                                                                          ((chunk ^ (t & 7)) << 4));
            uint32_t wv[4] = {bv.x, bv.y, bv.z, bv.w};
            if (kMasked) {
              // masked halves become bf16 -inf: (w & keep) | (~keep & -inf)
              const uint4 kv = c8 < kPre ? kpre[c8 < kPre ? c8 : 0]
                                         : reinterpret_cast<const uint4 *>(smem + L::kOffMaskWords + slot * (kBN / 2) * 4)[c8];
              const uint32_t keep[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) wv[e] = (wv[e] & keep[e]) | (~keep[e] & 0xFF80FF80u);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = c8 * 8 + 2 * e;
              x[c / 2] = ffma2(make_float2(__uint_as_float(sreg[c]), __uint_as_float(sreg[c + 1])), tau2,
                               make_float2(bf16lo_to_f32(wv[e]), bf16hi_to_f32(wv[e])));
            }
          }
        }
        // tile maximum: eight independent chains
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) m8[i] = fmaxf(x[i].x, x[i].y);
#pragma unroll
        for (int i = 8; i < kBN / 2; ++i) m8[i & 7] = max3f(m8[i & 7], x[i].x, x[i].y);
        const float mx = max3f(max3f(m8[0], m8[1], m8[2]), max3f(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        // The bias slot is released under a condition on mx, which depends on
        // every bias value of the tile: the arrive cannot issue before all of
        // the slot's shared-memory loads have returned, so the next TMA write
        // into the slot cannot overtake one still in flight.  (The pattern
        // never occurs: no maximum is this NaN.)
        if (__float_as_uint(mx) != 0x7FC0DEADu) {
          mbar_arrive(&bars[L::kBarBiasEmpty + slot]);
          if (kLateSFree) mbar_arrive(&bars[L::kBarSFree + w]);
        }
        m_true = fmaxf(m_true, mx);
        const bool need = mx > m_cur + kRescaleThreshold;
        float alpha = 1.f;
        if (need) {
          alpha = (m_cur == -INFINITY) ? 0.f : ex2_approx((m_cur - mx) * kLog2e);
          l *= alpha;
          m_cur = mx;
        }
        const float neg_m = (m_cur == -INFINITY) ? 0.f : -m_cur * kLog2e;
        const float2 l2e2 = make_float2(kLog2e, kLog2e), negm2 = make_float2(neg_m, neg_m);
        uint32_t pk[kBN / 2];
        float2 ls[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int i = 0; i < kBN / 2; ++i) {
          const float2 a = ffma2(x[i], l2e2, negm2);
          // every kExpEmuEvery-th key pair takes the software exp2 on the FMA pipe
          const float2 pv = (kExpEmuEvery > 0 && i % kExpEmuEvery == kExpEmuEvery - 1)
                                ? exp2_poly2(a)
                                : make_float2(ex2_approx(a.x), ex2_approx(a.y));
          ls[i & 3] = fadd2(ls[i & 3], pv);
          pk[i] = pack_bf16x2(pv.x, pv.y);
        }
        const float2 lsum2 = fadd2(fadd2(ls[0], ls[1]), fadd2(ls[2], ls[3]));
        l += lsum2.x + lsum2.y;

        // P(j) overwrites the P buffer that P V(j-1) read, possibly the last
        // one of the previous unit
        if (gt > 0) {
          ok = mbar_wait<false>(&bars[L::kBarODone + w], (gt - 1) & 1, wc);
          if (!ok) break;
          tc_fence_after_sync();
          if (j > 0 && __any_sync(0xffffffffu, need)) {
            // rescale this warp's rows of O (lanes without a new maximum use 1)
#pragma unroll
            for (int c = 0; c < D; c += 32) {
              uint32_t o[32];
              tmem_ld32(tO + c, o);
              tmem_wait_ld();
              reg_fence(o);
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(tO + c, o);
            }
          }
        }
#pragma unroll
        for (int c = 0; c < kBN / 2; c += 32) tmem_st32(tP + c, *reinterpret_cast<uint32_t(*)[32]>(&pk[c]));
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(&bars[L::kBarPFull + w]);
      }

      // -------------------------------------------------------------- epilogue
      // What does not need O is done before waiting for the last P V: the
      // unit's coordinates, 1/l and, with a gate at D = 32 and the
      // untransposed bias tile, the column factors sigmoid(g) / l of the row
      // (the exp2 unit works on them while the last P V runs; triangle
      // attention, starting node, 1.97 -> 1.84 ms at N = 1024).  The other
      // gated instances form the factors after reading O: there the early
      // factors add register spills (the ending node measured slower with
      // them, 1.91 -> 1.94 ms).
      const Unit un = decode_unit(p, u);  // derived here so it is not live across the tile loop
      const int row = un.q0 + w * kBM + t;
      const int b = un.b, h = un.h;
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      constexpr bool kEarlyGate = kGate && !kBiasT && D == 32;
      float sc[kGate ? D : 1];
      auto gate_factors = [&]() {
        const uint4 *gptr = reinterpret_cast<const uint4 *>(p.gate + b * p.gate_sb + h * p.gate_sh +
                                                            (int64_t)row * p.gate_sn);
        const uint8_t *grow_s = smem + L::kOffOut + (w * kBM + t) * L::kRowBytes;
        if (L::kOutStaged) cp_async_wait_all();
#pragma unroll
        for (int c = 0; c < D / 8; ++c) {
          const uint4 gv = L::kOutStaged ? *reinterpret_cast<const uint4 *>(grow_s + ((c ^ ((t >> 1) & 3)) << 4))
                                         : gptr[c];
          const uint32_t wv[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            sc[c * 8 + 2 * e] = inv_l * sigmoid_fast(bf16lo_to_f32(wv[e]));
            sc[c * 8 + 2 * e + 1] = inv_l * sigmoid_fast(bf16hi_to_f32(wv[e]));
          }
        }
      };
      if (kEpi == kEpiForward && kEarlyGate && row < p.Nq) gate_factors();
      if (ok) ok = mbar_wait<false>(&bars[L::kBarODone + w], (gt - 1) & 1, wc);
      if (!ok) break;
      tc_fence_after_sync();
      float o[D];
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        tmem_ld32(tO + c, r);
        tmem_wait_ld();
        reg_fence(r);
#pragma unroll
        for (int e = 0; e < 32; ++e) o[c + e] = __uint_as_float(r[e]);
      }
      // O is in registers: the next unit's first P V may overwrite it
      tc_fence_before_sync();
      mbar_arrive(&bars[L::kBarOFree + w]);
      if (kEpi == kEpiForward && L::kOutStaged && !kGate) {
        // the warp's staging rows were last read by the previous unit's store
        // (with a gate this was waited for at the unit's start)
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
      }
      if (row < p.Nq) {
        if (kEpi == kEpiForward) {
          if (kGate && !kEarlyGate) gate_factors();
          uint4 *op = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(p.out) + b * p.out_sb + h * p.out_sh +
                                                (int64_t)row * p.out_sn);
          // staged rows: this thread's row of the warpgroup's buffer, 16-byte
          // chunks swizzled by bits 7-8 of the row address
          uint8_t *srow = smem + L::kOffOut + (w * kBM + t) * L::kRowBytes;
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            uint32_t wv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = c * 8 + 2 * e;
              wv[e] = kGate ? pack_bf16x2(o[i] * sc[kGate ? i : 0], o[i + 1] * sc[kGate ? i + 1 : 0])
                            : pack_bf16x2(o[i] * inv_l, o[i + 1] * inv_l);
            }
            if (L::kOutStaged)
              *reinterpret_cast<uint4 *>(srow + ((c ^ ((t >> 1) & 3)) << 4)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            else
              op[c] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
          if (p.lse != nullptr)
            p.lse[b * p.lse_sb + h * p.lse_sh + (int64_t)row * p.lse_sn] = (l > 0.f) ? m_cur + logf(l) : -INFINITY;
        } else {
          float4 *op = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + b * p.out_sb + h * p.out_sh +
                                                  (int64_t)row * p.out_sn);
#pragma unroll
          for (int c = 0; c < D / 4; ++c)
            op[c] = make_float4(o[4 * c] * inv_l, o[4 * c + 1] * inv_l, o[4 * c + 2] * inv_l, o[4 * c + 3] * inv_l);
          const int64_t mi = b * p.lse_sb + h * p.lse_sh + (int64_t)row * p.lse_sn;
          p.lse[mi] = (l > 0.f) ? m_true : -INFINITY;
          p.l_part[mi] = (l > 0.f) ? l * ex2_approx((m_cur - m_true) * kLog2e) : 0.f;
        }
      }
      if (kEpi == kEpiForward && L::kOutStaged) {
        // the warp's 32 rows with one tensor store (rows past Nq are clipped)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int wq = warp & 3;
          tma_store_4d(&p.tm_out, smem + L::kOffOut + (w * kBM + 32 * wq) * L::kRowBytes, 0, un.q0 + w * kBM + 32 * wq,
                       h, b);
          bulk_commit_group();
        }
      }
    }
    // the output stores and gate copies are complete before the CTA ends
    if (kEpi == kEpiForward && L::kOutStaged && lane == 0) bulk_wait_group_all();
    if (kGate && L::kOutStaged) cp_async_wait_all();
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == kWarpMma) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace pba
